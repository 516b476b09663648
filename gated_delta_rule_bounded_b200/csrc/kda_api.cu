// kda_api.cu -- the C ABI: argument validation, kernel selection, status codes.
//
// Every check that can fail happens on the host before anything is launched,
// so a rejected call leaves the GPU untouched. Only launch failures return
// KDA_ERR_CUDA.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "kda.h"
#include "kda_internal.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_err[0] = '\0';
  return KDA_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(KDA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

size_t elem_size(kda_dtype dt) { return dt == KDA_F32 ? 4 : 2; }

bool valid_dtype(int dt) { return dt == KDA_F32 || dt == KDA_BF16; }

bool dim_supported(int64_t d) { return d >= 16 && d <= 256 && d % 16 == 0; }

// Contiguous [B,T,H,D] strides for a NULL strides pointer.
kda_strides contiguous(int64_t T, int64_t H, int64_t D) {
  kda_strides s;
  s.h = D;
  s.t = H * D;
  s.b = T * H * D;
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A token row (D contiguous elements) starts on a 16-byte boundary for every
// (b, t, h) when the base pointer and all three strides are 16-byte multiples.
// Dimensions of extent 1 never move the pointer, so their strides do not matter.
bool rows_aligned(const void* base, const kda_strides& s, size_t esize, int64_t B, int64_t T, int64_t H) {
  if (!aligned16(base)) return false;
  if (B > 1 && (s.b * (int64_t)esize) % 16 != 0) return false;
  if (T > 1 && (s.t * (int64_t)esize) % 16 != 0) return false;
  if (H > 1 && (s.h * (int64_t)esize) % 16 != 0) return false;
  return true;
}

bool strides_valid(const kda_strides& s) { return s.b >= 0 && s.t >= 0 && s.h >= 0; }

void put(int64_t dst[3], const kda_strides& s) {
  dst[0] = s.b;
  dst[1] = s.t;
  dst[2] = s.h;
}

}  // namespace

namespace kda {

int report_error(int code, const char* msg) { return fail(code, "%s", msg); }

}  // namespace kda

extern "C" {

const char* kda_last_error(void) { return g_err; }

const char* kda_version(void) { return "kda-b200 0.2 (sm_100a)"; }

int kda_selftest_wait_expiry(kda_stream_t stream) {
  cudaError_t e = kda::launch_wait_selftest(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kda_selftest_wait_expiry");
  return ok();
}

int kda_device_status(int* timed_out, int reset) {
  if (!timed_out) return fail(KDA_ERR_INVALID_ARG, "kda_device_status: null output");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "kda_device_status synchronize");
  int chunk_flag = 0, split_flag = 0, decode_flag = 0;
  e = kda::chunk_read_timeout(&chunk_flag, reset != 0);
  if (e == cudaSuccess) e = kda::split_read_timeout(&split_flag, reset != 0);
  if (e == cudaSuccess) e = kda::decode_read_timeout(&decode_flag, reset != 0);
  if (e != cudaSuccess) return cuda_fail(e, "kda_device_status read");
  *timed_out = (chunk_flag || split_flag || decode_flag) ? 1 : 0;
  return ok();
}

static int gate_impl(const char* fn, const void* logits, const kda_strides* logits_strides, kda_dtype dtype,
                     const float* A_log, float g_min, bool softplus, int64_t B, int64_t T, int64_t H, int64_t K,
                     void* out, const kda_strides* out_strides, kda_gate_kind out_kind, kda_stream_t stream) {
  if (B < 0 || T < 0 || H < 0 || K < 0) return fail(KDA_ERR_INVALID_ARG, "%s: negative size", fn);
  if (!valid_dtype(dtype)) return fail(KDA_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  if (out_kind != KDA_GATE_ALPHA && out_kind != KDA_GATE_LOG)
    return fail(KDA_ERR_INVALID_ARG, "%s: unknown out_kind %d", fn, (int)out_kind);
  if (!softplus && (!std::isfinite(g_min) || !(g_min < 0.f)))
    return fail(KDA_ERR_INVALID_ARG, "%s: g_min must be finite and < 0 (got %g)", fn, (double)g_min);
  if (B * T * H * K == 0) return ok();
  if (!logits || !A_log || !out) return fail(KDA_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (K % 4 != 0) return fail(KDA_ERR_UNSUPPORTED, "%s: K must be a multiple of 4 (got %lld)", fn, (long long)K);
  if (B * T * H >= (int64_t)INT32_MAX)
    return fail(KDA_ERR_UNSUPPORTED, "%s: B*T*H must be below 2^31 rows", fn);
  kda_strides zs = logits_strides ? *logits_strides : contiguous(T, H, K);
  kda_strides os = out_strides ? *out_strides : contiguous(T, H, K);
  if (!strides_valid(zs) || !strides_valid(os)) return fail(KDA_ERR_INVALID_ARG, "%s: negative stride", fn);
  const size_t es = elem_size(dtype);
  // bf16 rows are read four channels (8 bytes) at a time, fp32 rows 16 bytes.
  auto al = [&](const void* p, const kda_strides& s) {
    const size_t need = dtype == KDA_F32 ? 16 : 8;
    auto ok_mult = [&](int64_t st, int64_t ext) { return ext <= 1 || (st * (int64_t)es) % (int64_t)need == 0; };
    return (reinterpret_cast<uintptr_t>(p) % need) == 0 && ok_mult(s.b, B) && ok_mult(s.t, T) && ok_mult(s.h, H);
  };
  if (!al(logits, zs) || !al(out, os)) return fail(KDA_ERR_UNSUPPORTED, "%s: misaligned rows", fn);
  kda::GateParams p;
  p.z = logits;
  p.out = out;
  p.A_log = A_log;
  put(p.zs, zs);
  put(p.os, os);
  p.B = B;
  p.T = T;
  p.H = H;
  p.K = K;
  p.g_min = g_min;
  p.out_log = out_kind == KDA_GATE_LOG;
  p.softplus = softplus ? 1 : 0;
  cudaError_t e = kda::launch_gate(p, dtype, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

int kda_bounded_decay(const void* logits, const kda_strides* logits_strides, kda_dtype dtype,
                      const float* A_log, float g_min, int64_t B, int64_t T, int64_t H, int64_t K,
                      void* out, const kda_strides* out_strides, kda_gate_kind out_kind,
                      kda_stream_t stream) {
  return gate_impl("kda_bounded_decay", logits, logits_strides, dtype, A_log, g_min, false, B, T, H, K, out,
                   out_strides, out_kind, stream);
}

int kda_softplus_decay(const void* logits, const kda_strides* logits_strides, kda_dtype dtype,
                       const float* A_log, int64_t B, int64_t T, int64_t H, int64_t K,
                       void* out, const kda_strides* out_strides, kda_gate_kind out_kind,
                       kda_stream_t stream) {
  return gate_impl("kda_softplus_decay", logits, logits_strides, dtype, A_log, 0.f, true, B, T, H, K, out,
                   out_strides, out_kind, stream);
}

int kda_prefill_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                int64_t n_seq, kda_dtype dtype, size_t* bytes) {
  if (!bytes) return fail(KDA_ERR_INVALID_ARG, "kda_prefill_workspace_bytes: null output");
  if (B < 0 || T < 0 || H < 0 || K < 0 || V < 0 || n_seq < 0)
    return fail(KDA_ERR_INVALID_ARG, "kda_prefill_workspace_bytes: negative size");
  if (!valid_dtype(dtype)) return fail(KDA_ERR_INVALID_ARG, "kda_prefill_workspace_bytes: unknown dtype");
  *bytes = 0;
  if (dtype == KDA_BF16 && kda::chunk_supported((int)K, (int)V, dtype)) *bytes = kda::chunk_workspace_bytes(B, T, H, n_seq);
  return ok();
}

// The decay input of a scan: alpha, g = log alpha, or the logits z with A_log, g_min and an optional
// per-(head, channel) bias.
struct GateSpec {
  const float* data;
  int mode;
  const float* A_log;
  float g_min;
  unsigned flags;  // KDA_QK_L2NORM | KDA_BETA_LOGITS | KDA_STATE_VK | KDA_GATE_SOFTPLUS
  const float* dt_bias;
};

static int check_gate(const char* fn, const GateSpec& gs) {
  if (gs.mode != KDA_GATE_ALPHA && gs.mode != KDA_GATE_LOG && gs.mode != kda::GATE_LOGITS &&
      gs.mode != kda::GATE_SOFTPLUS)
    return fail(KDA_ERR_INVALID_ARG, "%s: unknown gate kind %d", fn, gs.mode);
  if (gs.mode == kda::GATE_LOGITS && (!std::isfinite(gs.g_min) || !(gs.g_min < 0.f)))
    return fail(KDA_ERR_INVALID_ARG, "%s: g_min must be finite and < 0 (got %g)", fn, (double)gs.g_min);
  if (gs.flags & ~(KDA_QK_L2NORM | KDA_BETA_LOGITS | KDA_STATE_VK | KDA_GATE_SOFTPLUS))
    return fail(KDA_ERR_INVALID_ARG, "%s: unknown flags 0x%x", fn, gs.flags);
  if (gs.dt_bias && !aligned16(gs.dt_bias))
    return fail(KDA_ERR_UNSUPPORTED, "%s: dt_bias must be 16-byte aligned", fn);
  return KDA_OK;
}

static int check_scan_common(const char* fn, kda_dtype dtype, const GateSpec& gs, int64_t H, int64_t K, int64_t V) {
  if (!valid_dtype(dtype)) return fail(KDA_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  int rc = check_gate(fn, gs);
  if (rc != KDA_OK) return rc;
  if (H <= 0) return fail(KDA_ERR_INVALID_ARG, "%s: H must be positive", fn);
  if (H > 65535) return fail(KDA_ERR_UNSUPPORTED, "%s: H must be at most 65535 (got %lld)", fn, (long long)H);
  if (!dim_supported(K) || !dim_supported(V))
    return fail(KDA_ERR_UNSUPPORTED, "%s: K and V must be multiples of 16 in [16,256] (K=%lld, V=%lld)", fn,
                (long long)K, (long long)V);
  return KDA_OK;
}

static int prefill_impl(const char* fn, const void* q, const void* k, const void* v, kda_dtype dtype,
                        const GateSpec& gs, const float* beta,
                        const float* initial_state, float* final_state,
                        const int32_t* cu_seqlens, int64_t n_seq,
                        int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                        const kda_layout* layout, void* o,
                        void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  const float* gate = gs.data;
  if (B < 0 || T < 0 || n_seq < 0) return fail(KDA_ERR_INVALID_ARG, "%s: negative size", fn);
  int rc = check_scan_common(fn, dtype, gs, H, K, V);
  if (rc != KDA_OK) return rc;
  int64_t N = B;
  if (cu_seqlens) {
    if (B != 1) return fail(KDA_ERR_INVALID_ARG, "%s: cu_seqlens requires B == 1 (got %lld)", fn, (long long)B);
    N = n_seq;
  }
  const int64_t state_elems = N * H * K * V;
  if (initial_state && final_state && initial_state != final_state) {
    const float* a0 = initial_state;
    const float* a1 = initial_state + state_elems;
    const float* b0 = final_state;
    const float* b1 = final_state + state_elems;
    if (a0 < b1 && b0 < a1) return fail(KDA_ERR_INVALID_ARG, "%s: initial_state and final_state overlap partially", fn);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B * T == 0 || N == 0) {
    // Empty scan: the final state is the initial state (or zeros).
    if (N > 0 && final_state) {
      cudaError_t e = kda::launch_state_copy(initial_state, final_state, state_elems, s);
      if (e != cudaSuccess) return cuda_fail(e, "kda_prefill state copy");
    }
    return ok();
  }
  if (!q || !k || !v || !gate || !beta || !o || ((gs.mode == kda::GATE_LOGITS || gs.mode == kda::GATE_SOFTPLUS) && !gs.A_log))
    return fail(KDA_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  kda_layout L;
  if (layout) {
    L = *layout;
  } else {
    L.q = contiguous(T, H, K);
    L.k = contiguous(T, H, K);
    L.gate = contiguous(T, H, K);
    L.v = contiguous(T, H, V);
    L.o = contiguous(T, H, V);
    L.beta = contiguous(T, H, 1);
  }
  const kda_strides* all[6] = {&L.q, &L.k, &L.v, &L.gate, &L.beta, &L.o};
  for (auto* st : all)
    if (!strides_valid(*st)) return fail(KDA_ERR_INVALID_ARG, "%s: negative stride", fn);
  const size_t es = elem_size(dtype);
  if (!rows_aligned(q, L.q, es, B, T, H) || !rows_aligned(k, L.k, es, B, T, H) ||
      !rows_aligned(v, L.v, es, B, T, H) || !rows_aligned(o, L.o, es, B, T, H) ||
      !rows_aligned(gate, L.gate, 4, B, T, H))
    return fail(KDA_ERR_UNSUPPORTED, "%s: token rows must start on 16-byte boundaries", fn);
  if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
    return fail(KDA_ERR_UNSUPPORTED, "%s: state pointers must be 16-byte aligned", fn);
  if (T > INT32_MAX) return fail(KDA_ERR_UNSUPPORTED, "%s: T too large", fn);

  kda::ScanParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.gate = gate;
  p.beta = beta;
  p.s0 = initial_state;
  p.sf = final_state;
  p.cu = cu_seqlens;
  p.o = o;
  put(p.qs, L.q);
  put(p.ks, L.k);
  put(p.vs, L.v);
  put(p.gs, L.gate);
  put(p.bs, L.beta);
  put(p.os, L.o);
  p.T = T;
  p.B = (int)B;
  p.H = (int)H;
  p.K = (int)K;
  p.V = (int)V;
  p.N = (int)N;
  p.gate_mode = gs.mode;
  p.A_log = gs.A_log;
  p.dt_bias = gs.dt_bias;
  p.g_min = gs.g_min;
  p.qk_l2norm = (gs.flags & KDA_QK_L2NORM) != 0;
  p.beta_sigmoid = (gs.flags & KDA_BETA_LOGITS) != 0;
  p.state_vk = (gs.flags & KDA_STATE_VK) != 0;

  cudaError_t e;
  if (workspace_bytes > 0 && !workspace) return fail(KDA_ERR_INVALID_ARG, "%s: workspace_bytes > 0 with a null workspace", fn);
  const bool chunked = dtype == KDA_BF16 && kda::chunk_supported((int)K, (int)V, dtype);
  if (chunked) {
    e = kda::launch_chunk(p, workspace, workspace_bytes, s);
  } else {
    e = kda::launch_recurrent(p, dtype, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "kda_prefill launch");
  return ok();
}

int kda_prefill(const void* q, const void* k, const void* v, kda_dtype dtype,
                const float* gate, kda_gate_kind gate_kind, const float* beta,
                const float* initial_state, float* final_state,
                const int32_t* cu_seqlens, int64_t n_seq,
                int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                const kda_layout* layout, void* o,
                void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  if (gate_kind != KDA_GATE_ALPHA && gate_kind != KDA_GATE_LOG)
    return fail(KDA_ERR_INVALID_ARG, "kda_prefill: unknown gate kind %d", (int)gate_kind);
  const GateSpec gs{gate, (int)gate_kind, nullptr, 0.f, 0u, nullptr};
  return prefill_impl("kda_prefill", q, k, v, dtype, gs, beta, initial_state, final_state, cu_seqlens, n_seq, B, T, H,
                      K, V, layout, o, workspace, workspace_bytes, stream);
}

int kda_prefill_logits(const void* q, const void* k, const void* v, kda_dtype dtype,
                       const float* logits, const float* A_log, const float* dt_bias, float g_min,
                       const float* beta, unsigned flags,
                       const float* initial_state, float* final_state,
                       const int32_t* cu_seqlens, int64_t n_seq,
                       int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                       const kda_layout* layout, void* o,
                       void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  const GateSpec gs{logits, (flags & KDA_GATE_SOFTPLUS) ? kda::GATE_SOFTPLUS : kda::GATE_LOGITS, A_log, g_min, flags,
                    dt_bias};
  return prefill_impl("kda_prefill_logits", q, k, v, dtype, gs, beta, initial_state, final_state, cu_seqlens, n_seq, B,
                      T, H, K, V, layout, o, workspace, workspace_bytes, stream);
}

static int decode_impl(const char* fn, const void* q, const void* k, const void* v, kda_dtype dtype,
                       const GateSpec& gs, const float* beta,
                       float* state, int64_t B, int64_t H, int64_t K, int64_t V,
                       const kda_layout* layout, void* o, kda_stream_t stream) {
  const float* gate = gs.data;
  if (B < 0) return fail(KDA_ERR_INVALID_ARG, "%s: negative size", fn);
  int rc = check_scan_common(fn, dtype, gs, H, K, V);
  if (rc != KDA_OK) return rc;
  if (B == 0) return ok();
  if (!q || !k || !v || !gate || !beta || !state || !o || ((gs.mode == kda::GATE_LOGITS || gs.mode == kda::GATE_SOFTPLUS) && !gs.A_log))
    return fail(KDA_ERR_INVALID_ARG, "%s: null pointer", fn);
  kda_layout L;
  if (layout) {
    L = *layout;
  } else {
    L.q = contiguous(1, H, K);
    L.k = contiguous(1, H, K);
    L.gate = contiguous(1, H, K);
    L.v = contiguous(1, H, V);
    L.o = contiguous(1, H, V);
    L.beta = contiguous(1, H, 1);
  }
  // Decode tensors have no time axis: the t stride is never used.
  kda_strides* all[6] = {&L.q, &L.k, &L.v, &L.gate, &L.beta, &L.o};
  for (auto* st : all) {
    st->t = 0;
    if (!strides_valid(*st)) return fail(KDA_ERR_INVALID_ARG, "%s: negative stride", fn);
  }
  const size_t es = elem_size(dtype);
  if (!rows_aligned(q, L.q, es, B, 1, H) || !rows_aligned(k, L.k, es, B, 1, H) ||
      !rows_aligned(v, L.v, es, B, 1, H) || !rows_aligned(o, L.o, es, B, 1, H) ||
      !rows_aligned(gate, L.gate, 4, B, 1, H) || !aligned16(state))
    return fail(KDA_ERR_UNSUPPORTED, "%s: rows and state must start on 16-byte boundaries", fn);
  kda::ScanParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.gate = gate;
  p.beta = beta;
  p.s0 = state;
  p.sf = state;
  p.cu = nullptr;
  p.o = o;
  put(p.qs, L.q);
  put(p.ks, L.k);
  put(p.vs, L.v);
  put(p.gs, L.gate);
  put(p.bs, L.beta);
  put(p.os, L.o);
  p.T = 1;
  p.B = (int)B;
  p.H = (int)H;
  p.K = (int)K;
  p.V = (int)V;
  p.N = (int)B;
  p.gate_mode = gs.mode;
  p.A_log = gs.A_log;
  p.dt_bias = gs.dt_bias;
  p.g_min = gs.g_min;
  p.qk_l2norm = (gs.flags & KDA_QK_L2NORM) != 0;
  p.beta_sigmoid = (gs.flags & KDA_BETA_LOGITS) != 0;
  p.state_vk = (gs.flags & KDA_STATE_VK) != 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = kda::decode_bulk_supported(p) ? kda::launch_decode_bulk(p, dtype, s) : kda::launch_recurrent(p, dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "kda_decode_step launch");
  return ok();
}

int kda_decode_step(const void* q, const void* k, const void* v, kda_dtype dtype,
                    const float* gate, kda_gate_kind gate_kind, const float* beta,
                    float* state, int64_t B, int64_t H, int64_t K, int64_t V,
                    const kda_layout* layout, void* o, kda_stream_t stream) {
  if (gate_kind != KDA_GATE_ALPHA && gate_kind != KDA_GATE_LOG)
    return fail(KDA_ERR_INVALID_ARG, "kda_decode_step: unknown gate kind %d", (int)gate_kind);
  const GateSpec gs{gate, (int)gate_kind, nullptr, 0.f, 0u, nullptr};
  return decode_impl("kda_decode_step", q, k, v, dtype, gs, beta, state, B, H, K, V, layout, o, stream);
}

int kda_decode_step_logits(const void* q, const void* k, const void* v, kda_dtype dtype,
                           const float* logits, const float* A_log, const float* dt_bias, float g_min,
                           const float* beta, unsigned flags,
                           float* state, int64_t B, int64_t H, int64_t K, int64_t V,
                           const kda_layout* layout, void* o, kda_stream_t stream) {
  const GateSpec gs{logits, (flags & KDA_GATE_SOFTPLUS) ? kda::GATE_SOFTPLUS : kda::GATE_LOGITS, A_log, g_min, flags,
                    dt_bias};
  return decode_impl("kda_decode_step_logits", q, k, v, dtype, gs, beta, state, B, H, K, V, layout, o, stream);
}

int kda_scan_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, int64_t n_seq,
                                      size_t* bytes) {
  if (!bytes) return fail(KDA_ERR_INVALID_ARG, "kda_scan_backward_workspace_bytes: null output");
  if (B < 0 || T < 0 || H < 0 || K < 0 || V < 0 || n_seq < 0)
    return fail(KDA_ERR_INVALID_ARG, "kda_scan_backward_workspace_bytes: negative size");
  *bytes = kda::backward_workspace_bytes(B, T, H, K, V, n_seq);
  return ok();
}

int kda_scan_backward(const void* q, const void* k, const void* v, kda_dtype dtype,
                      const float* gate, kda_gate_kind gate_kind, const float* beta,
                      const float* initial_state, const float* d_o, const float* d_final_state,
                      const int32_t* cu_seqlens, int64_t n_seq,
                      int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, const kda_layout* layout,
                      float* dq, float* dk, float* dv, float* dgate, float* dbeta, float* d_initial_state,
                      void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  const char* fn = "kda_scan_backward";
  if (B < 0 || T < 0 || H < 0 || n_seq < 0) return fail(KDA_ERR_INVALID_ARG, "%s: negative size", fn);
  int64_t N = B;  // sequences
  if (cu_seqlens) {
    if (B != 1) return fail(KDA_ERR_INVALID_ARG, "%s: cu_seqlens requires B == 1 (got %lld)", fn, (long long)B);
    N = n_seq;
  }
  if (!valid_dtype(dtype)) return fail(KDA_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  if (gate_kind != KDA_GATE_ALPHA && gate_kind != KDA_GATE_LOG)
    return fail(KDA_ERR_INVALID_ARG, "%s: unknown gate kind %d", fn, (int)gate_kind);
  if (!kda::backward_supported((int)K, (int)V))
    return fail(KDA_ERR_UNSUPPORTED, "%s: K and V must be 16, 32, 64 or 128 (K=%lld, V=%lld)", fn, (long long)K,
                (long long)V);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (N * H == 0) return ok();
  if (T == 0) {  // nothing to differentiate through: dS_0 = dS_T
    if (d_initial_state) {
      cudaError_t e = kda::launch_state_copy(d_final_state, d_initial_state, N * H * K * V, s);
      if (e != cudaSuccess) return cuda_fail(e, fn);
    }
    return ok();
  }
  if (!q || !k || !v || !gate || !beta || !d_o || !dq || !dk || !dv || !dgate || !dbeta)
    return fail(KDA_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  if (T > INT32_MAX) return fail(KDA_ERR_UNSUPPORTED, "%s: T too large", fn);
  const int64_t n_ws = cu_seqlens ? N : 0;
  const size_t need = kda::backward_workspace_bytes(B, T, H, K, V, n_ws);
  if (!workspace || workspace_bytes < need)
    return fail(KDA_ERR_INVALID_ARG, "%s: the workspace needs %zu bytes (got %zu)", fn, need, workspace_bytes);
  kda_layout L;
  if (layout) {
    L = *layout;
  } else {
    L.q = contiguous(T, H, K);
    L.k = contiguous(T, H, K);
    L.gate = contiguous(T, H, K);
    L.v = contiguous(T, H, V);
    L.o = contiguous(T, H, V);
    L.beta = contiguous(T, H, 1);
  }
  const kda_strides* all[5] = {&L.q, &L.k, &L.v, &L.gate, &L.beta};
  for (auto* st : all)
    if (!strides_valid(*st)) return fail(KDA_ERR_INVALID_ARG, "%s: negative stride", fn);
  const size_t es = elem_size(dtype);
  if (!rows_aligned(q, L.q, es, B, T, H) || !rows_aligned(k, L.k, es, B, T, H) ||
      !rows_aligned(v, L.v, es, B, T, H) || !rows_aligned(gate, L.gate, 4, B, T, H) || !aligned16(d_o) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dgate) || !aligned16(workspace) ||
      (initial_state && !aligned16(initial_state)) || (d_final_state && !aligned16(d_final_state)) ||
      (d_initial_state && !aligned16(d_initial_state)))
    return fail(KDA_ERR_UNSUPPORTED, "%s: rows and buffers must start on 16-byte boundaries", fn);
  kda::BwdParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.gate = gate;
  p.beta = beta;
  p.s0 = initial_state;
  p.d_o = d_o;
  p.d_sf = d_final_state;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dgate = dgate;
  p.dbeta = dbeta;
  p.ds0 = d_initial_state;
  p.cu = cu_seqlens;
  p.ckpt_slots = kda::backward_ckpt_slots(T, n_ws);
  p.ckpt = static_cast<float*>(workspace);
  p.scratch = p.ckpt + (size_t)(cu_seqlens ? H : B * H) * p.ckpt_slots * K * V;
  put(p.qs, L.q);
  put(p.ks, L.k);
  put(p.vs, L.v);
  put(p.gs, L.gate);
  put(p.bs, L.beta);
  p.T = T;
  p.B = (int)B;
  p.N = (int)N;
  p.H = (int)H;
  p.K = (int)K;
  p.V = (int)V;
  p.gate_log = gate_kind == KDA_GATE_LOG;
  cudaError_t e = kda::launch_scan_backward(p, dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

namespace {
// Workspace of the chunked backward: with packed sequences the forward's slots (T / 64 + n_seq + 1 per head)
// are laid out as one row of that many full chunks.
size_t chunked_bwd_bytes(int64_t B, int64_t T, int64_t H, int64_t n_seq) {
  if (n_seq > 0) return T * H == 0 ? 0 : kda::chunked_backward_workspace_bytes(1, 64 * (T / 64 + n_seq + 1), H);
  return B * T * H == 0 ? 0 : kda::chunked_backward_workspace_bytes(B, T, H);
}
}  // namespace

int kda_scan_backward_chunked_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, int64_t n_seq,
                                              size_t* bytes) {
  if (!bytes) return fail(KDA_ERR_INVALID_ARG, "kda_scan_backward_chunked_workspace_bytes: null output");
  if (B < 0 || T < 0 || H < 0 || K < 0 || V < 0 || n_seq < 0)
    return fail(KDA_ERR_INVALID_ARG, "kda_scan_backward_chunked_workspace_bytes: negative size");
  if (K != 128 || V != 128)
    return fail(KDA_ERR_UNSUPPORTED, "kda_scan_backward_chunked_workspace_bytes: K and V must be 128");
  *bytes = chunked_bwd_bytes(B, T, H, n_seq);
  return ok();
}

int kda_scan_backward_chunked(const void* q, const void* k, const void* v, kda_dtype dtype,
                              const float* gate, kda_gate_kind gate_kind, const float* beta,
                              const float* initial_state, const float* d_o, const float* d_final_state,
                              const int32_t* cu_seqlens, int64_t n_seq,
                              int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, const kda_layout* layout,
                              float* dq, float* dk, float* dv, float* dgate, float* dbeta, float* d_initial_state,
                              void* workspace, size_t workspace_bytes, kda_stream_t stream) {
  const char* fn = "kda_scan_backward_chunked";
  if (B < 0 || T < 0 || H < 0 || n_seq < 0) return fail(KDA_ERR_INVALID_ARG, "%s: negative size", fn);
  int64_t N = B;  // sequences
  if (cu_seqlens) {
    if (B != 1) return fail(KDA_ERR_INVALID_ARG, "%s: cu_seqlens requires B == 1 (got %lld)", fn, (long long)B);
    N = n_seq;
  }
  if (!valid_dtype(dtype)) return fail(KDA_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  if (gate_kind != KDA_GATE_ALPHA && gate_kind != KDA_GATE_LOG)
    return fail(KDA_ERR_INVALID_ARG, "%s: unknown gate kind %d", fn, (int)gate_kind);
  if (dtype != KDA_BF16 || K != 128 || V != 128)
    return fail(KDA_ERR_UNSUPPORTED, "%s: bf16 q, k, v with K = V = 128 only", fn);
  if (H > 65535) return fail(KDA_ERR_UNSUPPORTED, "%s: H must be at most 65535", fn);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (N * H == 0) return ok();
  if (T == 0) {  // nothing to differentiate through: dS_0 = dS_T
    if (d_initial_state) {
      cudaError_t e = kda::launch_state_copy(d_final_state, d_initial_state, N * H * K * V, s);
      if (e != cudaSuccess) return cuda_fail(e, fn);
    }
    return ok();
  }
  if (!q || !k || !v || !gate || !beta || !d_o || !dq || !dk || !dv || !dgate || !dbeta)
    return fail(KDA_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  const int64_t n_slots = cu_seqlens ? T / 64 + N + 1 : (T + 63) / 64 * B;
  if (T > INT32_MAX || n_slots * H > INT32_MAX / 2 || N > INT32_MAX)  // two CTAs per chunk-head in one kernel
    return fail(KDA_ERR_UNSUPPORTED, "%s: T too large", fn);
  const size_t need = chunked_bwd_bytes(B, T, H, cu_seqlens ? N : 0);
  if (!workspace || workspace_bytes < need)
    return fail(KDA_ERR_INVALID_ARG, "%s: the workspace needs %zu bytes (got %zu)", fn, need, workspace_bytes);
  kda_layout L;
  if (layout) {
    L = *layout;
  } else {
    L.q = contiguous(T, H, K);
    L.k = contiguous(T, H, K);
    L.gate = contiguous(T, H, K);
    L.v = contiguous(T, H, V);
    L.o = contiguous(T, H, V);
    L.beta = contiguous(T, H, 1);
  }
  const kda_strides* all[5] = {&L.q, &L.k, &L.v, &L.gate, &L.beta};
  for (auto* st : all)
    if (!strides_valid(*st)) return fail(KDA_ERR_INVALID_ARG, "%s: negative stride", fn);
  if (!rows_aligned(q, L.q, 2, B, T, H) || !rows_aligned(k, L.k, 2, B, T, H) || !rows_aligned(v, L.v, 2, B, T, H) ||
      !rows_aligned(gate, L.gate, 4, B, T, H) || !aligned16(d_o) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || !aligned16(dgate) || !aligned16(workspace) || (initial_state && !aligned16(initial_state)) ||
      (d_final_state && !aligned16(d_final_state)) || (d_initial_state && !aligned16(d_initial_state)))
    return fail(KDA_ERR_UNSUPPORTED, "%s: rows and buffers must start on 16-byte boundaries", fn);
  kda::ScanParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.gate = gate;
  p.beta = beta;
  p.s0 = initial_state;
  p.sf = nullptr;
  p.cu = cu_seqlens;
  p.o = nullptr;
  put(p.qs, L.q);
  put(p.ks, L.k);
  put(p.vs, L.v);
  put(p.gs, L.gate);
  put(p.bs, L.beta);
  p.T = T;
  p.B = (int)B;
  p.H = (int)H;
  p.K = (int)K;
  p.V = (int)V;
  p.N = (int)N;
  p.gate_mode = (int)gate_kind;
  p.A_log = nullptr;
  p.dt_bias = nullptr;
  p.g_min = 0.f;
  p.qk_l2norm = 0;
  p.beta_sigmoid = 0;
  p.state_vk = 0;
  if (!kda::split_maps_ok(p)) return fail(KDA_ERR_UNSUPPORTED, "%s: the q, k or gate layout admits no tensor map", fn);
  int cublas_status = 0;
  cudaError_t e = kda::launch_chunked_backward(p, d_o, d_final_state, dq, dk, dv, dgate, dbeta, d_initial_state,
                                               workspace, s, &cublas_status);
  if (cublas_status != 0) return fail(KDA_ERR_CUDA, "%s: cuBLAS status %d", fn, cublas_status);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

int kda_bounded_decay_backward(const float* logits, const float* A_log, float g_min, const float* d_log_decay,
                               int64_t B, int64_t T, int64_t H, int64_t K, float* d_logits, float* d_A_log,
                               kda_stream_t stream) {
  const char* fn = "kda_bounded_decay_backward";
  if (B < 0 || T < 0 || H < 0 || K < 0) return fail(KDA_ERR_INVALID_ARG, "%s: negative size", fn);
  if (!std::isfinite(g_min) || !(g_min < 0.f))
    return fail(KDA_ERR_INVALID_ARG, "%s: g_min must be finite and < 0 (got %g)", fn, (double)g_min);
  if (H == 0) return ok();
  if (!A_log || !d_A_log || (B * T * K > 0 && (!logits || !d_log_decay || !d_logits)))
    return fail(KDA_ERR_INVALID_ARG, "%s: null pointer", fn);
  cudaError_t e = kda::launch_bounded_decay_backward(logits, A_log, g_min, d_log_decay, B * T, (int)H, (int)K,
                                                     d_logits, d_A_log, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

}  // extern "C"
