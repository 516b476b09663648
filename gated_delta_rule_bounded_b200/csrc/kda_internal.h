// kda_internal.h -- host/device interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// Internal gate mode of a scan, next to KDA_GATE_ALPHA (0) and KDA_GATE_LOG (1): the gate tensor
// holds the decay logits z, and ScanParams::A_log / g_min complete the bounded gate.
constexpr int GATE_LOGITS = 2;
// The gate tensor holds logits z of Kimi Linear's unbounded gate, alpha = exp(-e^{A_h} softplus(z)).
// Per-token decay is then not bounded below, so scans in this mode take the token-by-token kernel.
constexpr int GATE_SOFTPLUS = 3;  // both logit modes (>= GATE_LOGITS) use the per-head scale e^{A_h}

// Everything a scan kernel needs, passed by value. Strides are in elements, for
// the B, T and H dimensions of each token tensor; the innermost dim is contiguous.
struct ScanParams {
  const void* q;
  const void* k;
  const void* v;
  const float* gate;  // alpha, g = log(alpha), or the logits z, per gate_mode
  const float* beta;
  const float* s0;    // [N,H,K,V] or nullptr (zeros)
  float* sf;          // [N,H,K,V] or nullptr (not written)
  const int32_t* cu;  // [N+1] packed offsets or nullptr
  void* o;
  int64_t qs[3], ks[3], vs[3], gs[3], bs[3], os[3];
  int64_t T;
  int B, H, K, V, N;
  int gate_mode;        // KDA_GATE_ALPHA, KDA_GATE_LOG, or GATE_LOGITS (gate holds decay logits z)
  const float* A_log;   // [H], logit gate modes only
  const float* dt_bias; // [H,K] or nullptr, logit gate modes only: added to z before the gate
  float g_min;          // GATE_LOGITS only
  int qk_l2norm;        // q, k are L2-normalised over K inside the kernels
  int beta_sigmoid;     // beta holds logits; the kernels use sigmoid(beta)
  int state_vk;         // states stored [N,H,V,K] (K contiguous) instead of [N,H,K,V]
  float* s_dump = nullptr;  // split path only: the state at every chunk start, fp32 [slot][H][K][V] (or null)
};

// Offset of state element (key row c, value column v) of a head whose state starts at `head_base`.
__host__ __device__ inline size_t state_at(const ScanParams& p, size_t head_base, int c, int v) {
  return p.state_vk ? head_base + (size_t)v * p.K + c : head_base + (size_t)c * p.V + v;
}

struct GateParams {
  const void* z;
  void* out;
  const float* A_log;
  int64_t zs[3], os[3];
  int64_t B, T, H, K;
  float g_min;
  int out_log;
  int softplus;  // Kimi Linear's unbounded gate instead of the bounded one (g_min unused)
};

// Gradients of the scan (backward.cu). Inputs as for the forward scan (per-element strides for B, T,
// H); d_o [B,T,H,V], d_sf [B,H,K,V] (or null) and every output fp32 and contiguous.
struct BwdParams {
  const void* q;
  const void* k;
  const void* v;
  const float* gate;  // alpha, or g = log(alpha) when gate_log != 0
  const float* beta;
  const float* s0;    // [B,H,K,V] or nullptr (zeros)
  const float* d_o;
  const float* d_sf;  // or nullptr (zeros)
  float *dq, *dk, *dv, *dgate, *dbeta;
  float* ds0;         // or nullptr (not written)
  float* ckpt;        // workspace: checkpoints, then the per-CTA segment scratch
  float* scratch;
  const int32_t* cu;  // [N + 1] sequence offsets (B == 1), or nullptr: one sequence per batch row
  int64_t ckpt_slots; // with cu: checkpoint slots per head
  int64_t qs[3], ks[3], vs[3], gs[3], bs[3];
  int64_t T;
  int B, N, H, K, V;  // N: sequences (B without cu)
  int gate_log;
};
bool backward_supported(int K, int V);
// Checkpoint slots per head: (T/32 rounded up + 1) per batch row without cu_seqlens; with n_seq packed
// sequences, floor(T/32) + 2 n_seq + 1 shared by the sequences of a head (sequence n starts at slot
// floor(cu[n]/32) + 2n, which keeps them disjoint).
int64_t backward_ckpt_slots(int64_t T, int64_t n_seq);
size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, int64_t n_seq);
cudaError_t launch_scan_backward(const BwdParams& p, kda_dtype dt, cudaStream_t s);
cudaError_t launch_bounded_decay_backward(const float* z, const float* A_log, float g_min, const float* dg,
                                          int64_t rows_bt, int H, int K, float* dz, float* dA, cudaStream_t s);

// Launchers return the launch status (cudaGetLastError after the launch).
cudaError_t launch_gate(const GateParams& p, kda_dtype dt, cudaStream_t s);
// Token-by-token kernel: the decode step (T = 1, s0 == sf) and the generic
// prefill path (fp32 inputs, any supported K and V).
cudaError_t launch_recurrent(const ScanParams& p, kda_dtype dt, cudaStream_t s);
// Decode step for K = V = 128 with whole-state bulk copies (persistent, one CTA per SM).
bool decode_bulk_supported(const ScanParams& p);
cudaError_t launch_decode_bulk(const ScanParams& p, kda_dtype dt, cudaStream_t s);
cudaError_t decode_read_timeout(int* flag, bool reset);
// Chunked prefill for bf16 inputs (bounded decay), tensor cores.
// With a workspace of chunk_workspace_bytes(...) it runs as two kernels (all chunks' state-independent
// operands in parallel, then the recurrence); without one, as a single fused kernel.
bool chunk_supported(int K, int V, kda_dtype dt);
size_t chunk_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t n_seq);
cudaError_t launch_chunk(const ScanParams& p, void* ws, size_t ws_bytes, cudaStream_t s);
size_t split_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N, bool varlen);
cudaError_t launch_chunk_split(const ScanParams& p, void* ws, cudaStream_t s);
// Gradients through the chunkwise form (backward_chunked.cu): bf16 q/k/v, K = V = 128, dense batch rows.
size_t chunked_backward_workspace_bytes(int64_t B, int64_t T, int64_t H);
cudaError_t launch_chunked_backward(const ScanParams& fwd, const float* d_o, const float* d_sf, float* dq, float* dk,
                                    float* dv, float* dgate, float* dbeta, float* ds0, void* ws, cudaStream_t s,
                                    int* cublas_status);
// Whether the driver accepts tensor maps of this call's q, k and gate layouts (the two-kernel path reads
// them by TMA); when it does not, the single fused kernel runs instead.
bool split_maps_ok(const ScanParams& p);
cudaError_t launch_wait_selftest(cudaStream_t s);  // one wait that expires (kda_selftest_wait_expiry)
cudaError_t split_read_timeout(int* flag, bool reset);
// Reads (and optionally clears) the chunk kernel's device-side timeout flag. Synchronous.
cudaError_t chunk_read_timeout(int* flag, bool reset);
// Records `msg` as the calling thread's kda_last_error() and returns `code`.
int report_error(int code, const char* msg);
// Copy initial state (or zeros) into final state for T == 0 calls.
cudaError_t launch_state_copy(const float* s0, float* sf, int64_t n, cudaStream_t s);

}  // namespace kda
