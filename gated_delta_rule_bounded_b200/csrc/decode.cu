// decode.cu -- the in-place decode step for K = V = 128, streaming whole head states through
// shared memory with bulk asynchronous copies.
//
// Per head ("Kimi K3: Bounded Decay and Delta Memory", eq. 1, one token):
//     Sbar = Diag(alpha) S;  delta = v - Sbar^T k;  S = Sbar + beta k delta^T;
//     o = S^T q = Sbar^T q + beta (k.q) delta
// The state of one (b, h) is a contiguous 64 KB block, so it moves as one bulk copy
// (cp.async.bulk, completion counted in bytes on an mbarrier; no multicast). One
// persistent CTA per SM walks heads blockIdx.x, blockIdx.x + gridDim.x, ... through a
// 3-stage ring: while head i is computed out of shared memory, head i+1 is loading
// and head i-1's updated state is being written back by a bulk store. Each thread
// owns a float4 column group of 16 key rows; the two key reductions are per-thread
// partial sums plus one shared-memory reduction over the 8 row groups. The state is
// read from and written to HBM exactly once. Waits are iteration-limited; an expired
// wait records a device flag and stops the CTA.
#include <atomic>

#include "common.cuh"
#include "gate_math.cuh"
#include "kda_internal.h"

namespace kda {

// Set to 1 by any decode CTA whose bounded wait on a bulk copy expired.
__device__ int g_decode_timeout = 0;

namespace {

constexpr int DK = 128, DV = 128, DNT = 256, NSTAGE = 3, ROWS = DK / 8;

template <typename TIn>
struct StageLayout {
  static constexpr int IN = DK * (int)sizeof(TIn);  // bytes of one q / k / v row
  static constexpr int STATE = 0;
  static constexpr int Q = DK * DV * 4;
  static constexpr int K = Q + IN;
  static constexpr int V = K + IN;
  static constexpr int A = V + IN;
  static constexpr int BYTES = A + DK * 4;          // + alpha row (fp32)
  static constexpr int RED = NSTAGE * BYTES;        // partial sums [2][8][128] + k.q, k.k, q.q [3][8]
  static constexpr int BAR = RED + (2 * 8 * DV + 24) * 4;
  static constexpr int SMEM = BAR + NSTAGE * 8;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait_bounded(bar, parity)) return true;
  atomicExch(&g_decode_timeout, 1);
  return false;
}

template <typename TIn>
struct HeadPtrs {
  const TIn *q, *k, *v;
  const float *a, *beta;
  float* state;
  TIn* o;
};

template <typename TIn>
__device__ __forceinline__ HeadPtrs<TIn> head_ptrs(const ScanParams& p, int head) {
  const int b = head / p.H, h = head % p.H;
  HeadPtrs<TIn> r;
  r.q = static_cast<const TIn*>(p.q) + b * p.qs[0] + h * p.qs[2];
  r.k = static_cast<const TIn*>(p.k) + b * p.ks[0] + h * p.ks[2];
  r.v = static_cast<const TIn*>(p.v) + b * p.vs[0] + h * p.vs[2];
  r.a = p.gate + b * p.gs[0] + h * p.gs[2];
  r.beta = p.beta + b * p.bs[0] + h * p.bs[2];
  r.state = p.sf + (size_t)head * DK * DV;
  r.o = static_cast<TIn*>(p.o) + b * p.os[0] + h * p.os[2];
  return r;
}

// One thread (tid 0) arms the stage's mbarrier with the byte count and issues the five copies.
template <typename TIn>
__device__ __forceinline__ void issue_stage(const ScanParams& p, int head, uint32_t stage_base, uint32_t bar) {
  using L = StageLayout<TIn>;
  const HeadPtrs<TIn> hp = head_ptrs<TIn>(p, head);
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"((uint32_t)(L::BYTES))
               : "memory");
  bulk_load(stage_base + L::STATE, hp.state, DK * DV * 4, bar);
  bulk_load(stage_base + L::Q, hp.q, L::IN, bar);
  bulk_load(stage_base + L::K, hp.k, L::IN, bar);
  bulk_load(stage_base + L::V, hp.v, L::IN, bar);
  bulk_load(stage_base + L::A, hp.a, DK * 4, bar);
}

// VK: the states are stored value-by-key ([V][K]) instead of key-by-value.
template <typename TIn, bool VK>
__global__ void __launch_bounds__(DNT, 1) decode_bulk_kernel(ScanParams p) {
  using L = StageLayout<TIn>;
  extern __shared__ __align__(128) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int tv = tid & 31, tk = tid >> 5;   // column group (4 columns), row group (16 rows)
  const int row0 = ROWS * tk, col0 = 4 * tv;
  const int nheads = p.B * p.H;
  const int n_my = blockIdx.x < nheads ? (nheads - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  float* red_a = reinterpret_cast<float*>(sm + L::RED);
  float* red_b = red_a + 8 * DV;
  float* red_kq = red_b + 8 * DV;
  float* red_kk = red_kq + 8;  // sums of k^2 and q^2 (in-kernel L2 normalisation)
  float* red_qq = red_kk + 8;
  const uint32_t bar0 = sb + L::BAR;

  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8 * s));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  int issued = 0;  // heads whose loads have been issued (meaningful in thread 0)
  if (tid == 0)
    for (; issued < NSTAGE && issued < n_my; ++issued)
      issue_stage<TIn>(p, blockIdx.x + issued * gridDim.x, sb + issued * L::BYTES, bar0 + 8 * issued);
  int done_heads = 0;
  float beta_next = n_my > 0 ? beta_value(__ldg(head_ptrs<TIn>(p, blockIdx.x).beta), p.beta_sigmoid) : 0.f;

  for (int i = 0; i < n_my; ++i) {
    const int head = blockIdx.x + i * gridDim.x;
    const float sc = p.gate_mode >= GATE_LOGITS ? expf(__ldg(p.A_log + head % p.H)) : 0.f;  // e^{A_h}
    const int s = i % NSTAGE;
    unsigned char* st = sm + s * L::BYTES;
    const float beta = beta_next;
    if (i + 1 < n_my) beta_next = beta_value(__ldg(head_ptrs<TIn>(p, head + gridDim.x).beta), p.beta_sigmoid);
    if (!__syncthreads_and(mbar_wait(bar0 + 8 * s, (i / NSTAGE) & 1))) break;
    done_heads = i + 1;

    const TIn* qs = reinterpret_cast<const TIn*>(st + L::Q);
    const TIn* ks = reinterpret_cast<const TIn*>(st + L::K);
    const TIn* vs = reinterpret_cast<const TIn*>(st + L::V);
    float* as = reinterpret_cast<float*>(st + L::A);
    // The staged gate row becomes alpha in place, once per head (each row is read by many threads).
    if (p.gate_mode != KDA_GATE_ALPHA) {
      for (int c = tid; c < DK; c += blockDim.x) {
        const float b = p.dt_bias ? __ldg(p.dt_bias + (size_t)(head % p.H) * DK + c) : 0.f;
        as[c] = gate_alpha(p.gate_mode, gate_input(p.gate_mode, as[c], b), sc, p.g_min);
      }
      __syncthreads();
    }
    float* S = reinterpret_cast<float*>(st + L::STATE);

    if constexpr (!VK) {
      float4 x[ROWS];
      float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
      float pkq = 0.f, pkk = 0.f, pqq = 0.f;
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const int row = row0 + r;
        const float a = as[row], kk = to_f32(ks[row]), qq = to_f32(qs[row]);
        x[r] = *reinterpret_cast<const float4*>(S + row * DV + col0);
        x[r].x *= a; x[r].y *= a; x[r].z *= a; x[r].w *= a;
        pa.x = fmaf(kk, x[r].x, pa.x); pa.y = fmaf(kk, x[r].y, pa.y);
        pa.z = fmaf(kk, x[r].z, pa.z); pa.w = fmaf(kk, x[r].w, pa.w);
        pb.x = fmaf(qq, x[r].x, pb.x); pb.y = fmaf(qq, x[r].y, pb.y);
        pb.z = fmaf(qq, x[r].z, pb.z); pb.w = fmaf(qq, x[r].w, pb.w);
        pkq = fmaf(kk, qq, pkq);
        pkk = fmaf(kk, kk, pkk);
        pqq = fmaf(qq, qq, pqq);
      }
      *reinterpret_cast<float4*>(red_a + tk * DV + col0) = pa;
      *reinterpret_cast<float4*>(red_b + tk * DV + col0) = pb;
      if (tv == 0) {
        red_kq[tk] = pkq;
        red_kk[tk] = pkk;
        red_qq[tk] = pqq;
      }
      __syncthreads();
      float4 A = make_float4(0.f, 0.f, 0.f, 0.f), Bq = A;
      float kq = 0.f, kk2 = 0.f, qq2 = 0.f;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float4 ya = *reinterpret_cast<const float4*>(red_a + g * DV + col0);
        const float4 yb = *reinterpret_cast<const float4*>(red_b + g * DV + col0);
        A.x += ya.x; A.y += ya.y; A.z += ya.z; A.w += ya.w;
        Bq.x += yb.x; Bq.y += yb.y; Bq.z += yb.z; Bq.w += yb.w;
        kq += red_kq[g];
        kk2 += red_kk[g];
        qq2 += red_qq[g];
      }
      // In-kernel L2 normalisation of k and q: every term is linear in each, so the scales apply to the
      // sums (k^T S, q^T S, k^T q) and to the rank-1 update.
      const float ik = p.qk_l2norm ? l2norm_scale(kk2) : 1.f, iq = p.qk_l2norm ? l2norm_scale(qq2) : 1.f;
      if (p.qk_l2norm) {
        A.x *= ik; A.y *= ik; A.z *= ik; A.w *= ik;
        Bq.x *= iq; Bq.y *= iq; Bq.z *= iq; Bq.w *= iq;
        kq *= ik * iq;
      }
      const float4 vv = load4(vs + col0);
      const float4 d = make_float4(vv.x - A.x, vv.y - A.y, vv.z - A.z, vv.w - A.w);
      if (tk == 0) {
        const float bkq = beta * kq;
        store4(head_ptrs<TIn>(p, head).o + col0, make_float4(fmaf(bkq, d.x, Bq.x), fmaf(bkq, d.y, Bq.y),
                                                            fmaf(bkq, d.z, Bq.z), fmaf(bkq, d.w, Bq.w)));
      }
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const int row = row0 + r;
        const float bk = beta * (to_f32(ks[row]) * ik);
        x[r].x = fmaf(bk, d.x, x[r].x); x[r].y = fmaf(bk, d.y, x[r].y);
        x[r].z = fmaf(bk, d.z, x[r].z); x[r].w = fmaf(bk, d.w, x[r].w);
        *reinterpret_cast<float4*>(S + row * DV + col0) = x[r];
      }
    } else {
      // Value-by-key state, S[v][k]: warp w owns value rows 16w .. 16w+15 and lane l the key columns
      // 4l .. 4l+3, so a warp reads each row as 512 contiguous bytes. The sums over k are warp
      // reductions: a reduce-scatter leaves lane l with row 16w + l's k^T Sbar (lanes 0-15) or
      // q^T Sbar (lanes 16-31), and delta goes back to every lane by shuffles.
      const int w = tid >> 5, l = tid & 31;
      const float4 a4 = *reinterpret_cast<const float4*>(as + 4 * l);
      const float4 k4 = load4(ks + 4 * l), q4 = load4(qs + 4 * l);
      float4 x[16];
      float red[32];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        x[r] = *reinterpret_cast<const float4*>(S + (16 * w + r) * DK + 4 * l);
        x[r].x *= a4.x; x[r].y *= a4.y; x[r].z *= a4.z; x[r].w *= a4.w;
        red[r] = fmaf(k4.x, x[r].x, fmaf(k4.y, x[r].y, fmaf(k4.z, x[r].z, k4.w * x[r].w)));
        red[16 + r] = fmaf(q4.x, x[r].x, fmaf(q4.y, x[r].y, fmaf(q4.z, x[r].z, q4.w * x[r].w)));
      }
#pragma unroll
      for (int step = 0; step < 5; ++step) {
        const int wd = 16 >> step;
        const bool up = (l & wd) != 0;
#pragma unroll
        for (int j = 0; j < wd; ++j) {
          const float send = up ? red[j] : red[j + wd];
          const float recv = __shfl_xor_sync(0xffffffffu, send, wd);
          red[j] = (up ? red[j + wd] : red[j]) + recv;
        }
      }
      float kq = fmaf(k4.x, q4.x, fmaf(k4.y, q4.y, fmaf(k4.z, q4.z, k4.w * q4.w)));
      float kk2 = fmaf(k4.x, k4.x, fmaf(k4.y, k4.y, fmaf(k4.z, k4.z, k4.w * k4.w)));
      float qq2 = fmaf(q4.x, q4.x, fmaf(q4.y, q4.y, fmaf(q4.z, q4.z, q4.w * q4.w)));
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) {
        kq += __shfl_xor_sync(0xffffffffu, kq, m);
        kk2 += __shfl_xor_sync(0xffffffffu, kk2, m);
        qq2 += __shfl_xor_sync(0xffffffffu, qq2, m);
      }
      const float ik = p.qk_l2norm ? l2norm_scale(kk2) : 1.f, iq = p.qk_l2norm ? l2norm_scale(qq2) : 1.f;
      const float mine = red[0] * (l < 16 ? ik : iq);  // k^T Sbar (l < 16) or q^T Sbar of row 16w + (l & 15)
      const float qs_row = __shfl_sync(0xffffffffu, mine, (l + 16) & 31);
      float delta = 0.f;
      if (l < 16) {
        const int vrow = 16 * w + l;
        delta = to_f32(vs[vrow]) - mine;
        const float o = fmaf(beta * (kq * ik * iq), delta, qs_row);
        head_ptrs<TIn>(p, head).o[vrow] = from_f32<TIn>(o);
      }
      const float bk = beta * ik;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float d = __shfl_sync(0xffffffffu, delta, r);
        x[r].x = fmaf(bk * k4.x, d, x[r].x); x[r].y = fmaf(bk * k4.y, d, x[r].y);
        x[r].z = fmaf(bk * k4.z, d, x[r].z); x[r].w = fmaf(bk * k4.w, d, x[r].w);
        *reinterpret_cast<float4*>(S + (16 * w + r) * DK + 4 * l) = x[r];
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();  // the updated state is in shared memory; the partial sums are consumed
    if (tid == 0) {
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(head_ptrs<TIn>(p, head).state),
                   "r"(sb + s * L::BYTES + L::STATE), "r"(DK * DV * 4)
                   : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      // Refill the stage of head i-1 (its write-back was committed one head ago) with head i-1+NSTAGE.
      const int j = i - 1 + NSTAGE;
      if (i >= 1 && j < n_my) {
        asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        const int sj = (i - 1) % NSTAGE;
        issue_stage<TIn>(p, blockIdx.x + j * gridDim.x, sb + sj * L::BYTES, bar0 + 8 * sj);
        issued = j + 1;
      }
    }
  }
  if (tid == 0) {
    // After an expired wait, give every load still in flight a bounded wait before the CTA's shared
    // memory goes away; then drain the write-backs.
    for (int j = done_heads; j < issued; ++j) mbar_wait(bar0 + 8 * (j % NSTAGE), (j / NSTAGE) & 1);
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
}

template <typename TIn>
cudaError_t launch_bulk(const ScanParams& p, cudaStream_t s) {
  using L = StageLayout<TIn>;
  static std::atomic<uint64_t> configured{0};
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;  // one configuration bit per device
  const uint64_t bit = 1ull << dev;
  if (!(configured.load(std::memory_order_relaxed) & bit)) {
    e = cudaFuncSetAttribute(decode_bulk_kernel<TIn, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_bulk_kernel<TIn, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int nheads = p.B * p.H;
  const int grid = nheads < sms ? nheads : sms;
  if (grid == 0) return cudaSuccess;
  if (p.state_vk)
    decode_bulk_kernel<TIn, true><<<grid, DNT, L::SMEM, s>>>(p);
  else
    decode_bulk_kernel<TIn, false><<<grid, DNT, L::SMEM, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool decode_bulk_supported(const ScanParams& p) {
  // Whole-state bulk copies need K = V = 128 and the state updated in place.
  return p.K == DK && p.V == DV && p.s0 == p.sf && p.sf != nullptr;
}

cudaError_t launch_decode_bulk(const ScanParams& p, kda_dtype dt, cudaStream_t s) {
  return dt == KDA_F32 ? launch_bulk<float>(p, s) : launch_bulk<__nv_bfloat16>(p, s);
}

cudaError_t decode_read_timeout(int* flag, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_decode_timeout, sizeof(int));
  if (e != cudaSuccess || !reset) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_decode_timeout, &zero, sizeof(int));
}

}  // namespace kda
