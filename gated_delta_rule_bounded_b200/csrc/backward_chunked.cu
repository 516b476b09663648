// backward_chunked.cu -- gradients of the scan through the chunkwise form, in parallel over chunks.
//
// The chunkwise form of eq. 1 ("Kimi K3: Bounded Decay and Delta Memory"; the "KDA cheat sheet",
// chunkwise form, eqs. 3-4) per chunk of n <= 64 tokens of one head, with G the chunk-local cumulative
// log-decay per channel, Gamma = e^G, gamma_C = e^{G_last}:
//   Mq[t][i] = sum_c q_tc k_ic e^{G_tc - G_ic} (i <= t),  Mk[t][i] = sum_c k_tc k_ic e^{G_tc - G_ic} (i < t),
//   T = (I + Diag(beta) Mk)^-1, TB = T Diag(beta), W = TB (K*Gamma), U = TB V - W S0,
//   O = (Q*Gamma) S0 + Mq U, S_C = Diag(gamma_C) S0 + (K*gamma_C/Gamma)^T U.
// Its adjoint, given dO and dS_C (the gradient at the chunk's end):
//   dU = Mq^T dO + KT dS_C,  dS0 = QG^T dO + Diag(gamma_C) dS_C - W^T dU        (KT = K*gamma_C/Gamma, QG = Q*Gamma)
//   dMq = tril(dO U^T), dQG = dO S0^T, dKT = U dS_C^T, dgamma_C = rowsum(dS_C * S0), dW = -dU S0^T,
//   dTB = dU V^T + dW KG^T, dV = TB^T dU, dKG = TB^T dW, dA = strict_tril(-T^T (dTB Diag(beta)) T^T),
//   dbeta = colsum(dTB * T) + rowsum(dA * Mk), dMk = Diag(beta) dA,
// and the bilinear forms Mq, Mk with the Gamma factors give dq, dk and dG; dlog(alpha) is dG's reverse
// cumulative sum within the chunk. dS0 of a chunk is dS_C of the one before, so the gradient of the state is
// one reverse recurrence over chunks; everything else is independent per chunk.
//
// Passes (one head per (batch row, head); b = (row * chunks + chunk) * H + head indexes a chunk of a head):
//   1. the forward's split kernels with the state at every chunk start kept (S0, fp32);
//   2. per chunk: fp32 copies of q, k, v, dO (zero past the end), the log2 cumulative decay, Q*Gamma,
//      K*Gamma, K*gamma_C/Gamma, gamma_C (prep_kernel); Mq and Mk with every decay ratio e^{G_t - G_i} <= 1
//      formed per pair and channel (pair_kernel); T and TB (inverse_kernel);
//   3. plain dense products of the chunk matrices as batched GEMMs (cuBLAS, fp32 with TF32 tensor cores);
//   4. the reverse recurrence over chunks for dS (dstate_kernel, value columns split over CTAs: the
//      recurrence is separable in the value index);
//   5. the remaining products, then per chunk the bilinear forms' gradients and the output rows
//      (assemble_kernel).
// Tokens past a sequence's end are zero-padded with alpha = 1 and beta = 0, which leaves every real row exact.
#include <cublas_v2.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int CC = 64;    // tokens per chunk
constexpr int D = 128;    // K = V
constexpr float LOG2E_F = 1.4426950408889634f;
constexpr float FLOOR2 = -126.f;  // per-token log2-decay floor (alpha = 0 included), as in the forward

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Bufs {
  float *Qf, *Kf, *Vf, *dOf, *G2, *QG, *KG, *KT, *gam, *bet;  // [NB][64][128] (KT [NB][128][64], gam [NB][128],
                                                              // bet [NB][64])
  float *Mq, *Mk, *Tm, *TB;                                   // [NB][64][64]
  float *W, *U, *dU, *dQG, *dKT, *dW, *dKG, *dV;              // [NB][64][128]
  float *S0, *dSC;                                            // [NB][128][128]
  float *dMq, *dTB, *X, *dA;                                  // [NB][64][64]
  float* dgC;                                                 // [NB][128]
};

struct BwdC {
  const void* q;
  const void* k;
  const void* v;
  const float* gate;
  const float* beta;
  const float* d_o;
  const float* d_sf;
  float *dq, *dk, *dv, *dgate, *dbeta, *ds0;
  int64_t qs[3], ks[3], vs[3], gs[3], bs[3];
  const int* cu;  // packed sequences (B = 1), or null
  int64_t T;
  int B, H, N, ncps;  // N sequences; ncps chunks per batch row without cu
  int gate_log;
};

// The clamped token range [c0, c1) of packed sequence s.
__device__ __forceinline__ void seq_tokens(const BwdC& a, int s, int64_t& c0, int64_t& c1) {
  c1 = min((int64_t)a.cu[s + 1], a.T);
  c0 = max((int64_t)0, min((int64_t)a.cu[s], c1));
}

// Chunk-head b -> batch row n (the row of the token tensors), chunk j of its sequence, head h, first token t0
// within the row and its number of real tokens nv. The chunks are in the forward split kernels' workspace
// order, b = slot * H + h: without cu_seqlens slot = n * ceil(T / 64) + j; with them, chunk j of sequence s
// sits at slot floor(c0 / 64) + s + j, and a slot between two sequences' runs has no tokens (nv = 0).
// PACKED (cu_seqlens given) is a template argument, so that the dense kernels carry no trace of the search.
template <bool PACKED>
__device__ __forceinline__ void chunk_of(const BwdC& a, int b, int& n, int& j, int& h, int& t0, int& nv) {
  h = b % a.H;
  if constexpr (!PACKED) {
    j = (b / a.H) % a.ncps;
    n = b / (a.H * a.ncps);
    t0 = j * CC;
    nv = (int)min((int64_t)CC, a.T - t0);
    return;
  }
  const int slot = b / a.H;
  n = 0;
  j = 0;
  t0 = 0;
  nv = 0;
  int lo = 0, hi = a.N - 1, sq = -1;  // the last sequence whose first slot is <= slot
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    int64_t c0, c1;
    seq_tokens(a, mid, c0, c1);
    if ((c0 >> 6) + mid <= slot) {
      sq = mid;
      lo = mid + 1;
    } else {
      hi = mid - 1;
    }
  }
  if (sq < 0) return;
  int64_t c0, c1;
  seq_tokens(a, sq, c0, c1);
  const int64_t jj = slot - ((c0 >> 6) + sq);
  if (jj * CC >= c1 - c0) return;
  j = (int)jj;
  t0 = (int)(c0 + jj * CC);
  nv = (int)min((int64_t)CC, c1 - t0);
}

__device__ __forceinline__ void unpack4(const float4 v, float o[4]) {
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}

// fp32 copies of the chunk's q, k, v, dO (zero past the end), the log2 cumulative decay (per-token floor at
// -126, zero past the end: alpha = 1), Q*Gamma, K*Gamma, K*gamma_C/Gamma (transposed, [c][t]), gamma_C and beta
// (zero past the end).
// Threads 0-127 walk the tokens for channel c (the cumulative sum), threads 128-255 copy v and dO; each takes
// 8 tokens' loads ahead of their stores.
template <bool PACKED>
__global__ void __launch_bounds__(256) prep_kernel(BwdC a, Bufs w) {
  const int b = blockIdx.x, tid = threadIdx.x;
  int n, j, h, t0, nv;
  chunk_of<PACKED>(a, b, n, j, h, t0, nv);
  const size_t mat = (size_t)b * CC * D;
  if (tid < D) {
    const int c = tid;
    float run = 0.f;
    for (int t8 = 0; t8 < CC; t8 += 8) {
      float x[8], qv[8], kv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t tt = t0 + t8 + u;
        const bool in = t8 + u < nv;
        x[u] = in ? a.gate[n * a.gs[0] + tt * a.gs[1] + h * a.gs[2] + c] : 0.f;
        qv[u] = in ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[n * a.qs[0] + tt * a.qs[1] + h * a.qs[2] + c]) : 0.f;
        kv[u] = in ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.k)[n * a.ks[0] + tt * a.ks[1] + h * a.ks[2] + c]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const size_t e = mat + (t8 + u) * D + c;
        run += t8 + u < nv ? fmaxf(a.gate_log ? x[u] * LOG2E_F : log2f(x[u]), FLOOR2) : 0.f;
        const float gm = ex2f(run);
        w.G2[e] = run;
        w.Qf[e] = qv[u];
        w.Kf[e] = kv[u];
        w.QG[e] = qv[u] * gm;
        w.KG[e] = kv[u] * gm;
      }
    }
    w.gam[(size_t)b * D + c] = ex2f(run);
    for (int t8 = 0; t8 < CC; t8 += 8) {  // KT transposed: [c][t]
      float kf[8], g2[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        kf[u] = w.Kf[mat + (t8 + u) * D + c];
        g2[u] = w.G2[mat + (t8 + u) * D + c];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) kf[u] *= ex2f(run - g2[u]);
      *reinterpret_cast<float4*>(w.KT + mat + c * CC + t8) = make_float4(kf[0], kf[1], kf[2], kf[3]);
      *reinterpret_cast<float4*>(w.KT + mat + c * CC + t8 + 4) = make_float4(kf[4], kf[5], kf[6], kf[7]);
    }
  } else {
    const int c = tid - D;
    for (int t8 = 0; t8 < CC; t8 += 8) {
      float vv[8], dov[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t tt = t0 + t8 + u;
        const bool in = t8 + u < nv;
        vv[u] = in ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.v)[n * a.vs[0] + tt * a.vs[1] + h * a.vs[2] + c]) : 0.f;
        dov[u] = in ? a.d_o[((n * a.T + tt) * a.H + h) * D + c] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        w.Vf[mat + (t8 + u) * D + c] = vv[u];
        w.dOf[mat + (t8 + u) * D + c] = dov[u];
      }
    }
  }
  if (tid < CC) {
    const int64_t tt = t0 + tid;
    w.bet[(size_t)b * CC + tid] = tid < nv ? a.beta[n * a.bs[0] + tt * a.bs[1] + h * a.bs[2]] : 0.f;
  }
}

// Packed sequences: the start state of a slot without tokens (between two sequences' runs), which the forward
// never writes, is zeroed so that every product stays finite there.
__global__ void __launch_bounds__(256) zero_empty_slots_kernel(BwdC a, Bufs w) {
  const int b = blockIdx.x;
  int n, j, h, t0, nv;
  chunk_of<true>(a, b, n, j, h, t0, nv);
  if (nv != 0) return;
  for (int e = threadIdx.x; e < D * D / 4; e += 256)
    reinterpret_cast<float4*>(w.S0 + (size_t)b * D * D)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Mq and Mk of one chunk, split over two CTAs by row quad (rows 4q .. 4q + 3; CTA `half` takes the quads of
// its parity). A warp takes one quad and 32 columns i at a time (a lane per i), channels 4 at a time. For the
// columns before the quad (i < 4q <= t) the decay ratio factors at the reference r = 4q - 1:
// 2^{G_t - G_i} = 2^{G_t - G_r} 2^{G_r - G_i}, both factors <= 1 (a factor that flushes to zero bounds the
// exact ratio, which is then below 2^-126 as well); q_t and k_t come pre-scaled by the first factor (QA, KA),
// so a pair costs two FMAs and a lane one exponential per channel. The 4x4 blocks on the diagonal form every
// ratio directly. Rows of k and G are padded to 132 floats (lane-indexed float4 loads hit distinct banks).
// About 100 KB of shared memory: two CTAs per SM.
constexpr int PAIR_SMEM = (2 * CC * 132 + 2 * (CC / 2) * D) * 4;
__global__ void __launch_bounds__(256, 2) pair_kernel(Bufs w) {
  constexpr int PR = 132;
  extern __shared__ __align__(16) float sp[];
  float* Ks = sp;              // [64][132]
  float* Gs = Ks + CC * PR;    // [64][132]
  float* QA = Gs + CC * PR;    // [32][128], the CTA's quads in order: q_t, then q_t 2^{G_t - G_r(t)}
  float* KA = QA + CC / 2 * D; // [32][128]: k_t 2^{G_t - G_r(t)}
  const int b = blockIdx.x >> 1, half = blockIdx.x & 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t mat = (size_t)b * CC * D, sq = (size_t)b * CC * CC;
  auto row_of = [&](int lr) { return 4 * (2 * (lr >> 2) + half) + (lr & 3); };  // local row -> token row
  {
    float4 kv[8], gv[8], qv[4];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      kv[m] = reinterpret_cast<const float4*>(w.Kf + mat)[tid + 256 * m];
      gv[m] = reinterpret_cast<const float4*>(w.G2 + mat)[tid + 256 * m];
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int e = tid + 256 * m, lr = e >> 5, c4 = e & 31;
      qv[m] = reinterpret_cast<const float4*>(w.Qf + mat + (size_t)row_of(lr) * D)[c4];
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int e = tid + 256 * m, t = e >> 5, c = 4 * (e & 31);
      *reinterpret_cast<float4*>(Ks + t * PR + c) = kv[m];
      *reinterpret_cast<float4*>(Gs + t * PR + c) = gv[m];
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int e = tid + 256 * m;
      reinterpret_cast<float4*>(QA)[e] = qv[m];
    }
  }
  __syncthreads();
  // the 4x4 diagonal blocks of the CTA's quads: warps 0-3, two quads a warp, a lane one pair (t, i)
  if (warp < 4) {
    const int qi = 2 * warp + (lane >> 4), r = (lane >> 2) & 3, ii = lane & 3;
    const int q = 2 * qi + half, t = 4 * q + r, i = 4 * q + ii;
    const float* qrow = QA + (4 * qi + r) * D;
    float mq = 0.f, mk = 0.f;
    if (ii <= r) {
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(qrow + c);
        const float4 kt = *reinterpret_cast<const float4*>(Ks + t * PR + c);
        const float4 gt = *reinterpret_cast<const float4*>(Gs + t * PR + c);
        const float4 kv = *reinterpret_cast<const float4*>(Ks + i * PR + c);
        const float4 gv = *reinterpret_cast<const float4*>(Gs + i * PR + c);
        float x = ex2f(gt.x - gv.x) * kv.x;
        mq = fmaf(qv.x, x, mq); mk = fmaf(kt.x, x, mk);
        x = ex2f(gt.y - gv.y) * kv.y;
        mq = fmaf(qv.y, x, mq); mk = fmaf(kt.y, x, mk);
        x = ex2f(gt.z - gv.z) * kv.z;
        mq = fmaf(qv.z, x, mq); mk = fmaf(kt.z, x, mk);
        x = ex2f(gt.w - gv.w) * kv.w;
        mq = fmaf(qv.w, x, mq); mk = fmaf(kt.w, x, mk);
      }
    }
    w.Mq[sq + t * CC + i] = ii <= r ? mq : 0.f;
    w.Mk[sq + t * CC + i] = ii < r ? mk : 0.f;
  }
  __syncthreads();  // raw q read; scale in place
#pragma unroll 2
  for (int e = tid; e < CC / 2 * D / 4; e += 256) {
    const int lr = e >> 5, c = 4 * (e & 31), t = row_of(lr);
    float4 qa = make_float4(0.f, 0.f, 0.f, 0.f), ka = qa;
    if (t >= 4) {
      const int r = (t & ~3) - 1;
      const float4 g = *reinterpret_cast<const float4*>(Gs + t * PR + c);
      const float4 gr = *reinterpret_cast<const float4*>(Gs + r * PR + c);
      const float4 qv = *reinterpret_cast<const float4*>(QA + lr * D + c);
      const float4 kv = *reinterpret_cast<const float4*>(Ks + t * PR + c);
      const float ax = ex2f(g.x - gr.x), ay = ex2f(g.y - gr.y), az = ex2f(g.z - gr.z), aw = ex2f(g.w - gr.w);
      qa = make_float4(qv.x * ax, qv.y * ay, qv.z * az, qv.w * aw);
      ka = make_float4(kv.x * ax, kv.y * ay, kv.z * az, kv.w * aw);
    }
    *reinterpret_cast<float4*>(QA + lr * D + c) = qa;
    *reinterpret_cast<float4*>(KA + lr * D + c) = ka;
  }
  __syncthreads();
  // warp w: quad q = 2w + half, columns 32 hf .. 32 hf + 31 for hf = 0, 1
  const int q = 2 * warp + half, tq = 4 * q;
  const float* qa_ = QA + 4 * warp * D;
  const float* ka_ = KA + 4 * warp * D;
#pragma unroll 1
  for (int hf = 0; hf < 2; ++hf) {
    const int i = 32 * hf + lane;
    float mq[4] = {0.f, 0.f, 0.f, 0.f}, mk[4] = {0.f, 0.f, 0.f, 0.f};
    if (32 * hf < tq) {  // some column before the quad
      const float* ki_ = Ks + i * PR;
      const float* gi_ = Gs + i * PR;
      const float* gr_ = Gs + (tq - 1) * PR;
#pragma unroll 2
      for (int c = 0; c < D; c += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(ki_ + c);
        const float4 gv = *reinterpret_cast<const float4*>(gi_ + c);
        const float4 gr = *reinterpret_cast<const float4*>(gr_ + c);
        const float kb0 = kv.x * ex2f(gr.x - gv.x), kb1 = kv.y * ex2f(gr.y - gv.y);
        const float kb2 = kv.z * ex2f(gr.z - gv.z), kb3 = kv.w * ex2f(gr.w - gv.w);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 qa = *reinterpret_cast<const float4*>(qa_ + r * D + c);
          const float4 ka = *reinterpret_cast<const float4*>(ka_ + r * D + c);
          mq[r] = fmaf(qa.x, kb0, fmaf(qa.y, kb1, fmaf(qa.z, kb2, fmaf(qa.w, kb3, mq[r]))));
          mk[r] = fmaf(ka.x, kb0, fmaf(ka.y, kb1, fmaf(ka.z, kb2, fmaf(ka.w, kb3, mk[r]))));
        }
      }
    }
    if (i < tq || i > tq + 3) {  // the quad's own columns are the diagonal pass's
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int t = tq + r;
        w.Mq[sq + t * CC + i] = i < tq ? mq[r] : 0.f;
        w.Mk[sq + t * CC + i] = i < tq ? mk[r] : 0.f;
      }
    }
  }
}

// T = (I + Diag(beta) Mk)^-1 (unit lower triangular) by forward substitution, one thread per column j, and
// TB = T Diag(beta).
__global__ void __launch_bounds__(64) inverse_kernel(Bufs w) {
  __shared__ float A[CC][CC + 1];
  const int b = blockIdx.x, j = threadIdx.x;
  const size_t sq = (size_t)b * CC * CC;
  for (int e = j; e < CC * CC; e += CC) {
    const int t = e / CC, i = e % CC;
    A[t][i] = w.bet[(size_t)b * CC + t] * w.Mk[sq + e];
  }
  __syncthreads();
  float x[CC];
#pragma unroll
  for (int i = 0; i < CC; ++i) {
    float s = 0.f;
#pragma unroll
    for (int l = 0; l < i; ++l) s = fmaf(A[i][l], x[l], s);  // x[l] = 0 for l < j
    x[i] = i < j ? 0.f : (i == j ? 1.f : -s);
  }
  const float bj = w.bet[(size_t)b * CC + j];
#pragma unroll
  for (int i = 0; i < CC; ++i) {
    w.Tm[sq + i * CC + j] = x[i];
    w.TB[sq + i * CC + j] = x[i] * bj;
  }
}

// 16-byte asynchronous global -> shared copies (the operand prefetch of the dS recurrence).
__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The reverse recurrence for dS over the chunks of one (batch row, head), value columns [32 s, 32 s + 32).
// The dO terms are independent of the recurrence and come in precomputed: X1 = Mq^T dO in dU and
// Y = QG^T dO - W^T X1 in dS_C's place. Per chunk, from the last:
//   dS_C = dS;  dU = X1 + KT dS;  dS <- Diag(gamma_C) dS + Y - W^T (KT dS),
// with dS_C and dU written over Y and X1 and dS0 of the first chunk to ds0. A thread holds a 4x4 block of dS;
// KT dS is split over the channel index between the two halves of the CTA (4x4 blocks each), so that every
// 16 FMAs take two 16-byte shared loads. Every operand of the next chunk (KT^T, W, the slices of Y and X1,
// gamma_C) is prefetched with cp.async into the other half of a double buffer.
constexpr int VS = 32;
constexpr int DS_KT = 0, DS_W = D * CC, DS_Y = 2 * D * CC, DS_X1 = DS_Y + D * VS, DS_G = DS_X1 + CC * VS;
constexpr int DS_OPS = DS_G + D;  // one chunk's operands
constexpr int DSTATE_SMEM = (2 * DS_OPS + D * VS + 2 * CC * VS) * 4;

__device__ __forceinline__ void dstate_prefetch(const Bufs& w, int b, int vsl, float* dst, int tid) {
  const size_t mat = (size_t)b * CC * D, st = (size_t)b * D * D;
  const float* kt = w.KT + mat;  // [128][64]
  const float* wm = w.W + mat;   // [64][128]
#pragma unroll
  for (int e = tid; e < CC * D / 4; e += 256) {
    cp_async16(dst + DS_KT + 4 * e, kt + 4 * e);
    cp_async16(dst + DS_W + 4 * e, wm + 4 * e);
  }
#pragma unroll
  for (int e = tid; e < D * VS / 4; e += 256) {  // Y[c][32 s ..]
    const int c = e >> 3, q = e & 7;
    cp_async16(dst + DS_Y + 4 * e, w.dSC + st + (size_t)c * D + vsl * VS + 4 * q);
  }
#pragma unroll
  for (int e = tid; e < CC * VS / 4; e += 256) {  // X1[i][32 s ..]
    const int i = e >> 3, q = e & 7;
    cp_async16(dst + DS_X1 + 4 * e, w.dU + mat + (size_t)i * D + vsl * VS + 4 * q);
  }
  if (tid < D / 4) cp_async16(dst + DS_G + 4 * tid, w.gam + (size_t)b * D + 4 * tid);
  cp_async_commit();
}


__global__ void __launch_bounds__(256, 1) dstate_kernel(BwdC a, Bufs w) {
  extern __shared__ __align__(16) float sd[];
  float* dSs = sd + 2 * DS_OPS;   // [128][VS]
  float* dUa = dSs + D * VS;      // [64][VS]: KT dS (channels 0-63, then the sum)
  float* dUb = dUa + CC * VS;     // [64][VS]: KT dS (channels 64-127)
  const int tid = threadIdx.x;
  const int nh = blockIdx.x, vsl = blockIdx.y;
  const int n = nh / a.H, h = nh % a.H;  // sequence, head
  int base, nch;                          // the sequence's first slot and its number of chunks
  if (a.cu) {
    int64_t s0, s1;
    seq_tokens(a, n, s0, s1);
    base = (int)((s0 >> 6) + n);
    nch = (int)((s1 - s0 + CC - 1) / CC);
  } else {
    base = n * a.ncps;
    nch = a.ncps;
  }
  const int c0 = 4 * (tid >> 3), v0 = 4 * (tid & 7);   // this thread's dS[c0 .. c0 + 3][v0 .. v0 + 3] of the slice
  const int half = tid >> 7, i0 = 4 * ((tid & 127) >> 3);  // KT dS: rows i0 .. i0 + 3, channels of this half
  const int vg = vsl * VS + v0;
  float dS[4][4];
  const size_t shead = ((size_t)n * a.H + h) * D * D;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float4 x = a.d_sf ? *reinterpret_cast<const float4*>(a.d_sf + shead + (size_t)(c0 + r) * D + vg)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    unpack4(x, dS[r]);
  }
  if (nch > 0) dstate_prefetch(w, (base + nch - 1) * a.H + h, vsl, sd + ((nch - 1) & 1) * DS_OPS, tid);
  for (int j = nch - 1; j >= 0; --j) {
    const int b = (base + j) * a.H + h;
    const size_t mat = (size_t)b * CC * D, st = (size_t)b * D * D;
    const float* buf = sd + (j & 1) * DS_OPS;
#pragma unroll
    for (int r = 0; r < 4; ++r)
      *reinterpret_cast<float4*>(dSs + (c0 + r) * VS + v0) = make_float4(dS[r][0], dS[r][1], dS[r][2], dS[r][3]);
    if (j > 0) {
      dstate_prefetch(w, b - a.H, vsl, sd + ((j - 1) & 1) * DS_OPS, tid);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // this chunk's operands have landed (Y and X1 among them: their places may be written)
#pragma unroll
    for (int r = 0; r < 4; ++r)
      *reinterpret_cast<float4*>(w.dSC + st + (size_t)(c0 + r) * D + vg) =
          make_float4(dS[r][0], dS[r][1], dS[r][2], dS[r][3]);
    {  // KT dS over this half's 64 channels
      const float* KTs = buf + DS_KT;
      float acc[4][4] = {};
#pragma unroll 8
      for (int cc = 64 * half; cc < 64 * half + 64; ++cc) {
        float kv[4], sv[4];
        unpack4(*reinterpret_cast<const float4*>(KTs + cc * CC + i0), kv);
        unpack4(*reinterpret_cast<const float4*>(dSs + cc * VS + v0), sv);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[r][u] = fmaf(kv[r], sv[u], acc[r][u]);
      }
      float* dst = half ? dUb : dUa;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        *reinterpret_cast<float4*>(dst + (i0 + r) * VS + v0) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    }
    __syncthreads();
#pragma unroll
    for (int q = tid; q < CC * VS / 4; q += 256) {  // the two halves summed; dU = X1 + KT dS
      const int i = q >> 3, v = 4 * (q & 7);
      const float4 x = *reinterpret_cast<const float4*>(dUa + i * VS + v);
      const float4 y = *reinterpret_cast<const float4*>(dUb + i * VS + v);
      const float4 z = make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w);
      *reinterpret_cast<float4*>(dUa + i * VS + v) = z;
      const float4 x1 = *reinterpret_cast<const float4*>(buf + DS_X1 + i * VS + v);
      *reinterpret_cast<float4*>(w.dU + mat + (size_t)i * D + vsl * VS + v) =
          make_float4(x1.x + z.x, x1.y + z.y, x1.z + z.z, x1.w + z.w);
    }
    __syncthreads();
    {  // dS <- gamma_C[c] dS[c][v] + Y[c][v] - sum_t W[t][c] (KT dS)[t][v]
      const float* Ws = buf + DS_W;
      float g[4];
      unpack4(*reinterpret_cast<const float4*>(buf + DS_G + c0), g);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float y[4];
        unpack4(*reinterpret_cast<const float4*>(buf + DS_Y + (c0 + r) * VS + v0), y);
#pragma unroll
        for (int u = 0; u < 4; ++u) dS[r][u] = fmaf(g[r], dS[r][u], y[u]);
      }
#pragma unroll 8
      for (int t = 0; t < CC; ++t) {
        float wv[4], ev[4];
        unpack4(*reinterpret_cast<const float4*>(Ws + t * D + c0), wv);
        unpack4(*reinterpret_cast<const float4*>(dUa + t * VS + v0), ev);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int u = 0; u < 4; ++u) dS[r][u] = fmaf(-wv[r], ev[u], dS[r][u]);
      }
    }
    __syncthreads();  // the buffer just read is the next prefetch's target
  }
  if (a.ds0) {
#pragma unroll
    for (int r = 0; r < 4; ++r)
      *reinterpret_cast<float4*>(a.ds0 + shead + (size_t)(c0 + r) * D + vg) =
          make_float4(dS[r][0], dS[r][1], dS[r][2], dS[r][3]);
  }
}

// dMq = tril(dMq) (diagonal kept); dgamma_C[c] = sum_v dS_C[c][v] S0[c][v] (a warp per row c); dv of the chunk's
// real rows (dV = TB^T dU, 8 loads ahead of their stores).
template <bool PACKED>
__global__ void __launch_bounds__(256) mask_dgc_kernel(BwdC a, Bufs w) {
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int n, j, h, t0, nv;
  chunk_of<PACKED>(a, b, n, j, h, t0, nv);
  const size_t sq = (size_t)b * CC * CC, st = (size_t)b * D * D, mat = (size_t)b * CC * D;
  float4 v[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) v[u] = reinterpret_cast<const float4*>(w.dV + mat)[tid + 256 * u];
  for (int e = tid; e < CC * CC; e += 256)
    if (e % CC > e / CC) w.dMq[sq + e] = 0.f;
  for (int c = warp; c < D; c += 8) {
    const float4 x = *reinterpret_cast<const float4*>(w.dSC + st + (size_t)c * D + 4 * lane);
    const float4 y = *reinterpret_cast<const float4*>(w.S0 + st + (size_t)c * D + 4 * lane);
    float s = x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    if (lane == 0) w.dgC[(size_t)b * D + c] = s;
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int pc = tid + 256 * u, t = pc >> 5, c4 = pc & 31;
    if (t < nv) *reinterpret_cast<float4*>(a.dv + ((n * a.T + t0 + t) * a.H + h) * D + 4 * c4) = v[u];
  }
}

// dT = dTB Diag(beta) in place (the X = T^T dT product follows), after dbeta's first term colsum(dTB * T)
// into dbeta_part.
__global__ void __launch_bounds__(64) dt_kernel(Bufs w, float* dbeta_part) {
  const int b = blockIdx.x, j = threadIdx.x;
  const size_t sq = (size_t)b * CC * CC;
  float s = 0.f;
  const float bj = w.bet[(size_t)b * CC + j];
  for (int t = 0; t < CC; ++t) {
    const float d = w.dTB[sq + t * CC + j];
    s = fmaf(d, w.Tm[sq + t * CC + j], s);
    w.X[sq + t * CC + j] = d * bj;  // dT, the next product's input
  }
  dbeta_part[(size_t)b * CC + j] = s;
}

// dA = strict_tril(dA) in place; dbeta = colsum(dTB * T) + rowsum(dA * Mk) written for the chunk's real rows;
// dMk = Diag(beta) dA (into dA). A warp per row t (lanes over i).
template <bool PACKED>
__global__ void __launch_bounds__(256) da_kernel(BwdC a, Bufs w, const float* dbeta_part) {
  const int b = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int n, j, h, t0, nv;
  chunk_of<PACKED>(a, b, n, j, h, t0, nv);
  const size_t sq = (size_t)b * CC * CC;
  for (int t = warp; t < CC; t += 8) {
    const float bt = w.bet[(size_t)b * CC + t];
    float s = 0.f;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = lane + 32 * hh;
      const float d = i < t ? w.dA[sq + t * CC + i] : 0.f;
      s = fmaf(d, w.Mk[sq + t * CC + i], s);
      w.dA[sq + t * CC + i] = d * bt;
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    if (lane == 0 && t < nv) a.dbeta[(n * a.T + t0 + t) * a.H + h] = dbeta_part[(size_t)b * CC + t] + s;
  }
}

// Per chunk: the gradients of the bilinear forms Mq, Mk, then dq, dk and dG -> dlog(alpha) (reverse cumulative
// sum) for the chunk's real rows.
// For channel c and the pairs (t, i <= t) with R = 2^{G2_tc - G2_ic}:
//   row forms (by t):    rq[t] = sum_i dMq[t][i] k_ic R,  rk[t] = sum_i dMk[t][i] k_ic R
//   column form (by i):  cs[i] = sum_t (dMq[t][i] q_tc + dMk[t][i] k_tc) R
// Threads 0-127 (one per channel) take the row forms, threads 128-255 the column form, each over 8x8 tiles of
// pairs with the tile's operands in registers; the row shares of dk and dG wait in shared memory for the column
// form. The per-channel columns of G, K and Q sit transposed in shared memory ([c][t], 16-byte groups
// XOR-swizzled by c so that a quarter warp's float4 loads hit distinct banks).
constexpr int ASM_T = D * CC;                             // one transposed [128][64] tile
constexpr int ASSEMBLE_SMEM = (3 * ASM_T + 2 * CC * CC + 3 * CC * D) * 4;

__device__ __forceinline__ int swz(int c, int t) { return c * CC + ((((t >> 2) ^ (c & 7))) << 2) + (t & 3); }
__device__ __forceinline__ void ld8(const float* X, int c, int t0, float v[8]) {
  const float4 x = *reinterpret_cast<const float4*>(X + swz(c, t0));
  const float4 y = *reinterpret_cast<const float4*>(X + swz(c, t0 + 4));
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w; v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}
__device__ __forceinline__ void ld8r(const float* row, float v[8]) {  // 8 consecutive floats (warp-uniform)
  const float4 x = *reinterpret_cast<const float4*>(row);
  const float4 y = *reinterpret_cast<const float4*>(row + 4);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w; v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}

// Tiles below the diagonal (I < T) put every row t after every column i, so with the reference G_ref = G2 at
// the block's last column, 2^{G_t - G_i} = 2^{G_t - G_ref} 2^{G_ref - G_i} with both factors <= 1 (a factor
// that flushes to zero bounds the exact ratio, which is then below 2^-126 as well): 16 exponentials per tile and
// channel instead of 64. The diagonal tiles form every ratio directly.

// Row forms of tile (rows 8T.., columns 8I..), I < T.
__device__ __forceinline__ void row_tile_off(const float* Gt_, const float* Kt_, const float* dMq, const float* dMk,
                                             int c, int T, int I, const float gt[8], float rq[8], float rk[8]) {
  float gi[8], kb[8];
  ld8(Gt_, c, 8 * I, gi);
  ld8(Kt_, c, 8 * I, kb);
  const float gref = gi[7];
#pragma unroll
  for (int ii = 0; ii < 8; ++ii) kb[ii] *= ex2f(gref - gi[ii]);
#pragma unroll
  for (int tt = 0; tt < 8; ++tt) {
    float mq[8], mk[8];
    ld8r(dMq + (8 * T + tt) * CC + 8 * I, mq);
    ld8r(dMk + (8 * T + tt) * CC + 8 * I, mk);
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) {
      sq = fmaf(mq[ii], kb[ii], sq);
      sk = fmaf(mk[ii], kb[ii], sk);
    }
    const float at = ex2f(gt[tt] - gref);
    rq[tt] = fmaf(at, sq, rq[tt]);
    rk[tt] = fmaf(at, sk, rk[tt]);
  }
}

// Row forms of the diagonal tile T.
__device__ __forceinline__ void row_tile_diag(const float* Gt_, const float* Kt_, const float* dMq, const float* dMk,
                                              int c, int T, const float gt[8], float rq[8], float rk[8]) {
  float ki[8];
  ld8(Kt_, c, 8 * T, ki);
#pragma unroll
  for (int tt = 0; tt < 8; ++tt) {
    float mq[8], mk[8];
    ld8r(dMq + (8 * T + tt) * CC + 8 * T, mq);
    ld8r(dMk + (8 * T + tt) * CC + 8 * T, mk);
#pragma unroll
    for (int ii = 0; ii <= tt; ++ii) {
      const float x = ex2f(gt[tt] - gt[ii]) * ki[ii];
      rq[tt] = fmaf(mq[ii], x, rq[tt]);
      rk[tt] = fmaf(mk[ii], x, rk[tt]);
    }
  }
}

// Column form of tile (rows 8T.., columns 8I..), I < T, without the column factor 2^{G_ref - G_i}.
__device__ __forceinline__ void col_tile_off(const float* Gt_, const float* Kt_, const float* Qt_, const float* dMq,
                                             const float* dMk, int c, int T, int I, float gref, float cs[8]) {
  float gt[8], aq[8], ak[8];
  ld8(Gt_, c, 8 * T, gt);
  ld8(Qt_, c, 8 * T, aq);
  ld8(Kt_, c, 8 * T, ak);
#pragma unroll
  for (int tt = 0; tt < 8; ++tt) {
    const float e = ex2f(gt[tt] - gref);
    aq[tt] *= e;
    ak[tt] *= e;
  }
#pragma unroll
  for (int tt = 0; tt < 8; ++tt) {
    float mq[8], mk[8];
    ld8r(dMq + (8 * T + tt) * CC + 8 * I, mq);
    ld8r(dMk + (8 * T + tt) * CC + 8 * I, mk);
#pragma unroll
    for (int ii = 0; ii < 8; ++ii) cs[ii] = fmaf(mq[ii], aq[tt], fmaf(mk[ii], ak[tt], cs[ii]));
  }
}

// Column form of the diagonal tile I.
__device__ __forceinline__ void col_tile_diag(const float* Kt_, const float* Qt_, const float* dMq, const float* dMk,
                                              int c, int I, const float gi[8], float cs[8]) {
  float qt[8], kt[8];
  ld8(Qt_, c, 8 * I, qt);
  ld8(Kt_, c, 8 * I, kt);
#pragma unroll
  for (int tt = 0; tt < 8; ++tt) {
    float mq[8], mk[8];
    ld8r(dMq + (8 * I + tt) * CC + 8 * I, mq);
    ld8r(dMk + (8 * I + tt) * CC + 8 * I, mk);
#pragma unroll
    for (int ii = 0; ii <= tt; ++ii) {
      const float wv = fmaf(mq[ii], qt[tt], mk[ii] * kt[tt]);
      cs[ii] = fmaf(ex2f(gi[tt] - gi[ii]), wv, cs[ii]);
    }
  }
}

template <bool PACKED>
__global__ void __launch_bounds__(256, 1) assemble_kernel(BwdC a, Bufs w) {
  extern __shared__ __align__(16) float sa[];
  float* Gt_ = sa;                  // [128][64] swizzled: G2 by channel
  float* Kt_ = Gt_ + ASM_T;         // [128][64] swizzled: k
  float* Qt_ = Kt_ + ASM_T;         // [128][64] swizzled: q
  float* dMq = Qt_ + ASM_T;         // [64][64]
  float* dMk = dMq + CC * CC;       // [64][64] (Diag(beta) dA)
  float* Cs = dMk + CC * CC;        // [64][128]: the column form
  float* DKr = Cs + CC * D;         // [64][128]: dk's row share
  float* DGr = DKr + CC * D;        // [64][128]: dG's row share
  const int b = blockIdx.x, tid = threadIdx.x;
  int n, j, h, t0, nv;
  chunk_of<PACKED>(a, b, n, j, h, t0, nv);
  const size_t mat = (size_t)b * CC * D, sq = (size_t)b * CC * CC;
  // dMq and dMk with cp.async; G2, k, q transposed through registers (a thread takes 4 consecutive tokens of
  // one channel, coalesced over the channel; every load in flight at once)
#pragma unroll
  for (int e = tid; e < CC * CC / 4; e += 256) {
    cp_async16(dMq + 4 * e, w.dMq + sq + 4 * e);
    cp_async16(dMk + 4 * e, w.dA + sq + 4 * e);
  }
  {
    float g[8][4], k[8][4], q[8][4];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int e = tid + 256 * m, c = e & 127, t4 = (e >> 7) * 4;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        g[m][u] = w.G2[mat + (t4 + u) * D + c];
        k[m][u] = w.Kf[mat + (t4 + u) * D + c];
        q[m][u] = w.Qf[mat + (t4 + u) * D + c];
      }
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int e = tid + 256 * m, c = e & 127, t4 = (e >> 7) * 4;
      *reinterpret_cast<float4*>(Gt_ + swz(c, t4)) = make_float4(g[m][0], g[m][1], g[m][2], g[m][3]);
      *reinterpret_cast<float4*>(Kt_ + swz(c, t4)) = make_float4(k[m][0], k[m][1], k[m][2], k[m][3]);
      *reinterpret_cast<float4*>(Qt_ + swz(c, t4)) = make_float4(q[m][0], q[m][1], q[m][2], q[m][3]);
    }
  }
  // dQG and dKG into the row-share buffers (each row thread reads its element, then writes its share over it)
#pragma unroll
  for (int e = tid; e < CC * D / 4; e += 256) {
    cp_async16(DGr + 4 * e, w.dQG + mat + 4 * e);
    cp_async16(DKr + 4 * e, w.dKG + mat + 4 * e);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  float dkt_kt = 0.f;  // row threads: sum_t dKT * KT, the share of G_last
  if (tid < D) {
    const int c = tid;
    float gl[8];
    ld8(Gt_, c, CC - 8, gl);
    for (int T = 0; T < CC / 8; ++T) {
      float gt[8], rq[8], rk[8], dkt[8];
      ld8(Gt_, c, 8 * T, gt);
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // dKT of the epilogue, loaded ahead of the tiles
        dkt[u] = w.dKT[mat + (8 * T + u) * D + c];
        rq[u] = rk[u] = 0.f;
      }
      for (int I = 0; I < T; ++I) row_tile_off(Gt_, Kt_, dMq, dMk, c, T, I, gt, rq, rk);
      row_tile_diag(Gt_, Kt_, dMq, dMk, c, T, gt, rq, rk);
      float qt[8], kt[8];
      ld8(Qt_, c, 8 * T, qt);
      ld8(Kt_, c, 8 * T, kt);
#pragma unroll
      for (int tt = 0; tt < 8; ++tt) {
        const int t = 8 * T + tt;
        const float gam_t = ex2f(gt[tt]), kts = ex2f(gl[7] - gt[tt]);
        const float dqg = DGr[t * D + c], dkg = DKr[t * D + c];
        // dk's and dG's row shares, completed by the column form below
        DKr[t * D + c] = rk[tt] + dkg * gam_t + dkt[tt] * kts;
        const float ktv = kt[tt] * kts;
        DGr[t * D + c] = qt[tt] * rq[tt] + kt[tt] * rk[tt] + dqg * qt[tt] * gam_t + dkg * kt[tt] * gam_t -
                         dkt[tt] * ktv;
        dkt_kt = fmaf(dkt[tt], ktv, dkt_kt);
        if (t < nv) a.dq[((n * a.T + t0 + t) * a.H + h) * D + c] = rq[tt] + dqg * gam_t;
      }
    }
  } else {
    const int c = tid - D;
    for (int I = 0; I < CC / 8; ++I) {
      float gi[8], cs[8], cd[8];
      ld8(Gt_, c, 8 * I, gi);
#pragma unroll
      for (int u = 0; u < 8; ++u) cs[u] = cd[u] = 0.f;
      col_tile_diag(Kt_, Qt_, dMq, dMk, c, I, gi, cd);
      for (int T = I + 1; T < CC / 8; ++T) col_tile_off(Gt_, Kt_, Qt_, dMq, dMk, c, T, I, gi[7], cs);
#pragma unroll
      for (int ii = 0; ii < 8; ++ii) Cs[(8 * I + ii) * D + c] = fmaf(ex2f(gi[7] - gi[ii]), cs[ii], cd[ii]);
    }
  }
  __syncthreads();
  if (tid < D) {
    // the column form into dk and dG, then dG -> dlog(alpha) by a reverse cumulative sum
    const int c = tid;
    float acc = dkt_kt + w.dgC[(size_t)b * D + c] * w.gam[(size_t)b * D + c];  // only G_last's share
    for (int t8 = CC - 8; t8 >= 0; t8 -= 8) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        x[u] = !a.gate_log && t8 + u < nv ? a.gate[n * a.gs[0] + (t0 + t8 + u) * a.gs[1] + h * a.gs[2] + c] : 1.f;
#pragma unroll
      for (int u = 7; u >= 0; --u) {
        const int t = t8 + u;
        const float kt = Kt_[swz(c, t)], cs = Cs[t * D + c];
        acc += DGr[t * D + c] - kt * cs;  // sum_{r >= t} dG[r]
        if (t < nv) {
          const size_t o = ((n * a.T + t0 + t) * a.H + h) * D + c;
          a.dk[o] = DKr[t * D + c] + cs;
          // dL/dalpha = dL/dlog(alpha) / alpha when alpha itself is the input
          a.dgate[o] = a.gate_log ? acc : (x[u] > 0.f ? acc / x[u] : 0.f);
        }
      }
    }
  }
}

// Row-major batched GEMM C = op(A) op(B) (alpha, beta as in cuBLAS) over `nb` matrices with the given strides,
// through column-major cuBLAS (C^T = op(B)^T op(A)^T), fp32 with TF32 tensor cores.
cublasStatus_t rm_gemm(cublasHandle_t hd, bool ta, bool tb, int M, int N, int K, float alpha, const float* A, int lda,
                       long long sA, const float* B, int ldb, long long sB, float beta, float* C, int ldc, long long sC,
                       int nb) {
  return cublasGemmStridedBatchedEx(hd, tb ? CUBLAS_OP_T : CUBLAS_OP_N, ta ? CUBLAS_OP_T : CUBLAS_OP_N, N, M, K, &alpha,
                                    B, CUDA_R_32F, ldb, sB, A, CUDA_R_32F, lda, sA, &beta, C, CUDA_R_32F, ldc, sC, nb,
                                    CUBLAS_COMPUTE_32F_FAST_TF32, CUBLAS_GEMM_DEFAULT);
}

// One cuBLAS handle per device, created on first use, and a per-device lock that a call holds from setting the
// handle's stream and workspace until its last product is enqueued (host threads sharing a device take turns;
// enqueueing does not wait for the GPU).
struct DeviceBlas {
  std::mutex use;
  cublasHandle_t handle = nullptr;
};

DeviceBlas* blas_for_device() {
  static std::mutex mu;
  static DeviceBlas blas[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!blas[dev].handle && cublasCreate(&blas[dev].handle) != CUBLAS_STATUS_SUCCESS) blas[dev].handle = nullptr;
  return blas[dev].handle ? &blas[dev] : nullptr;
}

constexpr size_t CUBLAS_WS = 32u << 20;  // handed to cuBLAS, so that its products allocate nothing per call
constexpr int NBUF = 33;

struct Layout {
  size_t off[NBUF];
  size_t total;
};

// Carves the workspace: the forward's operand blocks, its output, then the chunk buffers (256-byte aligned).
Layout carve(int64_t B, int64_t T, int64_t H) {
  Layout L{};
  const int64_t ncps = (T + CC - 1) / CC, NB = B * ncps * H;
  const size_t m128 = (size_t)NB * CC * D * 4, m64 = (size_t)NB * CC * CC * 4, mst = (size_t)NB * D * D * 4;
  const size_t sizes[] = {split_workspace_bytes(B, T, H, B, false), (size_t)B * T * H * D * 2,
                          m128, m128, m128, m128, m128, m128, m128, m128,        // Qf Kf Vf dOf G2 QG KG KT
                          (size_t)NB * D * 4, (size_t)NB * CC * 4,               // gam bet
                          m64, m64, m64, m64,                                    // Mq Mk Tm TB
                          m128, m128, m128, m128, m128, m128, m128, m128,        // W U dU dQG dKT dW dKG dV
                          mst, mst,                                              // S0 dSC
                          m64, m64, m64, m64,                                    // dMq dTB X dA
                          (size_t)NB * D * 4, (size_t)NB * CC * 4,               // dgC dbeta_part
                          CUBLAS_WS};                                            // cuBLAS's workspace
  size_t o = 0;
  static_assert(sizeof(sizes) / sizeof(sizes[0]) == NBUF, "one size per buffer");
  for (int i = 0; i < NBUF; ++i) {
    L.off[i] = o;
    o += (sizes[i] + 255) / 256 * 256;
  }
  L.total = o;
  return L;
}

}  // namespace

size_t chunked_backward_workspace_bytes(int64_t B, int64_t T, int64_t H) { return carve(B, T, H).total; }

cudaError_t launch_chunked_backward(const ScanParams& fwd, const float* d_o, const float* d_sf, float* dq, float* dk,
                                    float* dv, float* dgate, float* dbeta, float* ds0, void* ws, cudaStream_t s,
                                    int* cublas_status) {
  *cublas_status = 0;
  const int64_t B = fwd.B, T = fwd.T, H = fwd.H;
  const int ncps = (int)((T + CC - 1) / CC);
  // packed sequences: the forward's slot count; the layout is that of one row of n_slots full chunks
  const int64_t n_slots = fwd.cu ? T / CC + fwd.N + 1 : B * ncps;
  const int NB = (int)(n_slots * H);
  const Layout L = fwd.cu ? carve(1, n_slots * CC, H) : carve(B, T, H);
  unsigned char* base = static_cast<unsigned char*>(ws);
  auto F = [&](int i) { return reinterpret_cast<float*>(base + L.off[i]); };
  Bufs w;
  w.Qf = F(2); w.Kf = F(3); w.Vf = F(4); w.dOf = F(5); w.G2 = F(6); w.QG = F(7); w.KG = F(8); w.KT = F(9);
  w.gam = F(10); w.bet = F(11);
  w.Mq = F(12); w.Mk = F(13); w.Tm = F(14); w.TB = F(15);
  w.W = F(16); w.U = F(17); w.dU = F(18); w.dQG = F(19); w.dKT = F(20); w.dW = F(21); w.dKG = F(22); w.dV = F(23);
  w.S0 = F(24); w.dSC = F(25);
  w.dMq = F(26); w.dTB = F(27); w.X = F(28); w.dA = F(29);
  w.dgC = F(30);
  float* dbeta_part = F(31);

  // 1. the forward (kernels P and S) with the state at every chunk start kept
  ScanParams p = fwd;
  p.o = base + L.off[1];
  p.os[0] = T * H * D;
  p.os[1] = H * D;
  p.os[2] = D;
  p.sf = nullptr;
  p.s_dump = w.S0;
  cudaError_t e = launch_chunk_split(p, base + L.off[0], s);
  if (e != cudaSuccess) return e;

  BwdC a;
  a.q = fwd.q; a.k = fwd.k; a.v = fwd.v; a.gate = fwd.gate; a.beta = fwd.beta;
  a.d_o = d_o; a.d_sf = d_sf;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dgate = dgate; a.dbeta = dbeta; a.ds0 = ds0;
  for (int i = 0; i < 3; ++i) {
    a.qs[i] = fwd.qs[i]; a.ks[i] = fwd.ks[i]; a.vs[i] = fwd.vs[i]; a.gs[i] = fwd.gs[i]; a.bs[i] = fwd.bs[i];
  }
  a.cu = fwd.cu;
  a.T = T; a.B = (int)B; a.H = (int)H; a.N = fwd.N; a.ncps = ncps;
  a.gate_log = fwd.gate_mode == KDA_GATE_LOG;

  // 2. per-chunk preparation, Mq and Mk, T and TB
  if (fwd.cu) {
    prep_kernel<true><<<NB, 256, 0, s>>>(a, w);
    zero_empty_slots_kernel<<<NB, 256, 0, s>>>(a, w);
  } else {
    prep_kernel<false><<<NB, 256, 0, s>>>(a, w);
  }
  const int pair_smem = PAIR_SMEM;
  {
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!(configured.load() & (1ull << dev))) {
      const int dsm = DSTATE_SMEM;
      const int asm_ = ASSEMBLE_SMEM;
      if ((e = cudaFuncSetAttribute(pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pair_smem)) != cudaSuccess ||
          (e = cudaFuncSetAttribute(dstate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dsm)) != cudaSuccess ||
          (e = cudaFuncSetAttribute(assemble_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, asm_)) !=
              cudaSuccess ||
          (e = cudaFuncSetAttribute(assemble_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, asm_)) !=
              cudaSuccess)
        return e;
      configured.fetch_or(1ull << dev);
    }
  }
  pair_kernel<<<2 * NB, 256, pair_smem, s>>>(w);
  inverse_kernel<<<NB, 64, 0, s>>>(w);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  DeviceBlas* blas = blas_for_device();
  if (!blas) {
    *cublas_status = -1;
    return cudaErrorUnknown;
  }
  std::lock_guard<std::mutex> in_use(blas->use);
  cublasHandle_t hd = blas->handle;
  if (cublasSetStream(hd, s) != CUBLAS_STATUS_SUCCESS ||
      cublasSetWorkspace(hd, base + L.off[32], CUBLAS_WS) != CUBLAS_STATUS_SUCCESS) {
    *cublas_status = -2;
    return cudaErrorUnknown;
  }
  const long long s128 = (long long)CC * D, s64 = (long long)CC * CC, sst = (long long)D * D;
  cublasStatus_t cs = CUBLAS_STATUS_SUCCESS;
  auto G = [&](bool ta, bool tb, int M, int N, int K, float al, const float* A, int lda, long long sA, const float* Bm,
               int ldb, long long sB, float be, float* C, int ldc, long long sC) {
    if (cs == CUBLAS_STATUS_SUCCESS) cs = rm_gemm(hd, ta, tb, M, N, K, al, A, lda, sA, Bm, ldb, sB, be, C, ldc, sC, NB);
  };
  // 3. W = TB KG; U = TB V - W S0
  G(false, false, CC, D, CC, 1.f, w.TB, CC, s64, w.KG, D, s128, 0.f, w.W, D, s128);
  G(false, false, CC, D, CC, 1.f, w.TB, CC, s64, w.Vf, D, s128, 0.f, w.U, D, s128);
  G(false, false, CC, D, D, -1.f, w.W, D, s128, w.S0, D, sst, 1.f, w.U, D, s128);
  if (cs != CUBLAS_STATUS_SUCCESS) {
    *cublas_status = (int)cs;
    return cudaErrorUnknown;
  }
  // 4. the dO terms of the recurrence (X1 = Mq^T dO into dU, Y = QG^T dO - W^T X1 into dS_C), then the
  //    reverse recurrence over chunks for dS (completing dU = X1 + KT dS_C)
  G(true, false, CC, D, CC, 1.f, w.Mq, CC, s64, w.dOf, D, s128, 0.f, w.dU, D, s128);
  G(true, false, D, D, CC, 1.f, w.QG, D, s128, w.dOf, D, s128, 0.f, w.dSC, D, sst);
  G(true, false, D, D, CC, -1.f, w.W, D, s128, w.dU, D, s128, 1.f, w.dSC, D, sst);
  if (cs != CUBLAS_STATUS_SUCCESS) {
    *cublas_status = (int)cs;
    return cudaErrorUnknown;
  }
  {
    dstate_kernel<<<dim3((unsigned)((int64_t)fwd.N * H), D / VS), 256, DSTATE_SMEM, s>>>(a, w);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // 5. dMq = dO U^T; dQG = dO S0^T; dKT = U dS_C^T; dW = -dU S0^T; dTB = dU V^T + dW KG^T; dV = TB^T dU;
  //    dKG = TB^T dW; X = T^T dT; dA = -X T^T
  G(false, true, CC, CC, D, 1.f, w.dOf, D, s128, w.U, D, s128, 0.f, w.dMq, CC, s64);
  G(false, true, CC, D, D, 1.f, w.dOf, D, s128, w.S0, D, sst, 0.f, w.dQG, D, s128);
  G(false, true, CC, D, D, 1.f, w.U, D, s128, w.dSC, D, sst, 0.f, w.dKT, D, s128);
  G(false, true, CC, D, D, -1.f, w.dU, D, s128, w.S0, D, sst, 0.f, w.dW, D, s128);
  G(false, true, CC, CC, D, 1.f, w.dU, D, s128, w.Vf, D, s128, 0.f, w.dTB, CC, s64);
  G(false, true, CC, CC, D, 1.f, w.dW, D, s128, w.KG, D, s128, 1.f, w.dTB, CC, s64);
  G(true, false, CC, D, CC, 1.f, w.TB, CC, s64, w.dU, D, s128, 0.f, w.dV, D, s128);
  G(true, false, CC, D, CC, 1.f, w.TB, CC, s64, w.dW, D, s128, 0.f, w.dKG, D, s128);
  if (cs != CUBLAS_STATUS_SUCCESS) {
    *cublas_status = (int)cs;
    return cudaErrorUnknown;
  }
  if (fwd.cu)
    mask_dgc_kernel<true><<<NB, 256, 0, s>>>(a, w);
  else
    mask_dgc_kernel<false><<<NB, 256, 0, s>>>(a, w);
  dt_kernel<<<NB, 64, 0, s>>>(w, dbeta_part);  // X = dT = dTB Diag(beta); dbeta_part = colsum(dTB * T)
  // dA = -(T^T dT) T^T: the product T^T dT into dA, then -dA T^T into X (two products, reusing the buffers)
  G(true, false, CC, CC, CC, 1.f, w.Tm, CC, s64, w.X, CC, s64, 0.f, w.dA, CC, s64);
  G(false, true, CC, CC, CC, -1.f, w.dA, CC, s64, w.Tm, CC, s64, 0.f, w.X, CC, s64);
  if (cs != CUBLAS_STATUS_SUCCESS) {
    *cublas_status = (int)cs;
    return cudaErrorUnknown;
  }
  std::swap(w.dA, w.X);  // dA now names the result
  if (fwd.cu) {
    da_kernel<true><<<NB, 256, 0, s>>>(a, w, dbeta_part);
    assemble_kernel<true><<<NB, 256, ASSEMBLE_SMEM, s>>>(a, w);
  } else {
    da_kernel<false><<<NB, 256, 0, s>>>(a, w, dbeta_part);
    assemble_kernel<false><<<NB, 256, ASSEMBLE_SMEM, s>>>(a, w);
  }
  return cudaGetLastError();
}

}  // namespace kda
