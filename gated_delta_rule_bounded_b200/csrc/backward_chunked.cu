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
constexpr int PAD = 129;  // padded row length of the shared-memory [64][128] tiles (no bank conflicts)
constexpr float LOG2E_F = 1.4426950408889634f;
constexpr float FLOOR2 = -126.f;  // per-token log2-decay floor (alpha = 0 included), as in the forward

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Bufs {
  float *Qf, *Kf, *Vf, *dOf, *G2, *QG, *KG, *KT, *gam, *bet;  // [NB][64][128] (gam [NB][128], bet [NB][64])
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
  int64_t T;
  int B, H, ncps;
  int gate_log;
};

__device__ __forceinline__ void chunk_of(const BwdC& a, int b, int& n, int& j, int& h, int& t0, int& nv) {
  h = b % a.H;
  j = (b / a.H) % a.ncps;
  n = b / (a.H * a.ncps);
  t0 = j * CC;
  nv = (int)min((int64_t)CC, a.T - t0);
}

// fp32 copies of the chunk's q, k, v, dO (zero past the end), the log2 cumulative decay (per-token floor at
// -126, zero past the end: alpha = 1), Q*Gamma, K*Gamma, K*gamma_C/Gamma, gamma_C and beta (zero past the end).
__global__ void __launch_bounds__(256) prep_kernel(BwdC a, Bufs w) {
  __shared__ float Gs[CC][D];
  const int b = blockIdx.x, tid = threadIdx.x;
  int n, j, h, t0, nv;
  chunk_of(a, b, n, j, h, t0, nv);
  const size_t mat = (size_t)b * CC * D;
  if (tid < D) {
    const int c = tid;
    float run = 0.f;
    for (int t = 0; t < CC; ++t) {
      const bool in = t < nv;
      const int64_t tt = t0 + t;
      float l = 0.f, qv = 0.f, kv = 0.f;
      if (in) {
        const float x = a.gate[n * a.gs[0] + tt * a.gs[1] + h * a.gs[2] + c];
        l = fmaxf(a.gate_log ? x * LOG2E_F : log2f(x), FLOOR2);
        qv = __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[n * a.qs[0] + tt * a.qs[1] + h * a.qs[2] + c]);
        kv = __bfloat162float(static_cast<const __nv_bfloat16*>(a.k)[n * a.ks[0] + tt * a.ks[1] + h * a.ks[2] + c]);
      }
      run += l;
      Gs[t][c] = run;
      const float gm = ex2f(run);
      w.G2[mat + t * D + c] = run;
      w.Qf[mat + t * D + c] = qv;
      w.Kf[mat + t * D + c] = kv;
      w.QG[mat + t * D + c] = qv * gm;
      w.KG[mat + t * D + c] = kv * gm;
    }
    w.gam[(size_t)b * D + c] = ex2f(run);
    for (int t = 0; t < CC; ++t) w.KT[mat + t * D + c] = w.Kf[mat + t * D + c] * ex2f(run - Gs[t][c]);
  } else {
    const int c = tid - D;
    for (int t = 0; t < CC; ++t) {
      const bool in = t < nv;
      const int64_t tt = t0 + t;
      float vv = 0.f, dov = 0.f;
      if (in) {
        vv = __bfloat162float(static_cast<const __nv_bfloat16*>(a.v)[n * a.vs[0] + tt * a.vs[1] + h * a.vs[2] + c]);
        dov = a.d_o[((n * a.T + tt) * a.H + h) * D + c];
      }
      w.Vf[mat + t * D + c] = vv;
      w.dOf[mat + t * D + c] = dov;
    }
  }
  if (tid < CC) {
    const int64_t tt = t0 + tid;
    w.bet[(size_t)b * CC + tid] = tid < nv ? a.beta[n * a.bs[0] + tt * a.bs[1] + h * a.bs[2]] : 0.f;
  }
}

// Mq and Mk of one chunk, every pair (t, i <= t) summed over the channels with its decay ratio
// 2^{G2_tc - G2_ic} <= 1 formed directly (no range limit). A warp takes one row t and 32 columns i.
__global__ void __launch_bounds__(256) pair_kernel(Bufs w) {
  extern __shared__ float sp[];
  float* Qs = sp;
  float* Ks = Qs + CC * PAD;
  float* Gs = Ks + CC * PAD;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t mat = (size_t)b * CC * D;
  for (int e = tid; e < CC * D; e += 256) {
    const int t = e / D, c = e % D;
    Qs[t * PAD + c] = w.Qf[mat + e];
    Ks[t * PAD + c] = w.Kf[mat + e];
    Gs[t * PAD + c] = w.G2[mat + e];
  }
  __syncthreads();
  const size_t sq = (size_t)b * CC * CC;
  for (int u = warp; u < 2 * CC; u += 8) {
    const int t = u >> 1, i = (u & 1) * 32 + lane;
    float mq = 0.f, mk = 0.f;
    if (i <= t) {
      const float* qt = Qs + t * PAD;
      const float* kt = Ks + t * PAD;
      const float* gt = Gs + t * PAD;
      const float* ki = Ks + i * PAD;
      const float* gi = Gs + i * PAD;
#pragma unroll 4
      for (int c = 0; c < D; ++c) {
        const float r = ex2f(gt[c] - gi[c]) * ki[c];
        mq = fmaf(qt[c], r, mq);
        mk = fmaf(kt[c], r, mk);
      }
    }
    w.Mq[sq + t * CC + i] = mq;
    w.Mk[sq + t * CC + i] = i < t ? mk : 0.f;
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

// The reverse recurrence for dS over the chunks of one (batch row, head), value columns [32 s, 32 s + 32):
// dS_C of every chunk to dSC, dS0 of the first to ds0. A thread holds dS[c][16 columns].
constexpr int VS = 32;
__global__ void __launch_bounds__(256, 1) dstate_kernel(BwdC a, Bufs w) {
  extern __shared__ float sd[];
  float* Mq = sd;                 // [64][65]
  float* KT = Mq + CC * (CC + 1); // [64][129]
  float* QG = KT + CC * PAD;      // [64][129]
  float* Wm = QG + CC * PAD;      // [64][129]
  float* dOs = Wm + CC * PAD;     // [64][VS]
  float* dSs = dOs + CC * VS;     // [128][VS]
  float* dUs = dSs + D * VS;      // [64][VS]
  float* gm = dUs + CC * VS;      // [128]
  const int tid = threadIdx.x;
  const int nh = blockIdx.x, vsl = blockIdx.y;
  const int n = nh / a.H, h = nh % a.H;
  const int c = tid >> 1, v0 = (tid & 1) * 16;   // this thread's dS[c][v0 .. v0 + 15] of the slice
  const int vg = vsl * VS + v0;                  // global value column of v0
  float dS[16];
  const size_t shead = ((size_t)n * a.H + h) * D * D;
#pragma unroll
  for (int u = 0; u < 16; ++u) dS[u] = a.d_sf ? a.d_sf[shead + (size_t)c * D + vg + u] : 0.f;
  for (int j = a.ncps - 1; j >= 0; --j) {
    const int b = (n * a.ncps + j) * a.H + h;
    const size_t mat = (size_t)b * CC * D, sq = (size_t)b * CC * CC, st = (size_t)b * D * D;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      w.dSC[st + (size_t)c * D + vg + u] = dS[u];
      dSs[c * VS + v0 + u] = dS[u];
    }
    for (int e = tid; e < CC * CC; e += 256) Mq[(e / CC) * (CC + 1) + e % CC] = w.Mq[sq + e];
    for (int e = tid; e < CC * D; e += 256) {
      const int t = e / D, cc = e % D;
      KT[t * PAD + cc] = w.KT[mat + e];
      QG[t * PAD + cc] = w.QG[mat + e];
      Wm[t * PAD + cc] = w.W[mat + e];
    }
    for (int e = tid; e < CC * VS; e += 256) dOs[e] = w.dOf[mat + (e / VS) * D + vsl * VS + e % VS];
    if (tid < D) gm[tid] = w.gam[(size_t)b * D + tid];
    __syncthreads();
    // dU[i][v] = sum_t Mq[t][i] dO[t][v] + sum_c KT[i][c] dS[c][v]: a thread takes row i, 8 columns
    {
      const int i = tid >> 2, vq = (tid & 3) * 8;
      float acc[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = 0.f;
      for (int t = i; t < CC; ++t) {  // Mq[t][i] = 0 for t < i
        const float m = Mq[t * (CC + 1) + i];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = fmaf(m, dOs[t * VS + vq + u], acc[u]);
      }
      for (int cc = 0; cc < D; ++cc) {
        const float kt = KT[i * PAD + cc];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = fmaf(kt, dSs[cc * VS + vq + u], acc[u]);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) dUs[i * VS + vq + u] = acc[u];
    }
    __syncthreads();
    // dS0[c][v] = gamma_C[c] dS[c][v] + sum_t QG[t][c] dO[t][v] - sum_t W[t][c] dU[t][v]
    {
      const float g = gm[c];
#pragma unroll
      for (int u = 0; u < 16; ++u) dS[u] *= g;
      for (int t = 0; t < CC; ++t) {
        const float qg = QG[t * PAD + c], wv = Wm[t * PAD + c];
#pragma unroll
        for (int u = 0; u < 16; ++u) dS[u] = fmaf(qg, dOs[t * VS + v0 + u], fmaf(-wv, dUs[t * VS + v0 + u], dS[u]));
      }
    }
    __syncthreads();
  }
  if (a.ds0) {
#pragma unroll
    for (int u = 0; u < 16; ++u) a.ds0[shead + (size_t)c * D + vg + u] = dS[u];
  }
}

// dMq = tril(dMq) (diagonal kept); dgamma_C[c] = sum_v dS_C[c][v] S0[c][v].
__global__ void __launch_bounds__(256) mask_dgc_kernel(Bufs w) {
  const int b = blockIdx.x, tid = threadIdx.x;
  const size_t sq = (size_t)b * CC * CC, st = (size_t)b * D * D;
  for (int e = tid; e < CC * CC; e += 256)
    if (e % CC > e / CC) w.dMq[sq + e] = 0.f;
  if (tid < D) {
    float s = 0.f;
    for (int v = 0; v < D; ++v) s = fmaf(w.dSC[st + (size_t)tid * D + v], w.S0[st + (size_t)tid * D + v], s);
    w.dgC[(size_t)b * D + tid] = s;
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

// dA = strict_tril(dA) in place; dbeta = colsum(dTB * T) + rowsum(dA * Mk); dMk = Diag(beta) dA (into dA).
__global__ void __launch_bounds__(64) da_kernel(Bufs w, float* dbeta_part) {
  const int b = blockIdx.x, t = threadIdx.x;
  const size_t sq = (size_t)b * CC * CC;
  float s = 0.f;
  const float bt = w.bet[(size_t)b * CC + t];
  for (int i = 0; i < CC; ++i) {
    const float d = i < t ? w.dA[sq + t * CC + i] : 0.f;
    s = fmaf(d, w.Mk[sq + t * CC + i], s);
    w.dA[sq + t * CC + i] = d * bt;
  }
  dbeta_part[(size_t)b * CC + t] += s;
}

// Per chunk: the gradients of the bilinear forms Mq, Mk (every decay ratio formed per pair and channel), then
// dq, dk, dv, dbeta and dG -> dlog(alpha) (reverse cumulative sum) for the chunk's real rows. Thread c < 128
// owns channel c: the row forms as it walks t, the column forms accumulated in shared memory by column i.
__global__ void __launch_bounds__(256, 1) assemble_kernel(BwdC a, Bufs w, const float* dbeta_part) {
  extern __shared__ float sa[];
  float* Qs = sa;                   // [64][129]
  float* Ks = Qs + CC * PAD;        // [64][129]
  float* Gs = Ks + CC * PAD;        // [64][129]
  float* dMq = Gs + CC * PAD;       // [64][65]
  float* dMk = dMq + CC * (CC + 1); // [64][65] (Diag(beta) dA)
  float* Cq = dMk + CC * (CC + 1);  // [64][129]: sum_t dMq[t][i] q_tc R
  float* Ck = Cq + CC * PAD;        // [64][129]: sum_t dMk[t][i] k_tc R
  const int b = blockIdx.x, tid = threadIdx.x;
  int n, j, h, t0, nv;
  chunk_of(a, b, n, j, h, t0, nv);
  const size_t mat = (size_t)b * CC * D, sq = (size_t)b * CC * CC;
  for (int e = tid; e < CC * D; e += 256) {
    const int t = e / D, c = e % D;
    Qs[t * PAD + c] = w.Qf[mat + e];
    Ks[t * PAD + c] = w.Kf[mat + e];
    Gs[t * PAD + c] = w.G2[mat + e];
    Cq[t * PAD + c] = 0.f;
    Ck[t * PAD + c] = 0.f;
  }
  for (int e = tid; e < CC * CC; e += 256) {
    dMq[(e / CC) * (CC + 1) + e % CC] = w.dMq[sq + e];
    dMk[(e / CC) * (CC + 1) + e % CC] = w.dA[sq + e];
  }
  __syncthreads();
  if (tid < D) {
    const int c = tid;
    const float gl = Gs[(CC - 1) * PAD + c];
    float dkt_kt = 0.f;  // sum_t dKT * KT, the share of G_last
    for (int t = 0; t < CC; ++t) {
      const float gt = Gs[t * PAD + c], qt = Qs[t * PAD + c], kt = Ks[t * PAD + c];
      float rq = 0.f, rk = 0.f;
      for (int i = 0; i <= t; ++i) {
        const float r = ex2f(gt - Gs[i * PAD + c]);  // e^{G_t - G_i} <= 1 (G is non-increasing)
        const float ki = Ks[i * PAD + c];
        const float mq = dMq[t * (CC + 1) + i], mk = dMk[t * (CC + 1) + i];
        rq = fmaf(mq * ki, r, rq);
        rk = fmaf(mk * ki, r, rk);
        Cq[i * PAD + c] = fmaf(mq * qt, r, Cq[i * PAD + c]);
        Ck[i * PAD + c] = fmaf(mk * kt, r, Ck[i * PAD + c]);
      }
      const size_t e = mat + t * D + c;
      const float gam_t = ex2f(gt), kts = ex2f(gl - gt);
      const float dqg = w.dQG[e], dkg = w.dKG[e], dkt = w.dKT[e];
      const float dq = rq + dqg * gam_t;
      // dk's row share and dG's row share, completed by the column shares below
      w.dKG[e] = rk + dkg * gam_t + dkt * kts;
      const float ktv = kt * kts;
      w.dQG[e] = qt * rq + kt * rk + dqg * qt * gam_t + dkg * kt * gam_t - dkt * ktv;
      dkt_kt = fmaf(dkt, ktv, dkt_kt);
      if (t < nv) a.dq[((n * a.T + t0 + t) * a.H + h) * D + c] = dq;
    }
    // column shares, dk, and dG -> dlog(alpha) by a reverse cumulative sum
    float acc = dkt_kt + w.dgC[(size_t)b * D + c] * w.gam[(size_t)b * D + c];  // only G_last's share
    for (int t = CC - 1; t >= 0; --t) {
      const size_t e = mat + t * D + c;
      const float kt = Ks[t * PAD + c], cq = Cq[t * PAD + c], ck = Ck[t * PAD + c];
      const float dk = w.dKG[e] + cq + ck;
      const float dg = w.dQG[e] - kt * cq - kt * ck;
      acc += dg;  // sum_{r >= t} dG[r]
      if (t < nv) {
        const size_t o = ((n * a.T + t0 + t) * a.H + h) * D + c;
        a.dk[o] = dk;
        float dl = acc;
        if (!a.gate_log) {  // dL/dalpha = dL/dlog(alpha) / alpha
          const float x = a.gate[n * a.gs[0] + (t0 + t) * a.gs[1] + h * a.gs[2] + c];
          dl = x > 0.f ? acc / x : 0.f;
        }
        a.dgate[o] = dl;
      }
    }
  } else {
    const int c = tid - D;
    for (int t = 0; t < nv; ++t) a.dv[((n * a.T + t0 + t) * a.H + h) * D + c] = w.dV[mat + t * D + c];
    if (c < nv) a.dbeta[(n * a.T + t0 + c) * a.H + h] = dbeta_part[(size_t)b * CC + c];
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

cublasHandle_t handle_for_device() {
  static std::mutex mu;
  static cublasHandle_t handles[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!handles[dev] && cublasCreate(&handles[dev]) != CUBLAS_STATUS_SUCCESS) handles[dev] = nullptr;
  return handles[dev];
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
  const int NB = (int)(B * ncps * H);
  const Layout L = carve(B, T, H);
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
  a.T = T; a.B = (int)B; a.H = (int)H; a.ncps = ncps;
  a.gate_log = fwd.gate_mode == KDA_GATE_LOG;

  // 2. per-chunk preparation, Mq and Mk, T and TB
  prep_kernel<<<NB, 256, 0, s>>>(a, w);
  const int pair_smem = 3 * CC * PAD * 4;
  {
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!(configured.load() & (1ull << dev))) {
      const int dsm = (CC * (CC + 1) + 3 * CC * PAD + CC * VS + D * VS + CC * VS + D) * 4;
      const int asm_ = (3 * CC * PAD + 2 * CC * (CC + 1) + 2 * CC * PAD) * 4;
      if ((e = cudaFuncSetAttribute(pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pair_smem)) != cudaSuccess ||
          (e = cudaFuncSetAttribute(dstate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dsm)) != cudaSuccess ||
          (e = cudaFuncSetAttribute(assemble_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, asm_)) != cudaSuccess)
        return e;
      configured.fetch_or(1ull << dev);
    }
  }
  pair_kernel<<<NB, 256, pair_smem, s>>>(w);
  inverse_kernel<<<NB, 64, 0, s>>>(w);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  cublasHandle_t hd = handle_for_device();
  if (!hd) {
    *cublas_status = -1;
    return cudaErrorUnknown;
  }
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
  // 4. the reverse recurrence over chunks for dS
  {
    const int dsm = (CC * (CC + 1) + 3 * CC * PAD + CC * VS + D * VS + CC * VS + D) * 4;
    dstate_kernel<<<dim3((unsigned)(B * H), D / VS), 256, dsm, s>>>(a, w);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // 5. dU = Mq^T dO + KT dS_C; dMq = dO U^T; dQG = dO S0^T; dKT = U dS_C^T; dW = -dU S0^T;
  //    dTB = dU V^T + dW KG^T; dV = TB^T dU; dKG = TB^T dW; X = T^T dT; dA = -X T^T
  G(true, false, CC, D, CC, 1.f, w.Mq, CC, s64, w.dOf, D, s128, 0.f, w.dU, D, s128);
  G(false, false, CC, D, D, 1.f, w.KT, D, s128, w.dSC, D, sst, 1.f, w.dU, D, s128);
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
  mask_dgc_kernel<<<NB, 256, 0, s>>>(w);
  dt_kernel<<<NB, 64, 0, s>>>(w, dbeta_part);  // X = dT = dTB Diag(beta); dbeta_part = colsum(dTB * T)
  // dA = -(T^T dT) T^T: the product T^T dT into dA, then -dA T^T into X (two products, reusing the buffers)
  G(true, false, CC, CC, CC, 1.f, w.Tm, CC, s64, w.X, CC, s64, 0.f, w.dA, CC, s64);
  G(false, true, CC, CC, CC, -1.f, w.dA, CC, s64, w.Tm, CC, s64, 0.f, w.X, CC, s64);
  if (cs != CUBLAS_STATUS_SUCCESS) {
    *cublas_status = (int)cs;
    return cudaErrorUnknown;
  }
  std::swap(w.dA, w.X);  // dA now names the result
  da_kernel<<<NB, 64, 0, s>>>(w, dbeta_part);
  {
    const int asm_ = (3 * CC * PAD + 2 * CC * (CC + 1) + 2 * CC * PAD) * 4;
    assemble_kernel<<<NB, 256, asm_, s>>>(a, w, dbeta_part);
  }
  return cudaGetLastError();
}

}  // namespace kda
