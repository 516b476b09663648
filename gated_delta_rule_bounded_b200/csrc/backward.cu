// backward.cu -- gradients of the scan by the adjoint recurrence, token by token.
//
// Forward ("Kimi K3: Bounded Decay and Delta Memory", eq. 1), per token t:
//     Sbar = Diag(alpha) S_{t-1};  delta = v - Sbar^T k;  S_t = Sbar + beta k delta^T;  o_t = S_t^T q
// With G = dL/dS_t (the output's share q do^T added first), the adjoint step is
//     dq = S_t do;  c = G^T k;  dbeta = delta . c;  dv = beta c;
//     dk = beta G delta - Sbar (beta c);  dSbar = G - k (beta c)^T;
//     dalpha = rowsum(dSbar * S_{t-1});  G <- Diag(alpha) dSbar   (= dL/dS_{t-1})
// and dS_0 = G after the first token. One CTA owns one (batch row, head) and, like the forward
// token kernel, keeps a K x V state slice in registers (a thread: four consecutive value columns
// of K/8 key rows). Walking backwards needs S_{t-1} at every t: a forward pass stores the state
// every kSeg tokens (checkpoints), and each segment is recomputed forward from its checkpoint
// into a per-CTA scratch before the adjoint sweeps it in reverse. Sums over value columns are
// shuffles among the threads of a row group; sums over key rows go through shared memory.
#include "common.cuh"
#include "gate_math.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kGroups = 8;  // key-row groups
constexpr int kSeg = 32;    // tokens per checkpoint segment

template <int RPT, int VT>
struct BwdSmem {
  static constexpr int K = kGroups * RPT;
  static constexpr int A = 0, KK = A + K, Q = KK + K, V = Q + K, DO = V + VT, BETA = DO + VT;
  static constexpr int RED = (BETA + 4 + 3) & ~3;        // [kGroups][VT] column partial sums
  static constexpr int FLOATS = RED + kGroups * VT;
};

// Sum over the VT/4 column-group threads of one row group (consecutive lanes).
template <int VT>
__device__ __forceinline__ float rowgroup_sum(float x) {
#pragma unroll
  for (int m = VT / 8; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

template <int RPT, int VT>
__device__ __forceinline__ float4 colsum(const float* red, int col0) {
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int g = 0; g < kGroups; ++g) {
    const float4 x = *reinterpret_cast<const float4*>(red + g * VT + col0);
    s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
  }
  return s;
}

template <int RPT, int VT, typename TIn>
__global__ void __launch_bounds__(kGroups * (VT / 4)) scan_backward_kernel(BwdParams p) {
  using L = BwdSmem<RPT, VT>;
  constexpr int K = L::K, CG = VT / 4, NT = kGroups * CG;
  __shared__ __align__(16) float sm[L::FLOATS];
  float* sa = sm + L::A;
  float* sk = sm + L::KK;
  float* sq = sm + L::Q;
  float* sv = sm + L::V;
  float* sdo = sm + L::DO;
  float* red = sm + L::RED;

  const int tid = threadIdx.x, tv = tid % CG, tk = tid / CG;
  const int row0 = tk * RPT, col0 = 4 * tv;
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  const int64_t T = p.T;
  const int n_seg = (int)((T + kSeg - 1) / kSeg);
  const size_t slice = (size_t)K * VT;
  float* ckpt = p.ckpt + (size_t)bh * (n_seg + 1) * slice;  // state before token j*kSeg, j = 0..n_seg
  float* scr = p.scratch + (size_t)bh * kSeg * slice;       // states before each token of a segment
  const TIn* qb = static_cast<const TIn*>(p.q);
  const TIn* kb = static_cast<const TIn*>(p.k);
  const TIn* vb = static_cast<const TIn*>(p.v);
  auto tile = [&](float* base, int r) { return reinterpret_cast<float4*>(base + (size_t)(row0 + r) * VT + col0); };

  // Stages token t's alpha, k, v, beta (and q, do when `adj`).
  auto stage = [&](int64_t t, bool adj) {
    const int64_t ko = b * p.ks[0] + t * p.ks[1] + h * p.ks[2];
    const int64_t go = b * p.gs[0] + t * p.gs[1] + h * p.gs[2];
    const int64_t qo = b * p.qs[0] + t * p.qs[1] + h * p.qs[2];
    const int64_t vo = b * p.vs[0] + t * p.vs[1] + h * p.vs[2];
    for (int i = tid; i < K; i += NT) {
      const float gv = __ldg(p.gate + go + i);
      sa[i] = p.gate_log ? expf(gv) : gv;
      sk[i] = to_f32(kb[ko + i]);
      if (adj) sq[i] = to_f32(qb[qo + i]);
    }
    for (int j = tid; j < VT; j += NT) {
      sv[j] = to_f32(vb[vo + j]);
      if (adj) sdo[j] = p.d_o[((b * T + t) * p.H + h) * (int64_t)VT + j];
    }
    if (tid == 0) sm[L::BETA] = __ldg(p.beta + b * p.bs[0] + t * p.bs[1] + h * p.bs[2]);
  };

  // One forward step on the registers x (S_{t-1} -> S_t); token t already staged.
  auto forward_step = [&](float4 (&x)[RPT]) {
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float a = sa[row0 + r], kk = sk[row0 + r];
      x[r].x *= a; x[r].y *= a; x[r].z *= a; x[r].w *= a;
      pa.x = fmaf(kk, x[r].x, pa.x); pa.y = fmaf(kk, x[r].y, pa.y);
      pa.z = fmaf(kk, x[r].z, pa.z); pa.w = fmaf(kk, x[r].w, pa.w);
    }
    *reinterpret_cast<float4*>(red + tk * VT + col0) = pa;
    __syncthreads();
    const float4 A = colsum<RPT, VT>(red, col0);
    const float beta = sm[L::BETA];
    const float4 d = make_float4(sv[col0] - A.x, sv[col0 + 1] - A.y, sv[col0 + 2] - A.z, sv[col0 + 3] - A.w);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float bk = beta * sk[row0 + r];
      x[r].x = fmaf(bk, d.x, x[r].x); x[r].y = fmaf(bk, d.y, x[r].y);
      x[r].z = fmaf(bk, d.z, x[r].z); x[r].w = fmaf(bk, d.w, x[r].w);
    }
    __syncthreads();  // red and the staged token are free again
  };

  // ---- checkpoints: the state before every kSeg-th token --------------------------------------------
  float4 x[RPT];
  const size_t sbase = (size_t)bh * K * VT;
#pragma unroll
  for (int r = 0; r < RPT; ++r) x[r] = p.s0 ? *reinterpret_cast<const float4*>(p.s0 + sbase + (size_t)(row0 + r) * VT + col0)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t t = 0; t < T; ++t) {
    if (t % kSeg == 0) {
#pragma unroll
      for (int r = 0; r < RPT; ++r) *tile(ckpt + (size_t)(t / kSeg) * slice, r) = x[r];
    }
    stage(t, false);
    __syncthreads();
    forward_step(x);
  }

  // ---- adjoint, segment by segment from the end -------------------------------------------------------
  float4 G[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) G[r] = p.d_sf ? *reinterpret_cast<const float4*>(p.d_sf + sbase + (size_t)(row0 + r) * VT + col0)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int seg = n_seg - 1; seg >= 0; --seg) {
    const int64_t t0 = (int64_t)seg * kSeg, t1 = min(T, t0 + kSeg);
#pragma unroll
    for (int r = 0; r < RPT; ++r) x[r] = *tile(ckpt + (size_t)seg * slice, r);
    for (int64_t t = t0; t < t1; ++t) {  // recompute: scr[t - t0] = S_{t-1}
#pragma unroll
      for (int r = 0; r < RPT; ++r) *tile(scr + (size_t)(t - t0) * slice, r) = x[r];
      stage(t, false);
      __syncthreads();
      forward_step(x);
    }
    for (int64_t t = t1 - 1; t >= t0; --t) {
      stage(t, true);
#pragma unroll
      for (int r = 0; r < RPT; ++r) x[r] = *tile(scr + (size_t)(t - t0) * slice, r);  // S_{t-1}
      __syncthreads();
      const float beta = sm[L::BETA];
      // delta from Sbar = Diag(alpha) S_{t-1} (Sbar is recomputed from S_{t-1} where needed)
      auto sbar = [&](int r) {
        const float a = sa[row0 + r];
        return make_float4(a * x[r].x, a * x[r].y, a * x[r].z, a * x[r].w);
      };
      float4 pa = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const float kk = sk[row0 + r];
        const float4 xb = sbar(r);
        pa.x = fmaf(kk, xb.x, pa.x); pa.y = fmaf(kk, xb.y, pa.y);
        pa.z = fmaf(kk, xb.z, pa.z); pa.w = fmaf(kk, xb.w, pa.w);
      }
      *reinterpret_cast<float4*>(red + tk * VT + col0) = pa;
      __syncthreads();
      const float4 A = colsum<RPT, VT>(red, col0);
      const float4 d = make_float4(sv[col0] - A.x, sv[col0 + 1] - A.y, sv[col0 + 2] - A.z, sv[col0 + 3] - A.w);
      const float4 dov = *reinterpret_cast<const float4*>(sdo + col0);
      __syncthreads();  // red is reused below
      // G += q do^T (the output's share), dq = S_t do, and c = G^T k
      float4 pc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const float qq = sq[row0 + r], kk = sk[row0 + r], bk = beta * kk;
        G[r].x = fmaf(qq, dov.x, G[r].x); G[r].y = fmaf(qq, dov.y, G[r].y);
        G[r].z = fmaf(qq, dov.z, G[r].z); G[r].w = fmaf(qq, dov.w, G[r].w);
        const float4 xb = sbar(r);
        const float4 st = make_float4(fmaf(bk, d.x, xb.x), fmaf(bk, d.y, xb.y), fmaf(bk, d.z, xb.z), fmaf(bk, d.w, xb.w));
        const float dq = rowgroup_sum<VT>(st.x * dov.x + st.y * dov.y + st.z * dov.z + st.w * dov.w);
        if (tv == 0) p.dq[((b * T + t) * p.H + h) * (int64_t)K + row0 + r] = dq;
        pc.x = fmaf(kk, G[r].x, pc.x); pc.y = fmaf(kk, G[r].y, pc.y);
        pc.z = fmaf(kk, G[r].z, pc.z); pc.w = fmaf(kk, G[r].w, pc.w);
      }
      *reinterpret_cast<float4*>(red + tk * VT + col0) = pc;
      __syncthreads();
      const float4 c = colsum<RPT, VT>(red, col0);
      const float4 dd = make_float4(beta * c.x, beta * c.y, beta * c.z, beta * c.w);  // dL/d delta = dv
      // delta and c are per-column values, equal in every row group: each group forms the same dbeta.
      const float db = rowgroup_sum<VT>(d.x * c.x + d.y * c.y + d.z * c.z + d.w * c.w);
      if (tk == 0) {
        *reinterpret_cast<float4*>(p.dv + ((b * T + t) * p.H + h) * (int64_t)VT + col0) = dd;
        if (tv == 0) p.dbeta[(b * T + t) * p.H + h] = db;
      }
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const float kk = sk[row0 + r], a = sa[row0 + r];
        const float4 xb = sbar(r);
        const float dk = rowgroup_sum<VT>(beta * (G[r].x * d.x + G[r].y * d.y + G[r].z * d.z + G[r].w * d.w) -
                                          (xb.x * dd.x + xb.y * dd.y + xb.z * dd.z + xb.w * dd.w));
        const float4 ds = make_float4(G[r].x - kk * dd.x, G[r].y - kk * dd.y, G[r].z - kk * dd.z, G[r].w - kk * dd.w);
        const float da = rowgroup_sum<VT>(ds.x * x[r].x + ds.y * x[r].y + ds.z * x[r].z + ds.w * x[r].w);
        if (tv == 0) {
          const int64_t o = ((b * T + t) * p.H + h) * (int64_t)K + row0 + r;
          p.dk[o] = dk;
          p.dgate[o] = p.gate_log ? da * a : da;  // dL/dg = dL/dalpha * alpha
        }
        G[r] = make_float4(a * ds.x, a * ds.y, a * ds.z, a * ds.w);
      }
      __syncthreads();  // red and the staged token are free again
    }
  }
  if (p.ds0) {
#pragma unroll
    for (int r = 0; r < RPT; ++r) *reinterpret_cast<float4*>(p.ds0 + sbase + (size_t)(row0 + r) * VT + col0) = G[r];
  }
}

template <int RPT, int VT, typename TIn>
cudaError_t launch_b(const BwdParams& p, cudaStream_t s) {
  scan_backward_kernel<RPT, VT, TIn><<<(unsigned)(p.B * p.H), kGroups * (VT / 4), 0, s>>>(p);
  return cudaGetLastError();
}

template <int RPT, typename TIn>
cudaError_t launch_bv(const BwdParams& p, cudaStream_t s) {
  switch (p.V) {
    case 16: return launch_b<RPT, 16, TIn>(p, s);
    case 32: return launch_b<RPT, 32, TIn>(p, s);
    case 64: return launch_b<RPT, 64, TIn>(p, s);
    default: return launch_b<RPT, 128, TIn>(p, s);
  }
}

template <typename TIn>
cudaError_t launch_bk(const BwdParams& p, cudaStream_t s) {
  switch (p.K) {
    case 16: return launch_bv<2, TIn>(p, s);
    case 32: return launch_bv<4, TIn>(p, s);
    case 64: return launch_bv<8, TIn>(p, s);
    default: return launch_bv<16, TIn>(p, s);
  }
}

// Gate backward: dz = dg * g_min * s (1 - s) * e^A and dA_log[h] += dg * g_min * s (1 - s) * x,
// with x = e^A z and s = sigmoid(x) (the same device sigmoid as the forward gate).
__global__ void bounded_decay_backward_kernel(const float* __restrict__ z, const float* __restrict__ A_log,
                                              float g_min, const float* __restrict__ dg, int64_t rows, int H, int K,
                                              float* __restrict__ dz, float* __restrict__ dA) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * K; i += (int64_t)gridDim.x * blockDim.x) {
    const int h = (int)((i / K) % H);
    const float sc = expf(__ldg(A_log + h));
    const float x = sc * z[i];
    const float s = gate_sigmoid(x);
    const float w = dg[i] * g_min * s * (1.f - s);
    dz[i] = w * sc;
    atomicAdd(dA + h, w * x);
  }
}

}  // namespace

int64_t backward_segments(int64_t T) { return (T + kSeg - 1) / kSeg; }

bool backward_supported(int K, int V) {
  return (K == 16 || K == 32 || K == 64 || K == 128) && (V == 16 || V == 32 || V == 64 || V == 128);
}

size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V) {
  return (size_t)B * H * (size_t)(backward_segments(T) + 1 + kSeg) * (size_t)K * V * sizeof(float);
}

cudaError_t launch_scan_backward(const BwdParams& p, kda_dtype dt, cudaStream_t s) {
  return dt == KDA_F32 ? launch_bk<float>(p, s) : launch_bk<__nv_bfloat16>(p, s);
}

cudaError_t launch_bounded_decay_backward(const float* z, const float* A_log, float g_min, const float* dg,
                                          int64_t rows, int H, int K, float* dz, float* dA, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(dA, 0, sizeof(float) * H, s);
  if (e != cudaSuccess) return e;
  const int64_t n = rows * K;
  if (n == 0) return cudaSuccess;
  int64_t grid = (n + 255) / 256;
  if (grid > 148 * 8) grid = 148 * 8;
  bounded_decay_backward_kernel<<<(unsigned)grid, 256, 0, s>>>(z, A_log, g_min, dg, rows, H, K, dz, dA);
  return cudaGetLastError();
}

}  // namespace kda
