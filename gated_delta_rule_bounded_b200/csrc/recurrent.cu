// recurrent.cu -- token-by-token gated delta rule with a register-resident state.
//
// One CTA owns one (sequence, head, V-tile) and keeps that K x VT slice of the
// fp32 state in registers: a thread holds four consecutive columns (one float4)
// of rpt = K/8 consecutive key rows, so each warp streams whole 512-byte state
// rows with 16-byte loads. Per token ("Kimi K3: Bounded Decay and Delta Memory",
// eq. 1):
//     Sbar = Diag(alpha) S                  (fade: scales key rows)
//     a_j  = sum_i k_i Sbar_ij,  b_j = sum_i q_i Sbar_ij
//     delta_j = v_j - a_j
//     o_j  = b_j + beta (k.q) delta_j       (= (Sbar + beta k delta^T)^T q)
//     S    = Sbar + beta k delta^T
// The key-dimension sums are per-thread partial sums over its rows followed by
// one cross-row-group reduction in shared memory. Columns of S evolve
// independently, so V-tiles are exact.
//
// The decode step is this kernel with T = 1 and the state read and written in
// place: one read and one write of the state, which makes it HBM-bound. The
// same kernel serves the prefill of fp32 inputs (any supported K, V) with the
// state kept in registers across the whole sequence.
#include "common.cuh"
#include "gate_math.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kRowGroups = 8;

// Floats of one staging buffer, rounded up to a multiple of four so that both
// buffers keep their float4 partial-sum arrays 16-byte aligned.
__host__ __device__ constexpr int stage_floats(int K, int VT) {
  return (3 * K + VT + 2 * kRowGroups * VT + 3 * kRowGroups + 1 + 3) & ~3;
}

// RPT is the (maximum) number of key rows per thread; kExact marks K == 8 * RPT,
// which lets every row loop unroll without guards.
template <int RPT, int VT, bool kExact, typename TIn>
__global__ void __launch_bounds__(kRowGroups * (VT / 4), RPT <= 16 ? 2 : 1)
recurrent_kernel(ScanParams p) {
  constexpr int TV = VT / 4;  // threads along V, four columns each
  constexpr int NT = TV * kRowGroups;
  const int tid = threadIdx.x;
  const int tv = tid % TV, tk = tid / TV;
  const int n_vt = p.V / VT;
  int blk = blockIdx.x;
  const int vt = blk % n_vt;
  blk /= n_vt;
  const int h = blk % p.H;
  const float sc = p.gate_mode >= GATE_LOGITS ? expf(__ldg(p.A_log + h)) : 0.f;  // e^{A_h}
  const int n = blk / p.H;
  const int K = p.K, V = p.V;
  const int rpt = kExact ? RPT : K / kRowGroups;
  const int row0 = tk * rpt;
  const int col0 = vt * VT + tv * 4;

  int64_t t0 = 0, t1 = p.T, brow = n;
  if (p.cu) {
    // Offsets are clamped into [0, T] so that malformed offsets cannot address
    // memory outside the packed tensors.
    t1 = min((int64_t)p.cu[n + 1], p.T);
    t0 = max((int64_t)0, min((int64_t)p.cu[n], t1));
    brow = 0;
  }

  const size_t sbase = ((size_t)n * p.H + h) * (size_t)K * V;
  float4 S[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    S[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rpt && p.s0) {
      if (p.state_vk) {  // value-by-key: the four columns are K apart
        const float* s0 = p.s0 + sbase;
        S[r] = make_float4(s0[state_at(p, 0, row0 + r, col0)], s0[state_at(p, 0, row0 + r, col0 + 1)],
                           s0[state_at(p, 0, row0 + r, col0 + 2)], s0[state_at(p, 0, row0 + r, col0 + 3)]);
      } else {
        S[r] = ld_stream(p.s0 + sbase + (size_t)(row0 + r) * V + col0);
      }
    }
  }

  // Double-buffered per-token staging: gate, key, query, value tile, then the
  // cross-row-group partial sums.
  extern __shared__ float smem[];
  const int per_buf = stage_floats(K, VT);

  const TIn* qb = static_cast<const TIn*>(p.q);
  const TIn* kb = static_cast<const TIn*>(p.k);
  const TIn* vb = static_cast<const TIn*>(p.v);
  TIn* ob = static_cast<TIn*>(p.o);

  int parity = 0;
  for (int64_t t = t0; t < t1; ++t, parity ^= 1) {
    float* s_a = smem + parity * per_buf;
    float* s_k = s_a + K;
    float* s_q = s_k + K;
    float* s_v = s_q + K;
    float* red_a = s_v + VT;
    float* red_b = red_a + kRowGroups * VT;
    float* red_kq = red_b + kRowGroups * VT;
    float* red_kk = red_kq + kRowGroups;  // sums of k^2 and q^2 (in-kernel L2 normalisation)
    float* red_qq = red_kk + kRowGroups;
    float* s_beta = red_qq + kRowGroups;

    const int64_t qo = brow * p.qs[0] + t * p.qs[1] + h * p.qs[2];
    const int64_t ko = brow * p.ks[0] + t * p.ks[1] + h * p.ks[2];
    const int64_t go = brow * p.gs[0] + t * p.gs[1] + h * p.gs[2];
    const int64_t vo = brow * p.vs[0] + t * p.vs[1] + h * p.vs[2];
    for (int i = tid; i < K; i += NT) {
      s_a[i] = gate_alpha(p.gate_mode,
                         gate_input(p.gate_mode, __ldg(p.gate + go + i), p.dt_bias ? __ldg(p.dt_bias + (size_t)h * K + i) : 0.f),
                         sc, p.g_min);
      s_k[i] = to_f32(kb[ko + i]);
      s_q[i] = to_f32(qb[qo + i]);
    }
    for (int j = tid; j < VT; j += NT) s_v[j] = to_f32(vb[vo + vt * VT + j]);
    if (tid == 0) s_beta[0] = beta_value(__ldg(p.beta + brow * p.bs[0] + t * p.bs[1] + h * p.bs[2]), p.beta_sigmoid);
    __syncthreads();

    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
    float pkq = 0.f, pkk = 0.f, pqq = 0.f;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      if (r < rpt) {
        const int i = row0 + r;
        const float a = s_a[i], kk = s_k[i], qq = s_q[i];
        S[r].x *= a; S[r].y *= a; S[r].z *= a; S[r].w *= a;
        pa.x = fmaf(kk, S[r].x, pa.x); pa.y = fmaf(kk, S[r].y, pa.y);
        pa.z = fmaf(kk, S[r].z, pa.z); pa.w = fmaf(kk, S[r].w, pa.w);
        pb.x = fmaf(qq, S[r].x, pb.x); pb.y = fmaf(qq, S[r].y, pb.y);
        pb.z = fmaf(qq, S[r].z, pb.z); pb.w = fmaf(qq, S[r].w, pb.w);
        pkq = fmaf(kk, qq, pkq);
        pkk = fmaf(kk, kk, pkk);
        pqq = fmaf(qq, qq, pqq);
      }
    }
    *reinterpret_cast<float4*>(red_a + tk * VT + tv * 4) = pa;
    *reinterpret_cast<float4*>(red_b + tk * VT + tv * 4) = pb;
    if (tv == 0) {
      red_kq[tk] = pkq;
      red_kk[tk] = pkk;
      red_qq[tk] = pqq;
    }
    __syncthreads();

    float4 A = make_float4(0.f, 0.f, 0.f, 0.f), Bq = A;
    float kq = 0.f, kk2 = 0.f, qq2 = 0.f;
#pragma unroll
    for (int g = 0; g < kRowGroups; ++g) {
      float4 x = *reinterpret_cast<const float4*>(red_a + g * VT + tv * 4);
      float4 y = *reinterpret_cast<const float4*>(red_b + g * VT + tv * 4);
      A.x += x.x; A.y += x.y; A.z += x.z; A.w += x.w;
      Bq.x += y.x; Bq.y += y.y; Bq.z += y.z; Bq.w += y.w;
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
    const float beta = s_beta[0];
    float4 d;
    d.x = s_v[tv * 4 + 0] - A.x;
    d.y = s_v[tv * 4 + 1] - A.y;
    d.z = s_v[tv * 4 + 2] - A.z;
    d.w = s_v[tv * 4 + 3] - A.w;
    if (tk == 0) {
      const float bkq = beta * kq;
      float4 o = make_float4(fmaf(bkq, d.x, Bq.x), fmaf(bkq, d.y, Bq.y), fmaf(bkq, d.z, Bq.z),
                             fmaf(bkq, d.w, Bq.w));
      store4(ob + brow * p.os[0] + t * p.os[1] + h * p.os[2] + col0, o);
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      if (r < rpt) {
        const float bk = beta * (s_k[row0 + r] * ik);
        S[r].x = fmaf(bk, d.x, S[r].x); S[r].y = fmaf(bk, d.y, S[r].y);
        S[r].z = fmaf(bk, d.z, S[r].z); S[r].w = fmaf(bk, d.w, S[r].w);
      }
    }
  }

  if (p.sf) {
#pragma unroll
    for (int r = 0; r < RPT; ++r)
      if (r < rpt) {
        if (p.state_vk) {
          float* sf = p.sf + sbase;
          sf[state_at(p, 0, row0 + r, col0)] = S[r].x;
          sf[state_at(p, 0, row0 + r, col0 + 1)] = S[r].y;
          sf[state_at(p, 0, row0 + r, col0 + 2)] = S[r].z;
          sf[state_at(p, 0, row0 + r, col0 + 3)] = S[r].w;
        } else {
          st_stream(p.sf + sbase + (size_t)(row0 + r) * V + col0, S[r]);
        }
      }
  }
}

template <int RPT, int VT, typename TIn>
cudaError_t launch_rt(const ScanParams& p, cudaStream_t s) {
  constexpr int NT = kRowGroups * (VT / 4);
  const int per_buf = stage_floats(p.K, VT);
  const size_t smem = 2 * (size_t)per_buf * sizeof(float);
  const int64_t grid = (int64_t)p.N * p.H * (p.V / VT);
  if (grid == 0) return cudaSuccess;
  if (p.K == kRowGroups * RPT)
    recurrent_kernel<RPT, VT, true, TIn><<<(unsigned)grid, NT, smem, s>>>(p);
  else
    recurrent_kernel<RPT, VT, false, TIn><<<(unsigned)grid, NT, smem, s>>>(p);
  return cudaGetLastError();
}

template <int RPT, typename TIn>
cudaError_t launch_vt(const ScanParams& p, cudaStream_t s) {
  if (p.V % 128 == 0) return launch_rt<RPT, 128, TIn>(p, s);
  if (p.V % 64 == 0) return launch_rt<RPT, 64, TIn>(p, s);
  if (p.V % 32 == 0) return launch_rt<RPT, 32, TIn>(p, s);
  return launch_rt<RPT, 16, TIn>(p, s);
}

template <typename TIn>
cudaError_t launch_k(const ScanParams& p, cudaStream_t s) {
  const int rpt = p.K / kRowGroups;
  if (rpt <= 2) return launch_vt<2, TIn>(p, s);
  if (rpt <= 4) return launch_vt<4, TIn>(p, s);
  if (rpt <= 8) return launch_vt<8, TIn>(p, s);
  if (rpt <= 16) return launch_vt<16, TIn>(p, s);
  return launch_vt<32, TIn>(p, s);
}

}  // namespace

cudaError_t launch_recurrent(const ScanParams& p, kda_dtype dt, cudaStream_t s) {
  return dt == KDA_F32 ? launch_k<float>(p, s) : launch_k<__nv_bfloat16>(p, s);
}

namespace {
__global__ void state_copy_kernel(const float* __restrict__ s0, float* __restrict__ sf, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    sf[i] = s0 ? s0[i] : 0.f;
}
}  // namespace

cudaError_t launch_state_copy(const float* s0, float* sf, int64_t n, cudaStream_t s) {
  if (n == 0 || sf == nullptr || sf == s0) return cudaSuccess;
  int64_t grid = (n + 255) / 256;
  if (grid > 148 * 16) grid = 148 * 16;
  state_copy_kernel<<<(unsigned)grid, 256, 0, s>>>(s0, sf, n);
  return cudaGetLastError();
}

}  // namespace kda
