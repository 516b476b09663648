// chunk.cu -- chunked prefill of the bounded-decay gated delta rule (bf16 q/k/v).
//
// Math ("KDA cheat sheet", Chunkwise parallel form, eqs. 3-4, with the UT
// transform re-derived from eq. 1 of "Kimi K3: Bounded Decay and Delta
// Memory"). For a chunk of C = 64 tokens starting from state S0 (K x V), with
// G the chunk-local inclusive cumulative log-decay per channel and
// Gamma = exp(G):
//   A_kk[t,i] = beta_t sum_c k_tc k_ic exp(G_tc - G_ic)        (i < t)
//   A_qk[t,i] =        sum_c q_tc k_ic exp(G_tc - G_ic)        (i <= t)
//   T = (I + A_kk)^-1,  W = T Diag(beta)(K*Gamma),  Ut = T Diag(beta) V
//   U = Ut - W S0
//   O = (Q*Gamma) S0 + A_qk U
//   S = Diag(gamma_C) S0 + (K * gamma_C/Gamma)^T U
//
// Numerics of the decay ratios. exp(G_t - G_i) <= 1 for i <= t, but the
// factored form (q exp(G_t)) (k exp(-G_i)) overflows over 64 tokens (G reaches
// -320). The chunk is split into four 16-token blocks and every factor is
// taken against a block boundary: with s_a the token before block a and r_b
// the last token of block b,
//   q_t exp(G_t - G_ic) = [q_t exp(G_t - G_{s_a})] exp(G_{s_a} - G_{r_b}) [k_i exp(G_{r_b} - G_i)]
// for t in block a, i in block b <= a. The bracketed factors are <= 1; the
// middle per-channel factor is <= 1 off the diagonal and at most the decay of
// 15 tokens on it, which the lower bound on g (>= -5.5 here) keeps below
// e^83, inside the bf16/fp32 range ("KDA cheat sheet", Lower-bounded decay:
// the bound is what lets every tile, the diagonal included, be a dense matmul).
// Every other operand (Q*Gamma, K*Gamma, K*gamma_C/Gamma) is <= 1 times q or k.
//
// Kernel organisation. One CTA owns one (sequence, head, 128-wide V-tile) and
// walks its chunks in order; 8 warps; K = 128. The fp32 state lives in the
// accumulator registers of the state-update MMA (warp w owns key rows
// 16w..16w+15, all 128 value columns) and a bf16 copy in shared memory feeds
// the W*S and (Q*Gamma)*S products. All contractions are bf16 tensor-core MMAs
// with fp32 accumulation (mma.sync m16n8k16); the 64x64 triangular inverse is
// blocked forward substitution in fp32 on 16x16 blocks. The next chunk's q, k,
// g are fetched with cp.async as soon as the decay pass has consumed them, and
// its v and beta once the UT products are done, so loads overlap the MMAs.
// Tokens past the end of a sequence are zero-filled with g = 0 and beta = 0,
// which leaves the state unchanged.
#include <atomic>

#include "common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int C = 64;     // tokens per chunk
constexpr int KD = 128;   // key dim (rows of the state)
constexpr int VT = 128;   // value columns per CTA
constexpr int NTHREADS = 256;
constexpr float LOG2E = 1.4426950408889634f;
// Lower clamp of the per-token log2-decay: g >= -5.5 (natural log).
constexpr float G2_MIN = -5.5f * LOG2E;

// Shared-memory map (bytes). Regions are reused once their first content is dead.
constexpr int OFF_RAWQ = 0;                  // bf16 [64][128], plain rows
constexpr int OFF_RAWK = OFF_RAWQ + 16384;   // bf16 [64][128], plain rows
constexpr int OFF_RAWV = OFF_RAWK + 16384;   // bf16 [64][128], swizzled (ldmatrix source)
constexpr int OFF_RAWG = OFF_RAWV + 16384;   // f32  [64][128], plain rows
constexpr int OFF_BETA = OFF_RAWG + 32768;   // f32  [64]
constexpr int OFF_QE = OFF_BETA + 256;       // bf16 [64][128] q*exp(G_t - G_s)
constexpr int OFF_KE = OFF_QE + 16384;       // bf16 [64][128] k*exp(G_t - G_s); later U
constexpr int OFF_KC = OFF_KE + 16384;       // bf16 [64][128] k*exp(G_r - G_t)
constexpr int OFF_AKK = OFF_KC + 16384;      // f32 [64][64] A_kk; later T as bf16 [64][64]
constexpr int OFF_TF = OFF_AKK + 16384;      // f32 [64][64] T; later -W bf16 [64][128]; then O staging
constexpr int OFF_AQK = OFF_TF + 16384;      // bf16 [64][64] A_qk
constexpr int OFF_S = OFF_AQK + 8192;        // bf16 [128][128] state copy
constexpr int OFF_VEC = OFF_S + 32768;       // f32 per-channel vectors
constexpr int VEC_D = 0;                     // [10][128] exp(G_{s_a} - G_{r_b}), pairs a >= b
constexpr int VEC_GS = VEC_D + 10 * 128;     // [4][128]  exp(G_{s_a}) (Gamma at block starts)
constexpr int VEC_P = VEC_GS + 4 * 128;      // [4][128]  exp(G_C - G_{r_b})
constexpr int VEC_GAM = VEC_P + 4 * 128;     // [128]     exp(G_C) = gamma_C
constexpr int VEC_TOT = VEC_GAM + 128;       // [4][128]  per-block log2-decay sums
constexpr int VEC_FLOATS = VEC_TOT + 4 * 128;
constexpr int SMEM_BYTES = OFF_VEC + VEC_FLOATS * 4;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// ---------------------------------------------------------------------------------------------
// Small PTX helpers
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte chunk j of row r in a tile with 256-byte (128 x bf16) or 128-byte rows, XOR-swizzled
// so that eight consecutive rows at the same chunk fall in distinct bank groups.
__device__ __forceinline__ uint32_t swz256(int r, int j) { return r * 256 + ((j ^ (r & 7)) << 4); }
__device__ __forceinline__ uint32_t swz128(int r, int j) { return r * 128 + ((j ^ (r & 7)) << 4); }
__device__ __forceinline__ uint32_t swz256_e(int r, int c) { return swz256(r, c >> 3) + ((c & 7) << 1); }
__device__ __forceinline__ uint32_t swz128_e(int r, int c) { return swz128(r, c >> 3) + ((c & 7) << 1); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t scale2(uint32_t u, float s0, float s1) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  float2 f = __bfloat1622float2(v);
  return pack_bf16(f.x * s0, f.y * s1);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // n == 0 zero-fills the destination
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 4 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------

struct ChunkCtx {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* gate;
  const float* beta;
  int64_t qrow, krow, vrow, grow, boff;  // element offsets of token 0 of this (sequence, head)
  int64_t qst, kst, vst, gst, bst;       // element strides between tokens
};

// q, k, g of chunk c (tokens tc0 .. tc0+nv-1) into the raw buffers; rows >= nv are zero-filled.
__device__ __forceinline__ void load_qkg(const ChunkCtx& x, uint32_t sb, int64_t tc0, int nv, int tid) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid + NTHREADS * i;
    const int row = idx >> 4, piece = idx & 15;
    const bool ok = row < nv;
    const int64_t t = tc0 + (ok ? row : 0);
    cp_async16(sb + OFF_RAWQ + row * 256 + piece * 16, x.q + x.qrow + t * x.qst + piece * 8, ok);
    cp_async16(sb + OFF_RAWK + row * 256 + piece * 16, x.k + x.krow + t * x.kst + piece * 8, ok);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = tid + NTHREADS * i;
    const int row = idx >> 5, piece = idx & 31;
    const bool ok = row < nv;
    const int64_t t = tc0 + (ok ? row : 0);
    cp_async16(sb + OFF_RAWG + row * 512 + piece * 16, x.gate + x.grow + t * x.gst + piece * 4, ok);
  }
}

// v tile and beta of chunk c.
__device__ __forceinline__ void load_vb(const ChunkCtx& x, uint32_t sb, int64_t tc0, int nv, int tid) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid + NTHREADS * i;
    const int row = idx >> 4, piece = idx & 15;
    const bool ok = row < nv;
    const int64_t t = tc0 + (ok ? row : 0);
    cp_async16(sb + OFF_RAWV + swz256(row, piece), x.v + x.vrow + t * x.vst + piece * 8, ok);
  }
  if (tid < C) {
    const bool ok = tid < nv;
    const int64_t t = tc0 + (ok ? tid : 0);
    cp_async4(sb + OFF_BETA + tid * 4, x.beta + x.boff + t * x.bst, ok);
  }
}

__global__ void __launch_bounds__(NTHREADS, 1) chunk_prefill_kernel(ScanParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;

  const int n_vt = p.V / VT;
  int blk = blockIdx.x;
  const int vt = blk % n_vt;
  blk /= n_vt;
  const int h = blk % p.H;
  const int n = blk / p.H;

  int64_t t0 = 0, t1 = p.T, brow = n;
  if (p.cu) {
    t1 = min((int64_t)p.cu[n + 1], p.T);
    t0 = max((int64_t)0, min((int64_t)p.cu[n], t1));
    brow = 0;
  }
  const int n_chunks = (int)((t1 - t0 + C - 1) / C);

  ChunkCtx x;
  x.q = static_cast<const __nv_bfloat16*>(p.q);
  x.k = static_cast<const __nv_bfloat16*>(p.k);
  x.v = static_cast<const __nv_bfloat16*>(p.v);
  x.gate = p.gate;
  x.beta = p.beta;
  x.qrow = brow * p.qs[0] + h * p.qs[2];
  x.krow = brow * p.ks[0] + h * p.ks[2];
  x.vrow = brow * p.vs[0] + h * p.vs[2] + (int64_t)vt * VT;
  x.grow = brow * p.gs[0] + h * p.gs[2];
  x.boff = brow * p.bs[0] + h * p.bs[2];
  x.qst = p.qs[1];
  x.kst = p.ks[1];
  x.vst = p.vs[1];
  x.gst = p.gs[1];
  x.bst = p.bs[1];

  float* vec = reinterpret_cast<float*>(sm + OFF_VEC);
  const float* beta_s = reinterpret_cast<const float*>(sm + OFF_BETA);

  if (n_chunks > 0) {
    load_qkg(x, sb, t0, (int)min((int64_t)C, t1 - t0), tid);
    load_vb(x, sb, t0, (int)min((int64_t)C, t1 - t0), tid);
    cp_async_commit();
  }

  // State: warp owns key rows 16*warp + {g, g+8}; n8 tile j covers value columns 8j .. 8j+7.
  const size_t sbase = ((size_t)n * p.H + h) * (size_t)KD * p.V + (size_t)vt * VT;
  const int srow0 = 16 * warp + g, srow1 = srow0 + 8;
  float S[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int col = 8 * j + 2 * tq;
    if (p.s0) {
      const float2 a = *reinterpret_cast<const float2*>(p.s0 + sbase + (size_t)srow0 * p.V + col);
      const float2 b = *reinterpret_cast<const float2*>(p.s0 + sbase + (size_t)srow1 * p.V + col);
      S[j][0] = a.x; S[j][1] = a.y; S[j][2] = b.x; S[j][3] = b.y;
    } else {
      S[j][0] = S[j][1] = S[j][2] = S[j][3] = 0.f;
    }
    *reinterpret_cast<uint32_t*>(sm + OFF_S + swz256_e(srow0, col)) = pack_bf16(S[j][0], S[j][1]);
    *reinterpret_cast<uint32_t*>(sm + OFF_S + swz256_e(srow1, col)) = pack_bf16(S[j][2], S[j][3]);
  }

  const int m = warp & 3, nh = warp >> 2;  // 16-row block and 64-column half for the 64x128 products

  for (int c = 0; c < n_chunks; ++c) {
    const int64_t tc0 = t0 + (int64_t)c * C;
    const int nv = (int)min((int64_t)C, t1 - tc0);
    const bool has_next = c + 1 < n_chunks;
    const int64_t tn0 = tc0 + C;
    const int nvn = has_next ? (int)min((int64_t)C, t1 - tn0) : 0;

    cp_async_wait_all();
    __syncthreads();  // raw inputs of chunk c are in shared memory; the previous state copy is written

    // ---- decay pass: block-local cumulative log2-decay, scaled copies of q and k ----------------
    {
      const int ch = tid & 127, half = tid >> 7;
      const float* rg = reinterpret_cast<const float*>(sm + OFF_RAWG);
      const __nv_bfloat16* rq = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_RAWQ);
      const __nv_bfloat16* rk = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_RAWK);
#pragma unroll
      for (int bb = 0; bb < 2; ++bb) {
        const int a = half * 2 + bb;
        float pre[16];
        float run = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = a * 16 + i;
          float g2 = 0.f;
          if (t < nv) {
            const float gv = rg[t * 128 + ch];
            g2 = p.gate_log ? gv * LOG2E : lg2(gv);
            g2 = fmaxf(g2, G2_MIN);
          }
          run += g2;
          pre[i] = run;
        }
        vec[VEC_TOT + a * 128 + ch] = run;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = a * 16 + i;
          const float E = ex2(pre[i]);        // exp(G_t - G_{s_a}) <= 1
          const float F = ex2(run - pre[i]);  // exp(G_{r_a} - G_t) <= 1
          const float qv = __bfloat162float(rq[t * 128 + ch]);
          const float kv = __bfloat162float(rk[t * 128 + ch]);
          *reinterpret_cast<__nv_bfloat16*>(sm + OFF_QE + swz256_e(t, ch)) = __float2bfloat16_rn(qv * E);
          *reinterpret_cast<__nv_bfloat16*>(sm + OFF_KE + swz256_e(t, ch)) = __float2bfloat16_rn(kv * E);
          *reinterpret_cast<__nv_bfloat16*>(sm + OFF_KC + swz256_e(t, ch)) = __float2bfloat16_rn(kv * F);
        }
      }
    }
    __syncthreads();  // raw q, k, g consumed; block sums published

    if (has_next) load_qkg(x, sb, tn0, nvn, tid);
    cp_async_commit();

    if (tid < 128) {
      const int ch = tid;
      const float e0 = vec[VEC_TOT + ch];
      const float e1 = e0 + vec[VEC_TOT + 128 + ch];
      const float e2 = e1 + vec[VEC_TOT + 256 + ch];
      const float e3 = e2 + vec[VEC_TOT + 384 + ch];
      const float gs[4] = {0.f, e0, e1, e2};  // log2 Gamma at s_a
      const float ge[4] = {e0, e1, e2, e3};   // log2 Gamma at r_b
      int idx = 0;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b <= a; ++b) vec[VEC_D + (idx++) * 128 + ch] = ex2(gs[a] - ge[b]);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        vec[VEC_GS + a * 128 + ch] = ex2(gs[a]);
        vec[VEC_P + a * 128 + ch] = ex2(e3 - ge[a]);
      }
      vec[VEC_GAM + ch] = ex2(e3);
    }
    __syncthreads();  // decay vectors ready

    // ---- A_qk (warps 0-3) and A_kk (warps 4-7), 16x16 tiles (a, b), a >= b ----------------------
    {
      const int mat = warp >> 2;
      const uint32_t rows = sb + (mat ? OFF_KE : OFF_QE);
      for (int tile = warp & 3; tile < 10; tile += 4) {
        const int a = tile >= 6 ? 3 : (tile >= 3 ? 2 : (tile >= 1 ? 1 : 0));
        const int b = tile - a * (a + 1) / 2;
        const float* Dv = vec + VEC_D + tile * 128;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
          ldsm_x4(rows + swz256(16 * a + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
          const int c0 = 16 * kk + 2 * tq;
          const float d0 = Dv[c0], d1 = Dv[c0 + 1], d8 = Dv[c0 + 8], d9 = Dv[c0 + 9];
          a0 = scale2(a0, d0, d1);
          a1 = scale2(a1, d0, d1);
          a2 = scale2(a2, d8, d9);
          a3 = scale2(a3, d8, d9);
          ldsm_x4(sb + OFF_KC + swz256(16 * b + (lane & 7) + (lane >> 4) * 8, 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
          mma_bf16(acc[0], a0, a1, a2, a3, b0, b1);
          mma_bf16(acc[1], a0, a1, a2, a3, b2, b3);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
            const int t = 16 * a + g + 8 * hr;
            const int i0 = 16 * b + 8 * j + 2 * tq;
            float v0 = acc[j][2 * hr], v1 = acc[j][2 * hr + 1];
            if (mat == 0) {
              if (a == b) {
                v0 = (i0 <= t) ? v0 : 0.f;
                v1 = (i0 + 1 <= t) ? v1 : 0.f;
              }
              *reinterpret_cast<uint32_t*>(sm + OFF_AQK + swz128_e(t, i0)) = pack_bf16(v0, v1);
            } else {
              const float bt = beta_s[t];
              v0 = (a > b || i0 < t) ? v0 * bt : 0.f;
              v1 = (a > b || i0 + 1 < t) ? v1 * bt : 0.f;
              *reinterpret_cast<float2*>(sm + OFF_AKK + (t * 64 + i0) * 4) = make_float2(v0, v1);
            }
          }
      }
    }
    __syncthreads();  // A_qk, A_kk ready

    // ---- T = (I + A_kk)^-1 by blocked forward substitution (fp32) ----------------------------
    {
      const float* L = reinterpret_cast<const float*>(sm + OFF_AKK);
      float* Tm = reinterpret_cast<float*>(sm + OFF_TF);
      if (tid < 64) {
        const int a = tid >> 4, j = tid & 15;
        float xcol[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float s = (i == j) ? 1.f : 0.f;
#pragma unroll
          for (int l = 0; l < i; ++l) s -= L[(16 * a + i) * 64 + 16 * a + l] * xcol[l];
          xcol[i] = s;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[(16 * a + i) * 64 + 16 * a + j] = xcol[i];
      }
      __syncthreads();
#pragma unroll 1
      for (int d = 1; d <= 3; ++d) {
        const int nblk = 4 - d;
        // P_ab = sum_{j=b}^{a-1} L_aj T_jb, kept in the unused upper block (b, a) of Tm.
        for (int e = tid; e < nblk * 256; e += NTHREADS) {
          const int b = e >> 8, r = (e >> 4) & 15, cc = e & 15, a = b + d;
          float s = 0.f;
          for (int jb = b; jb < a; ++jb)
#pragma unroll
            for (int l = 0; l < 16; ++l) s += L[(16 * a + r) * 64 + 16 * jb + l] * Tm[(16 * jb + l) * 64 + 16 * b + cc];
          Tm[(16 * b + r) * 64 + 16 * a + cc] = s;
        }
        __syncthreads();
        // T_ab = -T_aa P_ab
        for (int e = tid; e < nblk * 256; e += NTHREADS) {
          const int b = e >> 8, r = (e >> 4) & 15, cc = e & 15, a = b + d;
          float s = 0.f;
#pragma unroll
          for (int l = 0; l < 16; ++l) s += Tm[(16 * a + r) * 64 + 16 * a + l] * Tm[(16 * b + l) * 64 + 16 * a + cc];
          Tm[(16 * a + r) * 64 + 16 * b + cc] = -s;
        }
        __syncthreads();
      }
      // T Diag(beta) to bf16 (the A_kk region is dead now): folding beta into T's columns lets
      // W and Ut take K*Gamma and V without a per-element beta scale. Only blocks on or below
      // the diagonal are read later.
      for (int e = tid; e < 64 * 32; e += NTHREADS) {
        const int r = e >> 5, c2 = (e & 31) * 2;
        const float2 tv = *reinterpret_cast<const float2*>(Tm + r * 64 + c2);
        *reinterpret_cast<uint32_t*>(sm + OFF_AKK + swz128_e(r, c2)) =
            pack_bf16(tv.x * beta_s[c2], tv.y * beta_s[c2 + 1]);
      }
    }
    __syncthreads();  // T (bf16) ready

    // ---- W = (T Diag(beta)) (K*Gamma) (stored negated), Ut = (T Diag(beta)) V (in registers) ----
    float accU[8][4];
    {
      float accW[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) accW[j][e] = accU[j][e] = 0.f;
      for (int kk = 0; kk <= m; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sb + OFF_AKK + swz128(16 * m + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
        const float* gsv = vec + VEC_GS + kk * 128;
        const int rr = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          const int col0 = 64 * nh + 16 * pp;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sb + OFF_KE + swz256(rr, (col0 >> 3) + (lane >> 4)), b0, b1, b2, b3);
          const float gs0 = gsv[col0 + g], gs1 = gsv[col0 + 8 + g];
          b0 = scale2(b0, gs0, gs0);
          b1 = scale2(b1, gs0, gs0);
          b2 = scale2(b2, gs1, gs1);
          b3 = scale2(b3, gs1, gs1);
          mma_bf16(accW[2 * pp], a0, a1, a2, a3, b0, b1);
          mma_bf16(accW[2 * pp + 1], a0, a1, a2, a3, b2, b3);
          ldsm_x4_t(sb + OFF_RAWV + swz256(rr, (col0 >> 3) + (lane >> 4)), b0, b1, b2, b3);
          mma_bf16(accU[2 * pp], a0, a1, a2, a3, b0, b1);
          mma_bf16(accU[2 * pp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = 64 * nh + 8 * j + 2 * tq;
        *reinterpret_cast<uint32_t*>(sm + OFF_TF + swz256_e(16 * m + g, col)) = pack_bf16(-accW[j][0], -accW[j][1]);
        *reinterpret_cast<uint32_t*>(sm + OFF_TF + swz256_e(16 * m + g + 8, col)) = pack_bf16(-accW[j][2], -accW[j][3]);
      }
    }
    __syncthreads();  // -W ready; v tile, beta and K*exp(...) are dead

    if (has_next) load_vb(x, sb, tn0, nvn, tid);
    cp_async_commit();

    // ---- U = Ut - W S ---------------------------------------------------------------------------
#pragma unroll 2
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sb + OFF_TF + swz256(16 * m + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
      const int rr = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sb + OFF_S + swz256(rr, 8 * nh + 2 * pp + (lane >> 4)), b0, b1, b2, b3);
        mma_bf16(accU[2 * pp], a0, a1, a2, a3, b0, b1);
        mma_bf16(accU[2 * pp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int col = 64 * nh + 8 * j + 2 * tq;
      *reinterpret_cast<uint32_t*>(sm + OFF_KE + swz256_e(16 * m + g, col)) = pack_bf16(accU[j][0], accU[j][1]);
      *reinterpret_cast<uint32_t*>(sm + OFF_KE + swz256_e(16 * m + g + 8, col)) = pack_bf16(accU[j][2], accU[j][3]);
    }
    __syncthreads();  // U ready

    // ---- O = (Q*Gamma) S + A_qk U ------------------------------------------------------------
    {
      float accO[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) accO[j][e] = 0.f;
      const float* gsv = vec + VEC_GS + m * 128;
#pragma unroll 2
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sb + OFF_QE + swz256(16 * m + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
        const int c0 = 16 * kk + 2 * tq;
        const float s0 = gsv[c0], s1 = gsv[c0 + 1], s8 = gsv[c0 + 8], s9 = gsv[c0 + 9];
        a0 = scale2(a0, s0, s1);
        a1 = scale2(a1, s0, s1);
        a2 = scale2(a2, s8, s9);
        a3 = scale2(a3, s8, s9);
        const int rr = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sb + OFF_S + swz256(rr, 8 * nh + 2 * pp + (lane >> 4)), b0, b1, b2, b3);
          mma_bf16(accO[2 * pp], a0, a1, a2, a3, b0, b1);
          mma_bf16(accO[2 * pp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      for (int kk = 0; kk <= m; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sb + OFF_AQK + swz128(16 * m + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
        const int rr = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sb + OFF_KE + swz256(rr, 8 * nh + 2 * pp + (lane >> 4)), b0, b1, b2, b3);
          mma_bf16(accO[2 * pp], a0, a1, a2, a3, b0, b1);
          mma_bf16(accO[2 * pp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = 64 * nh + 8 * j + 2 * tq;
        *reinterpret_cast<uint32_t*>(sm + OFF_TF + swz256_e(16 * m + g, col)) = pack_bf16(accO[j][0], accO[j][1]);
        *reinterpret_cast<uint32_t*>(sm + OFF_TF + swz256_e(16 * m + g + 8, col)) = pack_bf16(accO[j][2], accO[j][3]);
      }
    }
    __syncthreads();  // O staged; every read of the state copy for this chunk is done

    {
      __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(p.o);
      const int64_t orow = brow * p.os[0] + h * p.os[2] + (int64_t)vt * VT;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int idx = tid + NTHREADS * i;
        const int row = idx >> 4, piece = idx & 15;
        if (row < nv) {
          const uint4 val = *reinterpret_cast<const uint4*>(sm + OFF_TF + swz256(row, piece));
          *reinterpret_cast<uint4*>(ob + orow + (tc0 + row) * p.os[1] + piece * 8) = val;
        }
      }
    }

    // ---- S = Diag(gamma_C) S + (K * gamma_C/Gamma)^T U ------------------------------------------
    {
      const float gm0 = vec[VEC_GAM + srow0], gm1 = vec[VEC_GAM + srow1];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        S[j][0] *= gm0; S[j][1] *= gm0; S[j][2] *= gm1; S[j][3] *= gm1;
      }
      const int mi = lane >> 3;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(sb + OFF_KC + swz256(16 * kk + (mi >> 1) * 8 + (lane & 7), 2 * warp + (mi & 1)), a0, a1, a2, a3);
        const float p0 = vec[VEC_P + kk * 128 + srow0], p1 = vec[VEC_P + kk * 128 + srow1];
        a0 = scale2(a0, p0, p0);
        a1 = scale2(a1, p1, p1);
        a2 = scale2(a2, p0, p0);
        a3 = scale2(a3, p1, p1);
        const int rr = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int pp = 0; pp < 8; ++pp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sb + OFF_KE + swz256(rr, 2 * pp + (lane >> 4)), b0, b1, b2, b3);
          mma_bf16(S[2 * pp], a0, a1, a2, a3, b0, b1);
          mma_bf16(S[2 * pp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int col = 8 * j + 2 * tq;
        *reinterpret_cast<uint32_t*>(sm + OFF_S + swz256_e(srow0, col)) = pack_bf16(S[j][0], S[j][1]);
        *reinterpret_cast<uint32_t*>(sm + OFF_S + swz256_e(srow1, col)) = pack_bf16(S[j][2], S[j][3]);
      }
    }
  }
  cp_async_wait_all();

  if (p.sf) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int col = 8 * j + 2 * tq;
      *reinterpret_cast<float2*>(p.sf + sbase + (size_t)srow0 * p.V + col) = make_float2(S[j][0], S[j][1]);
      *reinterpret_cast<float2*>(p.sf + sbase + (size_t)srow1 * p.V + col) = make_float2(S[j][2], S[j][3]);
    }
  }
}

}  // namespace

bool chunk_supported(int K, int V, kda_dtype dt) { return dt == KDA_BF16 && K == KD && V % VT == 0; }

size_t chunk_workspace_bytes(int64_t, int64_t, int64_t, int64_t, int64_t, int64_t) { return 0; }

cudaError_t launch_chunk(const ScanParams& p, void*, size_t, cudaStream_t s) {
  // The shared-memory opt-in is per device; remember which devices have it.
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load(std::memory_order_relaxed) & bit)) {
    e = cudaFuncSetAttribute(chunk_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const int64_t grid = (int64_t)p.N * p.H * (p.V / VT);
  if (grid == 0) return cudaSuccess;
  chunk_prefill_kernel<<<(unsigned)grid, NTHREADS, SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
