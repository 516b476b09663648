// chunk.cu -- chunked prefill of the bounded-decay gated delta rule (bf16 q/k/v) on
// sm_100a: the per-chunk state products run on tcgen05 tensor cores with the
// fp32 state held in tensor memory (TMEM).
//
// Math ("KDA cheat sheet", Chunkwise parallel form, eqs. 3-4, with the UT
// transform re-derived from eq. 1 of "Kimi K3: Bounded Decay and Delta
// Memory"). For a chunk of C = 64 tokens starting from state S0 (K x V), with
// G the chunk-local inclusive cumulative log-decay per channel and Gamma = exp(G):
//   A_kk[t,i] = beta_t sum_c k_tc k_ic exp(G_tc - G_ic)        (i < t)
//   A_qk[t,i] =        sum_c q_tc k_ic exp(G_tc - G_ic)        (i <= t)
//   T' = (I + A_kk)^-1 Diag(beta),  W = T' (K*Gamma),  Ut = T' V
//   U = Ut - W S0,  O = (Q*Gamma) S0 + A_qk U,  S = Diag(gamma_C) S0 + (K * gamma_C/Gamma)^T U
//
// Decay ratios. exp(G_t - G_i) <= 1 for i <= t, but the factored form
// (q exp(G_t))(k exp(-G_i)) overflows over 64 tokens (G reaches -320). The
// chunk is split into four 16-token blocks and every factor is taken against
// a block boundary: with s_a the token before block a and r_b the last token
// of block b,
//   q_t exp(G_t - G_ic) = [q_t exp(G_t - G_{s_a})] exp(G_{s_a} - G_{r_b}) [k_i exp(G_{r_b} - G_i)]
// for t in block a, i in block b <= a. The bracketed factors are <= 1; the
// middle per-channel factor is <= 1 off the diagonal and at most the decay of
// 15 tokens on it, which the lower bound on g (clamped at -5.5 here) keeps
// below e^83, inside the bf16/fp32 range ("KDA cheat sheet", Lower-bounded
// decay: the bound is what lets every tile, the diagonal included, be a dense
// matmul). Q*Gamma, K*Gamma and K*gamma_C/Gamma are <= 1 times q or k.
//
// Organisation. One CTA (8 warps) owns one (sequence, head, 128-wide V-tile)
// and walks its chunks in order; K = 128. The state is kept transposed,
// S^T (V x K, fp32), in TMEM lanes 0..127 (one lane per value column), so
// every state product is an M = 128 tcgen05 MMA issued by one thread:
//   group 1:  W^T = (K*Gamma)^T T'^T,  U^T = V^T T'^T,  O^T = S^T (Q*Gamma)^T
//   group 2:  U^T += S^T (-W)^T
//   group 3:  O^T += U^T A_qk^T,       S^T += U^T (K*gamma_C/Gamma)   (S^T pre-scaled by gamma_C)
// Operands are bf16 tiles in shared memory in the 128-byte-swizzled canonical
// layouts; accumulators are fp32 in TMEM. Between groups all 8 warps move
// accumulators out of TMEM (one TMEM lane per thread, one contiguous smem row
// per thread). The decay pass and the 16x16 A_qk / A_kk tiles (whose operands
// need a different decay factor per block pair) stay on the SIMT pipes and
// mma.sync; the 64x64 triangular inverse is blocked forward substitution in
// fp32. The next chunk's q, k, g are loaded into registers while the MMAs of
// the current chunk run, and its v tile and beta by cp.async into a second
// buffer. Every wait on an mbarrier has an iteration limit; on expiry the
// kernel records the timeout in a device flag, stops, releases TMEM and
// returns. Tokens past the end of a sequence are zero-filled with g = 0 and
// beta = 0, which leaves the state unchanged.
#include <atomic>

#include "common.cuh"
#include "kda_internal.h"

namespace kda {

// Set to 1 by any chunk-kernel CTA whose bounded wait on an MMA completion expired.
__device__ int g_chunk_timeout = 0;

namespace {

constexpr int C = 64;     // tokens per chunk
constexpr int KD = 128;   // key dim
constexpr int VT = 128;   // value columns per CTA
constexpr int NTHREADS = 256;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float G2_MIN = -5.5f * LOG2E;  // lower clamp of the per-token log2-decay

// Shared-memory map (bytes). Every bf16 operand tile uses 128-byte rows with the
// 128-byte swizzle (16-byte chunk j of row r stored at chunk j ^ (r & 7)); tiles
// with 128 columns are two 64-column "atoms" stored one after the other.
constexpr int OFF_V = 0;          // 2 x 16K  v tile [i][v], two v-halves (MN-major A of U^T)
constexpr int OFF_QE = 32768;     // 16K  q*exp(G_t - G_s) [t][c]
constexpr int OFF_KE = 49152;     // 16K  k*exp(G_t - G_s) [t][c]; later T' and a bf16 copy of T
constexpr int OFF_TP = OFF_KE;        // 8K   T' = T Diag(beta), bf16 [t][i] (K-major B)
constexpr int OFF_TB = OFF_KE + 8192; // 8K   T, bf16 [t][i] (operand of the inverse's products)
constexpr int OFF_KC = 65536;     // 16K  k*exp(G_r - G_t) [t][c]
constexpr int OFF_AKK = 81920;    // 16K  A_kk fp32 [64][64]
constexpr int OFF_QG = 98304;     // 16K  Q*Gamma [t][c] (K-major B); later -W [c][t] (MN-major B)
constexpr int OFF_KG = 114688;    // 16K  K*Gamma [i][c] (MN-major A); later U [v][i] (K-major A)
constexpr int OFF_KT = 131072;    // 16K  K*gamma_C/Gamma [t][c] (MN-major B)
constexpr int OFF_AQK = 147456;   // 8K   A_qk bf16 [t][i] (K-major B)
constexpr int OFF_S = 155648;     // 32K  S bf16 [v][c], two c-atoms of [128][64] (K-major A)
constexpr int OFF_BETA = 188416;  // 2 x 64 fp32
constexpr int OFF_VEC = 188928;   // fp32 vectors
constexpr int VEC_D = 0;          // [10][128] bf16 exp(G_{s_a} - G_{r_b}), pairs a >= b (640 floats)
constexpr int VEC_GAM = 640;      // [128]     gamma_C
constexpr int VEC_TOT = 768;      // [4][128]  per-block log2-decay sums
constexpr int VEC_FLOATS = 1280;
constexpr int OFF_BAR = OFF_VEC + VEC_FLOATS * 4;  // mbarrier (8 B) + TMEM base (4 B)
constexpr int SMEM_BYTES = OFF_BAR + 64;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(OFF_S % 1024 == 0 && OFF_AQK % 1024 == 0 && OFF_KT % 1024 == 0, "swizzle atoms need 1 KB alignment");

// TMEM columns (fp32 accumulators; lanes 0..127).
constexpr uint32_t TM_S = 0;      // S^T [v][c], 128 columns
constexpr uint32_t TM_U = 128;    // U^T [v][t], 64 columns
constexpr uint32_t TM_O = 192;    // O^T [v][t], 64 columns
constexpr uint32_t TM_W = 256;    // W^T [c][t], 64 columns
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t WAIT_LIMIT = 1u << 22;

// ---------------------------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of element (r, c) in a tile of 128-byte rows (64 bf16 per atom); atom_bytes is the
// distance between the two 64-column atoms of a 128-column tile.
__device__ __forceinline__ uint32_t sw_e(int r, int c, int atom_bytes) {
  return (c >> 6) * atom_bytes + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1);
}
// Byte offset of the 16-byte chunk holding columns 8j..8j+7 of row r.
__device__ __forceinline__ uint32_t sw_chunk(int r, int j, int atom_bytes) {
  return (j >> 3) * atom_bytes + r * 128 + (((j & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

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
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
}
// Elementwise bf16x2 product (one rounding of the exact product).
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
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

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: 128-byte swizzle, start address, leading and stride byte offsets.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
               "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tm_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tm_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Waits for phase `parity` of the mbarrier with an iteration limit. Returns false (and records
// the timeout) when the limit expires.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t it = 0; it < WAIT_LIMIT; ++it) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done) : "r"(bar), "r"(parity) : "memory");
    if (done) return true;
  }
  atomicExch(&g_chunk_timeout, 1);
  return false;
}

__device__ __forceinline__ uint4 pack8(const uint32_t (&r)[32], int j, float sign) {
  uint4 w;
  w.x = pack_bf16(sign * __uint_as_float(r[8 * j + 0]), sign * __uint_as_float(r[8 * j + 1]));
  w.y = pack_bf16(sign * __uint_as_float(r[8 * j + 2]), sign * __uint_as_float(r[8 * j + 3]));
  w.z = pack_bf16(sign * __uint_as_float(r[8 * j + 4]), sign * __uint_as_float(r[8 * j + 5]));
  w.w = pack_bf16(sign * __uint_as_float(r[8 * j + 6]), sign * __uint_as_float(r[8 * j + 7]));
  return w;
}

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

// Registers holding one thread's share of a chunk's q, k, g: channels c0, c0+1 of the 16 tokens
// of block a (thread = (channel pair, block)).
struct Prefetch {
  float2 g[16];
  uint32_t q[16], k[16];
};

__device__ __forceinline__ void load_qkg(const ChunkCtx& x, int64_t tc0, int nv, int c0, int a, Prefetch& pf) {
  const int64_t t = tc0 + 16 * a;
  const float* gp = x.gate + x.grow + t * x.gst + c0;
  const __nv_bfloat16* qp = x.q + x.qrow + t * x.qst + c0;
  const __nv_bfloat16* kp = x.k + x.krow + t * x.kst + c0;
  const int imax = nv - 16 * a;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (i < imax) {
      pf.g[i] = *reinterpret_cast<const float2*>(gp);
      pf.q[i] = *reinterpret_cast<const uint32_t*>(qp);
      pf.k[i] = *reinterpret_cast<const uint32_t*>(kp);
    } else {
      pf.g[i] = make_float2(0.f, 0.f);
      pf.q[i] = pf.k[i] = 0u;
    }
    gp += x.gst;
    qp += x.qst;
    kp += x.kst;
  }
}

// v tile (into the MN-major operand layout) and beta of a chunk.
__device__ __forceinline__ void load_vb(const ChunkCtx& x, uint32_t vbase, uint32_t bbase, int64_t tc0, int nv,
                                        int tid) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid + NTHREADS * i;
    const int row = idx >> 4, piece = idx & 15;
    const bool ok = row < nv;
    const int64_t t = tc0 + (ok ? row : 0);
    cp_async16(vbase + (piece >> 3) * 8192 + row * 128 + (((piece & 7) ^ (row & 7)) << 4),
               x.v + x.vrow + t * x.vst + piece * 8, ok);
  }
  if (tid < C) {
    const bool ok = tid < nv;
    const int64_t t = tc0 + (ok ? tid : 0);
    cp_async4(bbase + tid * 4, x.beta + x.boff + t * x.bst, ok);
  }
}

// 16x16 block pairs (a, b), a >= b, of A_qk (rows from Qe) or A_kk (rows from Ke) against the Kc
// columns, with the per-pair decay factor D_ab applied to the row operand. The warp takes tiles
// first, first + stride, ... (nt of them) and runs their k-loops interleaved so the MMA chains
// overlap. A_qk is stored as a bf16 K-major operand (diagonal blocks masked to i <= t); A_kk as
// fp32 [64][64] with beta_t applied and diagonal blocks masked to i < t.
template <int NTMAX>
__device__ __forceinline__ void a_tiles(unsigned char* sm, uint32_t sb, const float* vec, int off_rows, int first,
                                        int stride, int nt, int lane, int g, int tq, const float* beta_s,
                                        bool is_qk) {
  int ta[NTMAX], tbk[NTMAX], tid_[NTMAX];
#pragma unroll
  for (int n = 0; n < NTMAX; ++n) {
    const int tile = first + stride * n;
    tid_[n] = tile;
    ta[n] = tile >= 6 ? 3 : (tile >= 3 ? 2 : (tile >= 1 ? 1 : 0));
    tbk[n] = tile - ta[n] * (ta[n] + 1) / 2;
  }
  const __nv_bfloat16* D16 = reinterpret_cast<const __nv_bfloat16*>(vec + VEC_D);
  float acc[NTMAX][2][4];
#pragma unroll
  for (int n = 0; n < NTMAX; ++n)
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[n][j][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
    for (int n = 0; n < NTMAX; ++n) {
      if (n < nt) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        const int ra = 16 * ta[n] + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldsm_x4(sb + off_rows + sw_chunk(ra, 2 * kk + (lane >> 4), 8192), a0, a1, a2, a3);
        const __nv_bfloat16* Dv = D16 + tid_[n] * 128 + 16 * kk + 2 * tq;
        const uint32_t d01 = *reinterpret_cast<const uint32_t*>(Dv);
        const uint32_t d89 = *reinterpret_cast<const uint32_t*>(Dv + 8);
        a0 = hmul2(a0, d01);
        a1 = hmul2(a1, d01);
        a2 = hmul2(a2, d89);
        a3 = hmul2(a3, d89);
        const int rb = 16 * tbk[n] + (lane & 7) + (lane >> 4) * 8;
        ldsm_x4(sb + OFF_KC + sw_chunk(rb, 2 * kk + ((lane >> 3) & 1), 8192), b0, b1, b2, b3);
        mma_bf16(acc[n][0], a0, a1, a2, a3, b0, b1);
        mma_bf16(acc[n][1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NTMAX; ++n) {
    if (n >= nt) continue;
    const int a = ta[n], b = tbk[n];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int t = 16 * a + g + 8 * hr;
        const int i0 = 16 * b + 8 * j + 2 * tq;
        float v0 = acc[n][j][2 * hr], v1 = acc[n][j][2 * hr + 1];
        if (is_qk) {
          if (a == b) {
            v0 = (i0 <= t) ? v0 : 0.f;
            v1 = (i0 + 1 <= t) ? v1 : 0.f;
          }
          *reinterpret_cast<uint32_t*>(sm + OFF_AQK + sw_e(t, i0, 8192)) = pack_bf16(v0, v1);
        } else {
          const float bt = beta_s[t];
          v0 = (a > b || i0 < t) ? v0 * bt : 0.f;
          v1 = (a > b || i0 + 1 < t) ? v1 * bt : 0.f;
          *reinterpret_cast<float2*>(sm + OFF_AKK + (t * 64 + i0) * 4) = make_float2(v0, v1);
        }
      }
  }
}

__global__ void __launch_bounds__(NTHREADS, 1) chunk_prefill_kernel(ScanParams p) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int quad = warp & 3, half = warp >> 2;   // TMEM lane quadrant, column half (epilogues)
  const int trow = 32 * quad + lane;             // the TMEM lane this thread moves

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
  const uint32_t bar = sb + OFF_BAR;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 8);

  // decay-pass ownership: channel pair (c0, c0+1) of block da
  const int c0 = 2 * (tid & 63), da = tid >> 6;

  Prefetch pf;
  if (n_chunks > 0) {
    const int nv0 = (int)min((int64_t)C, t1 - t0);
    load_vb(x, sb + OFF_V, sb + OFF_BETA, t0, nv0, tid);
    cp_async_commit();
    load_qkg(x, t0, nv0, c0, da, pf);
  }

  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(TM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tlane = tmem + ((uint32_t)(32 * quad) << 16);  // this warp's TMEM lane quadrant

  // Initial state: TMEM lane v = trow holds column v of S; this thread moves columns [64*half, +64).
  const size_t sbase = ((size_t)n * p.H + h) * (size_t)KD * p.V + (size_t)vt * VT;
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    const int cb = 64 * half + 32 * part;
    uint32_t r[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      r[j] = __float_as_uint(p.s0 ? p.s0[sbase + (size_t)(cb + j) * p.V + trow] : 0.f);
    tm_st32(tlane + TM_S + cb, r);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4*>(sm + OFF_S + sw_chunk(trow, (cb >> 3) + j, 16384)) = pack8(r, j, 1.f);
  }
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");

  uint32_t phase = 0;
  bool ok = true;

  for (int c = 0; c < n_chunks && ok; ++c) {
    const int64_t tc0 = t0 + (int64_t)c * C;
    const int nv = (int)min((int64_t)C, t1 - tc0);
    const bool has_next = c + 1 < n_chunks;
    const int64_t tn0 = tc0 + C;
    const int nvn = has_next ? (int)min((int64_t)C, t1 - tn0) : 0;
    const uint32_t vbuf = sb + OFF_V + (c & 1) * 16384;
    const float* beta_s = reinterpret_cast<const float*>(sm + OFF_BETA + (c & 1) * 256);

    cp_async_wait_all();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();  // v tile and beta of chunk c landed; the previous chunk is fully retired
    tc_fence_after();
    if (has_next) load_vb(x, sb + OFF_V + ((c + 1) & 1) * 16384, sb + OFF_BETA + ((c + 1) & 1) * 256, tn0, nvn, tid);
    cp_async_commit();

    // ---- decay pass, step 1: per-token log2-decay, retention and block sum for (c0, c0+1) ------
    float2 al[16];  // retention factors of this thread's 16 tokens (1 past the end of a sequence)
    {
      float2 run = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float2 l = make_float2(0.f, 0.f);
        if (16 * da + i < nv) {
          l.x = fmaxf(p.gate_log ? pf.g[i].x * LOG2E : lg2(pf.g[i].x), G2_MIN);
          l.y = fmaxf(p.gate_log ? pf.g[i].y * LOG2E : lg2(pf.g[i].y), G2_MIN);
        }
        run.x += l.x;
        run.y += l.y;
        al[i] = make_float2(ex2(l.x), ex2(l.y));
      }
      *reinterpret_cast<float2*>(vec + VEC_TOT + da * 128 + c0) = run;
    }
    __syncthreads();
    // ---- step 2: decay factors, scaled operand tiles, per-pair and per-chunk vectors ------------
    {
      float2 e[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) e[b] = *reinterpret_cast<const float2*>(vec + VEC_TOT + b * 128 + c0);
#pragma unroll
      for (int b = 1; b < 4; ++b) {
        e[b].x += e[b - 1].x;
        e[b].y += e[b - 1].y;
      }
      // e[b] = log2 Gamma at r_b; log2 Gamma at s_a is e[a-1] (0 for a = 0)
      const float2 gs = da == 0 ? make_float2(0.f, 0.f) : (da == 1 ? e[0] : (da == 2 ? e[1] : e[2]));
      const float2 eda = da == 0 ? e[0] : (da == 1 ? e[1] : (da == 2 ? e[2] : e[3]));
      __nv_bfloat16* D16 = reinterpret_cast<__nv_bfloat16*>(vec + VEC_D);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (b <= da) {
          const int pair = da * (da + 1) / 2 + b;
          *reinterpret_cast<uint32_t*>(D16 + pair * 128 + c0) = pack_bf16(ex2(gs.x - e[b].x), ex2(gs.y - e[b].y));
        }
      }
      if (da == 0) *reinterpret_cast<float2*>(vec + VEC_GAM + c0) = make_float2(ex2(e[3].x), ex2(e[3].y));
      const float2 GS = make_float2(ex2(gs.x), ex2(gs.y));
      const float2 PM = make_float2(ex2(e[3].x - eda.x), ex2(e[3].y - eda.y));
      // F_t = prod_{r > t in block} alpha_r (reverse running product), E_t = prod_{r <= t} alpha_r.
      float2 F[16];
      F[15] = make_float2(1.f, 1.f);
#pragma unroll
      for (int i = 14; i >= 0; --i) F[i] = make_float2(F[i + 1].x * al[i + 1].x, F[i + 1].y * al[i + 1].y);
      float2 E = make_float2(1.f, 1.f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 16 * da + i;
        E.x *= al[i].x;
        E.y *= al[i].y;
        const float2 qf = unpack_bf16(pf.q[i]), kf = unpack_bf16(pf.k[i]);
        const uint32_t off = sw_e(t, c0, 8192);
        const float qex = qf.x * E.x, qey = qf.y * E.y, kex = kf.x * E.x, key = kf.y * E.y;
        const float kfx = kf.x * F[i].x, kfy = kf.y * F[i].y;
        *reinterpret_cast<uint32_t*>(sm + OFF_QE + off) = pack_bf16(qex, qey);
        *reinterpret_cast<uint32_t*>(sm + OFF_KE + off) = pack_bf16(kex, key);
        *reinterpret_cast<uint32_t*>(sm + OFF_KC + off) = pack_bf16(kfx, kfy);
        *reinterpret_cast<uint32_t*>(sm + OFF_QG + off) = pack_bf16(qex * GS.x, qey * GS.y);
        *reinterpret_cast<uint32_t*>(sm + OFF_KG + off) = pack_bf16(kex * GS.x, key * GS.y);
        *reinterpret_cast<uint32_t*>(sm + OFF_KT + off) = pack_bf16(kfx * PM.x, kfy * PM.y);
      }
    }
    __syncthreads();  // scaled tiles and vectors ready; the q/k/g registers are free

    if (has_next) load_qkg(x, tn0, nvn, c0, da, pf);

    // ---- A_kk on all warps (block pairs (a, b), a >= b), then the inverse on warps 0-3 while
    //      warps 4-7 form A_qk --------------------------------------------------------------------
    {
      const int nt = warp < 2 ? 2 : 1;
      a_tiles<2>(sm, sb, vec, OFF_KE, warp, 8, nt, lane, g, tq, beta_s, /*is_qk=*/false);
    }
    __syncthreads();  // A_kk ready; Ke is dead

    if (warp < 4) {
      // T' = (I + A_kk)^-1 Diag(beta): the four 16x16 diagonal inverses by forward substitution in
      // fp32, then the blocks below the diagonal by distance d = 1, 2, 3 as tensor-core products
      // T_ab = -sum_{j=b}^{a-1} (T_aa L_aj) T_jb. A bf16 copy of T (second half of the Ke tile)
      // feeds the products; T' (first half of the Ke tile) is written from the fp32 values.
      const float* L = reinterpret_cast<const float*>(sm + OFF_AKK);
      const uint32_t tb = sb + OFF_TB;
      if (tid < 64) {
        const int a = tid >> 4, j = tid & 15;
        float xs[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) xs[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l)
#pragma unroll
          for (int i = l + 1; i < 16; ++i) xs[i] -= L[(16 * a + i) * 64 + 16 * a + l] * xs[l];
        const float bj = beta_s[16 * a + j];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t off = sw_e(16 * a + i, 16 * a + j, 8192);
          *reinterpret_cast<__nv_bfloat16*>(sm + OFF_TB + off) = __float2bfloat16_rn(xs[i]);
          *reinterpret_cast<__nv_bfloat16*>(sm + OFF_TP + off) = __float2bfloat16_rn(xs[i] * bj);
        }
      } else {
        // T' is lower triangular: zero its six blocks above the diagonal.
        for (int e = tid - 64; e < 6 * 64; e += 64) {
          const int pr = e >> 6, r = (e >> 2) & 15, q4 = e & 3;
          const int a = pr < 3 ? 0 : (pr < 5 ? 1 : 2);
          const int b = pr < 3 ? pr + 1 : (pr < 5 ? pr - 1 : 3);
          *reinterpret_cast<uint2*>(sm + OFF_TP + sw_e(16 * a + r, 16 * b + 4 * q4, 8192)) = make_uint2(0u, 0u);
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll 1
      for (int d = 1; d <= 3; ++d) {
        if (warp < 4 - d) {
          const int b = warp, a = b + d;
          float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          uint32_t t0, t1, t2, t3;  // A fragments of T_aa
          ldsm_x4(tb + sw_chunk(16 * a + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * a + (lane >> 4), 8192), t0, t1, t2, t3);
          for (int jb = b; jb < a; ++jb) {
            float P[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int j = 0; j < 2; ++j) {  // P = T_aa L_{a,jb}; B[k][n] = L[16a + k][16jb + n]
              const float* lp = L + (16 * a + 2 * tq) * 64 + 16 * jb + 8 * j + g;
              mma_bf16(P[j], t0, t1, t2, t3, pack_bf16(lp[0], lp[64]), pack_bf16(lp[8 * 64], lp[9 * 64]));
            }
            uint32_t b0, b1, b2, b3;  // B = T_{jb,b}
            ldsm_x4_t(tb + sw_chunk(16 * jb + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * b + (lane >> 4), 8192), b0, b1, b2, b3);
            const uint32_t p0 = pack_bf16(P[0][0], P[0][1]), p1 = pack_bf16(P[0][2], P[0][3]);
            const uint32_t p2 = pack_bf16(P[1][0], P[1][1]), p3 = pack_bf16(P[1][2], P[1][3]);
            mma_bf16(acc[0], p0, p1, p2, p3, b0, b1);
            mma_bf16(acc[1], p0, p1, p2, p3, b2, b3);
          }
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
              const int row = 16 * a + g + 8 * hr, col = 16 * b + 8 * j + 2 * tq;
              const float v0 = -acc[j][2 * hr], v1 = -acc[j][2 * hr + 1];
              const uint32_t off = sw_e(row, col, 8192);
              *reinterpret_cast<uint32_t*>(sm + OFF_TB + off) = pack_bf16(v0, v1);
              *reinterpret_cast<uint32_t*>(sm + OFF_TP + off) = pack_bf16(v0 * beta_s[col], v1 * beta_s[col + 1]);
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
    } else {
      a_tiles<3>(sm, sb, vec, OFF_QE, warp - 4, 4, (warp - 4) < 2 ? 3 : 2, lane, g, tq, beta_s, /*is_qk=*/true);
      // The MMA reads whole rows of A_qk: zero its six blocks above the diagonal.
      for (int e = tid - 128; e < 6 * 64; e += 128) {
        const int pr = e >> 6, r = (e >> 2) & 15, q4 = e & 3;  // block pair, row, group of 4 columns
        const int a = pr < 3 ? 0 : (pr < 5 ? 1 : 2);
        const int b = pr < 3 ? pr + 1 : (pr < 5 ? pr - 1 : 3);
        *reinterpret_cast<uint2*>(sm + OFF_AQK + sw_e(16 * a + r, 16 * b + 4 * q4, 8192)) = make_uint2(0u, 0u);
      }
    }
    fence_async_smem();
    __syncthreads();  // every operand of MMA group 1 is in shared memory

    // ---- MMA group 1: W^T, U^T = V^T T'^T, O^T = S^T (Q*Gamma)^T --------------------------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id_w = idesc_bf16(64, 1, 0);   // A MN-major, B K-major, N = 64
      constexpr uint32_t id_o = idesc_bf16(64, 0, 0);   // A K-major, B K-major, N = 64
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t bt = sdesc(sb + OFF_TP + ks * 32, 16, 1024);
        tc_mma(tmem + TM_W, sdesc(sb + OFF_KG + ks * 2048, 8192, 1024), bt, id_w, ks > 0);
        tc_mma(tmem + TM_U, sdesc(vbuf + ks * 2048, 8192, 1024), bt, id_w, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc_mma(tmem + TM_O, sdesc(sb + OFF_S + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
               sdesc(sb + OFF_QG + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id_o, ks > 0);
      tc_commit(bar);
    }
    ok = __syncthreads_and(mbar_wait(bar, phase));  // one decision for the whole CTA
    phase ^= 1;
    tc_fence_after();
    if (!ok) break;

    // ---- epilogue 1: -W to shared memory (MN-major B, row c holds W[0..63][c]) ---------------------
    {
      uint32_t r[32];
      tm_ld32(tlane + TM_W + 32 * half, r);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(sm + OFF_QG + sw_chunk(trow, 4 * half + j, 0)) = pack8(r, j, -1.f);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- MMA group 2: U^T += S^T (-W)^T; meanwhile S^T *= gamma_C in TMEM (group 2 reads the bf16
    //      copy of S, not TMEM) --------------------------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id_u = idesc_bf16(64, 0, 1);   // A K-major, B MN-major, N = 64
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc_mma(tmem + TM_U, sdesc(sb + OFF_S + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
               sdesc(sb + OFF_QG + ks * 2048, 8192, 1024), id_u, 1);
      tc_commit(bar);
    }
    {
      uint32_t r[32];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const int cb = 64 * half + 32 * part;
        tm_ld32(tlane + TM_S + cb, r);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 gm = *reinterpret_cast<const float4*>(vec + VEC_GAM + cb + 4 * j);
          r[4 * j + 0] = __float_as_uint(__uint_as_float(r[4 * j + 0]) * gm.x);
          r[4 * j + 1] = __float_as_uint(__uint_as_float(r[4 * j + 1]) * gm.y);
          r[4 * j + 2] = __float_as_uint(__uint_as_float(r[4 * j + 2]) * gm.z);
          r[4 * j + 3] = __float_as_uint(__uint_as_float(r[4 * j + 3]) * gm.w);
        }
        tm_st32(tlane + TM_S + cb, r);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    ok = __syncthreads_and(mbar_wait(bar, phase));  // one decision for the whole CTA
    phase ^= 1;
    tc_fence_after();
    if (!ok) break;

    // ---- epilogue 2: U to shared memory (K-major A, row v holds U[0..63][v]) ---------------------
    {
      uint32_t r[32];
      tm_ld32(tlane + TM_U + 32 * half, r);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(sm + OFF_KG + sw_chunk(trow, 4 * half + j, 0)) = pack8(r, j, 1.f);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- MMA group 3: O^T += U^T A_qk^T, S^T += U^T (K*gamma_C/Gamma) ----------------------------
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id_o = idesc_bf16(64, 0, 0);    // A K-major, B K-major, N = 64
      constexpr uint32_t id_s = idesc_bf16(128, 0, 1);   // A K-major, B MN-major, N = 128
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t au = sdesc(sb + OFF_KG + ks * 32, 16, 1024);
        tc_mma(tmem + TM_O, au, sdesc(sb + OFF_AQK + ks * 32, 16, 1024), id_o, 1);
        tc_mma(tmem + TM_S, au, sdesc(sb + OFF_KT + ks * 2048, 8192, 1024), id_s, 1);
      }
      tc_commit(bar);
    }
    ok = __syncthreads_and(mbar_wait(bar, phase));  // one decision for the whole CTA
    phase ^= 1;
    tc_fence_after();
    if (!ok) break;

    // ---- epilogue 3: O to global memory, S to its bf16 copy --------------------------------------
    {
      uint32_t r[32];
      tm_ld32(tlane + TM_O + 32 * half, r);
      const int64_t ost = p.os[1];
      __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.o) + brow * p.os[0] + h * p.os[2] + (int64_t)vt * VT + trow +
                          (tc0 + 32 * half) * ost;
      const int jmax = min(32, nv - 32 * half);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < jmax) *op = __float2bfloat16_rn(__uint_as_float(r[j]));
        op += ost;
      }
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const int cb = 64 * half + 32 * part;
        tm_ld32(tlane + TM_S + cb, r);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(sm + OFF_S + sw_chunk(trow, (cb >> 3) + j, 16384)) = pack8(r, j, 1.f);
      }
    }
    // (the barrier at the top of the next iteration orders these writes before their readers)
  }
  cp_async_wait_all();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (ok && p.sf) {
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int cb = 64 * half + 32 * part;
      uint32_t r[32];
      tm_ld32(tlane + TM_S + cb, r);
#pragma unroll
      for (int j = 0; j < 32; ++j) p.sf[sbase + (size_t)(cb + j) * p.V + trow] = __uint_as_float(r[j]);
    }
  }
  if (!ok) {
    // A wait expired: give any MMA still in flight one more bounded wait before releasing TMEM.
    mbar_wait(bar, phase);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TM_COLS));
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

cudaError_t chunk_read_timeout(int* flag, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_chunk_timeout, sizeof(int));
  if (e != cudaSuccess || !reset) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_chunk_timeout, &zero, sizeof(int));
}

}  // namespace kda
