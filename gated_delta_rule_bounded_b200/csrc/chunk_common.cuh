// chunk_common.cuh -- pieces shared by the chunked prefill kernels: PTX helpers for
// tcgen05/TMEM, ldmatrix/mma.sync and cp.async, the per-chunk decay pass, the 16x16
// A_qk / A_kk block pairs and the 64x64 triangular inverse. The math they implement is
// the chunkwise form of the "KDA cheat sheet" (eqs. 3-4) with the UT transform derived
// from eq. 1 of "Kimi K3: Bounded Decay and Delta Memory"; see chunk.cu for the notation.
#pragma once

#include "common.cuh"
#include "gate_math.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int C = 64;     // tokens per chunk
constexpr int KD = 128;   // key dim
constexpr int VT = 128;   // value columns per state tile
constexpr int NTHREADS = 256;
constexpr float LOG2E = 1.4426950408889634f;
// Range of the block-boundary factorisation. A per-token log2-decay below L2_FLOOR (alpha = 0 included) is
// raised to it: alpha < 2^-126 and alpha = 0 differ by less than fp32 resolves next to any other term. A
// 16-token block whose log2-decay sum on some channel is below BLOCK_SAFE would need a diagonal pair factor
// above 2^120; such blocks take the pairwise diagonal path (diag_pairwise) instead. A per-token bound of
// g >= -5 (the bounded gate at g_min = -5) keeps every block sum >= -115.4 in log2, inside the range.
constexpr float L2_FLOOR = -126.f;
constexpr float BLOCK_SAFE = -120.f;

// fp32 vector area written by the decay pass (offsets in floats).
constexpr int VEC_D = 0;          // [10][128] bf16 exp(G_{s_a} - G_{r_b}), pairs a >= b (640 floats)
constexpr int VEC_GAM = 640;      // [128]     gamma_C
constexpr int VEC_TOT = 768;      // [4][128]  per-block log2-decay sums
constexpr int VEC_FLAG = 1280;    // [8] int   per warp: one of its channels' block sums is below BLOCK_SAFE
constexpr int VEC_FLOATS = 1288;

// Shared-memory offsets (bytes) of the tiles the state-independent phases use. Every bf16
// tile has 128-byte rows with the 128-byte swizzle; 128-column tiles are two 8 KB atoms.
struct IntraLayout {
  int qe, ke, kc;   // row operands of A_qk / A_kk and the column operand, [t][c]
  int qg, kg, kt;   // Q*Gamma, K*Gamma, K*gamma_C/Gamma, [t][c]
  int akk;          // A_kk, fp32 [64][64]
  int aqk;          // A_qk, bf16 [t][i] (K-major operand)
  int tp, tb;       // T' = T Diag(beta) (K-major operand) and a bf16 copy of T, [t][i]
  int vec;          // fp32 vectors (VEC_*)
};

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

// Two fp32 lanes in one 64-bit register pair, and the packed fp32x2 product (two correctly rounded products,
// the same values as two scalar multiplies, in one instruction).
__device__ __forceinline__ uint64_t f2_bits(float2 v) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
  return r;
}
__device__ __forceinline__ float2 bits_f2(uint64_t r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
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
// The same MMA with A (K-major, M = 128 rows on the 128 lanes, two bf16 per 32-bit column) read from
// tensor memory at `a_tmem` instead of shared memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
               "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
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
__device__ __forceinline__ void tm_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tm_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

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
__device__ __forceinline__ void tm_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* timeout_flag) {
  if (mbar_try_wait_bounded(bar, parity)) return true;
  atomicExch(timeout_flag, 1);
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
// Inputs
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

// The logits' bias of channels (c0, c0 + 1) of head h, or zeros.
__device__ __forceinline__ float2 load_bias2(const ScanParams& p, int h, int c0) {
  if (!p.dt_bias || p.gate_mode < GATE_LOGITS) return make_float2(0.f, 0.f);
  return __ldg(reinterpret_cast<const float2*>(p.dt_bias + (size_t)h * KD + c0));
}

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

// v tile of a chunk into the MN-major operand layout ([i][v], two 64-column halves).
__device__ __forceinline__ void load_v(const ChunkCtx& x, uint32_t vbase, int64_t tc0, int nv, int tid) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid + NTHREADS * i;
    const int row = idx >> 4, piece = idx & 15;
    const bool ok = row < nv;
    const int64_t t = tc0 + (ok ? row : 0);
    cp_async16(vbase + (piece >> 3) * 8192 + row * 128 + (((piece & 7) ^ (row & 7)) << 4),
               x.v + x.vrow + t * x.vst + piece * 8, ok);
  }
}

// v tile and beta of a chunk.
__device__ __forceinline__ void load_vb(const ChunkCtx& x, uint32_t vbase, uint32_t bbase, int64_t tc0, int nv,
                                        int tid) {
  load_v(x, vbase, tc0, nv, tid);
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
// fp32 [64][64] with beta_t applied and diagonal blocks masked to i < t. The diagonal blocks of the
// blocks set in `pairwise` (bit a: block a) are not stored: diag_pairwise has written them.
template <int NTMAX>
__device__ __forceinline__ void a_tiles(unsigned char* sm, uint32_t sb, const IntraLayout& L, int off_rows, int first,
                                        int stride, int nt, int lane, int g, int tq, const float* beta_s,
                                        bool is_qk, int pairwise) {
  const float* vec = reinterpret_cast<const float*>(sm + L.vec);
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
        ldsm_x4(sb + L.kc + sw_chunk(rb, 2 * kk + ((lane >> 3) & 1), 8192), b0, b1, b2, b3);
        mma_bf16(acc[n][0], a0, a1, a2, a3, b0, b1);
        mma_bf16(acc[n][1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NTMAX; ++n) {
    if (n >= nt) continue;
    const int a = ta[n], b = tbk[n];
    if (a == b && ((pairwise >> a) & 1)) continue;
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
          *reinterpret_cast<uint32_t*>(sm + L.aqk + sw_e(t, i0, 8192)) = pack_bf16(v0, v1);
        } else {
          const float bt = beta_s[t];
          v0 = (a > b || i0 < t) ? v0 * bt : 0.f;
          v1 = (a > b || i0 + 1 < t) ? v1 * bt : 0.f;
          *reinterpret_cast<float2*>(sm + L.akk + (t * 64 + i0) * 4) = make_float2(v0, v1);
        }
      }
  }
}


// L2-normalises, in place, the q and k values a decay-pass thread holds (channels c0, c0+1 of the 16
// tokens of block da; warps 2da and 2da+1 hold the two halves of each token row) over all K = 128
// channels, rounding the results back to bf16. Each warp sums its half-rows by a reduce-scatter (lane
// L ends with token L/2), the two halves meet in `red` (256 floats), and one CTA barrier publishes them.
__device__ __forceinline__ void l2norm_qk(Prefetch& pf, float* red, int tid, int da) {
  const int lane = tid & 31, half = (tid >> 5) & 1;
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 x = unpack_bf16(which ? pf.k[i] : pf.q[i]);
      v[i] = x.x * x.x + x.y * x.y;
    }
#pragma unroll
    for (int step = 0; step < 4; ++step) {  // keep 8, 4, 2, 1 tokens
      const int w = 8 >> step, bit = 16 >> step;
      const bool up = (lane & bit) != 0;
#pragma unroll
      for (int j = 0; j < w; ++j) {
        const float send = up ? v[j] : v[j + w];
        const float recv = __shfl_xor_sync(0xffffffffu, send, bit);
        v[j] = (up ? v[j + w] : v[j]) + recv;
      }
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    if ((lane & 1) == 0) red[which * 128 + (da * 2 + half) * 16 + (lane >> 1)] = v[0];
  }
  __syncthreads();
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const float* r0 = red + which * 128 + da * 32;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float sc = l2norm_scale(r0[i] + r0[16 + i]);
      uint32_t& w = which ? pf.k[i] : pf.q[i];
      const float2 x = unpack_bf16(w);
      w = pack_bf16(x.x * sc, x.y * sc);
    }
  }
}

// The log2-decay of one channel from the gate value x in gate mode `mode` (alpha, g = log alpha, the
// bounded gate's logits z, or the unbounded gate's logits, both with sc = e^{A_h}), raised to L2_FLOOR.
__device__ __forceinline__ float log2_decay(int mode, float x, float sc, float g_min) {
  float l;
  if (mode == GATE_LOGITS)
    l = bounded_log_decay(sc, x, g_min) * LOG2E;
  else if (mode == GATE_SOFTPLUS)
    l = softplus_log_decay(sc, x) * LOG2E;
  else
    l = mode == KDA_GATE_LOG ? x * LOG2E : lg2(x);
  return fmaxf(l, L2_FLOOR);  // fmaxf(-inf, floor) = floor: alpha = 0 stays finite in log space
}

// log2_decay of two channels. For the bounded gate's logits it evaluates bounded_log_decay (gate_math.cuh)
// with packed fp32x2 products and sums -- the same operations in the same order, so the same values.
template <int MODE>
__device__ __forceinline__ float2 log2_decay2(float2 x, float sc, float g_min) {
  if constexpr (MODE == GATE_LOGITS) {
    const float2 xs = mul2(make_float2(sc, sc), x);
    const float2 a = mul2(make_float2(fabsf(xs.x), fabsf(xs.y)), make_float2(-1.4426950408889634f, -1.4426950408889634f));
    float2 t, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(t.x) : "f"(a.x));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(t.y) : "f"(a.y));
    const float2 d = add2(make_float2(1.f, 1.f), t);
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.x) : "f"(d.x));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.y) : "f"(d.y));
    const float2 tr = mul2(t, r);
    const float2 sg = make_float2(xs.x >= 0.f ? r.x : tr.x, xs.y >= 0.f ? r.y : tr.y);
    const float2 l = mul2(mul2(make_float2(g_min, g_min), sg), make_float2(LOG2E, LOG2E));
    return make_float2(fmaxf(l.x, L2_FLOOR), fmaxf(l.y, L2_FLOOR));
  } else {
    return make_float2(log2_decay(MODE, x.x, sc, g_min), log2_decay(MODE, x.y, sc, g_min));
  }
}

// Decay pass, step 1: the per-token log2-decay of channels (c0, c0+1) over the 16 tokens of block
// da (0 past the end of the sequence), their retention factors, and the block sum, published to
// VEC_TOT. `bias` is the logits' per-channel bias (0 without one). Each warp also records in VEC_FLAG
// whether one of its channels' block sums lies below BLOCK_SAFE (read back by pairwise_blocks after
// the caller's barrier). MODE is the gate mode, fixed at compile time.
template <int MODE>
__device__ __forceinline__ void decay_step1_t(unsigned char* sm, const IntraLayout& L, const Prefetch& pf, int nv,
                                              int da, float sc, float g_min, float2 bias, float2 (&al)[16], int c0) {
  float* vec = reinterpret_cast<float*>(sm + L.vec);
  float2 run = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float2 l = make_float2(0.f, 0.f);
    if (16 * da + i < nv) {
      const float2 x = MODE >= GATE_LOGITS ? add2(pf.g[i], bias) : pf.g[i];
      l = log2_decay2<MODE>(x, sc, g_min);
    }
    run = add2(run, l);
    al[i] = make_float2(ex2(l.x), ex2(l.y));
  }
  *reinterpret_cast<float2*>(vec + VEC_TOT + da * 128 + c0) = run;
  const unsigned out_of_range = __any_sync(0xffffffffu, run.x < BLOCK_SAFE || run.y < BLOCK_SAFE);
  if ((threadIdx.x & 31) == 0) reinterpret_cast<int*>(vec + VEC_FLAG)[threadIdx.x >> 5] = out_of_range ? 1 : 0;
}

// decay_step1_t for a gate mode known only at run time.
__device__ __forceinline__ void decay_step1(unsigned char* sm, const IntraLayout& L, const Prefetch& pf, int nv,
                                            int da, int c0, int mode, float sc, float g_min, float2 bias,
                                            float2 (&al)[16]) {
  switch (mode) {
    case GATE_LOGITS: decay_step1_t<GATE_LOGITS>(sm, L, pf, nv, da, sc, g_min, bias, al, c0); break;
    case GATE_SOFTPLUS: decay_step1_t<GATE_SOFTPLUS>(sm, L, pf, nv, da, sc, g_min, bias, al, c0); break;
    case KDA_GATE_LOG: decay_step1_t<KDA_GATE_LOG>(sm, L, pf, nv, da, sc, g_min, bias, al, c0); break;
    default: decay_step1_t<KDA_GATE_ALPHA>(sm, L, pf, nv, da, sc, g_min, bias, al, c0); break;
  }
}

// After decay_step1 and a barrier: bit a set when block a needs its diagonal blocks pairwise (the
// two warps 2a, 2a + 1 own its channels).
__device__ __forceinline__ int pairwise_blocks(const unsigned char* sm, const IntraLayout& L) {
  const int* f = reinterpret_cast<const int*>(sm + L.vec) + VEC_FLAG;
  int m = 0;
#pragma unroll
  for (int a = 0; a < 4; ++a) m |= (f[2 * a] | f[2 * a + 1]) << a;
  return m;
}

// The diagonal 16x16 blocks of A_qk and A_kk of the blocks set in `pairwise`, pair by pair, without the
// block-boundary factorisation (whose diagonal factor 2^{-block sum} is out of range there):
//   A_qk[t][j] = sum_c q_tc k_jc w_tjc (j <= t),  A_kk[t][j] = beta_t sum_c k_tc k_jc w_tjc (j < t),
//   w_tjc = prod_{m = j+1..t} alpha_mc,
// each w built as a running product (every factor <= 1, so nothing overflows and a decay that underflows
// gives the right limit, 0). Run by all 256 threads after decay_step2 (a CTA-uniform call): the thread that
// owns channels (c0, c0 + 1) of block da forms its two channels' share of all 32 entries of each column j
// (16 of A_qk, 16 of A_kk), a reduce-scatter over the warp leaves lane l with entry l, and the two warps of
// the block meet through unused (off-diagonal) parts of the A_kk area, written over by a_tiles later. The
// results go straight to A_kk (fp32) and A_qk (bf16); a_tiles then skips these diagonal blocks.
__device__ __forceinline__ void diag_pairwise(unsigned char* sm, const IntraLayout& L, const Prefetch& pf,
                                              const float2 (&al)[16], const float* beta_s, int da, int pairwise) {
  const int lane = threadIdx.x & 31, hw = (threadIdx.x >> 5) & 1;  // the block's first or second warp
  const bool mine = (pairwise >> da) & 1;
  float* akk = reinterpret_cast<float*>(sm + L.akk);
  // A row of the A_kk area that holds warp 2da + 1's entries of column j: row 16da + j, the columns of
  // blocks da + 1 and da + 2 (mod 4), never a diagonal block.
  auto scratch = [&](int j, int l) { return akk + (16 * da + j) * 64 + 16 * ((da + 1 + (l >> 4)) & 3) + (l & 15); };
  float res[16];
  if (mine) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 kj = unpack_bf16(pf.k[j]);
      float v[32];
#pragma unroll
      for (int t = 0; t < 16; ++t) v[t] = v[16 + t] = 0.f;
      float2 w = make_float2(kj.x, kj.y);  // k_j * w_tj
#pragma unroll
      for (int t = j; t < 16; ++t) {
        if (t > j) {
          w.x *= al[t].x;
          w.y *= al[t].y;
        }
        const float2 qt = unpack_bf16(pf.q[t]), kt = unpack_bf16(pf.k[t]);
        v[t] = fmaf(qt.x, w.x, qt.y * w.y);
        v[16 + t] = fmaf(kt.x, w.x, kt.y * w.y);
      }
      // reduce-scatter: lane l ends with the warp's total of entry l
#pragma unroll
      for (int m = 16, nl = 32; m >= 1; m >>= 1, nl >>= 1) {
        const bool up = (lane & m) != 0;
        const int hn = nl / 2;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (i < hn) {
            const float send = up ? v[i] : v[i + hn];
            const float keep = up ? v[i + hn] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
          }
        }
      }
      res[j] = v[0];
      if (hw) *scratch(j, lane) = v[0];
    }
  }
  __syncthreads();
  if (mine && !hw) {
    const int t = lane & 15;
    const float bt = beta_s[16 * da + t];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float sum = res[j] + *scratch(j, lane);
      if (lane < 16) {
        *reinterpret_cast<__nv_bfloat16*>(sm + L.aqk + sw_e(16 * da + t, 16 * da + j, 8192)) =
            __float2bfloat16_rn(t >= j ? sum : 0.f);
      } else {
        akk[(16 * da + t) * 64 + 16 * da + j] = t > j ? sum * bt : 0.f;
      }
    }
  }
  // The next barrier (the caller's) orders these writes before a_tiles and the inverse.
}

// Decay pass, step 2 (after a barrier): block-boundary decay vectors and the six scaled tiles
// Qe = q E, Ke = k E, Kc = k F, QG = q E GS, KG = k E GS, Kt = k F PM of this thread's elements,
// with E_t = exp(G_t - G_{s_a}), F_t = exp(G_{r_a} - G_t), GS = exp(G_{s_a}), PM = exp(G_C - G_{r_a}).
__device__ __forceinline__ void decay_step2(unsigned char* sm, const IntraLayout& L, const Prefetch& pf, int da,
                                            int c0, const float2 (&al)[16]) {
  float* vec = reinterpret_cast<float*>(sm + L.vec);
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
    *reinterpret_cast<uint32_t*>(sm + L.qe + off) = pack_bf16(qex, qey);
    *reinterpret_cast<uint32_t*>(sm + L.ke + off) = pack_bf16(kex, key);
    *reinterpret_cast<uint32_t*>(sm + L.kc + off) = pack_bf16(kfx, kfy);
    *reinterpret_cast<uint32_t*>(sm + L.qg + off) = pack_bf16(qex * GS.x, qey * GS.y);
    *reinterpret_cast<uint32_t*>(sm + L.kg + off) = pack_bf16(kex * GS.x, key * GS.y);
    *reinterpret_cast<uint32_t*>(sm + L.kt + off) = pack_bf16(kfx * PM.x, kfy * PM.y);
  }
}

// Zeroes the six 16x16 blocks above the diagonal of a [64][64] bf16 K-major tile, using the `count`
// threads with index `idx` in [0, count).
__device__ __forceinline__ void zero_upper_blocks(unsigned char* sm, int off, int idx, int count) {
  for (int e = idx; e < 6 * 64; e += count) {
    const int pr = e >> 6, r = (e >> 2) & 15, q4 = e & 3;  // block pair, row, group of 4 columns
    const int a = pr < 3 ? 0 : (pr < 5 ? 1 : 2);
    const int b = pr < 3 ? pr + 1 : (pr < 5 ? pr - 1 : 3);
    *reinterpret_cast<uint2*>(sm + off + sw_e(16 * a + r, 16 * b + 4 * q4, 8192)) = make_uint2(0u, 0u);
  }
}

// T' = (I + A_kk)^-1 Diag(beta), run by warps 0-3 (128 threads, named barrier 1): the four 16x16
// diagonal inverses by forward substitution in fp32, then the blocks below the diagonal by distance
// d = 1, 2, 3 as tensor-core products T_ab = -sum_{j=b}^{a-1} (T_aa L_aj) T_jb, reading the bf16
// copy of T and writing T' from the fp32 values.
__device__ __forceinline__ void inverse_warps0to3(unsigned char* sm, uint32_t sb, const IntraLayout& Ly,
                                                  const float* beta_s, int tid, int warp, int lane, int g, int tq) {
  const float* L = reinterpret_cast<const float*>(sm + Ly.akk);
  const uint32_t tb = sb + Ly.tb;
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
      *reinterpret_cast<__nv_bfloat16*>(sm + Ly.tb + off) = __float2bfloat16_rn(xs[i]);
      *reinterpret_cast<__nv_bfloat16*>(sm + Ly.tp + off) = __float2bfloat16_rn(xs[i] * bj);
    }
  } else {
    zero_upper_blocks(sm, Ly.tp, tid - 64, 64);  // T' is lower triangular
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
          *reinterpret_cast<uint32_t*>(sm + Ly.tb + off) = pack_bf16(v0, v1);
          *reinterpret_cast<uint32_t*>(sm + Ly.tp + off) = pack_bf16(v0 * beta_s[col], v1 * beta_s[col + 1]);
        }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
}

// The state-independent phases after the decay pass: A_kk on all warps; then the inverse on warps
// 0-3 while warps 4-7 form A_qk (and zero its upper blocks). Diagonal blocks set in `pairwise` are the
// ones diag_pairwise wrote. Ends with a CTA barrier.
__device__ __forceinline__ void intra_phases(unsigned char* sm, uint32_t sb, const IntraLayout& L, const float* beta_s,
                                             int tid, int warp, int lane, int g, int tq, int pairwise) {
  a_tiles<2>(sm, sb, L, L.ke, warp, 8, warp < 2 ? 2 : 1, lane, g, tq, beta_s, /*is_qk=*/false, pairwise);
  __syncthreads();  // A_kk ready; Ke is dead
  if (warp < 4) {
    inverse_warps0to3(sm, sb, L, beta_s, tid, warp, lane, g, tq);
  } else {
    a_tiles<3>(sm, sb, L, L.qe, warp - 4, 4, (warp - 4) < 2 ? 3 : 2, lane, g, tq, beta_s, /*is_qk=*/true, pairwise);
    zero_upper_blocks(sm, L.aqk, tid - 128, 128);  // the MMAs read whole rows of A_qk
  }
  __syncthreads();
}

}  // namespace
}  // namespace kda
