// chunk_split.cu -- chunked prefill in two kernels: the state-independent work of every chunk in
// parallel (kernel P), then the state recurrence (kernel S).
//
// The per-chunk quantities of the chunkwise form that do not depend on the carried state --
// the decay factors, A_qk and A_kk, T' = (I + A_kk)^-1 Diag(beta), W = T' (K*Gamma), Q*Gamma and
// K*gamma_C/Gamma -- are most of the arithmetic. In the fused kernel (chunk.cu) they sit on the
// sequential path of one CTA per (sequence, head). Here kernel P computes them for all chunks of all
// heads at once -- a persistent grid of two CTAs per SM walking the (chunk, head) items -- and writes
// each chunk's operand set as one 66,048-byte block to a workspace: the block is the exact image of the
// shared-memory tiles (128-byte swizzle included), so kernel S moves it with bulk copies (in two parts,
// fetched ahead) into a 1 KB-aligned buffer and feeds it straight to tcgen05. Kernel S keeps one CTA per
// (sequence, head, V-tile) with the transposed state S^T in TMEM and, per chunk:
//   U^T = V^T T'^T (no state needed: runs while the state is converted to bf16 and rescaled)
//   group A:  [U^T | O^T] += S^T [-W ; Q*Gamma]^T  (one N = 128 product)
//   group B:  [O^T | S^T] += U^T [A_qk ; (K*gamma_C/Gamma)^T]^T  (one N = 192 product; S^T pre-scaled)
// and writes each full chunk's O with one TMA tensor store. One thread issues a tcgen05 MMA only every
// ~100-180 cycles, nearly whatever its N, so the products that share an A operand are fused along N. The fused accumulators must be adjacent in TMEM -- [U | O] for group A and
// [O | S] for group B -- so the O and U buffers alternate with the chunk's parity around the fixed
// S, and kernel P writes each block's operand pairs in the order that chunk's parity needs.
// The price of the split is the workspace traffic (one write and one read of ~1 KB per token-head).
//
// Decays steep enough to put a 16-token block outside the range of the block-boundary factorisation (any
// gate: alpha near 0, g_min below about -5.2, Kimi Linear's unbounded gate) are detected per block by the
// decay pass, and those blocks' diagonal 16x16 tiles are formed pair by pair instead (diag_pairwise in
// chunk_common.cuh); every other factor stays <= 1 for any decay.
//
// Workspace slots. Chunk j of sequence n has slot n * ceil(T/64) + j without cu_seqlens, and
// floor(cu[n]/64) + n + j with them (unique: a sequence's slots end before the next one's begin).
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "chunk_common.cuh"

namespace kda {

// Set to 1 by any CTA of the split kernels whose bounded wait expired.
__device__ int g_split_timeout = 0;

namespace {

// One workspace block = the output region of kernel P = the operand buffer of kernel S. A pair (X, Y)
// of operands sharing a product is stored in that order for an even chunk index j and as (Y, X) for an
// odd one.
constexpr int WB_WQ = 0;         // 32K  two k-atoms (c) of 128 rows: (-W [t][c], Q*Gamma [t][c])
constexpr int WB_KA = 32768;     // 24K  MN-major, three 8K n-atoms of 64 rows (the K index t or i):
                                 //      (A_qk^T [i][t'], K*gamma_C/Gamma [t][c 0..63], [t][c 64..127])
constexpr int WB_TP = 57344;     // 8K   T' [t][i]
constexpr int WB_GAM = 65536;    // 512  gamma_C, fp32 [128]
constexpr int WB_BYTES = 66048;

// Kernel P shared memory (111,968 bytes: two CTAs fit on an SM), in three overlapping phases.
//  Inputs (TMA): q, k as [64-channel half][64 tokens][128 B] and the gate input as [half][64 tokens][256 B].
//  Operands (written by the decay pass once every input is in registers): the row operand KQ, the column
//   views VIEW and K*Gamma, all 128-byte-swizzled K-major tiles of 128-byte rows, two 64-channel halves.
//  After the A products: A_kk (fp32), A_qk^T, T and T' over the dead KQ and VIEW rows, and -W.
constexpr int P_QS = 0;                     // 16K q staging
constexpr int P_KS = 16384;                 // 16K k staging
constexpr int P_GS = 32768;                 // 32K gate-input staging (fp32)
constexpr int P_KQ = 0;                     // 32K row operand: [half][128 rows][128 B]
constexpr int VIEW_ROWS = 176;              // views 3, 0, 2, 1 at rows 0, 64, 80, 144
constexpr int VIEW_HALF = VIEW_ROWS * 128;  // 22,528
constexpr int P_VIEW = 32768;               // 44K column views: [half][176 rows][128 B]
constexpr int P_KG = 81920;                 // 16K K*Gamma [half][64 rows][128 B] (4K after VIEW: the second
                                            //     A product reads 32 rows past the views' end)
constexpr int P_DIAG = 98304;               // 8K  pairwise diagonal blocks, fp32 [A_kk | A_qk][block][t][j]
constexpr int P_VEC = 106496;               // vectors (VEC_*)
constexpr int P_BETA = P_VEC + VEC_FLOATS * 4;  // 256 beta
constexpr int P_GAM = P_BETA + 256;         // 512 gamma_C (bulk-stored with T')
constexpr int P_BAR = P_GAM + 512;          // mbarriers (inputs, MMA) and the TMEM base
constexpr int P_SMEM = P_BAR + 64;
constexpr int P_AKK = 0;                    // 16K A_kk fp32 [t][i] (beta_t applied, strictly lower)
constexpr int P_AQKT = 16384;               // 8K  A_qk^T bf16 [i][t] (zero above the diagonal of A_qk)
constexpr int P_TB = 24576;                 // 8K  T bf16 [t][i]
constexpr int P_TP = P_VIEW + 8192;         // 8K  T' bf16 [t][i]; the W product (M = 128) also reads the
                                            //     next 8K, whose rows it discards
constexpr int P_W = P_VIEW + VIEW_HALF + 8192;  // 16K -W bf16 [half][64 rows][128 B]
static_assert(P_GS + 32768 <= P_KG && P_VIEW + 2 * VIEW_HALF + 32 * 128 <= P_KG, "staging and view overrun");
static_assert(P_TP + 16384 <= P_VIEW + VIEW_HALF + 8192 && P_W >= P_VIEW + VIEW_HALF + 8192 && P_W + 16384 <= P_KG,
              "post-product tiles must not overlap the K*gamma_C/Gamma rows still being stored");
static_assert(P_KG % 1024 == 0 && P_VIEW % 1024 == 0 && VIEW_HALF % 1024 == 0 && P_TP % 1024 == 0 &&
              P_W % 1024 == 0 && P_AQKT % 1024 == 0 && P_TB % 1024 == 0, "swizzle atoms need 1 KB alignment");
static_assert(2 * (P_SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
constexpr uint32_t P_TM_COLS = 256;         // TMEM: A products at columns 0 and 64, W at 128
// The view scales of view_expand take the VEC_D area of the vectors (fp32 [6][128]) in kernel P.
static_assert(VEC_TOT >= VEC_D + 6 * 128, "view scales fit before the block sums");

// Kernel S shared memory: the operand blocks of two chunks and their v tiles.
constexpr int S_OPS = 0;                    // 2 x operand block (66048 B, padded to 66560)
constexpr int S_OPS_STRIDE = 66560;
constexpr int S_V = 2 * S_OPS_STRIDE;       // 2 x 16K v tile [i][v], two halves (MN-major A)
constexpr int S_BAR = S_V + 2 * 16384;      // mbarriers: part 1 x2, part 2 x2, mma; TMEM base
constexpr int S_OST = S_BAR + 1024;          // 2 x 16K output staging [64 tokens][128 values] bf16 (TMA store)
constexpr int S_SMEM = S_OST + 2 * 16384;
static_assert(S_SMEM <= 227 * 1024, "shared memory budget");
static_assert(WB_KA % 16 == 0 && WB_TP % 16 == 0 && WB_BYTES % 16 == 0, "bulk copies move 16-byte multiples");
static_assert(S_V % 1024 == 0 && S_OPS_STRIDE % 1024 == 0 && S_OST % 1024 == 0, "1 KB alignment");

// Kernel S tensor memory (columns; lane = value column v of the tile). S^T, U^T and O^T in fp32 are
// MMA accumulators, laid out [U_e | O_e | S | O_o | U_o] so that [U | O] and [O | S] are adjacent for
// chunks of either parity (e: even chunk index, o: odd). The bf16 copies of S^T and U^T (two values
// per column) are the A operands of the next products.
constexpr uint32_t TM_UE = 0;     // 64   U^T fp32 [v][t], even chunks
constexpr uint32_t TM_OE = 64;    // 64   O^T fp32 [v][t], even chunks
constexpr uint32_t TM_S = 128;    // 128  S^T fp32 [v][c]
constexpr uint32_t TM_OO = 256;   // 64   O^T, odd chunks
constexpr uint32_t TM_UO = 320;   // 64   U^T, odd chunks
constexpr uint32_t TM_SB = 384;   // 64   S^T bf16 (K = c)
constexpr uint32_t TM_UB = 448;   // 32   U^T bf16 (K = t)
constexpr uint32_t TM_COLS = 512;

__device__ __forceinline__ void seq_range(const ScanParams& p, int n, int64_t& t0, int64_t& t1, int64_t& brow) {
  t0 = 0;
  t1 = p.T;
  brow = n;
  if (p.cu) {
    t1 = min((int64_t)p.cu[n + 1], p.T);
    t0 = max((int64_t)0, min((int64_t)p.cu[n], t1));
    brow = 0;
  }
}

__device__ __forceinline__ int64_t slot_base(const ScanParams& p, int n, int64_t t0) {
  return p.cu ? (t0 >> 6) + n : (int64_t)n * ((p.T + C - 1) / C);
}

// Kernel P: slot s -> (sequence, chunk). Without cu_seqlens the slots are dense; with them, the
// sequence is the last one whose base slot is <= s (base slots increase with n).
__device__ __forceinline__ bool locate_slot(const ScanParams& p, int64_t s, int& n_out, int& j_out) {
  if (!p.cu) {
    const int64_t ncps = (p.T + C - 1) / C;
    n_out = (int)(s / ncps);
    j_out = (int)(s % ncps);
    return n_out < p.N && (int64_t)j_out * C < p.T;
  }
  int lo = 0, hi = p.N - 1, n = -1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    int64_t t0, t1, br;
    seq_range(p, mid, t0, t1, br);
    if (slot_base(p, mid, t0) <= s) {
      n = mid;
      lo = mid + 1;
    } else {
      hi = mid - 1;
    }
  }
  if (n < 0) return false;
  int64_t t0, t1, br;
  seq_range(p, n, t0, t1, br);
  const int64_t j = s - slot_base(p, n, t0);
  if (j * C >= t1 - t0) return false;
  n_out = n;
  j_out = (int)j;
  return true;
}

__device__ __forceinline__ void bulk_store(unsigned char* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------------------------------------
// Kernel P: the state-independent operands of one (chunk, head), tcgen05 products fed by TMA.
//
// Decay ratios. With e[a] the log2-decay of the chunk up to the end of block a (e[-1] = 0) and G_t the
// running log2-decay at token t, the ratio 2^{G_t - G_i} (t in block a, i <= t) is split at a reference
// point R_a of block a: [x_t 2^{G_t - R_a}] [k_i 2^{R_a - G_i}]. R_a = e[a], the end of block a, puts
// every factor of the column operand at or below 1 (i <= r_a) and bounds the row factor by the block's
// own decay (at most 2^120 for blocks within range, the g_min argument of the "KDA cheat sheet"). For a
// block out of range R_a = e[a - 1], the start: the row factor is then <= 1, the cross-block column
// factors 2^{e[a-1] - G_i} stay <= 1, and only the block's own diagonal tile is lost -- that one is
// formed pair by pair (diag_pairwise) and substituted when A_kk and A_qk are read back.
//
// Products. View a of the column operand holds k_i 2^{R_a - G_i} for the tokens i <= r_a of blocks
// 0..a (view 3 with R_3 = e[3] is K*gamma_C/Gamma, an operand of kernel S as well). The row operand KQ
// holds k_t 2^{G_t - R_a} and q_t 2^{G_t - R_a} for every block a. Two M = 128, N = 64, K = 128 products
// give every pair: rows [view 3 | view 0] against [K_3 | Q_3 | K_0 | Q_0], and [view 2 | view 1] against
// [K_2 | Q_2 | K_1 | Q_1] (the cross terms between different blocks are computed and discarded), so the
// accumulator lane is the column index i of A and the accumulator column the row index t. W = T' (K*Gamma)
// is a third product (M = 128 with the upper 64 rows discarded, N = 128, K = 64).
// First row of view a (views 3, 0 form the first product's A operand, 2, 1 the second's), and of block a's
// k rows in KQ (its q rows follow at +16; blocks 3, 0 form the first product's B operand, 2, 1 the second's).
__device__ __forceinline__ int view_base(int a) { return a == 3 ? 0 : (a == 0 ? 64 : (a == 2 ? 80 : 144)); }
__device__ __forceinline__ int kq_base(int a) { return a == 3 ? 0 : (a == 0 ? 32 : (a == 2 ? 64 : 96)); }

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int x, int h, int t, int b,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(h), "r"(t), "r"(b), "r"(bar)
      : "memory");
}

// Tensor maps of the three token tensors kernel P reads: q and k (bf16 boxes of 64 channels x 64
// tokens) and the gate input (fp32, same boxes).
struct PMaps {
  CUtensorMap q, k, g;
};

// Decay pass, step 2 of kernel P: the row operand KQ, K*Gamma (smem), Q*Gamma (straight to its place in the
// workspace block, qg_dst: [t][c] rows of 16 KB k-atoms), gamma_C, and block da's own rows of view da,
// k_i 2^{e[da] - G_i}, from which view_expand derives the other views. When block 3 is out of range view 3 is
// not K*gamma_C/Gamma (its reference is then the block's start), which goes straight to the workspace too
// (kt_dst: [t][c] rows of 8 KB n-atoms).
__device__ __forceinline__ void p_operands(unsigned char* sm, const Prefetch& pf, int da, int c0, int pairwise,
                                           const float2 (&al)[16], unsigned char* qg_dst, unsigned char* kt_dst) {
  float* vec = reinterpret_cast<float*>(sm + P_VEC);
  float2 e[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) e[b] = *reinterpret_cast<const float2*>(vec + VEC_TOT + b * 128 + c0);
#pragma unroll
  for (int b = 1; b < 4; ++b) {
    e[b].x += e[b - 1].x;
    e[b].y += e[b - 1].y;
  }
  // e[b] = log2 Gamma at the end of block b; the start of block a is e[a-1] (0 for a = 0)
  float2 R[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const float2 st = a == 0 ? make_float2(0.f, 0.f) : e[a - 1];
    R[a] = ((pairwise >> a) & 1) ? st : e[a];
  }
  const float2 gs = da == 0 ? make_float2(0.f, 0.f) : (da == 1 ? e[0] : (da == 2 ? e[1] : e[2]));
  const float2 eda = da == 0 ? e[0] : (da == 1 ? e[1] : (da == 2 ? e[2] : e[3]));
  const float2 Rd = da == 0 ? R[0] : (da == 1 ? R[1] : (da == 2 ? R[2] : R[3]));
  if (da == 0) *reinterpret_cast<float2*>(sm + P_GAM + 4 * c0) = make_float2(ex2(e[3].x), ex2(e[3].y));
  // Scales 2^{R_a - e[da]} (<= 1) of this block's rows in the views a > da, for view_expand:
  // fp32 [pair][128] in the VEC_D area, pair (a, b) at a (a - 1) / 2 + b.
#pragma unroll
  for (int a = 1; a < 4; ++a)
    if (a > da)
      *reinterpret_cast<float2*>(vec + VEC_D + (a * (a - 1) / 2 + da) * 128 + c0) =
          make_float2(ex2(R[a].x - eda.x), ex2(R[a].y - eda.y));
  const float2 GS = make_float2(ex2(gs.x), ex2(gs.y));               // Gamma at the start of the block
  const float2 DI = make_float2(ex2(gs.x - Rd.x), ex2(gs.y - Rd.y)); // 2^{G_start - R_da} (>= 1)
  const int rk = kq_base(da);
  float2 E = make_float2(1.f, 1.f);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int t = 16 * da + i;
    E = mul2(E, al[i]);
    const float2 qf = unpack_bf16(pf.q[i]), kf = unpack_bf16(pf.k[i]);
    const float2 rr = mul2(E, DI);   // 2^{G_t - R_da}
    const float2 gg = mul2(E, GS);   // Gamma_t
    const float2 kr = mul2(kf, rr), qr = mul2(qf, rr), kg = mul2(kf, gg), qg = mul2(qf, gg);
    *reinterpret_cast<uint32_t*>(sm + P_KQ + sw_e(rk + i, c0, 16384)) = pack_bf16(kr.x, kr.y);
    *reinterpret_cast<uint32_t*>(sm + P_KQ + sw_e(rk + 16 + i, c0, 16384)) = pack_bf16(qr.x, qr.y);
    *reinterpret_cast<uint32_t*>(sm + P_KG + sw_e(t, c0, 8192)) = pack_bf16(kg.x, kg.y);
    *reinterpret_cast<uint32_t*>(qg_dst + sw_e(t, c0, 16384)) = pack_bf16(qg.x, qg.y);
  }
  const bool kt_apart = (pairwise >> 3) & 1;
  const float2 PM = make_float2(ex2(e[3].x - eda.x), ex2(e[3].y - eda.y));  // 2^{e[3] - e[da]}
  const int vrow = view_base(da) + 16 * da;
  float2 F = make_float2(1.f, 1.f);  // 2^{e[da] - G_i}, tokens after i within the block
#pragma unroll
  for (int i = 15; i >= 0; --i) {
    const float2 kx = mul2(unpack_bf16(pf.k[i]), F);
    // block da's rows of view da (for an out-of-range block they are its discarded diagonal tile, and the
    // source of its rows in the later views)
    *reinterpret_cast<uint32_t*>(sm + P_VIEW + sw_e(vrow + i, c0, VIEW_HALF)) = pack_bf16(kx.x, kx.y);
    if (kt_apart) {
      const float2 kt = mul2(kx, PM);
      *reinterpret_cast<uint32_t*>(kt_dst + sw_e(16 * da + i, c0, 8192)) = pack_bf16(kt.x, kt.y);
    }
    F = mul2(F, al[i]);
  }
}

// T' = (I + A_kk)^-1 Diag(beta) on all eight warps of kernel P. The four 16 x 16 diagonal inverses by forward
// substitution in fp32 (warps 0-1; warps 2-3 zero T' above the diagonal), then the blocks below the diagonal
// from the 2 x 2 split into 32 x 32 halves, (I + A)^-1 = [[T1, 0], [-T2 A21 T1, T2]]: level 1 the blocks
// (1,0) and (3,2) of T1 and T2, T_ab = -T_aa A_ab T_bb; level 2 Y = A21 T1 into a bf16 scratch tile
// [32][32]; level 3 the lower-left quadrant -T2 Y. Each warp of a level takes one 16 x 8 half of a block
// (mma.sync, bf16 operands, fp32 sums); T (bf16) is the operand of the later levels, T' the output.
__device__ __forceinline__ void p_inverse(unsigned char* sm, uint32_t sb, const IntraLayout& Ly, const float* beta_s,
                                          int tid, int warp, int lane, int g, int tq, uint32_t yscr) {
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
  } else if (tid < 128) {
    zero_upper_blocks(sm, Ly.tp, tid - 64, 64);  // T' is lower triangular
  }
  __syncthreads();
  const int jh = warp & 1;  // this warp's 8-column half of its block
  // the B fragment (16 x 8, this warp's half) of a 16 x 16 bf16 block of T at block row r, block column b
  auto t_bfrag = [&](int r, int b, uint32_t& b0, uint32_t& b1) {
    uint32_t x0, x1, x2, x3;
    ldsm_x4_t(tb + sw_chunk(16 * r + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * b + (lane >> 4), 8192), x0, x1, x2, x3);
    b0 = jh ? x2 : x0;
    b1 = jh ? x3 : x1;
  };
  // -acc to T and T' at block (a, b), this warp's half
  auto store_t = [&](int a, int b, const float (&acc)[4]) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = 16 * a + g + 8 * hr, col = 16 * b + 8 * jh + 2 * tq;
      const float v0 = -acc[2 * hr], v1 = -acc[2 * hr + 1];
      const uint32_t off = sw_e(row, col, 8192);
      *reinterpret_cast<uint32_t*>(sm + Ly.tb + off) = pack_bf16(v0, v1);
      *reinterpret_cast<uint32_t*>(sm + Ly.tp + off) = pack_bf16(v0 * beta_s[col], v1 * beta_s[col + 1]);
    }
  };
  if (warp < 4) {  // level 1: T_10 (warps 0, 1) and T_32 (warps 2, 3)
    const int a = warp < 2 ? 1 : 3, b = a - 1;
    uint32_t t0, t1, t2, t3;  // A fragments of T_aa
    ldsm_x4(tb + sw_chunk(16 * a + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * a + (lane >> 4), 8192), t0, t1, t2, t3);
    float P[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int j = 0; j < 2; ++j) {  // P = T_aa A_ab; B[k][n] = A[16a + k][16b + n]
      const float* lp = L + (16 * a + 2 * tq) * 64 + 16 * b + 8 * j + g;
      mma_bf16(P[j], t0, t1, t2, t3, pack_bf16(lp[0], lp[64]), pack_bf16(lp[8 * 64], lp[9 * 64]));
    }
    uint32_t b0, b1;
    t_bfrag(b, b, b0, b1);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    mma_bf16(acc, pack_bf16(P[0][0], P[0][1]), pack_bf16(P[0][2], P[0][3]), pack_bf16(P[1][0], P[1][1]),
             pack_bf16(P[1][2], P[1][3]), b0, b1);
    store_t(a, b, acc);
  }
  __syncthreads();
  const int a = 2 + (warp >> 2), b = (warp >> 1) & 1;  // levels 2 and 3: block (a, b) of the lower-left quadrant
  {  // level 2: Y_ab = sum_{j=b}^{1} A_aj T_jb
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j < b) continue;
      const float* la = L + (16 * a + g) * 64 + 16 * j + 2 * tq;
      uint32_t b0, b1;
      t_bfrag(j, b, b0, b1);
      mma_bf16(acc, pack_bf16(la[0], la[1]), pack_bf16(la[8 * 64], la[8 * 64 + 1]), pack_bf16(la[8], la[9]),
               pack_bf16(la[8 * 64 + 8], la[8 * 64 + 9]), b0, b1);
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = 16 * (a - 2) + g + 8 * hr, col = 16 * b + 8 * jh + 2 * tq;
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(yscr + row * 64 + col * 2), "r"(pack_bf16(acc[2 * hr], acc[2 * hr + 1]))
                   : "memory");
    }
  }
  __syncthreads();
  {  // level 3: T_ab = -sum_{j=2}^{a} T_aj Y_jb
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 2; j < 4; ++j) {
      if (j > a) continue;
      uint32_t t0, t1, t2, t3, x0, x1, x2, x3;
      ldsm_x4(tb + sw_chunk(16 * a + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * j + (lane >> 4), 8192), t0, t1, t2, t3);
      ldsm_x4_t(yscr + (16 * (j - 2) + (lane & 7) + ((lane >> 3) & 1) * 8) * 64 + (16 * b + 8 * (lane >> 4)) * 2, x0, x1,
                x2, x3);
      mma_bf16(acc, t0, t1, t2, t3, jh ? x2 : x0, jh ? x3 : x1);
    }
    store_t(a, b, acc);
  }
}

// After p_operands and a barrier: the rows of block b in view a > b, as block b's rows of view b times the
// scale 2^{R_a - e[b]} of each channel (six block pairs of 16 rows x 128 channels, one 8-channel 16-byte
// piece per thread and pair; fp32 products rounded once to bf16).
__device__ __forceinline__ void view_expand(unsigned char* sm, int tid) {
  const float* vec = reinterpret_cast<const float*>(sm + P_VEC);
#pragma unroll
  for (int p = 0; p < 6; ++p) {
    const int a = p == 0 ? 1 : (p < 3 ? 2 : 3);
    const int b = p - a * (a - 1) / 2;
    const int row = tid >> 4, j = tid & 15;  // 16 rows x 16 pieces
    const uint4 src = *reinterpret_cast<const uint4*>(sm + P_VIEW + sw_chunk(view_base(b) + 16 * b + row, j, VIEW_HALF));
    const float4 s0 = *reinterpret_cast<const float4*>(vec + VEC_D + p * 128 + 8 * j);
    const float4 s1 = *reinterpret_cast<const float4*>(vec + VEC_D + p * 128 + 8 * j + 4);
    const float2 y0 = mul2(unpack_bf16(src.x), make_float2(s0.x, s0.y));
    const float2 y1 = mul2(unpack_bf16(src.y), make_float2(s0.z, s0.w));
    const float2 y2 = mul2(unpack_bf16(src.z), make_float2(s1.x, s1.y));
    const float2 y3 = mul2(unpack_bf16(src.w), make_float2(s1.z, s1.w));
    const uint4 dst = make_uint4(pack_bf16(y0.x, y0.y), pack_bf16(y1.x, y1.y), pack_bf16(y2.x, y2.y),
                                 pack_bf16(y3.x, y3.y));
    *reinterpret_cast<uint4*>(sm + P_VIEW + sw_chunk(view_base(a) + 16 * b + row, j, VIEW_HALF)) = dst;
  }
}

// The diagonal 16x16 tiles of the out-of-range blocks (bit a of `pairwise`), pair by pair, from the values the
// decay pass left in the staging area: q and k (bf16, prepared) and alpha (fp32, in place of the gate input),
// zero q, k and alpha = 1 past the sequence's end. One warp per (block, column j): lane l takes channels
// 2l, 2l + 1 of each 64-channel half, forms its share of A_qk[t][j] = sum_c q_tc k_jc w_tjc (t >= j) and
// A_kk[t][j] = sum_c k_tc k_jc w_tjc (t > j), w_tjc = prod_{m=j+1..t} alpha_mc, for the 16 rows t of the block,
// and a reduce-scatter over the warp leaves lane l with entry l. Results go to `out` as fp32
// [A_kk | A_qk][block][t][j], A_kk with beta_t applied. Kept out of line so that its registers do not
// weigh on the kernel's main path, which never calls it for chunks within range.
__device__ __noinline__ void p_diag_pairwise(const unsigned char* sm, int pairwise, const float* beta_s, float* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int blocks[4], nb = 0;
  for (int a = 0; a < 4; ++a)
    if ((pairwise >> a) & 1) blocks[nb++] = a;
  for (int item = warp; item < 16 * nb; item += NTHREADS / 32) {
    const int a = blocks[item >> 4], j = item & 15;
    const int rj = 16 * a + j;
    float kj[4], w[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + P_KS + h * 8192 + rj * 128 + lane * 4));
      kj[2 * h] = kv.x;
      kj[2 * h + 1] = kv.y;
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) w[m] = kj[m];
    float v[32];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float sq = 0.f, sk = 0.f;
      if (t >= j) {
        const int rt = 16 * a + t;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + P_QS + h * 8192 + rt * 128 + lane * 4));
          const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + P_KS + h * 8192 + rt * 128 + lane * 4));
          if (t > j) {
            const float2 al = *reinterpret_cast<const float2*>(sm + P_GS + h * 16384 + rt * 256 + lane * 8);
            w[2 * h] *= al.x;
            w[2 * h + 1] *= al.y;
          }
          sq = fmaf(qv.x, w[2 * h], fmaf(qv.y, w[2 * h + 1], sq));
          sk = fmaf(kv.x, w[2 * h], fmaf(kv.y, w[2 * h + 1], sk));
        }
      }
      v[t] = sq;
      v[16 + t] = sk;
    }
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
    const int t = lane & 15;
    if (lane < 16)
      out[1024 + (a * 16 + t) * 16 + j] = t >= j ? v[0] : 0.f;
    else
      out[(a * 16 + t) * 16 + j] = t > j ? v[0] * beta_s[16 * a + t] : 0.f;
  }
}

template <int MODE>  // the gate mode of p (KDA_GATE_ALPHA, KDA_GATE_LOG, GATE_LOGITS, GATE_SOFTPLUS)
__global__ void __launch_bounds__(NTHREADS, 2) chunk_intra_kernel(ScanParams p, unsigned char* ws,
                                                                  const __grid_constant__ PMaps maps, int64_t n_slots) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  constexpr IntraLayout LY{-1, -1, -1, -1, -1, -1, P_AKK, -1, P_TP, P_TB, P_VEC};
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  // Kernel S may be scheduled once every CTA of this grid has started; it reads the workspace only
  // after this whole grid has completed (griddepcontrol.wait).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const uint32_t bar_in = sb + P_BAR, bar_mma = sb + P_BAR + 8;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + P_BAR + 16);
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_in));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_mma));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(P_TM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  float* beta_s = reinterpret_cast<float*>(sm + P_BETA);
  const int c0 = 2 * (tid & 63), da = tid >> 6;
  const int hc = c0 >> 6, cc = c0 & 63;

  // Persistent: the CTA takes items (chunk slot, head) blockIdx.x, + gridDim.x, ... in head-major order.
  // bar_in completes once per item (phase parity n_done & 1), bar_mma twice (parity 0, then 1).
  const int64_t n_items = n_slots * p.H;
  bool ok = true;
  int n_done = 0;      // items whose inputs were requested
  int mma_groups = 0;  // product groups of the current item committed to bar_mma (thread 0)
  for (int64_t item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
    const int h = (int)(item / n_slots);
    const int64_t slot = item - (int64_t)h * n_slots;
    int n, j;
    if (!locate_slot(p, slot, n, j)) continue;  // uniform across the CTA
    const float gsc = MODE >= GATE_LOGITS ? expf(__ldg(p.A_log + h)) : 0.f;  // e^{A_h}
    int64_t t0, t1, brow;
    seq_range(p, n, t0, t1, brow);
    const int64_t tc0 = t0 + (int64_t)j * C;
    const int nv = (int)min((int64_t)C, t1 - tc0);
    unsigned char* blk = ws + ((size_t)slot * p.H + h) * WB_BYTES;
    const bool even = (j & 1) == 0;  // operand order within the block's pairs
    if (tid == 0) {
      // q, k and the gate input of the chunk's 64 tokens (rows past the tensor's end read as zeros; rows past
      // the sequence's end are zeroed below); 64 KB on one barrier. The previous item's readers of this
      // shared memory are done (the barrier at the end of the item).
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_in), "r"(65536) : "memory");
      const int tt = (int)tc0, bb = (int)brow;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tma_load_4d(sb + P_QS + half * 8192, &maps.q, 64 * half, h, tt, bb, bar_in);
        tma_load_4d(sb + P_KS + half * 8192, &maps.k, 64 * half, h, tt, bb, bar_in);
        tma_load_4d(sb + P_GS + half * 16384, &maps.g, 64 * half, h, tt, bb, bar_in);
      }
    }
    if (tid < C) {
      beta_s[tid] = tid < nv ? beta_value(__ldg(p.beta + brow * p.bs[0] + h * p.bs[2] + (tc0 + tid) * p.bs[1]),
                                          p.beta_sigmoid)
                             : 0.f;
    }
    ok = __syncthreads_and(mbar_wait(bar_in, n_done & 1, &g_split_timeout));
    int pairwise = 0;
    mma_groups = 0;
    if (ok) {
      Prefetch pf;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 16 * da + i;
        const bool v = t < nv;
        pf.q[i] = v ? *reinterpret_cast<const uint32_t*>(sm + P_QS + hc * 8192 + t * 128 + cc * 2) : 0u;
        pf.k[i] = v ? *reinterpret_cast<const uint32_t*>(sm + P_KS + hc * 8192 + t * 128 + cc * 2) : 0u;
        pf.g[i] = v ? *reinterpret_cast<const float2*>(sm + P_GS + hc * 16384 + t * 256 + cc * 4) : make_float2(0.f, 0.f);
      }
      if (p.qk_l2norm) l2norm_qk(pf, reinterpret_cast<float*>(sm + P_VEC) + VEC_D, tid, da);
      float2 al[16];
      decay_step1_t<MODE>(sm, LY, pf, nv, da, gsc, p.g_min, load_bias2(p, h, c0), al, c0);
      __syncthreads();  // block sums and flags published; every input is in registers
      pairwise = pairwise_blocks(sm, LY);
      if (pairwise) {  // CTA-uniform; never taken within range
        if ((pairwise >> da) & 1) {
          // the prepared inputs of this out-of-range block back into the staging area, alpha over the gate input
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int t = 16 * da + i;
            *reinterpret_cast<uint32_t*>(sm + P_QS + hc * 8192 + t * 128 + cc * 2) = pf.q[i];
            *reinterpret_cast<uint32_t*>(sm + P_KS + hc * 8192 + t * 128 + cc * 2) = pf.k[i];
            *reinterpret_cast<float2*>(sm + P_GS + hc * 16384 + t * 256 + cc * 4) = al[i];
          }
        }
        __syncthreads();
        p_diag_pairwise(sm, pairwise, beta_s, reinterpret_cast<float*>(sm + P_DIAG));
        __syncthreads();  // the staging area is read; the operands overwrite it next
      }
      p_operands(sm, pf, da, c0, pairwise, al, blk + WB_WQ + (even ? 8192 : 0), blk + WB_KA + (even ? 8192 : 0));
      __syncthreads();  // every block's own view rows and the view scales
      view_expand(sm, tid);
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      // ---- the A products: [view 3 | view 0] x [K_3 | Q_3 | K_0 | Q_0], [view 2 | view 1] x [K_2 | Q_2 | K_1 | Q_1]
      if (tid == 0) {
        constexpr uint32_t id_a = idesc_bf16(64, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t kv = (ks >> 2) * VIEW_HALF + (ks & 3) * 32, kq = (ks >> 2) * 16384 + (ks & 3) * 32;
          tc_mma(tmem, sdesc(sb + P_VIEW + kv, 16, 1024), sdesc(sb + P_KQ + kq, 16, 1024), id_a, ks > 0);
          tc_mma(tmem + 64, sdesc(sb + P_VIEW + 80 * 128 + kv, 16, 1024), sdesc(sb + P_KQ + 64 * 128 + kq, 16, 1024),
                 id_a, ks > 0);
        }
        tc_commit(bar_mma);
        mma_groups = 1;
      }
      ok = __syncthreads_and(mbar_wait(bar_mma, 0, &g_split_timeout));
      tc_fence_after();
    }
    if (ok) {
      // K*gamma_C/Gamma (view 3) goes to the workspace as kernel S's MN-major operand rows [t][c] (when block 3
      // is out of range the decay pass has stored it already).
      if (tid == 0 && !((pairwise >> 3) & 1)) {
        const uint32_t kt = WB_KA + (even ? 8192 : 0);
        bulk_store(blk + kt, sb + P_VIEW, 8192);
        bulk_store(blk + kt + 8192, sb + P_VIEW + VIEW_HALF, 8192);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
      // ---- read back: warps 0-3 the first product, 4-7 the second; TMEM lane L = 32 (warp & 3) + lane is
      // column i = L & 63 of A in view 3 or 0 (first product) and 2 or 1 (second)
      {
        const int L = 32 * (warp & 3) + lane, second = warp >> 2;
        const int a = second ? (L < 64 ? 2 : 1) : (L < 64 ? 3 : 0);
        const int i = L & 63;
        uint32_t r[32];
        tm_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 64 * second + (L < 64 ? 0 : 32), r);
        const bool from_pairs = ((pairwise >> a) & 1) && (i >> 4) == a;
        const float* dg = reinterpret_cast<const float*>(sm + P_DIAG);
        float* akk = reinterpret_cast<float*>(sm + P_AKK);
        float vq[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int t = 16 * a + jj;
          float vk = __uint_as_float(r[jj]);
          vq[jj] = __uint_as_float(r[16 + jj]);
          if (from_pairs) {
            vk = dg[(a * 16 + jj) * 16 + (i & 15)];
            vq[jj] = dg[1024 + (a * 16 + jj) * 16 + (i & 15)];
          } else {
            vk = i < t ? vk * beta_s[t] : 0.f;
            vq[jj] = i <= t ? vq[jj] : 0.f;
          }
          akk[t * 64 + i] = vk;
        }
        *reinterpret_cast<uint4*>(sm + P_AQKT + sw_chunk(i, 2 * a, 0)) =
            make_uint4(pack_bf16(vq[0], vq[1]), pack_bf16(vq[2], vq[3]), pack_bf16(vq[4], vq[5]), pack_bf16(vq[6], vq[7]));
        *reinterpret_cast<uint4*>(sm + P_AQKT + sw_chunk(i, 2 * a + 1, 0)) = make_uint4(
            pack_bf16(vq[8], vq[9]), pack_bf16(vq[10], vq[11]), pack_bf16(vq[12], vq[13]), pack_bf16(vq[14], vq[15]));
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();  // A_kk and A_qk^T complete
      if (tid == 0) {
        bulk_store(blk + WB_KA + (even ? 0 : 16384), sb + P_AQKT, 8192);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
      // ---- T' = (I + A_kk)^-1 Diag(beta) (the pairwise tiles' area is free again: scratch for the inverse)
      p_inverse(sm, sb, LY, beta_s, tid, warp, lane, g, tq, sb + P_DIAG);
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      // ---- W = T' (K*Gamma): A = T' (K-major [t][i], rows 64..127 discarded), B = K*Gamma (MN-major [i][c])
      if (tid == 0) {
        constexpr uint32_t id_w = idesc_bf16(128, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc_mma(tmem + 128, sdesc(sb + P_TP + ks * 32, 16, 1024), sdesc(sb + P_KG + ks * 2048, 8192, 1024), id_w,
                 ks > 0);
        tc_commit(bar_mma);
        mma_groups = 2;
        bulk_store(blk + WB_TP, sb + P_TP, 8192);
        bulk_store(blk + WB_GAM, sb + P_GAM, 512);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
      ok = __syncthreads_and(mbar_wait(bar_mma, 1, &g_split_timeout));
      tc_fence_after();
    }
    if (ok) {
      // ---- -W to [half][t][c] (warps 0, 1: channels 0-63; warps 4, 5: 64-127), then to the workspace
      if ((warp & 3) < 2) {
        const int t = 32 * (warp & 3) + lane, half = warp >> 2;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t r[32];
          tm_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 128 + 64 * half + 32 * part, r);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(sm + P_W + half * 8192 + sw_chunk(t, 4 * part + q4, 0)) = pack8(r, q4, -1.f);
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        const uint32_t wq = even ? 0 : 8192;
        bulk_store(blk + WB_WQ + wq, sb + P_W, 8192);
        bulk_store(blk + WB_WQ + 16384 + wq, sb + P_W + 8192, 8192);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    if (!ok) break;
    // The stores have read their shared memory, and every thread's generic writes are ordered before the
    // next item's TMA writes: the shared memory and TMEM are free for the next item.
    if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    ++n_done;
  }
  if (tid == 0) {
    if (!ok) {
      // A wait expired: give the loads and products that may still be in flight a bounded wait.
      mbar_wait(bar_in, n_done & 1, &g_split_timeout);
      if (mma_groups >= 1) mbar_wait(bar_mma, 0, &g_split_timeout);
      if (mma_groups >= 2) mbar_wait(bar_mma, 1, &g_split_timeout);
    }
    // Shared memory must stay valid until the stores have read it; their global writes complete before
    // the kernel does.
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(P_TM_COLS));
}

// One bulk copy completing on `bar` (the caller has announced the bytes with expect_tx).
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int x, int h, int t, int b) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(h), "r"(t), "r"(b), "r"(src)
               : "memory");
}

// O^T of one full chunk (TMEM columns [tm_o, tm_o + 64)) into the staging tile [t][v] (bf16, 256-byte rows):
// this thread's lane v, tokens 32*half... Ends with the proxy fence that orders these writes before the TMA
// store that reads them (issued after the next barrier).
__device__ __forceinline__ void stage_o(unsigned char* st, uint32_t tlane, uint32_t tm_o, int trow, int half) {
  uint32_t r[32];
  tm_ld32(tlane + tm_o + 32 * half, r);
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(st) + (32 * half) * VT + trow;
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) dst[jj * VT] = __float2bfloat16_rn(__uint_as_float(r[jj]));
  fence_async_smem();
}

// O^T of one chunk (TMEM columns [tm_o, tm_o + 64)) to o: this thread's lane v, tokens 32*half...
__device__ __forceinline__ void store_o(const ScanParams& p, uint32_t tlane, uint32_t tm_o, int64_t brow, int h, int vt,
                                       int trow, int half, int64_t tc0, int nv) {
  uint32_t r[32];
  tm_ld32(tlane + tm_o + 32 * half, r);
  const int64_t ost = p.os[1];
  __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.o) + brow * p.os[0] + h * p.os[2] + (int64_t)vt * VT + trow +
                      (tc0 + 32 * half) * ost;
  const int jmax = min(32, nv - 32 * half);
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) {
    if (jj < jmax) *op = __float2bfloat16_rn(__uint_as_float(r[jj]));
    op += ost;
  }
}

__global__ void __launch_bounds__(NTHREADS, 1) chunk_state_kernel(ScanParams p, const unsigned char* ws,
                                                                  const __grid_constant__ CUtensorMap omap,
                                                                  int use_omap) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int quad = warp & 3, half = warp >> 2;
  const int trow = 32 * quad + lane;

  const int n_vt = p.V / VT;
  int blk = blockIdx.x;
  const int vt = blk % n_vt;
  blk /= n_vt;
  const int h = blk % p.H;
  const int n = blk / p.H;
  int64_t t0, t1, brow;
  seq_range(p, n, t0, t1, brow);
  const int n_chunks = (int)((t1 - t0 + C - 1) / C);
  const int64_t sbase_slot = slot_base(p, n, t0);

  ChunkCtx x;
  x.v = static_cast<const __nv_bfloat16*>(p.v);
  x.beta = p.beta;
  x.vrow = brow * p.vs[0] + h * p.vs[2] + (int64_t)vt * VT;
  x.vst = p.vs[1];
  x.boff = 0;
  x.bst = 0;

  // Each operand block arrives in two parts, each with its own mbarrier per buffer: part 1 (-W, Q*Gamma,
  // T', gamma_C: used by the conversion and group A) and part 2 (A_qk^T, K*gamma_C/Gamma: group B). A buffer's
  // part 1 is refilled as soon as its chunk's group A is done, part 2 once its group B is, so part 1 and the
  // v tile are fetched about a chunk and a half ahead.
  const uint32_t bar_p1 = sb + S_BAR, bar_p2 = sb + S_BAR + 16, bar_mma = sb + S_BAR + 32;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + S_BAR + 40);
  auto block_src = [&](int c) { return ws + ((size_t)(sbase_slot + c) * p.H + h) * WB_BYTES; };
  auto load_part1 = [&](int c, int b) {  // thread 0
    const uint32_t dst = sb + S_OPS + b * S_OPS_STRIDE, bar = bar_p1 + 8 * b;
    const unsigned char* src = block_src(c);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(WB_KA + (WB_BYTES - WB_TP))
                 : "memory");
    bulk_copy(dst + WB_WQ, src + WB_WQ, WB_KA - WB_WQ, bar);
    bulk_copy(dst + WB_TP, src + WB_TP, WB_BYTES - WB_TP, bar);
  };
  auto load_part2 = [&](int c, int b) {  // thread 0
    const uint32_t dst = sb + S_OPS + b * S_OPS_STRIDE, bar = bar_p2 + 8 * b;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(WB_TP - WB_KA) : "memory");
    bulk_copy(dst + WB_KA, block_src(c) + WB_KA, WB_TP - WB_KA, bar);
  };

  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_p1));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_p1 + 8));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_p2));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_p2 + 8));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_mma));
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
  const uint32_t tlane = tmem + ((uint32_t)(32 * quad) << 16);

  // v tiles of chunks 0 and 1; one cp.async group per chunk from here on (empty past the end), so that at
  // the top of chunk c only chunk c+1's group may still be pending.
  if (n_chunks > 0) load_v(x, sb + S_V, t0, (int)min((int64_t)C, t1 - t0), tid);
  cp_async_commit();
  if (n_chunks > 1) load_v(x, sb + S_V + 16384, t0 + C, (int)min((int64_t)C, t1 - t0 - C), tid);
  cp_async_commit();

  // Initial state: TMEM lane v holds column v of S; this thread moves columns [64*half, +64).
  const size_t hbase = ((size_t)n * p.H + h) * (size_t)KD * p.V;  // this head's state
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    const int cb = 64 * half + 32 * part;
    uint32_t r[32];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj)
      r[jj] = __float_as_uint(p.s0 ? p.s0[state_at(p, hbase, cb + jj, vt * VT + trow)] : 0.f);
    tm_st32(tlane + TM_S + cb, r);
  }
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  // Everything above reads only the scan's inputs; the operand blocks are kernel P's output, so the
  // first block is fetched once that grid has completed (a no-op when launched without a dependency).
  if (tid == 0 && n_chunks > 0) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    load_part1(0, 0);
    load_part2(0, 0);
    if (n_chunks > 1) load_part1(1, 1);
  }

  // Each chunk's MMAs complete twice on bar_mma, group A then group B, and every completion is
  // waited for before the next group is issued: group A always completes phase parity 0, B parity 1.
  bool ok = true;
  for (int c = 0; c < n_chunks && ok; ++c) {
    const int64_t tc0 = t0 + (int64_t)c * C;
    const int nv = (int)min((int64_t)C, t1 - tc0);
    const int buf = c & 1;
    const uint32_t ops = sb + S_OPS + buf * S_OPS_STRIDE;
    const unsigned char* opsp = sm + S_OPS + buf * S_OPS_STRIDE;
    const uint32_t vbuf = sb + S_V + buf * 16384;
    const uint32_t tm_u = buf ? TM_UO : TM_UE;

    // The output staging buffer this chunk fills was read by the store of chunk c-3 (at most the store of chunk
    // c-2 stays in flight).
    if (tid == 0 && use_omap) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
    // The previous chunk's group B is done (TMEM S^T holds S_{c-1}); this chunk's part 1 and v have landed.
    bool w = c == 0 || mbar_wait(bar_mma, 1, &g_split_timeout);
    w = w && mbar_wait(bar_p1 + 8 * buf, (c >> 1) & 1, &g_split_timeout);
    asm volatile("cp.async.wait_group 1;" ::: "memory");  // this chunk's v tile
    fence_async_smem();
    ok = __syncthreads_and(w);
    tc_fence_after();
    if (!ok) break;

    // U^T = V^T T'^T needs no state: the tensor pipe runs it while the state is converted. (U's buffer was
    // last read by chunk c-2's conversion.)
    if (tid == 0) {
      constexpr uint32_t id_vt = idesc_bf16(64, 1, 0);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc_mma(tmem + tm_u, sdesc(vbuf + ks * 2048, 8192, 1024), sdesc(ops + WB_TP + ks * 32, 16, 1024), id_vt, ks > 0);
    }

    // S^T -> its bf16 copy (group A's operand), S^T *= gamma_C in place (group B accumulates on it), and this
    // chunk's O^T = 0 (group A accumulates on it; chunk c-2's output was read from that buffer in chunk c-1).
    {
      const float* gam = reinterpret_cast<const float*>(opsp + WB_GAM);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const int cb = 64 * half + 32 * part;
        uint32_t r[32], b16[16];
        tm_ld32(tlane + TM_S + cb, r);
        if (p.s_dump) {  // the chunk's start state, for the chunked gradients
          float* dst = p.s_dump + ((size_t)(sbase_slot + c) * p.H + h) * KD * p.V + (size_t)cb * p.V + vt * VT + trow;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) dst[(size_t)jj * p.V] = __uint_as_float(r[jj]);
        }
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) b16[jj] = pack_bf16(__uint_as_float(r[2 * jj]), __uint_as_float(r[2 * jj + 1]));
        tm_st16(tlane + TM_SB + cb / 2, b16);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float4 gm = *reinterpret_cast<const float4*>(gam + cb + 4 * jj);
          r[4 * jj + 0] = __float_as_uint(__uint_as_float(r[4 * jj + 0]) * gm.x);
          r[4 * jj + 1] = __float_as_uint(__uint_as_float(r[4 * jj + 1]) * gm.y);
          r[4 * jj + 2] = __float_as_uint(__uint_as_float(r[4 * jj + 2]) * gm.z);
          r[4 * jj + 3] = __float_as_uint(__uint_as_float(r[4 * jj + 3]) * gm.w);
        }
        tm_st32(tlane + TM_S + cb, r);
      }
      uint32_t z[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) z[jj] = 0u;
      tm_st32(tlane + (buf ? TM_OO : TM_OE) + 32 * half, z);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // Chunk c-1's group B is done: the other buffer's part 2 takes chunk c+1's.
    if (tid == 0 && c + 1 < n_chunks) load_part2(c + 1, buf ^ 1);

    // ---- group A: [U^T | O^T] += S^T [-W ; Q*Gamma]^T ---------------------------------------------------
    if (tid == 0) {
      constexpr uint32_t id_wq = idesc_bf16(128, 0, 0);
      const uint32_t d_a = buf ? TM_OO : TM_UE;  // [U_e | O_e] or [O_o | U_o]
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc_mma_ts(tmem + d_a, tmem + TM_SB + 8 * ks, sdesc(ops + WB_WQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                  id_wq, 1);
      tc_commit(bar_mma);
    }
    // meanwhile: the previous chunk's output, staged in shared memory for one TMA store (or stored directly)
    if (c > 0) {
      if (use_omap)
        stage_o(sm + S_OST + ((c - 1) & 1) * 16384, tlane, buf ? TM_OE : TM_OO, trow, half);
      else
        store_o(p, tlane, buf ? TM_OE : TM_OO, brow, h, vt, trow, half, tc0 - C, C);
    }

    ok = __syncthreads_and(mbar_wait(bar_mma, 0, &g_split_timeout));
    tc_fence_after();
    if (!ok) break;
    if (tid == 0 && use_omap && c > 0) {  // the staged output of chunk c-1: [64 tokens][128 values] bf16
      tma_store_4d(&omap, sb + S_OST + ((c - 1) & 1) * 16384, vt * VT, h, (int)(tc0 - C), (int)brow);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }

    // ---- U^T -> its bf16 copy ---------------------------------------------------------------------
    {
      uint32_t r[32], b16[16];
      tm_ld32(tlane + tm_u + 32 * half, r);
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) b16[jj] = pack_bf16(__uint_as_float(r[2 * jj]), __uint_as_float(r[2 * jj + 1]));
      tm_st16(tlane + TM_UB + 16 * half, b16);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    ok = __syncthreads_and(mbar_wait(bar_p2 + 8 * buf, (c >> 1) & 1, &g_split_timeout));  // and part 2 landed
    tc_fence_after();
    if (!ok) break;

    // ---- group B: [O^T | S^T] += U^T [A_qk ; (K*gamma_C/Gamma)^T]^T, B MN-major (rows: the K index) ------
    if (tid == 0) {
      constexpr uint32_t id_b = idesc_bf16(192, 0, 1);
      const uint32_t d_b = buf ? TM_S : TM_OE;  // [O_e | S] or [S | O_o]
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc_mma_ts(tmem + d_b, tmem + TM_UB + 8 * ks, sdesc(ops + WB_KA + ks * 2048, 8192, 1024), id_b, 1);
      tc_commit(bar_mma);
    }
    // Group A was done with this buffer's part 1 and v tile: refill them with chunk c+2's while group B runs.
    if (c + 2 < n_chunks) {
      if (tid == 0) load_part1(c + 2, buf);
      load_v(x, vbuf, tc0 + 2 * C, (int)min((int64_t)C, t1 - tc0 - 2 * C), tid);
    }
    cp_async_commit();
  }
  // The last chunk's group B, then its output.
  if (ok && n_chunks > 0) {
    ok = __syncthreads_and(mbar_wait(bar_mma, 1, &g_split_timeout));
    tc_fence_after();
    if (ok) {
      const int64_t tl = t0 + (int64_t)(n_chunks - 1) * C;
      store_o(p, tlane, ((n_chunks - 1) & 1) ? TM_OO : TM_OE, brow, h, vt, trow, half, tl, (int)(t1 - tl));
    }
  }
  cp_async_wait_all();
  if (tid == 0 && use_omap) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
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
      for (int jj = 0; jj < 32; ++jj) p.sf[state_at(p, hbase, cb + jj, vt * VT + trow)] = __uint_as_float(r[jj]);
    }
  }
  if (!ok && tid == 0) {
    // A wait expired: give the MMAs and operand loads that may still be in flight a bounded wait.
    mbar_wait(bar_mma, 0, &g_split_timeout);
    mbar_wait(bar_mma, 1, &g_split_timeout);
    for (int b = 0; b < 2; ++b) {
      mbar_wait(bar_p1 + 8 * b, 0, &g_split_timeout);
      mbar_wait(bar_p2 + 8 * b, 0, &g_split_timeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TM_COLS));
}

template <typename F>
cudaError_t set_smem_once(F* fn, int bytes, std::atomic<uint64_t>& configured) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;  // one configuration bit per device
  const uint64_t bit = 1ull << dev;
  if (!(configured.load(std::memory_order_relaxed) & bit)) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    // The largest carveout, so that kernel P's two CTAs per SM both fit.
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  return cudaSuccess;
}

}  // namespace

int64_t split_slots(int64_t B, int64_t T, int64_t N, bool varlen) {
  return varlen ? T / C + N + 1 : B * ((T + C - 1) / C);
}

size_t split_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N, bool varlen) {
  return (size_t)split_slots(B, T, N, varlen) * (size_t)H * (size_t)WB_BYTES;
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (no link-time libcuda dependency).
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// A [B,T,H,K] token tensor with element strides s = (b, t, h) as a 4-d tensor map (K, H, T, B) read in
// boxes of 64 channels x 64 tokens of one head. The stride of an extent-1 dimension never moves the
// pointer; it is given its contiguous value. Returns false when the driver refuses the layout.
bool token_map(CUtensorMap* m, const void* base, bool bf16, const int64_t s[3], int64_t B, int64_t T, int64_t H,
               int64_t K) {
  const EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const int64_t es = bf16 ? 2 : 4;
  const int64_t sh = H > 1 ? s[2] : K;
  const int64_t st = T > 1 ? s[1] : H * sh;
  const int64_t sbt = B > 1 ? s[0] : T * st;
  const cuuint64_t dims[4] = {(cuuint64_t)K, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)(sh * es), (cuuint64_t)(st * es), (cuuint64_t)(sbt * es)};
  const cuuint32_t box[4] = {64, 1, 64, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The bf16 output o [B,T,H,V] (element strides s = (b, t, h)) as a 4-d tensor map (V, H, T, B) written in
// boxes of 128 values x 64 tokens of one head (kernel S's tile of one chunk). False when the driver refuses the
// layout (kernel S then stores o directly).
bool out_map(CUtensorMap* m, void* base, const int64_t s[3], int64_t B, int64_t T, int64_t H, int64_t V) {
  const EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const int64_t sh = H > 1 ? s[2] : V;
  const int64_t st = T > 1 ? s[1] : H * sh;
  const int64_t sbt = B > 1 ? s[0] : T * st;
  const cuuint64_t dims[4] = {(cuuint64_t)V, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)(sh * 2), (cuuint64_t)(st * 2), (cuuint64_t)(sbt * 2)};
  const cuuint32_t box[4] = {(cuuint32_t)VT, 1, (cuuint32_t)C, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

bool split_maps_ok(const ScanParams& p) {
  PMaps m;
  return token_map(&m.q, p.q, true, p.qs, p.B, p.T, p.H, p.K) && token_map(&m.k, p.k, true, p.ks, p.B, p.T, p.H, p.K) &&
         token_map(&m.g, p.gate, false, p.gs, p.B, p.T, p.H, p.K);
}

cudaError_t launch_chunk_split(const ScanParams& p, void* ws, cudaStream_t s) {
  static std::atomic<uint64_t> cfg_p[4], cfg_s{0};
  auto intra = p.gate_mode == GATE_LOGITS    ? chunk_intra_kernel<GATE_LOGITS>
               : p.gate_mode == GATE_SOFTPLUS ? chunk_intra_kernel<GATE_SOFTPLUS>
               : p.gate_mode == KDA_GATE_LOG  ? chunk_intra_kernel<KDA_GATE_LOG>
                                              : chunk_intra_kernel<KDA_GATE_ALPHA>;
  cudaError_t e = set_smem_once(intra, P_SMEM, cfg_p[p.gate_mode & 3]);
  if (e == cudaSuccess) e = set_smem_once(chunk_state_kernel, S_SMEM, cfg_s);
  if (e != cudaSuccess) return e;
  const int64_t slots = split_slots(p.B, p.T, p.N, p.cu != nullptr);
  if (slots == 0 || p.N == 0) return cudaSuccess;
  PMaps maps;
  if (!token_map(&maps.q, p.q, true, p.qs, p.B, p.T, p.H, p.K) ||
      !token_map(&maps.k, p.k, true, p.ks, p.B, p.T, p.H, p.K) ||
      !token_map(&maps.g, p.gate, false, p.gs, p.B, p.T, p.H, p.K))
    return cudaErrorInvalidValue;  // callers check split_maps_ok first
  // Kernel P persistent: two CTAs per SM (its shared memory and registers allow two), each walking the items
  // with a fixed stride. The unbounded gate's items differ in cost (pairwise diagonal tiles where the decay is
  // steep, which depends on the head), so there each CTA takes one item and the hardware balances the load.
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t items = slots * p.H;
  if (items > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const unsigned gp = p.gate_mode == GATE_SOFTPLUS
                          ? (unsigned)items
                          : (unsigned)std::min<int64_t>(items, 2 * (int64_t)std::max(sms, 1));
  intra<<<gp, NTHREADS, P_SMEM, s>>>(p, static_cast<unsigned char*>(ws), maps, slots);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t grid = (int64_t)p.N * p.H * (p.V / VT);
  // Programmatic dependent launch: kernel S's CTAs set up (barriers, TMEM, initial state, first v tile)
  // while kernel P's last CTAs finish.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = S_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  CUtensorMap omap;
  std::memset(&omap, 0, sizeof(omap));
  const int use_omap = out_map(&omap, p.o, p.os, p.B, p.T, p.H, p.V) ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, chunk_state_kernel, p, static_cast<const unsigned char*>(ws), omap, use_omap);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

namespace {
// One thread waits on an mbarrier that expects one arrival which never comes: the bounded wait must
// give up and record the expiry in g_split_timeout.
__global__ void wait_expiry_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
  mbar_wait(b, 0, &g_split_timeout);
}
}  // namespace

cudaError_t launch_wait_selftest(cudaStream_t s) {
  wait_expiry_selftest_kernel<<<1, 1, 0, s>>>();
  return cudaGetLastError();
}

cudaError_t split_read_timeout(int* flag, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(flag, g_split_timeout, sizeof(int));
  if (e != cudaSuccess || !reset) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_split_timeout, &zero, sizeof(int));
}

}  // namespace kda
