// chunk_split.cu -- chunked prefill in two kernels: the state-independent work of every chunk in
// parallel (kernel P), then the state recurrence (kernel S).
//
// The per-chunk quantities of the chunkwise form that do not depend on the carried state --
// the decay factors, A_qk and A_kk, T' = (I + A_kk)^-1 Diag(beta), W = T' (K*Gamma), Q*Gamma and
// K*gamma_C/Gamma -- are most of the arithmetic. In the fused kernel (chunk.cu) they sit on the
// sequential path of one CTA per (sequence, head). Here kernel P computes them for all chunks of all
// heads at once, one CTA per (chunk, head) over every SM, and writes each chunk's operand set as
// one 66,048-byte block to a workspace: the block is the exact image of the shared-memory tiles
// (128-byte swizzle included), so kernel S moves it with a single bulk copy into a 1 KB-aligned
// buffer and feeds it straight to tcgen05. Kernel S keeps one CTA per (sequence, head, V-tile) with
// the transposed state S^T in TMEM and runs two MMA groups per chunk:
//   group A:  [U^T | O^T] = S^T [-W ; Q*Gamma]^T  (one N = 128 product),  U^T += V^T T'^T
//   group B:  [O^T | S^T] += U^T [A_qk ; (K*gamma_C/Gamma)^T]^T  (one N = 192 product; S^T pre-scaled)
// A tcgen05 MMA's time grows much more slowly than its N, so the products that share an A operand
// are fused along N. The fused accumulators must be adjacent in TMEM -- [U | O] for group A and
// [O | S] for group B -- so the O and U buffers alternate with the chunk's parity around the fixed
// S, and kernel P writes each block's operand pairs in the order that chunk's parity needs.
// The price of the split is the workspace traffic (one write and one read of ~1 KB per token-head).
//
// With Kimi Linear's unbounded gate (KDA_GATE_SOFTPLUS) a pre-pass, softplus_diag_kernel, first forms the
// diagonal 16x16 blocks of A_kk and A_qk pair by pair (their block-boundary factorisation would need the
// reciprocal of a whole block's decay, which that gate does not bound), and chunk_intra_kernel<true> takes
// them from the workspace in place of its own diagonal tiles; every other factor stays <= 1.
//
// Workspace slots. Chunk j of sequence n has slot n * ceil(T/64) + j without cu_seqlens, and
// floor(cu[n]/64) + n + j with them (unique: a sequence's slots end before the next one's begin).
#include <atomic>

#include "chunk_common.cuh"

namespace kda {

// Set to 1 by any CTA of the split kernels whose bounded wait expired.
__device__ int g_split_timeout = 0;

namespace {

// One workspace block = the output region of kernel P = the operand buffer of kernel S. All three
// operand regions are K-major; a pair (X, Y) is stored in that order for an even chunk index j and
// as (Y, X) for an odd one.
constexpr int WB_WQ = 0;         // 32K  two k-atoms (c) of 128 rows: (-W [t][c], Q*Gamma [t][c])
constexpr int WB_KA = 32768;     // 24K  one k-atom (t) of 192 rows: (A_qk [t'][t], (K*gamma_C/Gamma)^T [c][t])
constexpr int WB_TP = 57344;     // 8K   T' [t][i]
constexpr int WB_GAM = 65536;    // 512  gamma_C, fp32 [128]
constexpr int WB_BYTES = 66048;
// Unbounded gate only: the pairwise diagonal blocks of A_kk and A_qk (see softplus_diag_kernel), written
// into the T' region before kernel P runs; P reads them there before its final bulk store overwrites it.
constexpr int WB_DIAG = WB_TP;
static_assert(2 * 4 * 16 * 16 * 4 <= WB_GAM - WB_TP, "the diagonal blocks fit the T' region");

// Kernel P shared memory (104,192 bytes: two CTAs fit on an SM). Q*Gamma and K*gamma_C/Gamma
// never touch it: the decay pass writes them from registers straight into the workspace block.
constexpr int P_QE = 0;                     // 16K Qe [t][c]; after A_qk, -W [t][c] (two 8K atoms)
constexpr int P_KE = P_QE + 16384;          // 16K Ke [t][c]; after A_kk, the bf16 copy of T
constexpr int P_KC = P_KE + 16384;          // 16K Kc [t][c]
constexpr int P_KG = P_KC + 16384;          // 16K K*Gamma [i][c]
constexpr int P_AKK = P_KG + 16384;         // 16K A_kk fp32
constexpr int P_AQK = P_AKK + 16384;        // 8K  A_qk [t'][t]  } in block order for odd chunks, where
constexpr int P_TP = P_AQK + 8192;          // 8K  T'            } A_qk ends the KA region and T' and
constexpr int P_GAM = P_TP + 8192;          // 512 gamma_C       } gamma_C follow it
constexpr int P_BETA = P_GAM + 512;         // 256 beta
constexpr int P_VEC = P_BETA + 256;         // vectors
constexpr int P_SMEM = P_VEC + VEC_FLOATS * 4;
static_assert(P_TP - P_AQK == WB_TP - (WB_KA + 16384) && P_GAM - P_TP == WB_GAM - WB_TP, "odd-chunk tail order");
static_assert(P_TP % 1024 == 0 && P_AQK % 1024 == 0, "swizzle atoms need 1 KB alignment");
static_assert(2 * (P_SMEM + 1024) <= 228 * 1024, "two CTAs per SM");

// Kernel S shared memory: the operand blocks of two chunks and their v tiles.
constexpr int S_OPS = 0;                    // 2 x operand block (66048 B, padded to 66560)
constexpr int S_OPS_STRIDE = 66560;
constexpr int S_V = 2 * S_OPS_STRIDE;       // 2 x 16K v tile [i][v], two halves (MN-major A)
constexpr int S_BAR = S_V + 2 * 16384;      // mbarriers: ops0, ops1, mma; TMEM base
constexpr int S_SMEM = S_BAR + 64;
static_assert(S_SMEM <= 227 * 1024, "shared memory budget");
static_assert(S_V % 1024 == 0 && S_OPS_STRIDE % 1024 == 0, "swizzle atoms need 1 KB alignment");

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

// Decay pass, step 2 of kernel P: the same tiles as decay_step2 (chunk_common.cuh), with Q*Gamma and
// K*gamma_C/Gamma stored straight into their places in the workspace block. Q*Gamma goes to qg_dst
// as [t][c] rows of 16 KB k-atoms (a warp's 32 four-byte stores cover one 128-byte swizzled row);
// K*gamma_C/Gamma goes to kt_dst transposed, [c][t], one 16-byte piece per channel and 8 tokens.
// Tokens run forward for the E-scaled tiles and backward for the F-scaled ones, so no per-token F
// array is held in registers.
__device__ __forceinline__ void p_decay_step2(unsigned char* sm, const Prefetch& pf, int da, int c0,
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
  if (da == 0) *reinterpret_cast<float2*>(sm + P_GAM + 4 * c0) = make_float2(ex2(e[3].x), ex2(e[3].y));
  const float2 GS = make_float2(ex2(gs.x), ex2(gs.y));
  const float2 PM = make_float2(ex2(e[3].x - eda.x), ex2(e[3].y - eda.y));
  float2 E = make_float2(1.f, 1.f);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int t = 16 * da + i;
    E.x *= al[i].x;
    E.y *= al[i].y;
    const float2 qf = unpack_bf16(pf.q[i]), kf = unpack_bf16(pf.k[i]);
    const uint32_t off = sw_e(t, c0, 8192);
    const float qex = qf.x * E.x, qey = qf.y * E.y, kex = kf.x * E.x, key = kf.y * E.y;
    *reinterpret_cast<uint32_t*>(sm + P_QE + off) = pack_bf16(qex, qey);
    *reinterpret_cast<uint32_t*>(sm + P_KE + off) = pack_bf16(kex, key);
    *reinterpret_cast<uint32_t*>(sm + P_KG + off) = pack_bf16(kex * GS.x, key * GS.y);
    *reinterpret_cast<uint32_t*>(qg_dst + sw_e(t, c0, 16384)) = pack_bf16(qex * GS.x, qey * GS.y);
  }
  float2 F = make_float2(1.f, 1.f);
  float ktx[8], kty[8];  // K*gamma_C/Gamma of channels c0, c0+1 for the 8 tokens of one 16-byte piece
#pragma unroll
  for (int i = 15; i >= 0; --i) {
    const int t = 16 * da + i;
    const float2 kf = unpack_bf16(pf.k[i]);
    const float kfx = kf.x * F.x, kfy = kf.y * F.y;
    *reinterpret_cast<uint32_t*>(sm + P_KC + sw_e(t, c0, 8192)) = pack_bf16(kfx, kfy);
    ktx[i & 7] = kfx * PM.x;
    kty[i & 7] = kfy * PM.y;
    if ((i & 7) == 0) {  // tokens 16da + i .. +7 complete: piece j = 2da + i/8 of rows c0 and c0 + 1
      const int j = 2 * da + (i >> 3);
      const uint4 wx = make_uint4(pack_bf16(ktx[0], ktx[1]), pack_bf16(ktx[2], ktx[3]), pack_bf16(ktx[4], ktx[5]),
                                  pack_bf16(ktx[6], ktx[7]));
      const uint4 wy = make_uint4(pack_bf16(kty[0], kty[1]), pack_bf16(kty[2], kty[3]), pack_bf16(kty[4], kty[5]),
                                  pack_bf16(kty[6], kty[7]));
      *reinterpret_cast<uint4*>(kt_dst + sw_chunk(c0, j, 0)) = wx;
      *reinterpret_cast<uint4*>(kt_dst + sw_chunk(c0 + 1, j, 0)) = wy;
    }
    F.x *= al[i].x;
    F.y *= al[i].y;
  }
}

// Kimi Linear's unbounded gate (KDA_GATE_SOFTPLUS), g = -e^{A_h} softplus(z): the diagonal 16x16 blocks
// of A_kk and A_qk of one (chunk, head), pair by pair. Within a block exp(G_t - G_j) <= 1 for j <= t, but
// kernel P's block-boundary factorisation splits it as exp(G_t - G_s) exp(G_s - G_j), whose second factor
// grows with the decay of the whole block, which this gate does not bound. One warp per (block a, column
// j), lanes over the channels: A_qk[t][j] = sum_c q_tc k_jc exp(G_tc - G_jc) for t >= j and A_kk[t][j] =
// beta_t sum_c k_tc k_jc exp(G_tc - G_jc) for t > j, with q, k L2-normalised and rounded to bf16 first
// when the flag asks, and beta from its logits when the flag asks, as kernel P does.
constexpr int D_Q = 0, D_K = 16384, D_G = 32768, D_BETA = 65536, D_SMEM = D_BETA + 256;

__global__ void __launch_bounds__(NTHREADS, 3) softplus_diag_kernel(ScanParams p, unsigned char* ws) {
  extern __shared__ __align__(16) unsigned char sm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const int64_t slot = blockIdx.x;
  int n, jc;
  if (!locate_slot(p, slot, n, jc)) return;  // uniform across the CTA
  int64_t t0, t1, brow;
  seq_range(p, n, t0, t1, brow);
  const int64_t tc0 = t0 + (int64_t)jc * C;
  const int nv = (int)min((int64_t)C, t1 - tc0);
  float* out = reinterpret_cast<float*>(ws + ((size_t)slot * p.H + h) * WB_BYTES + WB_DIAG);
  const float sc = expf(__ldg(p.A_log + h));
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.k);
  __nv_bfloat16* sq = reinterpret_cast<__nv_bfloat16*>(sm + D_Q);
  __nv_bfloat16* sk = reinterpret_cast<__nv_bfloat16*>(sm + D_K);
  float* sg = reinterpret_cast<float*>(sm + D_G);
  float* sbeta = reinterpret_cast<float*>(sm + D_BETA);

  // Rows: warp w takes tokens w, w + 8, ...; lane l channels 4l .. 4l + 3, in two batches of four rows
  // whose loads are all issued before the first is used.
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint2 qv[4], kv[4];
    float4 zv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = warp + 8 * (4 * half + i);
      const int64_t t = tc0 + r;
      qv[i] = kv[i] = make_uint2(0u, 0u);
      zv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nv) {
        qv[i] = *reinterpret_cast<const uint2*>(qb + brow * p.qs[0] + t * p.qs[1] + h * p.qs[2] + 4 * lane);
        kv[i] = *reinterpret_cast<const uint2*>(kb + brow * p.ks[0] + t * p.ks[1] + h * p.ks[2] + 4 * lane);
        zv[i] = *reinterpret_cast<const float4*>(p.gate + brow * p.gs[0] + t * p.gs[1] + h * p.gs[2] + 4 * lane);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = warp + 8 * (4 * half + i);
      const float4 z = zv[i];
      const float4 lg = r < nv ? make_float4(softplus_log_decay(sc, z.x) * LOG2E, softplus_log_decay(sc, z.y) * LOG2E,
                                             softplus_log_decay(sc, z.z) * LOG2E, softplus_log_decay(sc, z.w) * LOG2E)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      uint2 qr = qv[i], kr = kv[i];
      if (p.qk_l2norm) {
        float2 q01 = unpack_bf16(qr.x), q23 = unpack_bf16(qr.y), k01 = unpack_bf16(kr.x), k23 = unpack_bf16(kr.y);
        float ssq = q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y;
        float ssk = k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
          ssq += __shfl_xor_sync(0xffffffffu, ssq, m);
          ssk += __shfl_xor_sync(0xffffffffu, ssk, m);
        }
        const float fq = l2norm_scale(ssq), fk = l2norm_scale(ssk);
        qr = make_uint2(pack_bf16(q01.x * fq, q01.y * fq), pack_bf16(q23.x * fq, q23.y * fq));
        kr = make_uint2(pack_bf16(k01.x * fk, k01.y * fk), pack_bf16(k23.x * fk, k23.y * fk));
      }
      *reinterpret_cast<uint2*>(sq + r * KD + 4 * lane) = qr;
      *reinterpret_cast<uint2*>(sk + r * KD + 4 * lane) = kr;
      *reinterpret_cast<float4*>(sg + r * KD + 4 * lane) = lg;
      if (lane == 0) {
        const int64_t t = tc0 + r;
        sbeta[r] = r < nv ? beta_value(__ldg(p.beta + brow * p.bs[0] + t * p.bs[1] + h * p.bs[2]), p.beta_sigmoid) : 0.f;
      }
    }
  }
  __syncthreads();
  // G: the running log2-decay within each 16-token block, one (block, channel) column per thread.
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int col = tid + NTHREADS * m, a = col >> 7, c = col & (KD - 1);
    float run = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float* x = sg + (16 * a + i) * KD + c;
      run += *x;
      *x = run;
    }
  }
  __syncthreads();
  // One warp per (block a, column j): each lane sums its four channels for every row t >= j of the block
  // (v[t] for A_qk, v[16 + t] for A_kk), then one reduce-scatter over the warp leaves lane l with the
  // total of entry l: A_qk[t = l][j] for l < 16, A_kk[t = l - 16][j] otherwise.
  for (int item = warp; item < 64; item += 8) {
    const int a = item >> 4, j = item & 15, rj = 16 * a + j;
    float kj[4], gj[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      kj[m] = __bfloat162float(sk[rj * KD + lane + 32 * m]);
      gj[m] = sg[rj * KD + lane + 32 * m];
    }
    float v[32];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float sqk = 0.f, skk = 0.f;
      if (t >= j) {  // uniform across the warp
        const int rt = 16 * a + t;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int c = lane + 32 * m;
          const float w = kj[m] * ex2(sg[rt * KD + c] - gj[m]);
          sqk = fmaf(__bfloat162float(sq[rt * KD + c]), w, sqk);
          skk = fmaf(__bfloat162float(sk[rt * KD + c]), w, skk);
        }
      }
      v[t] = sqk;
      v[16 + t] = skk;
    }
    int first = 0;
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
      if (up) first += hn;
    }
    // first == lane
    if (first < 16) {
      out[1024 + (a * 16 + first) * 16 + j] = v[0];
    } else {
      const int t = first - 16;
      out[(a * 16 + t) * 16 + j] = t > j ? v[0] * sbeta[16 * a + t] : 0.f;
    }
  }
}

// The four diagonal 16x16 blocks of A_kk and A_qk for the unbounded gate, formed pairwise by
// softplus_diag_kernel and stored as fp32 [A_kk | A_qk][block a][t][j] (A_kk with beta_t folded in, zero
// on and above the diagonal; A_qk zero above it) in the T' region of the chunk's workspace block.

// intra_phases (chunk_common.cuh) for the unbounded gate: the tile products run as usual, then the
// diagonal blocks, whose block-boundary factorisation needs exp(-decay of 16 tokens) and can overflow,
// are replaced by the pairwise values from `diag` before the inverse and the W phase read them.
__device__ __forceinline__ void unbounded_intra_phases(unsigned char* sm, uint32_t sb, const IntraLayout& L,
                                                       const float* beta_s, int tid, int warp, int lane, int g,
                                                       int tq, const float* diag) {
  float dk[4], dq[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    dk[r] = __ldg(diag + tid + NTHREADS * r);
    dq[r] = __ldg(diag + 1024 + tid + NTHREADS * r);
  }
  a_tiles<2>(sm, sb, L, L.ke, warp, 8, warp < 2 ? 2 : 1, lane, g, tq, beta_s, /*is_qk=*/false);
  __syncthreads();
  float* akk = reinterpret_cast<float*>(sm + L.akk);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int e = tid + NTHREADS * r, a = e >> 8, t = (e >> 4) & 15, j = e & 15;
    akk[(16 * a + t) * 64 + 16 * a + j] = dk[r];
  }
  __syncthreads();  // A_kk ready
  if (warp < 4) {
    inverse_warps0to3(sm, sb, L, beta_s, tid, warp, lane, g, tq);
  } else {
    a_tiles<3>(sm, sb, L, L.qe, warp - 4, 4, (warp - 4) < 2 ? 3 : 2, lane, g, tq, beta_s, /*is_qk=*/true);
    zero_upper_blocks(sm, L.aqk, tid - 128, 128);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int e = tid + NTHREADS * r, a = e >> 8, t = (e >> 4) & 15, j = e & 15;
    *reinterpret_cast<__nv_bfloat16*>(sm + L.aqk + sw_e(16 * a + t, 16 * a + j, 8192)) = __float2bfloat16_rn(dq[r]);
  }
  // The W phase does not read A_qk; the barrier before the bulk store publishes these writes.
}

template <bool UNBOUNDED>
__global__ void __launch_bounds__(NTHREADS, 2) chunk_intra_kernel(ScanParams p, unsigned char* ws) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  // qg and kt are not staged in shared memory by this kernel (p_decay_step2 stores them to the block).
  constexpr IntraLayout LY{P_QE, P_KE, P_KC, -1, P_KG, -1, P_AKK, P_AQK, P_TP, P_KE, P_VEC};
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  // Kernel S may be scheduled once every CTA of this grid has started; it reads the workspace only
  // after this whole grid has completed (griddepcontrol.wait).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int h = blockIdx.y;
  const float gsc = p.gate_mode >= GATE_LOGITS ? expf(__ldg(p.A_log + h)) : 0.f;  // e^{A_h}
  const int64_t slot = blockIdx.x;
  int n, j;
  if (!locate_slot(p, slot, n, j)) return;  // uniform across the CTA
  int64_t t0, t1, brow;
  seq_range(p, n, t0, t1, brow);
  const int64_t tc0 = t0 + (int64_t)j * C;
  const int nv = (int)min((int64_t)C, t1 - tc0);
  unsigned char* blk = ws + ((size_t)slot * p.H + h) * WB_BYTES;
  const bool even = (j & 1) == 0;  // operand pair order within the block

  ChunkCtx x;
  x.q = static_cast<const __nv_bfloat16*>(p.q);
  x.k = static_cast<const __nv_bfloat16*>(p.k);
  x.v = nullptr;
  x.gate = p.gate;
  x.beta = p.beta;
  x.qrow = brow * p.qs[0] + h * p.qs[2];
  x.krow = brow * p.ks[0] + h * p.ks[2];
  x.vrow = 0;
  x.grow = brow * p.gs[0] + h * p.gs[2];
  x.boff = brow * p.bs[0] + h * p.bs[2];
  x.qst = p.qs[1];
  x.kst = p.ks[1];
  x.vst = 0;
  x.gst = p.gs[1];
  x.bst = p.bs[1];

  const int c0 = 2 * (tid & 63), da = tid >> 6;
  float* beta_s = reinterpret_cast<float*>(sm + P_BETA);
  {
    Prefetch pf;
    load_qkg(x, tc0, nv, c0, da, pf);
    if (tid < C) beta_s[tid] = tid < nv ? beta_value(__ldg(x.beta + x.boff + (tc0 + tid) * x.bst), p.beta_sigmoid) : 0.f;
    if (p.qk_l2norm) l2norm_qk(pf, reinterpret_cast<float*>(sm + P_VEC) + VEC_D, tid, da);
    float2 al[16];
    decay_step1<UNBOUNDED>(sm, LY, pf, nv, da, c0, p.gate_mode, gsc, p.g_min, al);
    __syncthreads();
    p_decay_step2(sm, pf, da, c0, al, blk + WB_WQ + (even ? 8192 : 0), blk + WB_KA + (even ? 8192 : 0));
  }
  __syncthreads();
  if constexpr (UNBOUNDED) {
    unbounded_intra_phases(sm, sb, LY, beta_s, tid, warp, lane, g, tq, reinterpret_cast<const float*>(blk + WB_DIAG));
  } else {
    intra_phases(sm, sb, LY, beta_s, tid, warp, lane, g, tq);
  }

  // W = T' (K*Gamma) on mma.sync. Warp w owns columns 16w.. of all 64 rows, so every warp does the
  // same ten block products of the lower-triangular T'. -W is stored over the dead Qe tile as
  // [t][c], two 64-column atoms: the rows it takes in the block's K-major pair with Q*Gamma.
  {
    float acc[4][2][4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int jn = 0; jn < 2; ++jn)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[m][jn][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sb + P_KG + sw_chunk(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * warp + (lane >> 4), 8192), b0, b1,
                b2, b3);
#pragma unroll
      for (int m = kk; m < 4; ++m) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sb + P_TP + sw_chunk(16 * m + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * kk + (lane >> 4), 8192), a0, a1,
                a2, a3);
        mma_bf16(acc[m][0], a0, a1, a2, a3, b0, b1);
        mma_bf16(acc[m][1], a0, a1, a2, a3, b2, b3);
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int jn = 0; jn < 2; ++jn)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int t = 16 * m + g + 8 * hr, c = 16 * warp + 8 * jn + 2 * tq;
          *reinterpret_cast<uint32_t*>(sm + P_QE + sw_e(t, c, 8192)) =
              pack_bf16(-acc[m][jn][2 * hr], -acc[m][jn][2 * hr + 1]);
        }
  }
  fence_async_smem();
  __syncthreads();
  if (tid == 0) {
    const uint32_t wq = even ? 0 : 8192;
    bulk_store(blk + WB_WQ + wq, sb + P_QE, 8192);
    bulk_store(blk + WB_WQ + 16384 + wq, sb + P_QE + 8192, 8192);
    if (even) {
      bulk_store(blk + WB_KA, sb + P_AQK, 8192);
      bulk_store(blk + WB_TP, sb + P_TP, WB_BYTES - WB_TP);
    } else {
      bulk_store(blk + WB_KA + 16384, sb + P_AQK, WB_BYTES - (WB_KA + 16384));
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    // Shared memory must stay valid until the copies have read it; their global writes complete
    // before the kernel does.
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
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

__global__ void __launch_bounds__(NTHREADS, 1) chunk_state_kernel(ScanParams p, const unsigned char* ws) {
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

  const uint32_t bar_ops = sb + S_BAR, bar_mma = sb + S_BAR + 16;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + S_BAR + 24);
  auto block_src = [&](int c) { return ws + ((size_t)(sbase_slot + c) * p.H + h) * WB_BYTES; };

  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_ops));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_ops + 8));
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

  if (n_chunks > 0) {
    load_v(x, sb + S_V, t0, (int)min((int64_t)C, t1 - t0), tid);
    cp_async_commit();
  }

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
    bulk_load(sb + S_OPS, block_src(0), WB_BYTES, bar_ops);
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

    // The previous chunk's group B is done (TMEM S^T holds S_{c-1}); this chunk's operands have landed.
    bool w = c == 0 || mbar_wait(bar_mma, 1, &g_split_timeout);
    w = w && mbar_wait(bar_ops + 8 * buf, (c >> 1) & 1, &g_split_timeout);
    ok = __syncthreads_and(w);
    tc_fence_after();
    if (!ok) break;

    // S^T -> its bf16 copy (group A's operand) and S^T *= gamma_C in place (group B accumulates on it).
    {
      const float* gam = reinterpret_cast<const float*>(opsp + WB_GAM);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const int cb = 64 * half + 32 * part;
        uint32_t r[32], b16[16];
        tm_ld32(tlane + TM_S + cb, r);
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
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    cp_async_wait_all();  // this chunk's v tile
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // The other buffers' last readers (chunk c-1's MMAs) are done: prefetch chunk c+1 into them.
    if (c + 1 < n_chunks) {
      if (tid == 0) bulk_load(sb + S_OPS + (buf ^ 1) * S_OPS_STRIDE, block_src(c + 1), WB_BYTES, bar_ops + 8 * (buf ^ 1));
      load_v(x, sb + S_V + (buf ^ 1) * 16384, tc0 + C, (int)min((int64_t)C, t1 - tc0 - C), tid);
    }
    cp_async_commit();

    // ---- group A: [U^T | O^T] = S^T [-W ; Q*Gamma]^T, then U^T += V^T T'^T ---------------------------
    if (tid == 0) {
      constexpr uint32_t id_wq = idesc_bf16(128, 0, 0), id_vt = idesc_bf16(64, 1, 0);
      const uint32_t d_a = buf ? TM_OO : TM_UE;  // [U_e | O_e] or [O_o | U_o]
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc_mma_ts(tmem + d_a, tmem + TM_SB + 8 * ks, sdesc(ops + WB_WQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                  id_wq, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc_mma(tmem + tm_u, sdesc(vbuf + ks * 2048, 8192, 1024), sdesc(ops + WB_TP + ks * 32, 16, 1024), id_vt, 1);
      tc_commit(bar_mma);
    }
    // meanwhile: the previous chunk's output
    if (c > 0) store_o(p, tlane, buf ? TM_OE : TM_OO, brow, h, vt, trow, half, tc0 - C, C);

    ok = __syncthreads_and(mbar_wait(bar_mma, 0, &g_split_timeout));
    tc_fence_after();
    if (!ok) break;

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
    __syncthreads();
    tc_fence_after();

    // ---- group B: [O^T | S^T] += U^T [A_qk ; (K*gamma_C/Gamma)^T]^T -----------------------------------
    if (tid == 0) {
      constexpr uint32_t id_b = idesc_bf16(192, 0, 0);
      const uint32_t d_b = buf ? TM_S : TM_OE;  // [O_e | S] or [S | O_o]
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc_mma_ts(tmem + d_b, tmem + TM_UB + 8 * ks, sdesc(ops + WB_KA + ks * 32, 16, 1024), id_b, 1);
      tc_commit(bar_mma);
    }
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
    mbar_wait(bar_ops, 0, &g_split_timeout);
    mbar_wait(bar_ops + 8, 0, &g_split_timeout);
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
  const uint64_t bit = 1ull << (dev & 63);
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

cudaError_t launch_chunk_split(const ScanParams& p, void* ws, cudaStream_t s) {
  const bool unbounded = p.gate_mode == GATE_SOFTPLUS;
  static std::atomic<uint64_t> cfg_p{0}, cfg_pu{0}, cfg_d{0}, cfg_s{0};
  cudaError_t e = unbounded ? set_smem_once(chunk_intra_kernel<true>, P_SMEM, cfg_pu)
                            : set_smem_once(chunk_intra_kernel<false>, P_SMEM, cfg_p);
  if (e == cudaSuccess && unbounded) e = set_smem_once(softplus_diag_kernel, D_SMEM, cfg_d);
  if (e == cudaSuccess) e = set_smem_once(chunk_state_kernel, S_SMEM, cfg_s);
  if (e != cudaSuccess) return e;
  const int64_t slots = split_slots(p.B, p.T, p.N, p.cu != nullptr);
  if (slots == 0 || p.N == 0) return cudaSuccess;
  dim3 gp((unsigned)slots, (unsigned)p.H);
  if (unbounded) {
    softplus_diag_kernel<<<gp, NTHREADS, D_SMEM, s>>>(p, static_cast<unsigned char*>(ws));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    chunk_intra_kernel<true><<<gp, NTHREADS, P_SMEM, s>>>(p, static_cast<unsigned char*>(ws));
  } else {
    chunk_intra_kernel<false><<<gp, NTHREADS, P_SMEM, s>>>(p, static_cast<unsigned char*>(ws));
  }
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
  e = cudaLaunchKernelEx(&cfg, chunk_state_kernel, p, static_cast<const unsigned char*>(ws));
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
