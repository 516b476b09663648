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
// middle per-channel factor is <= 1 off the diagonal and the reciprocal of the
// block's whole decay on it, which a lower bound on g keeps in range (g >= -5
// gives at most e^80; "KDA cheat sheet", Lower-bounded decay: the bound is what
// lets every tile, the diagonal included, be a dense matmul). A block whose
// decay on some channel leaves that range (a steeper or unbounded gate, alpha
// near 0) gets its diagonal tiles pair by pair instead (diag_pairwise), with
// running products of alpha that never overflow. Q*Gamma, K*Gamma and
// K*gamma_C/Gamma are <= 1 times q or k.
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

#include "chunk_common.cuh"

namespace kda {

// Set to 1 by any chunk-kernel CTA whose bounded wait on an MMA completion expired.
__device__ int g_chunk_timeout = 0;

namespace {

// Shared-memory map of the fused kernel (bytes). Regions are reused once their first content is dead.
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
constexpr int OFF_VEC = 188928;   // fp32 vectors (VEC_*)
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

__global__ void __launch_bounds__(NTHREADS, 1) chunk_prefill_kernel(ScanParams p) {
  extern __shared__ __align__(1024) unsigned char sm[];
  const uint32_t sb = smem_u32(sm);
  constexpr IntraLayout LY{OFF_QE, OFF_KE, OFF_KC, OFF_QG, OFF_KG, OFF_KT, OFF_AKK, OFF_AQK, OFF_TP, OFF_TB, OFF_VEC};
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int quad = warp & 3, half = warp >> 2;   // TMEM lane quadrant, column half (epilogues)
  const int trow = 32 * quad + lane;             // the TMEM lane this thread moves

  const int n_vt = p.V / VT;
  int blk = blockIdx.x;
  const int vt = blk % n_vt;
  blk /= n_vt;
  const int h = blk % p.H;
  const float gsc = p.gate_mode >= GATE_LOGITS ? expf(__ldg(p.A_log + h)) : 0.f;  // e^{A_h}
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
  const float2 bias2 = load_bias2(p, h, c0);

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
  const size_t hbase = ((size_t)n * p.H + h) * (size_t)KD * p.V;  // this head's state
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    const int cb = 64 * half + 32 * part;
    uint32_t r[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      r[j] = __float_as_uint(p.s0 ? p.s0[state_at(p, hbase, cb + j, vt * VT + trow)] : 0.f);
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

    // ---- decay pass: block-local cumulative decay, scaled operand tiles, decay vectors -------------
    if (p.beta_sigmoid && tid < C) {  // beta of this chunk arrived as logits
      float* bw = reinterpret_cast<float*>(sm + OFF_BETA + (c & 1) * 256);
      bw[tid] = beta_value(bw[tid], 1);
    }
    if (p.qk_l2norm) l2norm_qk(pf, vec + VEC_D, tid, da);
    int pairwise;  // blocks whose diagonal tiles are formed pair by pair
    {
      float2 al[16];
      decay_step1(sm, LY, pf, nv, da, c0, p.gate_mode, gsc, p.g_min, bias2, al);
      __syncthreads();
      pairwise = pairwise_blocks(sm, LY);
      decay_step2(sm, LY, pf, da, c0, al);
      if (pairwise) diag_pairwise(sm, LY, pf, al, beta_s, da, pairwise);  // CTA-uniform
    }
    __syncthreads();  // scaled tiles and vectors ready; the q/k/g registers are free

    if (has_next) load_qkg(x, tn0, nvn, c0, da, pf);

    // ---- A_kk, then the inverse (warps 0-3) alongside A_qk (warps 4-7) ----------------------------
    intra_phases(sm, sb, LY, beta_s, tid, warp, lane, g, tq, pairwise);
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
    ok = __syncthreads_and(mbar_wait(bar, phase, &g_chunk_timeout));  // one decision for the whole CTA
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
    ok = __syncthreads_and(mbar_wait(bar, phase, &g_chunk_timeout));  // one decision for the whole CTA
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
    ok = __syncthreads_and(mbar_wait(bar, phase, &g_chunk_timeout));  // one decision for the whole CTA
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
      for (int j = 0; j < 32; ++j) p.sf[state_at(p, hbase, cb + j, vt * VT + trow)] = __uint_as_float(r[j]);
    }
  }
  if (!ok) {
    // A wait expired: give any MMA still in flight one more bounded wait before releasing TMEM.
    mbar_wait(bar, phase, &g_chunk_timeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TM_COLS));
}

}  // namespace

bool chunk_supported(int K, int V, kda_dtype dt) { return dt == KDA_BF16 && K == KD && V % VT == 0; }

size_t chunk_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t n_seq) {
  return split_workspace_bytes(B, T, H, n_seq > 0 ? n_seq : B, n_seq > 0);
}

cudaError_t launch_chunk(const ScanParams& p, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (ws != nullptr && ws_bytes >= split_workspace_bytes(p.B, p.T, p.H, p.N, p.cu != nullptr) && split_maps_ok(p))
    return launch_chunk_split(p, ws, s);
  // The shared-memory opt-in is per device; remember which devices have it.
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;  // one configuration bit per device
  const uint64_t bit = 1ull << dev;
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
