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
// into a per-CTA scratch before the adjoint sweeps it in reverse.
//
// The per-token work is short, so latency decides the speed: every segment's inputs (gate, k, v,
// beta, and q, do for the adjoint) are brought into shared memory with one batch of asynchronous
// copies, and during the adjoint the state S_{t-2} is copied from the scratch into a shared-memory
// ring while token t is processed. Sums over key rows go through shared memory; the per-row sums
// over value columns (dq, dk, dalpha) are warp reduce-scatters, one shuffle per value and level.
#include "common.cuh"
#include "gate_math.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kGroups = 8;  // key-row groups
constexpr int kSeg = 32;    // tokens per checkpoint segment

constexpr int align16(int x) { return (x + 15) & ~15; }

// Dynamic shared memory (byte offsets): one segment's inputs, the key-row partial sums and the
// two-slot ring of scratch states (slot, row r, thread: float4).
template <int RPT, int VT, typename TIn>
struct BwdSmem {
  static constexpr int K = kGroups * RPT;
  static constexpr int NT = kGroups * (VT / 4);
  static constexpr int GATE = 0;                                                  // float [kSeg][K]
  static constexpr int KK = GATE + kSeg * K * 4;                                  // TIn [kSeg][K]
  static constexpr int Q = align16(KK + kSeg * K * (int)sizeof(TIn));             // TIn [kSeg][K]
  static constexpr int V = align16(Q + kSeg * K * (int)sizeof(TIn));              // TIn [kSeg][VT]
  static constexpr int DO = align16(V + kSeg * VT * (int)sizeof(TIn));            // float [kSeg][VT]
  static constexpr int BETA = DO + kSeg * VT * 4;                                 // float [kSeg]
  static constexpr int RED = align16(BETA + kSeg * 4);                            // float [kGroups][VT]
  static constexpr int RING = align16(RED + kGroups * VT * 4);                    // float4 [2][RPT][NT]
  static constexpr int BYTES = RING + 2 * RPT * NT * 16;
};

__device__ __forceinline__ uint32_t shared_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(shared_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(shared_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Sum over the VT/4 column-group threads of one row group (consecutive lanes).
template <int VT>
__device__ __forceinline__ float rowgroup_sum(float x) {
#pragma unroll
  for (int m = VT / 8; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// Sums v[r] (r < N, one value per key row of this thread) over the CG threads of the row group.
// Each level exchanges half of the live values with the partner lane, so afterwards this lane
// holds the totals of NR = max(1, N / CG) consecutive rows starting at `first` in v[0..NR).
// With N < CG, CG / N lanes hold the same row; the one whose low bits are zero reports it (`own`).
template <int N, int CG>
__device__ __forceinline__ void rowgroup_reduce_scatter(float (&v)[N], int tv, int& first, bool& own) {
  first = 0;
  int n = N;
#pragma unroll
  for (int m = CG / 2; m >= 1; m >>= 1) {
    if (n > 1) {
      const bool up = (tv & m) != 0;
      const int hn = n / 2;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < hn) {
          const float send = up ? v[i] : v[i + hn];
          const float keep = up ? v[i + hn] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      if (up) first += hn;
      n = hn;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
  own = N >= CG || (tv & (CG / N - 1)) == 0;
}

// N consecutive per-row values (N = 2 or 4) from shared memory, as fp32: one vector load. All lanes
// of a warp read the same rows, so the load is a broadcast.
template <int N>
__device__ __forceinline__ void lds_rows(const float* p, float (&r)[N]) {
  if constexpr (N == 4) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    r[0] = x.x; r[1] = x.y; r[2] = x.z; r[3] = x.w;
  } else {
    const float2 x = *reinterpret_cast<const float2*>(p);
    r[0] = x.x; r[1] = x.y;
  }
}
template <int N>
__device__ __forceinline__ void lds_rows(const __nv_bfloat16* p, float (&r)[N]) {
  if constexpr (N == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    r[0] = __uint_as_float(x.x << 16); r[1] = __uint_as_float(x.x & 0xffff0000u);
    r[2] = __uint_as_float(x.y << 16); r[3] = __uint_as_float(x.y & 0xffff0000u);
  } else {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
    r[0] = __uint_as_float(x << 16); r[1] = __uint_as_float(x & 0xffff0000u);
  }
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

// LOGG: the gate is g = log(alpha). Then dL/dg = rowsum(dSbar * Sbar), so the adjoint keeps Sbar itself in
// the registers of S_{t-1} and never needs S_{t-1} again; with alpha given, dL/dalpha needs S_{t-1} and
// Sbar is formed where it is used.
template <int RPT, int VT, typename TIn, bool LOGG>
__global__ void __launch_bounds__(kGroups * (VT / 4), 1) scan_backward_kernel(BwdParams p) {
  using L = BwdSmem<RPT, VT, TIn>;
  constexpr int K = L::K, CG = VT / 4, NT = L::NT;
  constexpr int NR = RPT > CG ? RPT / CG : 1;  // rows per lane after a reduce-scatter
  constexpr int RG = RPT >= 4 ? 4 : RPT;       // rows per vector load of the per-row values
  extern __shared__ __align__(16) unsigned char smb[];
  float* sa = reinterpret_cast<float*>(smb + L::GATE);
  TIn* sk = reinterpret_cast<TIn*>(smb + L::KK);
  TIn* sq = reinterpret_cast<TIn*>(smb + L::Q);
  TIn* sv = reinterpret_cast<TIn*>(smb + L::V);
  float* sdo = reinterpret_cast<float*>(smb + L::DO);
  float* sbeta = reinterpret_cast<float*>(smb + L::BETA);
  float* red = reinterpret_cast<float*>(smb + L::RED);
  float4* ring = reinterpret_cast<float4*>(smb + L::RING);

  const int tid = threadIdx.x, tv = tid % CG, tk = tid / CG;
  const int row0 = tk * RPT, col0 = 4 * tv;
  const int bh = blockIdx.x, seq = bh / p.H, h = bh % p.H;  // (sequence or batch row, head)
  const int64_t T = p.T;  // tokens per batch row (the packed total with cu_seqlens)
  const size_t slice = (size_t)K * VT;
  // This CTA's tokens are ts .. ts + len - 1 of batch row b.
  int b = seq;
  int64_t ts = 0, len = T;
  float* ckpt;  // state before token ts + j*kSeg, j = 0..n_seg
  if (p.cu) {
    const int64_t t1 = min((int64_t)p.cu[seq + 1], T);
    ts = max((int64_t)0, min((int64_t)p.cu[seq], t1));
    len = t1 - ts;
    b = 0;
    ckpt = p.ckpt + ((size_t)h * p.ckpt_slots + (size_t)(ts / kSeg) + 2 * (size_t)seq) * slice;
  } else {
    ckpt = p.ckpt + (size_t)bh * ((T + kSeg - 1) / kSeg + 1) * slice;
  }
  const int n_seg = (int)((len + kSeg - 1) / kSeg);
  float* scr = p.scratch + (size_t)bh * kSeg * slice;  // states before each token of a segment
  const TIn* qb = static_cast<const TIn*>(p.q);
  const TIn* kb = static_cast<const TIn*>(p.k);
  const TIn* vb = static_cast<const TIn*>(p.v);
  auto tile = [&](float* base, int r) { return reinterpret_cast<float4*>(base + (size_t)(row0 + r) * VT + col0); };

  // Brings tokens t0 .. t0+n-1 into shared memory (q and do as well when `adj`) and turns the gate
  // into alpha. Every row starts on a 16-byte boundary (checked by the host).
  auto stage_segment = [&](int64_t t0, int n, bool adj) {
    constexpr int PK = K * (int)sizeof(TIn) / 16, PV = VT * (int)sizeof(TIn) / 16;  // 16-byte pieces per row
    for (int i = tid; i < n * (K / 4); i += NT) {
      const int tt = i / (K / 4), c = 4 * (i % (K / 4));
      cp_async16(sa + tt * K + c, p.gate + b * p.gs[0] + (t0 + tt) * p.gs[1] + h * p.gs[2] + c);
    }
    for (int i = tid; i < n * PK; i += NT) {
      const int tt = i / PK, c = (i % PK) * (16 / (int)sizeof(TIn));
      cp_async16(sk + tt * K + c, kb + b * p.ks[0] + (t0 + tt) * p.ks[1] + h * p.ks[2] + c);
      if (adj) cp_async16(sq + tt * K + c, qb + b * p.qs[0] + (t0 + tt) * p.qs[1] + h * p.qs[2] + c);
    }
    for (int i = tid; i < n * PV; i += NT) {
      const int tt = i / PV, c = (i % PV) * (16 / (int)sizeof(TIn));
      cp_async16(sv + tt * VT + c, vb + b * p.vs[0] + (t0 + tt) * p.vs[1] + h * p.vs[2] + c);
    }
    if (adj) {
      for (int i = tid; i < n * (VT / 4); i += NT) {
        const int tt = i / (VT / 4), c = 4 * (i % (VT / 4));
        cp_async16(sdo + tt * VT + c, p.d_o + ((b * T + t0 + tt) * p.H + h) * (int64_t)VT + c);
      }
    }
    for (int i = tid; i < n; i += NT) cp_async4(sbeta + i, p.beta + b * p.bs[0] + (t0 + i) * p.bs[1] + h * p.bs[2]);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    if (p.gate_log)
      for (int i = tid; i < n * K; i += NT) sa[i] = expf(sa[i]);
    __syncthreads();
  };

  // One forward step on the registers x (S_{t-1} -> S_t) for staged token tt.
  auto forward_step = [&](float4 (&x)[RPT], int tt) {
    const float* a_ = sa + tt * K + row0;
    const TIn* k_ = sk + tt * K + row0;
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int rr = 0; rr < RPT; rr += RG) {
      float av[RG], kv[RG];
      lds_rows<RG>(a_ + rr, av);
      lds_rows<RG>(k_ + rr, kv);
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        const int r = rr + j;
        const float a = av[j], kk = kv[j];
        x[r].x *= a; x[r].y *= a; x[r].z *= a; x[r].w *= a;
        pa.x = fmaf(kk, x[r].x, pa.x); pa.y = fmaf(kk, x[r].y, pa.y);
        pa.z = fmaf(kk, x[r].z, pa.z); pa.w = fmaf(kk, x[r].w, pa.w);
      }
    }
    *reinterpret_cast<float4*>(red + tk * VT + col0) = pa;
    __syncthreads();
    const float4 A = colsum<RPT, VT>(red, col0);
    const float beta = sbeta[tt];
    const TIn* v_ = sv + tt * VT;
    const float4 d = make_float4(to_f32(v_[col0]) - A.x, to_f32(v_[col0 + 1]) - A.y, to_f32(v_[col0 + 2]) - A.z,
                                 to_f32(v_[col0 + 3]) - A.w);
#pragma unroll
    for (int rr = 0; rr < RPT; rr += RG) {
      float kv[RG];
      lds_rows<RG>(k_ + rr, kv);
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        const int r = rr + j;
        const float bk = beta * kv[j];
        x[r].x = fmaf(bk, d.x, x[r].x); x[r].y = fmaf(bk, d.y, x[r].y);
        x[r].z = fmaf(bk, d.z, x[r].z); x[r].w = fmaf(bk, d.w, x[r].w);
      }
    }
    __syncthreads();  // red is free again
  };

  // ---- checkpoints: the state before every kSeg-th token --------------------------------------------
  float4 x[RPT];
  const size_t sbase = (size_t)bh * K * VT;
#pragma unroll
  for (int r = 0; r < RPT; ++r) x[r] = p.s0 ? *reinterpret_cast<const float4*>(p.s0 + sbase + (size_t)(row0 + r) * VT + col0)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int seg = 0; seg < n_seg; ++seg) {
    const int64_t t0 = ts + (int64_t)seg * kSeg;
    const int n = (int)min((int64_t)kSeg, ts + len - t0);
#pragma unroll
    for (int r = 0; r < RPT; ++r) *tile(ckpt + (size_t)seg * slice, r) = x[r];
    stage_segment(t0, n, false);
    for (int tt = 0; tt < n; ++tt) forward_step(x, tt);
    __syncthreads();  // the staged segment is free again
  }

  // ---- adjoint, segment by segment from the end -------------------------------------------------------
  float4 G[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) G[r] = p.d_sf ? *reinterpret_cast<const float4*>(p.d_sf + sbase + (size_t)(row0 + r) * VT + col0)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
  // This thread's float4 of row r in ring slot j (consecutive threads, consecutive 16 bytes).
  auto ring_at = [&](int j, int r) { return ring + (j * RPT + r) * NT + tid; };
  auto fetch = [&](int tt) {  // S_{t0+tt-1} from the scratch into ring slot tt & 1
#pragma unroll
    for (int r = 0; r < RPT; ++r) cp_async16(ring_at(tt & 1, r), tile(scr + (size_t)tt * slice, r));
    cp_async_commit();
  };
  for (int seg = n_seg - 1; seg >= 0; --seg) {
    const int64_t t0 = ts + (int64_t)seg * kSeg;
    const int n = (int)min((int64_t)kSeg, ts + len - t0);
#pragma unroll
    for (int r = 0; r < RPT; ++r) x[r] = *tile(ckpt + (size_t)seg * slice, r);
    stage_segment(t0, n, true);
    for (int tt = 0; tt < n; ++tt) {  // recompute: scr[tt] = S_{t0+tt-1}
#pragma unroll
      for (int r = 0; r < RPT; ++r) *tile(scr + (size_t)tt * slice, r) = x[r];
      forward_step(x, tt);
    }
    fetch(n - 1);  // this thread reads back only what it wrote itself
    for (int tt = n - 1; tt >= 0; --tt) {
      const int64_t t = t0 + tt;
      if (tt > 0) {
        fetch(tt - 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
#pragma unroll
      for (int r = 0; r < RPT; ++r) x[r] = *ring_at(tt & 1, r);  // S_{t-1}
      const float* a_ = sa + tt * K + row0;
      const TIn* k_ = sk + tt * K + row0;
      const TIn* q_ = sq + tt * K + row0;
      const TIn* v_ = sv + tt * VT;
      const float beta = sbeta[tt];
      // delta from Sbar = Diag(alpha) S_{t-1}: with LOGG x becomes Sbar here, otherwise Sbar is formed
      // from S_{t-1} where it is needed
      auto sbar = [&](int r, float a) {
        return LOGG ? x[r] : make_float4(a * x[r].x, a * x[r].y, a * x[r].z, a * x[r].w);
      };
      float4 pa = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int rr = 0; rr < RPT; rr += RG) {
        float av[RG], kv[RG];
        lds_rows<RG>(a_ + rr, av);
        lds_rows<RG>(k_ + rr, kv);
#pragma unroll
        for (int j = 0; j < RG; ++j) {
          const int r = rr + j;
          const float kk = kv[j];
          if (LOGG) {
            const float a = av[j];
            x[r].x *= a; x[r].y *= a; x[r].z *= a; x[r].w *= a;
          }
          const float4 xb = sbar(r, av[j]);
          pa.x = fmaf(kk, xb.x, pa.x); pa.y = fmaf(kk, xb.y, pa.y);
          pa.z = fmaf(kk, xb.z, pa.z); pa.w = fmaf(kk, xb.w, pa.w);
        }
      }
      *reinterpret_cast<float4*>(red + tk * VT + col0) = pa;
      __syncthreads();
      const float4 A = colsum<RPT, VT>(red, col0);
      const float4 d = make_float4(to_f32(v_[col0]) - A.x, to_f32(v_[col0 + 1]) - A.y, to_f32(v_[col0 + 2]) - A.z,
                                   to_f32(v_[col0 + 3]) - A.w);
      const float4 dov = *reinterpret_cast<const float4*>(sdo + tt * VT + col0);
      __syncthreads();  // red is reused below
      // G += q do^T (the output's share), dq = S_t do, and c = G^T k
      float4 pc = make_float4(0.f, 0.f, 0.f, 0.f);
      float rq[RPT];
#pragma unroll
      for (int rr = 0; rr < RPT; rr += RG) {
        float av[RG], kv[RG], qv[RG];
        lds_rows<RG>(a_ + rr, av);
        lds_rows<RG>(k_ + rr, kv);
        lds_rows<RG>(q_ + rr, qv);
#pragma unroll
        for (int j = 0; j < RG; ++j) {
          const int r = rr + j;
          const float qq = qv[j], kk = kv[j], bk = beta * kk;
          G[r].x = fmaf(qq, dov.x, G[r].x); G[r].y = fmaf(qq, dov.y, G[r].y);
          G[r].z = fmaf(qq, dov.z, G[r].z); G[r].w = fmaf(qq, dov.w, G[r].w);
          const float4 xb = sbar(r, av[j]);
          const float4 st = make_float4(fmaf(bk, d.x, xb.x), fmaf(bk, d.y, xb.y), fmaf(bk, d.z, xb.z), fmaf(bk, d.w, xb.w));
          rq[r] = st.x * dov.x + st.y * dov.y + st.z * dov.z + st.w * dov.w;
          pc.x = fmaf(kk, G[r].x, pc.x); pc.y = fmaf(kk, G[r].y, pc.y);
          pc.z = fmaf(kk, G[r].z, pc.z); pc.w = fmaf(kk, G[r].w, pc.w);
        }
      }
      *reinterpret_cast<float4*>(red + tk * VT + col0) = pc;
      const int64_t orow = ((b * T + t) * p.H + h) * (int64_t)K + row0;
      {
        int first;
        bool own;
        rowgroup_reduce_scatter<RPT, CG>(rq, tv, first, own);
        if (own) {
#pragma unroll
          for (int i = 0; i < NR; ++i) p.dq[orow + first + i] = rq[i];
        }
      }
      __syncthreads();
      const float4 c = colsum<RPT, VT>(red, col0);
      const float4 dd = make_float4(beta * c.x, beta * c.y, beta * c.z, beta * c.w);  // dL/d delta = dv
      // delta and c are per-column values, equal in every row group: each group forms the same dbeta.
      const float db = rowgroup_sum<VT>(d.x * c.x + d.y * c.y + d.z * c.z + d.w * c.w);
      if (tk == 0) {
        *reinterpret_cast<float4*>(p.dv + ((b * T + t) * p.H + h) * (int64_t)VT + col0) = dd;
        if (tv == 0) p.dbeta[(b * T + t) * p.H + h] = db;
      }
      float rk[RPT], ra[RPT];
#pragma unroll
      for (int rr = 0; rr < RPT; rr += RG) {
        float av[RG], kv[RG];
        lds_rows<RG>(a_ + rr, av);
        lds_rows<RG>(k_ + rr, kv);
#pragma unroll
        for (int j = 0; j < RG; ++j) {
          const int r = rr + j;
          const float kk = kv[j], a = av[j];
          const float4 xb = sbar(r, a);
          rk[r] = beta * (G[r].x * d.x + G[r].y * d.y + G[r].z * d.z + G[r].w * d.w) -
                  (xb.x * dd.x + xb.y * dd.y + xb.z * dd.z + xb.w * dd.w);
          const float4 ds = make_float4(G[r].x - kk * dd.x, G[r].y - kk * dd.y, G[r].z - kk * dd.z, G[r].w - kk * dd.w);
          ra[r] = ds.x * x[r].x + ds.y * x[r].y + ds.z * x[r].z + ds.w * x[r].w;  // LOGG: dL/dg, else dL/dalpha
          G[r] = make_float4(a * ds.x, a * ds.y, a * ds.z, a * ds.w);
        }
      }
      {
        int first;
        bool own;
        rowgroup_reduce_scatter<RPT, CG>(rk, tv, first, own);
        rowgroup_reduce_scatter<RPT, CG>(ra, tv, first, own);
        if (own) {
#pragma unroll
          for (int i = 0; i < NR; ++i) {
            p.dk[orow + first + i] = rk[i];
            p.dgate[orow + first + i] = ra[i];
          }
        }
      }
      __syncthreads();  // red is free again
    }
    __syncthreads();  // the staged segment is free again
  }
  if (p.ds0) {
#pragma unroll
    for (int r = 0; r < RPT; ++r) *reinterpret_cast<float4*>(p.ds0 + sbase + (size_t)(row0 + r) * VT + col0) = G[r];
  }
}

template <int RPT, int VT, typename TIn, bool LOGG>
cudaError_t launch_bg(const BwdParams& p, cudaStream_t s) {
  constexpr int bytes = BwdSmem<RPT, VT, TIn>::BYTES;
  static_assert(bytes <= 227 * 1024, "shared memory budget");
  auto kern = scan_backward_kernel<RPT, VT, TIn, LOGG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(p.N * p.H), kGroups * (VT / 4), bytes, s>>>(p);
  return cudaGetLastError();
}

template <int RPT, int VT, typename TIn>
cudaError_t launch_b(const BwdParams& p, cudaStream_t s) {
  return p.gate_log ? launch_bg<RPT, VT, TIn, true>(p, s) : launch_bg<RPT, VT, TIn, false>(p, s);
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
// with x = e^A z and s = sigmoid(x) (the same device sigmoid as the forward gate). One block per
// (head, slice of the rows); the block sums its share of dA_log[h] and adds it with one atomic.
template <int VW>
struct VecF;
template <>
struct VecF<1> {
  using T = float;
};
template <>
struct VecF<4> {
  using T = float4;
};

template <int VW>
__global__ void __launch_bounds__(256) bounded_decay_backward_kernel(const float* __restrict__ z,
                                                                     const float* __restrict__ A_log, float g_min,
                                                                     const float* __restrict__ dg, int64_t rows_bt,
                                                                     int H, int K, float* __restrict__ dz,
                                                                     float* __restrict__ dA) {
  using VT = typename VecF<VW>::T;
  constexpr int U = 4;  // independent elements in flight per thread
  const int h = blockIdx.x;
  const int tpr = K / VW;  // vectors per (b, t) row of this head
  const float sc = expf(__ldg(A_log + h));
  const int64_t n = rows_bt * tpr, stride = (int64_t)gridDim.y * blockDim.x;
  float acc = 0.f;
  for (int64_t e0 = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; e0 < n; e0 += U * stride) {
    VT zv[U], gv[U];
    int64_t off[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t e = e0 + u * stride;
      off[u] = -1;
      if (e < n) {
        const int64_t r = e / tpr;
        off[u] = ((r * H + h) * K) / VW + (e - r * tpr);
        zv[u] = reinterpret_cast<const VT*>(z)[off[u]];
        gv[u] = reinterpret_cast<const VT*>(dg)[off[u]];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (off[u] < 0) continue;
      const float* zf = reinterpret_cast<const float*>(&zv[u]);
      const float* gf = reinterpret_cast<const float*>(&gv[u]);
      VT out;
      float* of = reinterpret_cast<float*>(&out);
#pragma unroll
      for (int c = 0; c < VW; ++c) {
        const float x = sc * zf[c];
        const float s = gate_sigmoid(x);
        const float w = gf[c] * g_min * s * (1.f - s);
        of[c] = w * sc;
        acc = fmaf(w, x, acc);
      }
      reinterpret_cast<VT*>(dz)[off[u]] = out;
    }
  }
  __shared__ float part[8];
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
    atomicAdd(dA + h, t);
  }
}

}  // namespace

int64_t backward_ckpt_slots(int64_t T, int64_t n_seq) {
  return n_seq > 0 ? T / kSeg + 2 * n_seq + 1 : (T + kSeg - 1) / kSeg + 1;
}

bool backward_supported(int K, int V) {
  return (K == 16 || K == 32 || K == 64 || K == 128) && (V == 16 || V == 32 || V == 64 || V == 128);
}

size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V, int64_t n_seq) {
  const size_t slice = (size_t)K * V * sizeof(float);
  if (n_seq > 0)  // checkpoints shared per head, scratch per (sequence, head)
    return (size_t)H * backward_ckpt_slots(T, n_seq) * slice + (size_t)n_seq * H * kSeg * slice;
  return (size_t)B * H * (size_t)(backward_ckpt_slots(T, 0) + kSeg) * slice;
}

cudaError_t launch_scan_backward(const BwdParams& p, kda_dtype dt, cudaStream_t s) {
  return dt == KDA_F32 ? launch_bk<float>(p, s) : launch_bk<__nv_bfloat16>(p, s);
}

cudaError_t launch_bounded_decay_backward(const float* z, const float* A_log, float g_min, const float* dg,
                                          int64_t rows_bt, int H, int K, float* dz, float* dA, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(dA, 0, sizeof(float) * H, s);
  if (e != cudaSuccess) return e;
  if (rows_bt * K == 0) return cudaSuccess;
  const bool vec = K % 4 == 0 && ((reinterpret_cast<uintptr_t>(z) | reinterpret_cast<uintptr_t>(dg) |
                                   reinterpret_cast<uintptr_t>(dz)) & 15) == 0;
  const int64_t per_head = rows_bt * (vec ? K / 4 : K);
  int64_t ny = (per_head + 255) / 256;
  const int64_t cap = (148 * 8 + H - 1) / H;
  if (ny > cap) ny = cap;
  if (ny > 65535) ny = 65535;
  const dim3 grid((unsigned)H, (unsigned)ny);
  if (vec)
    bounded_decay_backward_kernel<4><<<grid, 256, 0, s>>>(z, A_log, g_min, dg, rows_bt, H, K, dz, dA);
  else
    bounded_decay_backward_kernel<1><<<grid, 256, 0, s>>>(z, A_log, g_min, dg, rows_bt, H, K, dz, dA);
  return cudaGetLastError();
}

}  // namespace kda
