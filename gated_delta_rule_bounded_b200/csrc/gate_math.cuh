// gate_math.cuh -- the bounded decay gate of "Kimi K3: Bounded Decay and Delta Memory" (Formula and
// conventions, eq. 5), g = g_min * sigmoid(e^{A_h} z), as one device function shared by the gate
// kernel and by every scan kernel that reads decay logits directly. Sharing it makes a scan fed
// with logits bit-identical to the gate kernel followed by a scan fed with its output.
#pragma once

#include "kda_internal.h"

namespace kda {

// sigmoid(x) = 1 / (1 + e^-x), branch-free and without overflow for either sign: with
// t = e^-|x| = 2^(-|x| log2 e) in [0, 1], sigmoid is 1 / (1 + t) for x >= 0 and t / (1 + t) for
// x < 0. The power of two and the reciprocal are the hardware approximations (ex2.approx and
// rcp.approx, about two and one ulp); 1 + t lies in [1, 2], where rcp.approx is well inside range.
__device__ __forceinline__ float gate_sigmoid(float x) {
  float t, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(-fabsf(x) * 1.4426950408889634f));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + t));
  return x >= 0.f ? r : t * r;
}

// g = g_min * sigmoid(sc * z) with sc = e^{A_h} (computed once per head as expf(A_log[h])).
__device__ __forceinline__ float bounded_log_decay(float sc, float z, float g_min) { return g_min * gate_sigmoid(sc * z); }

// Kimi Linear's unbounded gate, the contrast of the bounded one on the same page (and the "KDA cheat
// sheet", g_min table): g = -e^{A_h} softplus(z), softplus(z) = max(z, 0) + log(1 + e^{-|z|}).
__device__ __forceinline__ float softplus_log_decay(float sc, float z) {
  return -sc * (fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))));
}

// The write strength: beta itself, or sigmoid(beta) when the scan receives its logits.
__device__ __forceinline__ float beta_value(float b, int from_logits) { return from_logits ? gate_sigmoid(b) : b; }

// Scale that L2-normalises a q or k row with squared norm `ss` (x / sqrt(ss + 1e-6)).
__device__ __forceinline__ float l2norm_scale(float ss) { return rsqrtf(ss + 1e-6f); }

// The gate input of one channel: the logits plus the optional per-(head, channel) bias b ("KDA cheat
// sheet", How the inputs are produced: z = W_up W_down x + b), or alpha / g unchanged.
__device__ __forceinline__ float gate_input(int mode, float x, float b) { return mode >= GATE_LOGITS ? x + b : x; }

// The retention factor alpha of one channel for a scan in gate mode `mode`.
__device__ __forceinline__ float gate_alpha(int mode, float x, float sc, float g_min) {
  if (mode == GATE_SOFTPLUS) return expf(softplus_log_decay(sc, x));
  return mode == GATE_LOGITS ? expf(bounded_log_decay(sc, x, g_min)) : (mode == 1 ? expf(x) : x);
}

}  // namespace kda
