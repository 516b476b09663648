// gate.cu -- bounded decay gate ("Kimi K3: Bounded Decay and Delta Memory", eq. 5):
//   g = g_min * sigmoid(exp(A_h) * z),  alpha = exp(g).
// Elementwise and HBM-bound: a warp owns a (b, t, h) row and each lane four
// consecutive channels (16-byte fp32 or 8-byte bf16 accesses); the grid is a
// multiple of the SM count and strides over all rows.
#include "common.cuh"
#include "gate_math.cuh"
#include "kda_internal.h"

namespace kda {

// One warp per (b, t, h) row: the row's coordinates are decomposed once (32-bit
// arithmetic), A_log is read once, and the lanes stride over its K/4 channel
// quads. Each warp takes RPW consecutive rows per step and issues all their
// loads before any arithmetic, so every lane keeps RPW 16-byte loads in flight.
constexpr int RPW = 4;

template <typename T>
__global__ void __launch_bounds__(256) bounded_decay_kernel(GateParams p) {
  const int lane = threadIdx.x & 31;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t rows = (uint32_t)(p.B * p.T * p.H);
  const uint32_t H = (uint32_t)p.H, Tn = (uint32_t)p.T;
  const int quads = (int)(p.K / 4);
  for (uint32_t r0 = warp * RPW; r0 < rows; r0 += nwarps * RPW) {
    for (int c4 = lane; c4 < quads; c4 += 32) {
      float4 z[RPW];
      const T* zp[RPW];
      T* op[RPW];
      float scale[RPW];
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        const uint32_t r = min(r0 + i, rows - 1);  // clamped rows are recomputed, never out of range
        const uint32_t h = r % H, bt = r / H;
        const uint32_t t = bt % Tn, b = bt / Tn;
        zp[i] = static_cast<const T*>(p.z) + b * p.zs[0] + t * p.zs[1] + h * p.zs[2] + 4 * c4;
        op[i] = static_cast<T*>(p.out) + b * p.os[0] + t * p.os[1] + h * p.os[2] + 4 * c4;
        scale[i] = __ldg(p.A_log + h);
      }
#pragma unroll
      for (int i = 0; i < RPW; ++i) z[i] = load4(zp[i]);
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        if (r0 + i >= rows) break;
        const float sc = expf(scale[i]);
        float4 g;
        g.x = p.softplus ? softplus_log_decay(sc, z[i].x) : bounded_log_decay(sc, z[i].x, p.g_min);
        g.y = p.softplus ? softplus_log_decay(sc, z[i].y) : bounded_log_decay(sc, z[i].y, p.g_min);
        g.z = p.softplus ? softplus_log_decay(sc, z[i].z) : bounded_log_decay(sc, z[i].z, p.g_min);
        g.w = p.softplus ? softplus_log_decay(sc, z[i].w) : bounded_log_decay(sc, z[i].w, p.g_min);
        if (!p.out_log) {
          g.x = expf(g.x);
          g.y = expf(g.y);
          g.z = expf(g.z);
          g.w = expf(g.w);
        }
        store4(op[i], g);
      }
    }
  }
}

cudaError_t launch_gate(const GateParams& p, kda_dtype dt, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows = p.B * p.T * p.H;  // RPW rows per warp step, 8 warps per block
  const int64_t want = (rows + 8 * RPW - 1) / (8 * RPW);
  const int64_t cap = (int64_t)sms * 8;   // 8 resident 256-thread blocks per SM
  int grid = (int)(want < cap ? want : cap);
  if (grid < 1) grid = 1;
  if (dt == KDA_F32)
    bounded_decay_kernel<float><<<grid, 256, 0, s>>>(p);
  else
    bounded_decay_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
