// gate.cu -- bounded decay gate ("Kimi K3: Bounded Decay and Delta Memory", eq. 5):
//   g = g_min * sigmoid(exp(A_h) * z),  alpha = exp(g).
// Elementwise and HBM-bound: each thread handles four consecutive channels of a
// (b, t, h) row with 16-byte (fp32) or 8-byte (bf16) accesses; the grid is a
// multiple of the SM count and strides over all rows.
#include "common.cuh"
#include "kda_internal.h"

namespace kda {

__device__ __forceinline__ float gate_sigmoid(float x) {
  // Evaluated without overflow for either sign.
  if (x >= 0.f) return 1.f / (1.f + expf(-x));
  float e = expf(x);
  return e / (1.f + e);
}

template <typename T>
__global__ void __launch_bounds__(256) bounded_decay_kernel(GateParams p) {
  const int64_t quads = p.K / 4;
  const int64_t total = p.B * p.T * p.H * quads;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    int64_t c4 = i % quads;
    int64_t r = i / quads;
    int64_t h = r % p.H;
    r /= p.H;
    int64_t t = r % p.T;
    int64_t b = r / p.T;
    const T* zp = static_cast<const T*>(p.z) + b * p.zs[0] + t * p.zs[1] + h * p.zs[2] + 4 * c4;
    T* op = static_cast<T*>(p.out) + b * p.os[0] + t * p.os[1] + h * p.os[2] + 4 * c4;
    float scale = expf(__ldg(p.A_log + h));
    float4 z = load4(zp);
    float4 g;
    g.x = p.g_min * gate_sigmoid(scale * z.x);
    g.y = p.g_min * gate_sigmoid(scale * z.y);
    g.z = p.g_min * gate_sigmoid(scale * z.z);
    g.w = p.g_min * gate_sigmoid(scale * z.w);
    if (!p.out_log) {
      g.x = expf(g.x);
      g.y = expf(g.y);
      g.z = expf(g.z);
      g.w = expf(g.w);
    }
    store4(op, g);
  }
}

cudaError_t launch_gate(const GateParams& p, kda_dtype dt, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t total = p.B * p.T * p.H * (p.K / 4);
  int64_t want = (total + 255) / 256;
  int64_t cap = (int64_t)sms * 8;  // 8 resident 256-thread blocks per SM
  int grid = (int)(want < cap ? want : cap);
  if (grid < 1) grid = 1;
  if (dt == KDA_F32)
    bounded_decay_kernel<float><<<grid, 256, 0, s>>>(p);
  else
    bounded_decay_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
