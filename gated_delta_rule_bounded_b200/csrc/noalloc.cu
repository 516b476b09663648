// noalloc.cu -- kda_prefill_noalloc: the prefill for callers that cannot allocate device memory.
//
// kda_prefill's two-kernel path needs a device workspace (66,048 bytes per 64-token chunk and
// head) that the caller allocates. Some callers have no device allocator to hand: a plain C host
// that links only libkda and owns no CUDA allocator, or a serving loop that must not call
// cudaMalloc / cudaFree between steps because those calls synchronise the device. For them this
// entry point takes its workspace from a fixed scratch array compiled into the library (a
// file-scope __device__ array: the CUDA runtime provides one copy per device when it loads this
// file's module) and allocates nothing. Arguments, validation and kernels are kda_prefill's.
//
// Setup: the first call on a device looks up the scratch's device address with
// cudaGetSymbolAddress (which also loads this module on that device under lazy loading) and
// caches it; later calls on that device only read the cache. The cached address belongs to the
// device's primary context, so a device reset between calls is not supported. Under eager module
// loading the array is reserved on every device the library loads on, whether or not this call runs.
//
// Sharing: every call on a device uses the same array. The first kernel of a call writes every
// block the second kernel reads, so nothing in it has to start at zero, but two calls whose work
// overlaps on the GPU (different streams, or different host threads, without ordering between
// them) race on it.
#include <cstdio>
#include <mutex>

#include "kda.h"
#include "kda_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_prefill_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per device.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prefill_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int kda_prefill_noalloc(const void* q, const void* k, const void* v, kda_dtype dtype,
                                   const float* gate, kda_gate_kind gate_kind, const float* beta,
                                   const float* initial_state, float* final_state,
                                   const int32_t* cu_seqlens, int64_t n_seq,
                                   int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                   const kda_layout* layout, void* o, kda_stream_t stream) {
  size_t need = 0;
  int rc = kda_prefill_workspace_bytes(B, T, H, K, V, cu_seqlens ? n_seq : 0, dtype, &need);
  if (rc != KDA_OK) return rc;
  if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES) {
    char msg[320];
    snprintf(msg, sizeof(msg),
             "kda_prefill_noalloc: these sizes need %zu bytes of scratch but the library's static scratch holds "
             "%zu; call kda_prefill with a caller-allocated workspace instead",
             need, (size_t)KDA_NOALLOC_SCRATCH_BYTES);
    return kda::report_error(KDA_ERR_UNSUPPORTED, msg);
  }
  void* scratch = nullptr;
  if (need > 0) {
    cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
      char msg[320];
      snprintf(msg, sizeof(msg), "kda_prefill_noalloc: cudaGetSymbolAddress of the scratch failed: %s (%s)",
               cudaGetErrorName(e), cudaGetErrorString(e));
      return kda::report_error(KDA_ERR_CUDA, msg);
    }
  }
  return kda_prefill(q, k, v, dtype, gate, gate_kind, beta, initial_state, final_state, cu_seqlens, n_seq, B, T, H, K,
                     V, layout, o, scratch, need > 0 ? (size_t)KDA_NOALLOC_SCRATCH_BYTES : 0, stream);
}
