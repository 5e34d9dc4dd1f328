// swa_decode_noalloc: the decode step for callers that cannot allocate device
// memory.  The split-K decode needs scratch for its partial softmax states;
// swa_decode takes it from the caller, this entry point takes it from a fixed
// array compiled into the library instead.  See include/swa.h for the contract.
#include <cuda_runtime.h>

#include <cstddef>
#include <mutex>

#include "../../include/swa.h"
#include "swa_internal.h"

namespace {

constexpr size_t kScratchBytes = 8u << 20;  // 8 MiB, held by every GPU that loads the library

// The scratch itself.  Host code must not pass this name to a kernel: on the
// host it only stands for the symbol; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SWA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return SWA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SWA_OK;
}

}  // namespace

extern "C" {

int swa_decode_noalloc(const void* q, const void* kcache, const void* vcache, const void* sink_k,
                       const void* sink_v, const int32_t* pos, void* out, float* lse, int B, int Hq,
                       int Hkv, int d, int window, int n_sink, float scale, swa_stream_t stream) {
  // swa_decode's own argument checks first, so that an error does not depend on the size.
  int st = swa::decode_args_status(q, kcache, vcache, sink_k, sink_v, pos, out, lse, B, Hq, Hkv, d, window,
                                   n_sink, scale, SWA_DTYPE_BF16);
  if (st != SWA_OK) return st;
  if (B == 0) return SWA_OK;
  const size_t need = swa_decode_workspace_bytes(B, Hq, Hkv, d, window, n_sink);
  if (need == 0) return SWA_ERR_CUDA;                    // the device could not be queried
  if (need > kScratchBytes) return SWA_ERR_UNSUPPORTED;  // the fixed scratch is too small
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != SWA_OK) return st;
  return swa_decode(q, kcache, vcache, sink_k, sink_v, pos, out, lse, B, Hq, Hkv, d, window, n_sink,
                    scale, scratch, kScratchBytes, stream);
}

}  // extern "C"
