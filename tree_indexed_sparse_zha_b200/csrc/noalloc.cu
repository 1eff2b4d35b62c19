// zha_decode_noalloc: zha_decode with its workspace in a static device array.
//
// For callers that cannot hand the library a workspace: plugins loaded by a
// host that owns the device allocator and exposes none of it, and hot paths
// where an allocation is not allowed (cudaMalloc/cudaFree synchronise the
// device). The scratch is a static device array of this library: with the
// CUDA runtime's default lazy module loading its 64 MiB are reserved on a
// device only once a program calls this entry point there; with eager loading
// (CUDA_MODULE_LOADING=EAGER) every process that loads libzha reserves them on
// every device it uses, until exit.
#include <cuda_runtime.h>

#include <mutex>

#include "zha_internal.h"

namespace {

// Largest ZHA_OP_DECODE workspace this entry point serves (zha_workspace_bytes
// gives a geometry's need): e.g. B = 1, Hkv = 2, G = 8, b = 4, L = 6 fits up
// to about 2.19M tokens of context.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once per
// device (the first call on a device loads this module there). The address is
// kept for the life of the process: a device reset (cudaDeviceReset, or the
// primary context destroyed and re-created) between calls would leave it
// stale, so callers of this entry point must not reset the device.
zha_status static_scratch(void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return ZHA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return ZHA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return ZHA_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return ZHA_OK;
}

}  // namespace

extern "C" {

zha_status zha_decode_noalloc(const zha_config* cfg, const zha_cache* cache, const void* q,
                              double p, void* out, int32_t* level_counts, int32_t* dev_status,
                              void* stream) {
  size_t need = 0;
  zha_status st = zha_workspace_bytes(cfg, ZHA_OP_DECODE, 0, &need);
  if (st != ZHA_OK) return st;
  if (need > kStaticScratchBytes) return ZHA_ERR_WORKSPACE;  // geometry beyond the static size
  void* ws = nullptr;
  if ((st = static_scratch(&ws)) != ZHA_OK) return st;
  // Nothing in the decode workspace has to start at zero: the selection writes
  // every score, kept-list entry, bitmap word and counter before it is read,
  // so no clearing pass is needed between calls. Every launch stays on the
  // caller's stream: this entry point creates no streams or events either.
  return zha::decode_one_stream(cfg, cache, q, p, out, level_counts, ws, kStaticScratchBytes,
                                dev_status, stream);
}

}  // extern "C"
