// tria_decode_static: split-KV decode whose scratch is a fixed device array
// compiled into this library, for callers that cannot allocate device memory.
//
// Who needs it: code that owns no device allocator -- for example a plugin
// loaded into a host application that has already budgeted every byte of
// device memory, or a latency-critical loop that must not call cudaMalloc
// (which can synchronise the device). Such a caller still passes its inputs
// and outputs, but cannot hand tria_decode a workspace.
//
// How: the scratch that tria_decode takes from its caller lives here instead,
// in one file-scope __device__ array of TRIA_DECODE_STATIC_SCRATCH_BYTES. Every
// GPU that loads this library holds the array until the process exits. In
// host code the array's name is only a host-side stand-in, never a device
// address, so the device address is fetched once per device with
// cudaGetSymbolAddress (on the first call made while that device is current)
// and that address is what the kernels receive. Nothing here calls cudaMalloc,
// cudaFree or any allocating routine.
//
// Sharing: all calls on a device use the same array and it keeps whatever the
// last call left in it. The decode call clears the parts that must start at
// zero (error word and per-group counters) at the start of every call; the
// rest is fully rewritten before it is read. Two calls whose work overlaps on
// the GPU (different streams without ordering between them) race on the array.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "tria.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[TRIA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TRIA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TRIA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return TRIA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TRIA_OK;
}

}  // namespace

extern "C" int tria_decode_static(const void* q, const tria_kv_cache* cache, const int32_t* kv_len, int Hq,
                                  const int32_t* hi, const int32_t* keep, void* O, float* LSE, void* stream) {
  if (cache == nullptr) return TRIA_ERR_INVALID_ARG;
  const size_t need = tria_decode_workspace_bytes(cache->B, Hq, cache->Hkv, cache->D, cache->T, cache->capacity);
  if (need > TRIA_DECODE_STATIC_SCRATCH_BYTES) return TRIA_ERR_WORKSPACE;  // beyond the fixed maximum
  void* scratch = nullptr;
  const int s = scratch_address(&scratch);
  if (s != TRIA_OK) return s;
  return tria_decode(q, cache, kv_len, Hq, hi, keep, O, LSE, scratch, TRIA_DECODE_STATIC_SCRATCH_BYTES, stream);
}
