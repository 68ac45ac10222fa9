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
// address, so the device address is fetched with cudaGetSymbolAddress on the
// first call made in each CUDA context (a device's primary context, or a
// context the caller created and made current), and that address is what the
// kernels receive. Nothing here calls cudaMalloc, cudaFree or any allocating
// routine.
//
// Sharing: all calls in a context use the same array and it keeps whatever the
// last call left in it. The decode call clears the parts that must start at
// zero (error word and work counter) at the start of every call; the rest is
// fully rewritten before it is read. Two calls whose work overlaps on the GPU
// (different streams without ordering between them) race on the array.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>
#include <vector>

#include "tria.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[TRIA_DECODE_STATIC_SCRATCH_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

std::mutex g_scratch_mu;
// (context, device address of g_decode_scratch in that context)
std::vector<std::pair<CUcontext, void*>> g_scratch_addr;

// Device address of g_decode_scratch in the current context (looked up once per
// context; the lookup also brings up the device's primary context when no context
// is current yet).
int scratch_address(void** out) {
  CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr) return TRIA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return TRIA_ERR_CUDA;
  if (ctx != nullptr)
    for (const auto& e : g_scratch_addr)
      if (e.first == ctx) {
        *out = e.second;
        return TRIA_OK;
      }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return TRIA_ERR_CUDA;
  if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return TRIA_ERR_CUDA;
  g_scratch_addr.emplace_back(ctx, p);
  *out = p;
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

extern "C" int tria_decode_static_status(void* stream) {
  void* scratch = nullptr;
  const int s = scratch_address(&scratch);
  if (s != TRIA_OK) return s;
  return tria_workspace_status(scratch, stream);
}
