// Prefill from host buffers (tria_prefill_host): the runtime layer that overlaps the
// host<->device copies of a prompt with its kernels. It is built only on the C ABI of
// tria.h (tria_quantize_kv, tria_prefill_prepare, tria_prefill_attend) and the CUDA
// runtime's asynchronous copies and events.
//
// The unit of the pipeline is one (batch, KV head) group: its K and V rows, its G
// query heads' Q rows in, their O and LSE rows out. Every group is independent (its
// cache rows, its query heads and its outputs are its own), so group g's kernels run
// while group g + 1's inputs are copied in and group g - 1's outputs are copied out,
// through two to four staging slots in device memory (as many as the caller's
// staging buffer holds). The copies in set the pace; what runs after the last of them
// (the last unit's kernels and its copy out) is the pipeline's tail, so the last group
// is taken as two units of G / 2 query heads when G is a multiple of 4 (head pairs
// with the same boundaries stay together, so every head is computed by the same
// kernel as in a whole-group unit): the first writes the group's cache rows, the
// second only copies its queries in.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "tria.h"

namespace {

constexpr int kMinSlots = 2, kMaxSlots = 4;

struct Slots {
  size_t q, kv, o, lse, slot;   // bytes of each buffer of one slot, and of one whole slot
};

Slots slot_sizes(const tria_dims& d) {
  const int G = d.Hq / d.Hkv;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  Slots s;
  s.q = up(static_cast<size_t>(G) * d.S * d.D * 2);
  s.kv = up(static_cast<size_t>(d.S) * d.D * 2);
  s.o = s.q;
  s.lse = up(static_cast<size_t>(G) * d.S * 4);
  s.slot = s.q + 2 * s.kv + s.o + s.lse;
  return s;
}

bool dims_ok(const tria_dims* d) {
  return d != nullptr && d->B >= 1 && d->Hkv >= 1 && d->Hq >= d->Hkv && d->Hq % d->Hkv == 0 && d->S >= 1;
}

tria_dims group_dims(const tria_dims& d) {
  tria_dims g = d;
  g.B = 1;
  g.Hkv = 1;
  g.Hq = d.Hq / d.Hkv;
  return g;
}

// The cache rows of group (b, kvh) as a cache of one sequence and one KV head.
tria_kv_cache group_cache(const tria_kv_cache& c, int gi) {
  tria_kv_cache g = c;
  const size_t rows = static_cast<size_t>(gi) * c.capacity;
  g.k8 = c.k8 + rows * c.D;
  g.v8 = c.v8 + rows * c.D;
  g.k4 = c.k4 + rows * (c.D / 2);
  g.v4 = c.v4 + rows * (c.D / 2);
  g.k8_scale = c.k8_scale + rows;
  g.k4_scale = c.k4_scale + rows;
  g.v8_scale = c.v8_scale + rows;
  g.v4_scale = c.v4_scale + rows;
  g.B = 1;
  g.Hkv = 1;
  return g;
}

}  // namespace

extern "C" {

size_t tria_prefill_host_staging_bytes(const tria_dims* dims) {
  if (!dims_ok(dims)) return 0;
  return kMinSlots * slot_sizes(*dims).slot;
}

size_t tria_prefill_host_workspace_bytes(const tria_dims* dims) {
  if (!dims_ok(dims)) return 0;
  const tria_dims g = group_dims(*dims);
  return tria_prefill_workspace_bytes(&g);
}

int tria_prefill_host(const void* hQ, const void* hK, const void* hV, const tria_kv_cache* cache,
                      const tria_dims* dims, const int32_t* hi, const int32_t* keep, void* hO, float* hLSE,
                      void* staging, size_t staging_bytes, void* workspace, size_t workspace_bytes, void* stream,
                      void* copy_in_stream, void* copy_out_stream) {
  if (!dims_ok(dims) || cache == nullptr || hi == nullptr || keep == nullptr) return TRIA_ERR_INVALID_ARG;
  if (hQ == nullptr || hK == nullptr || hV == nullptr || hO == nullptr || hLSE == nullptr) return TRIA_ERR_INVALID_ARG;
  if (staging == nullptr || (reinterpret_cast<uintptr_t>(staging) & 255u) != 0) return TRIA_ERR_INVALID_ARG;
  if (copy_in_stream == nullptr || copy_out_stream == nullptr || copy_in_stream == stream ||
      copy_out_stream == stream || copy_in_stream == copy_out_stream)
    return TRIA_ERR_INVALID_ARG;
  const tria_dims& d = *dims;
  if (cache->block_table != nullptr) return TRIA_ERR_UNSUPPORTED;   // contiguous caches only
  if (cache->B != d.B || cache->Hkv != d.Hkv || cache->D != d.D || cache->T != d.T || cache->capacity < d.S)
    return TRIA_ERR_INVALID_ARG;
  const Slots sz = slot_sizes(d);
  if (staging_bytes < kMinSlots * sz.slot) return TRIA_ERR_INVALID_ARG;
  // a larger staging buffer buys more slots: the copies in run further ahead
  const int slots = static_cast<int>(std::min<size_t>(kMaxSlots, staging_bytes / sz.slot));
  const tria_dims gd = group_dims(d);
  const size_t ws_need = tria_prefill_workspace_bytes(&gd);
  if (ws_need == 0) return TRIA_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_need) return TRIA_ERR_INVALID_ARG;

  const cudaStream_t sc = static_cast<cudaStream_t>(stream);
  const cudaStream_t si = static_cast<cudaStream_t>(copy_in_stream);
  const cudaStream_t so = static_cast<cudaStream_t>(copy_out_stream);
  const int G = d.Hq / d.Hkv;
  const int groups = d.B * d.Hkv;
  const bool split_last = G % 4 == 0;
  const int units = groups + (split_last ? 1 : 0);
  const size_t kvbytes = static_cast<size_t>(d.S) * d.D * 2;
  const size_t head_q = static_cast<size_t>(d.S) * d.D * 2, head_l = static_cast<size_t>(d.S) * 4;   // per query head
  uint8_t* st = static_cast<uint8_t*>(staging);
  auto q_of = [&](int s) { return st + s * sz.slot; };
  auto k_of = [&](int s) { return q_of(s) + sz.q; };
  auto v_of = [&](int s) { return k_of(s) + sz.kv; };
  auto o_of = [&](int s) { return v_of(s) + sz.kv; };
  auto l_of = [&](int s) { return reinterpret_cast<float*>(o_of(s) + sz.o); };

  // Events: the start of the call on `stream`; per slot, inputs copied in, inputs
  // consumed (after the preparation), outputs written, outputs copied out.
  cudaEvent_t ev[1 + 4 * kMaxSlots] = {};
  int status = TRIA_OK;
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) status = TRIA_ERR_CUDA;
  cudaEvent_t start = ev[0];
  auto in_ready = [&](int s) { return ev[1 + 4 * s]; };
  auto in_free = [&](int s) { return ev[2 + 4 * s]; };
  auto out_ready = [&](int s) { return ev[3 + 4 * s]; };
  auto out_free = [&](int s) { return ev[4 + 4 * s]; };
  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess && status == TRIA_OK) status = TRIA_ERR_CUDA;
    return status == TRIA_OK;
  };
  auto ok_t = [&](int s) {
    if (s != TRIA_OK && status == TRIA_OK) status = s;
    return status == TRIA_OK;
  };

  // the copy streams start after the work already queued on `stream` (which may still
  // use the staging buffers of an earlier call)
  if (status == TRIA_OK && ok(cudaEventRecord(start, sc)) && ok(cudaStreamWaitEvent(si, start, 0)))
    ok(cudaStreamWaitEvent(so, start, 0));

  for (int ui = 0; ui < units && status == TRIA_OK; ++ui) {
    const int s = ui % slots;
    // unit ui: group gi, query heads [h0, h0 + nh) of it; the group's first unit writes its cache rows
    const bool second_half = split_last && ui == units - 1;
    const int gi = second_half ? groups - 1 : ui;
    const int nh = split_last && gi == groups - 1 ? G / 2 : G;
    const int h0 = second_half ? G / 2 : 0;
    const bool write_cache = h0 == 0;
    const int b = gi / d.Hkv, kvh = gi % d.Hkv;
    const size_t qrow0 = static_cast<size_t>(b) * d.Hq + static_cast<size_t>(kvh) * G + h0;   // first query head row
    tria_dims ud = gd;
    ud.Hq = nh;
    // inputs of unit ui into slot s, once unit ui - slots has consumed it
    if (ui >= slots && !ok(cudaStreamWaitEvent(si, in_free(s), 0))) break;
    if (write_cache) {
      if (!ok(cudaMemcpyAsync(k_of(s), static_cast<const uint8_t*>(hK) + gi * kvbytes, kvbytes, cudaMemcpyHostToDevice,
                              si)))
        break;
      if (!ok(cudaMemcpyAsync(v_of(s), static_cast<const uint8_t*>(hV) + gi * kvbytes, kvbytes, cudaMemcpyHostToDevice,
                              si)))
        break;
    }
    if (!ok(cudaMemcpyAsync(q_of(s), static_cast<const uint8_t*>(hQ) + qrow0 * head_q, nh * head_q,
                            cudaMemcpyHostToDevice, si)))
      break;
    if (!ok(cudaEventRecord(in_ready(s), si))) break;
    // kernels of unit ui: cache write (the group's first unit), preparation, fused
    // prefill into slot s's outputs (once unit ui - slots' outputs have been copied out of it)
    if (!ok(cudaStreamWaitEvent(sc, in_ready(s), 0))) break;
    if (ui >= slots && !ok(cudaStreamWaitEvent(sc, out_free(s), 0))) break;
    const tria_kv_cache gc = group_cache(*cache, gi);
    if (write_cache && !ok_t(tria_quantize_kv(k_of(s), v_of(s), d.S, 0, &gc, sc))) break;
    if (!ok_t(tria_prefill_prepare(q_of(s), &gc, &ud, workspace, workspace_bytes, sc))) break;
    if (!ok(cudaEventRecord(in_free(s), sc))) break;
    if (!ok_t(tria_prefill_attend(&gc, &ud, hi + kvh * G + h0, keep + kvh * G + h0, o_of(s), l_of(s), workspace,
                                  workspace_bytes, sc)))
      break;
    if (!ok(cudaEventRecord(out_ready(s), sc))) break;
    // outputs of unit ui to the host
    if (!ok(cudaStreamWaitEvent(so, out_ready(s), 0))) break;
    if (!ok(cudaMemcpyAsync(static_cast<uint8_t*>(hO) + qrow0 * head_q, o_of(s), nh * head_q, cudaMemcpyDeviceToHost,
                            so)))
      break;
    if (!ok(cudaMemcpyAsync(hLSE + qrow0 * d.S, l_of(s), nh * head_l, cudaMemcpyDeviceToHost, so))) break;
    if (!ok(cudaEventRecord(out_free(s), so))) break;
  }
  // `stream` completes after the last copy out (and after any copy in, on an early stop)
  cudaEvent_t tail_in = nullptr, tail_out = nullptr;
  if (cudaEventCreateWithFlags(&tail_in, cudaEventDisableTiming) == cudaSuccess) {
    if (cudaEventRecord(tail_in, si) == cudaSuccess) cudaStreamWaitEvent(sc, tail_in, 0);
    cudaEventDestroy(tail_in);
  }
  if (cudaEventCreateWithFlags(&tail_out, cudaEventDisableTiming) == cudaSuccess) {
    if (cudaEventRecord(tail_out, so) == cudaSuccess) cudaStreamWaitEvent(sc, tail_out, 0);
    cudaEventDestroy(tail_out);
  }
  for (auto& e : ev)
    if (e != nullptr) cudaEventDestroy(e);   // released once the work that records it completes
  return status;
}

}  // extern "C"
