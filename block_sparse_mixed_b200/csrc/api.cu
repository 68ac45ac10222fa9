// Host side of the C ABI declared in include/tria.h: argument checks, workspace
// layout, TMA descriptors and kernel launches. Nothing here allocates device
// memory; every buffer comes from the caller.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "load_plan.cuh"
#include "tria.h"

namespace tria {
namespace {

constexpr int kRowsPerTile = 128;   // query rows of a fused-prefill tile
constexpr int kCostLevels = 8192;   // levels of the decode's first-split cost estimate (in blocks)

// Whether the fused prefill may use the GQA-shared kernel (tria_prefill_gqa).
std::atomic<bool> g_prefill_gqa{true};

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// ---------------------------------------------------------------- device facts

struct DeviceInfo {
  bool ok = false;
  int sms = 0;
};

DeviceInfo device_info() {
  static std::mutex mu;
  static std::vector<DeviceInfo> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return {};
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  DeviceInfo& d = cache[dev];
  if (d.sms == 0) {
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    d.ok = (major == 10 && minor == 0);
    d.sms = sms > 0 ? sms : 1;
  }
  return d;
}

// ---------------------------------------------------------------- TMA descriptors

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

CUtensorMapSwizzle swizzle_for(int inner_bytes) {
  if (inner_bytes >= 128) return CU_TENSOR_MAP_SWIZZLE_128B;
  if (inner_bytes >= 64) return CU_TENSOR_MAP_SWIZZLE_64B;
  return CU_TENSOR_MAP_SWIZZLE_32B;
}

// 2-D map over a row-major [rows, inner] tensor; box = [box_inner, box_rows].
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
              uint64_t rows, uint32_t box_inner, uint32_t box_rows) {
  EncodeFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_for(static_cast<int>(box_inner) * elem_bytes), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- checks

bool shape_ok(int D, int T) { return (D == 64 || D == 128) && (T == 64 || T == 128); }

int check_cache(const tria_kv_cache* c) {
  if (c == nullptr) return TRIA_ERR_INVALID_ARG;
  if (c->B < 1 || c->Hkv < 1 || c->capacity < 1) return TRIA_ERR_INVALID_ARG;
  if (!shape_ok(c->D, c->T)) return TRIA_ERR_UNSUPPORTED;
  if (c->capacity % c->T != 0) return TRIA_ERR_INVALID_ARG;
  const void* ptrs[8] = {c->k8, c->k4, c->k8_scale, c->k4_scale, c->v8, c->v4, c->v8_scale, c->v4_scale};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return TRIA_ERR_INVALID_ARG;
  if (c->status == nullptr) return TRIA_ERR_INVALID_ARG;
  if (c->block_table != nullptr) {
    if (c->max_blocks < 1 || c->num_pages < 1 || c->capacity != c->max_blocks * c->T) return TRIA_ERR_INVALID_ARG;
    // TMA row coordinates and the page arithmetic are 32-bit
    if (static_cast<int64_t>(c->num_pages) * c->Hkv * c->T >= (int64_t(1) << 31)) return TRIA_ERR_UNSUPPORTED;
  } else if (static_cast<int64_t>(c->B) * c->Hkv * c->capacity >= (int64_t(1) << 31)) {
    return TRIA_ERR_UNSUPPORTED;
  }
  return TRIA_OK;
}

// Where the kernels find the cache's tokens.
CacheIndex cache_index(const tria_kv_cache& c) {
  CacheIndex ci{};
  ci.bt = c.block_table;
  ci.status = c.status;
  ci.cap = c.capacity;
  ci.Hkv = c.Hkv;
  ci.T = c.T;
  ci.max_blocks = c.max_blocks;
  ci.num_pages = c.num_pages;
  return ci;
}

int check_policy(const int32_t* hi, const int32_t* keep, int Hq) {
  if (hi == nullptr || keep == nullptr) return TRIA_ERR_INVALID_ARG;
  for (int h = 0; h < Hq; ++h)
    if (hi[h] < 0 || keep[h] < hi[h]) return TRIA_ERR_INVALID_ARG;
  return TRIA_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? TRIA_OK : TRIA_ERR_CUDA; }

// ---------------------------------------------------------------- workspace layouts

struct PrefillLayout {
  size_t ctrl, q8, q4, q8s, q4s, k4x, k8x, vt8, vt4, total;
};

PrefillLayout prefill_layout(const tria_dims& d) {
  PrefillLayout L{};
  const size_t qrows = static_cast<size_t>(d.B) * d.Hq * d.S;
  const size_t krows = static_cast<size_t>(d.B) * d.Hkv * d.S;
  size_t off = 0;
  L.ctrl = off; off += align_up(64);
  L.q8 = off; off += align_up(qrows * kQKRowBytes);
  L.q4 = off; off += align_up(qrows * kQKRowBytes);
  L.q8s = off; off += align_up(qrows * 4);
  L.q4s = off; off += align_up(qrows * 4);
  L.k4x = off; off += align_up(krows * kQKRowBytes);
  L.k8x = off; if (d.D < 128) off += align_up(krows * kQKRowBytes);
  L.vt8 = off; off += align_up(krows * d.D * 2);
  L.vt4 = off; off += align_up(krows * d.D * 2);
  L.total = off;
  return L;
}

int check_dims(const tria_dims* d) {
  if (d == nullptr) return TRIA_ERR_INVALID_ARG;
  if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->S < 1) return TRIA_ERR_INVALID_ARG;
  if (!shape_ok(d->D, d->T)) return TRIA_ERR_UNSUPPORTED;
  if (d->Hq % d->Hkv != 0) return TRIA_ERR_INVALID_ARG;
  if (d->Hq > kMaxHeads) return TRIA_ERR_UNSUPPORTED;
  if (d->S % d->T != 0) return TRIA_ERR_INVALID_ARG;
  // TMA coordinates are 32-bit
  if (static_cast<int64_t>(d->B) * d->Hq * d->S >= (int64_t(1) << 31)) return TRIA_ERR_UNSUPPORTED;
  return TRIA_OK;
}

struct DecodeLayout {
  size_t ctrl, part_o, part_ml, total;
  int max_items;
};

// Decode work items are bounded so that the partials fit a workspace sized from
// the shapes alone: at least two per group, at least 512 in all.
int decode_max_items(int groups) { return std::max(2 * groups, 512); }

DecodeLayout decode_layout(int B, int Hq, int Hkv, int D) {
  DecodeLayout L{};
  const size_t groups = static_cast<size_t>(B) * Hkv;
  const size_t G = static_cast<size_t>(Hq / Hkv);
  L.max_items = decode_max_items(static_cast<int>(groups));
  const size_t parts = static_cast<size_t>(L.max_items) * kDecodeSlices;
  size_t off = 0;
  L.ctrl = off; off += align_up(64);
  L.part_o = off; off += align_up(parts * G * D * 4);
  L.part_ml = off; off += align_up(parts * G * 2 * 4);
  L.total = off;
  return L;
}

// The decode's work plan (host side). nkept[g]: kept key blocks of group g = b * Hkv +
// kvh at its query position, the union over its G heads (block 0, then every block from
// the first one the widest band keeps to the diagonal). The split size bps asks for
// about six items per SM (at least 4 blocks), enlarged to the smallest size whose items
// fit max_items partial slots; split_start[g] is group g's first item and slot
// (ceil(nkept / bps) items each), and first_order lists the groups' first splits, the
// last phase of the launch, costliest first (a counting sort on the split's blocks plus,
// for a group of a single split, its widest 8-bit band once more). Returns the number
// of items.
int decode_plan(int B, int Hkv, int G, int T, const int32_t* kv_len, const int32_t* hi, const int32_t* keep, int sms,
                int max_items, int* bps_out, int* nkept, int* split_start, int16_t* first_order) {
  const int groups = B * Hkv;
  int64_t total = 0;
  for (int b = 0; b < B; ++b)
    for (int k = 0; k < Hkv; ++k) {
      const int ib = (kv_len[b] - 1) / T;
      int mk = 0;
      for (int h = 0; h < G; ++h) mk = std::max(mk, keep[k * G + h]);
      const int jb = first_band_block(ib, mk);
      nkept[b * Hkv + k] = ib == 0 ? 1 : 1 + (ib - jb + 1);
      total += nkept[b * Hkv + k];
    }
  const int64_t target_items = static_cast<int64_t>(sms) * 6;
  int bps = static_cast<int>(std::max<int64_t>(4, (total + target_items - 1) / target_items));
  auto count_items = [&](int b) {
    int64_t n = 0;
    for (int g = 0; g < groups; ++g) n += (nkept[g] + b - 1) / b;
    return n;
  };
  // the item count falls as the split size grows; at the largest group's size it is one
  // item per group, within the slots
  if (count_items(bps) > max_items) {
    int lo = bps, top = 1;
    for (int g = 0; g < groups; ++g) top = std::max(top, nkept[g]);
    while (lo < top) {
      const int mid = lo + (top - lo) / 2;
      if (count_items(mid) <= max_items) top = mid; else lo = mid + 1;
    }
    bps = lo;
  }
  int items = 0;
  for (int g = 0; g < groups; ++g) {
    split_start[g] = items;
    items += (nkept[g] + bps - 1) / bps;
  }
  split_start[groups] = items;
  std::vector<int> cost(groups), count(kCostLevels, 0);
  for (int g = 0; g < groups; ++g) {
    const int n = split_start[g + 1] - split_start[g];
    const int first = nkept[g] - (n - 1) * bps;
    int band = 0;
    if (n == 1)
      for (int h = 0; h < G; ++h) band = std::max(band, hi[(g % Hkv) * G + h]);
    cost[g] = static_cast<int>(std::min<int64_t>(static_cast<int64_t>(first) + band, kCostLevels - 1));
    ++count[cost[g]];
  }
  int at = 0;   // descending cost: start offsets from the top
  for (int c = kCostLevels - 1; c >= 0; --c) {
    const int n = count[c];
    count[c] = at;
    at += n;
  }
  for (int g = 0; g < groups; ++g) first_order[count[cost[g]]++] = static_cast<int16_t>(g);
  *bps_out = bps;
  return items;
}

}  // namespace
}  // namespace tria

using namespace tria;

extern "C" {

const char* tria_status_string(int status) {
  switch (status) {
    case TRIA_OK: return "ok";
    case TRIA_ERR_INVALID_ARG: return "invalid argument";
    case TRIA_ERR_UNSUPPORTED: return "unsupported shape or device";
    case TRIA_ERR_CUDA: return "CUDA error";
    case TRIA_ERR_TIMEOUT: return "device pipeline wait timed out";
    case TRIA_ERR_BOUNDS: return "device index check failed";
    case TRIA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

namespace {

// Planes of `rows` token rows after a 256-byte status block, in the order of the struct.
size_t planes_bytes(size_t rows, int D) {
  return align_up(64) + 2 * (align_up(rows * D) + align_up(rows * D / 2) + 2 * align_up(rows * 4));
}

void carve(tria_kv_cache* c, void* base, size_t rows, int D) {
  uint8_t* p = static_cast<uint8_t*>(base);
  c->status = reinterpret_cast<int*>(p); p += align_up(64);
  c->k8 = reinterpret_cast<int8_t*>(p); p += align_up(rows * D);
  c->k4 = p; p += align_up(rows * D / 2);
  c->k8_scale = reinterpret_cast<float*>(p); p += align_up(rows * 4);
  c->k4_scale = reinterpret_cast<float*>(p); p += align_up(rows * 4);
  c->v8 = reinterpret_cast<int8_t*>(p); p += align_up(rows * D);
  c->v4 = p; p += align_up(rows * D / 2);
  c->v8_scale = reinterpret_cast<float*>(p); p += align_up(rows * 4);
  c->v4_scale = reinterpret_cast<float*>(p);
}

}  // namespace

size_t tria_cache_bytes(int B, int Hkv, int D, int T, int capacity) {
  if (B < 1 || Hkv < 1 || !shape_ok(D, T) || capacity < 1 || capacity % T != 0) return 0;
  return planes_bytes(static_cast<size_t>(B) * Hkv * capacity, D);
}

int tria_cache_init(tria_kv_cache* c, void* base, size_t bytes, int B, int Hkv, int D, int T, int capacity) {
  if (c == nullptr || base == nullptr || !aligned256(base)) return TRIA_ERR_INVALID_ARG;
  const size_t need = tria_cache_bytes(B, Hkv, D, T, capacity);
  if (need == 0) return shape_ok(D, T) ? TRIA_ERR_INVALID_ARG : TRIA_ERR_UNSUPPORTED;
  if (bytes < need) return TRIA_ERR_INVALID_ARG;
  std::memset(c, 0, sizeof *c);
  carve(c, base, static_cast<size_t>(B) * Hkv * capacity, D);
  c->B = B; c->Hkv = Hkv; c->D = D; c->T = T; c->capacity = capacity;
  return TRIA_OK;
}

size_t tria_paged_cache_bytes(int num_pages, int Hkv, int D, int T) {
  if (num_pages < 1 || Hkv < 1 || !shape_ok(D, T)) return 0;
  return planes_bytes(static_cast<size_t>(num_pages) * Hkv * T, D);
}

int tria_paged_cache_init(tria_kv_cache* c, void* base, size_t bytes, int B, int Hkv, int D, int T, int num_pages,
                          const int32_t* block_table, int max_blocks) {
  if (c == nullptr || base == nullptr || !aligned256(base) || block_table == nullptr) return TRIA_ERR_INVALID_ARG;
  if (!shape_ok(D, T)) return TRIA_ERR_UNSUPPORTED;
  if (B < 1 || max_blocks < 1 || static_cast<int64_t>(max_blocks) * T >= (int64_t(1) << 31))
    return TRIA_ERR_INVALID_ARG;
  const size_t need = tria_paged_cache_bytes(num_pages, Hkv, D, T);
  if (need == 0 || bytes < need) return TRIA_ERR_INVALID_ARG;
  std::memset(c, 0, sizeof *c);
  carve(c, base, static_cast<size_t>(num_pages) * Hkv * T, D);
  c->B = B; c->Hkv = Hkv; c->D = D; c->T = T; c->capacity = max_blocks * T;
  c->block_table = block_table; c->max_blocks = max_blocks; c->num_pages = num_pages;
  return TRIA_OK;
}

int tria_cache_status(const tria_kv_cache* c, void* stream) {
  if (c == nullptr || c->status == nullptr) return TRIA_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return TRIA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, c->status, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) return TRIA_ERR_CUDA;
  if (cudaMemsetAsync(c->status, 0, sizeof word, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return TRIA_ERR_CUDA;
  return word;
}

int tria_quantize_rows(const void* X, int64_t rows, int D, int8_t* c8, float* s8, uint8_t* c4, float* s4,
                       void* stream) {
  if (D != 64 && D != 128) return TRIA_ERR_UNSUPPORTED;
  if (rows < 0 || X == nullptr || c8 == nullptr || s8 == nullptr) return TRIA_ERR_INVALID_ARG;
  if ((c4 == nullptr) != (s4 == nullptr)) return TRIA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(c8) || (c4 && !aligned16(c4)) || !aligned16(s8) || (s4 && !aligned16(s4)))
    return TRIA_ERR_INVALID_ARG;
  if (!device_info().ok) return TRIA_ERR_UNSUPPORTED;
  QuantArgs a{};
  a.X = static_cast<const __nv_bfloat16*>(X);
  a.rows = rows; a.cache = false;
  a.c8 = c8; a.ld8 = D; a.c4p = c4; a.c4u = nullptr; a.ld4u = 0; a.s8 = s8; a.s4 = s4;
  return cuda_status(launch_quant_rows(a, D, static_cast<cudaStream_t>(stream)));
}

int tria_quantize_kv(const void* K, const void* V, int S, int start, const tria_kv_cache* cache, void* stream) {
  const int cs = check_cache(cache);
  if (cs != TRIA_OK) return cs;
  if (K == nullptr || V == nullptr || !aligned16(K) || !aligned16(V)) return TRIA_ERR_INVALID_ARG;
  if (S < 1 || start < 0 || static_cast<int64_t>(start) + S > cache->capacity) return TRIA_ERR_INVALID_ARG;
  if (!device_info().ok) return TRIA_ERR_UNSUPPORTED;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // one launch for both tensors: K into the K planes, V (grid z = 1) into the V planes
  QuantArgs a{};
  a.X = static_cast<const __nv_bfloat16*>(K);
  a.rows = static_cast<int64_t>(cache->B) * cache->Hkv * S;
  a.cache = true;
  a.ci = cache_index(*cache);
  a.S = S;
  a.start = start;
  a.c8 = cache->k8;
  a.ld8 = cache->D;
  a.c4p = cache->k4;
  a.s8 = cache->k8_scale;
  a.s4 = cache->k4_scale;
  a.X2 = static_cast<const __nv_bfloat16*>(V);
  a.c8_2 = cache->v8;
  a.c4p_2 = cache->v4;
  a.s8_2 = cache->v8_scale;
  a.s4_2 = cache->v4_scale;
  return cuda_status(launch_quant_rows(a, cache->D, st));
}

int tria_count_tiles(int nb, int hi, int keep, int64_t* out) {
  if (out == nullptr || nb < 0 || hi < 0 || keep < hi) return TRIA_ERR_INVALID_ARG;
  out[0] = out[1] = out[2] = 0;
  for (int i = 0; i < nb; ++i)
    for (int j = 0; j <= i; ++j) {
      const int a = tile_action(i, j, hi, keep);
      if (a == ACT_INT8) ++out[0]; else if (a == ACT_INT4) ++out[1]; else if (a == ACT_SKIP) ++out[2];
    }
  return TRIA_OK;
}

int tria_decode_plan(int B, int Hq, int Hkv, int T, int capacity, const int32_t* kv_len, const int32_t* hi,
                     const int32_t* keep, int num_sms, int32_t* split_start, int32_t* first_order, int32_t* nkept,
                     int32_t* blocks_per_split, int32_t* n_items) {
  if (B < 1 || Hkv < 1 || Hq < 1 || Hq % Hkv != 0 || (T != 64 && T != 128) || capacity < 1 || capacity % T != 0 ||
      num_sms < 1 || kv_len == nullptr || split_start == nullptr || first_order == nullptr || nkept == nullptr ||
      blocks_per_split == nullptr || n_items == nullptr)
    return TRIA_ERR_INVALID_ARG;
  if (Hq > kMaxHeads || Hq / Hkv > 16 || B > kMaxBatch || static_cast<int64_t>(B) * Hkv > kMaxGroups)
    return TRIA_ERR_UNSUPPORTED;
  int s = check_policy(hi, keep, Hq);
  if (s != TRIA_OK) return s;
  for (int b = 0; b < B; ++b)
    if (kv_len[b] < 1 || kv_len[b] > capacity) return TRIA_ERR_INVALID_ARG;
  const int groups = B * Hkv;
  std::vector<int> nk(groups), ss(groups + 1);
  std::vector<int16_t> fo(groups);
  int bps = 0;
  const int items = decode_plan(B, Hkv, Hq / Hkv, T, kv_len, hi, keep, num_sms, decode_max_items(groups), &bps,
                                nk.data(), ss.data(), fo.data());
  for (int g = 0; g < groups; ++g) {
    nkept[g] = nk[g];
    split_start[g] = ss[g];
    first_order[g] = fo[g];
  }
  split_start[groups] = ss[groups];
  *blocks_per_split = bps;
  *n_items = items;
  return TRIA_OK;
}

int tria_prefill_load_plan(int nb, int T, int hi, int keep, int32_t* plan, int64_t capacity, int64_t* count) {
  if (count == nullptr || nb < 0 || (T != 64 && T != 128) || hi < 0 || keep < hi || capacity < 0)
    return TRIA_ERR_INVALID_ARG;
  const int nq = kRowsPerTile / T;
  int64_t n = 0;
  for (int i0 = 0; i0 < nb; i0 += nq) {
    const int q = std::min(nq, nb - i0);
    int j0, j1, plane;
    auto emit = [&]() {
      if (plan != nullptr && n < capacity) {
        int32_t* e = plan + 4 * n;
        e[0] = i0; e[1] = j0; e[2] = j1; e[3] = plane;
      }
      ++n;
    };
    const int64_t n0 = n;
    if (T == 128) {
      LoadPairs<1> lp;
      lp.init(i0, q, hi, keep);
      while (lp.next(j0, j1, plane)) emit();
      if (n - n0 != load_count<1>(i0, q, hi, keep)) return TRIA_ERR_BOUNDS;   // the kernel's count
    } else {
      LoadPairs<2> lp;
      lp.init(i0, q, hi, keep);
      while (lp.next(j0, j1, plane)) emit();
      if (n - n0 != load_count<2>(i0, q, hi, keep)) return TRIA_ERR_BOUNDS;
    }
  }
  *count = n;
  return TRIA_OK;
}

int tria_prefill_gqa(int enable) {
  const bool was = g_prefill_gqa.exchange(enable != 0);
  return was ? 1 : 0;
}

size_t tria_prefill_workspace_bytes(const tria_dims* dims) {
  if (check_dims(dims) != TRIA_OK) return 0;
  return prefill_layout(*dims).total;
}

namespace {

// Checks shared by the prefill calls; on success fills the layout and device facts.
int prefill_checks(const tria_kv_cache* cache, const tria_dims* dims, void* workspace, size_t workspace_bytes,
                   PrefillLayout* L, DeviceInfo* dev) {
  int s = check_dims(dims);
  if (s != TRIA_OK) return s;
  if ((s = check_cache(cache)) != TRIA_OK) return s;
  const tria_dims& d = *dims;
  if (cache->B != d.B || cache->Hkv != d.Hkv || cache->D != d.D || cache->T != d.T || cache->capacity < d.S)
    return TRIA_ERR_INVALID_ARG;
  *L = prefill_layout(d);
  if (workspace == nullptr || !aligned256(workspace) || workspace_bytes < L->total) return TRIA_ERR_WORKSPACE;
  *dev = device_info();
  if (!dev->ok) return TRIA_ERR_UNSUPPORTED;
  return TRIA_OK;
}

}  // namespace

int tria_prefill_prepare(const void* Q, const tria_kv_cache* cache, const tria_dims* dims, void* workspace,
                         size_t workspace_bytes, void* stream) {
  PrefillLayout L;
  DeviceInfo dev;
  int s = prefill_checks(cache, dims, workspace, workspace_bytes, &L, &dev);
  if (s != TRIA_OK) return s;
  if (Q == nullptr || !aligned16(Q)) return TRIA_ERR_INVALID_ARG;
  const tria_dims d = *dims;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int nb = d.S / d.T;
  const int64_t qrows = static_cast<int64_t>(d.B) * d.Hq * d.S;
  const int groups = d.B * d.Hkv;

  if (cudaMemsetAsync(ws + L.ctrl, 0, 64, st) != cudaSuccess) return TRIA_ERR_CUDA;

  // 1. Q codes, both planes, one int8 per value in 128-byte rows
  QuantArgs qa{};
  qa.X = static_cast<const __nv_bfloat16*>(Q);
  qa.rows = qrows; qa.cache = false;
  qa.c8 = reinterpret_cast<int8_t*>(ws + L.q8); qa.ld8 = kQKRowBytes;
  qa.c4p = nullptr; qa.c4u = reinterpret_cast<int8_t*>(ws + L.q4); qa.ld4u = kQKRowBytes;
  qa.s8 = reinterpret_cast<float*>(ws + L.q8s); qa.s4 = reinterpret_cast<float*>(ws + L.q4s);
  if (launch_quant_rows(qa, d.D, st) != cudaSuccess) return TRIA_ERR_CUDA;

  // 2. operand tiles from the cache: 4-bit K expanded, V dequantised and transposed per block
  PrepareArgs pa{};
  pa.k8 = cache->k8; pa.k4 = cache->k4; pa.v8 = cache->v8; pa.v4 = cache->v4;
  pa.v8s = cache->v8_scale; pa.v4s = cache->v4_scale;
  pa.k8x = d.D < 128 ? reinterpret_cast<int8_t*>(ws + L.k8x) : nullptr;
  pa.k4x = reinterpret_cast<int8_t*>(ws + L.k4x);
  pa.vt8 = reinterpret_cast<__nv_bfloat16*>(ws + L.vt8);
  pa.vt4 = reinterpret_cast<__nv_bfloat16*>(ws + L.vt4);
  pa.ci = cache_index(*cache); pa.S = d.S; pa.nb = nb; pa.groups = groups;
  if (launch_prepare(pa, d.D, d.T, st) != cudaSuccess) return TRIA_ERR_CUDA;
  return TRIA_OK;
}

int tria_prefill_attend(const tria_kv_cache* cache, const tria_dims* dims, const int32_t* hi, const int32_t* keep,
                        void* O, float* LSE, void* workspace, size_t workspace_bytes, void* stream) {
  PrefillLayout L;
  DeviceInfo dev;
  int s = prefill_checks(cache, dims, workspace, workspace_bytes, &L, &dev);
  if (s != TRIA_OK) return s;
  const tria_dims d = *dims;
  if ((s = check_policy(hi, keep, d.Hq)) != TRIA_OK) return s;
  if (O == nullptr || LSE == nullptr || !aligned16(O) || !aligned16(LSE)) return TRIA_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int nb = d.S / d.T;
  const int64_t qrows = static_cast<int64_t>(d.B) * d.Hq * d.S;
  const int groups = d.B * d.Hkv;
  // 3. the fused kernel
  PrefillMaps maps;
  const uint64_t krows = static_cast<uint64_t>(groups) * d.S;
  bool ok = make_map(&maps.q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.q8, kQKRowBytes, qrows, 128, 128) &&
            make_map(&maps.q4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.q4, kQKRowBytes, qrows, 128, 128) &&
            make_map(&maps.k4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.k4x, kQKRowBytes, krows, 128, d.T) &&
            make_map(&maps.v8, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + L.vt8, d.T,
                     static_cast<uint64_t>(groups) * nb * d.D, 64, d.D) &&
            make_map(&maps.v4, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ws + L.vt4, d.T,
                     static_cast<uint64_t>(groups) * nb * d.D, 64, d.D);
  const CacheIndex ci = cache_index(*cache);
  if (d.D == 128)
    ok = ok && make_map(&maps.k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cache->k8, 128,
                        static_cast<uint64_t>(ci.rows(cache->B)), 128, d.T);
  else
    ok = ok && make_map(&maps.k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.k8x, kQKRowBytes, krows, 128, d.T);
  if (!ok) return TRIA_ERR_CUDA;

  PrefillArgs a{};
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.S = d.S; a.G = d.Hq / d.Hkv; a.nb = nb;
  a.ci = ci; a.k8_in_cache = d.D == 128;
  a.cap = cache->capacity; a.cap8 = d.D == 128 ? cache->capacity : d.S;
  a.n_qtiles = (d.S + 127) / 128;
  a.n_units = d.B * d.Hq * a.n_qtiles;
  // Two query heads of a KV group share one CTA (and every K/V load) when their
  // boundaries coincide, for every such pair of the launch.
  bool gqa = g_prefill_gqa.load() && (a.G % 2 == 0);
  for (int h = 0; gqa && h < d.Hq; h += 2) gqa = hi[h] == hi[h + 1] && keep[h] == keep[h + 1];
  if (gqa) a.n_units = d.B * d.Hkv * (a.G / 2) * a.n_qtiles;
  a.qk_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d.D)));
  a.q8s = reinterpret_cast<const float*>(ws + L.q8s);
  a.q4s = reinterpret_cast<const float*>(ws + L.q4s);
  a.k8s = cache->k8_scale; a.k4s = cache->k4_scale;
  a.O = static_cast<__nv_bfloat16*>(O); a.LSE = LSE;
  a.err = reinterpret_cast<int*>(ws + L.ctrl);
  a.work = reinterpret_cast<int*>(ws + L.ctrl) + 4;
  for (int h = 0; h < d.Hq; ++h) { a.hi[h] = hi[h]; a.keep[h] = keep[h]; }
  if (cudaMemsetAsync(a.work, 0, sizeof(int), st) != cudaSuccess) return TRIA_ERR_CUDA;   // tile counter
  return cuda_status(gqa ? launch_prefill_gqa(a, maps, d.D, d.T, dev.sms, st)
                         : launch_prefill(a, maps, d.D, d.T, dev.sms, st));
}

int tria_prefill(const void* Q, const tria_kv_cache* cache, const tria_dims* dims, const int32_t* hi,
                 const int32_t* keep, void* O, float* LSE, void* workspace, size_t workspace_bytes, void* stream) {
  // arguments of the second call are checked before the first one runs
  int s = check_policy(hi, keep, dims != nullptr ? dims->Hq : 0);
  if (dims == nullptr || s != TRIA_OK) return dims == nullptr ? TRIA_ERR_INVALID_ARG : s;
  if (O == nullptr || LSE == nullptr || !aligned16(O) || !aligned16(LSE)) return TRIA_ERR_INVALID_ARG;
  if ((s = tria_prefill_prepare(Q, cache, dims, workspace, workspace_bytes, stream)) != TRIA_OK) return s;
  return tria_prefill_attend(cache, dims, hi, keep, O, LSE, workspace, workspace_bytes, stream);
}

size_t tria_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int T, int capacity) {
  if (B < 1 || B > kMaxBatch || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq > kMaxHeads) return 0;
  if (Hq / Hkv > 16 || static_cast<int64_t>(B) * Hkv > kMaxGroups || !shape_ok(D, T) || capacity < 1) return 0;
  return decode_layout(B, Hq, Hkv, D).total;
}

int tria_decode(const void* q, const tria_kv_cache* cache, const int32_t* kv_len, int Hq, const int32_t* hi,
                const int32_t* keep, void* O, float* LSE, void* workspace, size_t workspace_bytes, void* stream) {
  int s = check_cache(cache);
  if (s != TRIA_OK) return s;
  const int B = cache->B, Hkv = cache->Hkv, D = cache->D, T = cache->T;
  if (Hq < 1 || Hq % Hkv != 0) return TRIA_ERR_INVALID_ARG;
  if (Hq > kMaxHeads || Hq / Hkv > 16 || B > kMaxBatch || static_cast<int64_t>(B) * Hkv > kMaxGroups)
    return TRIA_ERR_UNSUPPORTED;
  if ((s = check_policy(hi, keep, Hq)) != TRIA_OK) return s;
  if (kv_len == nullptr) return TRIA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (kv_len[b] < 1 || kv_len[b] > cache->capacity) return TRIA_ERR_INVALID_ARG;
  if (q == nullptr || O == nullptr || LSE == nullptr || !aligned16(q) || !aligned16(O) || !aligned16(LSE))
    return TRIA_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(B, Hq, Hkv, D);
  if (workspace == nullptr || !aligned256(workspace) || workspace_bytes < L.total) return TRIA_ERR_WORKSPACE;
  const DeviceInfo dev = device_info();
  if (!dev.ok) return TRIA_ERR_UNSUPPORTED;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int G = Hq / Hkv;
  const int groups = B * Hkv;

  // the work plan: kept blocks per group, split size, each group's first item, the
  // order of the groups' first splits
  std::vector<int> nkept(groups);
  int bps = 0;
  DecodeArgs a{};
  const int items = decode_plan(B, Hkv, G, T, kv_len, hi, keep, dev.sms, L.max_items, &bps, nkept.data(),
                                a.split_start, a.first_order);
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.G = G; a.D = D; a.T = T;
  a.ci = cache_index(*cache);
  a.blocks_per_split = bps;
  a.qk_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k8 = cache->k8; a.k4 = cache->k4; a.k8s = cache->k8_scale; a.k4s = cache->k4_scale;
  a.v8 = cache->v8; a.v4 = cache->v4; a.v8s = cache->v8_scale; a.v4s = cache->v4_scale;
  a.part_o = reinterpret_cast<float*>(ws + L.part_o);
  a.part_ml = reinterpret_cast<float*>(ws + L.part_ml);
  a.work = reinterpret_cast<int*>(ws + L.ctrl) + 4;
  a.O = static_cast<__nv_bfloat16*>(O); a.LSE = LSE;
  a.err = reinterpret_cast<int*>(ws + L.ctrl);
  a.n_groups = groups;
  for (int h = 0; h < Hq; ++h) { a.hi[h] = hi[h]; a.keep[h] = keep[h]; }
  for (int b = 0; b < B; ++b) a.kv_len[b] = kv_len[b];
  a.n_items = items;

  DecodeMaps maps;
  const uint64_t rows = static_cast<uint64_t>(a.ci.rows(B));   // below 2^31 (check_cache)
  const bool ok = make_map(&maps.k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cache->k8, D, rows, D, T) &&
                  make_map(&maps.k4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cache->k4, D / 2, rows, D / 2, T) &&
                  make_map(&maps.v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cache->v8, D, rows, D, T) &&
                  make_map(&maps.v4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, cache->v4, D / 2, rows, D / 2, T);
  if (!ok) return TRIA_ERR_CUDA;
  if (cudaMemsetAsync(ws + L.ctrl, 0, 64, st) != cudaSuccess) return TRIA_ERR_CUDA;   // error word, work counter
  return cuda_status(launch_decode(a, maps, dev.sms, st));
}

int tria_workspace_status(const void* workspace, void* stream) {
  if (workspace == nullptr) return TRIA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TRIA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) return TRIA_ERR_CUDA;
  return word;
}

}  // extern "C"
