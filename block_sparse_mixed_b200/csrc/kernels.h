// Internal launch interface between the host API (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tria.h"

namespace tria {

constexpr int kMaxHeads = 256;     // Hq limit (policy arrays travel in kernel parameters)
constexpr int kMaxBatch = 1024;    // decode: kv_len travels in kernel parameters
constexpr int kMaxGroups = 2048;   // decode: B * Hkv
constexpr int kQKRowBytes = 128;   // Q/K code rows as the tensor cores read them (D padded to 128)
constexpr int kDecodeSlices = 8;   // decode: most compute warps per CTA (each writes its own partial)

// Where the cache keeps the tokens of one (sequence b, KV head): the contiguous
// layout [B, Hkv, cap] rows, or pages of T tokens x Hkv heads named by a block
// table. A page id outside [0, num_pages) sets TRIA_ERR_BOUNDS in the cache's
// status word and gives -1; callers then skip or redirect the access.
struct CacheIndex {
  const int32_t* bt;      // device [B, max_blocks] page of each logical block, or null (contiguous)
  int* status;            // the cache's device error word
  int64_t cap;            // contiguous: tokens per (b, kv head)
  int Hkv, T, max_blocks, num_pages;

  // Cache row of the first token of logical block j of (b, kvh).
  __device__ __forceinline__ int64_t block_row(int b, int kvh, int j) const {
    if (bt == nullptr) return (static_cast<int64_t>(b) * Hkv + kvh) * cap + static_cast<int64_t>(j) * T;
    const int p = (j >= 0 && j < max_blocks) ? bt[static_cast<int64_t>(b) * max_blocks + j] : -1;
    if (p < 0 || p >= num_pages) {
      atomicExch(status, TRIA_ERR_BOUNDS);
      return -1;
    }
    return (static_cast<int64_t>(p) * Hkv + kvh) * T;
  }
  // Rows of one plane of the cache.
  __host__ __device__ int64_t rows(int B) const {
    return bt == nullptr ? static_cast<int64_t>(B) * Hkv * cap : static_cast<int64_t>(num_pages) * Hkv * T;
  }
};

// Codec over rows. Output row of input row r: r itself (tokens of Q, or any rows),
// or, when `cache` is set, the cache row of token start + r % S of (b, kvh) =
// (r / S) / Hkv, (r / S) % Hkv.
struct QuantArgs {
  const __nv_bfloat16* X;
  int64_t rows;
  bool cache;         // rows of B * Hkv groups of S new tokens: grid (token blocks, groups, 1 or 2)
  CacheIndex ci;
  int64_t S;
  int64_t start;
  int8_t* c8;
  int ld8;            // bytes per c8 row (D or 128; bytes past D are zeroed)
  uint8_t* c4p;       // packed 4-bit codes, D/2 bytes per row (optional)
  int8_t* c4u;        // 4-bit codes one fp8 e4m3 byte each (optional; the prefill QK operand)
  int ld4u;
  float* s8;
  float* s4;          // null: skip the 4-bit plane
  int group0;         // cache path: group of grid row y = 0 (launches of at most 65,535 groups)
  // cache path, grid z = 1: a second tensor (V) into its own planes, same layout
  const __nv_bfloat16* X2;
  int8_t* c8_2;
  uint8_t* c4p_2;
  float* s8_2;
  float* s4_2;
};

struct PrepareArgs {
  const int8_t* k8;
  const uint8_t* k4;
  const int8_t* v8;
  const uint8_t* v4;
  const float* v8s;
  const float* v4s;
  int8_t* k8x;        // null when D == 128 (the cache plane is read directly)
  int8_t* k4x;        // [groups * S, 128]
  __nv_bfloat16* vt8; // [groups * nb, D, T] V of the 8-bit plane, dequantised, transposed per block
  __nv_bfloat16* vt4; // [groups * nb, D, T] the same for the 4-bit plane
  CacheIndex ci;
  int64_t S;          // prefill tokens per (b, kv head) (= nb * T)
  int64_t nb;
  int64_t groups;     // B * Hkv
};

struct PrefillArgs {
  int B, Hq, Hkv, S, G, nb;
  int64_t cap;            // contiguous cache: rows per (b, kv head), scale arrays
  int64_t cap8;           // rows per (b, kv head) behind the 8-bit K map (cap, or S when padded)
  int n_qtiles, n_units;
  float qk_log2;          // log2(e) / sqrt(D)
  const float* q8s;       // [B*Hq*S]
  const float* q4s;
  const float* k8s;       // cache scales [B*Hkv*cap]
  const float* k4s;
  __nv_bfloat16* O;
  float* LSE;
  int* err;
  int* work;              // next query tile (dynamic scheduling); zero before the launch
  int hi[kMaxHeads];
  int keep[kMaxHeads];
  CacheIndex ci;          // cache rows of the 8-bit K plane (D = 128) and of the K scales
  bool k8_in_cache;       // the 8-bit K map covers the cache plane (D = 128) or the padded copy (D = 64)
};

struct PrefillMaps {
  CUtensorMap q8, q4, k8, k4, v8, v4;
};

struct DecodeMaps {
  CUtensorMap k8, k4, v8, v4;
};

struct DecodeArgs {
  int B, Hq, Hkv, G, D, T;
  CacheIndex ci;
  int n_items;            // (group, split) work items
  int blocks_per_split;
  float qk_log2;
  const __nv_bfloat16* q; // [B, Hq, D]
  const int8_t* k8; const uint8_t* k4; const float* k8s; const float* k4s;
  const int8_t* v8; const uint8_t* v4; const float* v8s; const float* v4s;
  uint32_t magic[8];      // bit masks and biases of the code conversions, filled by the launcher
                          // (as kernel parameters they stay register operands of one lop3 each)
  int slices;             // compute warps per CTA: partials per item
  int stages;             // ring stages (from the shared memory available)
  float* part_o;          // [items, slices, G, D] unnormalised partial outputs (x 64)
  float* part_ml;         // [items, slices, G, 2] partial (max in log2 units, sum)
  int* work;              // next work item (dynamic scheduling); zero before the launch
  __nv_bfloat16* O;
  float* LSE;
  int* err;
  int n_groups;
  int hi[kMaxHeads];
  int keep[kMaxHeads];
  int kv_len[kMaxBatch];
  int split_start[kMaxGroups + 1];     // first work item of each group (groups = B*Hkv)
  int16_t first_order[kMaxGroups];     // the group of each item of the last phase (see item_range)
};

cudaError_t launch_quant_rows(const QuantArgs& a, int D, cudaStream_t stream);
cudaError_t launch_prepare(const PrepareArgs& a, int D, int T, cudaStream_t stream);
cudaError_t launch_prefill(const PrefillArgs& a, const PrefillMaps& maps, int D, int T, int num_sms,
                           cudaStream_t stream);
cudaError_t launch_prefill_gqa(const PrefillArgs& a, const PrefillMaps& maps, int D, int T, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& maps, int num_sms, cudaStream_t stream);

}  // namespace tria
