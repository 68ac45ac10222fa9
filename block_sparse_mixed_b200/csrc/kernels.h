// Internal launch interface between the host API (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tria {

constexpr int kMaxHeads = 256;     // Hq limit (policy arrays travel in kernel parameters)
constexpr int kMaxBatch = 1024;    // decode: kv_len travels in kernel parameters
constexpr int kMaxGroups = 2048;   // decode: B * Hkv
constexpr int kQKRowBytes = 128;   // Q/K code rows as the tensor cores read them (D padded to 128)
constexpr int kDecodeSlices = 8;   // decode: most compute warps per CTA (each writes its own partial)

// Codec over rows. Output row of input row r:
//   (r / rows_per_group) * group_stride + start + r % rows_per_group.
struct QuantArgs {
  const __nv_bfloat16* X;
  int64_t rows;
  int64_t rows_per_group;
  int64_t group_stride;
  int64_t start;
  int8_t* c8;
  int ld8;            // bytes per c8 row (D or 128; bytes past D are zeroed)
  uint8_t* c4p;       // packed 4-bit codes, D/2 bytes per row (optional)
  int8_t* c4u;        // 4-bit codes one fp8 e4m3 byte each (optional; the prefill QK operand)
  int ld4u;
  float* s8;
  float* s4;          // null: skip the 4-bit plane
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
  __nv_bfloat16* vt8; // [groups * nb, D, T]
  __nv_bfloat16* vt4;
  int64_t cap;        // cache tokens per (b, kv head)
  int64_t S;          // prefill tokens per (b, kv head) (= nb * T)
  int64_t nb;
};

struct PrefillArgs {
  int B, Hq, Hkv, S, G, nb;
  int64_t cap;            // cache rows per (b, kv head): scale arrays
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
};

struct PrefillMaps {
  CUtensorMap q8, q4, k8, k4, v8, v4;
};

struct DecodeMaps {
  CUtensorMap k8, k4, v8, v4;
};

struct DecodeArgs {
  int B, Hq, Hkv, G, D, T;
  int64_t cap;
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
};

cudaError_t launch_quant_rows(const QuantArgs& a, int D, cudaStream_t stream);
cudaError_t launch_prepare(const PrepareArgs& a, int D, int T, int groups, int nblocks, cudaStream_t stream);
cudaError_t launch_prefill(const PrefillArgs& a, const PrefillMaps& maps, int D, int T, int num_sms,
                           cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, const DecodeMaps& maps, int num_sms, cudaStream_t stream);

}  // namespace tria
