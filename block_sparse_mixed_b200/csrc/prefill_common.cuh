// Device helpers of the fused prefill kernels (per-head and GQA-shared): bounded
// drain waits, packed fp32x2 arithmetic and the two softmax passes over one
// thread's keys of a 128-key load.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace tria {
namespace pf {

// Bounded wait that ignores the abort flag: used on the way out to let copies and
// tensor-core ops already in flight land before the CTA releases its memory.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_timer();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer() - t0 > kWaitLimitNs) return;
  }
}

// ---- packed fp32x2 arithmetic (two scores per instruction) ----
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Softmax pass 1 over N keys of a row: y = float(acc) * s_k as packed pairs, and
// the maximum over the visible keys (n <= kmax when MASK).
// FP: S holds fp32 (the 4-bit plane's e4m3 product, an exact integer) instead of int32.
// (Converting the int32 sums through the bits of 1.5 * 2^23 and a packed subtraction,
// instead of the int-to-float conversion, measured slower at T = 128.)
template <int N, bool MASK, bool FP>
__device__ __forceinline__ float scores_and_max(const uint32_t (&r)[N], uint64_t (&y)[N / 2], const float* sk,
                                                int kmax) {
  auto cv = [](uint32_t v) { return FP ? __uint_as_float(v) : __int2float_rn(static_cast<int>(v)); };
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    const float4 s4 = *reinterpret_cast<const float4*>(sk + 4 * q);
    const uint64_t u01 = pk2(cv(r[4 * q]), cv(r[4 * q + 1]));
    const uint64_t u23 = pk2(cv(r[4 * q + 2]), cv(r[4 * q + 3]));
    y[2 * q] = mul2(u01, pk2(s4.x, s4.y));
    y[2 * q + 1] = mul2(u23, pk2(s4.z, s4.w));
    float v0, v1, v2, v3;
    up2(y[2 * q], v0, v1);
    up2(y[2 * q + 1], v2, v3);
    if (MASK) {
      const int n = 4 * q;
      v0 = n <= kmax ? v0 : -INFINITY;
      v1 = n + 1 <= kmax ? v1 : -INFINITY;
      v2 = n + 2 <= kmax ? v2 : -INFINITY;
      v3 = n + 3 <= kmax ? v3 : -INFINITY;
    }
    mx[(q % 2) * 2] = max3(mx[(q % 2) * 2], v0, v1);
    mx[(q % 2) * 2 + 1] = max3(mx[(q % 2) * 2 + 1], v2, v3);
  }
  return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// Softmax pass 2 over N keys: p = 2^(y * alpha - m) as bf16 pairs, stored as they
// are made into the thread's 128-byte P row (16-byte chunk c at c ^ swz), their
// fp32 sum accumulated in `acc`; masked keys (n > kmax when MASK) give 0.
template <int N, bool MASK>
__device__ __forceinline__ void probs(const uint64_t (&y)[N / 2], uint64_t al2, uint64_t nm2, int kmax,
                                      uint8_t* prow, int swz, uint64_t (&acc)[4]) {
#pragma unroll
  for (int c = 0; c < N / 8; ++c) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = 4 * c + e;
      float t0, t1;
      up2(fma2(y[k], al2, nm2), t0, t1);
      float e0 = fast_exp2(t0), e1 = fast_exp2(t1);
      if (MASK) {
        e0 = 2 * k <= kmax ? e0 : 0.0f;
        e1 = 2 * k + 1 <= kmax ? e1 : 0.0f;
      }
      acc[k % 4] = add2(acc[k % 4], pk2(e0, e1));
      w[e] = bf16x2(e0, e1);
    }
    *reinterpret_cast<uint4*>(prow + ((c ^ swz) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace pf
}  // namespace tria
