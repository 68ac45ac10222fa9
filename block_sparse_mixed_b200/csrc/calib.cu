// Synthetic per-head calibration of the boundaries (hi, keep) and the global
// allocator (rit.work TriAttention page, section "Как калибровка распределяет
// вычисления между головами", paragraphs one to three): each head's candidate
// boundary pairs are scored by the error they add after the output projection
// W_O, normalised by the layer's output energy, and priced by the work of the
// blocks they keep; a global allocator then spends extra work where it lowers
// the error most.
//
// Readings (the page gives no formulas): the reference output is the same
// attention with nothing skipped and every tile at 8 bits; the error of head h
// is sum over its rows of ||(O_c - O_ref) W_O[h]||^2 with W_O[h] the D rows of W_O
// that head h feeds, and the energy sum_h sum over rows of ||O_ref W_O[h]||^2
// (cross terms between heads dropped in both); a kept tile costs its query-key
// product and value aggregation (2 T^2 D operations each at 8 bits, half at 4
// bits) plus 4 T^2 for normalising its scores; the allocator starts every head at
// its cheapest candidate and repeatedly takes the single move to a costlier,
// lower-error candidate with the largest error decrease per unit of added cost
// that the budget allows (first in head-then-candidate order on equal ratios).
//
// On the GPU: the fused prefill computes every candidate's output for all heads
// at once (one launch per candidate, the Q codec and operand preparation shared),
// and ||dO W||^2 is evaluated as the quadratic form dO M dO^T with the per-head
// Gram matrix M = W_O[h] W_O[h]^T (D x D), so the projection to d_model is never
// materialised.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "tria.h"

namespace tria {
namespace {

constexpr int kGramRows = 8;     // rows of M per Gram CTA
constexpr int kGramK = 32;       // columns of W_O staged per step
constexpr int kErrRows = 256;    // rows of one head per error CTA

// M[h][i][j] = sum_k W[hD + i][k] W[hD + j][k], fp32, one CTA per (8 rows i, head h).
template <int D>
__global__ void __launch_bounds__(D) gram_kernel(const __nv_bfloat16* __restrict__ W, int d_model,
                                                 float* __restrict__ M) {
  __shared__ float tile[D][kGramK + 1];
  const int h = blockIdx.y, i0 = blockIdx.x * kGramRows, j = threadIdx.x;
  const __nv_bfloat16* Wh = W + static_cast<int64_t>(h) * D * d_model;
  float acc[kGramRows] = {};
  for (int k0 = 0; k0 < d_model; k0 += kGramK) {
    for (int e = threadIdx.x; e < D * kGramK; e += D) {
      const int r = e / kGramK, c = e % kGramK;
      tile[r][c] = k0 + c < d_model ? __bfloat162float(Wh[static_cast<int64_t>(r) * d_model + k0 + c]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kGramK; ++c) {
      const float wj = tile[j][c];
#pragma unroll
      for (int ii = 0; ii < kGramRows; ++ii) acc[ii] = fmaf(tile[i0 + ii][c], wj, acc[ii]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int ii = 0; ii < kGramRows; ++ii) M[(static_cast<int64_t>(h) * D + i0 + ii) * D + j] = acc[ii];
}

// partial[h][chunk] = sum over the chunk's rows of d M_h d^T, d = Oc - Oref (Oc null:
// d = Oref, the energy). Rows of head h are (b, s) of O [B, Hq, S, D]; a CTA of 2D
// threads takes two rows at a time, thread j forming (d M)_j and d_j (d M)_j.
template <int D>
__global__ void __launch_bounds__(2 * D) quad_form_kernel(const __nv_bfloat16* __restrict__ Oc,
                                                          const __nv_bfloat16* __restrict__ Oref,
                                                          const float* __restrict__ M, int B, int Hq, int S,
                                                          double* __restrict__ partial) {
  extern __shared__ float sm[];
  float* Ms = sm;                    // [D][D]
  float* ds = sm + D * D;            // [2][D]
  __shared__ double red[2 * D / 32];
  const int h = blockIdx.y;
  const int half = threadIdx.x / D, j = threadIdx.x % D;
  const float* Mh = M + static_cast<int64_t>(h) * D * D;
  for (int e = threadIdx.x; e < D * D; e += 2 * D) Ms[e] = Mh[e];
  const int64_t rows = static_cast<int64_t>(B) * S;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kErrRows;
  double acc = 0.0;
  for (int k = 0; k < kErrRows; k += 2) {
    const int64_t r = r0 + k + half;
    float d = 0.0f;
    if (r < rows) {
      const int64_t b = r / S, s = r % S;
      const int64_t off = ((b * Hq + h) * S + s) * D + j;
      d = __bfloat162float(Oref[off]);
      if (Oc != nullptr) d = __bfloat162float(Oc[off]) - d;
    }
    __syncthreads();                 // the previous rows' d are no longer read
    ds[half * D + j] = d;
    __syncthreads();
    float y = 0.0f;
    const float* dv = ds + half * D;
#pragma unroll 16
    for (int i = 0; i < D; ++i) y = fmaf(dv[i], Ms[i * D + j], y);
    acc += static_cast<double>(d) * static_cast<double>(y);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 2 * D / 32; ++w) t += red[w];
    partial[static_cast<int64_t>(h) * gridDim.x + blockIdx.x] = t;
  }
}

// Host: the cost of one candidate over nb x nb causal blocks.
int64_t candidate_cost(int nb, int T, int D, int hi, int keep) {
  const int64_t tt = static_cast<int64_t>(T) * T;
  const int64_t c8 = 4 * tt * D + 4 * tt, c4 = 2 * tt * D + 4 * tt;
  int64_t n8 = 0, n4 = 0;
  for (int i = 0; i < nb; ++i)
    for (int j = 0; j <= i; ++j) {
      const int a = tile_action(i, j, hi, keep);
      n8 += a == ACT_INT8;
      n4 += a == ACT_INT4;
    }
  return n8 * c8 + n4 * c4;
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct CalibLayout {
  size_t prefill, o_ref, o_c, lse, gram, partial, total;
  int chunks;
};

CalibLayout calib_layout(const tria_dims& d) {
  CalibLayout L{};
  const size_t orows = static_cast<size_t>(d.B) * d.Hq * d.S;
  L.chunks = static_cast<int>((static_cast<int64_t>(d.B) * d.S + kErrRows - 1) / kErrRows);
  size_t off = 0;
  L.prefill = off; off += align_up(tria_prefill_workspace_bytes(&d));
  L.o_ref = off; off += align_up(orows * d.D * 2);
  L.o_c = off; off += align_up(orows * d.D * 2);
  L.lse = off; off += align_up(orows * 4);
  L.gram = off; off += align_up(static_cast<size_t>(d.Hq) * d.D * d.D * 4);
  L.partial = off; off += align_up(static_cast<size_t>(d.Hq) * L.chunks * 8);
  L.total = off;
  return L;
}

template <int D>
cudaError_t launch_quad(const __nv_bfloat16* Oc, const __nv_bfloat16* Oref, const float* M, const tria_dims& d,
                        int chunks, double* partial, cudaStream_t st) {
  const int smem = (D * D + 2 * D) * 4;
  cudaError_t e = cudaFuncSetAttribute(quad_form_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  quad_form_kernel<D><<<dim3(chunks, d.Hq), 2 * D, smem, st>>>(Oc, Oref, M, d.B, d.Hq, d.S, partial);
  return cudaGetLastError();
}

// Sum of each head's partials in a fixed order (deterministic).
int read_partials(const double* dev, int Hq, int chunks, double* out, cudaStream_t st) {
  std::vector<double> h(static_cast<size_t>(Hq) * chunks);
  if (cudaMemcpyAsync(h.data(), dev, h.size() * 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return TRIA_ERR_CUDA;
  for (int k = 0; k < Hq; ++k) {
    double t = 0.0;
    for (int c = 0; c < chunks; ++c) t += h[static_cast<size_t>(k) * chunks + c];
    out[k] = t;
  }
  return TRIA_OK;
}

}  // namespace
}  // namespace tria

using namespace tria;

extern "C" {

int tria_calibration_costs(int nb, int T, int D, const int32_t* cand_hi, const int32_t* cand_keep, int C,
                           int64_t* cost) {
  if (nb < 0 || T < 1 || D < 1 || C < 0 || (C > 0 && (cand_hi == nullptr || cand_keep == nullptr || cost == nullptr)))
    return TRIA_ERR_INVALID_ARG;
  for (int c = 0; c < C; ++c) {
    if (cand_hi[c] < 0 || cand_keep[c] < cand_hi[c]) return TRIA_ERR_INVALID_ARG;
    cost[c] = candidate_cost(nb, T, D, cand_hi[c], cand_keep[c]);
  }
  return TRIA_OK;
}

int tria_allocate(const double* err, const int64_t* cost, int C, int H, int64_t budget, int32_t* choice) {
  if (C < 1 || H < 1 || err == nullptr || cost == nullptr || choice == nullptr) return TRIA_ERR_INVALID_ARG;
  auto E = [&](int c, int h) { return err[static_cast<int64_t>(c) * H + h]; };
  auto K = [&](int c, int h) { return cost[static_cast<int64_t>(c) * H + h]; };
  int64_t spent = 0;
  for (int h = 0; h < H; ++h) {     // the cheapest candidate (then the lower error, then the first)
    int best = 0;
    for (int c = 1; c < C; ++c)
      if (K(c, h) < K(best, h) || (K(c, h) == K(best, h) && E(c, h) < E(best, h))) best = c;
    choice[h] = best;
    spent += K(best, h);
  }
  while (true) {
    int bh = -1, bc = -1;
    double br = 0.0;
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < C; ++c) {
        const int64_t added = K(c, h) - K(choice[h], h);
        const double gain = E(choice[h], h) - E(c, h);
        if (added <= 0 || gain <= 0.0 || spent + added > budget) continue;
        const double ratio = gain / static_cast<double>(added);
        if (bh < 0 || ratio > br) {
          br = ratio;
          bh = h;
          bc = c;
        }
      }
    if (bh < 0) return TRIA_OK;
    spent += K(bc, bh) - K(choice[bh], bh);
    choice[bh] = bc;
  }
}

size_t tria_calibrate_workspace_bytes(const tria_dims* dims, int d_model) {
  if (dims == nullptr || d_model < 1 || tria_prefill_workspace_bytes(dims) == 0) return 0;
  return calib_layout(*dims).total;
}

int tria_calibrate(const void* Q, const tria_kv_cache* cache, const tria_dims* dims, const void* W_O, int d_model,
                   const int32_t* cand_hi, const int32_t* cand_keep, int C, double* err, double* energy,
                   void* workspace, size_t workspace_bytes, void* stream) {
  if (dims == nullptr || tria_prefill_workspace_bytes(dims) == 0) return TRIA_ERR_INVALID_ARG;
  const tria_dims d = *dims;
  if (W_O == nullptr || (reinterpret_cast<uintptr_t>(W_O) & 15u) != 0 || d_model < 1 || C < 1 ||
      cand_hi == nullptr || cand_keep == nullptr || err == nullptr || energy == nullptr)
    return TRIA_ERR_INVALID_ARG;
  for (int c = 0; c < C; ++c)
    if (cand_hi[c] < 0 || cand_keep[c] < cand_hi[c]) return TRIA_ERR_INVALID_ARG;
  const CalibLayout L = calib_layout(d);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < L.total)
    return TRIA_ERR_WORKSPACE;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* pws = ws + L.prefill;
  const size_t pbytes = L.o_ref - L.prefill;
  auto* o_ref = reinterpret_cast<__nv_bfloat16*>(ws + L.o_ref);
  auto* o_c = reinterpret_cast<__nv_bfloat16*>(ws + L.o_c);
  auto* lse = reinterpret_cast<float*>(ws + L.lse);
  auto* M = reinterpret_cast<float*>(ws + L.gram);
  auto* partial = reinterpret_cast<double*>(ws + L.partial);

  // Q codec and operand tiles: shared by every candidate
  int s = tria_prefill_prepare(Q, cache, dims, pws, pbytes, stream);
  if (s != TRIA_OK) return s;
  const auto* W = static_cast<const __nv_bfloat16*>(W_O);
  if (d.D == 128) gram_kernel<128><<<dim3(128 / kGramRows, d.Hq), 128, 0, st>>>(W, d_model, M);
  else gram_kernel<64><<<dim3(64 / kGramRows, d.Hq), 64, 0, st>>>(W, d_model, M);
  if (cudaGetLastError() != cudaSuccess) return TRIA_ERR_CUDA;
  auto quad = [&](const __nv_bfloat16* oc) {
    return d.D == 128 ? launch_quad<128>(oc, o_ref, M, d, L.chunks, partial, st)
                      : launch_quad<64>(oc, o_ref, M, d, L.chunks, partial, st);
  };

  const int nb = d.S / d.T;
  std::vector<int32_t> hi(d.Hq, nb), keep(d.Hq, nb);
  if ((s = tria_prefill_attend(cache, dims, hi.data(), keep.data(), o_ref, lse, pws, pbytes, stream)) != TRIA_OK)
    return s;
  if (quad(nullptr) != cudaSuccess) return TRIA_ERR_CUDA;
  if ((s = read_partials(partial, d.Hq, L.chunks, energy, st)) != TRIA_OK) return s;
  for (int c = 0; c < C; ++c) {
    std::fill(hi.begin(), hi.end(), cand_hi[c]);
    std::fill(keep.begin(), keep.end(), cand_keep[c]);
    if ((s = tria_prefill_attend(cache, dims, hi.data(), keep.data(), o_c, lse, pws, pbytes, stream)) != TRIA_OK)
      return s;
    if (quad(o_c) != cudaSuccess) return TRIA_ERR_CUDA;
    if ((s = read_partials(partial, d.Hq, L.chunks, err + static_cast<int64_t>(c) * d.Hq, st)) != TRIA_OK)
      return s;
  }
  return tria_workspace_status(pws, stream);
}

}  // extern "C"
