// Fused block-sparse mixed-precision causal prefill for sm_100a.
//
// What it computes (rit.work TriAttention page, section "Какие связи можно не
// считать, а какие нельзя удалять", and section "Как калибровка распределяет
// вычисления между головами", last paragraph): for every query row, softmax
// attention over the key blocks its query block keeps, each block at its own
// precision (8-bit near the diagonal, 4-bit in the next band, block 0 and the
// diagonal always 8-bit, far blocks skipped), reduced into one normalised
// output O and its natural log-sum-exp.
//
// How. A persistent CTA owns one 128-row query tile at a time (one query block
// of T = 128, or two query blocks of T = 64) of one (batch, query head). The
// key blocks the tile keeps are walked in ascending order; a key block whose
// rows need both planes is loaded once per plane. Warp roles:
//   warps 0-3  softmax: one TMEM lane (query row) per thread;
//   warp 4     producer: TMA loads of Q codes, K codes, V tiles and K scales,
//              only for kept (block, plane) pairs;
//   warp 5     MMA issuer: S = Q.K^T on tcgen05 kind::i8 (int32 in TMEM), then
//              O += P.V on tcgen05 kind::f16 (bf16 P read from TMEM, fp32 O in TMEM).
// S is double-buffered in TMEM so QK of load g+1 overlaps the softmax of load g.
// The softmax dequantises S with the row's Q scale and the key's K scale,
// applies the causal mask on the diagonal block, keeps a running maximum that
// is only raised when it grows by more than 2^8 (so O is rarely rescaled),
// writes P as bf16 over the S columns, and finally normalises O.
// Rows whose own tile action differs from the load's plane write P = 0.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace tria {
namespace {

constexpr int kRows = 128;             // query rows per tile (tcgen05 M)
constexpr int kThreads = 192;          // 4 softmax warps + producer warp + MMA warp
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kSlots = 2;              // S buffers in TMEM
constexpr int kTmemCols = 512;
constexpr int kOCol = 256;             // O accumulator columns [256, 256 + D)
constexpr float kRescaleLog2 = 8.0f;   // raise the running max only past this growth

template <int T, int D>
struct Cfg {
  static constexpr int kQBlocks = kRows / T;                 // query blocks per tile
  static constexpr int kKTile = T * kQKRowBytes;             // K codes per stage
  static constexpr int kVSub = D * 128;                      // one V sub-tile: D rows x 64 keys
  static constexpr int kVTile = D * T * 2;                   // all V sub-tiles of a stage
  static constexpr int kStageRaw = kKTile + kVTile + T * 4;
  static constexpr int kStage = (kStageRaw + 1023) / 1024 * 1024;
  static constexpr int kStages = T == 128 ? 3 : 4;
  static constexpr int kQTile = kRows * kQKRowBytes;
  static constexpr int kOffQ8 = 0;
  static constexpr int kOffQ4 = kQTile;
  static constexpr int kOffStage = 2 * kQTile;
  static constexpr int kOffBar = kOffStage + kStages * kStage;
  // barriers + alignment slack; never below 120 KB so that exactly one CTA (which
  // owns all 512 TMEM columns) is resident per SM
  static constexpr int kSmemNeed = kOffBar + 1024 + 1024;
  static constexpr int kSmem = kSmemNeed > 120 * 1024 ? kSmemNeed : 120 * 1024;
  static constexpr uint32_t kStageTx = kKTile + kVTile + T * 4;
  static constexpr uint32_t kIdescQK = idesc_i8(kRows, T);
  static constexpr uint32_t kIdescPV = idesc_bf16(kRows, D);
};

struct Bars {
  uint64_t q_full, q_empty, fin;
  uint64_t o_done[2];   // P.V of load g completes phase g/2 of o_done[g % 2]
  uint64_t kv_full[4], kv_empty[4];
  uint64_t s_full[kSlots], s_free[kSlots], p_full[kSlots];
  uint32_t tmem_base;
  int abort;
};

// The (key block, plane) loads of one query tile, in ascending key-block order;
// at a key block the 8-bit load (if any row needs it) comes before the 4-bit one.
struct LoadSeq {
  int i0, nq, hi, keep, j, jmax, jband, step;
  __device__ void init(int i0_, int nq_, int hi_, int keep_) {
    i0 = i0_; nq = nq_; hi = hi_; keep = keep_;
    jmax = i0 + nq - 1; j = 0; step = 0;
    jband = first_band_block(i0, keep);
  }
  __device__ bool next(int& jo, int& plane) {
    while (j <= jmax) {
      bool n8 = false, n4 = false;
      for (int q = 0; q < nq; ++q) {
        const int a = tile_action(i0 + q, j, hi, keep);
        n8 |= a == ACT_INT8;
        n4 |= a == ACT_INT4;
      }
      if (step == 0) {
        step = 1;
        if (n8) { jo = j; plane = 8; return true; }
      }
      step = 0;
      const int jj = j;
      j = (j == 0) ? jband : j + 1;
      if (n4) { jo = jj; plane = 4; return true; }
    }
    return false;
  }
};

struct Unit {
  int b, hq, kvh, i0, nq;
};

__device__ __forceinline__ Unit unit_of(const PrefillArgs& a, int w, int nqb) {
  Unit u;
  const int bh_count = a.B * a.Hq;
  const int qt = a.n_qtiles - 1 - w / bh_count;     // last query tiles first (longest rows)
  const int bh = w % bh_count;
  u.b = bh / a.Hq;
  u.hq = bh % a.Hq;
  u.kvh = u.hq / a.G;
  u.i0 = qt * nqb;
  u.nq = min(nqb, a.nb - u.i0);
  return u;
}

// Bounded wait that ignores the abort flag: used on the way out to let copies and
// tensor-core ops already in flight land before the CTA releases its memory.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_timer();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer() - t0 > kWaitLimitNs) return;
  }
}

template <int T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  using C = Cfg<T, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->fin, 1);
    mbar_init(&bars->o_done[0], 1);
    mbar_init(&bars->o_done[1], 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], 1);
      mbar_init(&bars->p_full[s], 128);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&maps.q8); prefetch_tensormap(&maps.q4);
    prefetch_tensormap(&maps.k8); prefetch_tensormap(&maps.k4);
    prefetch_tensormap(&maps.v8); prefetch_tensormap(&maps.v4);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  uint8_t* sQ8 = smem + C::kOffQ8;
  uint8_t* sQ4 = smem + C::kOffQ4;
  auto sK = [&](int s) { return smem + C::kOffStage + s * C::kStage; };
  auto sV = [&](int s) { return smem + C::kOffStage + s * C::kStage + C::kKTile; };
  auto sScale = [&](int s) {
    return reinterpret_cast<float*>(smem + C::kOffStage + s * C::kStage + C::kKTile + C::kVTile);
  };

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t g = 0, uloc = 0, q_issued = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < a.n_units && ok; w += gridDim.x, ++uloc) {
        const Unit u = unit_of(a, w, C::kQBlocks);
        if (uloc > 0 && !(ok = mbar_wait(&bars->q_empty, (uloc - 1) & 1, abort, a.err))) break;
        ++q_issued;
        const int qrow = (u.b * a.Hq + u.hq) * a.S + u.i0 * T;
        mbar_arrive_expect_tx(&bars->q_full, 2 * C::kQTile);
        tma_load_2d(sQ8, &maps.q8, &bars->q_full, 0, qrow);
        tma_load_2d(sQ4, &maps.q4, &bars->q_full, 0, qrow);
        LoadSeq seq;
        seq.init(u.i0, u.nq, a.hi[u.hq], a.keep[u.hq]);
        const int64_t grp = static_cast<int64_t>(u.b) * a.Hkv + u.kvh;
        int j, plane;
        while (seq.next(j, plane)) {
          const int st = g % C::kStages;
          if (g >= static_cast<uint32_t>(C::kStages) &&
              !(ok = mbar_wait(&bars->kv_empty[st], ((g / C::kStages) - 1) & 1, abort, a.err)))
            break;
          mbar_arrive_expect_tx(&bars->kv_full[st], C::kStageTx);
          const int krow = static_cast<int>(grp * (plane == 8 ? a.cap8 : static_cast<int64_t>(a.S)) +
                                            static_cast<int64_t>(j) * T);
          tma_load_2d(sK(st), plane == 8 ? &maps.k8 : &maps.k4, &bars->kv_full[st], 0, krow);
          const int vrow = static_cast<int>((grp * a.nb + j) * D);
#pragma unroll
          for (int q = 0; q < T / 64; ++q)
            tma_load_2d(sV(st) + q * C::kVSub, plane == 8 ? &maps.v8 : &maps.v4, &bars->kv_full[st], 64 * q,
                        vrow);
          const float* ks = (plane == 8 ? a.k8s : a.k4s) + grp * a.cap + static_cast<int64_t>(j) * T;
          bulk_load(sScale(st), ks, T * 4, &bars->kv_full[st]);
          ++g;
        }
      }
      // let every copy this CTA issued land before the block exits
      for (uint32_t k = (g > static_cast<uint32_t>(C::kStages) ? g - C::kStages : 0); k < g; ++k)
        drain_wait(&bars->kv_full[k % C::kStages], (k / C::kStages) & 1);
      if (q_issued > 0) drain_wait(&bars->q_full, (q_issued - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t g = 0, uloc = 0;
      bool ok = true;
      const uint32_t q8a = smem_u32(sQ8), q4a = smem_u32(sQ4);
      auto pv = [&](uint32_t gg, bool first) -> bool {
        const int st = gg % C::kStages, sl = gg % kSlots;
        if (!mbar_wait(&bars->p_full[sl], (gg / kSlots) & 1, abort, a.err)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_u32(sV(st));
#pragma unroll
        for (int s = 0; s < T / 16; ++s) {
          const uint64_t bdesc = sw128_desc(vbase + (s / 4) * C::kVSub + (s % 4) * 32);
          mma_bf16_ts(tmem + kOCol, tmem + sl * T + s * 8, bdesc, C::kIdescPV, (first && s == 0) ? 0u : 1u);
        }
        mma_commit(&bars->kv_empty[st]);
        mma_commit(&bars->s_free[sl]);
        mma_commit(&bars->o_done[gg % 2]);
        return true;
      };
      for (int w = blockIdx.x; w < a.n_units && ok; w += gridDim.x, ++uloc) {
        const Unit u = unit_of(a, w, C::kQBlocks);
        if (!(ok = mbar_wait(&bars->q_full, uloc & 1, abort, a.err))) break;
        tc_fence_after();
        LoadSeq seq;
        seq.init(u.i0, u.nq, a.hi[u.hq], a.keep[u.hq]);
        int j, plane, l = 0;
        while (seq.next(j, plane)) {
          const int st = g % C::kStages, sl = g % kSlots;
          if (!(ok = mbar_wait(&bars->kv_full[st], (g / C::kStages) & 1, abort, a.err))) break;
          if (g >= static_cast<uint32_t>(kSlots) &&
              !(ok = mbar_wait(&bars->s_free[sl], ((g / kSlots) - 1) & 1, abort, a.err)))
            break;
          tc_fence_after();
          const uint32_t abase = plane == 8 ? q8a : q4a;
          const uint32_t bbase = smem_u32(sK(st));
#pragma unroll
          for (int k = 0; k < kQKRowBytes / 32; ++k)
            mma_i8_ss(tmem + sl * T, sw128_desc(abase + 32 * k), sw128_desc(bbase + 32 * k), C::kIdescQK,
                      k > 0 ? 1u : 0u);
          mma_commit(&bars->s_full[sl]);
          if (l > 0 && !(ok = pv(g - 1, l == 1))) break;
          ++l;
          ++g;
        }
        if (!ok) break;
        if (l > 0 && !(ok = pv(g - 1, l == 1))) break;
        mma_commit(&bars->q_empty);
      }
      // wait for every tensor-core op this CTA issued before TMEM is released
      mma_commit(&bars->fin);
      drain_wait(&bars->fin, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int row = threadIdx.x;                        // TMEM lane = query row of the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t g = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < a.n_units && ok; w += gridDim.x) {
      const Unit u = unit_of(a, w, C::kQBlocks);
      const int qb = row / T;
      const int rl = row % T;
      const bool valid = qb < u.nq;
      const int ir = u.i0 + qb;
      const int64_t qrow = (static_cast<int64_t>(u.b) * a.Hq + u.hq) * a.S + static_cast<int64_t>(ir) * T + rl;
      const float a8 = valid ? a.q8s[qrow] * a.qk_log2 : 0.0f;
      const float a4 = valid ? a.q4s[qrow] * a.qk_log2 : 0.0f;
      const int hi = a.hi[u.hq], keep = a.keep[u.hq];
      float m_run = -INFINITY, l_run = 0.0f;
      LoadSeq seq;
      seq.init(u.i0, u.nq, hi, keep);
      int j, plane;
      while (seq.next(j, plane)) {
        const int st = g % C::kStages, sl = g % kSlots;
        if (!(ok = mbar_wait(&bars->kv_full[st], (g / C::kStages) & 1, abort, a.err))) break;
        if (!(ok = mbar_wait(&bars->s_full[sl], (g / kSlots) & 1, abort, a.err))) break;
        tc_fence_after();
        const int act = valid ? tile_action(ir, j, hi, keep) : ACT_NONE;
        const uint32_t s_addr = lane_addr + sl * T;
        if (act == plane) {
          uint32_t r[T];
#pragma unroll
          for (int c = 0; c < T / 32; ++c) tmem_ld32(s_addr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
          tmem_wait_ld();
          const float* ks = sScale(st);
          const float alpha = plane == 8 ? a8 : a4;
          const bool diag = (j == ir);
          float mx = -INFINITY;
#pragma unroll
          for (int n = 0; n < T; ++n) {
            float y = __int2float_rn(static_cast<int>(r[n])) * ks[n];
            if (diag && n > rl) y = -INFINITY;
            mx = fmaxf(mx, y);
            r[n] = __float_as_uint(y);
          }
          const float m_tile = mx * alpha;
          const bool raise = m_tile > m_run + kRescaleLog2;
          const float sc = raise ? fast_exp2(m_run - m_tile) : 1.0f;
          // TMEM loads/stores are warp-collective: the whole warp rescales its O rows
          // when any lane must (lanes that need not use the factor 1).
          if (__any_sync(0xffffffffu, raise && l_run > 0.0f)) {
            // O holds earlier loads of this tile: wait for the previous P.V first.
            if (!(ok = mbar_wait(&bars->o_done[(g - 1) % 2], ((g - 1) / 2) & 1, abort, a.err))) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(lane_addr + kOCol + 32 * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * sc);
              tmem_st32(lane_addr + kOCol + 32 * c, o);
            }
          }
          if (raise) {
            l_run *= sc;
            m_run = m_tile;
          }
          float sum = 0.0f;
#pragma unroll
          for (int c = 0; c < T / 64; ++c) {
            uint32_t pk[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const int n = 64 * c + 2 * k;
              const float y0 = __uint_as_float(r[n]), y1 = __uint_as_float(r[n + 1]);
              const float p0 = (diag && n > rl) ? 0.0f : fast_exp2(fmaf(y0, alpha, -m_run));
              const float p1 = (diag && n + 1 > rl) ? 0.0f : fast_exp2(fmaf(y1, alpha, -m_run));
              sum += p0 + p1;
              const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
              pk[k] = *reinterpret_cast<const uint32_t*>(&h);
            }
            tmem_st32(s_addr + 32 * c, pk);
          }
          l_run += sum;
        } else {
          uint32_t z[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) z[k] = 0u;
#pragma unroll
          for (int c = 0; c < T / 64; ++c) tmem_st32(s_addr + 32 * c, z);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[sl]);
        ++g;
      }
      if (!ok) break;
      // epilogue: wait for the last P.V of the tile, normalise, store. Having seen QK of
      // load gl complete, every P.V up to gl-2 is complete, so o_done[gl % 2] is at most
      // one phase short of the one awaited and its parity is unambiguous.
      const uint32_t gl = g - 1;
      if (!(ok = mbar_wait(&bars->o_done[gl % 2], (gl / 2) & 1, abort, a.err))) break;
      tc_fence_after();
      const float inv_l = valid ? 1.0f / l_run : 0.0f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(lane_addr + kOCol + 32 * c, o);
        tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(a.O + qrow * D + 32 * c);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(o[8 * k + 2 * e]) * inv_l,
                                                             __uint_as_float(o[8 * k + 2 * e + 1]) * inv_l);
              wv[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            dst[k] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        }
      }
      if (valid) a.LSE[qrow] = (m_run + log2f(l_run)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int T, int D>
cudaError_t launch_t(const PrefillArgs& a, const PrefillMaps& maps, int num_sms, cudaStream_t stream) {
  using C = Cfg<T, D>;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = a.n_units < num_sms ? a.n_units : num_sms;
  if (grid <= 0) return cudaSuccess;
  prefill_kernel<T, D><<<grid, kThreads, C::kSmem, stream>>>(a, maps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, const PrefillMaps& maps, int D, int T, int num_sms,
                           cudaStream_t stream) {
  if (T == 128 && D == 128) return launch_t<128, 128>(a, maps, num_sms, stream);
  if (T == 64 && D == 128) return launch_t<64, 128>(a, maps, num_sms, stream);
  if (T == 128 && D == 64) return launch_t<128, 64>(a, maps, num_sms, stream);
  return launch_t<64, 64>(a, maps, num_sms, stream);
}

}  // namespace tria
