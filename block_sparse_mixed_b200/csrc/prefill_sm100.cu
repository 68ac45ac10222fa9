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
// How. A persistent CTA takes 128-row query tiles (one query block of T = 128,
// or two query blocks of T = 64, of one (batch, query head)) from a kernel-wide
// counter, longest rows first. A tile's kept (key block, plane) pairs are walked
// by the producers only: first the 8-bit blocks, then the 4-bit ones, grouped into
// loads of 128 keys (one block at T = 128; any two blocks of one plane at T = 64,
// a lone block's copy in the second half masked). Warp roles:
//   warps 0-15  softmax, as two "pairs" of warpgroups that take the loads in
//               turn (pair p handles loads of parity p, with S slot p in TMEM, P
//               buffer p in shared memory and O accumulator p in TMEM). Inside a
//               pair, warpgroup `half` takes keys [64 half, 64 half + 64) of every
//               row (its own key block at T = 64); the two halves agree on the row
//               maximum through shared memory and a named barrier.
//   warp 16     producer: tile index and load count (a ring of 16 entries), the
//               tile's Q codes, then per load the K codes (a ring of 3 stages) and
//               the K scales with the load's blocks, plane and last-of-tile flag (a
//               ring of 4 stages). TMA, no multicast, only kept blocks.
//   warp 17     QK issuer: S = Q.K^T on tcgen05 (kind::i8 with int32 S for the
//               8-bit plane; kind::f8f6f4 on e4m3 operands, exact for 4-bit codes,
//               with fp32 S for the 4-bit plane). A pair's slot is refilled as soon
//               as the pair has read S into registers, so the next S of a pair is
//               computed while the pair still works on the current one.
//   warp 18     producer of the V tiles (a ring of 2 stages, one per pair).
//   warp 19     P.V issuer: O += P.V on kind::f16, bf16 P and V^T from shared memory,
//               both K-major, fp32 O in TMEM; each P.V frees its V stage, P buffer and
//               the accumulator for the pair's next load.
// Each ring is released as soon as its contents are used (K by the QK's
// completion, the scales after the softmax's first pass, V and P by the P.V's
// completion), so no stage is held across another role's round trip.
// The softmax dequantises S with the row's Q scale and the key's K scale, masks
// the diagonal block causally, keeps a running maximum that is only raised when
// it grows by more than 2^8 (so O is rarely rescaled), and writes P as bf16 into
// the pair's buffer in the swizzled K-major layout the tensor core reads. Rows
// whose own tile action differs from the load's plane write P = 0. The two
// accumulators of a row are merged and normalised in the tile epilogue.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "load_plan.cuh"
#include "prefill_common.cuh"

namespace tria {
namespace {

using namespace pf;

constexpr int kRows = 128;              // query rows per tile (tcgen05 M)
constexpr int kThreads = 640;           // 20 warps
constexpr int kSoftmaxWarps = 16;
constexpr int kPairWarps = 8;           // softmax warps of one pair (P arrivals per load, one per warp)
constexpr int kProducerWarp = 16;       // Q, K codes, K scales
constexpr int kMmaWarp = 17;            // QK issuer; allocates TMEM
constexpr int kVProducerWarp = 18;      // V tiles
constexpr int kPvWarp = 19;             // P.V issuer
// Register split (setmaxnreg): launched at 96 per thread (640 x 96 = 61,440; five
// warps per sub-partition x 32 x 96 = 15,360 of its 16,384); the four softmax
// warpgroups rise to 104 and the producer/MMA warpgroup drops to 64:
// 4 x 128 x 104 + 128 x 64 = 61,440, within the launch total.
constexpr int kRegsSoftmax = 104;
constexpr int kRegsOther = 64;
constexpr int kPairs = 2;               // softmax pairs = O accumulators in TMEM
constexpr int kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;    // raise the running max only past this growth

// O accumulator of pair p: D columns at 256 + 128 p.
__host__ __device__ constexpr uint32_t o_col(int p) { return p == 0 ? 256u : 384u; }

// A load carries 128 keys: one key block at T = 128, two key blocks of the same
// plane at T = 64 (the producer pairs them; a block left alone is loaded twice
// and its second copy masked). The tensor-core side is the same for both.
constexpr int kKeys = 128;

template <int T, int D>
struct Cfg {
  static constexpr int kQBlocks = kRows / T;                 // query blocks per tile
  static constexpr int kBlocksPerLoad = kKeys / T;           // key blocks per load
  static constexpr int kQTile = kRows * kQKRowBytes;         // Q codes of one plane
  static constexpr int kKTile = kKeys * kQKRowBytes;         // K codes of one load
  static constexpr int kVSub = D * 128;                      // one V sub-tile: D rows x 64 keys
  static constexpr int kVTile = D * kKeys * 2;               // both V sub-tiles of a load
  static constexpr int kPSub = kRows * 128;                  // one P sub-tile: 128 rows x 64 keys
  static constexpr int kPTile = kRows * kKeys * 2;           // P of one load (bf16)
  static constexpr int kScTile = kKeys * 4;                  // K scales of one load
  // Rings. K codes are released when the QK that reads them completes, V when
  // its P.V completes, and the K scales when the softmax has read them, so each
  // kind of operand is held only as long as it is used.
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;                         // = pairs: stage g % 2 is pair g % 2's
  static constexpr int kScStages = 4;
  static constexpr int kSlots = 2;                           // S slots in TMEM, one per pair
  static constexpr int kOffQ8 = 0;
  static constexpr int kOffQ4 = kQTile;
  static constexpr int kOffK = 2 * kQTile;
  static constexpr int kOffV = kOffK + kKStages * kKTile;
  static constexpr int kOffP = kOffV + kVStages * kVTile;    // P buffer of pair p at kOffP + p * kPTile
  static constexpr int kOffSc = kOffP + 2 * kPTile;
  static constexpr int kOffBar = kOffSc + kScStages * kScTile;
  static constexpr int kOffX = kOffBar + 1024;               // row-max and epilogue exchanges
  static constexpr int kXBytes = 2 * 2 * 128 * 4 + 2 * 2 * 2 * 2 * 128 * 4;   // 2 KB + 8 KB
  // never below 120 KB so that exactly one CTA (which owns all 512 TMEM columns)
  // is resident per SM
  static constexpr int kSmemNeed = kOffX + kXBytes + 1024;
  static constexpr int kSmem = kSmemNeed > 120 * 1024 ? kSmemNeed : 120 * 1024;
  static_assert(kSmemNeed <= 227 * 1024, "shared memory");
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0 && kKTile % 1024 == 0 &&
                    kVSub % 1024 == 0 && kPSub % 1024 == 0,
                "swizzled operand tiles start on 1024-byte boundaries");
  static constexpr uint32_t kIdescQK = idesc_i8(kRows, kKeys);       // 8-bit plane: int8, int32 S
  static constexpr uint32_t kIdescQK4 = idesc_e4m3(kRows, kKeys);    // 4-bit plane: e4m3, fp32 S (exact)
  static constexpr uint32_t kIdescPV = idesc_bf16(kRows, D);
};

constexpr int kUnitRing = 16;           // tiles published ahead of the consumers

struct Bars {
  uint64_t q_full, q_empty, fin, fin_pv;
  uint64_t o_fin;               // every P.V of the CTA's u-th tile: phase u
  uint64_t k_full[3], k_empty[3];       // K ring: emptied by the QK's completion
  uint64_t v_full[2], v_empty[2];       // V ring: emptied by the P.V's completion, which
                                        // also frees the pair's P buffer and O accumulator
  uint64_t sc_full[4], sc_empty[4];     // K scales + load info: emptied by the softmax pair
  uint64_t s_full[2], s_free[2];        // S slot written by QK / read out by the pair
  uint64_t p_full[2];                   // the pair's P buffer written
  uint32_t tmem_base;
  int abort;
  // Published by the producer so that the QK issuer, the P.V issuer and the
  // softmax need not walk the load sequence (the V producer walks it itself, from
  // the same tile entries): per K stage and per scale stage the load's key blocks and plane
  // (kLastLoad marks a tile's last load), visible after the stage's full barrier;
  // per tile u of this CTA, the tile's index and load count in ring entry
  // u % kUnitRing (index -1: no more tiles), visible after phase u / kUnitRing of
  // unit_ready[u % kUnitRing]. The ring cannot be lapped: a tile has at least one
  // load, and the producer runs at most a few loads ahead of the slowest reader.
  int4 k_info[3], sc_info[4];   // (j0, j1, plane | kLastLoad, 0)
  int unit_w[kUnitRing], unit_loads[kUnitRing];
  uint64_t unit_ready[kUnitRing];
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

constexpr int kLastLoad = 1 << 8;       // flag in info[].z next to the plane

struct Unit {
  int b, hq, kvh, i0, nq;
};

// Units: the last query tiles (longest rows) first, all (batch, head) of one tile
// index next to each other. (Going KV group by KV group, so that concurrent CTAs share
// one group's K/V band in L2, cut DRAM re-reads but measured slower.)
__device__ __forceinline__ Unit unit_of(const PrefillArgs& a, int w, int nqb) {
  Unit u;
  const int bh_count = a.B * a.Hq;
  const int qt = a.n_qtiles - 1 - w / bh_count;
  const int bh = w % bh_count;
  u.b = bh / a.Hq;
  u.hq = bh % a.Hq;
  u.kvh = u.hq / a.G;
  u.i0 = qt * nqb;
  u.nq = min(nqb, a.nb - u.i0);
  return u;
}

// PAGED: the cache is paged (block table); the contiguous instantiation keeps the
// producer's per-block arithmetic minimal, which measured worth 7% at T = 64.
template <int T, int D, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  using C = Cfg<T, D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, computed on the __shared__ array itself so that the
  // compiler keeps every access below in the shared address space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->fin, 1);
    mbar_init(&bars->fin_pv, 1);
    mbar_init(&bars->o_fin, 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < C::kScStages; ++s) {
      mbar_init(&bars->sc_full[s], 1);
      mbar_init(&bars->sc_empty[s], kPairWarps);
    }
    for (int r = 0; r < kUnitRing; ++r) mbar_init(&bars->unit_ready[r], 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], kPairWarps);
      mbar_init(&bars->p_full[s], kPairWarps);
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
  }
  if (warp == kVProducerWarp && lane == 0) {
    prefetch_tensormap(&maps.v8); prefetch_tensormap(&maps.v4);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // One CTA per SM allocates all 512 columns, so the allocation starts at lane 0,
  // column 0; TMEM addresses below are then compile-time constants plus uniform
  // offsets. A different base is reported as an error and the CTA does no work.
  constexpr uint32_t tmem = 0;
  if (bars->tmem_base != 0) {
    if (threadIdx.x == 0) atomicExch(a.err, TRIA_ERR_BOUNDS);
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(bars->tmem_base, kTmemCols);
    }
    return;
  }

  uint8_t* sQ8 = smem + C::kOffQ8;
  uint8_t* sQ4 = smem + C::kOffQ4;
  auto sK = [&](int s) { return smem + C::kOffK + s * C::kKTile; };
  auto sV = [&](int s) { return smem + C::kOffV + s * C::kVTile; };
  auto sP = [&](int p) { return smem + C::kOffP + p * C::kPTile; };
  auto sScale = [&](int s) { return reinterpret_cast<float*>(smem + C::kOffSc + s * C::kScTile); };

  if (warp >= kSoftmaxWarps) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    // The producer and MMA loops run on the whole warp, so that their operands are
    // warp-uniform (uniform registers); one elected lane issues the copies and the
    // tensor-core ops, and the same lane issues the commits that track them.
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, a.err));
    };
    if (warp == kProducerWarp) {
      // ---------------------------------------------------------- producer: Q, K, scales
      uint32_t g = 0, uloc = 0;
      bool ok = true;
      for (;; ++uloc) {
        // next tile from the kernel-wide counter (longest tiles first, see unit_of)
        int w = 0;
        if (lane == 0) w = atomicAdd(a.work, 1);
        w = __shfl_sync(0xffffffffu, w, 0);
        const int r = uloc % kUnitRing;
        if (w >= a.n_units) {
          if (elect_one()) {
            bars->unit_w[r] = -1;
            mbar_arrive(&bars->unit_ready[r]);
          }
          __syncwarp();
          break;
        }
        const Unit u = unit_of(a, w, C::kQBlocks);
        const int n_loads = load_count<C::kBlocksPerLoad>(u.i0, u.nq, a.hi[u.hq], a.keep[u.hq]);
        if (elect_one()) {
          bars->unit_w[r] = w;
          bars->unit_loads[r] = n_loads;
          mbar_arrive(&bars->unit_ready[r]);   // release: the entry is visible after the wait
        }
        __syncwarp();
        // the Q buffer is free once the last QK of the previous tile has completed
        if (uloc >= 1 && !(ok = warp_wait(&bars->q_empty, (uloc - 1) & 1))) break;
        const int qrow = (u.b * a.Hq + u.hq) * a.S + u.i0 * T;
        if (elect_one()) {
          mbar_arrive_expect_tx(&bars->q_full, 2 * C::kQTile);
          tma_load_2d(sQ8, &maps.q8, &bars->q_full, 0, qrow);
          tma_load_2d(sQ4, &maps.q4, &bars->q_full, 0, qrow);
        }
        __syncwarp();
        LoadPairs<C::kBlocksPerLoad> seq;
        seq.init(u.i0, u.nq, a.hi[u.hq], a.keep[u.hq]);
        const int64_t grp = static_cast<int64_t>(u.b) * a.Hkv + u.kvh;
        int j0, j1, plane, k_load = 0;
        while (seq.next(j0, j1, plane)) {
          const int ks = g % C::kKStages, ss = g % C::kScStages;
          if (g >= static_cast<uint32_t>(C::kKStages) &&
              !(ok = warp_wait(&bars->k_empty[ks], ((g / C::kKStages) - 1) & 1)))
            break;
          if (g >= static_cast<uint32_t>(C::kScStages) &&
              !(ok = warp_wait(&bars->sc_empty[ss], ((g / C::kScStages) - 1) & 1)))
            break;
          ++k_load;
          const CUtensorMap* kmap = plane == 8 ? &maps.k8 : &maps.k4;
          const bool k_in_cache = plane == 8 && a.k8_in_cache;    // else a workspace copy, [group][S] rows
          const float* ks_plane = plane == 8 ? a.k8s : a.k4s;
          // contiguous cache: rows of the load's blocks from one base per load
          const int64_t krow_base = grp * (plane == 8 ? a.cap8 : static_cast<int64_t>(a.S));
          const float* ks_base = ks_plane + grp * a.cap;
          if (elect_one()) {
            const int4 inf = make_int4(j0, j1, plane | (k_load == n_loads ? kLastLoad : 0), 0);
            bars->k_info[ks] = inf;    // released by the arrives below
            bars->sc_info[ss] = inf;
            mbar_arrive_expect_tx(&bars->k_full[ks], C::kKTile);
            mbar_arrive_expect_tx(&bars->sc_full[ss], C::kScTile);
            // 128 keys: one block at T = 128; two blocks of 64 at T = 64 (the second a
            // copy of the first when alone)
            const int jb[2] = {j0, (C::kBlocksPerLoad == 1 || j1 < 0) ? j0 : j1};
#pragma unroll
            for (int h = 0; h < C::kBlocksPerLoad; ++h) {
              if constexpr (PAGED) {   // the block's page (a bad page id reads page 0, reported)
                int64_t crow = a.ci.block_row(u.b, u.kvh, jb[h]);
                crow = crow < 0 ? 0 : crow;
                const int64_t krow = k_in_cache ? crow : grp * a.S + static_cast<int64_t>(jb[h]) * T;
                tma_load_2d(sK(ks) + h * T * kQKRowBytes, kmap, &bars->k_full[ks], 0, static_cast<int>(krow));
                bulk_load(sScale(ss) + h * T, ks_plane + crow, T * 4, &bars->sc_full[ss]);
              } else {
                tma_load_2d(sK(ks) + h * T * kQKRowBytes, kmap, &bars->k_full[ks], 0,
                            static_cast<int>(krow_base + static_cast<int64_t>(jb[h]) * T));
                bulk_load(sScale(ss) + h * T, ks_base + static_cast<int64_t>(jb[h]) * T, T * 4, &bars->sc_full[ss]);
              }
            }
          }
          __syncwarp();
          ++g;
        }
        if (!ok) break;
      }
      // let every copy this CTA issued land before the block exits
      for (uint32_t k = (g > static_cast<uint32_t>(C::kKStages) ? g - C::kKStages : 0); k < g; ++k)
        drain_wait(&bars->k_full[k % C::kKStages], (k / C::kKStages) & 1);
      for (uint32_t k = (g > static_cast<uint32_t>(C::kScStages) ? g - C::kScStages : 0); k < g; ++k)
        drain_wait(&bars->sc_full[k % C::kScStages], (k / C::kScStages) & 1);
      if (uloc >= 1) drain_wait(&bars->q_full, (uloc - 1) & 1);
    } else if (warp == kVProducerWarp) {
      // ---------------------------------------------------------- producer: V
      // Walks the same tiles (from the ring) and loads; a V stage is refilled only
      // when the P.V that read it has completed, which never holds up K or Q.
      uint32_t g = 0, uloc = 0;
      bool ok = true;
      for (;; ++uloc) {
        const int r = uloc % kUnitRing;
        if (!(ok = warp_wait(&bars->unit_ready[r], (uloc / kUnitRing) & 1))) break;
        const int w = __shfl_sync(0xffffffffu, bars->unit_w[r], 0);
        if (w < 0) break;
        const Unit u = unit_of(a, w, C::kQBlocks);
        LoadPairs<C::kBlocksPerLoad> seq;
        seq.init(u.i0, u.nq, a.hi[u.hq], a.keep[u.hq]);
        const int64_t grp = static_cast<int64_t>(u.b) * a.Hkv + u.kvh;
        int j0, j1, plane;
        while (seq.next(j0, j1, plane)) {
          const int vs = g % C::kVStages;
          if (g >= static_cast<uint32_t>(C::kVStages) &&
              !(ok = warp_wait(&bars->v_empty[vs], ((g / C::kVStages) - 1) & 1)))
            break;
          const CUtensorMap* vmap = plane == 8 ? &maps.v8 : &maps.v4;
          if (elect_one()) {
            mbar_arrive_expect_tx(&bars->v_full[vs], C::kVTile);
            if constexpr (C::kBlocksPerLoad == 1) {
              // one block of 128 keys as two V sub-tiles of 64 keys
              const int vrow = static_cast<int>((grp * a.nb + j0) * D);
              tma_load_2d(sV(vs), vmap, &bars->v_full[vs], 0, vrow);
              tma_load_2d(sV(vs) + C::kVSub, vmap, &bars->v_full[vs], 64, vrow);
            } else {
              const int jb[2] = {j0, j1 >= 0 ? j1 : j0};
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_2d(sV(vs) + h * C::kVSub, vmap, &bars->v_full[vs], 0, static_cast<int>((grp * a.nb + jb[h]) * D));
            }
          }
          __syncwarp();
          ++g;
        }
        if (!ok) break;
      }
      for (uint32_t k = (g > static_cast<uint32_t>(C::kVStages) ? g - C::kVStages : 0); k < g; ++k)
        drain_wait(&bars->v_full[k % C::kVStages], (k / C::kVStages) & 1);
    } else if (warp == kMmaWarp) {
      // ---------------------------------------------------------- QK issuer
      // A pair's next S is computed as soon as its current S has been read out, so
      // QK runs up to two loads ahead of P.V; the two streams are issued by two
      // warps and meet only through the barriers.
      uint32_t g = 0, uloc = 0;
      bool ok = true;
      const uint32_t q8a = smem_u32(sQ8), q4a = smem_u32(sQ4);
      for (;; ++uloc) {
        const int r = uloc % kUnitRing;
        if (!(ok = warp_wait(&bars->unit_ready[r], (uloc / kUnitRing) & 1))) break;
        if (__shfl_sync(0xffffffffu, bars->unit_w[r], 0) < 0) break;   // no more tiles
        if (!(ok = warp_wait(&bars->q_full, uloc & 1))) break;
        bool last = false;
        while (!last) {
          const int ks = g % C::kKStages, sl = g % C::kSlots;
          if (!(ok = warp_wait(&bars->k_full[ks], (g / C::kKStages) & 1))) break;
          // broadcast through a shuffle and a vote, so that the compiler sees the
          // loop, its counters and every operand derived from them as warp-uniform
          const int4 inf = bars->k_info[ks];
          const int plane = __shfl_sync(0xffffffffu, inf.z & 0xff, 0);
          last = __all_sync(0xffffffffu, (inf.z & kLastLoad) != 0);
          // the slot's previous S (load g - 2) has been read out by its pair
          if (g >= static_cast<uint32_t>(C::kSlots) &&
              !(ok = warp_wait(&bars->s_free[sl], ((g / C::kSlots) - 1) & 1)))
            break;
          tc_fence_after();
          const uint32_t abase = plane == 8 ? q8a : q4a;
          const uint64_t adesc = sw128_desc(abase), bdesc = sw128_desc(smem_u32(sK(ks)));
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < kQKRowBytes / 32; ++k)   // +32 bytes along K = +2 descriptor units
              if (plane == 8)
                mma_i8_ss(tmem + sl * kKeys, adesc + 2 * k, bdesc + 2 * k, C::kIdescQK, k > 0 ? 1u : 0u);
              else
                mma_f8_ss(tmem + sl * kKeys, adesc + 2 * k, bdesc + 2 * k, C::kIdescQK4, k > 0 ? 1u : 0u);
            mma_commit(&bars->s_full[sl]);
            mma_commit(&bars->k_empty[ks]);
            // the tile's last QK has read the Q buffer: the producer may refill it
            if (last) mma_commit(&bars->q_empty);
          }
          __syncwarp();
          ++g;
        }
        if (!ok) break;
      }
      // wait for every tensor-core op this warp issued before TMEM is released
      if (elect_one()) mma_commit(&bars->fin);
      __syncwarp();
      drain_wait(&bars->fin, 0);
    } else if (warp == kPvWarp) {
      // ---------------------------------------------------------- P.V issuer
      uint32_t g = 0, uloc = 0;
      bool ok = true;
      for (;; ++uloc) {
        const int r = uloc % kUnitRing;
        if (!(ok = warp_wait(&bars->unit_ready[r], (uloc / kUnitRing) & 1))) break;
        if (__shfl_sync(0xffffffffu, bars->unit_w[r], 0) < 0) break;   // no more tiles
        const int n = __shfl_sync(0xffffffffu, bars->unit_loads[r], 0);
        for (int l = 0; l < n; ++l, ++g) {
          const int pr = g % kPairs;   // pair = V stage = P buffer = O accumulator
          if (!(ok = warp_wait(&bars->p_full[pr], (g / kPairs) & 1))) break;
          if (!(ok = warp_wait(&bars->v_full[pr], (g / kPairs) & 1))) break;
          tc_fence_after();
          const uint64_t pdesc = sw128_desc(smem_u32(sP(pr)));
          const uint64_t vdesc = sw128_desc(smem_u32(sV(pr)));
          // the first P.V of a tile into an accumulator overwrites it: the tile's
          // loads l = 0 and l = 1 are the first of their pairs
          const bool first = l < kPairs;
          if (elect_one()) {
#pragma unroll
            for (int s = 0; s < kKeys / 16; ++s) {
              // +((s / 4) * sub-tile + (s % 4) * 32 bytes) in the descriptor's 16-byte units
              const uint64_t adv = static_cast<uint64_t>((s % 4) * 32 >> 4);
              const uint64_t ad = pdesc + adv + static_cast<uint64_t>(((s / 4) * C::kPSub) >> 4);
              const uint64_t bd = vdesc + adv + static_cast<uint64_t>(((s / 4) * C::kVSub) >> 4);
              mma_bf16_ss(tmem + o_col(pr), ad, bd, C::kIdescPV, (first && s == 0) ? 0u : 1u);
            }
            mma_commit(&bars->v_empty[pr]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit(&bars->o_fin);
        __syncwarp();
      }
      if (elect_one()) mma_commit(&bars->fin_pv);
      __syncwarp();
      drain_wait(&bars->fin_pv, 0);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax (warps 0-15)
    constexpr int TH = kKeys / 2;             // keys of this thread per load
    const int pair = warp / 8;                // load parity handled, S slot, O accumulator
    const int half = (warp / 4) % 2;          // which half of the keys
    const int sub = warp % 4;                 // TMEM lane quarter
    const int row = sub * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(sub * 32) << 16);
    const uint32_t my_s = lane_addr + half * TH;                     // + slot * kKeys: S columns of my keys
    const uint32_t my_o = lane_addr + o_col(pair) + half * (D / 2);  // O columns rescaled here
    const uint32_t pair_bar = 1 + pair * 4 + sub;                    // 64 threads: this row's pair
    const uint32_t row_bar = 9 + sub;                                // 128 threads: all four of the row
    // row maxima of loads: [pair][half][row]; epilogue (m, l): [tile parity][pair][half][2][row]
    float* xmax = reinterpret_cast<float*>(smem + C::kOffX);
    float* xepi = xmax + 2 * 2 * 128;
    // Every wait below is shared with the warps that meet this one in a named
    // barrier (the pair's other half per load, the row's four warps per tile): all
    // wait on the same phases and give up only at the time limit (mbar_wait_shared),
    // so a failure makes them leave at the same point and none is left in a barrier.
    auto wait = [&](uint64_t* bar, uint32_t parity) { return mbar_wait_shared(bar, parity, abort, a.err); };
    uint32_t g = 0, uloc = 0;
    bool ok = true;
    for (;; ++uloc) {
      // the CTA's next tile and its load count, published by the producer
      const int r = uloc % kUnitRing;
      if (!(ok = wait(&bars->unit_ready[r], (uloc / kUnitRing) & 1))) break;
      const int w = bars->unit_w[r];
      if (w < 0) break;                                 // no more tiles
      const Unit u = unit_of(a, w, C::kQBlocks);
      const int qb = row / T;
      const int rl = row % T;
      const bool valid = qb < u.nq;
      const int ir = u.i0 + qb;
      const int64_t qrow = (static_cast<int64_t>(u.b) * a.Hq + u.hq) * a.S + static_cast<int64_t>(ir) * T + rl;
      // the row's query scales, taken times log2(e) / sqrt(D) only where a load's plane
      // picks one: nothing before the first load's waits consumes the two reads
      const float q8s = valid ? a.q8s[qrow] : 0.0f;
      const float q4s = valid ? a.q4s[qrow] : 0.0f;
      const int hi = a.hi[u.hq], keep = a.keep[u.hq];
      float m_run = -INFINITY, l_run = 0.0f;     // m_run: shared by both halves of the pair
      // this tile's loads are g0 .. g0 + n - 1 in the CTA's order; the pair takes
      // those of its parity
      const uint32_t g0 = g, g_end = g0 + static_cast<uint32_t>(bars->unit_loads[r]);
      for (g = g0 + ((g0 % kPairs) == static_cast<uint32_t>(pair) ? 0u : 1u); g < g_end; g += kPairs) {
        const int sc = g % C::kScStages, sl = g % C::kSlots;   // sl = pair
        const uint32_t slot_col = static_cast<uint32_t>(sl * kKeys);
        if (!(ok = wait(&bars->sc_full[sc], (g / C::kScStages) & 1))) break;
        if (!(ok = wait(&bars->s_full[sl], (g / C::kSlots) & 1))) break;
        tc_fence_after();
        const int4 inf = bars->sc_info[sc];
        const int plane = inf.z & 0xff;
        // my keys: a half of the load's block at T = 128; at T = 64 the block of my
        // half (j1 < 0: none, the half holds a masked copy)
        const int jh = (C::kBlocksPerLoad == 1 || half == 0) ? inf.x : inf.y;
        const int koff = C::kBlocksPerLoad == 1 ? half * TH : 0;   // my first key inside block jh
        // rows whose tile with block jh has another action (or none) write P = 0;
        // uniform over the warp (its 32 rows are in one query block)
        const int act = (valid && jh >= 0) ? tile_action(ir, jh, hi, keep) : ACT_NONE;
        const bool active = act == plane;
        const float alpha = (plane == 8 ? q8s : q4s) * a.qk_log2;
        const int kmax = (jh == ir) ? rl - koff : TH;   // my keys [0, kmax] are visible
        float* xb = xmax + pair * 256;
        // Both halves exchange their maxima on every load (an inactive half offers
        // -inf) and take the same decision on the running maximum. Before writing
        // its maximum a half waits for the pair's previous P.V (below), which needed
        // the other half's previous P, written after that half read the last
        // exchange: one buffer is enough.
        float sc_o = 1.0f;
        bool rescale_o = false;
        auto exchange = [&](float m_half) {
          xb[half * 128 + row] = m_half;
          named_bar_sync(pair_bar, 64);
          const float mt = fmaxf(m_half, xb[(1 - half) * 128 + row]);
          const float m_tile = mt == -INFINITY ? -INFINITY : mt * alpha;
          const bool raise = m_tile > m_run + kRescaleLog2;
          sc_o = raise ? fast_exp2(m_run - m_tile) : 1.0f;
          rescale_o = raise && m_run != -INFINITY;
          if (raise) {
            l_run *= sc_o;
            m_run = m_tile;
          }
        };
        // The pair's S slot is released as soon as S is in registers, so the QK of
        // the pair's next load runs while this one is being processed; the scales
        // are released after the pass that reads them.
        auto release = [&](uint64_t* bar) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bar);
        };
        // The P.V of this pair's previous load (g - 2) reads this pair's P buffer and
        // writes its O accumulator: it must be complete before either is touched.
        // Its completion is phase (g / 2 - 1) of the pair's V stage barrier, which
        // cannot have run further ahead (the next phase needs this load's P).
        auto wait_prev_pv = [&]() -> bool {
          return g < static_cast<uint32_t>(kPairs) || wait(&bars->v_empty[sl], ((g / kPairs) - 1) & 1);
        };
        // my 128-byte row of the pair's P sub-tile `half` (K-major, 128-byte swizzle)
        uint8_t* prow = sP(pair) + half * C::kPSub + row * 128;
        if (active) {
          uint32_t rr[TH];
#pragma unroll
          for (int c = 0; c < TH / 32; ++c)
            tmem_ld32(my_s + slot_col + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&rr[32 * c]));
          tmem_wait_ld();
          tc_fence_before();
          release(&bars->s_free[sl]);
          const float* sk = sScale(sc) + half * TH;
          uint64_t y[TH / 2];
          const bool masked = kmax < TH - 1;
          float mh;
          if (plane == 8) mh = masked ? scores_and_max<TH, true, false>(rr, y, sk, kmax) : scores_and_max<TH, false, false>(rr, y, sk, kmax);
          else mh = masked ? scores_and_max<TH, true, true>(rr, y, sk, kmax) : scores_and_max<TH, false, true>(rr, y, sk, kmax);
          release(&bars->sc_empty[sc]);
          if (!(ok = wait_prev_pv())) break;
          exchange(mh);
          const uint64_t al2 = pk2(alpha, alpha), nm2 = pk2(-m_run, -m_run);
          uint64_t acc[4] = {0, 0, 0, 0};
          if (masked) probs<TH, true>(y, al2, nm2, kmax, prow, row & 7, acc);
          else probs<TH, false>(y, al2, nm2, kmax, prow, row & 7, acc);
          float s0, s1;
          up2(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), s0, s1);
          l_run += s0 + s1;
        } else {
          if (lane == 0) {
            mbar_arrive(&bars->s_free[sl]);
            mbar_arrive(&bars->sc_empty[sc]);
          }
          if (!(ok = wait_prev_pv())) break;
          exchange(-INFINITY);
#pragma unroll
          for (int c = 0; c < TH / 8; ++c) *reinterpret_cast<uint4*>(prow + (c << 4)) = make_uint4(0u, 0u, 0u, 0u);
        }
        // Rescale this half's O columns when the maximum rose. TMEM loads/stores are
        // warp-collective: the whole warp takes part when any lane must, lanes that
        // need not using the factor 1.
        if (__any_sync(0xffffffffu, rescale_o)) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t o[32];
            tmem_ld32(my_o + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * sc_o);
            tmem_st32(my_o + 32 * c, o);
          }
          tmem_wait_st();
        }
        // P (generic-proxy stores) must be visible to the tensor core's reads, and a
        // rescaled O complete (wait::st above), before the warp's one arrival
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[sl]);
      }
      if (!ok) break;
      g = g_end;
      // Epilogue: every P.V of this tile has completed (o_fin, one phase per tile; the
      // next tile's first P.V needs a P from after this epilogue, so the barrier is at
      // most one phase short).
      if (!(ok = wait(&bars->o_fin, uloc & 1))) break;
      tc_fence_after();
      float* xe = xepi + (uloc & 1) * (2 * 2 * 2 * 128);
      auto slot = [&](int p, int h, int v) { return xe + ((p * 2 + h) * 2 + v) * 128 + row; };
      *slot(pair, half, 0) = m_run;
      *slot(pair, half, 1) = l_run;
      named_bar_sync(row_bar, 128);
      const float m0 = *slot(0, 0, 0), m1 = *slot(1, 0, 0);
      const float l0 = *slot(0, 0, 1) + *slot(0, 1, 1);
      const float l1 = *slot(1, 0, 1) + *slot(1, 1, 1);
      const float m_all = fmaxf(m0, m1);
      // an accumulator that saw no kept key in this tile (l = 0) may hold stale values
      const bool use0 = l0 > 0.0f, use1 = l1 > 0.0f;
      const float w0 = use0 ? fast_exp2(m0 - m_all) : 0.0f;
      const float w1 = use1 ? fast_exp2(m1 - m_all) : 0.0f;
      // The two accumulators hold the tile's loads of even and odd position in either
      // order (which one takes the first load depends on the CTA's running load count,
      // so on the tiles it drew before): both products are rounded before the one
      // commutative add, here and for O, so the bits do not depend on that order
      // (a contracted fma(l0, w0, l1 * w1) would round only one of them).
      const float l_tot = __fmul_rn(l0, w0) + __fmul_rn(l1, w1);
      const float inv_l = valid ? 1.0f / l_tot : 0.0f;
      const float f0 = w0 * inv_l, f1 = w1 * inv_l;
      // this thread writes output columns [quarter * D/4, (quarter+1) * D/4)
      const int quarter = pair * 2 + half;
      constexpr int QC = D / 4;
      uint32_t o0[32], o1[32];
      if constexpr (QC == 32) {
        tmem_ld32(lane_addr + o_col(0) + quarter * QC, o0);
        tmem_ld32(lane_addr + o_col(1) + quarter * QC, o1);
      } else {
        tmem_ld16(lane_addr + o_col(0) + quarter * QC, o0);
        tmem_ld16(lane_addr + o_col(1) + quarter * QC, o1);
      }
      tmem_wait_ld();
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(a.O + qrow * D + quarter * QC);
#pragma unroll
        for (int k = 0; k < QC / 8; ++k) {
          uint32_t wv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i0 = 8 * k + 2 * e;
            const float v0 = (use0 ? __fmul_rn(__uint_as_float(o0[i0]), f0) : 0.0f) +
                             (use1 ? __fmul_rn(__uint_as_float(o1[i0]), f1) : 0.0f);
            const float v1 = (use0 ? __fmul_rn(__uint_as_float(o0[i0 + 1]), f0) : 0.0f) +
                             (use1 ? __fmul_rn(__uint_as_float(o1[i0 + 1]), f1) : 0.0f);
            wv[e] = bf16x2(v0, v1);
          }
          dst[k] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        if (quarter == 0) a.LSE[qrow] = (m_all + log2f(l_tot)) * 0.69314718055994531f;
      }
      // All four threads of the row read both accumulators: none may let the next
      // tile's first P.V (which overwrites them) start before the others have read.
      tc_fence_before();
      named_bar_sync(row_bar, 128);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int T, int D, bool PAGED>
cudaError_t launch_tp(const PrefillArgs& a, const PrefillMaps& maps, int num_sms, cudaStream_t stream) {
  using C = Cfg<T, D>;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<T, D, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = a.n_units < num_sms ? a.n_units : num_sms;
  if (grid <= 0) return cudaSuccess;
  prefill_kernel<T, D, PAGED><<<grid, kThreads, C::kSmem, stream>>>(a, maps);
  return cudaGetLastError();
}

template <int T, int D>
cudaError_t launch_t(const PrefillArgs& a, const PrefillMaps& maps, int num_sms, cudaStream_t stream) {
  return a.ci.bt != nullptr ? launch_tp<T, D, true>(a, maps, num_sms, stream)
                            : launch_tp<T, D, false>(a, maps, num_sms, stream);
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
