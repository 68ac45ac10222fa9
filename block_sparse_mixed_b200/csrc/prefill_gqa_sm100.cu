// Fused block-sparse mixed-precision causal prefill for sm_100a, GQA-shared:
// one CTA serves two query heads of one KV group whose boundaries coincide, so
// every kept K/V block it brings into shared memory serves both heads.
//
// What it computes is exactly what the per-head kernel (prefill_sm100.cu)
// computes: for every query row, softmax attention over the key blocks its query
// block keeps, each block at its own precision (rit.work TriAttention page,
// section "Какие связи можно не считать, а какие нельзя удалять", and section "Как
// калибровка распределяет вычисления между головами", last paragraph), with the
// query heads of a KV group reading the same K/V (llmis.ru chapter 3.5, section 4,
// "Grouped-Query Attention"). The heads of the pair share (hi, keep), so they keep
// the same tiles and one load sequence serves both.
//
// How it differs from the per-head kernel. A unit is (batch, KV group, head pair,
// 128-row query tile). The two softmax pairs of warpgroups belong to the two heads
// (pair p = head 2k + p) and each takes every load of the tile, with its own S slot,
// P buffer and O accumulator; the K and V stages and the K scales are shared, and a
// stage is released when both heads are done with it. The QK issuer issues the
// load's QK for both heads (two tcgen05.mma chains reading the same K tile), the
// P.V issuer the two P.V chains reading the same V tile. The Q buffer holds one
// plane of both heads at a time (the tile's 8-bit loads come first, then its 4-bit
// loads): the producer loads the 4-bit Q codes once the last 8-bit QK of the tile
// has completed. Each head's softmax state covers all the tile's loads, so the
// epilogue normalises one accumulator per head.
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

constexpr int kRows = 128;
constexpr int kThreads = 640;           // 16 softmax warps, producer, QK issuer, V producer, P.V issuer
constexpr int kSoftmaxWarps = 16;
constexpr int kPairWarps = 8;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kVProducerWarp = 18;
constexpr int kPvWarp = 19;
constexpr int kRegsSoftmax = 104;       // 4 x 128 x 104 + 128 x 64 = 61,440 = 640 x 96 at launch
constexpr int kRegsOther = 64;
constexpr int kHeads = 2;               // query heads per CTA = softmax pairs
constexpr int kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kKeys = 128;
constexpr int kUnitRing = 16;
constexpr int kLastLoad = 1 << 8;       // info.z flags next to the plane
constexpr int kLastOfPlane = 1 << 9;    // the tile's last load of this plane: its QK frees the Q buffer

// Output rows of one warp, coalesced. Lane l holds NC 16-byte chunks (chunk[c], 8
// bf16 values each) of row l of the warp's 32 rows, for the same columns in every
// row; row l goes to dst0 + l * row_stride (bytes), lanes whose row is not valid hold
// nothing to write. Written straight from the lanes, every store instruction would
// touch 32 rows; instead the warp passes the chunks through `scratch` (32 * NC * 16
// bytes of shared memory that only this warp uses) so that each store instruction
// writes 32 / NC whole row segments of NC * 16 bytes. Chunk c of row l is kept at
// position c ^ ((l / (8 / NC)) % NC) of its row, so that neither the writes of one
// chunk by all lanes nor the reads of 32 / NC consecutive rows meet a bank twice
// within a 128-byte wavefront.
template <int NC>
__device__ __forceinline__ void store_rows(const uint4 (&chunk)[NC], bool valid, uint8_t* scratch, uint8_t* dst0,
                                           int64_t row_stride, int lane) {
  static_assert(NC == 4 || NC == 8, "row segment of 64 or 128 bytes");
  constexpr int kRowsPerStore = 32 / NC;
  auto pos = [](int l, int c) { return l * NC * 16 + ((c ^ ((l / (8 / NC)) % NC)) << 4); };
#pragma unroll
  for (int c = 0; c < NC; ++c) *reinterpret_cast<uint4*>(scratch + pos(lane, c)) = chunk[c];
  const unsigned vmask = __ballot_sync(0xffffffffu, valid);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int l = i * kRowsPerStore + lane / NC, c = lane % NC;
    const uint4 v = *reinterpret_cast<const uint4*>(scratch + pos(l, c));
    if ((vmask >> l) & 1u) *reinterpret_cast<uint4*>(dst0 + l * row_stride + c * 16) = v;
  }
  __syncwarp();   // the scratch is free again for this warp's next writes
}

// S slot of head p: columns 128 p; O accumulator of head p: 256 + 128 p.
__host__ __device__ constexpr uint32_t s_col(int p) { return 128u * static_cast<uint32_t>(p); }
__host__ __device__ constexpr uint32_t o_col(int p) { return 256u + 128u * static_cast<uint32_t>(p); }

template <int T, int D>
struct Cfg {
  static constexpr int kQBlocks = kRows / T;
  static constexpr int kBlocksPerLoad = kKeys / T;
  static constexpr int kQHead = kRows * kQKRowBytes;         // one plane of one head's Q codes
  static constexpr int kKTile = kKeys * kQKRowBytes;
  static constexpr int kVSub = D * 128;                      // V^T sub-tile: D rows x 64 keys
  static constexpr int kVTile = D * kKeys * 2;
  static constexpr int kPSub = kRows * 128;
  static constexpr int kPTile = kRows * kKeys * 2;
  static constexpr int kScTile = kKeys * 4;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kScStages = 4;
  static constexpr int kOffQ = 0;                            // [head][128 rows][128 B], one plane
  static constexpr int kOffK = kHeads * kQHead;
  static constexpr int kOffV = kOffK + kKStages * kKTile;
  static constexpr int kOffP = kOffV + kVStages * kVTile;    // P buffer of head p at kOffP + p * kPTile
  static constexpr int kOffSc = kOffP + kHeads * kPTile;
  static constexpr int kOffBar = kOffSc + kScStages * kScTile;
  static constexpr int kOffX = kOffBar + 1024;
  static constexpr int kXBytes = kHeads * 2 * 128 * 4 + kHeads * 2 * 128 * 4;   // row maxima, epilogue sums
  static constexpr int kSmemNeed = kOffX + kXBytes + 1024;
  static constexpr int kSmem = kSmemNeed > 120 * 1024 ? kSmemNeed : 120 * 1024;
  static_assert(kSmemNeed <= 227 * 1024, "shared memory");
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0 && kKTile % 1024 == 0 &&
                    kVSub % 1024 == 0 && kPSub % 1024 == 0 && kQHead % 1024 == 0,
                "swizzled operand tiles start on 1024-byte boundaries");
  static constexpr uint32_t kIdescQK = idesc_i8(kRows, kKeys);
  static constexpr uint32_t kIdescQK4 = idesc_e4m3(kRows, kKeys);
  static constexpr uint32_t kIdescPV = idesc_bf16(kRows, D);
};

struct Bars {
  uint64_t q_full, q_empty, fin, fin_pv;
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[2], v_empty[2];
  uint64_t sc_full[4], sc_empty[4];
  uint64_t s_full[kHeads], s_free[kHeads];
  uint64_t p_full[kHeads];
  uint64_t pv_done[kHeads];     // head p's P.V of its n-th load: phase n
  uint32_t tmem_base;
  int abort;
  int4 k_info[3], sc_info[4];   // (j0, j1, plane | flags, 0)
  int unit_w[kUnitRing], unit_loads[kUnitRing];
  uint64_t unit_ready[kUnitRing];
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

struct Unit {
  int b, hq0, kvh, i0, nq;
};

// Units: (b, kv head, head pair, query tile), the last query tiles first.
__device__ __forceinline__ Unit unit_of(const PrefillArgs& a, int w, int nqb) {
  Unit u;
  const int pairs = a.G / kHeads;
  const int per_tile = a.B * a.Hkv * pairs;
  const int qt = a.n_qtiles - 1 - w / per_tile;
  const int r = w % per_tile;
  u.b = r / (a.Hkv * pairs);
  u.kvh = (r / pairs) % a.Hkv;
  u.hq0 = u.kvh * a.G + kHeads * (r % pairs);
  u.i0 = qt * nqb;
  u.nq = min(nqb, a.nb - u.i0);
  return u;
}

// PAGED: the cache is paged (block table); the contiguous instantiation keeps the
// producer's per-block arithmetic minimal, which measured worth 7% at T = 64.
template <int T, int D, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_gqa_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  using C = Cfg<T, D>;
  extern __shared__ uint8_t smem_raw[];
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
      mbar_init(&bars->sc_empty[s], kHeads * kPairWarps);
    }
    for (int r = 0; r < kUnitRing; ++r) mbar_init(&bars->unit_ready[r], 1);
    for (int p = 0; p < kHeads; ++p) {
      mbar_init(&bars->s_full[p], 1);
      mbar_init(&bars->s_free[p], kPairWarps);
      mbar_init(&bars->p_full[p], kPairWarps);
      mbar_init(&bars->pv_done[p], 1);
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

  auto sQ = [&](int h) { return smem + C::kOffQ + h * C::kQHead; };
  auto sK = [&](int s) { return smem + C::kOffK + s * C::kKTile; };
  auto sV = [&](int s) { return smem + C::kOffV + s * C::kVTile; };
  auto sP = [&](int p) { return smem + C::kOffP + p * C::kPTile; };
  auto sScale = [&](int s) { return reinterpret_cast<float*>(smem + C::kOffSc + s * C::kScTile); };

  if (warp >= kSoftmaxWarps) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, a.err));
    };
    if (warp == kProducerWarp) {
      // ---------------------------------------------------------- producer: Q, K, scales
      uint32_t g = 0, uloc = 0, qn = 0;    // loads, tiles, Q loads of this CTA
      bool ok = true;
      // Q codes of both heads, one plane, into the single Q buffer (once its previous
      // contents have been read by the QKs that used them)
      auto load_q = [&](const Unit& u, int plane) -> bool {
        if (qn >= 1 && !warp_wait(&bars->q_empty, (qn - 1) & 1)) return false;
        if (elect_one()) {
          mbar_arrive_expect_tx(&bars->q_full, kHeads * C::kQHead);
#pragma unroll
          for (int h = 0; h < kHeads; ++h) {
            const int qrow = (u.b * a.Hq + u.hq0 + h) * a.S + u.i0 * T;
            tma_load_2d(sQ(h), plane == 8 ? &maps.q8 : &maps.q4, &bars->q_full, 0, qrow);
          }
        }
        __syncwarp();
        ++qn;
        return true;
      };
      for (;; ++uloc) {
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
        const int hi = a.hi[u.hq0], keep = a.keep[u.hq0];
        const int n_loads = load_count<C::kBlocksPerLoad>(u.i0, u.nq, hi, keep);
        if (elect_one()) {
          bars->unit_w[r] = w;
          bars->unit_loads[r] = n_loads;
          mbar_arrive(&bars->unit_ready[r]);
        }
        __syncwarp();
        LoadPairs<C::kBlocksPerLoad> seq;
        seq.init(u.i0, u.nq, hi, keep);
        const int64_t grp = static_cast<int64_t>(u.b) * a.Hkv + u.kvh;
        int j0, j1, plane, k_load = 0;
        // one load ahead, so that a load knows whether it is the last of its plane
        int n0, n1, nplane;
        bool have = seq.next(j0, j1, plane);
        int cur_q_plane = 0;
        while (have) {
          const bool more = seq.next(n0, n1, nplane);
          const bool last_of_plane = !more || nplane != plane;
          if (plane != cur_q_plane) {
            if (!(ok = load_q(u, plane))) break;
            cur_q_plane = plane;
          }
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
            const int4 inf = make_int4(j0, j1, plane | (k_load == n_loads ? kLastLoad : 0) |
                                                   (last_of_plane ? kLastOfPlane : 0), 0);
            bars->k_info[ks] = inf;
            bars->sc_info[ss] = inf;
            mbar_arrive_expect_tx(&bars->k_full[ks], C::kKTile);
            mbar_arrive_expect_tx(&bars->sc_full[ss], C::kScTile);
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
          have = more;
          j0 = n0; j1 = n1; plane = nplane;
        }
        if (!ok) break;
      }
      for (uint32_t k = (g > static_cast<uint32_t>(C::kKStages) ? g - C::kKStages : 0); k < g; ++k)
        drain_wait(&bars->k_full[k % C::kKStages], (k / C::kKStages) & 1);
      for (uint32_t k = (g > static_cast<uint32_t>(C::kScStages) ? g - C::kScStages : 0); k < g; ++k)
        drain_wait(&bars->sc_full[k % C::kScStages], (k / C::kScStages) & 1);
      if (qn >= 1) drain_wait(&bars->q_full, (qn - 1) & 1);
    } else if (warp == kVProducerWarp) {
      // ---------------------------------------------------------- producer: V
      uint32_t g = 0, uloc = 0;
      bool ok = true;
      for (;; ++uloc) {
        const int r = uloc % kUnitRing;
        if (!(ok = warp_wait(&bars->unit_ready[r], (uloc / kUnitRing) & 1))) break;
        const int w = __shfl_sync(0xffffffffu, bars->unit_w[r], 0);
        if (w < 0) break;
        const Unit u = unit_of(a, w, C::kQBlocks);
        LoadPairs<C::kBlocksPerLoad> seq;
        seq.init(u.i0, u.nq, a.hi[u.hq0], a.keep[u.hq0]);
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
              const int vrow = static_cast<int>((grp * a.nb + j0) * D);
              tma_load_2d(sV(vs), vmap, &bars->v_full[vs], 0, vrow);
              tma_load_2d(sV(vs) + C::kVSub, vmap, &bars->v_full[vs], 64, vrow);
            } else {
              const int jb[2] = {j0, j1 >= 0 ? j1 : j0};
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_2d(sV(vs) + h * C::kVSub, vmap, &bars->v_full[vs], 0,
                            static_cast<int>((grp * a.nb + jb[h]) * D));
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
      // ---------------------------------------------------------- QK issuer (both heads per load)
      uint32_t g = 0, uloc = 0, qn = 0;
      bool ok = true, q_ready = false;
      const uint32_t qa[2] = {smem_u32(sQ(0)), smem_u32(sQ(1))};
      for (;; ++uloc) {
        const int r = uloc % kUnitRing;
        if (!(ok = warp_wait(&bars->unit_ready[r], (uloc / kUnitRing) & 1))) break;
        if (__shfl_sync(0xffffffffu, bars->unit_w[r], 0) < 0) break;
        bool last = false;
        while (!last) {
          const int ks = g % C::kKStages;
          if (!(ok = warp_wait(&bars->k_full[ks], (g / C::kKStages) & 1))) break;
          const int4 inf = bars->k_info[ks];
          const int plane = __shfl_sync(0xffffffffu, inf.z & 0xff, 0);
          last = __all_sync(0xffffffffu, (inf.z & kLastLoad) != 0);
          const bool last_of_plane = __all_sync(0xffffffffu, (inf.z & kLastOfPlane) != 0);
          if (!q_ready) {   // the Q codes of this plane (loaded after the previous plane's last QK)
            if (!(ok = warp_wait(&bars->q_full, qn & 1))) break;
            ++qn;
            q_ready = true;
          }
          const uint64_t bdesc = sw128_desc(smem_u32(sK(ks)));
#pragma unroll
          for (int p = 0; p < kHeads; ++p) {
            // head p's slot: its previous S has been read out by its pair
            if (g >= 1 && !(ok = warp_wait(&bars->s_free[p], (g - 1) & 1))) break;
            tc_fence_after();
            const uint64_t adesc = sw128_desc(qa[p]);
            if (elect_one()) {
#pragma unroll
              for (int k = 0; k < kQKRowBytes / 32; ++k)
                if (plane == 8)
                  mma_i8_ss(tmem + s_col(p), adesc + 2 * k, bdesc + 2 * k, C::kIdescQK, k > 0 ? 1u : 0u);
                else
                  mma_f8_ss(tmem + s_col(p), adesc + 2 * k, bdesc + 2 * k, C::kIdescQK4, k > 0 ? 1u : 0u);
              mma_commit(&bars->s_full[p]);
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) {
            mma_commit(&bars->k_empty[ks]);
            if (last_of_plane) mma_commit(&bars->q_empty);   // the producer may load the next plane's Q
          }
          __syncwarp();
          if (last_of_plane) q_ready = false;
          ++g;
        }
        if (!ok) break;
      }
      if (elect_one()) mma_commit(&bars->fin);
      __syncwarp();
      drain_wait(&bars->fin, 0);
    } else if (warp == kPvWarp) {
      // ---------------------------------------------------------- P.V issuer (both heads per load)
      uint32_t g = 0, uloc = 0;
      bool ok = true;
      for (;; ++uloc) {
        const int r = uloc % kUnitRing;
        if (!(ok = warp_wait(&bars->unit_ready[r], (uloc / kUnitRing) & 1))) break;
        if (__shfl_sync(0xffffffffu, bars->unit_w[r], 0) < 0) break;
        const int n = __shfl_sync(0xffffffffu, bars->unit_loads[r], 0);
        for (int l = 0; l < n; ++l, ++g) {
          const int vs = g % C::kVStages;
          if (!(ok = warp_wait(&bars->v_full[vs], (g / C::kVStages) & 1))) break;
          const uint64_t vdesc = sw128_desc(smem_u32(sV(vs)));
#pragma unroll
          for (int p = 0; p < kHeads; ++p) {
            if (!(ok = warp_wait(&bars->p_full[p], g & 1))) break;
            tc_fence_after();
            const uint64_t pdesc = sw128_desc(smem_u32(sP(p)));
            if (elect_one()) {
#pragma unroll
              for (int s = 0; s < kKeys / 16; ++s) {
                const uint64_t adv = static_cast<uint64_t>((s % 4) * 32 >> 4);
                const uint64_t ad = pdesc + adv + static_cast<uint64_t>(((s / 4) * C::kPSub) >> 4);
                const uint64_t bd = vdesc + adv + static_cast<uint64_t>(((s / 4) * C::kVSub) >> 4);
                mma_bf16_ss(tmem + o_col(p), ad, bd, C::kIdescPV, (l == 0 && s == 0) ? 0u : 1u);
              }
              mma_commit(&bars->pv_done[p]);   // frees head p's P buffer; O_p is up to date
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) mma_commit(&bars->v_empty[vs]);
          __syncwarp();
        }
        if (!ok) break;
      }
      if (elect_one()) mma_commit(&bars->fin_pv);
      __syncwarp();
      drain_wait(&bars->fin_pv, 0);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------ softmax (warps 0-15)
    constexpr int TH = kKeys / 2;
    const int pair = warp / 8;                // = head of the unit's pair
    const int half = (warp / 4) % 2;
    const int sub = warp % 4;
    const int row = sub * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(sub * 32) << 16);
    const uint32_t my_s = lane_addr + s_col(pair) + half * TH;
    const uint32_t my_o = lane_addr + o_col(pair) + half * (D / 2);
    const uint32_t pair_bar = 1 + pair * 4 + sub;       // 64 threads: this row's two halves
    float* xmax = reinterpret_cast<float*>(smem + C::kOffX) + pair * 256;   // [half][row]
    float* xsum = reinterpret_cast<float*>(smem + C::kOffX) + kHeads * 256 + pair * 256;
    auto wait = [&](uint64_t* bar, uint32_t parity) { return mbar_wait_shared(bar, parity, abort, a.err); };
    uint32_t g = 0, uloc = 0;
    bool ok = true;
    for (;; ++uloc) {
      const int r = uloc % kUnitRing;
      if (!(ok = wait(&bars->unit_ready[r], (uloc / kUnitRing) & 1))) break;
      const int w = bars->unit_w[r];
      if (w < 0) break;
      const Unit u = unit_of(a, w, C::kQBlocks);
      const int hq = u.hq0 + pair;
      const int qb = row / T;
      const int rl = row % T;
      const bool valid = qb < u.nq;
      const int ir = u.i0 + qb;
      const int64_t qrow = (static_cast<int64_t>(u.b) * a.Hq + hq) * a.S + static_cast<int64_t>(ir) * T + rl;
      const float a8 = valid ? a.q8s[qrow] * a.qk_log2 : 0.0f;
      const float a4 = valid ? a.q4s[qrow] * a.qk_log2 : 0.0f;
      const int hi = a.hi[hq], keep = a.keep[hq];
      float m_run = -INFINITY, l_run = 0.0f;
      const uint32_t g_end = g + static_cast<uint32_t>(bars->unit_loads[r]);
      for (; g < g_end; ++g) {
        const int sc = g % C::kScStages;
        if (!(ok = wait(&bars->sc_full[sc], (g / C::kScStages) & 1))) break;
        if (!(ok = wait(&bars->s_full[pair], g & 1))) break;
        tc_fence_after();
        const int4 inf = bars->sc_info[sc];
        const int plane = inf.z & 0xff;
        const int jh = (C::kBlocksPerLoad == 1 || half == 0) ? inf.x : inf.y;
        const int koff = C::kBlocksPerLoad == 1 ? half * TH : 0;
        const int act = (valid && jh >= 0) ? tile_action(ir, jh, hi, keep) : ACT_NONE;
        const bool active = act == plane;
        const float alpha = plane == 8 ? a8 : a4;
        const int kmax = (jh == ir) ? rl - koff : TH;
        float sc_o = 1.0f;
        bool rescale_o = false;
        auto exchange = [&](float m_half) {
          xmax[half * 128 + row] = m_half;
          named_bar_sync(pair_bar, 64);
          const float mt = fmaxf(m_half, xmax[(1 - half) * 128 + row]);
          const float m_tile = mt == -INFINITY ? -INFINITY : mt * alpha;
          const bool raise = m_tile > m_run + kRescaleLog2;
          sc_o = raise ? fast_exp2(m_run - m_tile) : 1.0f;
          rescale_o = raise && m_run != -INFINITY;
          if (raise) {
            l_run *= sc_o;
            m_run = m_tile;
          }
        };
        auto release = [&](uint64_t* bar) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bar);
        };
        // this head's previous P.V (load g - 1) reads its P buffer and writes O: done
        // before either is touched; it is phase g - 1 of pv_done[pair], which cannot run
        // further ahead (the next phase needs this load's P)
        auto wait_prev_pv = [&]() -> bool { return g < 1 || wait(&bars->pv_done[pair], (g - 1) & 1); };
        uint8_t* prow = sP(pair) + half * C::kPSub + row * 128;
        if (active) {
          uint32_t rr[TH];
#pragma unroll
          for (int c = 0; c < TH / 32; ++c)
            tmem_ld32(my_s + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&rr[32 * c]));
          tmem_wait_ld();
          tc_fence_before();
          release(&bars->s_free[pair]);
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
            mbar_arrive(&bars->s_free[pair]);
            mbar_arrive(&bars->sc_empty[sc]);
          }
          if (!(ok = wait_prev_pv())) break;
          exchange(-INFINITY);
#pragma unroll
          for (int c = 0; c < TH / 8; ++c) *reinterpret_cast<uint4*>(prow + (c << 4)) = make_uint4(0u, 0u, 0u, 0u);
        }
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
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[pair]);
      }
      if (!ok) break;
      // Epilogue: the tile's last P.V of this head (phase g_end - 1) has completed.
      if (!(ok = wait(&bars->pv_done[pair], (g_end - 1) & 1))) break;
      tc_fence_after();
      xsum[half * 128 + row] = l_run;
      named_bar_sync(pair_bar, 64);
      const float l_tot = xsum[row] + xsum[128 + row];
      const float inv_l = (valid && l_tot > 0.0f) ? 1.0f / l_tot : 0.0f;
      // this thread writes output columns [half * D/2, (half + 1) * D/2)
      constexpr int HC = D / 2;
      uint32_t o[HC];
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) tmem_ld32(my_o + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&o[32 * c]));
      tmem_wait_ld();
      {
        uint4 ch[HC / 8];
#pragma unroll
        for (int k = 0; k < HC / 8; ++k) {
          uint32_t wv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            wv[e] = bf16x2(__uint_as_float(o[8 * k + 2 * e]) * inv_l, __uint_as_float(o[8 * k + 2 * e + 1]) * inv_l);
          ch[k] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        // through the warp's own 32 rows of the head's P sub-tile: the head's last P.V
        // has completed, so the tensor core reads nothing there any more
        store_rows<HC / 8>(ch, valid, sP(pair) + half * C::kPSub + sub * 32 * 128,
                           reinterpret_cast<uint8_t*>(a.O + (qrow - lane) * D + half * HC), D * 2, lane);
        if (valid && half == 0) a.LSE[qrow] = (m_run + log2f(l_tot)) * 0.69314718055994531f;
      }
      // both halves have read the sums before the next tile's exchange overwrites them;
      // O_p is read before this pair's next P (and so the next P.V) is written
      tc_fence_before();
      named_bar_sync(pair_bar, 64);
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
  cudaError_t e =
      cudaFuncSetAttribute(prefill_gqa_kernel<T, D, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = a.n_units < num_sms ? a.n_units : num_sms;
  if (grid <= 0) return cudaSuccess;
  prefill_gqa_kernel<T, D, PAGED><<<grid, kThreads, C::kSmem, stream>>>(a, maps);
  return cudaGetLastError();
}

template <int T, int D>
cudaError_t launch_t(const PrefillArgs& a, const PrefillMaps& maps, int num_sms, cudaStream_t stream) {
  return a.ci.bt != nullptr ? launch_tp<T, D, true>(a, maps, num_sms, stream)
                            : launch_tp<T, D, false>(a, maps, num_sms, stream);
}

}  // namespace

cudaError_t launch_prefill_gqa(const PrefillArgs& a, const PrefillMaps& maps, int D, int T, int num_sms,
                               cudaStream_t stream) {
  if (T == 128 && D == 128) return launch_t<128, 128>(a, maps, num_sms, stream);
  if (T == 64 && D == 128) return launch_t<64, 128>(a, maps, num_sms, stream);
  if (T == 128 && D == 64) return launch_t<128, 64>(a, maps, num_sms, stream);
  return launch_t<64, 64>(a, maps, num_sms, stream);
}

}  // namespace tria
