// Load plan of a fused-prefill query tile: which key blocks, at which plane, go
// into each 128-key load, and in which order. Shared by the kernel's producers
// and the host-side plan query (tria_prefill_load_plan), so that host tests can
// check the plan the kernel follows against the tile policy.
#pragma once

#include "common.cuh"

namespace tria {

// The (key block, plane) loads of one query tile: first every block that some row
// of the tile reads at 8 bits (block 0, then ascending from the band), then every
// block read at 4 bits, ascending. Grouping by plane lets the pairing below join
// any two blocks of one plane, so a tile has at most one lone block per plane. The
// order of a row's key blocks does not change its softmax (the running maximum
// and sum are merged exactly up to rounding).
//
// Both sets are ranges, so the walk costs a few operations per block (the kernel's
// producer walks it on the critical path). With query blocks i in [i0, i0 + nq) and
// h = max(hi, 1) (the diagonal is 8-bit even when hi = 0):
//  * 8 bits: block 0, then [max(1, i0 - h + 1), i0 + nq - 1] -- for j <= i0 row i0 has
//    d = i0 - j < h, and j = i0 + 1 is the diagonal of the tile's second query block;
//  * 4 bits: when keep > h, [max(1, i0 - keep + 1), i0 + nq - 1 - h] -- the union over
//    the tile's query blocks i of [i - keep + 1, i - h], contiguous because those
//    blocks are consecutive; empty when keep <= h.
struct LoadSeq {
  int j, j_end, plane, lo4, hi4;
  __host__ __device__ void init(int i0, int nq, int hi, int keep) {
    const int h = hi > 1 ? hi : 1;
    const int lo8 = i0 - h + 1 > 1 ? i0 - h + 1 : 1;
    plane = 8;
    j = 0;                               // block 0 first, then [lo8, i0 + nq - 1]
    j_end = i0 + nq - 1;
    lo4 = i0 - keep + 1 > 1 ? i0 - keep + 1 : 1;
    hi4 = keep > h ? i0 + nq - 1 - h : 0;
    next8 = lo8;
  }
  int next8;
  // Blocks of each plane: block 0 and [lo8, j_end] at 8 bits, [lo4, hi4] at 4 bits.
  __host__ __device__ int count8() const { return 1 + (j_end >= next8 ? j_end - next8 + 1 : 0); }
  __host__ __device__ int count4() const { return hi4 >= lo4 ? hi4 - lo4 + 1 : 0; }
  __host__ __device__ bool next(int& jo, int& plane_out) {
    if (plane == 8) {
      if (j <= j_end) {
        jo = j;
        plane_out = 8;
        j = j == 0 ? (next8 > 1 ? next8 : 1) : j + 1;
        return true;
      }
      plane = 4;
      j = lo4;
    }
    if (j <= hi4) {
      jo = j++;
      plane_out = 4;
      return true;
    }
    return false;
  }
};

// The 128-key loads of a tile: with one key block per load (T = 128) the
// (block, plane) pairs of LoadSeq, each as (j, j); with two (T = 64) consecutive
// blocks of one plane merged into (j0, j1), and the last block of a plane's odd
// count alone as (j0, -1).
// Loads of a tile without walking it: per plane, blocks joined two by two at T = 64.
template <int BPL>
__host__ __device__ __forceinline__ int load_count(int i0, int nq, int hi, int keep) {
  LoadSeq q;
  q.init(i0, nq, hi, keep);
  const int n8 = q.count8(), n4 = q.count4();
  return BPL == 1 ? n8 + n4 : (n8 + 1) / 2 + (n4 + 1) / 2;
}

template <int BPL>
struct LoadPairs {
  LoadSeq seq;
  int pj, pplane;
  bool pending;
  __host__ __device__ void init(int i0, int nq, int hi, int keep) {
    seq.init(i0, nq, hi, keep);
    pending = false;
  }
  __host__ __device__ bool next(int& j0, int& j1, int& plane) {
    if constexpr (BPL == 1) {
      if (!seq.next(j0, plane)) return false;
      j1 = j0;
      return true;
    } else {
      int j, pl;
      while (seq.next(j, pl)) {
        if (!pending) {
          pj = j; pplane = pl; pending = true;
          continue;
        }
        if (pl == pplane) {            // merge with the pending block
          j0 = pj; j1 = j; plane = pl;
          pending = false;
          return true;
        }
        j0 = pj; j1 = -1; plane = pplane;   // emit the pending block alone
        pj = j; pplane = pl;
        return true;
      }
      if (pending) {
        j0 = pj; j1 = -1; plane = pplane;
        pending = false;
        return true;
      }
      return false;
    }
  }
};

}  // namespace tria
