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
struct LoadSeq {
  int i0, nq, hi, keep, j, jmax, jband, j8, plane;
  __host__ __device__ void init(int i0_, int nq_, int hi_, int keep_) {
    i0 = i0_; nq = nq_; hi = hi_; keep = keep_;
    jmax = i0 + nq - 1; j = 0; plane = 8;
    jband = first_band_block(i0, keep);
    // 8-bit blocks after block 0: d < hi or the diagonal, so none before i0 - hi + 1
    const int lo = i0 - hi + 1 < i0 ? i0 - hi + 1 : i0;
    j8 = lo > jband ? lo : jband;
  }
  __host__ __device__ bool next(int& jo, int& plane_out) {
    while (true) {
      if (j > jmax) {
        if (plane == 4) return false;
        plane = 4;                       // second pass: the 4-bit blocks of the band
        j = jband;
        continue;
      }
      const int want = plane == 8 ? ACT_INT8 : ACT_INT4;
      bool need = false;
      for (int q = 0; q < nq; ++q) need |= tile_action(i0 + q, j, hi, keep) == want;
      const int jj = j;
      j = (plane == 8 && j == 0) ? j8 : j + 1;
      if (need) { jo = jj; plane_out = plane; return true; }
    }
  }
};


// The 128-key loads of a tile: with one key block per load (T = 128) the
// (block, plane) pairs of LoadSeq, each as (j, j); with two (T = 64) consecutive
// blocks of one plane merged into (j0, j1), and the last block of a plane's odd
// count alone as (j0, -1).
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
