// compact.cuh -- the expert-offset scan of the compaction, as a block-level
// device routine run by the last routing CTA to finish.
//
// From the per-(32-token chunk, expert) kept-slot histogram it forms the
// per-expert counts, the exclusive offsets over experts (kept slots ordered
// by expert, then token), the per-(chunk, expert) base positions and the list
// of expert GEMM tiles (expert, first slot, rows <= tile_n) in expert order.
#pragma once

#include "ace_common.cuh"

namespace ace {

// Exclusive scan over the CTA in thread order; returns this thread's prefix,
// *total receives the sum.  All threads must call it.
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    s_warp[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int before = warp > 0 ? s_warp[warp - 1] : 0;
  *total = s_warp[nw - 1];
  __syncthreads();
  return before + incl - v;
}

struct ScanOut {
  int32_t* base;     // [nchunk][E]
  int32_t* counts;   // [E]
  int32_t* offsets;  // [E + 1]
  int32_t* n_kept;   // [1]
  int4* tiles;       // [max_tiles]
  int32_t* n_tiles;  // [1]
  int max_tiles, tile_n;
};

// Whole-CTA routine (every thread calls it; blockDim.x a multiple of 32 and
// at least E).  hist is read with L2-coherent loads: other CTAs wrote it.
__device__ __forceinline__ void scan_experts(const int32_t* hist, int nchunk, int E,
                                             const ScanOut& o) {
  __shared__ int s_warp[32];
  int tpe = 1;  // threads per expert (a power of two that divides 32)
  while (tpe < 32 && tpe * 2 * E <= (int)blockDim.x) tpe *= 2;
  const int e = threadIdx.x / tpe, g = threadIdx.x % tpe;
  const bool active = e < E;
  const int per = (nchunk + tpe - 1) / tpe;
  const int cb = min(nchunk, g * per), ce = min(nchunk, cb + per);
  int local = 0;
  if (active)
    for (int c = cb; c < ce; ++c) local += __ldcg(hist + (size_t)c * E + e);
  // prefix inside the expert's group of tpe consecutive lanes
  int incl = local;
  for (int sh = 1; sh < tpe; sh <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, sh, tpe);
    if (g >= sh) incl += n;
  }
  const int excl_in_group = incl - local;
  const int cnt = __shfl_sync(0xffffffffu, incl, tpe - 1, tpe);
  int total, total_tiles;
  const int off = block_excl_scan((active && g == 0) ? cnt : 0, s_warp, &total);
  const int ntile = (active && g == 0) ? (cnt + o.tile_n - 1) / o.tile_n : 0;
  const int toff = block_excl_scan(ntile, s_warp, &total_tiles);
  const int off_e = __shfl_sync(0xffffffffu, off, 0, tpe);
  if (active) {
    int run = off_e + excl_in_group;
    for (int c = cb; c < ce; ++c) {
      o.base[(size_t)c * E + e] = run;
      run += __ldcg(hist + (size_t)c * E + e);
    }
    if (g == 0) {
      o.counts[e] = cnt;
      o.offsets[e] = off;
      for (int q = 0; q < ntile; ++q) {
        if (toff + q < o.max_tiles)
          o.tiles[toff + q] =
              make_int4(e, off + q * o.tile_n, min(o.tile_n, cnt - q * o.tile_n), 0);
      }
    }
  }
  if (threadIdx.x == 0) {
    o.offsets[E] = total;
    *o.n_kept = total;
    *o.n_tiles = min(total_tiles, o.max_tiles);
  }
}

}  // namespace ace
