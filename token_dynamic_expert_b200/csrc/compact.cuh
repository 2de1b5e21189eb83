// compact.cuh -- the expert-offset scan of the compaction, as a block-level
// device routine run by the last routing CTA to finish.
//
// From the per-(expert, 32-token chunk) kept-slot histogram it forms the
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
  uint32_t* tile_done;  // [max_tiles] or NULL: per-tile counters, zeroed here
  int max_tiles, tile_n;
};

// Whole-CTA routine (every thread calls it; blockDim.x a multiple of 32, at
// least E, at most 1024).  hist and base are chunk-major, [nchunk][E]; hist
// is read with L2-coherent loads (other CTAs wrote it).
//
// The warps split the [nchunk][E] table into 32-expert columns (a lane per
// expert) times chunk ranges, so that every load and store of a warp covers
// 32 consecutive experts of one chunk and no step needs a shuffle:
//   pass 1: each warp sums its range per expert (s_part[range][e]);
//   then per expert: the count (sum over ranges), the exclusive offsets over
//   experts (a CTA scan) and the expert's GEMM tiles;
//   pass 2: each warp walks its range again, writing base[c][e] = offset of
//   e + kept slots of e in chunks before c.
// An expert of n kept slots gets ceil(n / tile_n) tiles of near-equal size
// (they differ by at most one slot), in slot order.
__device__ __forceinline__ void scan_experts(const int32_t* hist, int nchunk, int E,
                                             const ScanOut& o) {
  __shared__ int s_warp[32];
  __shared__ int s_cnt[1024], s_part[1024];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int ncol = (E + 31) / 32;              // 32-expert columns
  const int nrange = nw / ncol;                // chunk ranges (nw >= ncol since E <= 1024)
  const int per = (nchunk + nrange - 1) / nrange;
  const int col = warp % ncol, rg = warp / ncol;
  const int e = col * 32 + lane;
  const bool active = rg < nrange && e < E;
  const int c0 = rg * per, c1 = min(nchunk, c0 + per);
  // pass 1: per-range sums
  if (active) {
    int acc = 0;
#pragma unroll 8
    for (int c = c0; c < c1; ++c) acc += __ldcg(hist + (size_t)c * E + e);
    s_part[rg * E + e] = acc;
  }
  __syncthreads();
  // counts, offsets over experts, the tile list
  const int t = threadIdx.x;
  int cnt = 0;
  if (t < E)
    for (int r = 0; r < nrange; ++r) cnt += s_part[r * E + t];
  int total, total_tiles;
  const int off = block_excl_scan(cnt, s_warp, &total);
  const int ntile = t < E ? (cnt + o.tile_n - 1) / o.tile_n : 0;
  const int toff = block_excl_scan(ntile, s_warp, &total_tiles);
  if (t < E) {
    s_cnt[t] = off;  // from here on: the expert's offset
    o.counts[t] = cnt;
    o.offsets[t] = off;
    if (ntile > 0) {
      const int each = cnt / ntile, rem = cnt - each * ntile;
      for (int q = 0; q < ntile; ++q)
        if (toff + q < o.max_tiles)
          o.tiles[toff + q] = make_int4(t, off + q * each + min(q, rem), each + (q < rem ? 1 : 0), 0);
    }
  }
  if (t == 0) {
    o.offsets[E] = total;
    *o.n_kept = total;
    *o.n_tiles = min(total_tiles, o.max_tiles);
  }
  if (o.tile_done)
    for (int i = t; i < o.max_tiles; i += blockDim.x) o.tile_done[i] = 0u;
  __syncthreads();
  // pass 2: bases, from the expert's offset and the ranges before this one
  if (active) {
    int run = s_cnt[e];
    for (int r = 0; r < rg; ++r) run += s_part[r * E + e];
    int c = c0;
    for (; c + 8 <= c1; c += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = __ldcg(hist + (size_t)(c + j) * E + e);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        o.base[(size_t)(c + j) * E + e] = run;
        run += v[j];
      }
    }
    for (; c < c1; ++c) {
      o.base[(size_t)c * E + e] = run;
      run += __ldcg(hist + (size_t)c * E + e);
    }
  }
}

}  // namespace ace
