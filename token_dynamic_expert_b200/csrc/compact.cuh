// compact.cuh -- the expert-offset scan of the compaction, as a block-level
// device routine run by the last routing CTA to finish.
//
// From the per-(256-token range, expert) kept-slot counts it forms the
// per-expert counts, the exclusive offsets over experts (kept slots ordered
// by expert, then token), the base position of each (range, expert) run and
// the list of expert GEMM tiles (expert, first slot, rows <= tile_n) in
// expert order.  The row gather adds the counts of the chunks before a
// token's chunk within its range (from the chunk bitmaps).
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
  int32_t* rbase;    // [nrange][E]: offset of e + kept slots of e in ranges before r
  int32_t* counts;   // [E]
  int32_t* offsets;  // [E + 1]
  int32_t* n_kept;   // [1]
  int4* tiles;       // [max_tiles]: (expert, first slot, slots, index in expert << 16 | tiles of expert)
  int32_t* n_tiles;  // [1]
  uint32_t* tile_done;  // [max_tiles] or NULL: per-tile counters, zeroed here
  int max_tiles, tile_n;
};

// Whole-CTA routine (every thread calls it; blockDim.x a multiple of 32 and
// at least E / 2).  range_cnt [nrange][E] is read with L2-coherent loads
// (other CTAs' atomics built it).  With E <= blockDim.x thread i takes expert
// i and keeps the first kRegRanges of its range counts in registers, so each
// pass is one round of loads; otherwise thread i takes experts 2i and 2i + 1
// and the exclusive scan over experts runs over per-thread pairs.  An expert
// of n kept slots gets ceil(n / tile_n) tiles of near-equal size (they differ
// by one slot at most), in slot order, each tagged with its index within the
// expert and the expert's tile count.
constexpr int kRegRanges = 32;

__device__ __forceinline__ void write_tiles(const ScanOut& o, int e, int off, int cnt, int ntile,
                                            int toff) {
  if (ntile <= 0) return;
  const int each = cnt / ntile, rem = cnt - each * ntile;
  for (int q = 0; q < ntile; ++q)
    if (toff + q < o.max_tiles)
      o.tiles[toff + q] = make_int4(e, off + q * each + min(q, rem), each + (q < rem ? 1 : 0),
                                    (q << 16) | ntile);
}

__device__ __forceinline__ void scan_experts(const int32_t* range_cnt, int nrange, int E,
                                             const ScanOut& o) {
  __shared__ int s_warp[32];
  const int t = threadIdx.x;
  int total, total_tiles;
  if (E <= (int)blockDim.x) {
    const bool on = t < E;
    int rc[kRegRanges];
    int cnt = 0;
#pragma unroll
    for (int r = 0; r < kRegRanges; ++r) {
      rc[r] = (on && r < nrange) ? __ldcg(range_cnt + (size_t)r * E + t) : 0;
      cnt += rc[r];
    }
    for (int r = kRegRanges; r < nrange; ++r)
      if (on) cnt += __ldcg(range_cnt + (size_t)r * E + t);
    const int off = block_excl_scan(cnt, s_warp, &total);
    const int ntile = on ? (cnt + o.tile_n - 1) / o.tile_n : 0;
    const int toff = block_excl_scan(ntile, s_warp, &total_tiles);
    if (on) {
      o.counts[t] = cnt;
      o.offsets[t] = off;
      write_tiles(o, t, off, cnt, ntile, toff);
      int run = off;
#pragma unroll
      for (int r = 0; r < kRegRanges; ++r)
        if (r < nrange) {
          o.rbase[(size_t)r * E + t] = run;
          run += rc[r];
        }
      for (int r = kRegRanges; r < nrange; ++r) {
        const size_t at = (size_t)r * E + t;
        const int c = __ldcg(range_cnt + at);
        o.rbase[at] = run;
        run += c;
      }
    }
  } else {
    const int e0 = 2 * t;
    int cnt[2] = {0, 0};
#pragma unroll 16
    for (int r = 0; r < nrange; ++r)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        if (e0 + j < E) cnt[j] += __ldcg(range_cnt + (size_t)r * E + e0 + j);
    const int off0 = block_excl_scan(cnt[0] + cnt[1], s_warp, &total);
    int ntile[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) ntile[j] = e0 + j < E ? (cnt[j] + o.tile_n - 1) / o.tile_n : 0;
    const int toff0 = block_excl_scan(ntile[0] + ntile[1], s_warp, &total_tiles);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int e = e0 + j;
      if (e >= E) continue;
      const int off = off0 + (j ? cnt[0] : 0);
      o.counts[e] = cnt[j];
      o.offsets[e] = off;
      write_tiles(o, e, off, cnt[j], ntile[j], toff0 + (j ? ntile[0] : 0));
    }
    int run[2] = {off0, off0 + cnt[0]};
#pragma unroll 8
    for (int r = 0; r < nrange; ++r)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        if (e0 + j < E) {
          const size_t at = (size_t)r * E + e0 + j;
          const int c = __ldcg(range_cnt + at);
          o.rbase[at] = run[j];
          run[j] += c;
        }
  }
  if (t == 0) {
    o.offsets[E] = total;
    *o.n_kept = total;
    *o.n_tiles = min(total_tiles, o.max_tiles);
  }
  if (o.tile_done)
    for (int i = t; i < o.max_tiles; i += blockDim.x) o.tile_done[i] = 0u;
}

}  // namespace ace
