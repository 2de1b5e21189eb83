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
// least E, at most 1024).  hist is expert-major, [E][nchunk], and read with
// L2-coherent loads (other CTAs wrote it); base is chunk-major, [nchunk][E].
// A warp takes four experts at a time: their chunk counts are summed (pass 1)
// and, once the offsets over experts are known, scanned over the chunks in
// segments of 32 (pass 2).
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

__device__ __forceinline__ void scan_experts(const int32_t* hist, int nchunk, int E,
                                             const ScanOut& o) {
  __shared__ int s_warp[32];
  __shared__ int s_cnt[1024], s_off[1024];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  constexpr int kEpw = 4;  // experts a warp handles at once
  // pass 1: per-expert counts
  for (int eb = warp; eb < E; eb += kEpw * nw) {
    int acc[kEpw] = {0, 0, 0, 0};
#pragma unroll 8
    for (int c = lane; c < nchunk; c += 32)
#pragma unroll
      for (int j = 0; j < kEpw; ++j) {
        const int e = eb + j * nw;
        if (e < E) acc[j] += __ldcg(hist + (size_t)e * nchunk + c);
      }
#pragma unroll
    for (int j = 0; j < kEpw; ++j) {
#pragma unroll
      for (int sh = 16; sh > 0; sh >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], sh);
      const int e = eb + j * nw;
      if (lane == 0 && e < E) s_cnt[e] = acc[j];
    }
  }
  __syncthreads();
  // offsets over experts and the tile list
  const int t = threadIdx.x;
  const int cnt = t < E ? s_cnt[t] : 0;
  int total, total_tiles;
  const int off = block_excl_scan(cnt, s_warp, &total);
  const int ntile = t < E ? (cnt + o.tile_n - 1) / o.tile_n : 0;
  const int toff = block_excl_scan(ntile, s_warp, &total_tiles);
  if (t < E) {
    s_off[t] = off;
    o.counts[t] = cnt;
    o.offsets[t] = off;
    for (int q = 0; q < ntile; ++q)
      if (toff + q < o.max_tiles)
        o.tiles[toff + q] = make_int4(t, off + q * o.tile_n, min(o.tile_n, cnt - q * o.tile_n), 0);
  }
  if (t == 0) {
    o.offsets[E] = total;
    *o.n_kept = total;
    *o.n_tiles = min(total_tiles, o.max_tiles);
  }
  if (o.tile_done)
    for (int i = t; i < o.max_tiles; i += blockDim.x) o.tile_done[i] = 0u;
  __syncthreads();
  // pass 2: base[e][c] = offset of e + kept slots of e in chunks before c
  // (expert-major, so a warp's stores over consecutive chunks coalesce).  The
  // loads of kGroups 32-chunk groups go out together before their scans: one
  // CTA runs this, so its time is round trips to L2, not bandwidth.
  constexpr int kGroups = 8;
  for (int eb = warp; eb < E; eb += kEpw * nw) {
    int carry[kEpw];
#pragma unroll
    for (int j = 0; j < kEpw; ++j) carry[j] = eb + j * nw < E ? s_off[eb + j * nw] : 0;
    for (int c0 = 0; c0 < nchunk; c0 += 32 * kGroups) {
      int v[kEpw][kGroups];
#pragma unroll
      for (int j = 0; j < kEpw; ++j) {
        const int e = eb + j * nw;
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          const int c = c0 + g * 32 + lane;
          v[j][g] = (e < E && c < nchunk) ? __ldcg(hist + (size_t)e * nchunk + c) : 0;
        }
      }
#pragma unroll
      for (int j = 0; j < kEpw; ++j) {
        const int e = eb + j * nw;
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          const int c = c0 + g * 32 + lane;
          const int incl = warp_incl_scan(v[j][g], lane);
          if (e < E && c < nchunk) o.base[(size_t)e * nchunk + c] = carry[j] + incl - v[j][g];
          carry[j] += __shfl_sync(0xffffffffu, incl, 31);
        }
      }
    }
  }
}

}  // namespace ace
