// compact.cu -- deterministic compaction of the kept (token, expert) slots.
//
// Kept slots are ordered by expert, then by token.  The routing kernel left,
// per chunk c of 32 tokens and expert e, a bitmap of the chunk's tokens that
// kept a slot of e (a token routes to an expert at most once) and its
// population count.  From these:
//   k_scan     one CTA: per-expert counts, exclusive offsets over experts,
//              per-(chunk, expert) base positions, and the list of GEMM tiles
//              (expert, first slot, rows <= kTileN) in expert order.
//   k_scatter  one CTA per chunk: position of slot (t, i) of expert e =
//              base[c][e] + popcount(bitmap[c][e] below t); writes the slot
//              tables.
//   k_gather   copies x_t into row `pos` of the gathered matrix Xp.
// No result depends on the order atomics resolve in.
#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {

// Exclusive scan over the CTA in thread order; returns this thread's prefix,
// *total receives the sum.  All threads must call it.
__device__ int block_excl_scan(int v, int* s_warp, int* total) {
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

__global__ void __launch_bounds__(1024) k_scan(const int32_t* __restrict__ hist, int nchunk,
                                               int E, int tile_n, int max_tiles,
                                               int32_t* __restrict__ base,
                                               int32_t* __restrict__ counts,
                                               int32_t* __restrict__ offsets,
                                               int32_t* __restrict__ n_kept,
                                               int4* __restrict__ tiles,
                                               int32_t* __restrict__ n_tiles) {
  __shared__ int s_warp[32];
  int tpe = 1;  // threads per expert (a power of two that divides 32)
  while (tpe < 32 && tpe * 2 * E <= (int)blockDim.x) tpe *= 2;
  const int e = threadIdx.x / tpe, g = threadIdx.x % tpe;
  const bool active = e < E;
  const int per = (nchunk + tpe - 1) / tpe;
  const int cb = min(nchunk, g * per), ce = min(nchunk, cb + per);
  int local = 0;
  if (active)
    for (int c = cb; c < ce; ++c) local += hist[(size_t)c * E + e];
  // prefix inside the expert's group of tpe consecutive lanes
  int incl = local;
  for (int o = 1; o < tpe; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o, tpe);
    if (g >= o) incl += n;
  }
  const int excl_in_group = incl - local;
  const int cnt = __shfl_sync(0xffffffffu, incl, tpe - 1, tpe);
  int total, total_tiles;
  const int off = block_excl_scan((active && g == 0) ? cnt : 0, s_warp, &total);
  const int ntile = (active && g == 0) ? (cnt + tile_n - 1) / tile_n : 0;
  const int toff = block_excl_scan(ntile, s_warp, &total_tiles);
  const int off_e = __shfl_sync(0xffffffffu, off, 0, tpe);
  if (active) {
    int run = off_e + excl_in_group;
    for (int c = cb; c < ce; ++c) {
      base[(size_t)c * E + e] = run;
      run += hist[(size_t)c * E + e];
    }
    if (g == 0) {
      counts[e] = cnt;
      offsets[e] = off;
      for (int q = 0; q < ntile; ++q) {
        if (toff + q < max_tiles)
          tiles[toff + q] = make_int4(e, off + q * tile_n, min(tile_n, cnt - q * tile_n), 0);
      }
    }
  }
  if (threadIdx.x == 0) {
    offsets[E] = total;
    *n_kept = total;
    *n_tiles = min(total_tiles, max_tiles);
  }
}

cudaError_t launch_scan(const int32_t* hist, int nchunk, int E, int tile_n, int max_tiles,
                        int32_t* base, int32_t* counts, int32_t* offsets, int32_t* n_kept,
                        int4* tiles, int32_t* n_tiles, cudaStream_t s) {
  k_scan<<<1, 1024, 0, s>>>(hist, nchunk, E, tile_n, max_tiles, base, counts, offsets, n_kept,
                            tiles, n_tiles);
  return cudaGetLastError();
}

template <typename T>
__global__ void __launch_bounds__(256) k_scatter(
    int Tn, int k, int E, int d, const int32_t* __restrict__ idx, const float* __restrict__ gate,
    const uint8_t* __restrict__ keep, const uint32_t* __restrict__ bitmap,
    const int32_t* __restrict__ base, const T* __restrict__ x, int32_t* __restrict__ slot_token,
    int32_t* __restrict__ slot_rank, float* __restrict__ slot_gate,
    int32_t* __restrict__ slot_of, T* __restrict__ xp, int cap, uint32_t* status) {
  const int c = blockIdx.x;
  for (int s = threadIdx.x; s < kChunk * k; s += blockDim.x) {
    const int tl = s / k, i = s - tl * k;
    const int t = c * kChunk + tl;
    if (t >= Tn) continue;
    const size_t o = (size_t)t * k + i;
    int pos = -1;
    if (keep[o]) {
      const int e = idx[o];
      if (e < 0 || e >= E) {
        raise_flag(status, ACE_FLAG_BAD_INDEX);
      } else {
        const uint32_t bits = bitmap[(size_t)c * E + e];
        pos = base[(size_t)c * E + e] + __popc(bits & ((1u << tl) - 1u));
        if (pos >= cap) {
          raise_flag(status, ACE_FLAG_OVERFLOW);
          pos = -1;
        } else {
          slot_token[pos] = t;
          slot_rank[pos] = i;
          slot_gate[pos] = gate[o];
        }
      }
    }
    slot_of[o] = pos;
  }
}

// Xp[pos] = x[slot_token[pos]] for pos < n_kept: 4 rows per CTA, 16-byte
// vectors.  Launched over the worst-case slot count; CTAs past n_kept exit.
template <typename T>
__global__ void __launch_bounds__(256) k_gather(int d, const int32_t* __restrict__ n_kept,
                                                const int32_t* __restrict__ slot_token,
                                                const T* __restrict__ x, T* __restrict__ xp) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 6);
  if (row >= *n_kept) return;
  const int t = slot_token[row];
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)row * d);
  const int vpr = d * (int)sizeof(T) / 16;
  for (int v = threadIdx.x & 63; v < vpr; v += 64) dst[v] = src[v];
}

cudaError_t launch_scatter(ace_dtype dt, int T, int k, int E, int d, const int32_t* idx,
                           const float* gate, const uint8_t* keep, const uint32_t* bitmap,
                           const int32_t* base, const void* x, int32_t* slot_token,
                           int32_t* slot_rank, float* slot_gate, int32_t* slot_of, void* xp,
                           uint32_t* status, cudaStream_t s) {
  dim3 grid(cdiv(T, kChunk));
  const int cap = T * k;
  if (dt == ACE_BF16)
    k_scatter<__nv_bfloat16><<<grid, 256, 0, s>>>(
        T, k, E, d, idx, gate, keep, bitmap, base, (const __nv_bfloat16*)x, slot_token, slot_rank,
        slot_gate, slot_of, (__nv_bfloat16*)xp, cap, status);
  else
    k_scatter<float><<<grid, 256, 0, s>>>(T, k, E, d, idx, gate, keep, bitmap, base,
                                          (const float*)x, slot_token, slot_rank, slot_gate,
                                          slot_of, (float*)xp, cap, status);
  return cudaGetLastError();
}

cudaError_t launch_gather(ace_dtype dt, int cap, int d, const int32_t* n_kept,
                          const int32_t* slot_token, const void* x, void* xp, cudaStream_t s) {
  dim3 grid(cdiv(cap, 4));
  if (dt == ACE_BF16)
    k_gather<__nv_bfloat16><<<grid, 256, 0, s>>>(d, n_kept, slot_token, (const __nv_bfloat16*)x,
                                                 (__nv_bfloat16*)xp);
  else
    k_gather<float><<<grid, 256, 0, s>>>(d, n_kept, slot_token, (const float*)x, (float*)xp);
  return cudaGetLastError();
}

}  // namespace ace
