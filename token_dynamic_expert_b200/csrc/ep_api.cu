// ep_api.cu -- the expert half of the layer on its own: the SwiGLU experts
// of one layer run over kept slots that arrive already grouped by expert, as
// they do on the rank that owns those experts in expert-parallel dispatch
// ([ACE] "Conclusion", future directions: distributed expert dispatch; the
// kept slots go to their experts' owner and the outputs come back for the
// gate-weighted combine).  Same expert kernels as the forward; the slot
// tiles come from the caller's offsets instead of the routing's scan.
#include <string.h>

#include "ace_common.cuh"
#include "ace_internal.h"
#include "compact.cuh"

namespace ace {
namespace {

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct ExpLayout {
  size_t status, h, tiles, n_tiles, tile_done, total;
  int max_tiles;
};

ExpLayout exp_layout(const ace_layer& L, int max_slots) {
  ExpLayout o;
  memset(&o, 0, sizeof(o));
  const size_t S = (size_t)(max_slots > 0 ? max_slots : 1);
  const size_t es = L.dtype == ACE_BF16 ? 2 : 4;
  o.max_tiles = L.E + cdiv((int)S, kTileN);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  o.status = take(256);
  o.h = take(S * (size_t)L.m * es);
  o.tiles = take((size_t)o.max_tiles * sizeof(int4));
  o.n_tiles = take(4);
  o.tile_done = take((size_t)o.max_tiles * 4);
  o.total = off;
  return o;
}

// The experts' own checks (the router, gamma and k play no part here).
ace_status check_expert_layer(const ace_layer* L) {
  if (!L) return ACE_ERR_INVALID_ARG;
  if (L->d <= 0 || L->E <= 0 || L->m <= 0) return ACE_ERR_INVALID_ARG;
  if (L->dtype != ACE_BF16 && L->dtype != ACE_F32) return ACE_ERR_INVALID_ARG;
  if (L->E > kMaxE) return ACE_ERR_UNSUPPORTED;
  if (!L->w_gate || !L->w_up || !L->w_down) return ACE_ERR_INVALID_ARG;
  if (!is_aligned(L->w_gate, 16) || !is_aligned(L->w_up, 16) || !is_aligned(L->w_down, 16))
    return ACE_ERR_INVALID_ARG;
  const int q = L->dtype == ACE_BF16 ? 128 : 64;
  if (L->d % q != 0 || L->m % q != 0) return ACE_ERR_UNSUPPORTED;
  return ACE_OK;
}

// One CTA: the expert tiles (expert, first slot, rows <= tile_n) from the
// caller's offsets [E + 1], in expert order.  Offsets that do not rise from 0
// to S give no tiles and ACE_FLAG_BAD_INDEX.
__global__ void k_tiles_from_offsets(const int32_t* __restrict__ offsets, int E, int S, int tile_n,
                                     int4* __restrict__ tiles, int32_t* __restrict__ n_tiles,
                                     int max_tiles, uint32_t* __restrict__ tile_done,
                                     uint32_t* status) {
  __shared__ int s_warp[32];
  __shared__ int s_bad;
  const int t = threadIdx.x;
  if (t == 0) s_bad = (offsets[0] != 0 || offsets[E] != S) ? 1 : 0;
  __syncthreads();
  int off = 0, cnt = 0;
  if (t < E) {
    off = offsets[t];
    cnt = offsets[t + 1] - off;
    if (off < 0 || cnt < 0 || off + cnt > S) s_bad = 1;
  }
  __syncthreads();
  const bool bad = s_bad != 0;
  const int ntile = (t < E && !bad) ? (cnt + tile_n - 1) / tile_n : 0;
  int total = 0;
  const int toff = block_excl_scan(ntile, s_warp, &total);
  if (ntile > 0) {  // near-equal tiles, as the forward's compaction makes them
    const int each = cnt / ntile, rem = cnt - each * ntile;
    for (int q = 0; q < ntile; ++q)
      if (toff + q < max_tiles)
        tiles[toff + q] = make_int4(t, off + q * each + min(q, rem), each + (q < rem ? 1 : 0),
                                    (q << 16) | ntile);
  }
  if (t == 0) {
    *n_tiles = min(total, max_tiles);
    if (bad) raise_flag(status, ACE_FLAG_BAD_INDEX);
  }
  for (int i = t; i < max_tiles; i += blockDim.x) tile_done[i] = 0u;
}

}  // namespace
}  // namespace ace

using namespace ace;

extern "C" {

size_t ace_experts_workspace_size(const ace_layer* layer, int max_slots) {
  if (check_expert_layer(layer) != ACE_OK || max_slots < 0) return 0;
  return exp_layout(*layer, max_slots).total;
}

ace_status ace_moe_experts(const ace_layer* layer, const void* xp, int S, const int32_t* offsets,
                           const float* slot_gate, void* yslot, void* ws, size_t ws_bytes,
                           void* stream) {
  const ace_status st = check_expert_layer(layer);
  if (st != ACE_OK) return st;
  if (S < 0) return ACE_ERR_INVALID_ARG;
  if (S > 0 && (!xp || !offsets || !slot_gate || !yslot || !is_aligned(xp, 16) ||
                !is_aligned(yslot, 16) || !is_aligned(offsets, 4) || !is_aligned(slot_gate, 4)))
    return ACE_ERR_INVALID_ARG;
  if (!ws || !is_aligned(ws, 256)) return ACE_ERR_WORKSPACE;
  const ace_layer& L = *layer;
  const ExpLayout ly = exp_layout(L, S);
  if (ws_bytes < ly.total) return ACE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(w + ly.status);
  if (launch_clear_words(status, 64, s) != cudaSuccess) return ACE_ERR_CUDA;
  if (S == 0) return ACE_OK;
  int4* tiles = reinterpret_cast<int4*>(w + ly.tiles);
  int32_t* n_tiles = reinterpret_cast<int32_t*>(w + ly.n_tiles);
  uint32_t* tile_done = reinterpret_cast<uint32_t*>(w + ly.tile_done);
  const int threads = ((L.E + 1 + 31) / 32) * 32;
  const bool fused = L.dtype == ACE_BF16 && (long long)S < 128LL * L.E;
  k_tiles_from_offsets<<<1, threads > 1024 ? 1024 : threads, 0, s>>>(
      offsets, L.E, S, kTileN, tiles, n_tiles, ly.max_tiles, tile_done, status);
  if (cudaGetLastError() != cudaSuccess) return ACE_ERR_CUDA;
  const int num_sms = device_sm_count();
  cudaError_t e;
  if (fused) {
    // small tiles: both GEMMs in one launch, as the forward does
    e = launch_experts_fused(L, S, xp, w + ly.h, yslot, tiles, n_tiles, ly.max_tiles, slot_gate,
                             tile_done, status, num_sms, s);
  } else if (L.dtype == ACE_BF16) {
    e = launch_experts_sm100(L, S, xp, w + ly.h, yslot, tiles, n_tiles, ly.max_tiles, slot_gate,
                             status, num_sms, s, nullptr);
  } else {
    e = launch_experts_simt(L, xp, w + ly.h, yslot, tiles, n_tiles, ly.max_tiles, slot_gate, s);
  }
  return e == cudaSuccess ? ACE_OK : ACE_ERR_CUDA;
}

ace_status ace_moe_combine(int T, int k, int d, ace_dtype dtype, const int32_t* slot_of,
                           const void* yslot, int n_rows, void* y, void* ws, size_t ws_bytes,
                           void* stream) {
  if (dtype != ACE_BF16 && dtype != ACE_F32) return ACE_ERR_INVALID_ARG;
  // rows are read and written as 16-byte vectors
  const int vec = dtype == ACE_BF16 ? 8 : 4;
  if (T < 0 || k < 1 || k > kMaxK || d <= 0 || d % vec != 0 || n_rows < 0)
    return ACE_ERR_INVALID_ARG;
  if (T > 0 && (!slot_of || !y || !is_aligned(slot_of, 4) || !is_aligned(y, 16) ||
                (n_rows > 0 && (!yslot || !is_aligned(yslot, 16)))))
    return ACE_ERR_INVALID_ARG;
  if (!ws || !is_aligned(ws, 256) || ws_bytes < 256) return ACE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(ws);
  if (launch_clear_words(status, 64, s) != cudaSuccess) return ACE_ERR_CUDA;
  return launch_combine(dtype, T, k, d, slot_of, yslot, n_rows, y, status, s) == cudaSuccess
             ? ACE_OK
             : ACE_ERR_CUDA;
}

}  // extern "C"
