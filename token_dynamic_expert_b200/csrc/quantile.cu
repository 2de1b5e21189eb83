// quantile.cu -- quantile mapping of a skip budget to the threshold tau, on
// the device ([ACE] "Efficiency Results", Table 6: the threshold for a target
// skip rate is a quantile of the calibration scores).
//
// Candidates are the scores of the non-top-1 slots of a score pool
// [n_tok][k] (column 0, the top-1 slot, is never skipped).  With the
// candidates sorted ascending c_(1) <= ... <= c_(N), tau = c_(n+1): exactly n
// slots satisfy c < tau when no two scores tie; n <= 0 gives c_(1) (nothing
// skipped) and n >= N gives +inf (every candidate skipped).
//
// Selection of the (n+1)-th smallest is an exact radix select on the
// order-preserving 32-bit keys of the floats: four passes, one per byte from
// the most significant, each a histogram of the candidates that match the
// bytes chosen so far (k_tau_hist, grid-stride, shared-memory bins) followed by
// a one-CTA pick of the byte holding the wanted rank (k_tau_pick).
#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {
namespace {

struct TauState {
  uint32_t prefix, mask;
  unsigned long long rank;  // rank still wanted among the matching candidates
};

__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__global__ void __launch_bounds__(256) k_tau_hist(const float* __restrict__ score, long long n_el,
                                                  int k, int shift, const TauState* st,
                                                  uint32_t* __restrict__ hist) {
  __shared__ uint32_t bins[256];
  bins[threadIdx.x] = 0u;
  __syncthreads();
  const uint32_t prefix = st->prefix, mask = st->mask;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_el; i += stride) {
    if (i % k == 0) continue;  // top-1 slot
    const uint32_t key = fkey(__ldg(score + i));
    if ((key & mask) == prefix) atomicAdd(&bins[(key >> shift) & 0xffu], 1u);
  }
  __syncthreads();
  const uint32_t c = bins[threadIdx.x];
  if (c) atomicAdd(&hist[threadIdx.x], c);
}

__global__ void __launch_bounds__(256) k_tau_pick(const uint32_t* __restrict__ hist, int shift,
                                                  TauState* st, float* tau_out) {
  __shared__ unsigned long long incl[256];
  const int b = threadIdx.x;
  incl[b] = hist[b];
  __syncthreads();
  for (int o = 1; o < 256; o <<= 1) {  // inclusive scan of the bins
    const unsigned long long v = b >= o ? incl[b - o] : 0ull;
    __syncthreads();
    incl[b] += v;
    __syncthreads();
  }
  const unsigned long long r = st->rank;
  const unsigned long long before = b > 0 ? incl[b - 1] : 0ull;
  __syncthreads();
  if (before <= r && r < incl[b]) {  // exactly one bin holds rank r
    st->rank = r - before;
    st->prefix |= (uint32_t)b << shift;
    st->mask |= 0xffu << shift;
    if (shift == 0) *tau_out = key_to_float(st->prefix);
  }
}

__global__ void k_tau_init(TauState* st, long long rank, float* tau_out, int infinite) {
  st->prefix = 0u;
  st->mask = 0u;
  st->rank = (unsigned long long)rank;
  if (infinite) *tau_out = __uint_as_float(0x7f800000u);
}

}  // namespace

size_t tau_workspace_size() { return 256 + 4 * 256 * sizeof(uint32_t); }

cudaError_t launch_tau_quantile(const float* score, int n_tok, int k, long long n_skip,
                                float* tau, void* ws, int num_sms, cudaStream_t s) {
  const long long n_el = (long long)n_tok * k;
  const long long N = (long long)n_tok * (k - 1);
  TauState* st = reinterpret_cast<TauState*>(ws);
  uint32_t* hist = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + 256);
  const long long rank = n_skip <= 0 ? 0 : n_skip;
  if (N == 0 || rank >= N) {  // every candidate skipped (or none exist)
    k_tau_init<<<1, 1, 0, s>>>(st, 0, tau, 1);
    return cudaGetLastError();
  }
  cudaError_t e = cudaMemsetAsync(hist, 0, 4 * 256 * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  k_tau_init<<<1, 1, 0, s>>>(st, rank, tau, 0);
  long long blocks = (n_el + 255) / 256;
  const long long cap = 4LL * num_sms;
  if (blocks > cap) blocks = cap;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    k_tau_hist<<<(int)blocks, 256, 0, s>>>(score, n_el, k, shift, st, hist + pass * 256);
    k_tau_pick<<<1, 256, 0, s>>>(hist + pass * 256, shift, st, tau);
  }
  return cudaGetLastError();
}

}  // namespace ace
