// combine.cu -- the gate-weighted combine of the kept slots.
//
// y_t = sum over the kept slots i of token t, in rank order, of
// Yslot[pos(t, i)], where the down-projection epilogue already multiplied
// each slot row by its gate g_{t,i} (and rounded it to the storage type).
// Skipped slots (pos = -1) drop out of the sum; the survivors are not
// re-normalised.  fp32 sum, one rounding to the output type.  A position
// outside the n_rows rows of Yslot raises ACE_FLAG_BAD_INDEX and drops out as
// well.
#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {

// Kept slots whose rows one thread loads before it adds any of them
constexpr int kCombineBatch = 8;
constexpr int kCombineCtasPerSm = 4;  // 256 threads of <= 64 registers

// T: the storage type of Yslot and y; one 16-byte vector per thread and step.
// A persistent grid walks the tokens t = blockIdx.x, + gridDim.x, ...  Warp 0
// lists each token's kept positions in rank order (a ballot over the k
// ranks) into one of two shared buffers, and loads the next token's slot
// positions while the CTA works on this one, so the only round trip per token
// is the rows'.  A thread issues the loads of up to kCombineBatch rows
// together and then adds them in rank order: the same sum, in the same order,
// as one rank at a time.
template <typename T>
__global__ void __launch_bounds__(256, kCombineCtasPerSm) k_combine(int Tn, int k, int d,
                                                 const int32_t* __restrict__ slot_of,
                                                 const T* __restrict__ yslot, int n_rows,
                                                 T* __restrict__ y, uint32_t* status) {
  constexpr int V = 16 / (int)sizeof(T);
  __shared__ int s_pos[2][kMaxK];
  __shared__ int s_n[2];
  const int lane = threadIdx.x & 31;
  const bool lister = threadIdx.x < 32;
  int p_next = -1;  // warp 0: slot position of rank `lane` of the next token
  if (lister && lane < k && (int)blockIdx.x < Tn) p_next = slot_of[(size_t)blockIdx.x * k + lane];
  const int nv = d / V;
  int buf = 0;
  for (int t = blockIdx.x; t < Tn; t += gridDim.x, buf ^= 1) {
    if (lister) {
      int p = p_next;
      if (p >= n_rows) {
        raise_flag(status, ACE_FLAG_BAD_INDEX);
        p = -1;
      }
      const uint32_t kept = __ballot_sync(0xffffffffu, p >= 0);
      if (p >= 0) s_pos[buf][__popc(kept & ((1u << lane) - 1u))] = p;
      if (lane == 0) s_n[buf] = __popc(kept);
      const int tn = t + (int)gridDim.x;
      p_next = (lane < k && tn < Tn) ? slot_of[(size_t)tn * k + lane] : -1;
    }
    // the buffer written here was last read two tokens ago, before the
    // previous token's barrier
    __syncthreads();
    const int n = s_n[buf];
    for (int iv = threadIdx.x; iv < nv; iv += blockDim.x) {
      float acc[V];
#pragma unroll
      for (int c = 0; c < V; ++c) acc[c] = 0.f;
      for (int r0 = 0; r0 < n; r0 += kCombineBatch) {
        uint4 q[kCombineBatch];
#pragma unroll
        for (int j = 0; j < kCombineBatch; ++j)
          if (r0 + j < n)
            q[j] = reinterpret_cast<const uint4*>(yslot + (size_t)s_pos[buf][r0 + j] * d)[iv];
#pragma unroll
        for (int j = 0; j < kCombineBatch; ++j) {
          if (r0 + j < n) {
            const T* e = reinterpret_cast<const T*>(&q[j]);
#pragma unroll
            for (int c = 0; c < V; ++c) acc[c] += to_f(e[c]);
          }
        }
      }
      uint4 o;
      T* oe = reinterpret_cast<T*>(&o);
#pragma unroll
      for (int c = 0; c < V; ++c) oe[c] = from_f<T>(acc[c]);
      reinterpret_cast<uint4*>(y + (size_t)t * d)[iv] = o;
    }
  }
}

cudaError_t launch_combine(ace_dtype dt, int T, int k, int d, const int32_t* slot_of,
                           const void* yslot, int n_rows, void* y, uint32_t* status,
                           cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int grid = min(T, kCombineCtasPerSm * device_sm_count());
  if (dt == ACE_BF16)
    k_combine<__nv_bfloat16><<<grid, 256, 0, s>>>(T, k, d, slot_of,
                                                  (const __nv_bfloat16*)yslot, n_rows,
                                                  (__nv_bfloat16*)y, status);
  else
    k_combine<float><<<grid, 256, 0, s>>>(T, k, d, slot_of, (const float*)yslot, n_rows,
                                          (float*)y, status);
  return cudaGetLastError();
}

}  // namespace ace
