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

// T: the storage type of Yslot and y; one 16-byte vector per thread and step
template <typename T>
__global__ void __launch_bounds__(256) k_combine(int Tn, int k, int d,
                                                 const int32_t* __restrict__ slot_of,
                                                 const T* __restrict__ yslot, int n_rows,
                                                 T* __restrict__ y, uint32_t* status) {
  constexpr int V = 16 / (int)sizeof(T);
  __shared__ int s_pos[kMaxK];
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    int p = slot_of[(size_t)t * k + threadIdx.x];
    if (p >= n_rows) {
      raise_flag(status, ACE_FLAG_BAD_INDEX);
      p = -1;
    }
    s_pos[threadIdx.x] = p;
  }
  __syncthreads();
  const int nv = d / V;
  for (int iv = threadIdx.x; iv < nv; iv += blockDim.x) {
    float acc[V];
#pragma unroll
    for (int c = 0; c < V; ++c) acc[c] = 0.f;
    for (int r = 0; r < k; ++r) {
      const int p = s_pos[r];
      if (p < 0) continue;
      const uint4 q = reinterpret_cast<const uint4*>(yslot + (size_t)p * d)[iv];
      const T* e = reinterpret_cast<const T*>(&q);
#pragma unroll
      for (int c = 0; c < V; ++c) acc[c] += to_f(e[c]);
    }
    uint4 o;
    T* oe = reinterpret_cast<T*>(&o);
#pragma unroll
    for (int c = 0; c < V; ++c) oe[c] = from_f<T>(acc[c]);
    reinterpret_cast<uint4*>(y + (size_t)t * d)[iv] = o;
  }
}

cudaError_t launch_combine(ace_dtype dt, int T, int k, int d, const int32_t* slot_of,
                           const void* yslot, int n_rows, void* y, uint32_t* status,
                           cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (dt == ACE_BF16)
    k_combine<__nv_bfloat16><<<T, 256, 0, s>>>(T, k, d, slot_of, (const __nv_bfloat16*)yslot,
                                               n_rows, (__nv_bfloat16*)y, status);
  else
    k_combine<float><<<T, 256, 0, s>>>(T, k, d, slot_of, (const float*)yslot, n_rows, (float*)y,
                                       status);
  return cudaGetLastError();
}

}  // namespace ace
