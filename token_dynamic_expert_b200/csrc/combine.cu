// combine.cu -- the gate-weighted combine of the kept slots.
//
// y_t = sum over the kept slots i of token t, in rank order, of
// Yslot[pos(t, i)], where the down-projection epilogue already multiplied
// each slot row by its gate g_{t,i}.  Skipped slots (pos = -1) drop out of
// the sum; the survivors are not re-normalised.  fp32 sum, one rounding to
// the output type.  A position outside the n_rows rows of Yslot raises
// ACE_FLAG_BAD_INDEX and drops out as well.
#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {

template <typename T>
__global__ void __launch_bounds__(256) k_combine(int Tn, int k, int d,
                                                 const int32_t* __restrict__ slot_of,
                                                 const float* __restrict__ yslot, int n_rows,
                                                 T* __restrict__ y, uint32_t* status) {
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
  const int d4 = d >> 2;
  for (int i4 = threadIdx.x; i4 < d4; i4 += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < k; ++r) {
      const int p = s_pos[r];
      if (p < 0) continue;
      const float4 v = reinterpret_cast<const float4*>(yslot + (size_t)p * d)[i4];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    T* yo = y + (size_t)t * d + 4 * i4;
    yo[0] = from_f<T>(acc.x);
    yo[1] = from_f<T>(acc.y);
    yo[2] = from_f<T>(acc.z);
    yo[3] = from_f<T>(acc.w);
  }
}

cudaError_t launch_combine(ace_dtype dt, int T, int k, int d, const int32_t* slot_of,
                           const float* yslot, int n_rows, void* y, uint32_t* status,
                           cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (dt == ACE_BF16)
    k_combine<__nv_bfloat16><<<T, 256, 0, s>>>(T, k, d, slot_of, yslot, n_rows,
                                               (__nv_bfloat16*)y, status);
  else
    k_combine<float><<<T, 256, 0, s>>>(T, k, d, slot_of, yslot, n_rows, (float*)y, status);
  return cudaGetLastError();
}

}  // namespace ace
