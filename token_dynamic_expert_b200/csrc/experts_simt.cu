// experts_simt.cu -- SwiGLU experts on CUDA cores, for fp32 layers.
//
// [ACE] "Theoretical Foundation", eq. for f_{l,e}: per kept slot,
//   h = SiLU(x W^gate) (.) (x W^up)        (k_simt_gateup)
//   Yslot = g * (h W^down)                 (k_simt_down)
// One CTA per (tile, 64 output columns); each thread owns one output column
// and walks the tile's slots.  Used for fp32 layers, which are small; bf16
// layers run on the tcgen05 kernels.
#include <math.h>

#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {

template <typename T>
__global__ void __launch_bounds__(256) k_simt_gateup(const T* __restrict__ wg,
                                                     const T* __restrict__ wu, int d, int m,
                                                     const T* __restrict__ xp, T* __restrict__ h,
                                                     const int4* __restrict__ tiles,
                                                     const int32_t* __restrict__ n_tiles) {
  if ((int)blockIdx.x >= *n_tiles) return;
  const int4 tl = tiles[blockIdx.x];
  const int e = tl.x, row0 = tl.y, n = tl.z;
  const int j = blockIdx.y * 64 + (threadIdx.x & 63), grp = threadIdx.x >> 6;
  if (j >= m) return;
  const T* g = wg + ((size_t)e * m + j) * d;
  const T* u = wu + ((size_t)e * m + j) * d;
  for (int r = grp; r < n; r += 4) {
    const T* xr = xp + (size_t)(row0 + r) * d;
    float a = 0.f, b = 0.f;
    for (int i = 0; i < d; ++i) {
      const float xv = to_f(xr[i]);
      a = fmaf(xv, to_f(g[i]), a);
      b = fmaf(xv, to_f(u[i]), b);
    }
    h[(size_t)(row0 + r) * m + j] = from_f<T>(a / (1.0f + expf(-a)) * b);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_simt_down(const T* __restrict__ wd, int d, int m,
                                                   const T* __restrict__ h,
                                                   T* __restrict__ yslot,
                                                   const float* __restrict__ slot_gate,
                                                   const int4* __restrict__ tiles,
                                                   const int32_t* __restrict__ n_tiles) {
  if ((int)blockIdx.x >= *n_tiles) return;
  const int4 tl = tiles[blockIdx.x];
  const int e = tl.x, row0 = tl.y, n = tl.z;
  const int i = blockIdx.y * 64 + (threadIdx.x & 63), grp = threadIdx.x >> 6;
  if (i >= d) return;
  const T* w = wd + ((size_t)e * d + i) * m;
  for (int r = grp; r < n; r += 4) {
    const T* hr = h + (size_t)(row0 + r) * m;
    float acc = 0.f;
    for (int j = 0; j < m; ++j) acc = fmaf(to_f(hr[j]), to_f(w[j]), acc);
    yslot[(size_t)(row0 + r) * d + i] = from_f<T>(slot_gate[row0 + r] * acc);
  }
}

cudaError_t launch_experts_simt(const ace_layer& L, const void* xp, void* h, void* yslot,
                                const int4* tiles, const int32_t* n_tiles, int max_tiles,
                                const float* slot_gate, cudaStream_t s) {
  dim3 g1(max_tiles, cdiv(L.m, 64)), g2(max_tiles, cdiv(L.d, 64));
  if (L.dtype == ACE_F32) {
    k_simt_gateup<float><<<g1, 256, 0, s>>>((const float*)L.w_gate, (const float*)L.w_up, L.d,
                                            L.m, (const float*)xp, (float*)h, tiles, n_tiles);
    k_simt_down<float><<<g2, 256, 0, s>>>((const float*)L.w_down, L.d, L.m, (const float*)h,
                                          (float*)yslot, slot_gate, tiles, n_tiles);
  } else {
    k_simt_gateup<__nv_bfloat16><<<g1, 256, 0, s>>>(
        (const __nv_bfloat16*)L.w_gate, (const __nv_bfloat16*)L.w_up, L.d, L.m,
        (const __nv_bfloat16*)xp, (__nv_bfloat16*)h, tiles, n_tiles);
    k_simt_down<__nv_bfloat16><<<g2, 256, 0, s>>>((const __nv_bfloat16*)L.w_down, L.d, L.m,
                                                  (const __nv_bfloat16*)h,
                                                  (__nv_bfloat16*)yslot, slot_gate, tiles,
                                                  n_tiles);
  }
  return cudaGetLastError();
}

}  // namespace ace
