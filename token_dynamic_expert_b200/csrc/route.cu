// route.cu -- the online routing half of the ACE MoE forward.
//
//   k_rmsnorm        1/rms_t, and (when asked) x_t = RMSNorm(u_t) * gamma
//                    rounded to the storage type ([ACE] "Theoretical
//                    Foundation": x = xbar Gamma_l).  The forward's consumers
//                    (the routers, the row gather) form x from u and 1/rms
//                    themselves.
//   k_router_logits  l_{t,e} = x_t . w_e, fp32 CUDA-core GEMM over a K split
//                    (fp32 layers; bf16 layers use the tensor-core router in
//                    router_sm100.cu)
//   k_topk_mask      per token: top-k by logit, gates, ACE scores
//                    c = g * max(A^GSP, A^RCR), skip mask with the top-1 slot
//                    always kept ([ACE] "3. Conservative Fusion"; [NEWS]:
//                    table lookups, the gate and scalar operations), plus the
//                    per-chunk expert bitmaps the compaction consumes.
//
// The router logits use the unrounded fp32 x (u * (1/rms) * gamma); the
// experts consume x rounded to the storage type.
#include <float.h>
#include <math.h>

#include "ace_common.cuh"
#include "ace_internal.h"
#include "compact.cuh"

namespace ace {

// ------------------------------------------------------------------ RMSNorm
// One warp per token, 16-byte loads and stores (d is a multiple of 64).
// x (nullable) receives xhat(u, 1/rms, gamma) rounded to the storage type.
// As the forward's first kernel it also zeroes the call's status words
// (clear[0 .. n_clear)) and the top-k kernel's bitmaps and range counts
// (zero[0 .. n_zero)), which no kernel of the forward touches before it, and
// (w3 non-null, bf16 layers) forms the tensor-core router's operand: the
// router rows with gamma folded in, w'_ek = gamma_k w_ek in fp32, as three
// bf16 terms hi + mid + lo (each the rounding of what the previous terms
// leave) at w3[term * E + e][k].
template <typename T>
__global__ void __launch_bounds__(256) k_rmsnorm(const T* __restrict__ u, int Tn, int d,
                                                 const float* __restrict__ gamma, float eps,
                                                 float* __restrict__ inv_rms, T* __restrict__ x,
                                                 uint32_t* __restrict__ clear, int n_clear,
                                                 uint32_t* __restrict__ zero, size_t n_zero,
                                                 const __nv_bfloat16* __restrict__ wr, int E,
                                                 __nv_bfloat16* __restrict__ w3) {
  constexpr int V = 16 / sizeof(T);
  if (blockIdx.x == 0 && (int)threadIdx.x < n_clear) clear[threadIdx.x] = 0u;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_zero;
       i += (size_t)gridDim.x * blockDim.x)
    zero[i] = 0u;
  if (w3 != nullptr) {
    const int vpr = d / 8;
    const size_t nvec = (size_t)E * vpr;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec;
         i += (size_t)gridDim.x * blockDim.x) {
      const int e = (int)(i / vpr), v = (int)(i - (size_t)e * vpr);
      const uint4 q = reinterpret_cast<const uint4*>(wr + (size_t)e * d)[v];
      const __nv_bfloat16* wv = reinterpret_cast<const __nv_bfloat16*>(&q);
      uint4 oh, om, ol;
      __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(&oh);
      __nv_bfloat16* mi = reinterpret_cast<__nv_bfloat16*>(&om);
      __nv_bfloat16* lo = reinterpret_cast<__nv_bfloat16*>(&ol);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float wf = __fmul_rn(gamma[v * 8 + c], __bfloat162float(wv[c]));
        h[c] = __float2bfloat16_rn(wf);
        const float r1 = __fsub_rn(wf, __bfloat162float(h[c]));
        mi[c] = __float2bfloat16_rn(r1);
        lo[c] = __float2bfloat16_rn(__fsub_rn(r1, __bfloat162float(mi[c])));
      }
      reinterpret_cast<uint4*>(w3 + (size_t)e * d)[v] = oh;
      reinterpret_cast<uint4*>(w3 + (size_t)(E + e) * d)[v] = om;
      reinterpret_cast<uint4*>(w3 + (size_t)(2 * E + e) * d)[v] = ol;
    }
  }
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= Tn) return;
  const uint4* ur = reinterpret_cast<const uint4*>(u + (size_t)t * d);
  const int nv = d / V;
  float ss = 0.f;
  for (int v = lane; v < nv; v += 32) {
    const uint4 q = ur[v];
    const T* e = reinterpret_cast<const T*>(&q);
#pragma unroll
    for (int c = 0; c < V; ++c) {
      const float f = to_f(e[c]);
      ss = fmaf(f, f, ss);
    }
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)d + eps);
  if (lane == 0) inv_rms[t] = r;
  if (x == nullptr) return;
  uint4* xr = reinterpret_cast<uint4*>(x + (size_t)t * d);
  for (int v = lane; v < nv; v += 32) {
    const uint4 q = ur[v];
    const T* e = reinterpret_cast<const T*>(&q);
    uint4 o;
    T* oe = reinterpret_cast<T*>(&o);
#pragma unroll
    for (int c = 0; c < V; ++c) oe[c] = from_f<T>(xhat(to_f(e[c]), r, gamma[v * V + c]));
    xr[v] = o;
  }
}

cudaError_t launch_rmsnorm(ace_dtype dt, const void* u, int T, int d, const float* gamma,
                           float eps, float* inv_rms, void* x, uint32_t* clear, int n_clear,
                           uint32_t* zero, size_t n_zero, const void* wr, int E, void* w3,
                           cudaStream_t s) {
  dim3 grid(cdiv(T, 8));
  if (n_clear > 256) return cudaErrorInvalidValue;
  if (dt == ACE_BF16)
    k_rmsnorm<__nv_bfloat16><<<grid, 256, 0, s>>>(
        (const __nv_bfloat16*)u, T, d, gamma, eps, inv_rms, (__nv_bfloat16*)x, clear, n_clear,
        zero, n_zero, (const __nv_bfloat16*)wr, E, (__nv_bfloat16*)w3);
  else
    k_rmsnorm<float><<<grid, 256, 0, s>>>((const float*)u, T, d, gamma, eps, inv_rms, (float*)x,
                                          clear, n_clear, zero, n_zero, nullptr, 0, nullptr);
  return cudaGetLastError();
}

// ------------------------------------------------------------ router logits
// part[split][t][e] = sum over k in split's range of xhat[t][k] * w[e][k],
// xhat = u * inv_rms * gamma.  64 x 64 output tile, 4 x 4 per thread.
template <typename T>
__global__ void __launch_bounds__(256) k_router_logits(const T* __restrict__ u,
                                                       const float* __restrict__ inv_rms,
                                                       const float* __restrict__ gamma,
                                                       const T* __restrict__ wr, int Tn, int d,
                                                       int E, int kper, float* __restrict__ part) {
  __shared__ float As[kRouterBK][kRouterBT + 4];
  __shared__ float Bs[kRouterBK][kRouterBE + 4];
  const int t0 = blockIdx.x * kRouterBT, e0 = blockIdx.y * kRouterBE, split = blockIdx.z;
  const int kbeg = split * kper, kend = kbeg + kper;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int lr = tid >> 2, lk = (tid & 3) * 8;
  const bool arow = (t0 + lr) < Tn, brow = (e0 + lr) < E;
  const float rr = arow ? inv_rms[t0 + lr] : 0.f;
  const T* ua = u + (size_t)(arow ? t0 + lr : 0) * d;
  const T* wb = wr + (size_t)(brow ? e0 + lr : 0) * d;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = kbeg; k0 < kend; k0 += kRouterBK) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int kk = k0 + lk + j;
      As[lk + j][lr] = arow ? xhat(to_f(ua[kk]), rr, gamma[kk]) : 0.f;
      Bs[lk + j][lr] = brow ? to_f(wb[kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRouterBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = part + (size_t)split * Tn * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= Tn) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) out[(size_t)t * E + e] = acc[i][j];
    }
  }
}

int router_splitk(int T, int d, int E, int num_sms) {
  const int tiles = cdiv(T, kRouterBT) * cdiv(E, kRouterBE);
  int s = cdiv(2 * num_sms, tiles);
  if (s > kMaxSplitK) s = kMaxSplitK;
  if (s < 1) s = 1;
  while (s > 1 && (d % (s * kRouterBK)) != 0) --s;
  return s;
}

cudaError_t launch_router_logits(ace_dtype dt, const void* u, const float* inv_rms,
                                 const float* gamma, const void* wr, int T, int d, int E,
                                 int splitk, float* part, cudaStream_t s) {
  dim3 grid(cdiv(T, kRouterBT), cdiv(E, kRouterBE), splitk);
  const int kper = d / splitk;
  if (dt == ACE_BF16)
    k_router_logits<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)u, inv_rms, gamma,
                                                        (const __nv_bfloat16*)wr, T, d, E, kper,
                                                        part);
  else
    k_router_logits<float><<<grid, 256, 0, s>>>((const float*)u, inv_rms, gamma,
                                                (const float*)wr, T, d, E, kper, part);
  return cudaGetLastError();
}

// -------------------------------------------------------- top-k and the mask
// One warp per token, eight tokens per CTA.  Lane l holds the logits of
// experts l, l+32, ...  Selection order is (logit descending, expert index
// ascending); slot 0 is the top-1 expert.  Each kept slot sets its token's bit
// in the chunk bitmap bitmap[t / 32][e] and counts itself in the range count
// range_cnt[t / 256][e] (integer atomics: the results do not depend on their
// order; both arrays are zeroed by RMSNorm).  The last CTA to finish runs the
// expert-offset scan over the range counts.
constexpr int kTopkWarps = 8;

// DEEP: every split's loads of a lane in flight at once (64 loads, 128
// registers, two CTAs an SM) for the many-split launches of short token
// counts; otherwise four splits at a time in 64 registers (four CTAs an SM),
// for the few-split launches of long ones.
template <int V, bool DEEP>
__global__ void __launch_bounds__(kTopkWarps * 32, DEEP ? 2 : 4) k_topk_mask(
    const float* __restrict__ part, int splitk, int Tn, int E, int k,
    const float* __restrict__ bias, const FuseTables ft, float tau, int renorm,
    int32_t* __restrict__ idx, float* __restrict__ gate, float* __restrict__ score,
    uint8_t* __restrict__ keep, uint32_t* __restrict__ bitmap, int32_t* __restrict__ range_cnt,
    float* __restrict__ logits_out, uint32_t* status, uint32_t* done_ctr, ScanOut so) {
  __shared__ int s_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t < Tn) {
    // the lane's fused factors and bias, loaded beside the partial sums
    float fv[V], bv[V];
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const int e = lane + 32 * q;
      fv[q] = e < E ? fused_factor(ft, e) : 0.f;
      bv[q] = (e < E && bias) ? bias[e] : 0.f;
    }
    // split-K partial sums in split order
    constexpr int kUnroll = DEEP ? (V >= 4 ? 64 / V : 16) : (V >= 8 ? 2 : 4);
    float v[V];
#pragma unroll
    for (int q = 0; q < V; ++q) v[q] = 0.f;
#pragma unroll kUnroll
    for (int sp = 0; sp < splitk; ++sp) {
      const float* pr = part + ((size_t)sp * Tn + t) * E;
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int e = lane + 32 * q;
        if (e < E) v[q] += pr[e];
      }
    }
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const int e = lane + 32 * q;
      if (e < E) {
        if (bias) v[q] += bv[q];
        if (logits_out) logits_out[(size_t)t * E + e] = v[q];
      } else {
        v[q] = -INFINITY;
      }
    }
    int my_e = 0;
    float my_v = -INFINITY;
    topk_sorted(v, E, k, lane, my_e, my_v, status);
    // the factor of the selected expert, from the lane that holds it
    float fac = 0.f;
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const float x = __shfl_sync(0xffffffffu, fv[q], my_e & 31);
      if ((my_e >> 5) == q) fac = x;
    }
    const float v0 = __shfl_sync(0xffffffffu, my_v, 0);  // the top-1 logit is the maximum
    const float ex = (lane < k) ? expf(my_v - v0) : 0.f;
    float denom;
    if (renorm) {
      denom = warp_sum(ex);
    } else {
      float z = 0.f;
#pragma unroll
      for (int q = 0; q < V; ++q) z += (lane + 32 * q < E) ? expf(v[q] - v0) : 0.f;
      denom = warp_sum(z);
    }
    if (lane < k) {
      const float g = ex / denom;
      const float sc = g * fac;
      const bool kept = (lane == 0) || !(sc < tau);
      const size_t o = (size_t)t * k + lane;
      idx[o] = my_e;
      gate[o] = g;
      score[o] = sc;
      keep[o] = kept ? 1 : 0;
      if (kept) {
        atomicOr(&bitmap[(size_t)(t / kChunk) * E + my_e], 1u << (t % kChunk));
        atomicAdd(&range_cnt[(size_t)(t / kRangeTok) * E + my_e], 1);
      }
    }
  }
  if (done_ctr == nullptr) return;
  // the last CTA to finish runs the expert-offset scan (each CTA's atomics
  // are ordered before its arrival count)
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t prev;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(prev) : "l"(done_ctr) : "memory");
    s_last = prev == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last) scan_experts(range_cnt, (Tn + kRangeTok - 1) / kRangeTok, E, so);
}

cudaError_t launch_topk_mask(const float* part, int splitk, int T, int E, int k,
                             const float* bias, const FuseTables& ft, float tau, int renorm,
                             int32_t* idx, float* gate, float* score, uint8_t* keep,
                             uint32_t* bitmap, int32_t* range_cnt, float* logits_out,
                             uint32_t* status, uint32_t* done_ctr, const ScanOut* so,
                             cudaStream_t s) {
  dim3 grid(cdiv(T, kTopkWarps));
  const ScanOut sv = so ? *so : ScanOut{};
  if (so == nullptr) done_ctr = nullptr;
#define ACE_TOPK(V)                                                                          \
  if (splitk > 4)                                                                            \
    k_topk_mask<V, true><<<grid, kTopkWarps * 32, 0, s>>>(                                   \
        part, splitk, T, E, k, bias, ft, tau, renorm, idx, gate, score, keep, bitmap,        \
        range_cnt, logits_out, status, done_ctr, sv);                                        \
  else                                                                                       \
    k_topk_mask<V, false><<<grid, kTopkWarps * 32, 0, s>>>(                                  \
        part, splitk, T, E, k, bias, ft, tau, renorm, idx, gate, score, keep, bitmap,        \
        range_cnt, logits_out, status, done_ctr, sv)
  if (E <= 32) {
    ACE_TOPK(1);
  } else if (E <= 64) {
    ACE_TOPK(2);
  } else if (E <= 128) {
    ACE_TOPK(4);
  } else if (E <= 256) {
    ACE_TOPK(8);
  } else {  // 16 logits a lane: the shallow form would spill
    k_topk_mask<16, true><<<grid, kTopkWarps * 32, 0, s>>>(
        part, splitk, T, E, k, bias, ft, tau, renorm, idx, gate, score, keep, bitmap, range_cnt,
        logits_out, status, done_ctr, sv);
  }
#undef ACE_TOPK
  return cudaGetLastError();
}

}  // namespace ace
