// compact.cu -- deterministic compaction of the kept (token, expert) slots.
//
// Kept slots are ordered by expert, then by token.  The routing kernel left,
// per chunk c of 32 tokens and expert e, a bitmap of the chunk's tokens that
// kept a slot of e (a token routes to an expert at most once), its
// population count, and (its last CTA, compact.cuh) the base position of
// each (chunk, expert) run.  Here, one CTA per group of 4 tokens:
//   position of slot (t, i) of expert e = base[e][c] + popcount(bitmap[c][e]
//   below t); the slot tables are written and x_t is copied into row
//   `position` of the gathered matrix Xp.
// No result depends on the order atomics resolve in.
#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {

constexpr int kScatterTok = 4;  // tokens per CTA

template <typename T>
__global__ void __launch_bounds__(256) k_scatter_gather(
    int Tn, int k, int E, int d, const int32_t* __restrict__ idx, const float* __restrict__ gate,
    const uint8_t* __restrict__ keep, const uint32_t* __restrict__ bitmap,
    const int32_t* __restrict__ base, const T* __restrict__ x, size_t x_stride,
    int32_t* __restrict__ slot_token, int32_t* __restrict__ slot_rank,
    float* __restrict__ slot_gate, int32_t* __restrict__ slot_of, T* __restrict__ xp, int cap,
    uint32_t* status) {
  __shared__ int s_pos[kScatterTok * kMaxK], s_tok[kScatterTok * kMaxK];
  __shared__ int s_n;
  const int t0 = blockIdx.x * kScatterTok;
  const int c = t0 / kChunk;
  if (threadIdx.x == 0) s_n = 0;
  __syncthreads();
  if ((int)threadIdx.x < kScatterTok * k) {
    const int tq = threadIdx.x / k, i = threadIdx.x - tq * k;
    const int t = t0 + tq, tl = t - c * kChunk;
    if (t < Tn) {
      const size_t o = (size_t)t * k + i;
      int pos = -1;
      if (keep[o]) {
        const int e = idx[o];
        if (e < 0 || e >= E) {
          raise_flag(status, ACE_FLAG_BAD_INDEX);
        } else {
          const uint32_t bits = bitmap[(size_t)c * E + e];
          pos = base[(size_t)e * ((Tn + kChunk - 1) / kChunk) + c] +
                __popc(bits & ((1u << tl) - 1u));
          if (pos >= cap) {
            raise_flag(status, ACE_FLAG_OVERFLOW);
            pos = -1;
          } else {
            slot_token[pos] = t;
            slot_rank[pos] = i;
            slot_gate[pos] = gate[o];
            const int j = atomicAdd(&s_n, 1);  // copy list: order does not matter
            s_pos[j] = pos;
            s_tok[j] = t;
          }
        }
      }
      slot_of[o] = pos;
    }
  }
  __syncthreads();
  // Xp[pos] = x[t]: 16-byte vectors, four loads in flight per thread
  const int n = s_n;
  const int vpr = d * (int)sizeof(T) / 16;
  const int total = n * vpr;
  for (int q0 = threadIdx.x; q0 < total; q0 += 4 * blockDim.x) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = q0 + u * blockDim.x;
      if (q < total) {
        const int j = q / vpr, w = q - j * vpr;
        v[u] = reinterpret_cast<const uint4*>(x + (size_t)s_tok[j] * x_stride)[w];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = q0 + u * blockDim.x;
      if (q < total) {
        const int j = q / vpr, w = q - j * vpr;
        reinterpret_cast<uint4*>(xp + (size_t)s_pos[j] * d)[w] = v[u];
      }
    }
  }
}

cudaError_t launch_scatter_gather(ace_dtype dt, int T, int k, int E, int d, const int32_t* idx,
                                  const float* gate, const uint8_t* keep, const uint32_t* bitmap,
                                  const int32_t* base, const void* x, size_t x_stride,
                                  int32_t* slot_token, int32_t* slot_rank, float* slot_gate,
                                  int32_t* slot_of, void* xp, uint32_t* status, cudaStream_t s) {
  dim3 grid(cdiv(T, kScatterTok));
  const int cap = T * k;
  if (dt == ACE_BF16)
    k_scatter_gather<__nv_bfloat16><<<grid, 256, 0, s>>>(
        T, k, E, d, idx, gate, keep, bitmap, base, (const __nv_bfloat16*)x, x_stride, slot_token,
        slot_rank, slot_gate, slot_of, (__nv_bfloat16*)xp, cap, status);
  else
    k_scatter_gather<float><<<grid, 256, 0, s>>>(T, k, E, d, idx, gate, keep, bitmap, base,
                                                 (const float*)x, x_stride, slot_token, slot_rank,
                                                 slot_gate, slot_of, (float*)xp, cap, status);
  return cudaGetLastError();
}

}  // namespace ace
