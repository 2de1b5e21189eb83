// compact.cu -- deterministic compaction of the kept (token, expert) slots.
//
// Kept slots are ordered by expert, then by token.  The routing kernel left,
// per chunk c of 32 tokens and expert e, a bitmap of the chunk's tokens that
// kept a slot of e (a token routes to an expert at most once), and (its last
// CTA, compact.cuh) the base position rbase[r][e] of each 256-token range r.
// Here, one CTA per group of 4 tokens:
//   position of slot (t, i) of expert e = rbase[r][e]
//       + popcount(bitmap[c'][e]) over the range's chunks c' before t's chunk c
//       + popcount(bitmap[c][e] below t);
// the slot tables are written and x_t = xhat(u_t, 1/rms_t, gamma), rounded to
// the storage type, is formed once per token and written into row
// `position` of the gathered matrix Xp for each of its kept slots.
// No result depends on the order atomics resolve in.
#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {

constexpr int kScatterTok = 4;  // tokens per CTA

template <typename T>
__global__ void __launch_bounds__(256) k_scatter_gather(
    int Tn, int k, int E, int d, const int32_t* __restrict__ idx, const float* __restrict__ gate,
    const uint8_t* __restrict__ keep, const uint32_t* __restrict__ bitmap,
    const int32_t* __restrict__ rbase, const T* __restrict__ u, const float* __restrict__ inv_rms,
    const float* __restrict__ gamma, int32_t* __restrict__ slot_token,
    int32_t* __restrict__ slot_rank, float* __restrict__ slot_gate, int32_t* __restrict__ slot_of,
    T* __restrict__ xp, int cap, uint32_t* status) {
  __shared__ int s_pos[kScatterTok][kMaxK];
  __shared__ int s_n[kScatterTok];
  const int t0 = blockIdx.x * kScatterTok;
  const int c = t0 / kChunk;
  // Xp[pos] = x_t: one 16-byte vector of u per thread and step (four in
  // flight), turned into x and stored to each kept slot of the token.  The
  // first step's loads do not depend on the positions, so they are issued
  // before the positions are worked out.
  constexpr int V = 16 / (int)sizeof(T);
  const int vpr = d / V;
  const int total = kScatterTok * vpr;
  uint4 v[4];
  float r[4];
  auto load_step = [&](int q0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = q0 + j * (int)blockDim.x;
      const int tq = q / vpr, w = q - tq * vpr, t = t0 + tq;
      r[j] = 0.f;
      if (q < total && t < Tn) {
        v[j] = reinterpret_cast<const uint4*>(u + (size_t)t * d)[w];
        r[j] = inv_rms[t];
      }
    }
  };
  load_step(threadIdx.x);
  if (threadIdx.x < kScatterTok) s_n[threadIdx.x] = 0;
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
          const int c0 = (t / kRangeTok) * (kRangeTok / kChunk);
          pos = rbase[(size_t)(t / kRangeTok) * E + e] +
                __popc(bitmap[(size_t)c * E + e] & ((1u << tl) - 1u));
#pragma unroll
          for (int j = 0; j < kRangeTok / kChunk - 1; ++j)
            if (c0 + j < c) pos += __popc(bitmap[(size_t)(c0 + j) * E + e]);
          if (pos >= cap) {
            raise_flag(status, ACE_FLAG_OVERFLOW);
            pos = -1;
          } else {
            slot_token[pos] = t;
            slot_rank[pos] = i;
            slot_gate[pos] = gate[o];
            const int j = atomicAdd(&s_n[tq], 1);  // copy list: order does not matter
            s_pos[tq][j] = pos;
          }
        }
      }
      slot_of[o] = pos;
    }
  }
  __syncthreads();
  for (int q0 = threadIdx.x; q0 < total; q0 += 4 * blockDim.x) {
    if (q0 != (int)threadIdx.x) load_step(q0);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = q0 + j * blockDim.x;
      const int tq = q / vpr, w = q - tq * vpr;
      if (q < total && t0 + tq < Tn) {
        const T* e = reinterpret_cast<const T*>(&v[j]);
        uint4 o;
        T* oe = reinterpret_cast<T*>(&o);
        float gg[V];  // gamma is 16-byte aligned (checked with the layer)
#pragma unroll
        for (int h = 0; h < V / 4; ++h) {
          const float4 g4 = reinterpret_cast<const float4*>(gamma + (size_t)w * V)[h];
          gg[4 * h] = g4.x;
          gg[4 * h + 1] = g4.y;
          gg[4 * h + 2] = g4.z;
          gg[4 * h + 3] = g4.w;
        }
#pragma unroll
        for (int cc = 0; cc < V; ++cc) oe[cc] = from_f<T>(xhat(to_f(e[cc]), r[j], gg[cc]));
        const int n = s_n[tq];
        for (int i = 0; i < n; ++i) reinterpret_cast<uint4*>(xp + (size_t)s_pos[tq][i] * d)[w] = o;
      }
    }
  }
}

cudaError_t launch_scatter_gather(ace_dtype dt, int T, int k, int E, int d, const int32_t* idx,
                                  const float* gate, const uint8_t* keep, const uint32_t* bitmap,
                                  const int32_t* rbase, const void* u, const float* inv_rms,
                                  const float* gamma, int32_t* slot_token, int32_t* slot_rank,
                                  float* slot_gate, int32_t* slot_of, void* xp, uint32_t* status,
                                  cudaStream_t s) {
  dim3 grid(cdiv(T, kScatterTok));
  const int cap = T * k;
  if (dt == ACE_BF16)
    k_scatter_gather<__nv_bfloat16><<<grid, 256, 0, s>>>(
        T, k, E, d, idx, gate, keep, bitmap, rbase, (const __nv_bfloat16*)u, inv_rms, gamma,
        slot_token, slot_rank, slot_gate, slot_of, (__nv_bfloat16*)xp, cap, status);
  else
    k_scatter_gather<float><<<grid, 256, 0, s>>>(T, k, E, d, idx, gate, keep, bitmap, rbase,
                                                 (const float*)u, inv_rms, gamma, slot_token,
                                                 slot_rank, slot_gate, slot_of, (float*)xp, cap,
                                                 status);
  return cudaGetLastError();
}

}  // namespace ace
