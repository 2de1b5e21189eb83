// ace_common.cuh -- device helpers shared by the libace kernels (sm_100a).
//
// Thin inline-PTX wrappers for the Blackwell data path: mbarriers, TMA tiled
// loads, tcgen05 (TMEM allocation, MMA, commit, TMEM loads) and the global
// timer used to bound every wait.  Also the workspace layout shared by the
// host entry points and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ace.h"

namespace ace {

// ----------------------------------------------------------------- numerics
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------ status word
__device__ __forceinline__ void raise_flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// Upper bound for any pipeline wait before the kernel gives up, sets
// ACE_FLAG_TIMEOUT and drains (nanoseconds of %globaltimer).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ smem
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------ programmatic launches
// In a launch with programmatic stream serialisation allowed: wait until the
// previous kernel of the stream has completed and its memory is visible (a
// no-op in any other launch), and let the next such launch be scheduled.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `bar` with parity `parity` to complete.
// Returns false (and raises ACE_FLAG_TIMEOUT once, setting *abort) when the
// limit passes or another role of the CTA already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                          volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (global_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      raise_flag(status, ACE_FLAG_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Wait for a phase whose completion is already owed (copies or MMAs this
// thread issued), so that a CTA leaving early lets them land first: no abort
// check, the fixed limit only.  False if the limit passed.
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

// -------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled load of the box at (x = inner coordinate, y) into smem; completes
// `bytes` of transaction on `bar`.  x * element size must be a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* m, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------- tcgen05
// TMEM allocation: one full warp; the allocated column base is written to
// `holder` in shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* holder, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(holder)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored the way a
// 128-byte-swizzled TMA box of 64 bf16 columns leaves it: rows of 128 B,
// groups of 8 rows 1024 B apart (SBO), tile base 1024-B aligned.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)1 << 16;                    // leading byte offset (16 B, unused)
  d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset
  d |= (uint64_t)1 << 46;                    // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                    // 128-byte swizzle
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32
// accumulate, both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                          // D format fp32
         | (1u << 7)                        // A format bf16
         | (1u << 10)                       // B format bf16
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- fusion
// The per-expert factor F(A^GSP, A^RCR)(e) of the fused score c = g F: the
// gates are non-negative, so fusing the two views' scores g A^GSP and
// g A^RCR by max / min / mean / one view equals fusing the tables.
struct FuseTables {
  const float* amax;   // max(A^GSP, A^RCR), or NULL
  const float* a_gsp;  // or NULL
  const float* a_rcr;  // or NULL
  int fusion;          // ace_fusion
};

__device__ __forceinline__ float fused_factor(const FuseTables& f, int e) {
  switch (f.fusion) {
    case ACE_FUSE_MIN: return fminf(f.a_gsp[e], f.a_rcr[e]);
    case ACE_FUSE_MEAN: return 0.5f * (f.a_gsp[e] + f.a_rcr[e]);
    case ACE_FUSE_GSP: return f.a_gsp[e];
    case ACE_FUSE_RCR: return f.a_rcr[e];
    default:
      if (f.amax) return f.amax[e];
      if (f.a_gsp && f.a_rcr) return fmaxf(f.a_gsp[e], f.a_rcr[e]);
      return 1.0f;
  }
}

// The normalised, scaled input element x = (u * (1/rms)) * gamma in fp32,
// each product rounded (no contraction into an FMA): every kernel that forms
// x from u uses this, so they all hold the same bits.
__device__ __forceinline__ float xhat(float u, float inv_rms, float gamma) {
  return __fmul_rn(__fmul_rn(u, inv_rms), gamma);
}

// ---------------------------------------------------------------- top-k
// order-preserving map of a float to an unsigned key (larger float, larger key)
__device__ __forceinline__ uint32_t fkey(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Warp-wide top-k of the logits held as v[q] = logit of expert lane + 32 q:
// k rounds of (largest key by redux.max, then the smallest expert index among
// the lanes holding it by redux.min).  Lane i < k receives rank i.
template <int NV>
__device__ __forceinline__ void topk_select(const float (&v)[NV], int nq, int E, int k, int lane,
                                            int& sel_e, float& sel_v, uint32_t* status) {
  uint32_t taken = 0u;
  for (int i = 0; i < k; ++i) {
    uint32_t bk = 0u;
    int be = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      if (q >= nq) break;
      const int e = lane + 32 * q;
      if (e < E && !((taken >> q) & 1u)) {
        const uint32_t kk = fkey(v[q]);
        if (kk > bk || be == 0x7fffffff) {  // lower index wins ties: q ascends
          bk = kk;
          be = e;
        }
      }
    }
    const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
    const int we = (int)__reduce_min_sync(0xffffffffu, (bk == mk) ? (uint32_t)be : 0x7fffffffu);
    int e_sel = we;
    if (e_sel < 0 || e_sel >= E) {
      raise_flag(status, ACE_FLAG_BAD_INDEX);
      e_sel = 0;
    }
    if ((e_sel & 31) == lane) taken |= 1u << (e_sel >> 5);
    if (lane == i) sel_e = e_sel;
  }
  // the selected logits: lane i < k fetches v of expert sel_e from its owner lane
  float mine = -INFINITY;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const float x = __shfl_sync(0xffffffffu, v[q], sel_e & 31);
    if ((sel_e >> 5) == q) mine = x;
  }
  sel_v = mine;
}

// inverse of fkey: the float whose key is k
__device__ __forceinline__ float fkey_inv(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// The same selection as topk_select (same ranks, same tie rule: the lower
// expert index wins) for a compile-time count NV of logits per lane, in fewer
// instructions.  Each lane packs its candidates as (key << 32 | ~expert), so
// that one unsigned compare orders them by logit and then by lower index, and
// sorts them once, largest first, with Batcher's odd-even merge network
// (19 compare-exchanges for NV = 8).  Each of the k rounds then looks only at
// the lanes' list heads: the largest key by redux.max, the smallest expert
// index among the heads that carry it by redux.max of ~expert, and the owner
// lane pops its head.  Experts e >= E carry the packed value 0, below every
// real candidate.  The selected logit comes back exactly from its key.
template <int NV>
__device__ __forceinline__ void topk_sorted(const float (&v)[NV], int E, int k, int lane,
                                            int& sel_e, float& sel_v, uint32_t* status) {
  uint64_t c[NV];
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int e = lane + 32 * q;
    c[q] = e < E ? ((uint64_t)fkey(v[q]) << 32) | (uint64_t)(~(uint32_t)e) : 0ull;
  }
#pragma unroll
  for (int p = 1; p < NV; p <<= 1)
#pragma unroll
    for (int kk = p; kk >= 1; kk >>= 1)
#pragma unroll
      for (int j = kk % p; j + kk < NV; j += 2 * kk)
#pragma unroll
        for (int i = 0; i < kk; ++i) {
          const int a = i + j, b = i + j + kk;
          if (b < NV && a / (2 * p) == b / (2 * p)) {
            const uint64_t x = c[a], y = c[b];
            const bool sw = y > x;
            c[a] = sw ? y : x;
            c[b] = sw ? x : y;
          }
        }
  for (int i = 0; i < k; ++i) {
    const uint32_t hk = (uint32_t)(c[0] >> 32);
    const uint32_t mk = __reduce_max_sync(0xffffffffu, hk);
    const uint32_t ne = __reduce_max_sync(0xffffffffu, hk == mk ? (uint32_t)c[0] : 0u);
    int e_sel = (int)~ne;
    const bool valid = e_sel >= 0 && e_sel < E;
    if (!valid) {
      raise_flag(status, ACE_FLAG_BAD_INDEX);
      e_sel = 0;
    }
    const bool pop = valid && (e_sel & 31) == lane;
#pragma unroll
    for (int q = 0; q + 1 < NV; ++q) c[q] = pop ? c[q + 1] : c[q];
    if (pop) c[NV - 1] = 0ull;
    if (lane == i) {
      sel_e = e_sel;
      sel_v = fkey_inv(mk);
    }
  }
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }
__device__ __forceinline__ uint32_t warp_id() { return threadIdx.x >> 5; }

}  // namespace ace
