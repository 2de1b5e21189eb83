// experts_sm100.cu -- grouped SwiGLU expert GEMMs over the kept slots on
// Blackwell tensor cores (tcgen05 + TMEM + TMA), bf16 in, fp32 accumulate.
//
// [ACE] "Theoretical Foundation", eq. for f_{l,e}: for the kept slots of
// expert e (rows row0 .. row0+n-1 of the gathered matrix Xp):
//   MODE 0:  H = SiLU(Xp W^gate_e) (.) (Xp W^up_e)      -> bf16 [S][m]
//   MODE 1:  Yslot = g * (H W^down_e)                   -> bf16 [S][d]
//
// Operand roles are swapped ("swap-AB"): weight rows sit on the MMA's M side
// (128, the tensor-core M) and the expert's kept slots on N (16..256, rounded
// up to a multiple of 16), because an expert receives tens of slots while its
// weight matrices have hundreds of rows.  The accumulator lives in tensor
// memory: TMEM lane = weight row, column = slot.
//
// MODE 0 stacks 64 rows of W^gate and the same 64 rows of W^up into one
// 128-row A tile, so a work item covers 64 intermediate columns: lanes 0-63
// accumulate the gate pre-activations, lanes 64-127 the up projections.  The
// epilogue pairs them through a small shared-memory exchange.  Work items are
// (tile, 64-column block) in MODE 0 and (tile, 128-row block of W^down) in
// MODE 1, dealt round-robin to one persistent CTA per SM; the small items
// keep the last wave short.
//
// The gate/up launch runs on CTA pairs (tcgen05.mma.cta_group::2, see
// k_experts_pair below); the down launch on single CTAs.
//
// Warp roles:
//   warp 0      TMA producer: weight rows (128 x 64 bf16 per stage) and the
//               tile's slot rows (64-row boxes, only as many as it needs),
//               128-byte swizzle, mbarrier transaction counts.
//   warp 1      TMEM allocator and MMA issuer (one thread): 4 MMAs of K=16
//               per stage; tcgen05.commit frees the stage and, after the last
//               stage of an item, hands the accumulator to the epilogue.
//   warps 2..   epilogue: tcgen05.ld 16 columns at a time, SiLU(.)*up or
//               gate scaling, global stores; 4 warps in the gate/up (pair)
//               kernel, 8 in the down kernel.
// Two TMEM accumulators of 256 columns alternate between items, so the
// epilogue of one item overlaps the main loop of the next.  The stage count
// adapts to the largest slot tile of the launch (more stages when tiles are
// small, to keep more weight bytes in flight).  Every mbarrier wait is bounded
// in time; a wait that runs out raises ACE_FLAG_TIMEOUT, the CTA drains what
// it issued and exits.
#include <math.h>

#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {
namespace {

constexpr int kBM = 128;                    // MMA M (weight rows per A tile)
constexpr int kBK = 64;                     // K per stage: one 128-B swizzle row of bf16
constexpr int kBoxN = 64;                   // slot rows per B TMA box (fewer, larger loads)
constexpr int kAStage = kBM * kBK * 2;      // 16 KB
constexpr int kBoxBytes = kBoxN * kBK * 2;  // 8 KB
constexpr int kMaxStages = 8;
constexpr int kStageBudget = 200 * 1024;
// per epilogue group: 2 buffers x (gate, up) x 64 rows x 8 floats; two groups
constexpr int kXchgGroupFloats = 2 * 2 * 64 * 8;
constexpr int kXchgBytes = 2 * kXchgGroupFloats * 4;
// 8 epilogue warps, two per TMEM lane quarter taking alternate 16-slot groups
// (in the gate/up epilogue each group of four pairs gate with up values
// through its own exchange buffers and named barrier): the epilogue (a bf16
// store per slot and output column) is the slower side of the pipeline.
// The one-CTA gate/up form keeps 4.
constexpr int kEpiWarps1 = 8;
constexpr int kThreads1 = 64 + 32 * kEpiWarps1;
constexpr int kThreads = kThreads1;  // the CTA-pair kernel
constexpr uint32_t kTmemCols = 512;         // two accumulators of 256 columns
constexpr int kSmemBytes = 1024 + kStageBudget + kXchgBytes + 512;

__device__ __forceinline__ float silu(float a) { return a / (1.0f + expf(-a)); }

// Item w of a launch of (tile, row block) items.  An expert's tiles sit
// together in the tile list and each tile entry carries (its index within
// the expert << 16 | the expert's tile count) in .w, so the items can run
// row block by row block with the expert's tiles side by side: neighbouring
// items then stream the same weight rows at the same time, and the second
// tile of an expert reads them from L2 instead of HBM.
__device__ __forceinline__ void item_of(const int4* __restrict__ tiles, int n_tiles, int ipt,
                                        int w, int& ti, int& it) {
  const int t0 = w / ipt;
  const int4 a = tiles[t0];
  const int gs = t0 - min(a.w >> 16, t0);             // the expert's first tile
  const int gn = max(1, min(a.w & 0xffff, n_tiles - gs));
  const int l = w - gs * ipt;
  it = min(l / gn, ipt - 1);
  ti = gs + l % gn;
}

// named barrier of one group of four epilogue warps (ids 1 and 2)
__device__ __forceinline__ void epilogue_bar(int group) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + group) : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(kThreads1, 1)
    k_experts(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
              const __grid_constant__ CUtensorMap tmB, const int4* __restrict__ tiles,
              const int32_t* __restrict__ n_tiles_ptr, int max_tiles, int rows_per_expert,
              int K, int items_per_tile, void* __restrict__ out, int out_ld,
              const float* __restrict__ slot_gate, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* xchg = reinterpret_cast<float*>(smem + kStageBudget);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStageBudget + kXchgBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kMaxStages;
  uint64_t* tfull = bars + 2 * kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* s_maxn = reinterpret_cast<int*>(tmem_holder + 2);

  const int warp = (int)warp_id(), lane = (int)lane_id();
  int n_tiles = *n_tiles_ptr;
  if (n_tiles > max_tiles || n_tiles < 0) {
    if (threadIdx.x == 0) raise_flag(status, ACE_FLAG_BAD_INDEX);
    n_tiles = n_tiles < 0 ? 0 : max_tiles;
  }
  const int total = n_tiles * items_per_tile;
  if ((int)blockIdx.x >= total) return;  // uniform across the CTA: no work, no TMEM
  const int ksteps = K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], MODE == 1 ? 32 * kEpiWarps1 : 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *s_maxn = 1;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    if (MODE == 0) tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // largest slot tile of the launch -> stage size and count
  {
    int mx = 1;
    for (int i = threadIdx.x; i < n_tiles; i += blockDim.x) mx = max(mx, tiles[i].z);
    atomicMax(s_maxn, mx);
  }
  __syncthreads();
  const int maxbox = (min(*s_maxn, kTileN) + kBoxN - 1) / kBoxN;
  const int stage_bytes = kAStage + maxbox * kBoxBytes;
  int NS = kStageBudget / stage_bytes;
  NS = NS > kMaxStages ? kMaxStages : NS;
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights: streamed once
      const uint64_t pol_x = policy_evict_last();   // slot rows: reused by every row block
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int w = blockIdx.x; w < total && !*abort_flag; w += gridDim.x) {
        int ti, it;
        item_of(tiles, n_tiles, items_per_tile, w, ti, it);
        const int4 tl = tiles[ti];
        const int nbox = (tl.z + kBoxN - 1) / kBoxN;
        const uint32_t bytes = kAStage + nbox * kBoxBytes;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, status, abort_flag)) break;
          uint8_t* sa = smem + stage * stage_bytes;
          uint8_t* sb = sa + kAStage;
          mbar_expect_tx(&full[stage], bytes);
          if (MODE == 0) {  // 64 gate rows over 64 up rows of the same columns
            const int r = tl.x * rows_per_expert + it * 64;
            tma_load_2d(sa, &tmA0, kb * kBK, r, &full[stage], pol_w);
            tma_load_2d(sa + kAStage / 2, &tmA1, kb * kBK, r, &full[stage], pol_w);
          } else {
            tma_load_2d(sa, &tmA0, kb * kBK, tl.x * rows_per_expert + it * kBM, &full[stage],
                        pol_w);
          }
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(sb + b * kBoxBytes, &tmB, kb * kBK, tl.y + b * kBoxN, &full[stage], pol_x);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == NS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {  // let every copy this thread started land before exiting
        for (int s = 0; s < NS; ++s)
          if ((issued >> s) & 1u) mbar_drain(&full[s], (issued_par >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        int ti, it;
        item_of(tiles, n_tiles, items_per_tile, w, ti, it);
        const int4 tl = tiles[ti];
        const int npad = (tl.z + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kBM, npad);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d0 = tmem + (uint32_t)acc * 256u;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&full[stage], phase, status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * stage_bytes);
          const uint32_t b0 = a0 + kAStage;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16(d0, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc,
                     (kb | kk) != 0);
          mma_commit(&empty[stage]);
          if (++stage == NS) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // wait for every MMA this thread issued before TMEM is released
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
  } else if (MODE == 1 || warp < 6) {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    // MODE 1: the two warps of a quarter take alternate 16-slot groups
    const int g0 = MODE == 1 ? ((warp - 2) >> 2) * 16 : 0, gstep = MODE == 1 ? 32 : 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    int xb = 0;  // exchange buffer parity (MODE 0)
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      int ti, it;
      item_of(tiles, n_tiles, items_per_tile, w, ti, it);
      const int4 tl = tiles[ti];
      const int row0 = tl.y, n = tl.z;
      if (!mbar_wait(&tfull[acc], acc_phase, status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * 256u;
      if (MODE == 0) {
        const bool is_gate = q < 2;
        const int r = (q & 1) * 32 + lane;  // intermediate row within the 64-block
        const int col = it * 64 + r;
        __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(out);
        for (int c0 = 0; c0 < n; c0 += 16) {
          float v[16];
          tmem_ld16(tbase + (uint32_t)c0, v);
          tmem_ld_wait();
          float* xg = xchg + xb * 1024;  // gate values of columns 8..15
          float* xu = xg + 512;          // up values of columns 0..7
          float4* mine = reinterpret_cast<float4*>((is_gate ? xg : xu) + r * 8);
          const int off = is_gate ? 8 : 0;
          mine[0] = make_float4(v[off + 0], v[off + 1], v[off + 2], v[off + 3]);
          mine[1] = make_float4(v[off + 4], v[off + 5], v[off + 6], v[off + 7]);
          epilogue_bar(0);
          const float4* other = reinterpret_cast<const float4*>((is_gate ? xu : xg) + r * 8);
          const float4 o0 = other[0], o1 = other[1];
          const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
          const int base = is_gate ? c0 : c0 + 8;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float g = is_gate ? v[c] : ov[c];
            const float u = is_gate ? ov[c] : v[8 + c];
            if (base + c < n)
              H[(size_t)(row0 + base + c) * out_ld + col] = __float2bfloat16_rn(silu(g) * u);
          }
          xb ^= 1;
        }
      } else {
        const int col = it * kBM + q * 32 + lane;
        __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(out) + col;
        for (int c0 = g0; c0 < n; c0 += gstep) {
          float v[16];
          tmem_ld16(tbase + (uint32_t)c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; c += 2) {  // two slots per conversion
            const int slot = row0 + c0 + c;
            const float ga = c0 + c < n ? slot_gate[slot] : 0.f;
            const float gb = c0 + c + 1 < n ? slot_gate[slot + 1] : 0.f;
            const __nv_bfloat162 pr = __floats2bfloat162_rn(ga * v[c], gb * v[c + 1]);
            if (c0 + c < n) Y[(size_t)slot * out_ld] = pr.x;
            if (c0 + c + 1 < n) Y[(size_t)(slot + 1) * out_ld] = pr.y;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------- two-SM (CTA pair) form
// The same grouped GEMMs with tcgen05.mma.cta_group::2: a cluster of two
// CTAs on two SMs works on one item with M = 256.  CTA r of the pair holds
// 128 of the A rows (MODE 0: 64 gate + 64 up rows of its 64 intermediate
// columns; MODE 1: 128 rows of W^down) and half of the tile's slot rows
// (B rows r * N/2 .. (r + 1) * N/2 - 1), and accumulates its 128 rows x N
// slots in its own TMEM.  Each slot-row byte a CTA loads now feeds a
// 256-row MMA, so a stage holds 2/3 of the bytes of the one-SM form for the
// same MMA work on each SM, and the accumulators stay double-buffered.
//   * Both CTAs' TMA loads of a stage complete on the leader's (rank 0)
//     full barrier; the leader's producer arms it for the bytes of both.
//   * The leader's MMA thread issues the 256-row MMAs and commits, to both
//     CTAs at once (multicast), the release of a stage and the readiness of
//     an accumulator.
//   * Each CTA's epilogue reads its own TMEM and arrives on the leader's
//     accumulator-empty barrier.
// Every wait is bounded.  The CTAs of a pair always meet at the closing
// cluster barrier (no early exit), after which they free their TMEM
// together.  No TMA multicast.
constexpr uint32_t kPeerMask = 0xFEFFFFFFu;  // the leader's copy of a barrier address

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* m, int x,
                                                 int y, uint32_t leader_bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(leader_bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` in both CTAs of the pair once every tcgen05 operation this
// thread issued has completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  const uint16_t mask = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void arrive_on_leader(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   smem_u32(bar) & kPeerMask)
               : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_experts_pair(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2,
                   const int4* __restrict__ tiles,
                   const int32_t* __restrict__ n_tiles_ptr, int max_tiles, int rows_per_expert,
                   int K, int items_per_tile, int out_rows, void* __restrict__ out, int out_ld,
                   const float* __restrict__ slot_gate, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* xchg = reinterpret_cast<float*>(smem + kStageBudget);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStageBudget + kXchgBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kMaxStages;
  uint64_t* tfull = bars + 2 * kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* s_maxn = reinterpret_cast<int*>(tmem_holder + 2);

  const int warp = (int)warp_id(), lane = (int)lane_id();
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  int n_tiles = *n_tiles_ptr;
  if (n_tiles > max_tiles || n_tiles < 0) {
    if (threadIdx.x == 0) raise_flag(status, ACE_FLAG_BAD_INDEX);
    n_tiles = n_tiles < 0 ? 0 : max_tiles;
  }
  const int total = n_tiles * items_per_tile;
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  const int ksteps = K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full[s], 1);   // the leader's producer arms it; both CTAs' bytes land on it
      mbar_init(&empty[s], 1);  // one multicast commit per release
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 32 * kEpiWarps1);  // both CTAs' epilogue threads (the leader's copy counts)
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *s_maxn = 1;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    if (MODE == 0) tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {  // the same warp in both CTAs
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  {
    int mx = 1;
    for (int i = threadIdx.x; i < n_tiles; i += blockDim.x) mx = max(mx, tiles[i].z);
    atomicMax(s_maxn, mx);
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  // stage: this CTA's 128 A rows, then its half of the slot rows (the same
  // offsets in both CTAs: the MMA reads both halves at them)
  const int maxhalf = ((min(*s_maxn, kTileN) + 15) & ~15) / 2;
  const int maxbox = (maxhalf + kBoxN - 1) / kBoxN;
  const int stage_bytes = kAStage + maxbox * kBoxBytes;
  int NS = kStageBudget / stage_bytes;
  NS = NS > kMaxStages ? kMaxStages : NS;
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int w = pair; w < total && !*abort_flag; w += npairs) {
        int ti, it;
        item_of(tiles, n_tiles, items_per_tile, w, ti, it);
        const int4 tl = tiles[ti];
        const int half = ((tl.z + 15) & ~15) / 2;
        const int nbox = (half + kBoxN - 1) / kBoxN;
        // a half of 65-128 rows comes as one box of twice the rows (tmB2): the
        // same bytes in the same place from half the loads
        const bool wide = nbox == 2;
        const int brow = tl.y + (int)rank * half;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, status, abort_flag)) break;
          uint8_t* sa = smem + stage * stage_bytes;
          uint8_t* sb = sa + kAStage;
          if (leader) mbar_expect_tx(&full[stage], 2u * (uint32_t)(kAStage + nbox * kBoxBytes));
          const uint32_t lbar = smem_u32(&full[stage]) & kPeerMask;
          if (MODE == 0) {  // 64 gate rows over 64 up rows of this CTA's 64 columns
            const int r = tl.x * rows_per_expert + it * 128 + (int)rank * 64;
            tma_load_2d_pair(sa, &tmA0, kb * kBK, r, lbar, pol_w);
            tma_load_2d_pair(sa + kAStage / 2, &tmA1, kb * kBK, r, lbar, pol_w);
          } else {
            tma_load_2d_pair(sa, &tmA0, kb * kBK,
                             tl.x * rows_per_expert + it * 256 + (int)rank * kBM, lbar, pol_w);
          }
          if (wide)
            tma_load_2d_pair(sb, &tmB2, kb * kBK, brow, lbar, pol_x);
          else
            for (int b = 0; b < nbox; ++b)
              tma_load_2d_pair(sb + b * kBoxBytes, &tmB, kb * kBK, brow + b * kBoxN, lbar, pol_x);
          if (++stage == NS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int w = pair; w < total && ok; w += npairs) {
        int ti, it;
        item_of(tiles, n_tiles, items_per_tile, w, ti, it);
        const int4 tl = tiles[ti];
        const int npad = (tl.z + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, npad);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d0 = tmem + (uint32_t)acc * 256u;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&full[stage], phase, status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * stage_bytes);
          const uint32_t b0 = a0 + kAStage;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16_pair(d0, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32),
                          idesc, (kb | kk) != 0);
          mma_commit_pair(&empty[stage]);
          if (++stage == NS) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // every MMA this thread issued has completed before TMEM is released
      asm volatile(
          "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              smem_u32(drain))
          : "memory");
      mbar_drain(drain, 0);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;           // TMEM lane quarter this warp may read
    const int grp = (warp - 2) >> 2;  // its group: alternate 16-slot column groups
    int acc = 0;
    uint32_t acc_phase = 0;
    int xb = 0;
    for (int w = pair; w < total; w += npairs) {
      int ti, it;
      item_of(tiles, n_tiles, items_per_tile, w, ti, it);
      const int4 tl = tiles[ti];
      const int row0 = tl.y, n = tl.z;
      if (!mbar_wait(&tfull[acc], acc_phase, status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * 256u;
      if (MODE == 0) {
        const bool is_gate = q < 2;
        const int r = (q & 1) * 32 + lane;
        const int col = it * 128 + (int)rank * 64 + r;
        __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(out);
        for (int c0 = grp * 16; c0 < n; c0 += 32) {
          float v[16];
          tmem_ld16(tbase + (uint32_t)c0, v);
          tmem_ld_wait();
          float* xg = xchg + grp * kXchgGroupFloats + xb * 1024;
          float* xu = xg + 512;
          float4* mine = reinterpret_cast<float4*>((is_gate ? xg : xu) + r * 8);
          const int off = is_gate ? 8 : 0;
          mine[0] = make_float4(v[off + 0], v[off + 1], v[off + 2], v[off + 3]);
          mine[1] = make_float4(v[off + 4], v[off + 5], v[off + 6], v[off + 7]);
          epilogue_bar(grp);
          const float4* other = reinterpret_cast<const float4*>((is_gate ? xu : xg) + r * 8);
          const float4 o0 = other[0], o1 = other[1];
          const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
          const int base = is_gate ? c0 : c0 + 8;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float g = is_gate ? v[c] : ov[c];
            const float u = is_gate ? ov[c] : v[8 + c];
            if (base + c < n)
              H[(size_t)(row0 + base + c) * out_ld + col] = __float2bfloat16_rn(silu(g) * u);
          }
          xb ^= 1;
        }
      } else {
        const int col = it * 256 + (int)rank * kBM + q * 32 + lane;
        __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(out);
        for (int c0 = grp * 16; c0 < n; c0 += 32) {
          float v[16];
          tmem_ld16(tbase + (uint32_t)c0, v);
          tmem_ld_wait();
          if (col < out_rows) {
#pragma unroll
            for (int c = 0; c < 16; ++c)
              if (c0 + c < n) {
                const int slot = row0 + c0 + c;
                Y[(size_t)slot * out_ld + col] = __float2bfloat16_rn(slot_gate[slot] * v[c]);
              }
          }
        }
      }
      tc_fence_before();
      arrive_on_leader(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
  __syncthreads();
  if (*abort_flag) {
    // a wait ran out somewhere: copies this CTA started may still be landing
    // (their completion counts on the leader's barriers), so give them time
    if (threadIdx.x == 0) {
      const uint64_t t0 = global_ns();
      while (global_ns() - t0 < 100000ull) {
      }
    }
    __syncthreads();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs are done with TMEM and with each other's barriers
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ----------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 matrix [rows][cols] (row-major), box of box_rows x 64 columns,
// 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t set_smem_attr() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_experts<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e == cudaSuccess) done = true;
  return e;
}

template <int MODE>
cudaError_t launch_pair(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                        const CUtensorMap& b2, const int4* tiles, const int32_t* n_tiles, int max_tiles,
                        int rows_per_expert, int K, int items_per_tile, int out_rows, void* out,
                        int out_ld, const float* slot_gate, uint32_t* status, int num_sms,
                        cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_experts_pair<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(num_sms & ~1));  // whole pairs
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_experts_pair<MODE>, a0, a1, b, b2, tiles, n_tiles, max_tiles,
                            rows_per_expert, K, items_per_tile, out_rows, out, out_ld, slot_gate,
                            status);
}

}  // namespace

cudaError_t launch_experts_sm100(const ace_layer& L, int cap_slots, const void* xp, void* h,
                                 void* yslot, const int4* tiles, const int32_t* n_tiles,
                                 int max_tiles, const float* slot_gate, uint32_t* status,
                                 int num_sms, cudaStream_t s, cudaEvent_t ev_mid) {
  CUtensorMap mg, mu, mx, mx2, md, mh;
  const uint64_t E = (uint64_t)L.E, d = (uint64_t)L.d, m = (uint64_t)L.m;
  if (!make_map(&mg, L.w_gate, E * m, d, 64) || !make_map(&mu, L.w_up, E * m, d, 64) ||
      !make_map(&mx, xp, (uint64_t)cap_slots, d, kBoxN) ||
      !make_map(&mx2, xp, (uint64_t)cap_slots, d, 2 * kBoxN) ||
      !make_map(&md, L.w_down, E * d, m, kBM) || !make_map(&mh, h, (uint64_t)cap_slots, m, kBoxN))
    return cudaErrorInvalidValue;
  cudaError_t e;
  // gate/up on CTA pairs: items of 128 intermediate columns (m % 128 == 0
  // for bf16 layers).  Down stays on single CTAs: the pair form measured
  // slower there, with 8 epilogue warps and bf16 outputs too (0.185 vs
  // 0.158 ms at 8192 tokens, 256 experts; 0.173 vs 0.156 ms at 4096
  // tokens, 0% skip).
  if ((e = launch_pair<0>(mg, mu, mx, mx2, tiles, n_tiles, max_tiles, L.m, L.d, L.m / 128, L.m, h,
                          L.m, slot_gate, status, num_sms, s)) != cudaSuccess)
    return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
  if ((e = set_smem_attr<1>()) != cudaSuccess) return e;
  k_experts<1><<<num_sms, kThreads1, kSmemBytes, s>>>(md, md, mh, tiles, n_tiles, max_tiles, L.d,
                                                     L.m, L.d / kBM, yslot, L.d, slot_gate, status);
  return cudaGetLastError();
}

}  // namespace ace
