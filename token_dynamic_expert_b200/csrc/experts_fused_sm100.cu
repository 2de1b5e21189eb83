// experts_fused_sm100.cu -- both grouped SwiGLU expert GEMMs of the prefill
// ([ACE] "Theoretical Foundation", eq. for f_{l,e}) in one persistent kernel:
//   gate/up items:  H = SiLU(Xp W^gate_e) (.) (Xp W^up_e)    -> bf16 [S][m]
//   down items:     Yslot = g * (H W^down_e)                 -> bf16 [S][d]
//
// The operands, tiles, warp roles, TMEM accumulators and epilogues are those
// of the two-launch version (experts_sm100.cu): swap-AB, weight rows on the
// MMA's M = 128, the expert's slots on N <= 256, TMA with 128-byte swizzle,
// one thread issuing tcgen05.mma, two 256-column accumulators alternating.
// What differs is the work list: every gate/up item (tile, 64-column block)
// comes first, then every down item (tile, 128-row block of W^down), dealt
// round-robin to one CTA per SM.  A down item needs the h rows of its tile,
// so the gate/up epilogue counts, per tile, the items it has written
// (release add after a proxy fence: the down item reads h with TMA), and the
// producer of a down item waits (bounded) until its tile's count is
// complete.  The gate/up tail of the launch then overlaps the first down
// items instead of idling SMs, and there is one launch instead of two.
// Gate/up items all precede down items in every CTA's order, so no wait can
// be on an item that has not been dealt, and the launch is cooperative, so
// every CTA that owes a tile its gate/up items is resident.
#include <math.h>

#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {
namespace {

constexpr int kBM = 128;                    // MMA M (weight rows per A tile)
constexpr int kBK = 64;                     // K per stage: one 128-B swizzle row of bf16
constexpr int kBoxN = 32;                   // slot rows per B TMA box
constexpr int kAStage = kBM * kBK * 2;      // 16 KB
constexpr int kBoxBytes = kBoxN * kBK * 2;  // 4 KB
constexpr int kMaxStages = 8;
constexpr int kStageBudget = 200 * 1024;
constexpr int kXchgBytes = 2 * 2 * 64 * 8 * 4;  // 2 buffers x (gate, up) x 64 rows x 8 floats
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;         // two accumulators of 256 columns
constexpr int kSmemBytes = 1024 + kStageBudget + kXchgBytes + 512;

__device__ __forceinline__ float silu(float a) { return a / (1.0f + expf(-a)); }

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

struct FusedArgs {
  const int4* tiles;
  const int32_t* n_tiles;
  int max_tiles, m, d;
  __nv_bfloat16* h;        // [S][m]
  __nv_bfloat16* yslot;    // [S][d]
  const float* slot_gate;  // [S]
  uint32_t* tile_done;     // [max_tiles] gate/up items written per tile (zeroed)
  uint32_t* status;
  uint64_t peer_wait_ns;   // limit of a down item's wait for its tile's h rows
};

__global__ void __launch_bounds__(kThreads, 1)
    k_experts_fused(const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmU,
                    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmD,
                    const __grid_constant__ CUtensorMap tmH, const FusedArgs a) {
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
  uint64_t* epi = drain + 1;  // the four epilogue warps' exchange points
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* s_maxn = reinterpret_cast<int*>(tmem_holder + 2);

  const int warp = (int)warp_id(), lane = (int)lane_id();
  int n_tiles = *a.n_tiles;
  if (n_tiles > a.max_tiles || n_tiles < 0) {
    if (threadIdx.x == 0) raise_flag(a.status, ACE_FLAG_BAD_INDEX);
    n_tiles = n_tiles < 0 ? 0 : a.max_tiles;
  }
  const int items0 = a.m / 64, items1 = a.d / kBM;  // per tile: gate/up, down
  const int total0 = n_tiles * items0;
  const int total = total0 + n_tiles * items1;
  if ((int)blockIdx.x >= total) return;  // uniform across the CTA: no work, no TMEM

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&tfull[q], 1);
      mbar_init(&tempty[q], 128);
    }
    mbar_init(drain, 1);
    mbar_init(epi, 128);
    *abort_flag = 0;
    *s_maxn = 1;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmG);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmD);
    tma_prefetch_desc(&tmH);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  {  // largest slot tile of the launch -> stage size and count
    int mx = 1;
    for (int i = threadIdx.x; i < n_tiles; i += blockDim.x) mx = max(mx, a.tiles[i].z);
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
        const bool down = w >= total0;
        const int wi = down ? w - total0 : w;
        const int per = down ? items1 : items0;
        const int ti = wi / per, it = wi - ti * per;
        const int4 tl = a.tiles[ti];
        const int nbox = (tl.z + kBoxN - 1) / kBoxN;
        const uint32_t bytes = kAStage + nbox * kBoxBytes;
        if (down) {  // the tile's h rows are complete once all its gate/up items counted
          const uint64_t t0 = global_ns();
          bool ready = true;
          while (ld_acquire_u32(a.tile_done + ti) < (uint32_t)items0) {
            if (*abort_flag || global_ns() - t0 > a.peer_wait_ns) {
              if (!*abort_flag) raise_flag(a.status, ACE_FLAG_TIMEOUT);
              *abort_flag = 1;
              ready = false;
              break;
            }
          }
          if (!ready) break;
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        const int ksteps = (down ? a.m : a.d) / kBK;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, a.status, abort_flag)) break;
          uint8_t* sa = smem + stage * stage_bytes;
          uint8_t* sb = sa + kAStage;
          mbar_expect_tx(&full[stage], bytes);
          if (!down) {  // 64 gate rows over 64 up rows of the same columns
            const int r = tl.x * a.m + it * 64;
            tma_load_2d(sa, &tmG, kb * kBK, r, &full[stage], pol_w);
            tma_load_2d(sa + kAStage / 2, &tmU, kb * kBK, r, &full[stage], pol_w);
            for (int b = 0; b < nbox; ++b)
              tma_load_2d(sb + b * kBoxBytes, &tmX, kb * kBK, tl.y + b * kBoxN, &full[stage],
                          pol_x);
          } else {
            tma_load_2d(sa, &tmD, kb * kBK, tl.x * a.d + it * kBM, &full[stage], pol_w);
            for (int b = 0; b < nbox; ++b)
              tma_load_2d(sb + b * kBoxBytes, &tmH, kb * kBK, tl.y + b * kBoxN, &full[stage],
                          pol_x);
          }
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
        const bool down = w >= total0;
        const int wi = down ? w - total0 : w;
        const int4 tl = a.tiles[wi / (down ? items1 : items0)];
        const int npad = (tl.z + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kBM, npad);
        const int ksteps = (down ? a.m : a.d) / kBK;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, a.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d0 = tmem + (uint32_t)acc * 256u;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&full[stage], phase, a.status, abort_flag)) {
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
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    int acc = 0;
    uint32_t acc_phase = 0, ephase = 0;
    int xb = 0;  // exchange buffer parity (gate/up items)
    // the epilogue warps meet on an mbarrier (bounded waits) rather than a
    // named barrier, so a warp that gives up cannot strand the others
    auto epi_sync = [&]() -> bool {
      mbar_arrive(epi);
      const bool ok = mbar_wait(epi, ephase, a.status, abort_flag);
      ephase ^= 1u;
      return ok;
    };
    bool ok = true;
    for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
      const bool down = w >= total0;
      const int wi = down ? w - total0 : w;
      const int per = down ? items1 : items0;
      const int ti = wi / per, it = wi - ti * per;
      const int4 tl = a.tiles[ti];
      const int row0 = tl.y, n = tl.z;
      if (!mbar_wait(&tfull[acc], acc_phase, a.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * 256u;
      if (!down) {
        const bool is_gate = q < 2;
        const int r = (q & 1) * 32 + lane;  // intermediate row within the 64-block
        const int col = it * 64 + r;
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
          if (!(ok = epi_sync())) break;
          const float4* other = reinterpret_cast<const float4*>((is_gate ? xu : xg) + r * 8);
          const float4 o0 = other[0], o1 = other[1];
          const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
          const int base = is_gate ? c0 : c0 + 8;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float g = is_gate ? v[c] : ov[c];
            const float u = is_gate ? ov[c] : v[8 + c];
            if (base + c < n)
              a.h[(size_t)(row0 + base + c) * a.m + col] = __float2bfloat16_rn(silu(g) * u);
          }
          xb ^= 1;
        }
        if (!ok) break;
        // this item's h block is written: count it for the tile (down items
        // read h through TMA, the async proxy)
        asm volatile("fence.proxy.async.global;" ::: "memory");
        if (!(ok = epi_sync())) break;
        if (warp == 2 && lane == 0)
          asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(a.tile_done + ti)
                       : "memory");
      } else {
        const int col = it * kBM + q * 32 + lane;
        for (int c0 = 0; c0 < n; c0 += 16) {
          float v[16];
          tmem_ld16(tbase + (uint32_t)c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (c0 + c < n) {
              const int slot = row0 + c0 + c;
              a.yslot[(size_t)slot * a.d + col] = __float2bfloat16_rn(a.slot_gate[slot] * v[c]);
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

// ----------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// bf16 matrix [rows][cols] (row-major), box of box_rows x 64 columns,
// 128-byte swizzle.
bool fused_map(CUtensorMap* mp, const void* base, uint64_t rows, uint64_t cols,
               uint32_t box_rows) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_experts_fused(const ace_layer& L, int cap_slots, const void* xp, void* h,
                                 void* yslot, const int4* tiles, const int32_t* n_tiles,
                                 int max_tiles, const float* slot_gate, uint32_t* tile_done,
                                 uint32_t* status, int num_sms, cudaStream_t s) {
  CUtensorMap mg, mu, mx, md, mh;
  const uint64_t E = (uint64_t)L.E, d = (uint64_t)L.d, m = (uint64_t)L.m;
  if (!fused_map(&mg, L.w_gate, E * m, d, 64) || !fused_map(&mu, L.w_up, E * m, d, 64) ||
      !fused_map(&mx, xp, (uint64_t)cap_slots, d, kBoxN) ||
      !fused_map(&md, L.w_down, E * d, m, kBM) ||
      !fused_map(&mh, h, (uint64_t)cap_slots, m, kBoxN))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k_experts_fused,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  FusedArgs a;
  a.tiles = tiles;
  a.n_tiles = n_tiles;
  a.max_tiles = max_tiles;
  a.m = L.m;
  a.d = L.d;
  a.h = static_cast<__nv_bfloat16*>(h);
  a.yslot = static_cast<__nv_bfloat16*>(yslot);
  a.slot_gate = slot_gate;
  a.tile_done = tile_done;
  a.status = status;
  a.peer_wait_ns = peer_wait_ns();
  // down items wait on other CTAs' gate/up items: a cooperative launch makes
  // every CTA of the grid resident at once (one per SM)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_experts_fused, mg, mu, mx, md, mh, a);
}

}  // namespace ace
