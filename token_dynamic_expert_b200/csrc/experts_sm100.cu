// experts_sm100.cu -- grouped SwiGLU expert GEMMs over the kept slots on
// Blackwell tensor cores (tcgen05 + TMEM + TMA), bf16 in, fp32 accumulate.
//
// [ACE] "Theoretical Foundation", eq. for f_{l,e}: for the kept slots of
// expert e (rows row0 .. row0+n-1 of the gathered matrix Xp):
//   MODE 0:  H = SiLU(Xp W^gate_e) (.) (Xp W^up_e)      -> bf16 [S][m]
//   MODE 1:  Yslot = g * (H W^down_e)                   -> fp32 [S][d]
//
// Operand roles are swapped ("swap-AB"): the weight rows sit on the MMA's M
// side (128 rows per tile, the tensor-core M) and the expert's kept slots on
// N (16..256, rounded up to a multiple of 16), because an expert typically
// receives tens of slots while its weight matrix has hundreds of rows.  The
// accumulator lives in tensor memory: TMEM lane = weight row, column = slot.
//
// One persistent CTA per SM, 6 warps:
//   warp 0      TMA producer: weight tile(s) 128 x 64 and the slot tile
//               (32-row boxes, only as many as the tile's slots need) per
//               stage, 128-byte swizzle, mbarrier transaction counts.
//   warp 1      TMEM allocator and MMA issuer (one thread): 4 MMAs of K=16
//               per 64-wide stage; tcgen05.commit frees the stage and, after
//               the last stage of a work item, signals the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of 16 columns at a time, SiLU(.)*up or
//               gate scaling, stores to global memory.
// Work items are (tile, 128-row block of the weight) pairs, dealt round-robin.
// MODE 0 keeps two accumulators (gate, up) of up to 256 columns each; MODE 1
// double-buffers one accumulator so the epilogue overlaps the next item.
// Every mbarrier wait is bounded in time; a wait that runs out raises
// ACE_FLAG_TIMEOUT, the CTA drains what it issued and exits.
#include <math.h>
#include <stdio.h>

#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {
namespace {

constexpr int kBM = 128;                   // weight rows per work item (UMMA M)
constexpr int kBK = 64;                    // K per stage: one 128-B swizzle row of bf16
constexpr int kBoxN = 32;                  // slot rows per B TMA box
constexpr int kAStage = kBM * kBK * 2;     // 16 KB
constexpr int kBStage = kTileN * kBK * 2;  // 32 KB
constexpr int kBoxBytes = kBoxN * kBK * 2; // 4 KB
constexpr int kThreads = 192;

template <int MODE>
struct Cfg;
template <>
struct Cfg<0> {
  static constexpr int NA = 2;      // A operands per stage (gate, up)
  static constexpr int NS = 3;      // pipeline stages
  static constexpr int NACC = 1;    // accumulator buffers
};
template <>
struct Cfg<1> {
  static constexpr int NA = 1;
  static constexpr int NS = 4;
  static constexpr int NACC = 2;
};
constexpr uint32_t kTmemCols = 512;

template <int MODE>
constexpr int smem_bytes() {
  return 1024 /*alignment slack*/ + Cfg<MODE>::NS * (Cfg<MODE>::NA * kAStage + kBStage) + 256;
}

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > kWaitLimitNs) return false;
  return true;
}

__device__ __forceinline__ float silu(float a) { return a / (1.0f + expf(-a)); }

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_experts(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
              const __grid_constant__ CUtensorMap tmB, const int4* __restrict__ tiles,
              const int32_t* __restrict__ n_tiles_ptr, int max_tiles, int rows_per_expert,
              int K, int mtiles, void* __restrict__ out, int out_ld,
              const float* __restrict__ slot_gate, uint32_t* status) {
  using C = Cfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA0 = smem;
  uint8_t* sA1 = smem + C::NS * kAStage;  // MODE 0 only
  uint8_t* sB = smem + C::NS * C::NA * kAStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + C::NS * kBStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::NS;
  uint64_t* tfull = bars + 2 * C::NS;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = (int)warp_id(), lane = (int)lane_id();
  int n_tiles = *n_tiles_ptr;
  if (n_tiles > max_tiles || n_tiles < 0) {
    if (threadIdx.x == 0) raise_flag(status, ACE_FLAG_BAD_INDEX);
    n_tiles = n_tiles < 0 ? 0 : max_tiles;
  }
  const int total = n_tiles * mtiles;
  if ((int)blockIdx.x >= total) return;  // uniform across the CTA: no work, no TMEM
  const int ksteps = K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
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
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights: streamed once
      const uint64_t pol_x = policy_evict_last();   // slot rows: reused by every row block
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int w = blockIdx.x; w < total && !*abort_flag; w += gridDim.x) {
        const int ti = w / mtiles, mt = w - ti * mtiles;
        const int4 tl = tiles[ti];
        const int nbox = (tl.z + kBoxN - 1) / kBoxN;
        const uint32_t bytes = C::NA * kAStage + nbox * kBoxBytes;
        const int arow = tl.x * rows_per_expert + mt * kBM;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, status, abort_flag)) break;
          mbar_expect_tx(&full[stage], bytes);
          tma_load_2d(sA0 + stage * kAStage, &tmA0, kb * kBK, arow, &full[stage], pol_w);
          if (MODE == 0)
            tma_load_2d(sA1 + stage * kAStage, &tmA1, kb * kBK, arow, &full[stage], pol_w);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(sB + stage * kBStage + b * kBoxBytes, &tmB, kb * kBK, tl.y + b * kBoxN,
                        &full[stage], pol_x);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {  // let every copy this thread started land before exiting
        for (int s = 0; s < C::NS; ++s)
          if ((issued >> s) & 1u) mbar_wait_drain(&full[s], (issued_par >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int4 tl = tiles[w / mtiles];
        const int npad = (tl.z + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kBM, npad);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d0 = tmem + (MODE == 1 ? (uint32_t)acc * 256u : 0u);
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&full[stage], phase, status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA0 + stage * kAStage);
          const uint32_t a1 = smem_u32(sA1 + stage * kAStage);
          const uint32_t b = smem_u32(sB + stage * kBStage);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t accum = (kb | kk) != 0;
            const uint64_t db = sw128_kmajor_desc(b + kk * 32);
            mma_bf16(d0, sw128_kmajor_desc(a0 + kk * 32), db, idesc, accum);
            if (MODE == 0) mma_bf16(tmem + 256u, sw128_kmajor_desc(a1 + kk * 32), db, idesc, accum);
          }
          mma_commit(&empty[stage]);
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        if (C::NACC == 2) {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        } else {
          acc_phase ^= 1u;
        }
      }
      // wait for every MMA this thread issued before TMEM is released
      mma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const int ti = w / mtiles, mt = w - ti * mtiles;
      const int4 tl = tiles[ti];
      const int row0 = tl.y, n = tl.z;
      if (!mbar_wait(&tfull[acc], acc_phase, status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (MODE == 1 ? (uint32_t)acc * 256u : 0u);
      const int col = mt * kBM + row;
      for (int c0 = 0; c0 < n; c0 += 16) {
        float g[16];
        tmem_ld16(tbase + (uint32_t)c0, g);
        if (MODE == 0) {
          float u[16];
          tmem_ld16(tbase + 256u + (uint32_t)c0, u);
          tmem_ld_wait();
          __nv_bfloat16* H = reinterpret_cast<__nv_bfloat16*>(out);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (c0 + c < n)
              H[(size_t)(row0 + c0 + c) * out_ld + col] = __float2bfloat16_rn(silu(g[c]) * u[c]);
        } else {
          tmem_ld_wait();
          float* Y = reinterpret_cast<float*>(out);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (c0 + c < n) {
              const int slot = row0 + c0 + c;
              Y[(size_t)slot * out_ld + col] = slot_gate[slot] * g[c];
            }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (C::NACC == 2) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        acc_phase ^= 1u;
      }
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
  static int done = -1;  // per process; the attribute is per function and device-agnostic here
  if (done == 1) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_experts<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem_bytes<MODE>());
  if (e == cudaSuccess) done = 1;
  return e;
}

}  // namespace

cudaError_t launch_experts_sm100(const ace_layer& L, int cap_slots, const void* xp, void* h,
                                 float* yslot, const int4* tiles, const int32_t* n_tiles,
                                 int max_tiles, const float* slot_gate, uint32_t* status,
                                 int num_sms, cudaStream_t s, cudaEvent_t ev_mid) {
  CUtensorMap mg, mu, mx, md, mh;
  const uint64_t E = (uint64_t)L.E, d = (uint64_t)L.d, m = (uint64_t)L.m;
  if (!make_map(&mg, L.w_gate, E * m, d, kBM) || !make_map(&mu, L.w_up, E * m, d, kBM) ||
      !make_map(&mx, xp, (uint64_t)cap_slots, d, kBoxN) ||
      !make_map(&md, L.w_down, E * d, m, kBM) || !make_map(&mh, h, (uint64_t)cap_slots, m, kBoxN))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if ((e = set_smem_attr<0>()) != cudaSuccess) return e;
  if ((e = set_smem_attr<1>()) != cudaSuccess) return e;
  const int grid = num_sms;
  k_experts<0><<<grid, kThreads, smem_bytes<0>(), s>>>(mg, mu, mx, tiles, n_tiles, max_tiles,
                                                      L.m, L.d, L.m / kBM, h, L.m, slot_gate,
                                                      status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
  k_experts<1><<<grid, kThreads, smem_bytes<1>(), s>>>(md, md, mh, tiles, n_tiles, max_tiles,
                                                      L.d, L.m, L.d / kBM, yslot, L.d, slot_gate,
                                                      status);
  return cudaGetLastError();
}

}  // namespace ace
