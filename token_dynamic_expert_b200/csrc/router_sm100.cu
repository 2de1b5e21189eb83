// router_sm100.cu -- router logits l = x . w_e on tcgen05 tensor cores with
// fp32-level accuracy.
//
// The logits decide the top-k and, through the gates, the skip mask, so they
// must carry fp32 precision ([ACE] "3. Conservative Fusion": a slot is
// skipped by comparing g * A against tau).  With x_t = r_t (u_t (.) gamma) and
// r_t = 1 / rms(u_t) ([ACE] "Theoretical Foundation"), the logit is
//   l_te = r_t * sum_k u_tk (gamma_k w_ek),
// so gamma is folded into the router rows: w'_ek = gamma_k w_ek in fp32 enters
// as three bf16 terms w' = hi + mid + lo (each the round-to-nearest of what
// the previous terms leave, 24 significant bits together; RMSNorm forms them
// for the call), and u is bf16, so every product u_tk * term is exact in fp32.
// A long tensor-core accumulation would still lose low bits, so the sum is cut
// into 64-column chunks: per chunk, 12 MMAs (3 terms x 4 K-steps of 16)
// accumulate into a fresh TMEM buffer, and the epilogue adds the chunk result
// into fp32 registers.  The error is then that of an fp32 sum over the chunk
// values.  The epilogue multiplies each token's sum by r_t.
//
// Tile: 128 tokens (MMA M) x 128 experts (N), K split into `splits` ranges
// whose fp32 partial sums part[split][t][e] the top-k kernel adds in split
// order.  A stage is the 128 x 64 u tile and the three 128 x 64 term tiles of
// the tile's router rows, one TMA box each.  Warps: 0 TMA producer, 1 MMA
// issuer (TMEM allocator), 2..9 epilogue (two warps per TMEM lane quarter, 64
// columns each).  Two TMEM buffers of 128 columns alternate between chunks.
// Bounded waits throughout.
#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {
namespace {

constexpr int rBM = 128, rBN = 128, rBK = 64, rNS = 3;
constexpr int rATile = rBM * rBK * 2;           // 16 KB: u
constexpr int rBTile = rBN * rBK * 2;           // 16 KB per term
constexpr int rStage = rATile + 3 * rBTile;     // 64 KB
constexpr int rSmem = 1024 + rNS * rStage + 256;
constexpr int rThreads = 320;
constexpr uint32_t rTmemCols = 256;

__global__ void __launch_bounds__(rThreads, 1)
    k_router_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const float* __restrict__ inv_rms, int Tn, int d, int E, int splits,
                float* __restrict__ part, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + rNS * rStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + rNS;
  uint64_t* tfull = bars + 2 * rNS;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = (int)warp_id(), lane = (int)lane_id();
  const int mt_n = (Tn + rBM - 1) / rBM, nt_n = (E + rBN - 1) / rBN;
  const int nchunks = d / rBK, cps = nchunks / splits;
  const int total = mt_n * nt_n * splits;
  if ((int)blockIdx.x >= total) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < rNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 256);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, rTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int w = blockIdx.x; w < total && !*abort_flag; w += gridDim.x) {
        const int s = w % splits, nt = (w / splits) % nt_n, mt = w / (splits * nt_n);
        for (int c = s * cps; c < (s + 1) * cps; ++c) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, status, abort_flag)) break;
          uint8_t* st = smem + stage * rStage;
          mbar_expect_tx(&full[stage], rStage);
          tma_load_2d(st, &tmA, c * rBK, mt * rBM, &full[stage], pol);
#pragma unroll
          for (int term = 0; term < 3; ++term)  // the term blocks are E rows apart
            tma_load_2d(st + rATile + term * rBTile, &tmB, c * rBK, term * E + nt * rBN,
                        &full[stage], pol);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == rNS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < rNS; ++s)
          if ((issued >> s) & 1u) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(&full[s], (issued_par >> s) & 1u))
              if (global_ns() - t0 > kWaitLimitNs) break;
          }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(rBM, rBN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t chunk = 0;  // running chunk count: buffer and parity
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        for (int c = 0; c < cps; ++c, ++chunk) {
          const uint32_t buf = chunk & 1u, bpar = (chunk >> 1) & 1u;
          if (!mbar_wait(&tempty[buf], bpar ^ 1u, status, abort_flag) ||
              !mbar_wait(&full[stage], phase, status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * rStage);
          const uint32_t b0 = a0 + rATile;
          const uint32_t dcol = tmem + buf * (uint32_t)rBN;
          // smallest term first: the accumulator stays small while the low
          // terms are added
#pragma unroll
          for (int ti = 0; ti < 3; ++ti)
#pragma unroll
            for (int kk = 0; kk < rBK / 16; ++kk)
              mma_bf16(dcol, sw128_kmajor_desc(a0 + kk * 32),
                       sw128_kmajor_desc(b0 + (2 - ti) * rBTile + kk * 32), idesc,
                       (ti | kk) != 0);
          mma_commit(&empty[stage]);
          mma_commit(&tfull[buf]);
          if (++stage == rNS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      mma_commit(drain);
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(drain, 0))
        if (global_ns() - t0 > kWaitLimitNs) break;
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int ew = warp - 2;               // 0..7
    const int q = warp & 3;                // TMEM lane quarter of this warp
    const int half = ew >> 2;              // columns [64 half, 64 half + 64)
    const int row = q * 32 + lane;
    uint32_t chunk = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const int s = w % splits, nt = (w / splits) % nt_n, mt = w / (splits * nt_n);
      float acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.f;
      bool ok = true;
      for (int c = 0; c < cps; ++c, ++chunk) {
        const uint32_t buf = chunk & 1u, bpar = (chunk >> 1) & 1u;
        if (!mbar_wait(&tfull[buf], bpar, status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + buf * (uint32_t)rBN + half * 64;
        float v[4][16];
#pragma unroll
        for (int g = 0; g < 4; ++g) tmem_ld16(tb + g * 16, v[g]);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[g * 16 + j] += v[g][j];
        tc_fence_before();
        mbar_arrive(&tempty[buf]);
      }
      if (!ok) break;
      const int t = mt * rBM + row;
      const int e0 = nt * rBN + half * 64;
      if (t < Tn) {
        const float r = inv_rms[t];
        float* out = part + ((size_t)s * Tn + t) * E;
        if (e0 + 64 <= E && (E % 4) == 0) {
#pragma unroll
          for (int j = 0; j < 64; j += 4)
            *reinterpret_cast<float4*>(out + e0 + j) =
                make_float4(r * acc[j], r * acc[j + 1], r * acc[j + 2], r * acc[j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (e0 + j < E) out[e0 + j] = r * acc[j];
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, rTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool rmap(CUtensorMap* mp, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
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
  cuuint32_t box[2] = {(cuuint32_t)rBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int router_tc_splits(int T, int d, int E, int num_sms) {
  const int tiles = cdiv(T, rBM) * cdiv(E, rBN);
  const int nchunks = d / rBK;
  int s = 1;
  while (s * 2 <= nchunks && tiles * s < num_sms && (nchunks % (s * 2)) == 0 && s < 16) s *= 2;
  return s;
}

cudaError_t launch_router_tc(const void* u, const float* inv_rms, const void* w3, int T, int d,
                             int E, int splits, float* part, uint32_t* status, int num_sms,
                             cudaStream_t s) {
  CUtensorMap ma, mb;
  if (!rmap(&ma, u, (uint64_t)T, (uint64_t)d, rBM) ||
      !rmap(&mb, w3, (uint64_t)3 * E, (uint64_t)d, rBN))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e =
        cudaFuncSetAttribute(k_router_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, rSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int items = cdiv(T, rBM) * cdiv(E, rBN) * splits;
  const int grid = items < num_sms ? items : num_sms;
  k_router_tc<<<grid, rThreads, rSmem, s>>>(ma, mb, inv_rms, T, d, E, splits, part, status);
  return cudaGetLastError();
}

}  // namespace ace
