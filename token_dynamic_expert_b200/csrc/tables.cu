// tables.cu -- offline construction of ACE's per-expert tables on B200.
//
// Global Spectral Proxy ([ACE] "Methodology 1"):
//   a^up   = ||Gamma W^up|| ||Gamma W^gate W^down||
//   a^gate = ||Gamma W^gate|| ||Gamma W^up W^down||
//   A^GSP(e) = sqrt(a^up a^gate)_e / (mean_j sqrt(a^up a^gate)_j + eps)
// The Frobenius norms come from m x m Gram matrices built on tcgen05 tensor
// cores (K = d contractions, fp32 accumulate):
//   G_g = W_g Gamma^2 W_g^T,  G_u = W_u Gamma^2 W_u^T   (W_* stored [m][d])
//   D   = W^down (W^down)^T                              (page orientation)
//   ||Gamma W||_F^2 = tr(G),  ||Gamma W W^down||_F^2 = <G, D>  (trace identity)
// Gamma^2 W is not exactly bf16, so it enters as a two-term bf16 split
// (hi + lo, relative residual below 2^-16) concatenated along K.
// The largest singular values (the constants of the bound on ||f(x)|| in
// [ACE] "Theoretical Foundation", and the spectral GSP variant) come from
// power iteration on the same Grams: from v_0 = 1/sqrt(m), v <- G v/||G v||,
// sigma = sqrt(v^T G v); for a product, v <- G (D v)/||.||, sigma^2 = ||G D v||.
//
// Router-Conditioned Refinement ([ACE] "Methodology 2"):
//   q_e = (w_e - mean_j w_j) / (RMS(w_e - mean_j w_j) + eps) * rho
//   a~_e = ||f_e(q_e)|| / (||q_e|| + eps),  f applies Gamma to q
//   A^RCR(e) = a~_e / (mean_j a~_j + eps)
// by batched GEMVs over every expert's weights.
#include <math.h>

#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {
namespace {

// ------------------------------------------------------ operand preparation
// WdT[b][j][i] = W_down[e0+b][i][j]: the K-major copy of W^down's rows.
__global__ void __launch_bounds__(256) k_transpose_wd(const __nv_bfloat16* __restrict__ wd,
                                                      int e0, int d, int m,
                                                      __nv_bfloat16* __restrict__ wdt) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int b = blockIdx.z;
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const __nv_bfloat16* src = wd + (size_t)(e0 + b) * d * m;
  __nv_bfloat16* dst = wdt + (size_t)b * m * d;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) tile[r][tx] = src[(size_t)(i0 + r) * m + j0 + tx];
  __syncthreads();
  for (int r = ty; r < 32; r += 8) dst[(size_t)(j0 + r) * d + i0 + tx] = tile[tx][r];
}

// Y[b][j][0:d] = hi(gamma^2 * W[e0+b][j][:]),  Y[b][j][d:2d] = lo (the rest).
__global__ void __launch_bounds__(256) k_split_scaled(const __nv_bfloat16* __restrict__ w,
                                                      const float* __restrict__ gamma, int e0,
                                                      int d, int m, __nv_bfloat16* __restrict__ y) {
  const size_t b = blockIdx.y;
  const size_t n = (size_t)m * d;
  const __nv_bfloat16* src = w + (size_t)(e0 + b) * n;
  for (size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x; q < n;
       q += (size_t)gridDim.x * blockDim.x) {
    const int j = (int)(q / d), i = (int)(q % d);
    const float g = gamma[i];
    const float v = __bfloat162float(src[q]) * (g * g);
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    __nv_bfloat16* row = y + (b * m + j) * (size_t)(2 * d);
    row[i] = hi;
    row[d + i] = lo;
  }
}

// -------------------------------------------------------- tcgen05 Gram GEMM
// C[b] (m x m, fp32) = A_b B_b^T over K, A_b rows from map A (row b*a_rows +
// r, column k mod Ka), B_b rows from map B (row b*b_rows + r).  128 x 256
// tiles, 4 stages, double-buffered TMEM accumulator; same warp roles as the
// expert GEMMs (producer, MMA issuer, 4 epilogue warps).
constexpr int gBM = 128, gBN = 256, gBK = 64, gNS = 4;
constexpr int gAStage = gBM * gBK * 2, gBStage = gBN * gBK * 2;
constexpr int gSmem = 1024 + gNS * (gAStage + gBStage) + 256;

__global__ void __launch_bounds__(192, 1)
    k_gram(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           int nbatch, int m, int a_rows, int b_rows, int Ka, int K, float* __restrict__ C,
           uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + gNS * gAStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + gNS * gBStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + gNS;
  uint64_t* tfull = bars + 2 * gNS;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = (int)warp_id(), lane = (int)lane_id();
  const int mt_n = m / gBM, nt_n = (m + gBN - 1) / gBN;
  const int total = nbatch * mt_n * nt_n;
  if ((int)blockIdx.x >= total) return;
  const int ksteps = K / gBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < gNS; ++s) {
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
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int w = blockIdx.x; w < total && !*abort_flag; w += gridDim.x) {
        const int b = w / (mt_n * nt_n), r = w - b * mt_n * nt_n;
        const int mt = r / nt_n, nt = r - mt * nt_n;
        const int arow = b * a_rows + mt * gBM, brow = b * b_rows + nt * gBN;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, status, abort_flag)) break;
          mbar_expect_tx(&full[stage], gAStage + gBStage);
          tma_load_2d(sA + stage * gAStage, &tmA, (kb * gBK) % Ka, arow, &full[stage], pol);
          tma_load_2d(sB + stage * gBStage, &tmB, kb * gBK, brow, &full[stage], pol);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == gNS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < gNS; ++s)
          if ((issued >> s) & 1u) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(&full[s], (issued_par >> s) & 1u))
              if (global_ns() - t0 > kWaitLimitNs) break;
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int r = w % (mt_n * nt_n);
        const int nt = r % nt_n;
        const int ncols = min(gBN, m - nt * gBN);
        const uint32_t idesc = idesc_bf16_f32(gBM, ncols);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d0 = tmem + (uint32_t)acc * 256u;
        for (int kb = 0; kb < ksteps; ++kb) {
          if (!mbar_wait(&full[stage], phase, status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * gAStage);
          const uint32_t b0 = smem_u32(sB + stage * gBStage);
#pragma unroll
          for (int kk = 0; kk < gBK / 16; ++kk)
            mma_bf16(d0, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), idesc,
                     (kb | kk) != 0);
          mma_commit(&empty[stage]);
          if (++stage == gNS) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      mma_commit(drain);
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(drain, 0))
        if (global_ns() - t0 > kWaitLimitNs) break;
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const int b = w / (mt_n * nt_n), r = w - b * mt_n * nt_n;
      const int mt = r / nt_n, nt = r - mt * nt_n;
      const int ncols = min(gBN, m - nt * gBN);
      if (!mbar_wait(&tfull[acc], acc_phase, status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * 256u;
      float* crow = C + ((size_t)b * m + mt * gBM + row) * m + nt * gBN;
      for (int c0 = 0; c0 < ncols; c0 += 16) {
        float v[16];
        tmem_ld16(tbase + (uint32_t)c0, v);
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(crow + c0);
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
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
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------- Gram reductions
__device__ double block_sum_d(double v, double* s_buf) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane == 0) s_buf[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < nw; ++i) t += s_buf[i];
  __syncthreads();
  if (threadIdx.x == 0) s_buf[0] = t;
  __syncthreads();
  t = s_buf[0];
  __syncthreads();
  return t;
}

// stats[e][0..3] = tr(G_g), tr(G_u), <G_g, D>, <G_u, D>  (fp64 sums)
__global__ void __launch_bounds__(1024) k_gram_stats(const float* __restrict__ Gg,
                                                     const float* __restrict__ Gu,
                                                     const float* __restrict__ D, int m, int e0,
                                                     double* __restrict__ stats) {
  __shared__ double s_buf[32];
  const int b = blockIdx.x;
  const size_t off = (size_t)b * m * m, n = (size_t)m * m;
  double tg = 0, tu = 0, pg = 0, pu = 0;
  for (size_t q = threadIdx.x; q < n; q += blockDim.x) {
    const double g = Gg[off + q], u = Gu[off + q], dd = D[off + q];
    pg += g * dd;
    pu += u * dd;
  }
  for (int j = threadIdx.x; j < m; j += blockDim.x) {
    tg += Gg[off + (size_t)j * m + j];
    tu += Gu[off + (size_t)j * m + j];
  }
  tg = block_sum_d(tg, s_buf);
  tu = block_sum_d(tu, s_buf);
  pg = block_sum_d(pg, s_buf);
  pu = block_sum_d(pu, s_buf);
  if (threadIdx.x == 0) {
    double* s = stats + (size_t)(e0 + b) * 8;
    s[0] = tg;
    s[1] = tu;
    s[2] = pg;
    s[3] = pu;
  }
}

// --------------------------------------------------------- power iteration
// Block (b, q) of a batch: q = 0, 1, 2 -> sigma of G_g[b], G_u[b], D[b]
// (sqrt of the dominant eigenvalue, by v <- P v/||P v||, then sqrt(v^T P v));
// q = 3, 4 -> sigma of the products Gamma W_g W^down, Gamma W_u W^down
// (v <- G (D v)/||.||, then sqrt(||G D v||)).  sig[(e0+b)*5 + q].
__global__ void __launch_bounds__(512) k_power(const float* __restrict__ Gg,
                                                const float* __restrict__ Gu,
                                                const float* __restrict__ Dm, int m, int e0,
                                                int iters, float* __restrict__ sig) {
  extern __shared__ float sv[];  // v [m], t [m]
  __shared__ double s_buf[32];
  float* v = sv;
  float* t = sv + m;
  const int b = blockIdx.x, q = blockIdx.y;
  const size_t mm = (size_t)m * m;
  const float* P0 = (q == 0 || q == 3) ? Gg + b * mm : (q == 1 || q == 4) ? Gu + b * mm : Dm + b * mm;
  const float* P1 = q >= 3 ? Dm + b * mm : nullptr;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float v0 = 1.0f / sqrtf((float)m);
  for (int j = threadIdx.x; j < m; j += blockDim.x) v[j] = v0;
  __syncthreads();
  // y = P x: a warp takes two rows at a time and issues all of its 16-byte
  // loads of both rows before the arithmetic (m is a multiple of 128)
  auto matvec = [&](const float* P, const float* x, float* y) {
    const int m4 = m / 4;
    for (int r = 2 * warp; r < m; r += 2 * nw) {
      const float4* r0 = reinterpret_cast<const float4*>(P + (size_t)r * m);
      const float4* r1 = reinterpret_cast<const float4*>(P + (size_t)(r + 1) * m);
      float s0 = 0.f, s1 = 0.f;
      for (int base = 0; base < m4; base += 32 * 8) {
        float4 a0[8], a1[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = base + lane + 32 * i;
          a0[i] = c < m4 ? __ldg(r0 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
          a1[i] = c < m4 ? __ldg(r1 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = base + lane + 32 * i;
          if (c >= m4) continue;
          const float4 xv = reinterpret_cast<const float4*>(x)[c];
          s0 = fmaf(a0[i].x, xv.x, fmaf(a0[i].y, xv.y, fmaf(a0[i].z, xv.z, fmaf(a0[i].w, xv.w, s0))));
          s1 = fmaf(a1[i].x, xv.x, fmaf(a1[i].y, xv.y, fmaf(a1[i].z, xv.z, fmaf(a1[i].w, xv.w, s1))));
        }
      }
      s0 = warp_sum(s0);
      s1 = warp_sum(s1);
      if (lane == 0) {
        y[r] = s0;
        y[r + 1] = s1;
      }
    }
    __syncthreads();
  };
  double nrm = 0.0;
  for (int it = 0; it <= iters; ++it) {
    if (P1) {
      matvec(P1, v, t);  // t = D v
      matvec(P0, t, v);  // v = G t
      for (int j = threadIdx.x; j < m; j += blockDim.x) t[j] = v[j];
      __syncthreads();
    } else {
      matvec(P0, v, t);  // t = P v
    }
    double ss = 0.0;
    for (int j = threadIdx.x; j < m; j += blockDim.x) ss += (double)t[j] * t[j];
    ss = block_sum_d(ss, s_buf);
    nrm = sqrt(ss);
    if (it == iters || nrm == 0.0) break;
    const float inv = (float)(1.0 / nrm);
    for (int j = threadIdx.x; j < m; j += blockDim.x) v[j] = t[j] * inv;
    __syncthreads();
  }
  float out;
  if (P1) {
    out = (float)sqrt(nrm);
  } else {  // ||A v_K||^2 = v_K^T G v_K with t = G v_K (v_K is v unless the loop broke early)
    double vg = 0.0;
    for (int j = threadIdx.x; j < m; j += blockDim.x) vg += (double)v[j] * t[j];
    vg = block_sum_d(vg, s_buf);
    out = nrm == 0.0 ? 0.f : (float)sqrt(fmax(vg, 0.0));
  }
  if (threadIdx.x == 0) sig[(size_t)(e0 + b) * 5 + q] = out;
}

// Gram matrices on CUDA cores for fp32 layers (small shapes):
//   G_g[b][j][j'] = sum_i gamma_i^2 W_g[j][i] W_g[j'][i] (likewise G_u),
//   D[b][j][j'] = sum_i W_d[i][j] W_d[i][j'].
template <typename T>
__global__ void __launch_bounds__(256) k_gram_simt(const T* __restrict__ wg, const T* __restrict__ wu,
                                                   const T* __restrict__ wd,
                                                   const float* __restrict__ gamma, int e0, int d,
                                                   int m, float* __restrict__ Gg,
                                                   float* __restrict__ Gu, float* __restrict__ Dm) {
  const int b = blockIdx.z;
  const int j = blockIdx.y * 16 + (threadIdx.x >> 4), jj = blockIdx.x * 16 + (threadIdx.x & 15);
  if (j >= m || jj >= m) return;
  const size_t e = (size_t)(e0 + b);
  const T* g1 = wg + (e * m + j) * d;
  const T* g2 = wg + (e * m + jj) * d;
  const T* u1 = wu + (e * m + j) * d;
  const T* u2 = wu + (e * m + jj) * d;
  const T* w = wd + e * d * m;
  float sg = 0.f, su = 0.f, sd = 0.f;
  for (int i = 0; i < d; ++i) {
    const float gg = gamma[i] * gamma[i];
    sg = fmaf(to_f(g1[i]) * gg, to_f(g2[i]), sg);
    su = fmaf(to_f(u1[i]) * gg, to_f(u2[i]), su);
    sd = fmaf(to_f(w[(size_t)i * m + j]), to_f(w[(size_t)i * m + jj]), sd);
  }
  const size_t o = ((size_t)b * m + j) * m + jj;
  Gg[o] = sg;
  Gu[o] = su;
  Dm[o] = sd;
}

// ------------------------------------------------------------------- RCR
// q_e, z_e = q_e * gamma (fp32) and ||q_e|| for every expert of the layer.
template <typename T>
__global__ void __launch_bounds__(256) k_rcr_prototype(const T* __restrict__ wr,
                                                       const float* __restrict__ gamma, int E,
                                                       int d, float eps, float rho,
                                                       float* __restrict__ z,
                                                       double* __restrict__ stats) {
  __shared__ double s_buf[32];
  const int e = blockIdx.x;
  double ss = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    double mean = 0.0;
    for (int j = 0; j < E; ++j) mean += (double)to_f(wr[(size_t)j * d + i]);
    mean /= E;
    const double wt = (double)to_f(wr[(size_t)e * d + i]) - mean;
    z[(size_t)e * d + i] = (float)wt;
    ss += wt * wt;
  }
  ss = block_sum_d(ss, s_buf);
  const double rms = sqrt(ss / d);
  const double scale = rho / (rms + eps);
  double qq = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const double q = (double)z[(size_t)e * d + i] * scale;
    qq += q * q;
    z[(size_t)e * d + i] = (float)(q * gamma[i]);
  }
  qq = block_sum_d(qq, s_buf);
  if (threadIdx.x == 0) stats[(size_t)e * 8 + 4] = sqrt(qq);
}

// h[e][j] = SiLU(W_g[e][j] . z_e) * (W_u[e][j] . z_e); one warp per row,
// 16-byte loads.
template <typename T>
__global__ void __launch_bounds__(256) k_rcr_gateup(const T* __restrict__ wg, const T* __restrict__ wu,
                                                    const float* __restrict__ z, int d, int m,
                                                    float* __restrict__ h) {
  constexpr int V = 16 / sizeof(T);
  const int e = blockIdx.y;
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (j >= m) return;
  const uint4* g = reinterpret_cast<const uint4*>(wg + ((size_t)e * m + j) * d);
  const uint4* u = reinterpret_cast<const uint4*>(wu + ((size_t)e * m + j) * d);
  const float* ze = z + (size_t)e * d;
  float a = 0.f, b = 0.f;
  for (int v = lane; v < d / V; v += 32) {
    const uint4 gv = g[v], uv = u[v];
    const T* gp = reinterpret_cast<const T*>(&gv);
    const T* up = reinterpret_cast<const T*>(&uv);
#pragma unroll
    for (int c = 0; c < V; ++c) {
      const float x = ze[v * V + c];
      a = fmaf(to_f(gp[c]), x, a);
      b = fmaf(to_f(up[c]), x, b);
    }
  }
  a = warp_sum(a);
  b = warp_sum(b);
  if (lane == 0) h[(size_t)e * m + j] = a / (1.0f + expf(-a)) * b;
}

// o2[e][blk] = sum over the block's 8 rows i of (W_d[e][i] . h_e)^2.
template <typename T>
__global__ void __launch_bounds__(256) k_rcr_down(const T* __restrict__ wd, const float* __restrict__ h,
                                                  int d, int m, float* __restrict__ o2) {
  constexpr int V = 16 / sizeof(T);
  __shared__ float s_part[8];
  const int e = blockIdx.y;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  float s = 0.f;
  if (i < d) {
    const uint4* w = reinterpret_cast<const uint4*>(wd + ((size_t)e * d + i) * m);
    const float* he = h + (size_t)e * m;
    for (int v = lane; v < m / V; v += 32) {
      const uint4 wv = w[v];
      const T* wp = reinterpret_cast<const T*>(&wv);
#pragma unroll
      for (int c = 0; c < V; ++c) s = fmaf(to_f(wp[c]), he[v * V + c], s);
    }
    s = warp_sum(s);
  }
  if (lane == 0) s_part[threadIdx.x >> 5] = s * s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int q = 0; q < 8; ++q) t += s_part[q];
    o2[(size_t)e * gridDim.x + blockIdx.x] = t;
  }
}

// ---------------------------------------------------------------- finalize
// stats[e]: 0 tr(G_g) 1 tr(G_u) 2 <G_g,D> 3 <G_u,D> 4 ||q|| ; sig[e][0..4]:
// sigma(G_g), sigma(G_u), sigma(D), sigma(G_g D), sigma(G_u D).
__global__ void __launch_bounds__(512) k_finalize(const double* __restrict__ stats,
                                                  const float* __restrict__ o2, int nblk_o,
                                                  const float* __restrict__ sig, int E, int spectral,
                                                  float eps, float* __restrict__ a_gsp,
                                                  float* __restrict__ a_rcr,
                                                  float* __restrict__ amax,
                                                  float* __restrict__ sigma_out) {
  __shared__ double s_buf[32];
  __shared__ double s_gsp[kMaxE], s_rcr[kMaxE];
  double sum_g = 0.0, sum_r = 0.0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const double* s = stats + (size_t)e * 8;
    double up, gate;
    if (spectral) {
      up = (double)sig[e * 5 + 1] * (double)sig[e * 5 + 3];
      gate = (double)sig[e * 5 + 0] * (double)sig[e * 5 + 4];
    } else {
      up = sqrt(fmax(s[1], 0.0)) * sqrt(fmax(s[2], 0.0));
      gate = sqrt(fmax(s[0], 0.0)) * sqrt(fmax(s[3], 0.0));
    }
    const double at = sqrt(up * gate);
    double o = 0.0;
    for (int q = 0; q < nblk_o; ++q) o += (double)o2[(size_t)e * nblk_o + q];
    const double ar = sqrt(o) / (s[4] + eps);
    s_gsp[e] = at;
    s_rcr[e] = ar;
    sum_g += at;
    sum_r += ar;
  }
  sum_g = block_sum_d(sum_g, s_buf);
  sum_r = block_sum_d(sum_r, s_buf);
  const double mg = sum_g / E, mr = sum_r / E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const float g = (float)(s_gsp[e] / (mg + eps));
    const float r = (float)(s_rcr[e] / (mr + eps));
    a_gsp[e] = g;
    a_rcr[e] = r;
    amax[e] = fmaxf(g, r);
    if (sigma_out) {
      sigma_out[e * 3 + 0] = sig[e * 5 + 0];
      sigma_out[e * 3 + 1] = sig[e * 5 + 1];
      sigma_out[e * 3 + 2] = sig[e * 5 + 2];
    }
  }
}

// ----------------------------------------------------------- host helpers
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool map2d(CUtensorMap* mp, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)gBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TabLayout {
  size_t wdt, yg, yu, G, stats, z, h, o2, sig, total;
  int eb;  // experts per batch
};

TabLayout tab_layout(const ace_layer& L) {
  TabLayout t{};
  const size_t d = L.d, m = L.m, E = L.E;
  t.eb = (int)(E < 64 ? E : 64);
  const size_t eb = (size_t)t.eb;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 1024);
    return at;
  };
  take(256);  // status word (offset 0, as in the forward workspace)
  t.wdt = take(eb * m * d * 2);
  t.yg = take(eb * m * 2 * d * 2);
  t.yu = take(eb * m * 2 * d * 2);
  t.G = take(3 * eb * m * m * 4);  // [G_g batch][G_u batch][D batch]
  t.stats = take(E * 8 * 8);
  t.z = take(E * d * 4);
  t.h = take(E * m * 4);
  t.o2 = take(E * (d / 8) * 4);
  t.sig = take(E * 5 * 4);
  t.total = off;
  return t;
}

}  // namespace

size_t tables_workspace_size(const ace_layer& L) { return tab_layout(L).total; }

ace_status build_tables_impl(const ace_layer* layers, int n_layers, const ace_table_opts& o,
                             float* a_gsp, float* a_rcr, float* amax, float* sigma, void* ws,
                             size_t ws_bytes, cudaStream_t s) {
  const ace_layer& L0 = layers[0];
  const TabLayout t = tab_layout(L0);
  if (ws_bytes < t.total) return ACE_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(w);
  if (cudaMemsetAsync(status, 0, 4, s) != cudaSuccess) return ACE_ERR_CUDA;
  const bool bf16 = L0.dtype == ACE_BF16;
  if (bf16) {
    static bool attr = false;
    if (!attr) {
      if (cudaFuncSetAttribute(k_gram, cudaFuncAttributeMaxDynamicSharedMemorySize, gSmem) !=
          cudaSuccess)
        return ACE_ERR_CUDA;
      attr = true;
    }
  }
  const int d = L0.d, m = L0.m, E = L0.E, eb = t.eb;
  const int num_sms = device_sm_count();
  const bool spectral = o.gsp_norm == ACE_GSP_SPECTRAL;
  const int nq = spectral ? 5 : (sigma ? 3 : 0);  // power iterations per expert
  __nv_bfloat16* wdt = reinterpret_cast<__nv_bfloat16*>(w + t.wdt);
  __nv_bfloat16* yg = reinterpret_cast<__nv_bfloat16*>(w + t.yg);
  __nv_bfloat16* yu = reinterpret_cast<__nv_bfloat16*>(w + t.yu);
  float* Gg = reinterpret_cast<float*>(w + t.G);
  float* Gu = Gg + (size_t)eb * m * m;
  float* Dm = Gu + (size_t)eb * m * m;
  double* stats = reinterpret_cast<double*>(w + t.stats);
  float* z = reinterpret_cast<float*>(w + t.z);
  float* h = reinterpret_cast<float*>(w + t.h);
  float* o2 = reinterpret_cast<float*>(w + t.o2);
  float* sig = reinterpret_cast<float*>(w + t.sig);

  for (int l = 0; l < n_layers; ++l) {
    const ace_layer& L = layers[l];
    // ---- GSP: Gram matrices per batch of experts, their traces and inner
    // products, and the power iterations
    for (int e0 = 0; e0 < E; e0 += eb) {
      const int nb = (E - e0) < eb ? (E - e0) : eb;
      if (bf16) {
        k_transpose_wd<<<dim3(m / 32, d / 32, nb), 256, 0, s>>>(
            (const __nv_bfloat16*)L.w_down, e0, d, m, wdt);
        k_split_scaled<<<dim3(256, nb), 256, 0, s>>>((const __nv_bfloat16*)L.w_gate, L.gamma, e0,
                                                      d, m, yg);
        k_split_scaled<<<dim3(256, nb), 256, 0, s>>>((const __nv_bfloat16*)L.w_up, L.gamma, e0,
                                                      d, m, yu);
        if (cudaGetLastError() != cudaSuccess) return ACE_ERR_CUDA;
        CUtensorMap ma_g, mb_g, ma_u, mb_u, ma_d, mb_d;
        const __nv_bfloat16* wg0 = (const __nv_bfloat16*)L.w_gate + (size_t)e0 * m * d;
        const __nv_bfloat16* wu0 = (const __nv_bfloat16*)L.w_up + (size_t)e0 * m * d;
        if (!map2d(&ma_g, wg0, (uint64_t)nb * m, d, gBM) ||
            !map2d(&mb_g, yg, (uint64_t)nb * m, 2 * d, gBN) ||
            !map2d(&ma_u, wu0, (uint64_t)nb * m, d, gBM) ||
            !map2d(&mb_u, yu, (uint64_t)nb * m, 2 * d, gBN) ||
            !map2d(&ma_d, wdt, (uint64_t)nb * m, d, gBM) ||
            !map2d(&mb_d, wdt, (uint64_t)nb * m, d, gBN))
          return ACE_ERR_CUDA;
        const int tiles = nb * (m / gBM) * ((m + gBN - 1) / gBN);
        const int grid = tiles < num_sms ? tiles : num_sms;
        // G = W (hi + lo)^T: A = W used for both halves of K (column k mod d)
        k_gram<<<grid, 192, gSmem, s>>>(ma_g, mb_g, nb, m, m, m, d, 2 * d, Gg, status);
        k_gram<<<grid, 192, gSmem, s>>>(ma_u, mb_u, nb, m, m, m, d, 2 * d, Gu, status);
        k_gram<<<grid, 192, gSmem, s>>>(ma_d, mb_d, nb, m, m, m, d, d, Dm, status);
      } else {
        k_gram_simt<float><<<dim3(cdiv(m, 16), cdiv(m, 16), nb), 256, 0, s>>>(
            (const float*)L.w_gate, (const float*)L.w_up, (const float*)L.w_down, L.gamma, e0, d,
            m, Gg, Gu, Dm);
      }
      k_gram_stats<<<nb, 1024, 0, s>>>(Gg, Gu, Dm, m, e0, stats);
      if (nq > 0)
        k_power<<<dim3(nb, nq), 512, 2 * m * sizeof(float), s>>>(Gg, Gu, Dm, m, e0,
                                                                 o.power_iters, sig);
      if (cudaGetLastError() != cudaSuccess) return ACE_ERR_CUDA;
    }
    // ---- RCR: prototypes, then f(q) by batched GEMVs
    if (bf16) {
      k_rcr_prototype<__nv_bfloat16><<<E, 256, 0, s>>>((const __nv_bfloat16*)L.w_router, L.gamma,
                                                       E, d, o.eps, o.rho, z, stats);
      k_rcr_gateup<__nv_bfloat16><<<dim3(cdiv(m, 8), E), 256, 0, s>>>(
          (const __nv_bfloat16*)L.w_gate, (const __nv_bfloat16*)L.w_up, z, d, m, h);
      k_rcr_down<__nv_bfloat16><<<dim3(d / 8, E), 256, 0, s>>>((const __nv_bfloat16*)L.w_down,
                                                               h, d, m, o2);
    } else {
      k_rcr_prototype<float><<<E, 256, 0, s>>>((const float*)L.w_router, L.gamma, E, d, o.eps,
                                               o.rho, z, stats);
      k_rcr_gateup<float><<<dim3(cdiv(m, 8), E), 256, 0, s>>>(
          (const float*)L.w_gate, (const float*)L.w_up, z, d, m, h);
      k_rcr_down<float><<<dim3(d / 8, E), 256, 0, s>>>((const float*)L.w_down, h, d, m, o2);
    }
    k_finalize<<<1, 512, 0, s>>>(stats, o2, d / 8, sig, E, spectral ? 1 : 0, o.eps,
                                 a_gsp + (size_t)l * E, a_rcr + (size_t)l * E,
                                 amax + (size_t)l * E, sigma ? sigma + (size_t)l * E * 3 : nullptr);
    if (cudaGetLastError() != cudaSuccess) return ACE_ERR_CUDA;
  }
  return ACE_OK;
}

}  // namespace ace
