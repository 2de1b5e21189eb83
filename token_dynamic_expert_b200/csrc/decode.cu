// decode.cu -- the ACE MoE layer forward for a handful of tokens (T <= 8).
//
// At decode sizes the layer is bound by reading the weights of the experts
// that survive skipping ([ExFold] abstract: decode is limited by the memory
// traffic of the activated experts), so one persistent cooperative kernel
// streams exactly those bytes once, spread over every SM:
//   phase A  x = RMSNorm(u) * gamma into shared memory (the warp of token t
//            normalises its row), router logits, one warp per expert spread
//            over the CTAs (its weight row fetched before x is ready)
//   -- grid barrier --
//   phase B  every CTA, redundantly: top-k, gates, ACE scores and the skip
//            mask ([ACE] "3. Conservative Fusion", top-1 always kept), the
//            kept slots sorted by (expert, token), the distinct experts
//   phase C  gate/up ([ACE] eq. f): the surviving (expert, row) pairs, in
//            stages of 4 row pairs dealt round robin to the CTAs, stream
//            through a shared-memory ring by bulk copies issued from a
//            producer warp; each ring slot has 2-3 fixed compute warps that
//            split the hidden size and form, on the tensor cores, the dots of
//            every token with the stage's 8 rows, then write
//            h = SiLU(x W^gate) (.) x W^up for the tokens that kept the
//            expert; once the ring drains, the first W^down stages of phase D
//            are issued
//   -- grid barrier --
//   phase D  down + combine: the CTA's output rows of every surviving
//            expert's W^down, with the h rows of the expert's kept slots,
//            stream through the ring; each slot's warps form h W^down on the
//            tensor cores and add g * (h W^down) into per-warp sums, which
//            are added in warp order at the end
// The grid barrier is a generation counter in the workspace with a bounded
// spin; the launch is cooperative so every CTA is resident.  Every mbarrier
// wait is bounded as well.  Numerics follow the prefill path: fp32 router on
// the unrounded x, experts on bf16(x), h rounded to bf16, fp32 sums.
#include <limits.h>
#include <math.h>

#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {
namespace {

constexpr int kCompWarps = 16;                      // compute warps
constexpr int kDecThreads = (kCompWarps + 1) * 32;  // + one producer warp
constexpr int kRing = 6;                            // most stages of the phase-C ring
constexpr int kRingD = 8;                           // most stages of the phase-D ring
constexpr int kSmemBudget = 226 * 1024;             // dynamic + static shared memory
constexpr int kStagePairs = 4;                      // (gate, up) row pairs per phase-C stage
constexpr int kStageRows = 2 * kStagePairs;         // staged rows: 4 gate, then 4 up
constexpr int kMaxSlots = kDecodeMaxT * kMaxK;

// Bytes between the rows of bf16(x) and between the staged weight rows of a
// phase-C stage: 2d + 64.  The hidden size is a multiple of 128, so 2d is a
// multiple of 256 and the padding puts rows n and n + 1 64 bytes apart modulo
// 128: the 16-byte loads of a quarter warp (two rows, four consecutive
// 16-byte pieces of each) then hit distinct banks.
__host__ __device__ constexpr int row_stride(int d) { return 2 * d + 64; }
// A phase-C stage (rows j0 .. j0 + 3 of W^gate and W^up) is four groups of
// two consecutive rows, one bulk copy each: gate j0, j0 + 1 | gate j0 + 2,
// j0 + 3 | up j0, j0 + 1 | up j0 + 2, j0 + 3, the groups 4d + 64 bytes apart.
// MMA column n (0 .. 7) is group 2 (n >> 2) + (n & 1), row (n >> 1) & 1 of
// it, i.e. gate pairs 0, 2, 1, 3 then up pairs 0, 2, 1, 3: the columns that a
// quarter warp reads together (n even, n + 1) are one group apart, 64 bytes
// modulo 128, so their 16-byte loads hit distinct banks.
__host__ __device__ constexpr int group_stride(int d) { return 4 * d + 64; }
__host__ __device__ constexpr int col_offset(int n, int d) {
  return ((n >> 2) * 2 + (n & 1)) * group_stride(d) + ((n >> 1) & 1) * 2 * d;
}
constexpr int kStageBytes = 4 * group_stride(2048);  // bytes per ring slot (d <= 2048)
// Phase C splits the hidden size of a stage over at most kPartsC warps; the
// partial dots of parts 1 .. kPartsC - 1 meet part 0 in shared memory, two
// buffers per slot (by fill parity)
constexpr int kPartsC = 3;
constexpr int kPartBytes = kRing * 2 * (kPartsC - 1) * 32 * 8;
// Phase D splits the expert size of a stage over at most kPartsD warps
constexpr int kPartsD = 4;

struct DecodeArgs {
  const float* gamma;
  const __nv_bfloat16* wr;
  const float* bias;
  const __nv_bfloat16* wg;
  const __nv_bfloat16* wu;
  const __nv_bfloat16* wd;
  FuseTables ft;
  const __nv_bfloat16* u;
  __nv_bfloat16* y;
  int T, d, E, m, k;
  float tau, eps_rms;
  int renorm;
  float* logits;          // [T][E]
  __nv_bfloat16* h;       // [T*k][m]
  int32_t* idx;           // [T][k]
  float* gate;            // [T][k]
  float* score;           // [T][k]
  uint8_t* keep;          // [T][k]
  int32_t* offsets;       // [E+1]
  int32_t* slot_token;    // [T*k]
  int32_t* slot_rank;     // [T*k]
  int32_t* slot_of;       // [T][k]
  int32_t* n_kept;        // [1]
  uint32_t* sync;             // [16] the launch epoch and its cross-CTA counters
  uint32_t* status;           // the call's status word (written at the end)
  int keep_status;            // add the flags to the status word, else replace it
  unsigned long long* trace;  // optional [grid][8] phase stamps
  uint64_t peer_wait_ns;      // limit of a grid-barrier wait
  int nring;                  // stages of the copy ring for this call
  int region;                 // byte offset of the region after the ring
  int part_off;               // byte offset of phase C's partial dots
  size_t dyn_bytes;           // dynamic shared memory of the launch
};

struct DecShared {
  uint64_t full_c[kRing], empty_c[kRing], full_d[kRingD], empty_d[kRingD];
  int n_slots;                 // kept slots
  int n_uexp;                  // distinct experts among them
  int slot_e[kMaxSlots];
  int slot_t[kMaxSlots];
  int slot_r[kMaxSlots];
  float slot_g[kMaxSlots];
  int uexp[kMaxSlots];         // distinct experts, ascending
  int ufirst[kMaxSlots + 1];   // first slot of each distinct expert
  int t_idx[kMaxSlots];        // per (token, rank): expert, gate, score, keep, slot
  float t_gate[kMaxSlots];
  float t_score[kMaxSlots];
  int t_keep[kMaxSlots];
  int t_pos[kMaxSlots];
  uint32_t tok_mask[kMaxE];    // per expert: bit t set when token t kept a slot of it
  float fac[kMaxE];            // per expert: the fused table factor F(A^GSP, A^RCR)
  int e_base[kMaxE];           // per expert: its first slot
  uint64_t in_bar;             // phase A: u, gamma and the router rows have landed
  int slot_stage[kRing];       // phase C: the stage a ring slot holds (-1: no more)
  int abort;
  uint32_t flags;              // ACE_FLAG_* bits this CTA raised
  uint32_t epoch;              // the launch's epoch (word 0 of the sync words)
  int fast;                    // the sync words are marked clean for this epoch
  // bulk copies the producer issued, so that a CTA leaving early lets them land
  int n_c_issued;              // phase-C stages (ring slot = stage % nring)
  int n_c_marked;              // phase-C end marks after them (one more phase per slot)
  int n_d_issued;              // phase-D W^down stages (ring slot = expert % nring_d)
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// global -> shared bulk copy completing `bytes` of transaction on `bar`
// (addresses 16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// the same, with an L2 eviction-priority policy for the copied lines
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Expert weights are read once per call: their lines go first when L2 needs
// room, so they do not push out what the call reads again (h, the logits,
// the tables, the kernel's code)
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void stamp(const DecodeArgs& a, int i) {
  if (a.trace && threadIdx.x == 0) a.trace[blockIdx.x * 8 + i] = global_ns();
}

// Cross-CTA words of a launch (sync: 16 words in the caller's workspace).
//   word 0      the launch epoch e
//   word 1      e ^ kCleanMark when words 2-4 are clean (zero)
//   words 2-4   arrivals, departures and raised flags (fast path)
//   words 6-11  the same as 64-bit words tagged with e ^ kTagMark in the
//               high half (slow path)
// The last CTA to depart writes the launch's flags into the status word,
// zeroes words 2-4, and marks them clean for epoch e + 1.  So the words need
// no clearing before a launch (nor a kernel to clear them: inside a CUDA
// graph that node costs about a microsecond per layer), and a launch that gave
// up part way through still leaves them clean.  A workspace whose words were
// never written (or were cleared, or hold anything else) lacks the mark; every
// CTA reads the mark before any CTA writes a word, so they all take the slow
// path, where the first CTA to touch a word whose tag is not this launch's
// re-tags it with a zero count.  A uniform fill (all zero or all ones bytes)
// can match neither mark; other garbage matches one with odds 2^-32.
constexpr uint32_t kCleanMark = 0x5bd1e995u;
constexpr uint32_t kTagMark = 0x9e3779b9u;

__device__ __forceinline__ uint32_t ld_acquire32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t add_acq_rel32(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ uint32_t add_release32(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.release.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ uint64_t ld_acquire64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t ld_relaxed64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t cas_acq_rel64(uint64_t* p, uint64_t cmp, uint64_t val) {
  uint64_t old;
  asm volatile("atom.acq_rel.gpu.global.cas.b64 %0, [%1], %2, %3;"
               : "=l"(old) : "l"(p), "l"(cmp), "l"(val) : "memory");
  return old;
}
__device__ __forceinline__ uint64_t add_acq_rel64(uint64_t* p, uint64_t v) {
  uint64_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
__device__ __forceinline__ bool tagged(uint64_t v, uint32_t e) {
  return (uint32_t)(v >> 32) == (e ^ kTagMark);
}
__device__ __forceinline__ uint64_t tag_of(uint32_t e) { return (uint64_t)(e ^ kTagMark) << 32; }

// Slow path: adds one to the count of epoch e in word w; returns the count
// before.
__device__ uint32_t epoch_add(uint64_t* w, uint32_t e) {
  uint64_t v = ld_relaxed64(w);
  for (;;) {
    // once tagged e, a word keeps the tag for the rest of the launch
    if (tagged(v, e)) return (uint32_t)add_acq_rel64(w, 1ull);
    const uint64_t seen = cas_acq_rel64(w, v, tag_of(e) | 1ull);
    if (seen == v) return 0u;
    v = seen;
  }
}

// Slow path: ORs `bits` into the flags of epoch e in word w.
__device__ void epoch_or(uint64_t* w, uint32_t e, uint32_t bits) {
  uint64_t v = ld_relaxed64(w);
  for (;;) {
    const uint64_t want = tag_of(e) | ((tagged(v, e) ? (uint32_t)v : 0u) | bits);
    if (want == v) return;
    const uint64_t seen = cas_acq_rel64(w, v, want);
    if (seen == v) return;
    v = seen;
  }
}

// Called once by thread 0 of every CTA as it leaves (normally or after a
// failed wait), when the CTA's flags are final and it touches no more
// cross-CTA word.
__device__ void depart(const DecodeArgs& a, DecShared& sh) {
  uint32_t* w = a.sync;
  uint64_t* w64 = reinterpret_cast<uint64_t*>(a.sync);
  const uint32_t e = sh.epoch;
  bool last;
  if (sh.fast) {
    if (sh.flags) atomicOr(w + 4, sh.flags);
    last = add_acq_rel32(w + 3, 1u) == gridDim.x - 1;
  } else {
    if (sh.flags) epoch_or(w64 + 5, e, sh.flags);
    last = epoch_add(w64 + 4, e) == gridDim.x - 1;
  }
  if (last) {
    // the last CTA out: every other CTA has published its flags and left its
    // barriers
    uint32_t flags;
    if (sh.fast) {
      flags = ld_acquire32(w + 4);
    } else {
      const uint64_t p = ld_acquire64(w64 + 5);
      flags = tagged(p, e) ? (uint32_t)p : 0u;
    }
    if (a.keep_status) {
      if (flags) atomicOr(a.status, flags);
    } else {
      *reinterpret_cast<volatile uint32_t*>(a.status) = flags;
    }
    // (the next launch starts after this one ends, which orders these)
    w[2] = 0u;
    w[3] = 0u;
    w[4] = 0u;
    w[1] = (e + 1u) ^ kCleanMark;
    w[0] = e + 1u;
  }
}

// Grid-wide barrier number `n` (1, 2, ...) over co-resident CTAs: it opens
// when the launch's arrival count reaches n * gridDim.x.  False when the
// bounded wait ran out (ACE_FLAG_TIMEOUT raised) or an earlier wait failed.
__device__ bool grid_barrier(const DecodeArgs& a, DecShared& sh, uint32_t n) {
  __syncthreads();
  if (threadIdx.x == 0 && !sh.abort) {
    const uint32_t e = sh.epoch, target = n * gridDim.x;
    uint32_t* w = a.sync + 2;
    uint64_t* w64 = reinterpret_cast<uint64_t*>(a.sync) + 3;
    const uint32_t before = sh.fast ? add_release32(w, 1u) : epoch_add(w64, e);
    if (before + 1 < target) {
      const uint64_t t0 = global_ns();
      for (;;) {
        bool open;
        if (sh.fast) {
          open = ld_acquire32(w) >= target;
        } else {
          const uint64_t v = ld_acquire64(w64);
          open = tagged(v, e) && (uint32_t)v >= target;
        }
        if (open) break;
        if (global_ns() - t0 > a.peer_wait_ns) {
          raise_flag(&sh.flags, ACE_FLAG_TIMEOUT);
          sh.abort = 1;
          break;
        }
      }
    }
  }
  __syncthreads();
  return !sh.abort;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const DecodeArgs& a,
                                         DecShared& sh) {
  return mbar_wait(bar, parity, &sh.flags, &sh.abort);
}

// Waits (fixed limit) until the last fill of every ring slot that received
// one has landed: n fills went to slots f % nring, fill f completing the
// slot's phase f / nring.
__device__ void drain_ring(uint64_t* full, int nring, int n) {
  for (int f = n - nring > 0 ? n - nring : 0; f < n; ++f) mbar_drain(&full[f % nring], (f / nring) & 1);
}

// Called by the producer thread before the CTA leaves: every bulk copy it
// issued has landed, so none writes shared memory after the CTA is gone.
__device__ void drain_copies(DecShared& sh, int nring, int nring_d) {
  // phase C: stages, then end marks (no bytes; they complete on arrival) as
  // the slots' last fills, so the waited parities are those of the last phases
  drain_ring(sh.full_c, nring, sh.n_c_issued + sh.n_c_marked);
  drain_ring(sh.full_d, nring_d, sh.n_d_issued);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& q, float (&f)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(p[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

__device__ __forceinline__ void lds8(const float* p, float (&f)[8]) {
  const float4 a0 = reinterpret_cast<const float4*>(p)[0];
  const float4 a1 = reinterpret_cast<const float4*>(p)[1];
  f[0] = a0.x; f[1] = a0.y; f[2] = a0.z; f[3] = a0.w;
  f[4] = a1.x; f[5] = a1.y; f[6] = a1.z; f[7] = a1.w;
}

__device__ __forceinline__ float silu(float a) { return a / (1.0f + expf(-a)); }

// c += A * B for one m16n8k16 tile, bf16 operands, fp32 accumulators; A's
// rows 8 .. 15 are zero (fragments a1, a3), so c[2], c[3] stay zero
__device__ __forceinline__ void mma_bf16_m16n8k16(float (&c)[4], uint32_t a0, uint32_t a2,
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}



// c += A * B for one m16n8k16 tile, bf16 operands, fp32 accumulators, all
// sixteen rows of A
__device__ __forceinline__ void mma_bf16_m16n8k16_full(float (&c)[4], uint32_t a0, uint32_t a1,
                                                       uint32_t a2, uint32_t a3, uint32_t b0,
                                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Named barrier `id` over `count` threads that also ANDs `v` over them: every
// participant gets the same answer, so a group of warps can leave a loop
// together.
__device__ __forceinline__ bool bar_red_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// Phase-D geometry of a CTA with `rows` output rows (the same on the host,
// which sizes shared memory, and in the kernel): a stage holds the rows of
// one expert's W^down and the h rows of its kept slots (at most T)
__host__ __device__ inline size_t dstage_bytes(int rows, int T, int m) {
  return ((size_t)rows * m * 2 + (size_t)T * m * 2 + 1023) & ~(size_t)1023;
}
// per-warp sums of phase D: [warp][16 rows][T tokens] fp32
__host__ __device__ constexpr size_t dacc_bytes(int T) { return (size_t)kCompWarps * 16 * T * 4; }

// NT = the call's token count.
template <int NT>
__global__ void __launch_bounds__(kDecThreads, 1) k_decode(const DecodeArgs a) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ DecShared sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d, E = a.E, m = a.m, k = a.k;
  const int G = gridDim.x;
  const bool producer = warp == kCompWarps;
  const int nring = a.nring;
  uint8_t* ring = dsm;
  // phase A lives inside the ring: the unrounded x (fp32), then the staged
  // inputs u (bf16), gamma (fp32) and the CTA's router rows (bf16)
  float* xf = reinterpret_cast<float*>(dsm);
  __nv_bfloat16* us = reinterpret_cast<__nv_bfloat16*>(dsm + (size_t)NT * d * 4);
  float* gs = reinterpret_cast<float*>(dsm + (size_t)NT * d * 6);
  __nv_bfloat16* wrs = reinterpret_cast<__nv_bfloat16*>(dsm + (size_t)NT * d * 6 + (size_t)d * 4);
  __nv_bfloat16* xb = reinterpret_cast<__nv_bfloat16*>(dsm + a.region);  // bf16(x)
  const int n_router_warps = (E + G - 1) / G;
  // router rows of this CTA: experts blockIdx.x + G * r, r < n_mine
  const int n_mine = (int)blockIdx.x < E ? min(n_router_warps, (E - 1 - (int)blockIdx.x) / G + 1) : 0;
  // phase C: each ring slot has wps_c consumer warps, which split the hidden
  // size of the slot's stages
  const int wps_c = min(kPartsC, kCompWarps / nring);
  // phase D: the CTA's output rows i0 .. i1 - 1 (warp w of a slot's MMA
  // covers all of them, <= 16); each ring slot has wps_d consumer warps,
  // which split the expert size
  const int rows_per_cta = (d + G - 1) / G;
  const int i0 = min(d, (int)blockIdx.x * rows_per_cta), i1 = min(d, i0 + rows_per_cta);
  const int nrows = i1 - i0;
  const uint32_t dbytes = (uint32_t)(nrows * m * 2);
  const size_t dstage = dstage_bytes(nrows, NT, m);
  const int nring_d = (int)min((size_t)kRingD, (a.dyn_bytes - 1024 - dacc_bytes(NT)) / dstage);
  const int wps_d = min(min(kPartsD, kCompWarps / nring_d), m / 32);
  if (threadIdx.x == 0) {
    sh.abort = 0;
    sh.flags = 0u;
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sh.full_c[i], 1);
      mbar_init(&sh.empty_c[i], wps_c);  // the slot's warps
    }
    for (int i = 0; i < kRingD; ++i) {
      mbar_init(&sh.full_d[i], 1);
      mbar_init(&sh.empty_d[i], wps_d);
    }
    mbar_init(&sh.in_bar, 1);
    sh.n_c_issued = sh.n_d_issued = sh.n_c_marked = 0;
    fence_barrier_init();
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh.tok_mask[e] = 0u;
  // The launch may begin while the previous kernel of the stream drains
  // (programmatic stream serialisation): the work above touches shared memory
  // only, and nothing in global memory is read or written before this wait,
  // which returns once that kernel has completed and its writes are visible.
  // The next launch may then be scheduled; its CTAs take an SM only as this
  // launch's CTAs leave (one CTA fills an SM's shared memory).
  grid_dependency_wait();
  if (threadIdx.x == 0) {
    allow_dependent_launch();
    volatile const uint32_t* vs = a.sync;
    sh.epoch = vs[0];
    sh.fast = vs[1] == (sh.epoch ^ kCleanMark);
    // one round trip for every input of phase A
    mbar_expect_tx(&sh.in_bar, (uint32_t)(NT * d * 2 + d * 4 + n_mine * d * 2));
    bulk_g2s(us, a.u, (uint32_t)(NT * d * 2), &sh.in_bar);
    bulk_g2s(gs, a.gamma, (uint32_t)(d * 4), &sh.in_bar);
    for (int r = 0; r < n_mine; ++r)
      bulk_g2s(wrs + (size_t)r * d, a.wr + (size_t)((int)blockIdx.x + G * r) * d,
               (uint32_t)(d * 2), &sh.in_bar);
  }
  stamp(a, 0);
  __syncthreads();  // barrier inits are visible

  // ---------------------------------------------------------- phase A
  // the fused table factors, read while the inputs are in flight (by the
  // last warps, so the token warps start normalising as soon as u lands);
  // phase B then looks them up in shared memory
  for (int e = kDecThreads - 1 - (int)threadIdx.x; e < E; e += kDecThreads)
    sh.fac[e] = fused_factor(a.ft, e);
  const bool in_ok = wait_bar(&sh.in_bar, 0, a, sh);
  if (__syncthreads_or(!in_ok)) {
    if (threadIdx.x == 0) depart(a, sh);
    return;
  }
  if (warp < NT) {  // token warps: x = u / rms(u) * gamma
    const int t = warp;
    const uint4* ur = reinterpret_cast<const uint4*>(us + (size_t)t * d);
    const float4* gp = reinterpret_cast<const float4*>(gs);
    float ss = 0.f;
    for (int v = lane; v < d / 8; v += 32) {
      float f[8];
      bf16x8_to_f32(ur[v], f);
#pragma unroll
      for (int c = 0; c < 8; ++c) ss = fmaf(f[c], f[c], ss);
    }
    ss = warp_sum(ss);
    stamp(a, 7);
    const float r = 1.0f / sqrtf(ss / (float)d + a.eps_rms);
    for (int v = lane; v < d / 8; v += 32) {
      float f[8];
      bf16x8_to_f32(ur[v], f);
      const float4 g0 = gp[2 * v], g1 = gp[2 * v + 1];
      const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      float xv[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) xv[c] = xhat(f[c], r, gg[c]);
      float4* xo = reinterpret_cast<float4*>(xf + t * d + v * 8);
      xo[0] = make_float4(xv[0], xv[1], xv[2], xv[3]);
      xo[1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
      uint4 bq;
      __nv_bfloat16* bp = reinterpret_cast<__nv_bfloat16*>(&bq);
#pragma unroll
      for (int c = 0; c < 8; ++c) bp[c] = __float2bfloat16_rn(xv[c]);
      reinterpret_cast<uint4*>(xb + (size_t)t * (row_stride(d) / 2))[v] = bq;
    }
  }
  __syncthreads();
  stamp(a, 1);
  // router: the (row, token) dots of this CTA's staged rows, one per compute
  // warp (counting down from the last one)
  for (int it = kCompWarps - 1 - warp; warp < kCompWarps && it < n_mine * NT; it += kCompWarps) {
    const int r = it / NT, t = it - r * NT;
    const int my_e = (int)blockIdx.x + G * r;
    const uint4* wrow = reinterpret_cast<const uint4*>(wrs + (size_t)r * d);
    float acc = 0.f;
    for (int v = lane; v < d / 8; v += 32) {
      float w[8], xv[8];
      bf16x8_to_f32(wrow[v], w);
      lds8(xf + t * d + v * 8, xv);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc = fmaf(xv[c], w[c], acc);
    }
    const float sm = warp_sum(acc);
    if (lane == 0) a.logits[(size_t)t * E + my_e] = sm + (a.bias ? a.bias[my_e] : 0.f);
  }
  if (!grid_barrier(a, sh, 1)) {
    if (threadIdx.x == 0) depart(a, sh);
    return;
  }
  stamp(a, 2);

  // ---------------------------------------------------------- phase B
  const int nq = (E + 31) / 32;
  if (warp < NT) {
    const int t = warp;
    float v[kMaxE / 32];
#pragma unroll
    for (int q = 0; q < kMaxE / 32; ++q) {
      const int e = lane + 32 * q;
      v[q] = (q < nq && e < E) ? a.logits[(size_t)t * E + e] : -INFINITY;
    }
    int sel_e = 0;
    float sel_v = -INFINITY;
    topk_select(v, nq, E, k, lane, sel_e, sel_v, &sh.flags);
    const float v0 = __shfl_sync(0xffffffffu, sel_v, 0);
    const float ex = lane < k ? expf(sel_v - v0) : 0.f;
    float denom;
    if (a.renorm) {
      denom = warp_sum(ex);
    } else {
      float z = 0.f;
#pragma unroll
      for (int q = 0; q < kMaxE / 32; ++q)
        if (q < nq) z += (lane + 32 * q < E) ? expf(v[q] - v0) : 0.f;
      denom = warp_sum(z);
    }
    if (lane < k) {
      const float g = ex / denom;
      const float sc = g * sh.fac[sel_e];
      sh.t_idx[t * k + lane] = sel_e;
      sh.t_gate[t * k + lane] = g;
      sh.t_score[t * k + lane] = sc;
      const bool kept = (lane == 0) || !(sc < a.tau);
      sh.t_keep[t * k + lane] = kept;
      if (kept) atomicOr(&sh.tok_mask[sel_e], 1u << t);  // distinct experts per token
    }
  }
  __syncthreads();
  // counting sort of the kept slots by (expert, token): per-expert counts
  // are the popcounts of the token masks; one warp scans them over experts
  // (consecutive experts per lane) into first-slot bases and the list of
  // distinct experts
  const int TK = NT * k;
  if (warp == 0) {
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int cnt = 0, nue = 0;
    for (int e = e0; e < e1; ++e) {
      const uint32_t mk = sh.tok_mask[e];
      cnt += __popc(mk);
      nue += mk != 0u;
    }
    int ci = cnt, ui = nue;  // inclusive scans over lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int c2 = __shfl_up_sync(0xffffffffu, ci, o);
      const int u2 = __shfl_up_sync(0xffffffffu, ui, o);
      if (lane >= o) {
        ci += c2;
        ui += u2;
      }
    }
    int base = ci - cnt, ub = ui - nue;
    for (int e = e0; e < e1; ++e) {
      const uint32_t mk = sh.tok_mask[e];
      sh.e_base[e] = base;
      if (mk != 0u) {
        sh.uexp[ub] = e;
        sh.ufirst[ub] = base;
        ++ub;
      }
      base += __popc(mk);
    }
    if (lane == 31) {
      sh.n_slots = ci;
      sh.n_uexp = ui;
      sh.ufirst[ui] = ci;
    }
  }
  __syncthreads();
  if ((int)threadIdx.x < TK) {
    const int s = threadIdx.x;
    int pos = -1;
    if (sh.t_keep[s]) {
      const int e = sh.t_idx[s], t = s / k;
      pos = sh.e_base[e] + __popc(sh.tok_mask[e] & ((1u << t) - 1u));
      sh.slot_e[pos] = e;
      sh.slot_t[pos] = t;
      sh.slot_r[pos] = s % k;
      sh.slot_g[pos] = sh.t_gate[s];
    }
    sh.t_pos[s] = pos;
  }
  __syncthreads();
  stamp(a, 3);
  const int S = sh.n_slots, U = sh.n_uexp;

  // ---------------------------------------------------------- phase C
  const int P = U * m;  // surviving (expert, row) pairs
  const int n_stages = P / kStagePairs;  // m % 8 == 0: a stage never spans two experts
  const int rs = row_stride(d);
  // phase D's stages (its first ones are filled while phase C ends): the
  // CTA's W^down rows of one surviving expert, then the h rows of that
  // expert's kept slots (consecutive in h); the per-warp sums follow the ring
  uint8_t* ring_d = dsm;
  // stages that lie inside phase C's ring (free once its last stage is
  // consumed), clear of bf16(x) and the partial dots that phase C still reads
  const int n_pre = (nrows > 0 && dstage <= (size_t)a.region)
                        ? min(min(nring_d, U), (int)((size_t)a.region / dstage))
                        : 0;
  if (producer) {
    if (lane == 0) {
      // The CTA's stages are blockIdx.x + G * ls, ls = 0, 1, ...: a fixed
      // round robin (the CTAs' counts differ by one at most), so the issue
      // loop never waits on anything but a free slot.  (A grid-wide counter
      // that hands out stages costs an atomic round trip per stage, which
      // under full DRAM load is longer than a stage's streaming time.)
      int ls = 0;  // this CTA's stages so far
      bool ok = true;
      for (;; ++ls) {
        const int gst = (int)blockIdx.x + G * ls;
        if (gst >= n_stages) break;
        const int slot = ls % nring;
        if (!(ok = wait_bar(&sh.empty_c[slot], ((ls / nring) & 1) ^ 1u, a, sh))) break;
        sh.slot_stage[slot] = gst;
        // rows j0 .. j0 + 3 of W^gate, then of W^up, two rows per copy
        const int pa = gst * kStagePairs, ui = pa / m, j0 = pa - ui * m;
        const size_t off = ((size_t)sh.uexp[ui] * m + j0) * d;
        mbar_expect_tx(&sh.full_c[slot], (uint32_t)(kStageRows * d * 2));
        uint8_t* sg = ring + (size_t)slot * kStageBytes;
        const int gsz = group_stride(d);
        const uint64_t pol = evict_first_policy();
        bulk_g2s_hint(sg, a.wg + off, (uint32_t)(d * 4), &sh.full_c[slot], pol);
        bulk_g2s_hint(sg + gsz, a.wg + off + 2 * (size_t)d, (uint32_t)(d * 4), &sh.full_c[slot], pol);
        bulk_g2s_hint(sg + 2 * gsz, a.wu + off, (uint32_t)(d * 4), &sh.full_c[slot], pol);
        bulk_g2s_hint(sg + 3 * gsz, a.wu + off + 2 * (size_t)d, (uint32_t)(d * 4), &sh.full_c[slot],
                      pol);
      }
      sh.n_c_issued = ls;
      // End marks: the next fill of every slot carries stage -1 and no bytes
      // (a plain arrival completes its phase), so each slot's warps learn that
      // there is no more.  A slot is marked once its last stage is consumed;
      // after the marks every phase-C stage is consumed.
      for (int j = 0; j < nring && ok; ++j) {
        const int lsj = ls + j, slot = lsj % nring;
        if (!(ok = wait_bar(&sh.empty_c[slot], ((lsj / nring) & 1) ^ 1u, a, sh))) break;
        sh.slot_stage[slot] = -1;
        mbar_arrive(&sh.full_c[slot]);
        sh.n_c_marked = j + 1;
      }
      if (ok && n_pre > 0) {
        // the first W^down stages go into the drained ring
        for (int ui = 0; ui < n_pre && ok; ++ui) {
          // the stage's h rows follow after the second grid barrier, on the
          // same phase of the barrier
          const uint32_t hb = (uint32_t)((sh.ufirst[ui + 1] - sh.ufirst[ui]) * m * 2);
          mbar_expect_tx(&sh.full_d[ui], dbytes + hb);
          bulk_g2s_hint(ring_d + (size_t)ui * dstage, a.wd + ((size_t)sh.uexp[ui] * d + i0) * m,
                        dbytes, &sh.full_d[ui], evict_first_policy());
          sh.n_d_issued = ui + 1;
        }
      }
    }
  } else {
    // Each ring slot has wps_c fixed consumer warps (parts), which take its
    // fills in order (fill f of slot s is the CTA's stage f * nring + s) until
    // an end mark: a warp only ever waits for the next phase of its own slot,
    // so no wait can see an older phase, and waiting warps sleep in the
    // barrier instead of polling.  Part p forms, on the tensor cores
    // (m16n8k16, bf16 operands, fp32 accumulation), the dots of the call's
    // tokens (MMA rows; rows NT .. 15 are zero) with the stage's 8 rows (MMA
    // columns: 4 gate, 4 up) over its share of the hidden size, 32-wide
    // blocks b0 .. b1 - 1.  In each block, lane (g, q) holds the elements
    // 8q .. 8q + 7 of token g's bf16(x) and of the row of column g; the block's two
    // MMAs take elements 8q + {0..3} and 8q + {4..7} as the k of their
    // fragments, the same permutation of the block's 32 k on both operands,
    // so each MMA sums exact products of matching elements.  Parts 1, 2 leave
    // their dots in shared memory; after a named barrier over the slot's
    // warps (which also tells every part whether to go on), part 0 adds them
    // in part order and writes h = SiLU(gate) * up for the tokens that kept
    // the stage's expert.
    const int slot = warp / wps_c, part = warp % wps_c;
    const int g = lane >> 2, q = lane & 3;
    const int nblk = d / 32;
    const int b0 = part * nblk / wps_c, b1 = (part + 1) * nblk / wps_c;
    const uint8_t* xrow = reinterpret_cast<const uint8_t*>(xb) + (size_t)g * rs + 16 * q;
    float2* partial = reinterpret_cast<float2*>(dsm + a.part_off);  // [kRing][2][kPartsC - 1][32]
    if (slot < nring) {
      for (int f = 0;; ++f) {
        // lane 0 waits (bounded); once the phase is complete every lane takes
        // its acquire with one test (the phase stays complete until all of
        // the slot's warps release it)
        int ok = 1;
        if (lane == 0) ok = wait_bar(&sh.full_c[slot], f & 1, a, sh);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        int gst = -1;
        if (ok) {
          mbar_try_wait(&sh.full_c[slot], f & 1);
          gst = sh.slot_stage[slot];
        }
        const bool go = ok && gst >= 0;  // (gst < 0: end mark)
        float d0 = 0.f, d1 = 0.f;
        if (go) {
          const uint8_t* wrow = ring + (size_t)slot * kStageBytes + col_offset(g, d) + 16 * q;
          float c[4][4];  // four accumulators (blocks mod 4), so the MMA chains overlap
#pragma unroll
          for (int j = 0; j < 4; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.f;
          int blk = b0;
          for (; blk + 4 <= b1; blk += 4) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 xv = make_uint4(0u, 0u, 0u, 0u);
              if (g < NT) xv = *reinterpret_cast<const uint4*>(xrow + (blk + j) * 64);
              const uint4 wv = *reinterpret_cast<const uint4*>(wrow + (blk + j) * 64);
              mma_bf16_m16n8k16(c[j], xv.x, xv.y, wv.x, wv.y);
              mma_bf16_m16n8k16(c[j], xv.z, xv.w, wv.z, wv.w);
            }
          }
          for (; blk < b1; ++blk) {
            uint4 xv = make_uint4(0u, 0u, 0u, 0u);
            if (g < NT) xv = *reinterpret_cast<const uint4*>(xrow + blk * 64);
            const uint4 wv = *reinterpret_cast<const uint4*>(wrow + blk * 64);
            mma_bf16_m16n8k16(c[0], xv.x, xv.y, wv.x, wv.y);
            mma_bf16_m16n8k16(c[0], xv.z, xv.w, wv.z, wv.w);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.empty_c[slot]);  // the warp's reads of the slot are done
          // token g with staged rows 2q, 2q + 1
          d0 = (c[0][0] + c[1][0]) + (c[2][0] + c[3][0]);
          d1 = (c[0][1] + c[1][1]) + (c[2][1] + c[3][1]);
          if (part > 0)
            partial[((slot * 2 + (f & 1)) * (kPartsC - 1) + part - 1) * 32 + lane] =
                make_float2(d0, d1);
        }
        if (!bar_red_and(1 + slot, wps_c * 32, go)) break;
        if (part == 0) {
          for (int p2 = 1; p2 < wps_c; ++p2) {
            const float2 v = partial[((slot * 2 + (f & 1)) * (kPartsC - 1) + p2 - 1) * 32 + lane];
            d0 += v.x;
            d1 += v.y;
          }
          // lanes q = 0, 1 hold the gate dots of pairs q (column 2q) and
          // q + 2 (column 2q + 1); the matching up dots are two lanes up
          const float u0 = __shfl_down_sync(0xffffffffu, d0, 2);
          const float u1 = __shfl_down_sync(0xffffffffu, d1, 2);
          if (q < 2 && g < NT) {
            const int pa = gst * kStagePairs, ui = pa / m, j0 = pa - ui * m;
            const uint32_t mk = sh.tok_mask[sh.uexp[ui]];
            if ((mk >> g) & 1u) {
              const int si = sh.ufirst[ui] + __popc(mk & ((1u << g) - 1u));
              __nv_bfloat16* hp = a.h + (size_t)si * m + j0 + q;
              hp[0] = __float2bfloat16_rn(silu(d0) * u0);
              hp[2] = __float2bfloat16_rn(silu(d1) * u1);
            }
          }
        }
      }
    }
  }
  __syncthreads();  // every kept slot's h of this CTA's stages is written
  // h is read back by bulk copies (the async proxy) after the grid barrier
  asm volatile("fence.proxy.async.global;" ::: "memory");
  stamp(a, 4);
  if (!grid_barrier(a, sh, 2)) {
    if (producer && lane == 0) {
      // the pre-issued stages expect their h rows too: copy them (whatever h
      // holds) so that their phases complete, then let everything land
      for (int ui = 0; ui < sh.n_d_issued; ++ui) {
        const int s0 = sh.ufirst[ui];
        bulk_g2s(ring_d + (size_t)ui * dstage + dbytes, a.h + (size_t)s0 * m,
                 (uint32_t)((sh.ufirst[ui + 1] - s0) * m * 2), &sh.full_d[ui]);
      }
      drain_copies(sh, nring, nring_d);
    }
    if (threadIdx.x == 0) depart(a, sh);
    return;
  }
  stamp(a, 5);

  // ---------------------------------------------------------- phase D
  // a ring of stages that each hold the CTA's output rows of one surviving
  // expert's W^down and the h rows of its kept slots; the W^down rows of the
  // first n_pre stages were issued at the end of phase C
  if (nrows > 0) {
    if (producer) {
      if (lane == 0) {
        asm volatile("fence.proxy.async.global;" ::: "memory");  // h is read by bulk copies
        for (int ui = 0; ui < sh.n_d_issued; ++ui) {
          const int s0 = sh.ufirst[ui];
          const uint32_t hb = (uint32_t)((sh.ufirst[ui + 1] - s0) * m * 2);
          bulk_g2s(ring_d + (size_t)ui * dstage + dbytes, a.h + (size_t)s0 * m, hb,
                   &sh.full_d[ui]);
        }
        for (int ui = sh.n_d_issued; ui < U; ++ui) {
          const int slot = ui % nring_d;
          if (!wait_bar(&sh.empty_d[slot], ((ui / nring_d) & 1) ^ 1u, a, sh)) break;
          const int s0 = sh.ufirst[ui];
          const uint32_t hb = (uint32_t)((sh.ufirst[ui + 1] - s0) * m * 2);
          uint8_t* st = ring_d + (size_t)slot * dstage;
          mbar_expect_tx(&sh.full_d[slot], dbytes + hb);
          bulk_g2s_hint(st, a.wd + ((size_t)sh.uexp[ui] * d + i0) * m, dbytes, &sh.full_d[slot],
                        evict_first_policy());
          bulk_g2s(st + dbytes, a.h + (size_t)s0 * m, hb, &sh.full_d[slot]);
          sh.n_d_issued = ui + 1;
        }
      }
    } else {
      // Each ring slot has wps_d fixed consumer warps (parts), which take its
      // fills (experts slot, slot + nring_d, ...) in order; part p covers the
      // 32-wide blocks kb0 .. kb1 - 1 of the expert size.  One MMA tile per
      // block pair of k: A = the stage's W^down rows (MMA rows: the CTA's
      // output rows, rows nrows .. 15 zero), B = the stage's h rows (MMA
      // columns: the expert's kept slots, columns nt .. 7 zero), with the
      // same permutation of each block's 32 k on both operands as in phase C.
      // The warp then adds g * (h W^down) of each kept slot into its own sums
      // [16 rows][NT tokens] in shared memory (its lanes own distinct cells:
      // a token keeps an expert once), experts in ascending order.
      const int slot = warp / wps_d, part = warp % wps_d;
      const int g = lane >> 2, q = lane & 3;
      const int nbm = m / 32;
      const int kb0 = part * nbm / wps_d, kb1 = (part + 1) * nbm / wps_d;
      float* acc = reinterpret_cast<float*>(ring_d + (size_t)nring_d * dstage) + warp * 16 * NT;
      const bool ra = g < nrows, rb = g + 8 < nrows;
      if (slot < nring_d) {
        for (int i = lane; i < 16 * NT; i += 32) acc[i] = 0.f;
        __syncwarp();
        for (int ui = slot; ui < U; ui += nring_d) {
          const int f = ui / nring_d;
          int ok = 1;
          if (lane == 0) ok = wait_bar(&sh.full_d[slot], f & 1, a, sh);
          if (!__shfl_sync(0xffffffffu, ok, 0)) break;
          mbar_try_wait(&sh.full_d[slot], f & 1);
          const int s0 = sh.ufirst[ui], nt = sh.ufirst[ui + 1] - s0;  // <= NT
          const uint8_t* st = ring_d + (size_t)slot * dstage;
          const uint8_t* ar0 = st + (size_t)g * m * 2 + 16 * q;  // W^down row i0 + g
          const uint8_t* ar1 = ar0 + (size_t)8 * m * 2;            // row i0 + g + 8
          const uint8_t* br = st + dbytes + (size_t)g * m * 2 + 16 * q;  // h of slot s0 + g
          const bool hb = g < nt;
          float c[2][4];
#pragma unroll
          for (int j = 0; j < 2; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.f;
          for (int blk = kb0; blk < kb1; blk += 2) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              if (blk + j < kb1) {
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                const uint4 av = ra ? *reinterpret_cast<const uint4*>(ar0 + (blk + j) * 64) : z;
                const uint4 av8 = rb ? *reinterpret_cast<const uint4*>(ar1 + (blk + j) * 64) : z;
                const uint4 hv = hb ? *reinterpret_cast<const uint4*>(br + (blk + j) * 64) : z;
                mma_bf16_m16n8k16_full(c[j], av.x, av8.x, av.y, av8.y, hv.x, hv.y);
                mma_bf16_m16n8k16_full(c[j], av.z, av8.z, av.w, av8.w, hv.z, hv.w);
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.empty_d[slot]);  // the warp's reads of the slot are done
          // lane (g, q): rows g, g + 8 with the slots s0 + 2q, s0 + 2q + 1
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int col = 2 * q + e2;
            if (col < nt) {
              const int t = sh.slot_t[s0 + col];
              const float gq = sh.slot_g[s0 + col];
              if (ra) acc[g * NT + t] = fmaf(gq, c[0][e2] + c[1][e2], acc[g * NT + t]);
              if (rb) acc[(g + 8) * NT + t] = fmaf(gq, c[0][2 + e2] + c[1][2 + e2], acc[(g + 8) * NT + t]);
            }
          }
        }
      }
    }
  }
  __syncthreads();  // every warp's sums are in
  if (producer && lane == 0) drain_copies(sh, nring, nring_d);  // (all consumed unless aborted)
  if (nrows > 0 && (int)threadIdx.x < nrows * NT) {
    // output row i0 + r of token t: the consumer warps' sums in warp order
    const int r = threadIdx.x / NT, t = threadIdx.x - r * NT;
    const float* acc0 = reinterpret_cast<const float*>(ring_d + (size_t)nring_d * dstage);
    float v = 0.f;
    for (int w = 0; w < nring_d * wps_d; ++w) v += acc0[(w * 16 + r) * NT + t];
    a.y[(size_t)t * d + i0 + r] = __float2bfloat16_rn(v);
  }
  stamp(a, 6);

  // debug / compaction outputs (CTA 0, off the critical path)
  if (blockIdx.x == 0) {
    if ((int)threadIdx.x < TK) {
      const int s = threadIdx.x;
      a.idx[s] = sh.t_idx[s];
      a.gate[s] = sh.t_gate[s];
      a.score[s] = sh.t_score[s];
      a.keep[s] = (uint8_t)sh.t_keep[s];
      a.slot_of[s] = sh.t_pos[s];
    }
    if ((int)threadIdx.x < S) {
      a.slot_token[threadIdx.x] = sh.slot_t[threadIdx.x];
      a.slot_rank[threadIdx.x] = sh.slot_r[threadIdx.x];
    }
    for (int e = threadIdx.x; e <= E; e += blockDim.x) a.offsets[e] = e < E ? sh.e_base[e] : S;
    if (threadIdx.x == 0) *a.n_kept = S;
  }
  if (threadIdx.x == 0) depart(a, sh);
}

template <int NT>
cudaError_t launch_nt(cudaLaunchConfig_t& cfg, const DecodeArgs& a, size_t smem) {
  static size_t attr_bytes = 0;  // largest dynamic shared memory enabled so far
  if (smem > attr_bytes) {
    cudaError_t e = cudaFuncSetAttribute(k_decode<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr_bytes = smem;
  }
  return cudaLaunchKernelEx(&cfg, k_decode<NT>, a);
}

}  // namespace

// Dynamic shared memory in phase C: [ring of nring 33 KB stages | bf16(x)
// [T][d], padded rows | partial dots].  The unrounded fp32 x and the staged
// inputs of phase A live inside the ring.  Phase D reuses all of it: [its
// ring | per-warp sums].
static size_t region_bytes(int T, int d) {
  return (size_t)T * row_stride(d) + kPartBytes;  // bf16(x), partial dots
}

static int ring_stages(int T, int d) {
  const size_t avail = (size_t)kSmemBudget - sizeof(DecShared) - 1024 - region_bytes(T, d);
  const int n = (int)(avail / kStageBytes);
  // any depth: each slot's warps wait on its fills in order
  return n > kRing ? kRing : n;
}

// All the shared memory a CTA can have: phase C uses its ring and bf16(x),
// phase D the whole of it (h, then as many W^down stages as fit).
size_t decode_smem_bytes(int T, int d, int m, int k, int E, int num_sms) {
  (void)T, (void)d, (void)m, (void)k, (void)E, (void)num_sms;
  return (size_t)kSmemBudget - sizeof(DecShared);
}

bool decode_fits(int T, int d, int m, int k, int E, int num_sms) {
  // the bf16 shape rule of every entry point (d and m multiples of 128) also
  // keeps the staged rows and the MMA blocks of phase C whole
  if (T < 1 || T > kDecodeMaxT || d > 2048 || d % 128 != 0 || m % 128 != 0) return false;
  const int n = ring_stages(T, d);
  if (n < 2) return false;
  // phase A inside the ring: x (fp32), u (bf16), gamma, the router rows
  const size_t staged = (size_t)T * d * 6 + (size_t)d * 4 +
                        (size_t)((E + num_sms - 1) / num_sms) * d * 2;
  if (staged > (size_t)n * kStageBytes) return false;
  const int rows = (d + num_sms - 1) / num_sms;                    // phase-D rows per CTA
  if (rows > kCompWarps) return false;
  // phase D: at least two stages of W^down rows and an expert's h rows, and
  // the per-warp sums
  return decode_smem_bytes(T, d, m, k, E, num_sms) >=
         1024 + dacc_bytes(T) + 2 * dstage_bytes(rows, T, m);
}

cudaError_t launch_decode(const ace_layer& L, int fusion, const void* u, int T, float tau,
                          int renorm,
                          float eps_rms, void* y, float* logits, void* h, int32_t* idx,
                          float* gate, float* score, uint8_t* keep, int32_t* offsets,
                          int32_t* slot_token, int32_t* slot_rank, int32_t* slot_of,
                          int32_t* n_kept, uint32_t* sync, uint32_t* status, bool keep_status,
                          unsigned long long* trace, int num_sms, cudaStream_t s) {
  DecodeArgs a;
  a.gamma = L.gamma;
  a.wr = (const __nv_bfloat16*)L.w_router;
  a.bias = L.router_bias;
  a.wg = (const __nv_bfloat16*)L.w_gate;
  a.wu = (const __nv_bfloat16*)L.w_up;
  a.wd = (const __nv_bfloat16*)L.w_down;
  a.ft.amax = L.amax;
  a.ft.a_gsp = L.a_gsp;
  a.ft.a_rcr = L.a_rcr;
  a.ft.fusion = fusion;
  a.u = (const __nv_bfloat16*)u;
  a.y = (__nv_bfloat16*)y;
  a.T = T;
  a.d = L.d;
  a.E = L.E;
  a.m = L.m;
  a.k = L.k;
  a.tau = tau;
  a.eps_rms = eps_rms;
  a.renorm = renorm;
  a.logits = logits;
  a.h = (__nv_bfloat16*)h;
  a.idx = idx;
  a.gate = gate;
  a.score = score;
  a.keep = keep;
  a.offsets = offsets;
  a.slot_token = slot_token;
  a.slot_rank = slot_rank;
  a.slot_of = slot_of;
  a.n_kept = n_kept;
  a.sync = sync;
  a.status = status;
  a.keep_status = keep_status ? 1 : 0;
  a.trace = trace;
  a.peer_wait_ns = peer_wait_ns();
  a.nring = ring_stages(T, L.d);
  a.region = a.nring * kStageBytes;
  a.part_off = a.region + T * row_stride(L.d);
  const size_t smem = decode_smem_bytes(T, L.d, L.m, L.k, L.E, num_sms);
  a.dyn_bytes = smem;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  switch (T) {
    case 1: return launch_nt<1>(cfg, a, smem);
    case 2: return launch_nt<2>(cfg, a, smem);
    case 3: return launch_nt<3>(cfg, a, smem);
    case 4: return launch_nt<4>(cfg, a, smem);
    case 5: return launch_nt<5>(cfg, a, smem);
    case 6: return launch_nt<6>(cfg, a, smem);
    case 7: return launch_nt<7>(cfg, a, smem);
    case 8: return launch_nt<8>(cfg, a, smem);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ace
