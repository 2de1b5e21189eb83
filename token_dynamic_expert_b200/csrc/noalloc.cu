// noalloc.cu -- ace_moe_decode_noalloc: the decode forward (T <= 8 tokens,
// bf16 layers) with its scratch memory in a fixed, file-scope device array,
// for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: plugins inside a host framework that
// owns every device allocation and hands out no allocator, or serving loops
// that must not allocate once they are running (an allocation can
// synchronise the device and stall every stream).  They still own their
// inputs and outputs; only the scratch comes from here.
//
// The array lives for the life of the process on every GPU that loads the
// library.  Host code cannot use the array's name as a device address (on the
// host it is a stand-in), so the first call on each device, with that device
// current, asks the runtime for the array's device address once and caches
// it.  Do that first call before any stream capture.
#include <mutex>

#include "ace_common.cuh"
#include "ace_internal.h"

namespace ace {
namespace {

// Upper bound of the scratch this entry point can use: the decode kernel's
// router logits, bf16 gated intermediates and slot tables for up to 8 tokens.
constexpr size_t kStaticScratchBytes = 512 * 1024;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

struct StaticLayout {
  size_t logits, h, idx, gate, score, keep, offsets, slot_token, slot_rank, slot_of, n_kept, total;
};

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

StaticLayout static_layout(int T, int E, int k, int m) {
  StaticLayout o{};
  size_t off = 256;  // status word at 0, grid-barrier counter at byte 64
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  const size_t tk = (size_t)T * k;
  o.logits = take((size_t)T * E * 4);
  o.h = take(tk * m * 2);
  o.idx = take(tk * 4);
  o.gate = take(tk * 4);
  o.score = take(tk * 4);
  o.keep = take(tk);
  o.offsets = take(((size_t)E + 1) * 4);
  o.slot_token = take(tk * 4);
  o.slot_rank = take(tk * 4);
  o.slot_of = take(tk * 4);
  o.n_kept = take(4);
  o.total = off;
  return o;
}

// Device address of the array on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace ace

using namespace ace;

extern "C" ace_status ace_moe_decode_noalloc(const ace_layer* layer, const void* u, int T,
                                             const ace_fwd_opts* opts, void* y, void* stream) {
  // the same layer checks and shape rule as ace_moe_forward
  const ace_status st = validate_layer(layer, true);
  if (st != ACE_OK) return st;
  if (!opts || !u || !y) return ACE_ERR_INVALID_ARG;
  const ace_layer& L = *layer;
  if (L.dtype != ACE_BF16) return ACE_ERR_UNSUPPORTED;
  if (T < 1 || T > kDecodeMaxT) return ACE_ERR_INVALID_ARG;
  if (check_fusion(L, (int)opts->fusion) != ACE_OK) return ACE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(u) | reinterpret_cast<uintptr_t>(y)) % 16 != 0)
    return ACE_ERR_INVALID_ARG;
  {
    const uint8_t *ub = (const uint8_t*)u, *yb = (const uint8_t*)y;
    const size_t bytes = (size_t)T * L.d * 2;
    if (ub < yb + bytes && yb < ub + bytes) return ACE_ERR_INVALID_ARG;
  }
  const int num_sms = device_sm_count();
  if (!decode_fits(T, L.d, L.m, L.k, L.E, num_sms)) return ACE_ERR_UNSUPPORTED;
  const StaticLayout ly = static_layout(T, L.E, L.k, L.m);
  if (ly.total > kStaticScratchBytes) return ACE_ERR_UNSUPPORTED;  // beyond the fixed scratch

  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return ACE_ERR_CUDA;
  uint8_t* w = static_cast<uint8_t*>(base);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word and the decode kernel's cross-CTA words (byte 64) start
  // from zero
  if (launch_clear_words(w, 64, s) != cudaSuccess) return ACE_ERR_CUDA;
  auto at = [&](size_t off) { return w + off; };
  if (launch_decode(L, (int)opts->fusion, u, T, opts->tau, opts->renorm_topk, opts->eps_rms, y,
                    reinterpret_cast<float*>(at(ly.logits)), at(ly.h),
                    reinterpret_cast<int32_t*>(at(ly.idx)), reinterpret_cast<float*>(at(ly.gate)),
                    reinterpret_cast<float*>(at(ly.score)), at(ly.keep),
                    reinterpret_cast<int32_t*>(at(ly.offsets)),
                    reinterpret_cast<int32_t*>(at(ly.slot_token)),
                    reinterpret_cast<int32_t*>(at(ly.slot_rank)),
                    reinterpret_cast<int32_t*>(at(ly.slot_of)),
                    reinterpret_cast<int32_t*>(at(ly.n_kept)),
                    reinterpret_cast<uint32_t*>(w) + 16, reinterpret_cast<uint32_t*>(w), false,
                    nullptr, num_sms, s) != cudaSuccess)
    return ACE_ERR_CUDA;
  return ACE_OK;
}

extern "C" ace_status ace_noalloc_read_status(uint32_t* flags, void* stream) {
  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return ACE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, base, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return ACE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ACE_ERR_CUDA;
  if (flags) *flags = v;
  if (v & ACE_FLAG_TIMEOUT) return ACE_ERR_TIMEOUT;
  if (v & (ACE_FLAG_BAD_INDEX | ACE_FLAG_OVERFLOW)) return ACE_ERR_DEVICE_FAULT;
  return ACE_OK;
}
