// ace_api.cu -- the C ABI of libace (declared in include/ace.h): argument
// validation, the workspace layout, and the launch sequence of the forward.
#include <string.h>

#include <atomic>

#include "ace_common.cuh"
#include "ace_internal.h"
#include "compact.cuh"

namespace ace {

// Zeroes n 32-bit words.  A kernel rather than cudaMemsetAsync: inside a CUDA
// graph a memset node before a kernel node costs ~3 us of dependency
// latency on B200, a kernel node ~1 us.
__global__ void k_clear_words(uint32_t* p, int n) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) p[i] = 0u;
}

cudaError_t launch_clear_words(void* p, int n_words, cudaStream_t s) {
  k_clear_words<<<1, 64, 0, s>>>(static_cast<uint32_t*>(p), n_words);
  return cudaGetLastError();
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

static size_t esize(ace_dtype dt) { return dt == ACE_BF16 ? 2 : 4; }

int router_splits_for(const ace_layer& L, int T, int num_sms) {
  return L.dtype == ACE_BF16 ? router_tc_splits(T, L.d, L.E, num_sms)
                             : router_splitk(T, L.d, L.E, num_sms);
}

FwdLayout fwd_layout(const ace_layer& L, int max_tokens, int num_sms) {
  FwdLayout o;
  memset(&o, 0, sizeof(o));
  const size_t T = (size_t)(max_tokens > 0 ? max_tokens : 1), k = (size_t)L.k, E = (size_t)L.E;
  const size_t d = (size_t)L.d, m = (size_t)L.m, es = esize(L.dtype);
  const size_t nchunk = (T + kChunk - 1) / kChunk, cap = T * k;
  // largest split-K x tokens product over the token counts this workspace serves
  // (the split count only changes at multiples of the router's token tile)
  size_t part = 0;
  const int rbt = L.dtype == ACE_BF16 ? 128 : kRouterBT;
  for (int gx = 1; gx <= cdiv((int)T, rbt); ++gx) {
    const int t = gx == cdiv((int)T, rbt) ? (int)T : gx * rbt;
    const size_t p = (size_t)router_splits_for(L, t, num_sms) * (size_t)t * E;
    if (p > part) part = p;
  }
  o.max_tokens = (int)T;
  o.part_floats = (int)part;
  o.max_tiles = (int)E + cdiv((int)cap, kTileN);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  o.status = take(256);
  o.part = take(part * 4);
  o.inv_rms = take(T * 4);
  o.rw3 = take(L.dtype == ACE_BF16 ? 3 * E * d * 2 : 0);  // gamma-folded router rows, 3 terms
  o.idx = take(cap * 4);
  o.gate = take(cap * 4);
  o.score = take(cap * 4);
  o.keep = take(cap);
  // bitmap and range_cnt adjacent: RMSNorm zeroes them as one block
  const size_t nrange = (T + kRangeTok - 1) / kRangeTok;
  o.bitmap = take((nchunk + nrange) * E * 4);
  o.range_cnt = o.bitmap + nchunk * E * 4;
  o.rbase = take(nrange * E * 4);
  o.counts = take(E * 4);
  o.offsets = take((E + 1) * 4);
  o.n_kept = take(4);
  o.tiles = take((size_t)o.max_tiles * 16);
  o.n_tiles = take(4);
  o.tile_done = take((size_t)o.max_tiles * 4);
  o.slot_token = take(cap * 4);
  o.slot_rank = take(cap * 4);
  o.slot_gate = take(cap * 4);
  o.slot_of = take(cap * 4);
  o.xp = take(cap * d * es);
  o.h = take(cap * m * es);
  o.yslot = take(cap * d * es);
  o.total = off;
  return o;
}

}  // namespace ace

using namespace ace;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

ace_status check_layer(const ace_layer* L, bool need_experts) {
  if (!L) return ACE_ERR_INVALID_ARG;
  if (L->d <= 0 || L->E <= 0 || L->m <= 0 || L->k <= 0) return ACE_ERR_INVALID_ARG;
  if (L->k > L->E || L->k > kMaxK) return ACE_ERR_INVALID_ARG;
  if (L->dtype != ACE_BF16 && L->dtype != ACE_F32) return ACE_ERR_INVALID_ARG;
  if (!L->gamma || !L->w_router) return ACE_ERR_INVALID_ARG;
  if (L->E > kMaxE) return ACE_ERR_UNSUPPORTED;
  if (L->d % 64 != 0 || L->m % 64 != 0) return ACE_ERR_UNSUPPORTED;
  if (need_experts) {
    if (!L->w_gate || !L->w_up || !L->w_down) return ACE_ERR_INVALID_ARG;
    if (!aligned(L->w_gate, 16) || !aligned(L->w_up, 16) || !aligned(L->w_down, 16))
      return ACE_ERR_INVALID_ARG;
    if (L->dtype == ACE_BF16 && (L->d % 128 != 0 || L->m % 128 != 0)) return ACE_ERR_UNSUPPORTED;
  }
  if (!aligned(L->w_router, 16) || !aligned(L->gamma, 16)) return ACE_ERR_INVALID_ARG;
  return ACE_OK;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Limit of the waits in which a CTA waits on other CTAs (ace_set_peer_wait_limit_ns).
std::atomic<uint64_t> g_peer_wait_ns{kWaitLimitNs};

}  // namespace

namespace ace {
ace_status validate_layer(const ace_layer* L, bool need_experts) {
  return check_layer(L, need_experts);
}
uint64_t peer_wait_ns() { return g_peer_wait_ns.load(std::memory_order_relaxed); }
}  // namespace ace

namespace ace {
// The fusion rule is known and the tables it reads are present.
ace_status check_fusion(const ace_layer& L, int fusion) {
  const bool need_g = fusion == ACE_FUSE_MIN || fusion == ACE_FUSE_MEAN || fusion == ACE_FUSE_GSP;
  const bool need_r = fusion == ACE_FUSE_MIN || fusion == ACE_FUSE_MEAN || fusion == ACE_FUSE_RCR;
  if (fusion < ACE_FUSE_MAX || fusion > ACE_FUSE_RCR) return ACE_ERR_INVALID_ARG;
  if ((need_g && !L.a_gsp) || (need_r && !L.a_rcr)) return ACE_ERR_INVALID_ARG;
  if ((L.amax && !aligned(L.amax, 4)) || (L.a_gsp && !aligned(L.a_gsp, 4)) ||
      (L.a_rcr && !aligned(L.a_rcr, 4)))
    return ACE_ERR_INVALID_ARG;
  return ACE_OK;
}
}  // namespace ace

namespace {

ace_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = e;
  return ACE_ERR_CUDA;
}

#define ACE_CK(call)                                \
  do {                                              \
    const cudaError_t ace_e_ = (call);              \
    if (ace_e_ != cudaSuccess) return cuda_fail(ace_e_); \
  } while (0)

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

// Word of the status block counting finished routing CTAs (zeroed per call).
constexpr size_t kDoneCtrWord = 32;

// Status words a call zeroes before its kernels run: all 64 of the block, or
// (a layer stack keeping one status word across layers) words 16-63.
struct StatusClear {
  uint32_t* p;
  int n;
};
StatusClear status_clear(const FwdLayout& ly, void* ws, bool keep_status) {
  uint32_t* w = at<uint32_t>(ws, ly.status);
  return keep_status ? StatusClear{w + 16, 48} : StatusClear{w, 64};
}

// The routing half shared by the forward and the score query; with_scan adds
// the compaction's expert-offset scan (run by the routing's last CTA).  x_out
// (nullable) receives x rounded to the storage type.  The first kernel zeroes
// the status words `clr` (T > 0 here).
ace_status run_routing(const ace_layer& L, const void* u, int T, const ace_fwd_opts& o,
                       const FwdLayout& ly, void* ws, int num_sms, float* logits_dbg,
                       bool with_scan, void* x_out, StatusClear clr, cudaStream_t s) {
  const int splitk = router_splits_for(L, T, num_sms);
  const bool tc = L.dtype == ACE_BF16;
  const size_t n_zero = ((size_t)cdiv(T, kChunk) + (size_t)cdiv(T, kRangeTok)) * (size_t)L.E;
  ACE_CK(launch_rmsnorm(L.dtype, u, T, L.d, L.gamma, o.eps_rms, at<float>(ws, ly.inv_rms), x_out,
                        clr.p, clr.n, at<uint32_t>(ws, ly.bitmap), n_zero, L.w_router, L.E,
                        tc ? at<void>(ws, ly.rw3) : nullptr, s));
  if (tc)
    ACE_CK(launch_router_tc(u, at<float>(ws, ly.inv_rms), at<void>(ws, ly.rw3), T, L.d, L.E,
                            splitk, at<float>(ws, ly.part), at<uint32_t>(ws, ly.status), num_sms,
                            s));
  else
    ACE_CK(launch_router_logits(L.dtype, u, at<float>(ws, ly.inv_rms), L.gamma, L.w_router, T,
                                L.d, L.E, splitk, at<float>(ws, ly.part), s));
  ScanOut so{};
  so.rbase = at<int32_t>(ws, ly.rbase);
  so.counts = at<int32_t>(ws, ly.counts);
  so.offsets = at<int32_t>(ws, ly.offsets);
  so.n_kept = at<int32_t>(ws, ly.n_kept);
  so.tiles = at<int4>(ws, ly.tiles);
  so.n_tiles = at<int32_t>(ws, ly.n_tiles);
  so.tile_done = at<uint32_t>(ws, ly.tile_done);
  so.max_tiles = ly.max_tiles;
  so.tile_n = kTileN;
  FuseTables ft{L.amax, L.a_gsp, L.a_rcr, (int)o.fusion};
  ACE_CK(launch_topk_mask(at<float>(ws, ly.part), splitk, T, L.E, L.k, L.router_bias, ft,
                          o.tau, o.renorm_topk, at<int32_t>(ws, ly.idx), at<float>(ws, ly.gate),
                          at<float>(ws, ly.score), at<uint8_t>(ws, ly.keep),
                          at<uint32_t>(ws, ly.bitmap), at<int32_t>(ws, ly.range_cnt), logits_dbg,
                          at<uint32_t>(ws, ly.status), at<uint32_t>(ws, ly.status) + kDoneCtrWord,
                          with_scan ? &so : nullptr, s));
  return ACE_OK;
}

ace_status check_common(const ace_layer* layer, const void* u, int T, const ace_fwd_opts* opts,
                        void* ws, bool need_experts) {
  ace_status st = check_layer(layer, need_experts);
  if (st != ACE_OK) return st;
  if (!opts || T < 0) return ACE_ERR_INVALID_ARG;
  st = check_fusion(*layer, opts->fusion);
  if (st != ACE_OK) return st;
  if (T > 0 && (!u || !aligned(u, 16))) return ACE_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256)) return ACE_ERR_WORKSPACE;
  return ACE_OK;
}

// Both expert GEMMs in one launch when the slot tiles are small: fewer than
// 128 slots per expert on average before skipping (T k < 128 E).  There the
// GEMMs stream weights and the fused kernel's down items fill the gate/up
// tail (measured 254 -> 249 us at 1024 tokens); with larger tiles the down
// items wait on many CTAs' gate/up items and two launches are faster
// (705 vs 759 us at 8192 tokens, 256 experts).
bool fused_experts(const ace_layer& L, int T) { return (long long)T * L.k < 128LL * L.E; }

// The prefill launch sequence: RMSNorm, router, top-k + mask (its last CTA
// runs the expert-offset scan), slot tables + row gather, expert GEMMs,
// combine.
ace_status run_prefill(const ace_layer& L, const void* u, int T, const ace_fwd_opts& o, void* y,
                       const FwdLayout& ly, void* ws, int num_sms, ace_debug_out* dbg,
                       StatusClear clr, cudaEvent_t ev_b, cudaEvent_t ev_m, cudaEvent_t ev_e,
                       cudaStream_t s) {
  ace_status st = run_routing(L, u, T, o, ly, ws, num_sms, dbg ? dbg->logits : nullptr, true,
                              nullptr, clr, s);
  if (st != ACE_OK) return st;
  ACE_CK(launch_scatter_gather(
      L.dtype, T, L.k, L.E, L.d, at<int32_t>(ws, ly.idx), at<float>(ws, ly.gate),
      at<uint8_t>(ws, ly.keep), at<uint32_t>(ws, ly.bitmap), at<int32_t>(ws, ly.rbase), u,
      at<float>(ws, ly.inv_rms), L.gamma, at<int32_t>(ws, ly.slot_token),
      at<int32_t>(ws, ly.slot_rank), at<float>(ws, ly.slot_gate), at<int32_t>(ws, ly.slot_of),
      at<void>(ws, ly.xp), at<uint32_t>(ws, ly.status), s));
  if (ev_b) ACE_CK(cudaEventRecord(ev_b, s));
  if (L.dtype == ACE_BF16 && fused_experts(L, T)) {
    // one launch for both expert GEMMs; "mid" is recorded after it as well
    ACE_CK(launch_experts_fused(L, T * L.k, at<void>(ws, ly.xp), at<void>(ws, ly.h),
                                at<void>(ws, ly.yslot), at<int4>(ws, ly.tiles),
                                at<int32_t>(ws, ly.n_tiles), ly.max_tiles,
                                at<float>(ws, ly.slot_gate), at<uint32_t>(ws, ly.tile_done),
                                at<uint32_t>(ws, ly.status), num_sms, s));
    if (ev_m) ACE_CK(cudaEventRecord(ev_m, s));
  } else if (L.dtype == ACE_BF16) {
    if (launch_experts_sm100(L, T * L.k, at<void>(ws, ly.xp), at<void>(ws, ly.h),
                             at<void>(ws, ly.yslot), at<int4>(ws, ly.tiles),
                             at<int32_t>(ws, ly.n_tiles), ly.max_tiles,
                             at<float>(ws, ly.slot_gate), at<uint32_t>(ws, ly.status), num_sms,
                             s, ev_m) != cudaSuccess)
      return cuda_fail(cudaGetLastError());
  } else {
    ACE_CK(launch_experts_simt(L, at<void>(ws, ly.xp), at<void>(ws, ly.h), at<void>(ws, ly.yslot),
                               at<int4>(ws, ly.tiles), at<int32_t>(ws, ly.n_tiles), ly.max_tiles,
                               at<float>(ws, ly.slot_gate), s));
    if (ev_m) ACE_CK(cudaEventRecord(ev_m, s));
  }
  if (ev_e) ACE_CK(cudaEventRecord(ev_e, s));
  ACE_CK(launch_combine(L.dtype, T, L.k, L.d, at<int32_t>(ws, ly.slot_of), at<void>(ws, ly.yslot),
                        T * L.k, y, at<uint32_t>(ws, ly.status), s));
  return ACE_OK;
}


}  // namespace

extern "C" {

size_t ace_workspace_size(const ace_layer* layer, int max_tokens) {
  if (check_layer(layer, false) != ACE_OK || max_tokens < 0) return 0;
  return fwd_layout(*layer, max_tokens, device_sm_count()).total;
}

}  // extern "C"

namespace {

// The forward of one layer.  keep_status: leave the status word as it is
// (a layer of a stack adds its flags to those of the layers before it).
ace_status forward_impl(const ace_layer* layer, const void* u, int T, const ace_fwd_opts* opts,
                        void* y, void* ws, size_t ws_bytes, ace_debug_out* dbg, void* stream,
                        bool keep_status) {
  ace_status st = check_common(layer, u, T, opts, ws, true);
  if (st != ACE_OK) return st;
  if (T > 0 && (!y || !aligned(y, 16))) return ACE_ERR_INVALID_ARG;
  const ace_layer& L = *layer;
  const size_t es = esize(L.dtype);
  if (T > 0) {  // u and y may not overlap
    const uint8_t *ub = (const uint8_t*)u, *yb = (const uint8_t*)y;
    const size_t bytes = (size_t)T * L.d * es;
    if (ub < yb + bytes && yb < ub + bytes) return ACE_ERR_INVALID_ARG;
  }
  const int num_sms = device_sm_count();
  const FwdLayout ly = fwd_layout(L, T, num_sms);
  if (ws_bytes < ly.total) return ACE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool decode = T > 0 && L.dtype == ACE_BF16 && T <= kDecodeMaxT &&
                      decode_fits(T, L.d, L.m, L.k, L.E, num_sms);
  // status word (offset 0), the decode kernel's cross-CTA words (byte 64)
  // and the routing CTAs' completion count (byte 128).  The decode kernel
  // needs no clearing: its words carry their launch's epoch, and it writes
  // the status word itself as it finishes.  The prefill's first kernel
  // zeroes them; with no token there is no kernel, so a clear runs instead.
  const StatusClear clr = status_clear(ly, ws, keep_status);
  if (!decode && T == 0) ACE_CK(launch_clear_words(clr.p, clr.n, s));
  if (T == 0) return ACE_OK;
  cudaEvent_t ev_b = dbg ? static_cast<cudaEvent_t>(dbg->ev_experts_begin) : nullptr;
  cudaEvent_t ev_m = dbg ? static_cast<cudaEvent_t>(dbg->ev_experts_mid) : nullptr;
  cudaEvent_t ev_e = dbg ? static_cast<cudaEvent_t>(dbg->ev_experts_end) : nullptr;

  if (decode) {
    // decode: one cooperative kernel streams the surviving experts' weights
    if (ev_b) ACE_CK(cudaEventRecord(ev_b, s));
    if (ev_m) ACE_CK(cudaEventRecord(ev_m, s));
    ACE_CK(launch_decode(L, (int)opts->fusion, u, T, opts->tau, opts->renorm_topk, opts->eps_rms, y,
                         at<float>(ws, ly.part), at<void>(ws, ly.h), at<int32_t>(ws, ly.idx),
                         at<float>(ws, ly.gate), at<float>(ws, ly.score), at<uint8_t>(ws, ly.keep),
                         at<int32_t>(ws, ly.offsets), at<int32_t>(ws, ly.slot_token),
                         at<int32_t>(ws, ly.slot_rank), at<int32_t>(ws, ly.slot_of),
                         at<int32_t>(ws, ly.n_kept), at<uint32_t>(ws, ly.status) + 16,
                         at<uint32_t>(ws, ly.status), keep_status, dbg ? dbg->trace : nullptr,
                         num_sms, s));
    if (ev_e) ACE_CK(cudaEventRecord(ev_e, s));
  } else {
    st = run_prefill(L, u, T, *opts, y, ly, ws, num_sms, dbg, clr, ev_b, ev_m, ev_e, s);
    if (st != ACE_OK) return st;
  }
  if (dbg) {
    const size_t tk = (size_t)T * L.k;
    auto cp = [&](void* dst, size_t off, size_t bytes) -> bool {
      return !dst || cudaMemcpyAsync(dst, at<void>(ws, off), bytes, cudaMemcpyDeviceToDevice, s) ==
                         cudaSuccess;
    };
    if (!cp(dbg->topk_idx, ly.idx, tk * 4) || !cp(dbg->gate, ly.gate, tk * 4) ||
        !cp(dbg->score, ly.score, tk * 4) || !cp(dbg->keep, ly.keep, tk) ||
        !cp(dbg->expert_offsets, ly.offsets, ((size_t)L.E + 1) * 4) ||
        !cp(dbg->slot_token, ly.slot_token, tk * 4) || !cp(dbg->slot_rank, ly.slot_rank, tk * 4) ||
        !cp(dbg->n_kept, ly.n_kept, 4))
      return ACE_ERR_CUDA;
    if (dbg->logits && decode &&
        !cp(dbg->logits, ly.part, (size_t)T * L.E * 4))
      return ACE_ERR_CUDA;
  }
  return ACE_OK;
}

// Stack workspace: [the largest layer workspace | activations A | B], each
// 256-byte aligned; the layer workspace starts at 0 so its status word is
// the stack's.
struct StackLayout {
  size_t layer_ws, act0, act1, total;
};

bool stack_layout(const ace_layer* layers, int n, int max_tokens, int num_sms, StackLayout* o) {
  if (!layers || n < 1 || max_tokens < 0) return false;
  size_t lw = 0;
  for (int l = 0; l < n; ++l) {
    if (check_layer(&layers[l], true) != ACE_OK) return false;
    if (layers[l].d != layers[0].d || layers[l].dtype != layers[0].dtype) return false;
    const size_t b = fwd_layout(layers[l], max_tokens, num_sms).total;
    if (b > lw) lw = b;
  }
  const size_t act = align_up((size_t)(max_tokens > 0 ? max_tokens : 1) * layers[0].d *
                                  esize(layers[0].dtype), 256);
  o->layer_ws = align_up(lw, 256);
  o->act0 = o->layer_ws;
  o->act1 = o->act0 + act;
  o->total = o->act1 + act;
  return true;
}

}  // namespace

extern "C" {

ace_status ace_moe_forward(const ace_layer* layer, const void* u, int T, const ace_fwd_opts* opts,
                           void* y, void* ws, size_t ws_bytes, ace_debug_out* dbg,
                           void* stream) {
  return forward_impl(layer, u, T, opts, y, ws, ws_bytes, dbg, stream, false);
}

size_t ace_stack_workspace_size(const ace_layer* layers, int n_layers, int max_tokens) {
  StackLayout ly;
  if (!stack_layout(layers, n_layers, max_tokens, device_sm_count(), &ly)) return 0;
  return ly.total;
}

ace_status ace_moe_stack_forward(const ace_layer* layers, int n_layers, const void* u, int T,
                                 const ace_fwd_opts* opts, void* y, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (!layers || n_layers < 1 || !opts || T < 0) return ACE_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256)) return ACE_ERR_WORKSPACE;
  for (int l = 0; l < n_layers; ++l) {
    if (check_layer(&layers[l], true) != ACE_OK) return check_layer(&layers[l], true);
    if (layers[l].d != layers[0].d || layers[l].dtype != layers[0].dtype)
      return ACE_ERR_INVALID_ARG;
    const ace_status fs = check_fusion(layers[l], opts[l].fusion);
    if (fs != ACE_OK) return fs;
  }
  if (T > 0 && (!u || !y || !aligned(u, 16) || !aligned(y, 16))) return ACE_ERR_INVALID_ARG;
  const size_t bytes = (size_t)T * layers[0].d * esize(layers[0].dtype);
  if (T > 0) {
    const uint8_t *ub = (const uint8_t*)u, *yb = (const uint8_t*)y;
    if (ub < yb + bytes && yb < ub + bytes) return ACE_ERR_INVALID_ARG;
  }
  StackLayout ly;
  if (!stack_layout(layers, n_layers, T, device_sm_count(), &ly)) return ACE_ERR_INVALID_ARG;
  if (ws_bytes < ly.total) return ACE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ACE_CK(launch_clear_words(ws, 1, s));  // the status word, once for the stack
  if (T == 0) return ACE_OK;
  uint8_t* base = static_cast<uint8_t*>(ws);
  const void* in = u;
  for (int l = 0; l < n_layers; ++l) {
    void* out = l == n_layers - 1 ? y : base + ((l & 1) ? ly.act1 : ly.act0);
    const ace_status st = forward_impl(&layers[l], in, T, &opts[l], out, ws, ly.layer_ws, nullptr,
                                       stream, true);
    if (st != ACE_OK) return st;
    in = out;
  }
  return ACE_OK;
}

ace_status ace_moe_scores(const ace_layer* layer, const void* u, int T, const ace_fwd_opts* opts,
                          float* score, int32_t* topk_idx, void* ws, size_t ws_bytes,
                          void* stream) {
  ace_status st = check_common(layer, u, T, opts, ws, false);
  if (st != ACE_OK) return st;
  if (T > 0 && !score) return ACE_ERR_INVALID_ARG;
  const ace_layer& L = *layer;
  const int num_sms = device_sm_count();
  const FwdLayout ly = fwd_layout(L, T, num_sms);
  if (ws_bytes < ly.total) return ACE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const StatusClear clr = status_clear(ly, ws, false);
  if (T == 0) {
    ACE_CK(launch_clear_words(clr.p, clr.n, s));
    return ACE_OK;
  }
  st = run_routing(L, u, T, *opts, ly, ws, num_sms, nullptr, false, nullptr, clr, s);
  if (st != ACE_OK) return st;
  const size_t tk = (size_t)T * L.k;
  ACE_CK(cudaMemcpyAsync(score, at<void>(ws, ly.score), tk * 4, cudaMemcpyDeviceToDevice, s));
  if (topk_idx)
    ACE_CK(cudaMemcpyAsync(topk_idx, at<void>(ws, ly.idx), tk * 4, cudaMemcpyDeviceToDevice, s));
  return ACE_OK;
}

ace_status ace_moe_route(const ace_layer* layer, const void* u, int T, const ace_fwd_opts* opts,
                         void* x, int32_t* idx, float* gate, uint8_t* keep, void* ws,
                         size_t ws_bytes, void* stream) {
  ace_status st = check_common(layer, u, T, opts, ws, false);
  if (st != ACE_OK) return st;
  if (T > 0 && (!x || !idx || !gate || !keep || !aligned(x, 16) || !aligned(idx, 4) ||
                !aligned(gate, 4)))
    return ACE_ERR_INVALID_ARG;
  const ace_layer& L = *layer;
  const int num_sms = device_sm_count();
  const FwdLayout ly = fwd_layout(L, T, num_sms);
  if (ws_bytes < ly.total) return ACE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const StatusClear clr = status_clear(ly, ws, false);
  if (T == 0) {
    ACE_CK(launch_clear_words(clr.p, clr.n, s));
    return ACE_OK;
  }
  st = run_routing(L, u, T, *opts, ly, ws, num_sms, nullptr, false, x, clr, s);
  if (st != ACE_OK) return st;
  const size_t tk = (size_t)T * L.k;
  ACE_CK(cudaMemcpyAsync(idx, at<void>(ws, ly.idx), tk * 4, cudaMemcpyDeviceToDevice, s));
  ACE_CK(cudaMemcpyAsync(gate, at<void>(ws, ly.gate), tk * 4, cudaMemcpyDeviceToDevice, s));
  ACE_CK(cudaMemcpyAsync(keep, at<void>(ws, ly.keep), tk, cudaMemcpyDeviceToDevice, s));
  return ACE_OK;
}

size_t ace_tau_workspace_size(void) { return tau_workspace_size(); }

ace_status ace_tau_quantile(const float* score, int n_tok, int k, int64_t n_skip, float* tau,
                            void* ws, size_t ws_bytes, void* stream) {
  if (n_tok < 0 || k < 1 || k > kMaxK || !tau) return ACE_ERR_INVALID_ARG;
  if (n_tok > 0 && !score) return ACE_ERR_INVALID_ARG;
  if (!aligned(tau, 4) || (score && !aligned(score, 4))) return ACE_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < tau_workspace_size()) return ACE_ERR_WORKSPACE;
  ACE_CK(launch_tau_quantile(score, n_tok, k, (long long)n_skip, tau, ws, device_sm_count(),
                             static_cast<cudaStream_t>(stream)));
  return ACE_OK;
}

ace_status ace_read_status(void* ws, size_t ws_bytes, uint32_t* flags, void* stream) {
  if (!ws || ws_bytes < 4) return ACE_ERR_WORKSPACE;
  uint32_t v = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return ACE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ACE_ERR_CUDA;
  if (flags) *flags = v;
  if (v & ACE_FLAG_TIMEOUT) return ACE_ERR_TIMEOUT;
  if (v & (ACE_FLAG_BAD_INDEX | ACE_FLAG_OVERFLOW)) return ACE_ERR_DEVICE_FAULT;
  return ACE_OK;
}

const char* ace_status_str(ace_status s) {
  switch (s) {
    case ACE_OK: return "ACE_OK";
    case ACE_ERR_INVALID_ARG: return "ACE_ERR_INVALID_ARG";
    case ACE_ERR_WORKSPACE: return "ACE_ERR_WORKSPACE";
    case ACE_ERR_CUDA: return "ACE_ERR_CUDA";
    case ACE_ERR_UNSUPPORTED: return "ACE_ERR_UNSUPPORTED";
    case ACE_ERR_DEVICE_FAULT: return "ACE_ERR_DEVICE_FAULT";
    case ACE_ERR_TIMEOUT: return "ACE_ERR_TIMEOUT";
    case ACE_ERR_IO: return "ACE_ERR_IO";
  }
  return "ACE_UNKNOWN_STATUS";
}

uint64_t ace_set_peer_wait_limit_ns(uint64_t ns) {
  return g_peer_wait_ns.exchange(ns == 0 ? kWaitLimitNs : ns);
}

const char* ace_version(void) { return "0.2.0"; }

const char* ace_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

size_t ace_tables_workspace_size(const ace_layer* layer) {
  if (check_layer(layer, true) != ACE_OK) return 0;
  return tables_workspace_size(*layer);
}

ace_status ace_build_tables(const ace_layer* layers, int n_layers, const ace_table_opts* opts,
                            float* a_gsp, float* a_rcr, float* amax, float* sigma, void* ws,
                            size_t ws_bytes, void* stream) {
  if (!layers || n_layers <= 0 || !opts) return ACE_ERR_INVALID_ARG;
  if (!a_gsp || !a_rcr || !amax) return ACE_ERR_INVALID_ARG;
  if (opts->gsp_norm != ACE_GSP_FRO && opts->gsp_norm != ACE_GSP_SPECTRAL)
    return ACE_ERR_INVALID_ARG;
  if (opts->power_iters < 0 || !(opts->eps >= 0.f)) return ACE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    const ace_status st = check_layer(&layers[l], true);
    if (st != ACE_OK) return st;
    const ace_layer& a = layers[0];
    const ace_layer& b = layers[l];
    if (a.d != b.d || a.E != b.E || a.m != b.m || a.dtype != b.dtype) return ACE_ERR_INVALID_ARG;
  }
  if (layers[0].m > 4096) return ACE_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256)) return ACE_ERR_WORKSPACE;
  return build_tables_impl(layers, n_layers, *opts, a_gsp, a_rcr, amax, sigma, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream));
}

}  // extern "C"
