// ace_internal.h -- host-side declarations shared by the libace translation
// units: the forward workspace layout and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ace.h"

namespace ace {

constexpr int kChunk = 32;        // tokens per compaction chunk (one bit each)
constexpr int kRangeTok = 256;    // tokens per range of the kept-slot counts (8 chunks)
constexpr int kMaxE = 512;        // experts per layer the routing kernel holds
constexpr int kMaxK = 16;         // top-k limit
constexpr int kTileN = 256;       // kept slots per expert tile (GEMM N limit)
constexpr int kRouterBT = 64;     // router GEMM tile: tokens
constexpr int kRouterBE = 64;     // router GEMM tile: experts
constexpr int kRouterBK = 32;     // router GEMM K step
constexpr int kMaxSplitK = 16;
constexpr int kDecodeMaxT = 8;    // token counts served by the decode kernel

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// Split of the router GEMM's K dimension for T tokens: enough CTAs to cover
// the GPU twice, each split a multiple of the K step.
int router_splitk(int T, int d, int E, int num_sms);
// The K split the forward uses for this layer's router (CUDA-core router for
// fp32 layers, tensor-core router for bf16 layers).
int router_splits_for(const ace_layer& L, int T, int num_sms);

// Byte offsets of the forward's scratch arrays inside the caller's
// workspace.  Everything is sized for max_tokens and no skipping.
struct FwdLayout {
  size_t status, part, inv_rms, rw3, tile_done, idx, gate, score, keep, bitmap, range_cnt, rbase,
      counts,
      offsets, n_kept, tiles, n_tiles, slot_token, slot_rank, slot_gate, slot_of, xp, h,
      yslot, total;
  int max_tokens, part_floats, max_tiles;
};
FwdLayout fwd_layout(const ace_layer& L, int max_tokens, int num_sms);

int device_sm_count();
// The argument and shape checks of a layer (need_experts: the expert weights
// are read as well), shared by every entry point.
ace_status validate_layer(const ace_layer* L, bool need_experts);
// Current limit (ns) of the waits in which a CTA waits on other CTAs: the
// decode kernel's grid barriers and the fused expert kernel's wait for a
// tile's h rows.  Read when a call enqueues its kernels.
uint64_t peer_wait_ns();
// Zeroes n_words 32-bit words on the stream (the status block of a call).
cudaError_t launch_clear_words(void* p, int n_words, cudaStream_t s);
ace_status check_fusion(const ace_layer& L, int fusion);

// ---------------------------------------------------------------- launchers
// 1/rms per token, x (nullable); zeroes clear[0 .. n_clear) (n_clear <= 256)
// and zero[0 .. n_zero); w3 (nullable, bf16 layers): gamma (.) w_router as
// three bf16 terms [3][E][d]
cudaError_t launch_rmsnorm(ace_dtype dt, const void* u, int T, int d, const float* gamma,
                           float eps, float* inv_rms, void* x, uint32_t* clear, int n_clear,
                           uint32_t* zero, size_t n_zero, const void* wr, int E, void* w3,
                           cudaStream_t s);
// Tensor-core router (bf16 layers): part[split][t][e] from u [T][d] (bf16),
// 1/rms and the three-term router operand w3 [3][E][d].
int router_tc_splits(int T, int d, int E, int num_sms);
cudaError_t launch_router_tc(const void* u, const float* inv_rms, const void* w3, int T, int d,
                             int E, int splits, float* part, uint32_t* status, int num_sms,
                             cudaStream_t s);
cudaError_t launch_router_logits(ace_dtype dt, const void* u, const float* inv_rms,
                                 const float* gamma, const void* wr, int T, int d, int E,
                                 int splitk, float* part, cudaStream_t s);
struct ScanOut;
struct FuseTables;
cudaError_t launch_topk_mask(const float* part, int splitk, int T, int E, int k,
                             const float* bias, const FuseTables& ft, float tau, int renorm,
                             int32_t* idx, float* gate, float* score, uint8_t* keep,
                             uint32_t* bitmap, int32_t* range_cnt, float* logits_out,
                             uint32_t* status, uint32_t* done_ctr, const ScanOut* so,
                             cudaStream_t s);
// Slot tables and the gathered rows Xp[pos] = x[t]; x rows are x_stride
// elements apart.
cudaError_t launch_scatter_gather(ace_dtype dt, int T, int k, int E, int d, const int32_t* idx,
                                  const float* gate, const uint8_t* keep, const uint32_t* bitmap,
                                  const int32_t* rbase, const void* u, const float* inv_rms,
                                  const float* gamma, int32_t* slot_token, int32_t* slot_rank,
                                  float* slot_gate, int32_t* slot_of, void* xp, uint32_t* status,
                                  cudaStream_t s);
// yslot [S][d] in the layer's storage type
cudaError_t launch_experts_sm100(const ace_layer& L, int cap_slots, const void* xp, void* h,
                                 void* yslot, const int4* tiles, const int32_t* n_tiles,
                                 int max_tiles, const float* slot_gate, uint32_t* status,
                                 int num_sms, cudaStream_t s, cudaEvent_t ev_mid);
// Both expert GEMMs in one persistent kernel (bf16 layers): gate/up items
// first, then down items, each down item waiting for its tile's h rows.
cudaError_t launch_experts_fused(const ace_layer& L, int cap_slots, const void* xp, void* h,
                                 void* yslot, const int4* tiles, const int32_t* n_tiles,
                                 int max_tiles, const float* slot_gate, uint32_t* tile_done,
                                 uint32_t* status, int num_sms, cudaStream_t s);
cudaError_t launch_experts_simt(const ace_layer& L, const void* xp, void* h, void* yslot,
                                const int4* tiles, const int32_t* n_tiles, int max_tiles,
                                const float* slot_gate, cudaStream_t s);
size_t decode_smem_bytes(int T, int d, int m, int k, int E, int num_sms);
bool decode_fits(int T, int d, int m, int k, int E, int num_sms);
cudaError_t launch_decode(const ace_layer& L, int fusion, const void* u, int T, float tau,
                          int renorm,
                          float eps_rms, void* y, float* logits, void* h, int32_t* idx,
                          float* gate, float* score, uint8_t* keep, int32_t* offsets,
                          int32_t* slot_token, int32_t* slot_rank, int32_t* slot_of,
                          int32_t* n_kept, uint32_t* sync, uint32_t* status, bool keep_status,
                          unsigned long long* trace, int num_sms, cudaStream_t s);
size_t tables_workspace_size(const ace_layer& L);
ace_status build_tables_impl(const ace_layer* layers, int n_layers, const ace_table_opts& o,
                             float* a_gsp, float* a_rcr, float* amax, float* sigma, void* ws,
                             size_t ws_bytes, cudaStream_t s);
size_t tau_workspace_size();
cudaError_t launch_tau_quantile(const float* score, int n_tok, int k, long long n_skip,
                                float* tau, void* ws, int num_sms, cudaStream_t s);
// yslot [n_rows][d] and y [T][d] in the storage type dt
cudaError_t launch_combine(ace_dtype dt, int T, int k, int d, const int32_t* slot_of,
                           const void* yslot, int n_rows, void* y, uint32_t* status,
                           cudaStream_t s);

}  // namespace ace
