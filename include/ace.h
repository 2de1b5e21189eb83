/*
 * ace.h -- C ABI of libace: the forward pass of a routed SwiGLU
 * mixture-of-experts layer with ACE per-token expert skipping, and the
 * offline construction of ACE's per-expert tables, on NVIDIA B200 (sm_100a).
 *
 * Method: "ACE: Adaptive Calibration-Free Expert Skipping for MoE-based
 * LLMs" (picx.dev whiteboard summary of arXiv 2609.05228), cited as [ACE]
 * with its section, and the news article "ACE Skips Low-Contribution MoE
 * Experts Per Token" (ainews.surl.tw), cited as [NEWS].
 *
 * Conventions for every entry point
 *   - Pointers marked (device) are CUDA device pointers owned by the caller;
 *     the library never frees, retains or writes through a weight pointer
 *     (checkpoint preservation, [ACE] "Practical Implications").
 *   - The library allocates no device memory: scratch space is the caller's
 *     workspace `ws` of at least the size the matching *_workspace_size
 *     query returns, 256-byte aligned.  A workspace needs no initialisation
 *     and may hold anything between calls: every call brings the words it
 *     shares between CTAs to a known state itself (the decode kernel without
 *     a clearing launch, see ace_moe_forward).
 *   - Weight, gamma, activation and output pointers are 16-byte aligned
 *     (the kernels move them in 16-byte vectors and bulk copies); tables
 *     are 4-byte aligned.  A misaligned pointer is ACE_ERR_INVALID_ARG.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; nothing synchronises the
 *     host except ace_read_status.  No call allocates or synchronises, so
 *     the forward can be captured in a CUDA graph.
 *   - Argument errors are detected on the host before anything is launched
 *     and return ACE_ERR_INVALID_ARG / ACE_ERR_WORKSPACE /
 *     ACE_ERR_UNSUPPORTED.  Launch failures return ACE_ERR_CUDA.  Errors a
 *     kernel detects (an index out of range, a pipeline wait that exceeded
 *     its time limit) set bits in a status word inside the workspace; read
 *     them with ace_read_status.
 *   - Matrices are row-major.  Layouts (with the page's row-vector
 *     convention: W^gate, W^up are d x m and W^down is m x d):
 *       gamma      [d]        fp32   RMSNorm scale (diagonal of Gamma_l)
 *       w_router   [E][d]     dtype  row e is the router vector w_{l,e}
 *       router_bias[E]        fp32   optional, added to the logits
 *       w_gate     [E][m][d]  dtype  w_gate[e][j][i] = W^gate_{l,e}[i][j]
 *       w_up       [E][m][d]  dtype  likewise
 *       w_down     [E][d][m]  dtype  w_down[e][i][j] = W^down_{l,e}[j][i]
 *       u, y       [T][d]     dtype  layer input and output rows
 */
#ifndef ACE_H_
#define ACE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ACE_API __attribute__((visibility("default")))
#else
#define ACE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ACE_OK = 0,
  ACE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer    */
  ACE_ERR_WORKSPACE = 2,    /* workspace missing, too small or misaligned   */
  ACE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed         */
  ACE_ERR_UNSUPPORTED = 4,  /* valid but not implemented (shape, dtype)     */
  ACE_ERR_DEVICE_FAULT = 5, /* a kernel flagged an out-of-range index       */
  ACE_ERR_TIMEOUT = 6,      /* a kernel's bounded wait ran out              */
  ACE_ERR_IO = 7            /* a tables file could not be written or read,
                               or is not an intact tables file              */
} ace_status;

/* device status bits (ace_read_status) */
#define ACE_FLAG_BAD_INDEX 0x1u    /* an expert/slot index outside its range */
#define ACE_FLAG_TIMEOUT 0x2u      /* a pipeline wait exceeded its limit     */
#define ACE_FLAG_OVERFLOW 0x4u     /* more kept slots than the workspace holds */

typedef enum { ACE_BF16 = 0, ACE_F32 = 1 } ace_dtype;

/* GSP norm: Frobenius exactly as printed in [ACE] "Methodology 1", or the
 * spectral norm (largest singular value, power iteration). */
typedef enum { ACE_GSP_FRO = 0, ACE_GSP_SPECTRAL = 1 } ace_gsp_norm;

/* Fusion of the two views' scores s^GSP = g A^GSP(e), s^RCR = g A^RCR(e)
 * into the score c that is compared with tau.  MAX is ACE's rule
 * ([ACE] "3. Conservative Fusion": a slot is skipped only when both views
 * call it low, i.e. the intersection of the two low sets).  The others are
 * the pages' ablations: MIN (skipped when either view calls it low, the
 * union) and MEAN (the arithmetic mean of the two scores) in the fusion
 * ablation (Table 5), and a single view, GSP or RCR, in the component
 * ablation (Table 4).  Gates are non-negative, so c = g F(A^GSP, A^RCR)(e)
 * with F = max, min, mean, first or second. */
typedef enum {
  ACE_FUSE_MAX = 0,
  ACE_FUSE_MIN = 1,
  ACE_FUSE_MEAN = 2,
  ACE_FUSE_GSP = 3,
  ACE_FUSE_RCR = 4
} ace_fusion;

/* One MoE layer: shapes, weights (device) and its ACE table. */
typedef struct {
  int d;                   /* hidden size                                  */
  int E;                   /* routed experts                               */
  int m;                   /* expert intermediate size                     */
  int k;                   /* experts per token (top-k), 1 <= k <= E, <= 16 */
  ace_dtype dtype;         /* storage and activation type                  */
  const float* gamma;      /* [d]                                          */
  const void* w_router;    /* [E][d]                                       */
  const float* router_bias;/* [E] or NULL                                  */
  const void* w_gate;      /* [E][m][d]                                    */
  const void* w_up;        /* [E][m][d]                                    */
  const void* w_down;      /* [E][d][m]                                    */
  const float* amax;       /* [E] max(A^GSP, A^RCR) from ace_build_tables,
                              the table of ACE_FUSE_MAX; NULL only for
                              callers that want the raw gates as scores
                              (1.0 then), or that give a_gsp and a_rcr      */
  const float* a_gsp;      /* [E] A^GSP, or NULL; needed by ACE_FUSE_MIN,
                              _MEAN and _GSP                                */
  const float* a_rcr;      /* [E] A^RCR, or NULL; needed by ACE_FUSE_MIN,
                              _MEAN and _RCR                                */
} ace_layer;

/* Forward options. */
typedef struct {
  float tau;           /* skip threshold: slot i > 0 is skipped iff its
                          fused score c_i < tau ([ACE] "Conservative
                          Fusion"; tau comes from the caller, one per layer
                          and skip budget, [ACE] "Efficiency Results")    */
  int renorm_topk;     /* 1: gates renormalised over the top-k (the gate of
                          slot i is p_i / sum_topk p); 0: raw softmax p_i    */
  ace_fusion fusion;   /* how c is formed (ace_fusion); MAX reads
                          layer->amax when it is set, else
                          max(a_gsp, a_rcr); the other rules read a_gsp
                          and/or a_rcr and return ACE_ERR_INVALID_ARG when
                          a table they need is NULL                       */
  float eps_rms;       /* RMSNorm epsilon (1e-6 in the shipped workloads)  */
} ace_fwd_opts;

/* Optional copies of the forward's intermediates (device pointers, each may
 * be NULL).  Sizes use the call's T, k, E. */
typedef struct {
  int32_t* topk_idx;       /* [T][k] expert of slot (t, i); i = 0 is top-1 */
  float* gate;             /* [T][k] gate g_{t,i}                          */
  float* score;            /* [T][k] fused score c (opts->fusion)          */
  uint8_t* keep;           /* [T][k] 1 = kept, 0 = skipped                 */
  int32_t* expert_offsets; /* [E+1] first kept slot of each expert         */
  int32_t* slot_token;     /* [T*k] token of each kept slot (first n_kept)  */
  int32_t* slot_rank;      /* [T*k] rank i of each kept slot               */
  int32_t* n_kept;         /* [1]   number of kept slots                   */
  float* logits;           /* [T][E] router logits (bias included)          */
  /* Optional cudaEvent_t handles (passed as void*) recorded on the call's
   * stream right before the gate/up expert GEMM, between it and the down
   * GEMM, and right after the down GEMM: live kernel timing for profilers
   * and benchmarks.  When both GEMMs run as one kernel (small slot tiles:
   * T k < 128 E), "mid" is recorded after that kernel, like "end".  NULL =
   * not recorded. */
  void* ev_experts_begin;
  void* ev_experts_mid;
  void* ev_experts_end;
  /* Optional trace (device, uint64 [grid][8]): the decode kernel (T <= 8)
   * writes the %globaltimer value (ns) of each CTA at its phase boundaries:
   * start, x ready, after the first grid barrier, after the slot list,
   * after gate/up, after the second barrier, end, and (entry 7) after the
   * first token's sum of squares.  NULL = off. */
  unsigned long long* trace;
} ace_debug_out;

/* Table-build options ([ACE] "Methodology 1-2"). */
typedef struct {
  ace_gsp_norm gsp_norm; /* ACE_GSP_FRO (default) or ACE_GSP_SPECTRAL       */
  float eps;             /* epsilon of the layer normalisations and of RCR  */
  float rho;             /* RCR prototype scale rho_l (1.0 by default)      */
  int power_iters;       /* power-iteration steps (200 by default)          */
} ace_table_opts;

/* ------------------------------------------------------------------------
 * ace_workspace_size
 *   Bytes of workspace ace_moe_forward / ace_moe_scores need for `layer`
 *   and up to `max_tokens` tokens per call.  Returns 0 for an invalid
 *   layer.  The size covers the worst case (no slot skipped).
 * ---------------------------------------------------------------------- */
ACE_API size_t ace_workspace_size(const ace_layer* layer, int max_tokens);

/* ------------------------------------------------------------------------
 * ace_moe_forward -- one MoE layer forward with ACE skipping.
 *   [ACE] "Theoretical Foundation" (x = xbar Gamma and the SwiGLU expert
 *   f_{l,e}), "Methodology 1-2" (scores s = g A), "3. Conservative Fusion"
 *   (max-fusion, top-1 always kept); [NEWS] (online stage: table lookups,
 *   the token's gate and scalar operations).
 *   Per token t: x_t = RMSNorm(u_t) * gamma; logits x_t . w_e (+ b_e); the
 *   top-k experts by logit (ties: lower index first); gates; scores
 *   c = g * F(A^GSP, A^RCR)(e) by opts->fusion (ACE: F = max, the table
 *   layer->amax); slot i is kept iff i == 0 or !(c < tau); the kept
 *   slots are grouped by expert (then token), run through their SwiGLU
 *   experts, and y_t = sum over kept i, in rank order, of g_i f_{e_i}(x_t).
 *   Skipped slots drop out without re-normalising the others.
 *   u (device) [T][d], y (device) [T][d], both layer->dtype; they must not
 *   overlap.  0 <= T <= max_tokens of the workspace.  T == 0 is a no-op.
 *   dbg may be NULL.
 *   bf16 layers run the expert GEMMs on tcgen05 tensor cores and need
 *   d % 128 == 0 and m % 128 == 0; fp32 layers use CUDA cores.
 *   Calls of 1-8 tokens on bf16 layers (d <= 2048) take the decode route:
 *   one cooperative kernel whose grid barriers count in 64 bytes of the
 *   workspace's status block; its last CTA writes the status word and
 *   leaves those words zeroed and marked for the next call, so the route
 *   launches nothing before the kernel.  The kernel may start while the
 *   previous kernel of the stream is ending (programmatic stream
 *   serialisation), but it reads and writes no global memory until that
 *   kernel has completed, so stream order holds for every argument.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_moe_forward(const ace_layer* layer, const void* u, int T,
                           const ace_fwd_opts* opts, void* y, void* ws,
                           size_t ws_bytes, ace_debug_out* dbg, void* stream);

/* ------------------------------------------------------------------------
 * ace_stack_workspace_size -- bytes of workspace ace_moe_stack_forward
 *   needs for the n_layers layers (same d and dtype) and up to max_tokens
 *   tokens; 0 for invalid layers.
 * ---------------------------------------------------------------------- */
ACE_API size_t ace_stack_workspace_size(const ace_layer* layers, int n_layers, int max_tokens);

/* ------------------------------------------------------------------------
 * ace_moe_stack_forward -- n_layers MoE layers in sequence, the output of
 *   each the input of the next (u_{l+1} = y_l), as in a decode step through
 *   the model's MoE layers ([ACE] "Efficiency Results", Table 7: the
 *   per-token latency over every layer).  The paper has no entry point of
 *   its own for this; it is the layer forward repeated, each layer with its
 *   own options opts[l] (tau per layer).  Every layer's forward is exactly
 *   ace_moe_forward's (same kernels, same results), so the stack equals
 *   n_layers calls with the outputs fed back.  The intermediate
 *   activations alternate between two [T][d] buffers inside ws; u (device)
 *   [T][d] is only read, y (device) [T][d] receives the last layer's
 *   output; they must not overlap.  The status word (ace_read_status on
 *   ws) holds the flags of every layer of the call.  Asynchronous; no
 *   allocation, no synchronisation, so it can be captured in a CUDA graph.
 *   Argument errors (any layer's) return before anything is launched.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_moe_stack_forward(const ace_layer* layers, int n_layers, const void* u,
                                         int T, const ace_fwd_opts* opts, void* y, void* ws,
                                         size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * ace_moe_scores -- only the routing half of the forward: fused scores
 *   c (opts->fusion; the gate alone under ACE_FUSE_MAX when layer->amax,
 *   a_gsp and a_rcr are all NULL) of every slot,
 *   for building tau by quantile mapping ([ACE] "Efficiency Results",
 *   Table 6).  score (device) [T][k] fp32, column 0 = top-1 slot;
 *   topk_idx (device) [T][k] int32 or NULL.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_moe_scores(const ace_layer* layer, const void* u, int T,
                          const ace_fwd_opts* opts, float* score,
                          int32_t* topk_idx, void* ws, size_t ws_bytes,
                          void* stream);

/* ------------------------------------------------------------------------
 * ace_moe_route -- the routing half of the forward with its decisions, the
 *   first step of expert-parallel dispatch ([ACE] "Conclusion", future
 *   directions: distributed expert dispatch): a rank routes its own tokens,
 *   then sends each kept slot to the rank that owns the slot's expert.
 *   Same kernels as ace_moe_forward, so the same bits.
 *   x (device) [T][d] layer->dtype, 16-byte aligned: the experts' input
 *   rows (bf16(x) for bf16 layers, x for fp32 layers); idx (device) [T][k]
 *   int32 experts, column 0 = top-1; gate (device) [T][k] fp32 gates;
 *   keep (device) [T][k] uint8, 1 = kept (top-1 always).  Workspace: at
 *   least ace_workspace_size(layer, T) bytes.  The expert weights are not
 *   read and may be NULL.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_moe_route(const ace_layer* layer, const void* u, int T,
                                 const ace_fwd_opts* opts, void* x, int32_t* idx,
                                 float* gate, uint8_t* keep, void* ws, size_t ws_bytes,
                                 void* stream);

/* ------------------------------------------------------------------------
 * ace_experts_workspace_size -- bytes of workspace ace_moe_experts needs for
 *   up to max_slots slots of `layer`; 0 for an invalid expert layer.
 *
 * ace_moe_experts -- the SwiGLU experts of `layer` on S kept slots grouped by
 *   expert, the owner's step of expert-parallel dispatch:
 *     yslot[s] = slot_gate[s] * f_e(xp[s])  for offsets[e] <= s < offsets[e+1]
 *   with f_e as in ace_moe_forward ([ACE] "Theoretical Foundation", the
 *   SwiGLU expert).  `layer` holds only the experts the caller owns (E of
 *   them, d, m, dtype and the three expert matrices); the router, gamma and
 *   k are not read.  xp (device) [S][d] layer->dtype, 16-byte aligned;
 *   offsets (device) [E+1] int32, rising from 0 to S (otherwise
 *   ACE_FLAG_BAD_INDEX is raised and nothing is computed); slot_gate
 *   (device) [S] fp32; yslot (device) [S][d] layer->dtype, 16-byte aligned.
 *   Same kernels and numerics as the forward's expert GEMMs (fp32
 *   accumulation; h and each yslot row rounded to the storage type).
 *   Device flags: ace_read_status on ws.
 * ---------------------------------------------------------------------- */
ACE_API size_t ace_experts_workspace_size(const ace_layer* layer, int max_slots);
ACE_API ace_status ace_moe_experts(const ace_layer* layer, const void* xp, int S,
                                   const int32_t* offsets, const float* slot_gate,
                                   void* yslot, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * ace_moe_combine -- the forward's combine on slot outputs the caller
 *   gathered (in expert-parallel dispatch: the outputs of a rank's kept
 *   slots, back from their experts' owners):
 *     y_t = sum over i = 0 .. k-1 with slot_of[t][i] >= 0, in that order, of
 *           yslot[slot_of[t][i]]
 *   in fp32, rounded once to dtype ([ACE] "Theoretical Foundation": the
 *   gate-weighted sum of the kept experts; the gates are already in yslot,
 *   skipped slots drop out without re-normalising).
 *   slot_of (device) [T][k] int32, -1 for a skipped slot; yslot (device)
 *   [n_rows][d] dtype, 16-byte aligned (ace_moe_experts' output); y (device)
 *   [T][d] dtype, 16-byte aligned; d a multiple of 8 (bf16) or 4 (fp32).
 *   An index >= n_rows raises ACE_FLAG_BAD_INDEX and drops out.  ws: at
 *   least 256 bytes (its status word; ace_read_status).
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_moe_combine(int T, int k, int d, ace_dtype dtype, const int32_t* slot_of,
                                   const void* yslot, int n_rows, void* y, void* ws,
                                   size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * ace_moe_decode_noalloc -- the decode forward (1 <= T <= 8 tokens, bf16
 *   layers) for callers that cannot allocate device memory.  The paper has
 *   no counterpart: this is a deployment variant of ace_moe_forward.
 *   Some callers cannot call cudaMalloc: plugins inside a host framework
 *   that owns every device allocation and gives them no allocator, or
 *   serving loops that must not allocate once running (an allocation can
 *   synchronise the device).  This entry point takes the inputs and outputs
 *   from the caller (layer weights and amax table, u [T][d], y [T][d],
 *   device pointers as for ace_moe_forward) and uses, instead of a
 *   workspace, a scratch array of 512 KiB compiled into the library
 *   (static device memory, present on every GPU that loads the library
 *   until the process exits).  It allocates nothing and calls no allocating
 *   library routine.
 *   - The first call on a device, with that device current, looks up the
 *     array's device address once; make that first call before any stream
 *     capture.
 *   - Every call shares the one array and leaves its last contents there;
 *     each call zeroes what must start at zero.  Calls whose GPU work
 *     overlaps (on different streams or host threads) race on the array:
 *     serialise them.
 *   - The layer checks and shape rule are ace_moe_forward's (bf16 layers
 *     need d % 128 == 0 and m % 128 == 0).  Shapes whose scratch exceeds the
 *     array (router logits T x E fp32, gated intermediates T x k x m bf16,
 *     slot tables), non-bf16 layers and shapes the decode kernel does not
 *     serve return ACE_ERR_UNSUPPORTED before anything is launched; bad
 *     pointers return ACE_ERR_INVALID_ARG.
 *   - Device-detected flags go to a status word in the array; read them
 *     with ace_noalloc_read_status.  The kernel's waits are bounded as
 *     elsewhere.
 *   Results equal ace_moe_forward's for the same inputs.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_moe_decode_noalloc(const ace_layer* layer, const void* u, int T,
                                          const ace_fwd_opts* opts, void* y, void* stream);

/* ------------------------------------------------------------------------
 * ace_noalloc_read_status -- synchronise `stream` and return the device
 *   status word of the most recent ace_moe_decode_noalloc call on the
 *   current device (ACE_FLAG_* bits in *flags, which may be NULL), read
 *   from the library's scratch array; ACE_ERR_TIMEOUT / ACE_ERR_DEVICE_FAULT
 *   when the corresponding bit is set, else ACE_OK.  Allocates nothing.
 *   Like the array itself, the word is shared by every call on the device:
 *   read it before the next call is enqueued.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_noalloc_read_status(uint32_t* flags, void* stream);

/* ------------------------------------------------------------------------
 * ace_tables_workspace_size
 *   Bytes of workspace ace_build_tables needs for layers shaped like
 *   `layer` (d, E, m, dtype).
 * ---------------------------------------------------------------------- */
ACE_API size_t ace_tables_workspace_size(const ace_layer* layer);

/* ------------------------------------------------------------------------
 * ace_build_tables -- offline ACE statistics of n_layers layers (all with
 *   the same d, E, m, dtype), [ACE] "Methodology 1" (GSP) and
 *   "Methodology 2" (RCR):
 *     a^up   = ||Gamma W^up|| ||Gamma W^gate W^down||
 *     a^gate = ||Gamma W^gate|| ||Gamma W^up W^down||
 *     A^GSP(e) = sqrt(a^up a^gate)_e / (mean_j sqrt(a^up a^gate)_j + eps)
 *     q_e = (w_e - mean_j w_j) / (RMS(w_e - mean_j w_j) + eps) * rho
 *     A^RCR(e) = a~_e / (mean_j a~_j + eps), a~_e = ||f_e(q_e)|| / (||q_e|| + eps)
 *   Outputs (device, fp32, [n_layers][E]): a_gsp, a_rcr, amax = max of the
 *   two (the table ace_moe_forward reads).  sigma (device, [n_layers][E][3]
 *   or NULL) receives the largest singular values of Gamma W^gate,
 *   Gamma W^up and W^down (the constants of the bound on ||f(x)|| in
 *   [ACE] "Theoretical Foundation"), by power iteration from the all-ones
 *   vector in R^m for opts->power_iters steps.  Weights are only read.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_build_tables(const ace_layer* layers, int n_layers,
                            const ace_table_opts* opts, float* a_gsp,
                            float* a_rcr, float* amax, float* sigma, void* ws,
                            size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Tables files: ace_build_tables's outputs kept on disk, so a table build
 *   (which depends only on the frozen weights, [ACE] "Practical
 *   Implications") is done once and reloaded.  Host pointers, fp32:
 *   a_gsp, a_rcr, amax [n_layers][E]; sigma [n_layers][E][3] or NULL.
 *   Format: a 32-byte header (magic "ACETBL\0\x01", version 1, n_layers,
 *   E, flags bit 0 = sigma present, FNV-1a 64 hash of the payload), then
 *   the arrays in that order, little-endian.
 *
 * ace_tables_save -- writes the file under path + ".tmp" and renames it
 *   into place (a crash never leaves a torn file).  ACE_ERR_IO when the
 *   file cannot be written.
 * ace_tables_info -- the file's n_layers, E and whether it holds sigma (any
 *   output pointer may be NULL).  ACE_ERR_IO for a missing, truncated,
 *   corrupted (hash mismatch) or foreign file.
 * ace_tables_load -- reads a file of exactly n_layers x E into the arrays;
 *   ACE_ERR_INVALID_ARG when the shape differs or sigma is asked for and
 *   absent, ACE_ERR_IO as for ace_tables_info.  Nothing is written to the
 *   arrays unless the whole file checks out.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_tables_save(const char* path, int n_layers, int E, const float* a_gsp,
                                   const float* a_rcr, const float* amax, const float* sigma);
ACE_API ace_status ace_tables_info(const char* path, int* n_layers, int* E, int* has_sigma);
ACE_API ace_status ace_tables_load(const char* path, int n_layers, int E, float* a_gsp,
                                   float* a_rcr, float* amax, float* sigma);

/* ------------------------------------------------------------------------
 * ace_tau_workspace_size -- bytes of workspace ace_tau_quantile needs
 *   (a constant: the selection state and four 256-bin histograms).
 * ---------------------------------------------------------------------- */
ACE_API size_t ace_tau_workspace_size(void);

/* ------------------------------------------------------------------------
 * ace_tau_quantile -- quantile mapping of a skip budget to the threshold,
 *   on the device ([ACE] "Efficiency Results", Table 6: the threshold for a
 *   target skip rate is read off the score distribution of calibration
 *   tokens).
 *   score (device) [n_tok][k] fp32: a score pool as ace_moe_scores writes
 *   it, column 0 the top-1 slot, which is never a candidate.  The
 *   candidates are the other n_tok * (k - 1) scores; sorted ascending
 *   c_(1) <= ... <= c_(N), *tau = c_(n_skip + 1), so exactly n_skip slots of
 *   the pool satisfy c < tau when no scores tie (with ties, fewer).
 *   n_skip <= 0 gives c_(1) (nothing skipped); n_skip >= N, or N == 0,
 *   gives +inf (every candidate skipped).  The result is one of the pool's
 *   values, bit for bit: an exact radix select on the order-preserving
 *   integer keys of the floats (NaN scores order above +inf).
 *   tau (device) receives one fp32.  ws (device, 256-byte aligned,
 *   >= ace_tau_workspace_size() bytes) is scratch; its contents need no
 *   initialisation.  n_tok >= 0, 1 <= k <= 16; NULL score (n_tok > 0) or
 *   tau returns ACE_ERR_INVALID_ARG, a short or misaligned ws
 *   ACE_ERR_WORKSPACE.  Asynchronous on `stream`; allocates nothing.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_tau_quantile(const float* score, int n_tok, int k, int64_t n_skip,
                                    float* tau, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * ace_read_status -- synchronise `stream` and return the device status
 *   word that the most recent call using `ws` left there (ACE_FLAG_* bits in
 *   *flags; every forward, scores or tables call clears it when it starts).
 *   Returns ACE_ERR_TIMEOUT / ACE_ERR_DEVICE_FAULT when the corresponding
 *   bit is set, else ACE_OK.  flags may be NULL.
 * ---------------------------------------------------------------------- */
ACE_API ace_status ace_read_status(void* ws, size_t ws_bytes, uint32_t* flags,
                           void* stream);

/* Human-readable name of a status code (static storage). */
ACE_API const char* ace_status_str(ace_status s);

/* ------------------------------------------------------------------------
 * ace_set_peer_wait_limit_ns -- time limit of the waits in which one CTA of
 *   a kernel waits for other CTAs of the same launch: the decode kernel's
 *   two grid barriers (T <= 8) and, in the prefill's fused expert kernel, a
 *   down item's wait for the h rows of its tile.  The paper has no
 *   counterpart: it is a robustness setting of this implementation.
 *   Default 2 s (ns == 0 restores it).  A wait that runs out sets
 *   ACE_FLAG_TIMEOUT in the call's status word; the kernel then lets every
 *   copy it issued land, frees its tensor memory and returns, so the
 *   context stays usable and the next call runs normally (outputs of the
 *   timed-out call are undefined).  Process-wide; read when a call enqueues
 *   its kernels, so a captured CUDA graph keeps the value of its capture.
 *   Waits inside one CTA (on its own copies and MMAs) keep the fixed 2 s
 *   bound.  Returns the previous limit.
 * ---------------------------------------------------------------------- */
ACE_API uint64_t ace_set_peer_wait_limit_ns(uint64_t ns);

/* Name and description of the CUDA runtime error behind the most recent
 * ACE_ERR_CUDA returned on the calling thread ("no error" if none), static
 * storage. */
ACE_API const char* ace_last_cuda_error(void);

/* Library version, "major.minor.patch" (static storage). */
ACE_API const char* ace_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ACE_H_ */
