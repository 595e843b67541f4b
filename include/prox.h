/*
 * prox.h -- C ABI of the B200 (sm_100a) Prox sparse SwiGLU FFN decode step.
 *
 * Source of every operation below: "Prox: Training-Free FFN Activation
 * Sparsity via Approximate Intermediate-Channel Salience in LLMs" (Liu et al.),
 * cited as *Prox* with its section or equation.
 *
 * Conventions shared by all entry points
 * --------------------------------------
 *  - Pointers are DEVICE pointers unless the parameter name ends in `_host`.
 *  - bf16 and fp16 values are passed as their uint16_t bit patterns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    All work is enqueued on it in stream order; functions whose comment says
 *    "synchronises" wait for the stream before returning.
 *  - The caller owns every buffer it passes and must keep it alive until the
 *    enqueued work has finished.  The library owns the layer handle, its
 *    repacked weights and its workspace (allocated in prox_layer_create, freed
 *    in prox_layer_destroy); prox_ffn_forward and prox_dense_ffn allocate
 *    nothing and never synchronise.
 *  - Weight shapes are in math layout: W_gate, W_up are [d_model, d_ff] and
 *    W_down is [d_ff, d_model], all row-major.  Activations are fp32.
 *  - Shape rules (else PROX_EINVAL, checked before any launch):
 *    d_model > 0 and d_model % 128 == 0; d_ff > 0 and d_ff % 32 == 0;
 *    d_model <= 16384; d_ff <= 32768; 1 <= k <= d_ff; pointers 16-byte aligned.
 *    Stage 1 keeps a table entry per kept input row of its share in shared
 *    memory beside its copy ring (at least two 8-row tiles per warp), which
 *    bounds ceil(d_ff/512) * d_model <= 15535 * (number of SMs), and the
 *    scoring takes one channel per thread, which bounds d_ff <= 512 * (number
 *    of SMs): on a 148-SM B200 every shape the rules above admit (at most
 *    64 * 16384 = 1.05 M <= 2.29 M).  On a device with fewer SMs
 *    prox_layer_create returns PROX_EUNSUPPORTED beyond them.
 *  - Errors: every call returns a prox_status; prox_last_error() copies a
 *    message for the calling thread's last failure.  No C++ exception crosses
 *    this boundary.  Device-side checks (an index out of range in a caller's
 *    mask, a bounded wait that ran out) never trap: they set the layer's error
 *    word, read with prox_layer_error().
 *  - A layer handle is used by one stream at a time (its workspace is shared
 *    by the calls on it).
 */
#ifndef PROX_H_
#define PROX_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PROX_API __attribute__((visibility("default")))
#else
#define PROX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum prox_status {
  PROX_OK = 0,
  PROX_EINVAL = 1,       /* bad argument (shape, pointer, k, s1 ...) */
  PROX_ENOMEM = 2,       /* device allocation failed */
  PROX_ECUDA = 3,        /* a CUDA runtime call failed */
  PROX_EUNSUPPORTED = 4, /* device is not sm_100 or a limit is exceeded */
  PROX_EDEVICE = 5       /* a device-side check fired (see prox_layer_error) */
} prox_status;

/* Device error word bits (prox_layer_error). */
#define PROX_DEVERR_MASK_INDEX 0x1  /* a channel index outside [0, d_ff) */
#define PROX_DEVERR_WAIT_TIMEOUT 0x2 /* a bounded pipeline wait ran out */

typedef struct prox_layer prox_layer; /* opaque */

/* Static description of a created layer (all host values). */
typedef struct prox_layer_info {
  int d_model, d_ff, group, k, max_batch;
  float tau_x;
  int stage1_col_slices, stage1_ctas; /* Stage-1 column slices and CTAs */
  int stage2_ctas, stage2_ring_slots;      /* Stage-2 grid and TMA ring depth */
  size_t weight_bytes;    /* bf16 gate/up records + bf16 W_down             */
  size_t proxy_bytes;     /* INT4 codes + fp16 scales                        */
  size_t workspace_bytes; /* scratch owned by the handle                     */
  int mask_mode;          /* PROX_MASK_TOPK or PROX_MASK_THRESHOLD           */
  float tau_s;            /* Stage-2 score threshold (threshold mode)        */
  int activation;         /* PROX_ACT_*                                      */
  int stage2_source;      /* PROX_STAGE2_EXACT or PROX_STAGE2_PROXY_VALUES   */
} prox_layer_info;

/* Stage-2 channel rule: per-token top-k (Prox App. A.6), or the fixed
 * layer-wise score threshold m_s = 1[|s~_j| >= tau_s] of Prox §4.1 (a
 * token-adaptive channel count). */
#define PROX_MASK_TOPK 0
#define PROX_MASK_THRESHOLD 1

/* Gate activation of the GLU, used by the Stage-1 score, Stage 2 and the
 * dense baseline alike.  SwiGLU (Prox §2.1) is the default; Prox §5 applies
 * the method unchanged to GeGLU FFNs, whose gate is GELU, here either
 * GELU(z) = z Phi(z) (Phi the standard normal CDF) or its tanh form
 * 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))) (Hendrycks & Gimpel,
 * "Gaussian Error Linear Units", §2). */
#define PROX_ACT_SILU 0
#define PROX_ACT_GELU_TANH 1
#define PROX_ACT_GELU_ERF 2

/* Where Stage 2 takes the selected channels' values from.  EXACT is the
 * method (Prox §4.1).  PROXY_VALUES is ablation A3 of Prox §5.2: Stage 2
 * skips the exact gate/up projections and feeds the selected Stage-1 proxy
 * values s~_j = act(g~_j) u~_j straight into the down projection,
 * y = sum_{j in S} s~_j W_down[j, :]. */
#define PROX_STAGE2_EXACT 0
#define PROX_STAGE2_PROXY_VALUES 1

/* ------------------------------------------------------------------------
 * Offline preparation
 * ------------------------------------------------------------------------ */

/* INT4 proxy of one weight matrix (Prox §4.3 "Hardware-Aware Implementation":
 * symmetric INT4 proxies of W_up and W_gate kept resident on the GPU; this
 * build quantises in groups of `group` consecutive input rows per channel).
 *
 * For every group g of rows and channel j:
 *   amax = max_{i in g} |W[i,j]|,  S[g,j] = fp16_nearest_even(amax / 7),
 *   Q[i,j] = clamp(round_half_even(W[i,j] / S[g,j]), -7, 7)   (0 when S = 0).
 * W: bf16 [d_model, d_ff].  codes: uint8 [d_model, d_ff/2]; byte b of row i
 * holds channel 2b in its low nibble and 2b+1 in its high nibble, each stored
 * as Q + 8.  scales: fp16 [d_model/group, d_ff].  group must be 128.
 * amax/7 must be finite in fp16 (|W| < 458752).  Stream-ordered; no sync. */
PROX_API prox_status prox_pack_proxy(const uint16_t* W, int d_model, int d_ff, int group,
                            uint8_t* codes, uint16_t* scales, void* stream);

/* Per-layer Stage-1 input threshold (Prox App. A.7 "Calibration data and
 * scale": the threshold is the empirical quantile of the calibration
 * activations; §4.1 uses it as tau_x).
 *
 * tau = the order statistic of rank floor(s1 * n) (0-based, ascending) of the
 * n = n_tok * d_model values |X_cal|; s1 = 0 gives tau = 0.  Exact (radix
 * select on the fp32 bit patterns).  X_cal: fp32 [n_tok, d_model] on the
 * device.  tau_host: one float written on return.  Allocates its scratch
 * (a few KB) stream-ordered and synchronises the stream. */
PROX_API prox_status prox_calibrate_thresholds(const float* X_cal, int n_tok, int d_model, float s1,
                                      float* tau_host, void* stream);

/* The calibration above without any allocation.  The Prox pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory at the moment they calibrate -- a host process whose device
 * memory belongs to another allocator (a serving framework that has reserved
 * it all for its own pool), or a latency-critical path where cudaMalloc's
 * implicit device-wide synchronisation and cudaMallocAsync's pool growth are
 * not acceptable.  Same quantile, same exactness as
 * prox_calibrate_thresholds.  Its scratch is a fixed static __device__ array
 * of 2056 uint32 (8 KB) per device, which every device that loads the
 * library holds until the process exits.  Set-up: the first call made on a
 * device (with that device current) looks up the array's device address with
 * cudaGetSymbolAddress and caches it per device and CUDA context.  A device
 * reset (cudaDeviceReset) or a new primary context makes the next call look
 * the address up again.
 * Every call zeroes the histogram it needs before counting, so nothing has to
 * start at zero.  Calls that overlap on one device (other streams, other
 * threads) share that scratch and race: serialise them.  X_cal: fp32
 * [n_tok, d_model] in device memory of the current device, 16-byte aligned;
 * n_tok * d_model must stay below 2^31 (the counters are 32-bit), else
 * PROX_EINVAL with a message.  tau_dev: one float in device memory of the
 * current device, written in stream order (nothing synchronises).  A pointer
 * to host memory or to another device gives PROX_EINVAL.  Allocates nothing:
 * no cudaMalloc, cudaMallocAsync or cudaFree. */
PROX_API prox_status prox_calibrate_thresholds_noalloc(const float* X_cal, int n_tok, int d_model,
                                                       float s1, float* tau_dev, void* stream);

/* ------------------------------------------------------------------------
 * Layer handle
 * ------------------------------------------------------------------------ */

/* Repack one SwiGLU FFN layer into library-owned buffers:
 *  - gate/up channel records: record j = [W_gate[:, j] | W_up[:, j]], bf16;
 *  - W_down rows (bf16 [d_ff, d_model], unchanged);
 *  - INT4 proxies of W_gate and W_up (prox_pack_proxy), interleaved so that
 *    one input row i of both proxies is a single contiguous run of d_ff bytes;
 *  - workspace for max_batch tokens.
 * tau_x: Stage-1 threshold; k: channels kept per token by the top-k mask.
 * Inputs may be freed once the call returns (it synchronises `stream`). */
PROX_API prox_status prox_layer_create(const uint16_t* W_gate, const uint16_t* W_up,
                              const uint16_t* W_down, int d_model, int d_ff, float tau_x,
                              int k, int max_batch, void* stream, prox_layer** out_host);

/* Frees the layer's device buffers (on the layer's device, switching to it
 * and back if another one is current) and the handle.  The frees are
 * cudaFree calls, which wait for work still running on the device.  NULL is
 * accepted (PROX_OK); the handle may not be used afterwards. */
PROX_API prox_status prox_layer_destroy(prox_layer* layer);

/* Change the threshold or k of an existing layer (host-side; affects calls
 * enqueued afterwards).  tau_x must be finite and >= 0, k in [1, d_ff], else
 * PROX_EINVAL and the layer is unchanged. */
PROX_API prox_status prox_layer_set_tau(prox_layer* layer, float tau_x);
PROX_API prox_status prox_layer_set_k(prox_layer* layer, int k);

/* Chooses the Stage-2 rule: PROX_MASK_TOPK (uses k) or PROX_MASK_THRESHOLD
 * (uses tau_s, a finite value >= 0; Prox §4.1).  Host only. */
PROX_API prox_status prox_layer_set_mask(prox_layer* layer, int mode, float tau_s);

/* Chooses the gate activation (PROX_ACT_*; else PROX_EINVAL).  Host only;
 * takes effect from the next enqueued call. */
PROX_API prox_status prox_layer_set_activation(prox_layer* layer, int act);

/* Chooses the Stage-2 value source of prox_ffn_forward and
 * prox_ffn_forward_host (PROX_STAGE2_*; else PROX_EINVAL).  Host only.
 * prox_forward_with_mask and prox_dense_ffn always compute exact values. */
PROX_API prox_status prox_layer_set_stage2(prox_layer* layer, int source);

/* Copies the layer's shapes, current settings, launch geometry and byte
 * counts into info_host (host memory, caller-owned).  Host only; NULL
 * arguments give PROX_EINVAL. */
PROX_API prox_status prox_layer_get_info(const prox_layer* layer, prox_layer_info* info_host);

/* Reads (and clears) the layer's device error word; synchronises `stream`. */
PROX_API prox_status prox_layer_error(prox_layer* layer, int32_t* word_host, void* stream);

/* Realised statistics accumulated since the last call (Prox App. A.7
 * "Runtime sparsity"): the sum of n_x over tokens, the number of tokens and
 * the sum of selected Stage-2 channels (realised s1 = 1 - sum_nx/(tokens*d),
 * s2 = 1 - sum_sel/(tokens*d_ff)).  Any output may be NULL.  Synchronises
 * `stream` and resets. */
PROX_API prox_status prox_layer_stats(prox_layer* layer, int64_t* sum_nx_host, int64_t* tokens_host,
                             int64_t* sum_sel_host, void* stream);

/* ------------------------------------------------------------------------
 * Cost model and sparsity allocation (host only: no device work, no stream)
 * ------------------------------------------------------------------------ */

/* Effective FFN sparsity of a (s1, s2) pair under the normalised cost model
 * of Prox §4.2: the dense gate, up and down projections cost one unit each
 * (C_Dense = 3); Stage 1 runs two INT4 proxy projections over the kept
 * (1 - s1) share of the inputs at alpha units each, Stage 2 three exact
 * projections over the kept (1 - s2) share of the channels:
 *   C_Prox = 2 alpha (1 - s1) + 3 (1 - s2),  e = 1 - C_Prox / 3
 *          = s2 - 2 alpha (1 - s1) / 3.
 * s1, s2 in [0, 1] and alpha >= 0 (finite), else PROX_EINVAL. */
PROX_API prox_status prox_effective_sparsity(double s1, double s2, double alpha, double* e_host);

/* The allocation policy of Prox §4.2 (operating points in App. A.4): for a
 * target effective sparsity e, set s2 = s_ref and solve the relation above
 * for s1; if that s1 lies outside [s1_min, s1_max], clamp it to the nearer
 * bound and re-solve s2 = e + 2 alpha (1 - s1) / 3.  The paper's setting is
 * alpha = 1/3, s_ref = 0.7, [s1_min, s1_max] = [0, 0.7].
 * PROX_EINVAL when alpha <= 0, s_ref is outside [0, 1], the bounds are not
 * 0 <= s1_min <= s1_max <= 1, any argument is not finite, or the re-solved
 * s2 leaves [0, 1] (no allocation within the bounds reaches e). */
PROX_API prox_status prox_allocate_sparsity(double e, double alpha, double s_ref, double s1_min,
                                            double s1_max, double* s1_host, double* s2_host);

/* Runtime sparsity from accumulated mask counts (Prox App. A.7, "Runtime
 * sparsity"), with the counts prox_layer_stats returns:
 *   s1^ = 1 - sum_nx / (tokens d_model),  s2^ = 1 - sum_sel / (tokens d_ff),
 *   e^  = s2^ - 2 alpha (1 - s1^) / 3.
 * tokens >= 1, 0 <= sum_nx <= tokens d_model, 0 <= sum_sel <= tokens d_ff,
 * d_model, d_ff >= 1, alpha >= 0 (finite), else PROX_EINVAL.  Any output may
 * be NULL. */
PROX_API prox_status prox_runtime_sparsity(int64_t sum_nx, int64_t sum_sel, int64_t tokens,
                                           int d_model, int d_ff, double alpha, double* s1_host,
                                           double* s2_host, double* e_host);

/* ------------------------------------------------------------------------
 * The decode step
 * ------------------------------------------------------------------------ */

/* Prox two-stage sparse FFN (Prox §4.1), B tokens each with its own masks;
 * act is the layer's gate activation (SiLU unless prox_layer_set_activation
 * chose GELU):
 *   Stage 1: m_x = 1[|x_i| >= tau_x]; g~ = Π_in(x, W~_gate, m_x),
 *            u~ = Π_in(x, W~_up, m_x); score_j = |act(g~_j) u~_j|;
 *            idx_s = the k channels of largest score, ties to the lower
 *            index (Prox App. A.6, per-token top-k), ascending; or, in
 *            threshold mode, every channel with score_j >= tau_s.
 *   Stage 2: for j in idx_s: s_j = act(x W_gate[:, j]) (x W_up[:, j]) with the
 *            full x (or s~_j in PROX_STAGE2_PROXY_VALUES mode);
 *            out = sum_j s_j W_down[j, :].
 * x, out: fp32 [B, d_model] (out may not alias x).  B <= max_batch.
 * One cooperative kernel per token on every SM (Stage 1, the cut, Stage 2 and
 * the output sum; the CTAs hand each other tagged words, no grid barrier),
 * each launch programmatically dependent on the previous one in the stream.
 * Token b's result does not depend on the other tokens of the call. */
PROX_API prox_status prox_ffn_forward(const prox_layer* layer, const float* x, float* out, int B,
                             void* stream);

/* Dense GLU baseline FFN(x) = (x W_up ⊙ act(x W_gate)) W_down (Prox §2.1),
 * on the same bf16 buffers (Stage 2 with every channel kept). */
PROX_API prox_status prox_dense_ffn(const prox_layer* layer, const float* x, float* out, int B,
                           void* stream);

/* The largest batch whose tokens take their Stage 1 from the batch-1 kernel
 * in prox_ffn_forward_batch (see there). */
#define PROX_BATCH_PER_TOKEN_STAGE1 4

/* The same step for B tokens at once, reading every weight byte the batch
 * needs once (the pages' kernels are batch 1 only, Prox §5.3 "Discussion";
 * the masks are still per token, Prox §4.1 and App. A.6):
 *   the union of the tokens' kept input rows is read once from the INT4
 *   proxies, each token contributing only its own kept rows; each token then
 *   takes its own top-k (or threshold) channel mask; the union of the
 *   selected channels' gate/up records and W_down rows is read once, each
 *   token contributing only through the channels it selected.
 * Batches of at most PROX_BATCH_PER_TOKEN_STAGE1 tokens take each token's
 * Stage 1 and mask from the batch-1 kernel instead (reading each token's own
 * kept rows: fewer bytes and less decoding than the union at small B; their
 * masks are then exactly the batch-1 masks).
 * The products run on the tensor cores (bf16 operands, fp32 accumulation,
 * x and the intermediate values split into two bf16 parts so that they carry
 * 16 significant bits); the sums are taken in another order than
 * prox_ffn_forward's, so scores and outputs agree with it to rounding and the
 * masks wherever no two scores are that close.  Exact Stage 2 only
 * (PROX_STAGE2_PROXY_VALUES gives PROX_EUNSUPPORTED).  x, out: fp32
 * [B, d_model], out not aliasing x; 1 <= B <= min(max_batch, 16); the layer
 * must have been created with max_batch > 1 (else PROX_EINVAL).  The scratch
 * is the layer's: calls on one layer must be stream-ordered.  No library
 * counterpart in the pages: this is the batched serving path they leave
 * open. */
PROX_API prox_status prox_ffn_forward_batch(const prox_layer* layer, const float* x, float* out, int B,
                                            void* stream);

/* Dense GLU baseline for B tokens reading every weight once: the batched
 * step's gate/up and down products over every channel with every token
 * keeping it (Prox §2.1).  Same arguments and limits as
 * prox_ffn_forward_batch. */
PROX_API prox_status prox_dense_ffn_batch(const prox_layer* layer, const float* x, float* out, int B,
                                          void* stream);

/* The union sizes of the layer's last prox_ffn_forward_batch: rows_host =
 * input rows some token kept, channels_host = channels some token selected
 * (the bytes that call streamed follow from them).  Synchronises `stream`;
 * PROX_EINVAL on a layer without the batched step or NULL outputs. */
PROX_API prox_status prox_batch_union_sizes(const prox_layer* layer, int32_t* rows_host,
                                            int32_t* channels_host, void* stream);

/* Same as prox_ffn_forward for n_tok tokens whose inputs and outputs live in
 * HOST memory (pinned memory makes the copies asynchronous): copies each
 * chunk of tokens to the device, runs the step and copies the results back.
 * Synchronises `stream` before returning. */
PROX_API prox_status prox_ffn_forward_host(prox_layer* layer, const float* x_host, float* out_host,
                                  int n_tok, void* stream);

/* prox_ffn_forward for one token with cudaEvent_t events_host[2] (passed as
 * void*) recorded right before and right after the token's kernel, which is
 * launched without programmatic overlap so the interval is its duration.
 * phase_ns (device, may be NULL): uint64 [stage1_ctas][24] receiving, per CTA,
 * the SM's cycle count (clock64) at: 0 kernel entry, 1 the previous kernel of
 * the stream complete, 8 kept rows compacted, 9 Stage-1 row loop done,
 * 2 Stage-1 partials written, 16 every CTA's partials written (phase 0),
 * 3 the partials of thread 0's channel received, 10 the CTA's channels scored
 * and counted, 17 every CTA's scores counted (phase 1), 14 the coarse
 * histogram complete, 15 the top-k cut found, 18 every CTA's count written
 * (phase 2), 4 the CTA's Stage-2 channels known, 11 Stage-2 ring set up,
 * 12 gate/up phase done, 5 partial output row written, 19 every partial row
 * written (phase 3), 6 the partial rows of the CTA's columns received,
 * 7 output written, 21 exit; slots 22 and 23 hold the GPU global timer (ns)
 * at entry and exit, which place the cycle counts on one time line; slot 13
 * holds the CTA's number of Stage-2 channels; slots not reached are 0. */
PROX_API prox_status prox_ffn_forward_profiled(const prox_layer* layer, const float* x, float* out,
                                               void* const* events_host, uint64_t* phase_ns,
                                               void* stream);

/* ------------------------------------------------------------------------
 * Test taps: the same kernels, exposing intermediate results
 * ------------------------------------------------------------------------ */

/* Stage 1 of one token.  idx_x: int32 [d_model] (first n_x entries valid,
 * ascending); n_x: one int32; g_tilde, u_tilde: fp32 [d_ff] proxy
 * pre-activations; idx_s: int32 [k], ascending.  Any output may be NULL. */
PROX_API prox_status prox_debug_stage1(prox_layer* layer, const float* x, int32_t* idx_x, int32_t* n_x,
                              float* g_tilde, float* u_tilde, int32_t* idx_s, void* stream);

/* Proxy scores |act(g~) u~| (Prox §4.1, Stage 1) of B tokens x [B, d_model]
 * into scores [B, d_ff] (fp32, device), with the layer's tau_x.  The input to
 * calibrating tau_s (Prox App. A.7, Algorithm 1: the s2-quantile of these
 * scores over the calibration tokens, e.g. with prox_calibrate_thresholds).
 * Stream-ordered; any B >= 1 (the tokens run one after another). */
PROX_API prox_status prox_layer_proxy_scores(const prox_layer* layer, const float* x, int B,
                                             float* scores, void* stream);

/* Test tap: the Stage-2 channels one token selects under the layer's current
 * rule, ascending, into idx_s [d_ff] (device) and their number into n_s (one
 * int32 on the device).  Same kernels as the forward step. */
PROX_API prox_status prox_debug_mask(const prox_layer* layer, const float* x, int32_t* idx_s,
                                     int32_t* n_s, void* stream);

/* Stage 2 of one token on a caller-given channel list idx_s (int32 [k], any
 * order, entries in [0, d_ff)); s_sp (fp32 [k], may be NULL) receives
 * act(g) u for each listed channel.  Always the exact Stage 2. */
PROX_API prox_status prox_forward_with_mask(prox_layer* layer, const float* x, const int32_t* idx_s,
                                   int k, float* out, float* s_sp, void* stream);

/* Test-only: the per-token channel masks of the layer's last
 * prox_ffn_forward_batch, int32 [B][d_ff] (1 = selected) into the device
 * buffer masks (caller-owned).  Stream-ordered; PROX_EINVAL on a layer
 * without the batched step, NULL masks or B outside [1, 16]. */
PROX_API prox_status prox_debug_batch_masks(const prox_layer* layer, int32_t* masks, int B, void* stream);

/* Test-only fault injection on the host: the nth device allocation that
 * prox_layer_create makes from now on (1 = the next one; a create makes nine:
 * four weight buffers, four packing temporaries, the workspace) fails as if
 * the device were out of memory, so the caller sees PROX_ENOMEM and the
 * library frees whatever it had allocated; 0 cancels a pending injection.
 * Process-wide; nothing fails on the device.  nth < 0 gives PROX_EINVAL. */
PROX_API prox_status prox_debug_fail_alloc(int nth);

/* Host-only plan of the per-token kernel for d_model x d_ff over num_sms
 * SMs, as prox_layer_create would make it on such a device (no GPU needed):
 * out_host (host, int32 [6]) receives the Stage-1 column slices, the kept-row
 * capacity per CTA, the Stage-1 copy depth (8-row tiles in flight per warp),
 * the Stage-2 ring slots, the Stage-2 consumer groups and the launch's
 * dynamic shared memory in bytes.  Errors as prox_layer_create:
 * PROX_EINVAL for a shape outside the rules, PROX_EUNSUPPORTED when the shape
 * needs more shared memory per CTA, or more channels per CTA, than
 * num_sms SMs give.  For tests of the shape rules. */
PROX_API prox_status prox_debug_token_geometry(int d_model, int d_ff, int num_sms, int32_t* out_host);

/* Test-only exercise of the bounded device waits, with no fault: launches one
 * CTA that adds one to the layer's launch counter and waits for a second
 * addition that never comes.  The wait runs out after its bound (2e8 SM
 * cycles, about 0.1 s), sets PROX_DEVERR_WAIT_TIMEOUT in the layer's error
 * word and the kernel returns.  prox_layer_error then reports the bit and, as
 * after any timeout, clears the launch counter, the histograms and the tagged
 * exchange words so that the next token runs clean.  Stream-ordered. */
PROX_API prox_status prox_debug_wait_timeout(prox_layer* layer, void* stream);

/* ------------------------------------------------------------------------
 * Harness kernels
 * ------------------------------------------------------------------------ */

/* Unit-gain RMSNorm y / sqrt(mean(y^2) + eps) of `rows` vectors of length d,
 * used to chain stacked layers (not part of the paper's FFN). */
PROX_API prox_status prox_rmsnorm(const float* y, float* x_out, int rows, int d, float eps,
                         void* stream);

/* Streaming device copy of `bytes` (multiple of 16, 16-byte aligned) used to
 * measure the HBM copy bandwidth that rooflines are quoted against. */
PROX_API prox_status prox_copy(const void* src, void* dst, size_t bytes, void* stream);

/* Copies the calling thread's last error message into msg_host (NUL-terminated,
 * at most n bytes); returns the full message length. */
PROX_API size_t prox_last_error(char* msg_host, size_t n);

/* Library version string (static storage). */
PROX_API const char* prox_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PROX_H_ */
