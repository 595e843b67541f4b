// Host-side internals of the Prox library: the layer handle, its buffers and
// the kernel launchers that the C ABI (prox_api.cu) strings together.
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "prox.h"

namespace prox {

constexpr int kGroup = 128;          // proxy quantisation group (input rows)
constexpr int kHistBins = 2048;      // calibration radix levels: 11 bits
constexpr int kScoreShift = 18;      // top-k select, first radix level: score bits [30:18]
constexpr int kScoreBins = 8192;
constexpr int kBucketCap = 128;      // (key, channel) entries kept per fine histogram bin
constexpr int kStage1Warps = 16;     // Stage-1 warps per CTA (one CTA per SM)
constexpr int kSelectSlice = 256;    // channels per select CTA (and per rank-offset entry)
constexpr int kMaxSlices = 160;      // >= d_ff / kSelectSlice + 1
constexpr int kStage2Consumers = 16;  // Stage-2 consumer warps (+1 producer warp)
constexpr int kTokenThreads = (kStage2Consumers + 1) * 32;  // threads of the per-token kernel
constexpr int kPhaseStamps = 24;     // phase stamp slots per CTA of the per-token kernel
constexpr int kMaxCtas = 256;        // per-token kernel grid (one CTA per SM) at most
constexpr size_t kStage2SmemBudget = 208 * 1024;  // Stage-2 ring and tables
constexpr int kMaxDModel = 16384;
constexpr int kMaxDff = 32768;       // bounds the select's slice table (kMaxSlices)
constexpr int kSmemPerSm = 233472;   // shared memory per SM on sm_100 (228 KB)
constexpr int kMaxSmemPerBlock = 232448;  // opt-in dynamic shared memory per CTA (227 KB)
constexpr int kHostChunkTokens = 64; // staging chunk of prox_ffn_forward_host
constexpr int kBatchMax = 16;        // tokens of one batched (union) step

// Per-token scratch of one layer (device memory owned by the handle).
struct Workspace {
  float* scores = nullptr;        // |act(g~) u~| [F]
  float* s_tilde = nullptr;       // act(g~) u~ [F], signed (proxy-values Stage 2 only)
  float* g_dbg = nullptr;         // debug g~ [F]
  float* u_dbg = nullptr;         // debug u~ [F]
  int32_t* sel_mask = nullptr;    // [F] debug: 1 where the channel is selected
  int32_t* idx_s = nullptr;       // [F] debug: selected channels (first k valid)
  unsigned long long* stats = nullptr;  // [3] sum n_x, tokens, sum of selected channels
  // What the CTAs of one per-token launch exchange (one contiguous range,
  // cleared after a wait ran out).  Tagged words: payload | launch tag << 32.
  uint32_t* hist = nullptr;       // [2][kScoreBins] scores' bits 30..18, by launch parity
  uint32_t* chist = nullptr;      // [2][kCoarseBins] scores' bits 30..24, by launch parity
  unsigned long long* bucket = nullptr;  // [kScoreBins][kBucketCap][2] tagged (key, channel)
  unsigned long long* st64 = nullptr;    // [F] tagged bits of act(g~) u~
  unsigned long long* sel_list = nullptr;  // [F] tagged selected channels, at each CTA's range start
  unsigned long long* sel_cnt = nullptr;   // [kMaxCtas] tagged selected count per CTA
  unsigned long long* s1_part = nullptr;   // [P][2][1024] tagged Stage-1 partial sums
  unsigned long long* ypart = nullptr;     // [P][d] tagged Stage-2 partial output rows
  unsigned long long* gbar = nullptr;  // launch counter: every CTA adds 1 when it ends
  void* xchg = nullptr;           // the exchange range, for clearing
  size_t xchg_bytes = 0;
  int* err = nullptr;             // device error word
  float* stage_in = nullptr;      // host-path staging [kHostChunkTokens][d]
  float* stage_out = nullptr;
  void* base = nullptr;           // single allocation holding all of the above
  size_t bytes = 0;
};

// Scratch of the batched step (batch.cu), allocated when max_batch > 1.
// Token-major arrays have kBatchMax rows; Fp = d_ff rounded up to 64.
struct BatchWs {
  __nv_bfloat16* xu_hi = nullptr;  // [16][d] x^ of the union rows (kept or 0), bf16 hi part
  __nv_bfloat16* xu_lo = nullptr;  //          ... and the rest
  __nv_bfloat16* xf_hi = nullptr;  // [16][d] x split the same way
  __nv_bfloat16* xf_lo = nullptr;
  int* urow = nullptr;             // [d] the union rows, ascending
  int* gstart = nullptr;           // [G] first union entry of each quantisation group
  int* gcount = nullptr;           // [G] union rows in each group
  int* cnt = nullptr;              // [4] union rows, union channels
  int* rcount = nullptr;           // [d / 256] union rows per block of 256 rows
  int* ccount = nullptr;           // [d_ff / 256] union channels per block of 256
  float* part1 = nullptr;          // [S1][16][2][F] Stage-1 sums per row split
  float* scores = nullptr;         // [16][F]
  int32_t* smask = nullptr;        // [16][F] per-token channel masks (1 = selected)
  int* ulist = nullptr;            // [F] the union channels, ascending
  uint32_t* utok = nullptr;        // [F] the tokens that selected each
  float* gup = nullptr;            // [Fp / 64 * KS][64][16][2] gate / up sums per work item
  __nv_bfloat16* hh = nullptr;     // [16][Fp] h per token and union entry, hi part
  __nv_bfloat16* hl = nullptr;     //                                      ... lo part
  float* yp = nullptr;             // [S5][16][d] down partials per entry split
};

}  // namespace prox

struct prox_layer {
  int d = 0, F = 0, G = 0, k = 0, max_batch = 0;
  float tau = 0.f;
  int mask_mode = 0;     // PROX_MASK_TOPK or PROX_MASK_THRESHOLD
  float tau_s = 0.f;     // Stage-2 score threshold (threshold mode)
  int act = 0;           // PROX_ACT_*: gate activation of the GLU
  int stage2_source = 0; // PROX_STAGE2_EXACT or PROX_STAGE2_PROXY_VALUES
  int device = 0, num_sms = 0;
  // Per-token kernel: P CTAs (one per SM), token_smem bytes of shared memory.
  int P = 0;
  size_t token_smem = 0;
  // Stage-1 geometry: C column slices, at most s1_lmax rows per CTA, s1_depth
  // k-tiles in flight per Stage-1 warp
  int C = 0, s1_lmax = 0, s1_depth = 0;
  // Stage-2 geometry
  int ring_slots = 0, stage2_groups = 1;
  // library-owned weights
  uint16_t* wgu = nullptr;   // bf16 [F][2d]: gate column j | up column j
  uint16_t* wd = nullptr;    // bf16 [F][d]
  uint8_t* pq = nullptr;     // INT4 codes [C][d][512 B], gate/up interleaved per 16 B
  uint16_t* ps = nullptr;    // fp16 scales [G][F/32][2][32]
  prox::Workspace ws;
  // batched step: row splits of its Stage 1, entry splits of its down product
  int b_s1 = 0, b_s5 = 0, b_ks = 1;
  void* bws_base = nullptr;
  prox::BatchWs bws;
};

namespace prox {

// ---- launchers (each returns the CUDA error of its launch) ----------------
struct Stage1Taps {
  float* g = nullptr;       // g~ [F]
  float* u = nullptr;       // u~ [F]
  int32_t* idx_x = nullptr; // kept input rows, ascending [d]
  int32_t* n_x = nullptr;   // their number
  float* s_tilde = nullptr; // signed proxy values act(g~) u~ [F]
};
// One launch of the per-token kernel: which phases run and on what.
struct TokenLaunch {
  const float* x = nullptr;
  float* out = nullptr;         // output row (Stage-2 modes, not select_only)
  bool stage1 = true;           // Stage 1 runs (threshold, proxies, scores)
  int mode = 1;                 // -1 Stage 1 only, 0 given list `idx`, 1 top-k, 2 dense, 3 threshold
  float tau_s = 0.f;            // mode 3: channels with score >= tau_s
  const int32_t* idx = nullptr;
  int k = 0;
  int32_t* sel_mask = nullptr;  // top-k / threshold: 1/0 per channel written here (debug)
  float* s_sp = nullptr;        // optional act(g) u per listed channel
  bool proxy_values = false;    // ablation: s~ of Stage 1 instead of the exact s
  bool select_only = false;     // stop after selecting
  Stage1Taps taps;
  unsigned long long* phase_ns = nullptr;  // optional phase stamps [P][kPhaseStamps]
};

cudaError_t setup_token_kernels();
// The batched step (batch.cu): B <= kBatchMax tokens, union loads; dense =
// every channel for every token (the batched dense baseline).
cudaError_t setup_batch_kernels();
void choose_batch_splits(int d, int F, int num_sms, int* s1, int* s5, int* ks);
bool batch_fits(int F, int num_sms, int ks);
size_t batch_ws_bytes(int d, int F, int s1, int s5, int ks);
void carve_batch_ws(void* base, int d, int F, int s1, int s5, int ks, BatchWs* w);
cudaError_t launch_batch(const prox_layer* L, const float* X, float* Y, int B, bool dense,
                         cudaStream_t s);
// Batches up to this size take each token's Stage 1 and mask from the
// per-token kernel (select only) instead of the union Stage 1.
constexpr int kBatchPerTokenStage1 = PROX_BATCH_PER_TOKEN_STAGE1;
cudaError_t launch_barrier_probe(const prox_layer* L, cudaStream_t s);
cudaError_t launch_token(const prox_layer* L, const TokenLaunch& m, cudaStream_t s, bool pdl);

cudaError_t launch_pack_proxy(const uint16_t* W, int d, int F, uint8_t* codes,
                              uint16_t* scales, cudaStream_t s);
cudaError_t launch_interleave_proxy(const uint8_t* cg, const uint8_t* cu, const uint16_t* sg,
                                    const uint16_t* su, int d, int F, uint8_t* pq,
                                    uint16_t* ps, cudaStream_t s);
cudaError_t launch_gateup_records(const uint16_t* Wg, const uint16_t* Wu, int d, int F,
                                  uint16_t* wgu, cudaStream_t s);

// Calibration: exact order statistic of |X| at 0-based ascending rank `rank`.
// `scratch` holds kHistBins + 4 uint32 (zeroed by the caller).
// Device address of the calibration scratch kept in a static __device__
// array (kHistBins + 8 words) of the current device.
cudaError_t calibrate_static_scratch(uint32_t** ptr);
cudaError_t launch_calibrate(const float* X, size_t n, unsigned long long rank,
                             uint32_t* scratch, float* tau_dev, cudaStream_t s);

cudaError_t launch_rmsnorm(const float* y, float* x, int rows, int d, float eps,
                           cudaStream_t s);
cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t s);
cudaError_t launch_mask_to_list(const int32_t* mask, int n, int32_t* list, int32_t* count,
                                cudaStream_t s);

// Stage-1 column slices, per-CTA row capacity and ring depth for a shape on
// `num_sms` SMs (one CTA each).
void choose_stage1_grid(int d, int F, int num_sms, int* C, int* lmax, int* depth);
size_t stage1_smem_bytes(int lmax, int depth, int d);
size_t stage1_part_floats(int P);
// Stage-2 ring depth, consumer groups and shared memory for d_model = d.
void choose_stage2(int d, int F, int num_sms, int* slots, int* groups, size_t* smem);

}  // namespace prox
