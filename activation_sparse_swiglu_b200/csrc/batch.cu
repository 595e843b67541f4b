// The batched Prox FFN step: B <= 16 decode tokens, each with its own input
// mask and its own Stage-2 channel mask (Prox §4.1 applied per token; the
// pages' kernels are batch-1 only, Prox §5.3 "Discussion"), reading every
// weight byte the batch needs once:
//
//   prepare:  per token the kept rows |x_b,i| >= tau_x; their union U (rows
//             any token keeps), with x^_b,i = x_b,i where token b keeps row i
//             and 0 elsewhere, and the full x, both split into bf16 hi + lo
//             (x = hi + lo to 2^-16 relative: the products below are exact);
//   stage 1:  the INT4 proxies over the union rows, once, for all tokens:
//             D[output][token] = sum over the rows of a quantisation group of
//             code x x^, scaled per (group, channel) by the fp16 scale;
//   scores:   per token and channel |act(g~) u~|; the exact per-token top-k
//             (or the score threshold) gives each token its channel mask;
//   union:    the channels any token selected, with the tokens that did;
//   gate/up:  the union channels' bf16 records, once, for all tokens, with
//             h_b,j = act(g) u for the tokens that selected j and 0 elsewhere;
//   down:     the union channels' W_down rows, once: y_b = sum_j h_b,j W_down[j].
//
// The contractions are small matrix products (16 tokens wide); they run on
// the tensor cores with mma.sync (m16n8k16, bf16 in, fp32 accumulate), the
// skinny shape needing no more: every operand tile is staged in shared memory
// by cp.async and the matrix side read by ldmatrix.  The dense batched
// baseline is the gate/up and down kernels over every channel with every
// token selecting it.
#include "prox_device.cuh"
#include "prox_internal.h"
#include "select.cuh"

namespace prox {
namespace {

constexpr int NB = kBatchMax;  // the token (n) width of every product: 16

// ---------------------------------------------------------------------------
// small primitives
// ---------------------------------------------------------------------------

__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// A fragment (16 x 16, row-major) of a tile stored [m][k] (k contiguous).
__device__ __forceinline__ void ldsm_a(uint32_t (&a)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(smem_u32(row_addr)));
}
// A fragment of a tile stored [k][m] (m contiguous): the transposing load.
__device__ __forceinline__ void ldsm_a_trans(uint32_t (&a)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(smem_u32(row_addr)));
}
// D (16 x 8 fp32) += A (16 x 16 bf16) B (16 x 8 bf16).
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Lane l's row address for an x4 ldmatrix of the 16 x 16 A block at (m0, k0):
// matrix q = l / 8 covers m0 + 8 (q & 1), k0 + 8 (q >> 1); its row l % 8.
// [m][k] storage (ld = row stride in elements):
__device__ __forceinline__ const __nv_bfloat16* a_row_mk(const __nv_bfloat16* t, int ld, int m0, int k0) {
  const int l = threadIdx.x & 31, q = l >> 3, r = l & 7;
  return t + (size_t)(m0 + r + 8 * (q & 1)) * ld + k0 + 8 * (q >> 1);
}
// [k][m] storage:
__device__ __forceinline__ const __nv_bfloat16* a_row_km(const __nv_bfloat16* t, int ld, int m0, int k0) {
  const int l = threadIdx.x & 31, q = l >> 3, r = l & 7;
  return t + (size_t)(k0 + r + 8 * (q >> 1)) * ld + m0 + 8 * (q & 1);
}

// The 16 x 16 tile's product with the token block: B operand from a [n][k]
// tile (k contiguous, hi and lo parts), both n8 halves.  acc[h] is the
// D fragment of tokens 8h .. 8h+7.
__device__ __forceinline__ void mma_tokens(float (&acc)[2][4], const uint32_t (&a)[4],
                                           const __nv_bfloat16* bhi, const __nv_bfloat16* blo, int ldb,
                                           int k0) {
  const int l = threadIdx.x & 31, g = l >> 2, t = l & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const __nv_bfloat16* rh = bhi + (size_t)(8 * h + g) * ldb + k0 + 2 * t;
    const __nv_bfloat16* rl = blo + (size_t)(8 * h + g) * ldb + k0 + 2 * t;
    mma_bf16(acc[h], a, *reinterpret_cast<const uint32_t*>(rh), *reinterpret_cast<const uint32_t*>(rh + 8));
    mma_bf16(acc[h], a, *reinterpret_cast<const uint32_t*>(rl), *reinterpret_cast<const uint32_t*>(rl + 8));
  }
}

// fp32 -> bf16 hi + bf16 lo, hi + lo = v to 2^-16 relative.
__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16* hi, __nv_bfloat16* lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  *hi = h;
  *lo = __float2bfloat16_rn(v - __bfloat162float(h));
}

// ---------------------------------------------------------------------------
// prepare: the union of kept rows, x^ (union-compacted) and x, split hi / lo
// ---------------------------------------------------------------------------

// One CTA of 1024 threads.  Rows in rounds of 1024 (one per thread, coalesced);
// the union rows are compacted in ascending order with a running offset.
// Writes urow[n_u], xu_hi/lo[16][d] (columns < n_u), xf_hi/lo[16][d],
// gstart/gcount per quantisation group and cnt[0] = n_u; adds the kept rows
// and the tokens to the layer's statistics.
__global__ void __launch_bounds__(1024) batch_prepare_kernel(const float* __restrict__ X, int B, int d,
                                                             float tau, BatchWs w,
                                                             unsigned long long* stats) {
  __shared__ int s_scan[40];
  const int tid = threadIdx.x;
  const int G = d / kGroup;
  for (int g = tid; g < G; g += blockDim.x) w.gcount[g] = 0;
  __syncthreads();
  int base = 0;
  unsigned kept_total = 0;
  for (int r0 = 0; r0 < d; r0 += blockDim.x) {
    const int r = r0 + tid;
    float xv[NB];
    bool any = false;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      xv[b] = (r < d && b < B) ? __ldg(X + (size_t)b * d + r) : 0.f;
      const bool keep = fabsf(xv[b]) >= tau && r < d && b < B;
      kept_total += keep ? 1u : 0u;
      any = any || keep;
    }
    if (r < d)
#pragma unroll
      for (int b = 0; b < NB; ++b) split_bf16(xv[b], w.xf_hi + (size_t)b * d + r, w.xf_lo + (size_t)b * d + r);
    int total;
    const int pos = base + block_exclusive_scan(any ? 1 : 0, s_scan, &total);
    if (any) {
      w.urow[pos] = r;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float v = fabsf(xv[b]) >= tau ? xv[b] : 0.f;
        split_bf16(v, w.xu_hi + (size_t)b * d + pos, w.xu_lo + (size_t)b * d + pos);
      }
      atomicAdd(w.gcount + r / kGroup, 1);
    }
    base += total;
  }
  __syncthreads();
  // group starts: the union rows are ascending, so group g's rows are
  // [gstart[g], gstart[g] + gcount[g]) with gstart the prefix of the counts
  if (tid == 0) {
    int acc = 0;
    for (int g = 0; g < G; ++g) {
      w.gstart[g] = acc;
      acc += w.gcount[g];
    }
    w.cnt[0] = base;
  }
  // block total of the kept rows
  unsigned tk;
  block_exclusive_scan(kept_total, reinterpret_cast<unsigned*>(s_scan), &tk);
  if (tid == 0 && stats) {
    atomicAdd(stats, (unsigned long long)tk);
    atomicAdd(stats + 1, (unsigned long long)B);
  }
}

// ---------------------------------------------------------------------------
// stage 1 over the union rows
// ---------------------------------------------------------------------------

constexpr int S1_THREADS = 512;   // 16 warps, two 16-output tiles each
constexpr int S1_OUT = 512;       // outputs per CTA: half a slice (256 channels of each proxy)
constexpr int S1_KT = 32;         // union rows per tile (never across a group)
constexpr int S1_STAGES = 4;      // raw code tiles in flight
constexpr int S1_LDS = S1_OUT + 8;
constexpr int S1_LDB = S1_KT + 8;
constexpr int S1_MAX_TILES = 4 * (kMaxDModel / kGroup);

struct S1Smem {
  uint8_t raw[S1_STAGES][S1_KT][256];            // codes of the half slice, per union row
  __nv_bfloat16 S[S1_KT][S1_LDS];                // decoded codes, [row][output]
  __nv_bfloat16 bhi[NB][S1_LDB], blo[NB][S1_LDB];  // x^ of the tile's rows, [token][row]
  int t_i0[S1_MAX_TILES];
  short t_len[S1_MAX_TILES];
  short t_grp[S1_MAX_TILES];
  int ntiles;
};

// Grid (2 C, S1 splits): CTA (hs, s) takes the outputs of half slice hs and
// the quantisation groups [G s / S1, G (s + 1) / S1); writes
// part1[s][token][gate|up][channel] (the group-scaled sums of its groups).
__global__ void __launch_bounds__(S1_THREADS) batch_stage1_kernel(const uint8_t* __restrict__ pq,
                                                                  const __half* __restrict__ ps, int d,
                                                                  int F, BatchWs w) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  S1Smem& sm = *reinterpret_cast<S1Smem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hs = blockIdx.x, slice = hs >> 1, half = hs & 1;
  const int S1 = gridDim.y, s = blockIdx.y;
  const int G = d / kGroup;
  const int g0 = (int)((long long)G * s / S1), g1 = (int)((long long)G * (s + 1) / S1);
  // the CTA's tiles: each group's union rows in runs of at most S1_KT
  if (tid == 0) {
    int n = 0;
    for (int g = g0; g < g1; ++g) {
      const int c = w.gcount[g], st = w.gstart[g];
      for (int j = 0; j < c; j += S1_KT) {
        sm.t_i0[n] = st + j;
        sm.t_len[n] = (short)min(S1_KT, c - j);
        sm.t_grp[n] = (short)g;
        ++n;
      }
    }
    sm.ntiles = n;
  }
  for (int i = tid; i < S1_KT * S1_LDS; i += S1_THREADS) (&sm.S[0][0])[i] = __float2bfloat16_rn(0.f);
  __syncthreads();
  const int nt = sm.ntiles;
  const uint8_t* slice_base = pq + (size_t)slice * d * 512 + half * 256;

  // tile t's codes: row k of the tile (k < len) into raw[t % STAGES][k]
  auto issue = [&](int t) {
    if (t < nt) {
      const int k = tid >> 4, c16 = tid & 15;  // 32 rows x 16 chunks of 16 B
      if (k < sm.t_len[t]) {
        const int row = __ldg(w.urow + sm.t_i0[t] + k);
        cp16(&sm.raw[t % S1_STAGES][k][c16 * 16], slice_base + (size_t)row * 512 + c16 * 16);
      }
    }
    cp_commit();
  };
#pragma unroll
  for (int t = 0; t < S1_STAGES - 1; ++t) issue(t);

  float acc[2][2][4], tot[2][2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][h][e] = tot[i][h][e] = 0.f;

  const int g = lane >> 2;
  for (int t = 0; t < nt; ++t) {
    issue(t + S1_STAGES - 1);
    cp_wait<S1_STAGES - 1>();
    __syncthreads();  // tile t's codes are in; the previous tile's products are done
    const int len = sm.t_len[t], i0 = sm.t_i0[t];
    // decode: 32 rows x 64 words, 4 words per thread; word wd of row k holds
    // outputs 8 wd .. 8 wd + 7 (nibble p is output 8 wd + p); the code is q + 8
    for (int j = tid; j < S1_KT * 64; j += S1_THREADS) {
      const int k = j >> 6, wd = j & 63;
      if (k < len) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(&sm.raw[t % S1_STAGES][k][wd * 4]);
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const uint32_t b = v >> (8 * p);  // nibbles 2p (low) and 2p + 1
          const uint32_t pair = (b & 0xFu) | ((b & 0xF0u) << 12) | 0x43004300u;  // bf16 128 + code
          __nv_bfloat162 q = *reinterpret_cast<const __nv_bfloat162*>(&pair);
          q = __hsub2(q, __floats2bfloat162_rn(136.f, 136.f));  // exact: q in [-8, 7]
          o[p] = *reinterpret_cast<const uint32_t*>(&q);
        }
        *reinterpret_cast<uint4*>(&sm.S[k][wd * 8]) = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
        *reinterpret_cast<uint4*>(&sm.S[k][wd * 8]) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    {
      const int n = tid >> 5, k = tid & 31;  // 16 tokens x 32 rows
      const bool ok = k < len;
      sm.bhi[n][k] = ok ? w.xu_hi[(size_t)n * d + i0 + k] : __float2bfloat16_rn(0.f);
      sm.blo[n][k] = ok ? w.xu_lo[(size_t)n * d + i0 + k] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m0 = warp * 32 + i * 16;
#pragma unroll
      for (int k0 = 0; k0 < S1_KT; k0 += 16) {
        if (k0 < len) {
          uint32_t a[4];
          ldsm_a_trans(a, a_row_km(&sm.S[0][0], S1_LDS, m0, k0));
          mma_tokens(acc[i], a, &sm.bhi[0][0], &sm.blo[0][0], S1_LDB, k0);
        }
      }
    }
    // the group's last tile: scale its sums per (group, output) and add them
    if (t + 1 == nt || sm.t_grp[t + 1] != sm.t_grp[t]) {
      const int grp = sm.t_grp[t];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int m = warp * 32 + i * 16 + g + 8 * r;  // output of the half slice
          const int blk = (slice * 512 + half * 256) / 32 + (m >> 6);  // < F / 32 for real channels
          const float sc = blk < F / 32 ? __half2float(__ldg(ps + ((size_t)grp * (F / 32) + blk) * 64 + (m & 63)))
                                        : 0.f;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tot[i][h][2 * r] = fmaf(sc, acc[i][h][2 * r], tot[i][h][2 * r]);
            tot[i][h][2 * r + 1] = fmaf(sc, acc[i][h][2 * r + 1], tot[i][h][2 * r + 1]);
            acc[i][h][2 * r] = acc[i][h][2 * r + 1] = 0.f;
          }
        }
      }
    }
  }
  cp_wait<0>();
  // part1[s][token][kind][channel]: output m is kind (m & 63) >> 5 of channel
  // slice * 512 + half * 256 + (m >> 6) * 32 + (m & 31)
  const int t4 = lane & 3;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int m = warp * 32 + i * 16 + g + 8 * r;
      const int kind = (m & 63) >> 5;
      const int ch = slice * 512 + half * 256 + (m >> 6) * 32 + (m & 31);
      if (ch < F)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int n = 8 * h + 2 * t4 + c;
            w.part1[(((size_t)s * NB + n) * 2 + kind) * F + ch] = tot[i][h][2 * r + c];
          }
    }
}

// ---------------------------------------------------------------------------
// scores, per-token masks, union of the selected channels
// ---------------------------------------------------------------------------

// One thread per (channel, token < B): g~, u~ summed over the Stage-1 splits
// in split order, score |act(g~) u~|; under the threshold rule the mask too.
__global__ void batch_score_kernel(BatchWs w, int F, int S1, int act, int threshold, float tau_s) {
  const int ch = blockIdx.x * blockDim.x + threadIdx.x, b = blockIdx.y;
  if (ch >= F) return;
  float g = 0.f, u = 0.f;
  for (int s = 0; s < S1; ++s) {
    g += w.part1[(((size_t)s * NB + b) * 2 + 0) * F + ch];
    u += w.part1[(((size_t)s * NB + b) * 2 + 1) * F + ch];
  }
  const float sc = fabsf(act_f32(g, act) * u);
  w.scores[(size_t)b * F + ch] = sc;
  if (threshold) w.smask[(size_t)b * F + ch] = sc >= tau_s ? 1 : 0;
}

// One CTA per token: the exact top-k of its F scores (ties to the lower
// channel), by the radix select of select.cuh over keys held in shared memory.
__global__ void __launch_bounds__(1024) batch_topk_kernel(BatchWs w, int F, int k) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SelectScratch& sc = *reinterpret_cast<SelectScratch*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + ((sizeof(SelectScratch) + 15) & ~(size_t)15));
  const int b = blockIdx.x, tid = threadIdx.x;
  const float* src = w.scores + (size_t)b * F;
  for (int j = tid; j < F; j += blockDim.x) keys[j] = __float_as_uint(src[j]);
  __syncthreads();
  const int per = (F + (int)blockDim.x - 1) / (int)blockDim.x;
  const int j0 = min(tid * per, F), j1 = min(j0 + per, F);
  auto all = [&](auto fn) {
    for (int j = j0; j < j1; ++j) fn(keys[j], j);
  };
  TopkCut cut;
  int n_eq, k_eq;
  radix_kth(all, k, sc, &cut.T, &n_eq, &k_eq);
  cut.tie_cut = k_eq < n_eq ? radix_tie(all, cut.T, k_eq, sc) : F;
  for (int j = tid; j < F; j += blockDim.x) w.smask[(size_t)b * F + j] = selected(keys[j], j, cut) ? 1 : 0;
}

// One CTA of 1024 threads: the channels some token selected, ascending, with
// the bit set of the tokens that did; cnt[1] = their number.  Adds the
// selected (token, channel) pairs to the layer's statistics.
__global__ void __launch_bounds__(1024) batch_union_kernel(BatchWs w, int F, int B,
                                                           unsigned long long* stats) {
  __shared__ int s_scan[40];
  const int tid = threadIdx.x;
  int base = 0;
  unsigned nsel = 0;
  for (int c0 = 0; c0 < F; c0 += blockDim.x) {
    const int ch = c0 + tid;
    uint32_t bits = 0u;
    if (ch < F)
      for (int b = 0; b < B; ++b) bits |= w.smask[(size_t)b * F + ch] ? (1u << b) : 0u;
    nsel += __popc(bits);
    int total;
    const int pos = base + block_exclusive_scan(bits ? 1 : 0, s_scan, &total);
    if (bits) {
      w.ulist[pos] = ch;
      w.utok[pos] = bits;
    }
    base += total;
  }
  if (tid == 0) w.cnt[1] = base;
  unsigned ts;
  block_exclusive_scan(nsel, reinterpret_cast<unsigned*>(s_scan), &ts);
  if (tid == 0 && stats) atomicAdd(stats + 2, (unsigned long long)ts);
}

// ---------------------------------------------------------------------------
// gate/up over the union channels (or every channel: dense)
// ---------------------------------------------------------------------------

constexpr int GU_THREADS = 256;  // 8 warps: gate / up x four 16-channel tiles
constexpr int GU_M = 64;         // channels per CTA
constexpr int GU_KT = 64;        // d_model elements per stage
constexpr int GU_STAGES = 3;
constexpr int GU_LDA = GU_KT + 8;

struct GuSmem {
  __nv_bfloat16 a[GU_STAGES][2][GU_M][GU_LDA];     // gate, up column slices [channel][k]
  __nv_bfloat16 bhi[GU_STAGES][NB][GU_LDA], blo[GU_STAGES][NB][GU_LDA];  // x [token][k]
};

// CTA c: union entries [64 c, 64 c + 64) (dense: channels).  Writes
// hh / hl[token][entry] = h split hi / lo, h = act(g) u for the tokens that
// selected the channel and 0 for the others (and for entries past the union).
__global__ void __launch_bounds__(GU_THREADS) batch_gateup_kernel(const __nv_bfloat16* __restrict__ wgu, int d,
                                                                  int F, int B, int act, int dense,
                                                                  BatchWs w) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  GuSmem& sm = *reinterpret_cast<GuSmem*>(smem_raw);
  const int n_s = dense ? F : w.cnt[1];
  const int e0 = blockIdx.x * GU_M, Fp = (F + 63) & ~63;
  if (e0 >= n_s) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kind = warp >> 2, m0 = (warp & 3) * 16;
  const int nkt = d / GU_KT;

  auto channel = [&](int e) { return dense ? min(e, F - 1) : __ldg(w.ulist + min(e, n_s - 1)); };
  auto issue = [&](int kt) {
    if (kt < nkt) {
      const int st = kt % GU_STAGES, k0 = kt * GU_KT;
      // 2 x 64 channels x 8 chunks, then 2 x 16 tokens x 8 chunks: 1280 copies
      for (int j = tid; j < 1280; j += GU_THREADS) {
        if (j < 1024) {
          const int kd = j >> 9, m = (j >> 3) & 63, c = j & 7;
          const size_t col = (size_t)channel(e0 + m) * 2 * d + (size_t)kd * d + k0 + c * 8;
          cp16(&sm.a[st][kd][m][c * 8], wgu + col);
        } else {
          const int jj = j - 1024, lo = jj >> 7, n = (jj >> 3) & 15, c = jj & 7;
          const __nv_bfloat16* src = (lo ? w.xf_lo : w.xf_hi) + (size_t)n * d + k0 + c * 8;
          cp16(lo ? &sm.blo[st][n][c * 8] : &sm.bhi[st][n][c * 8], src);
        }
      }
    }
    cp_commit();
  };
#pragma unroll
  for (int kt = 0; kt < GU_STAGES - 1; ++kt) issue(kt);
  float acc[2][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
  for (int kt = 0; kt < nkt; ++kt) {
    issue(kt + GU_STAGES - 1);
    cp_wait<GU_STAGES - 1>();
    __syncthreads();
    const int st = kt % GU_STAGES;
#pragma unroll
    for (int k0 = 0; k0 < GU_KT; k0 += 16) {
      uint32_t a[4];
      ldsm_a(a, a_row_mk(&sm.a[st][kind][0][0], GU_LDA, m0, k0));
      mma_tokens(acc, a, &sm.bhi[st][0][0], &sm.blo[st][0][0], GU_LDA, k0);
    }
    __syncthreads();
  }
  cp_wait<0>();
  __syncthreads();
  // g and u through shared memory: gu[kind][channel][token]
  float* gu = reinterpret_cast<float*>(smem_raw);
  {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          gu[(kind * GU_M + m0 + g + 8 * r) * NB + 8 * h + 2 * t + c] = acc[h][2 * r + c];
  }
  __syncthreads();
  for (int j = tid; j < GU_M * NB; j += GU_THREADS) {
    const int m = j / NB, n = j % NB, e = e0 + m;
    float h = 0.f;
    if (e < n_s && n < B) {
      const bool sel = dense || ((__ldg(w.utok + e) >> n) & 1u);
      if (sel) h = act_f32(gu[m * NB + n], act) * gu[(GU_M + m) * NB + n];
    }
    if (e < ((n_s + GU_M - 1) / GU_M) * GU_M)
      split_bf16(h, w.hh + (size_t)n * Fp + e, w.hl + (size_t)n * Fp + e);
  }
}

// ---------------------------------------------------------------------------
// down over the union channels, then the split sum
// ---------------------------------------------------------------------------

constexpr int DN_THREADS = 256;  // 8 warps, one 16-column tile each
constexpr int DN_M = 128;        // output columns per CTA
constexpr int DN_KT = 64;        // union entries per stage
constexpr int DN_STAGES = 3;
constexpr int DN_LDA = DN_M + 8;
constexpr int DN_LDB = DN_KT + 8;

struct DnSmem {
  __nv_bfloat16 a[DN_STAGES][DN_KT][DN_LDA];        // W_down rows' column slices [entry][column]
  __nv_bfloat16 bhi[DN_STAGES][NB][DN_LDB], blo[DN_STAGES][NB][DN_LDB];  // h [token][entry]
};

// Grid (d / 128, S5): CTA (cb, s) takes columns [128 cb, 128 cb + 128) and the
// entry tiles [T s / S5, T (s + 1) / S5) of the T = ceil(n / 64) tiles;
// writes yp[s][token][column].
__global__ void __launch_bounds__(DN_THREADS) batch_down_kernel(const __nv_bfloat16* __restrict__ wd, int d,
                                                                int F, int dense, BatchWs w) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DnSmem& sm = *reinterpret_cast<DnSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_s = dense ? F : w.cnt[1];
  const int S5 = gridDim.y, s = blockIdx.y, col0 = blockIdx.x * DN_M, Fp = (F + 63) & ~63;
  const int T = (n_s + DN_KT - 1) / DN_KT;
  const int t0 = (int)((long long)T * s / S5), t1 = (int)((long long)T * (s + 1) / S5);
  const int nt = t1 - t0;
  auto channel = [&](int e) { return dense ? min(e, F - 1) : __ldg(w.ulist + min(e, n_s - 1)); };
  auto issue = [&](int it) {
    if (it < nt) {
      const int st = it % DN_STAGES, e0 = (t0 + it) * DN_KT;
      // 64 entries x 16 chunks, then 2 x 16 tokens x 8 chunks: 1280 copies
      for (int j = tid; j < 1280; j += DN_THREADS) {
        if (j < 1024) {
          const int k = j >> 4, c = j & 15;
          cp16(&sm.a[st][k][c * 8], wd + (size_t)channel(e0 + k) * d + col0 + c * 8);
        } else {
          const int jj = j - 1024, lo = jj >> 7, n = (jj >> 3) & 15, c = jj & 7;
          const __nv_bfloat16* src = (lo ? w.hl : w.hh) + (size_t)n * Fp + e0 + c * 8;
          cp16(lo ? &sm.blo[st][n][c * 8] : &sm.bhi[st][n][c * 8], src);
        }
      }
    }
    cp_commit();
  };
#pragma unroll
  for (int it = 0; it < DN_STAGES - 1; ++it) issue(it);
  float acc[2][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
  const int m0 = warp * 16;
  for (int it = 0; it < nt; ++it) {
    issue(it + DN_STAGES - 1);
    cp_wait<DN_STAGES - 1>();
    __syncthreads();
    const int st = it % DN_STAGES;
#pragma unroll
    for (int k0 = 0; k0 < DN_KT; k0 += 16) {
      uint32_t a[4];
      ldsm_a_trans(a, a_row_km(&sm.a[st][0][0], DN_LDA, m0, k0));
      mma_tokens(acc, a, &sm.bhi[st][0][0], &sm.blo[st][0][0], DN_LDB, k0);
    }
    __syncthreads();
  }
  cp_wait<0>();
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < 2; ++c)
        w.yp[((size_t)s * NB + 8 * h + 2 * t + c) * d + col0 + m0 + g + 8 * r] = acc[h][2 * r + c];
}

// y[b][col] = the split partials added in split order.
__global__ void batch_reduce_kernel(BatchWs w, int d, int B, int S5, float* __restrict__ Y) {
  const int col = blockIdx.x * blockDim.x + threadIdx.x, b = blockIdx.y;
  if (col >= d || b >= B) return;
  float v = 0.f;
  for (int s = 0; s < S5; ++s) v += w.yp[((size_t)s * NB + b) * d + col];
  Y[(size_t)b * d + col] = v;
}

}  // namespace
}  // namespace prox

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

namespace prox {

namespace {
size_t topk_smem(int F) { return ((sizeof(SelectScratch) + 15) & ~(size_t)15) + (size_t)F * 4; }
size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }
}  // namespace

void choose_batch_splits(int d, int F, int num_sms, int* s1, int* s5) {
  const int hs = 2 * ((F + 511) / 512);  // half slices
  const int G = d / kGroup;
  *s1 = std::max(1, std::min(G, (2 * num_sms + hs - 1) / hs));
  const int cb = d / DN_M;
  *s5 = std::max(1, (2 * num_sms + cb - 1) / cb);
}

size_t batch_ws_bytes(int d, int F, int s1, int s5) {
  const size_t Fp = (size_t)((F + 63) & ~63), G = (size_t)d / kGroup;
  return 4 * al256((size_t)NB * d * 2) + al256((size_t)d * 4) + 2 * al256(G * 4) + al256(16) +
         al256((size_t)s1 * NB * 2 * F * 4) + al256((size_t)NB * F * 4) + al256((size_t)NB * F) +
         2 * al256((size_t)F * 4) + 2 * al256((size_t)NB * Fp * 2) + al256((size_t)s5 * NB * d * 4);
}

void carve_batch_ws(void* base, int d, int F, int s1, int s5, BatchWs* w) {
  const size_t Fp = (size_t)((F + 63) & ~63), G = (size_t)d / kGroup;
  char* p = static_cast<char*>(base);
  auto take = [&](size_t bytes) {
    char* q = p;
    p += al256(bytes);
    return q;
  };
  w->xu_hi = reinterpret_cast<__nv_bfloat16*>(take((size_t)NB * d * 2));
  w->xu_lo = reinterpret_cast<__nv_bfloat16*>(take((size_t)NB * d * 2));
  w->xf_hi = reinterpret_cast<__nv_bfloat16*>(take((size_t)NB * d * 2));
  w->xf_lo = reinterpret_cast<__nv_bfloat16*>(take((size_t)NB * d * 2));
  w->urow = reinterpret_cast<int*>(take((size_t)d * 4));
  w->gstart = reinterpret_cast<int*>(take(G * 4));
  w->gcount = reinterpret_cast<int*>(take(G * 4));
  w->cnt = reinterpret_cast<int*>(take(16));
  w->part1 = reinterpret_cast<float*>(take((size_t)s1 * NB * 2 * F * 4));
  w->scores = reinterpret_cast<float*>(take((size_t)NB * F * 4));
  w->smask = reinterpret_cast<uint8_t*>(take((size_t)NB * F));
  w->ulist = reinterpret_cast<int*>(take((size_t)F * 4));
  w->utok = reinterpret_cast<uint32_t*>(take((size_t)F * 4));
  w->hh = reinterpret_cast<__nv_bfloat16*>(take((size_t)NB * Fp * 2));
  w->hl = reinterpret_cast<__nv_bfloat16*>(take((size_t)NB * Fp * 2));
  w->yp = reinterpret_cast<float*>(take((size_t)s5 * NB * d * 4));
}

cudaError_t setup_batch_kernels() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(batch_stage1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(S1Smem))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(batch_gateup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(GuSmem))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(batch_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(DnSmem))) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(batch_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)topk_smem(kMaxDff));
}

cudaError_t launch_batch(const prox_layer* L, const float* X, float* Y, int B, bool dense,
                         cudaStream_t s) {
  const BatchWs& w = L->bws;
  const int d = L->d, F = L->F;
  const __nv_bfloat16* wgu = reinterpret_cast<const __nv_bfloat16*>(L->wgu);
  const __nv_bfloat16* wd = reinterpret_cast<const __nv_bfloat16*>(L->wd);
  batch_prepare_kernel<<<1, 1024, 0, s>>>(X, B, d, L->tau, w, dense ? nullptr : L->ws.stats);
  if (!dense) {
    batch_stage1_kernel<<<dim3(2 * ((F + 511) / 512), L->b_s1), S1_THREADS, sizeof(S1Smem), s>>>(
        L->pq, reinterpret_cast<const __half*>(L->ps), d, F, w);
    const bool thr = L->mask_mode == PROX_MASK_THRESHOLD;
    batch_score_kernel<<<dim3((F + 255) / 256, B), 256, 0, s>>>(w, F, L->b_s1, L->act, thr ? 1 : 0,
                                                                L->tau_s);
    if (!thr) batch_topk_kernel<<<B, 1024, topk_smem(F), s>>>(w, F, L->k);
    batch_union_kernel<<<1, 1024, 0, s>>>(w, F, B, L->ws.stats);
  }
  batch_gateup_kernel<<<(F + GU_M - 1) / GU_M, GU_THREADS, sizeof(GuSmem), s>>>(wgu, d, F, B, L->act,
                                                                                dense ? 1 : 0, w);
  batch_down_kernel<<<dim3(d / DN_M, L->b_s5), DN_THREADS, sizeof(DnSmem), s>>>(wd, d, F, dense ? 1 : 0, w);
  batch_reduce_kernel<<<dim3((d + 255) / 256, B), 256, 0, s>>>(w, d, B, L->b_s5, Y);
  return cudaGetLastError();
}

}  // namespace prox
