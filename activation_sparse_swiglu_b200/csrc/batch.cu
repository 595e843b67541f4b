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

// Two kernels over blocks of 256 rows (two quantisation groups each).
// prepare_count: x split into xf_hi / xf_lo for the 16 token slots (0 past
// B), and each block's number of union rows in rcount[block]; adds the kept
// (token, row) pairs and the tokens to the layer's statistics.
__global__ void __launch_bounds__(256) batch_prepare_count_kernel(const float* __restrict__ X, int B, int d,
                                                                  float tau, BatchWs w,
                                                                  unsigned long long* stats, int count_kept) {
  __shared__ int s_red[8];
  const int r = blockIdx.x * 256 + threadIdx.x;
  bool any = false;
  int kept = 0;
  if (r < d) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float v = b < B ? __ldg(X + (size_t)b * d + r) : 0.f;
      const bool keep = b < B && fabsf(v) >= tau;
      kept += keep ? 1 : 0;
      any = any || keep;
      split_bf16(v, w.xf_hi + (size_t)b * d + r, w.xf_lo + (size_t)b * d + r);
    }
  }
  const int n_any = __syncthreads_count(any);
  // the block's kept pairs: warp sums, then warp 0
  int kw = kept;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kw += __shfl_xor_sync(0xffffffffu, kw, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = kw;
  __syncthreads();
  if (threadIdx.x == 0) {
    w.rcount[blockIdx.x] = n_any;
    int kt = 0;
    for (int i = 0; i < 8; ++i) kt += s_red[i];
    if (stats) {
      if (count_kept) atomicAdd(stats, (unsigned long long)kt);
      if (blockIdx.x == 0) atomicAdd(stats + 1, (unsigned long long)B);
    }
  }
}

// prepare_place: block j's union rows go to [sum of rcount[< j], ...) in
// ascending order: urow, xu_hi / xu_lo (x where the token keeps the row, else
// 0), gstart / gcount of its two groups; the last block writes cnt[0].
__global__ void __launch_bounds__(256) batch_prepare_place_kernel(const float* __restrict__ X, int B, int d,
                                                                  float tau, BatchWs w) {
  __shared__ int s_scan[40];
  const int blk = blockIdx.x, tid = threadIdx.x, r = blk * 256 + tid;
  int off = 0;
  if (tid < 32) {
    for (int j = tid; j < blk; j += 32) off += w.rcount[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) off += __shfl_xor_sync(0xffffffffu, off, o);
    if (tid == 0) s_scan[36] = off;
  }
  float xv[NB];
  bool any = false;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    xv[b] = (r < d && b < B) ? __ldg(X + (size_t)b * d + r) : 0.f;
    any = any || (r < d && b < B && fabsf(xv[b]) >= tau);
  }
  __syncthreads();
  off = s_scan[36];
  int total;
  const int pre = block_exclusive_scan(any ? 1 : 0, s_scan, &total);
  if (any) {
    const int pos = off + pre;
    w.urow[pos] = r;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float v = (b < B && fabsf(xv[b]) >= tau) ? xv[b] : 0.f;
      split_bf16(v, w.xu_hi + (size_t)b * d + pos, w.xu_lo + (size_t)b * d + pos);
    }
  }
  // the first group's count is the exclusive prefix at thread 128
  __shared__ int s_half;
  if (tid == 128) s_half = pre;
  __syncthreads();
  const int G = d / kGroup;
  if (tid == 0) {
    const int h0 = d - blk * 256 >= 256 ? s_half : total;  // a last block of 128 rows: one group
    w.gstart[2 * blk] = off;
    w.gcount[2 * blk] = h0;
    if (2 * blk + 1 < G) {
      w.gstart[2 * blk + 1] = off + h0;
      w.gcount[2 * blk + 1] = total - h0;
    }
    if (blk == gridDim.x - 1) w.cnt[0] = off + total;
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
  int scan[40];
  int ntiles;
};

// The half slice's output held at stored position m of the decoded tile
// (each word's outputs are stored 0 4 1 5 2 6 3 7).
__device__ __forceinline__ int s1_output(int m) {
  const int j = m & 7;
  return (m & ~7) | (j >> 1) | ((j & 1) << 2);
}

// Grid (2 C, S1 splits): CTA (hs, s) takes the outputs of half slice hs and
// the quantisation groups [G s / S1, G (s + 1) / S1); writes
// part1[s][token][gate|up][channel] (the group-scaled sums of its groups).
__global__ void __launch_bounds__(S1_THREADS, 2) batch_stage1_kernel(const uint8_t* __restrict__ pq,
                                                                  const __half* __restrict__ ps, int d,
                                                                  int F, BatchWs w) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  S1Smem& sm = *reinterpret_cast<S1Smem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hs = blockIdx.x, slice = hs >> 1, half = hs & 1;
  const int S1 = gridDim.y, s = blockIdx.y;
  const int G = d / kGroup;
  const int g0 = (int)((long long)G * s / S1), g1 = (int)((long long)G * (s + 1) / S1);
  // the CTA's tiles: each group's union rows in runs of at most S1_KT, listed
  // in parallel (thread j takes group g0 + j)
  {
    const int j = tid, g = g0 + j;
    const int c = g < g1 ? w.gcount[g] : 0, st = g < g1 ? w.gstart[g] : 0;
    const int n = (c + S1_KT - 1) / S1_KT;
    int tot;
    const int at = block_exclusive_scan(n, reinterpret_cast<int*>(sm.scan), &tot);
    for (int q = 0; q < n; ++q) {
      sm.t_i0[at + q] = st + q * S1_KT;
      sm.t_len[at + q] = (short)min(S1_KT, c - q * S1_KT);
      sm.t_grp[at + q] = (short)g;
    }
    if (tid == 0) sm.ntiles = tot;
  }
  for (int i = tid; i < S1_KT * S1_LDS; i += S1_THREADS) (&sm.S[0][0])[i] = __float2bfloat16_rn(0.f);
  __syncthreads();
  const int nt = sm.ntiles;
  const uint8_t* slice_base = pq + (size_t)slice * d * 512 + half * 256;

  // tile t's codes: row k = tid / 16 of the tile (k < len) into
  // raw[t % STAGES][k]; the row index is loaded a tile ahead (row_of)
  auto row_of = [&](int t) {
    const int k = tid >> 4;
    return (t < nt && k < sm.t_len[t]) ? __ldg(w.urow + sm.t_i0[t] + k) : -1;
  };
  auto issue = [&](int t, int row) {
    if (row >= 0) {
      const int k = tid >> 4, c16 = tid & 15;  // 32 rows x 16 chunks of 16 B
      cp16(&sm.raw[t % S1_STAGES][k][c16 * 16], slice_base + (size_t)row * 512 + c16 * 16);
    }
    cp_commit();
  };
  // tile t's x^ (token tid / 32, row tid % 32), fetched a tile ahead
  auto fetch_x = [&](int t, __nv_bfloat16& hi, __nv_bfloat16& lo) {
    const int n = tid >> 5, k = tid & 31;
    hi = lo = __float2bfloat16_rn(0.f);
    if (t < nt && k < sm.t_len[t]) {
      hi = w.xu_hi[(size_t)n * d + sm.t_i0[t] + k];
      lo = w.xu_lo[(size_t)n * d + sm.t_i0[t] + k];
    }
  };
  // the fp16 scales of this lane's four outputs in group grp
  const int g = lane >> 2;
  auto fetch_scales = [&](int grp, float (&sc)[2][2]) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int m = s1_output(warp * 32 + i * 16 + g + 8 * r);
        const int blk = (slice * 512 + half * 256) / 32 + (m >> 6);  // < F / 32 for real channels
        sc[i][r] = blk < F / 32 ? __half2float(__ldg(ps + ((size_t)grp * (F / 32) + blk) * 64 + (m & 63))) : 0.f;
      }
  };
#pragma unroll
  for (int t = 0; t < S1_STAGES - 1; ++t) issue(t, row_of(t));
  int row_next = row_of(S1_STAGES - 1);
  __nv_bfloat16 xh, xl;
  fetch_x(0, xh, xl);
  float scl[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  if (nt > 0) fetch_scales(sm.t_grp[0], scl);

  float acc[2][2][4], tot[2][2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][h][e] = tot[i][h][e] = 0.f;

  for (int t = 0; t < nt; ++t) {
    issue(t + S1_STAGES - 1, row_next);
    row_next = row_of(t + S1_STAGES);
    cp_wait<S1_STAGES - 1>();
    __syncthreads();  // tile t's codes are in; the previous tile's products are done
    const int len = sm.t_len[t];
    sm.bhi[tid >> 5][tid & 31] = xh;
    sm.blo[tid >> 5][tid & 31] = xl;
    fetch_x(t + 1, xh, xl);
    // decode: 32 rows x 64 words, 4 words per thread; word wd of row k holds
    // outputs 8 wd .. 8 wd + 7 (nibble p is output 8 wd + p; the code is
    // q + 8).  Nibbles p and p + 4 sit 16 bits apart, so one mask-and-or puts
    // both into a bf16 pair 128 + code; the stored order of the word's
    // outputs is therefore 0 4 1 5 2 6 3 7 (s1_output maps it back).
    for (int j = tid; j < S1_KT * 64; j += S1_THREADS) {
      const int k = j >> 6, wd = j & 63;
      if (k < len) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(&sm.raw[t % S1_STAGES][k][wd * 4]);
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const uint32_t pair = ((v >> (4 * p)) & 0x000F000Fu) | 0x43004300u;  // bf16 128 + code
          __nv_bfloat162 q = *reinterpret_cast<const __nv_bfloat162*>(&pair);
          q = __hsub2(q, __floats2bfloat162_rn(136.f, 136.f));  // exact: q in [-8, 7]
          o[p] = *reinterpret_cast<const uint32_t*>(&q);
        }
        *reinterpret_cast<uint4*>(&sm.S[k][wd * 8]) = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
        *reinterpret_cast<uint4*>(&sm.S[k][wd * 8]) = make_uint4(0u, 0u, 0u, 0u);
      }
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
    // the group's last tile: scale its sums per (group, output) and add them;
    // the next group's scales are fetched right away
    if (t + 1 == nt || sm.t_grp[t + 1] != sm.t_grp[t]) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tot[i][h][2 * r] = fmaf(scl[i][r], acc[i][h][2 * r], tot[i][h][2 * r]);
            tot[i][h][2 * r + 1] = fmaf(scl[i][r], acc[i][h][2 * r + 1], tot[i][h][2 * r + 1]);
            acc[i][h][2 * r] = acc[i][h][2 * r + 1] = 0.f;
          }
      if (t + 1 < nt) fetch_scales(sm.t_grp[t + 1], scl);
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
      const int m = s1_output(warp * 32 + i * 16 + g + 8 * r);
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
// channel).  A most-significant-digit-first radix select over the keys (the
// scores' bits), 8 bits per level, each level a shared-memory histogram of
// the keys that match the digits fixed so far; then, among the keys equal to
// the k-th largest, the lowest-indexed ones up to the rank still wanted.
constexpr int TK_THREADS = 1024;
__global__ void __launch_bounds__(TK_THREADS) batch_topk_kernel(BatchWs w, int F, int k) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw);  // [F]
  __shared__ int hist[256];
  __shared__ int s_pick[4];
  __shared__ int s_scan[40];
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* src = w.scores + (size_t)b * F;
  for (int j = tid; j < F; j += TK_THREADS) keys[j] = __float_as_uint(src[j]);
  uint32_t prefix = 0u, pmask = 0u;
  int krem = k, n_eq = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int j = tid; j < F; j += TK_THREADS) {
      const uint32_t key = keys[j];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255 - 8 l .. 248 - 8 l (descending)
      int c[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * lane - i];
        sum += c[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int above = incl - sum;
      if (above < krem && incl >= krem) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above < krem && above + c[i] >= krem) {
            s_pick[0] = 255 - 8 * lane - i;
            s_pick[1] = krem - above;
            s_pick[2] = c[i];
            above = krem;  // done
          } else {
            above += c[i];
          }
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_pick[0] << shift;
    pmask |= 255u << shift;
    krem = s_pick[1];
    n_eq = s_pick[2];
    __syncthreads();
  }
  // ties: the krem lowest channels among the n_eq keys equal to prefix
  int tie_cut = F;
  if (krem < n_eq) {
    const int per = (F + TK_THREADS - 1) / TK_THREADS;
    const int j0 = min(tid * per, F), j1 = min(j0 + per, F);
    int c = 0;
    for (int j = j0; j < j1; ++j) c += keys[j] == prefix;
    int tot;
    const int before = block_exclusive_scan(c, s_scan, &tot);
    if (before < krem && before + c >= krem) {
      int seen = before;
      for (int j = j0; j < j1; ++j)
        if (keys[j] == prefix && ++seen == krem) s_pick[3] = j;
    }
    __syncthreads();
    tie_cut = s_pick[3];
  }
  TopkCut cut;
  cut.T = prefix;
  cut.tie_cut = tie_cut;
  for (int j = tid; j < F; j += TK_THREADS) w.smask[(size_t)b * F + j] = selected(keys[j], j, cut) ? 1 : 0;
}

// The channels some token selected, ascending, with the bit set of the
// tokens that did, in two kernels over blocks of 256 channels like prepare:
// union_count writes each block's count to ccount and adds the selected
// (token, channel) pairs to the layer's statistics; union_place writes
// ulist / utok and, in the last block, cnt[1].
__device__ __forceinline__ uint32_t token_bits(const BatchWs& w, int F, int B, int ch) {
  uint32_t bits = 0u;
  if (ch < F)
    for (int b = 0; b < B; ++b) bits |= w.smask[(size_t)b * F + ch] ? (1u << b) : 0u;
  return bits;
}

__global__ void __launch_bounds__(256) batch_union_count_kernel(BatchWs w, int F, int B,
                                                                unsigned long long* stats) {
  __shared__ int s_red[8];
  const int ch = blockIdx.x * 256 + threadIdx.x;
  const uint32_t bits = token_bits(w, F, B, ch);
  const int n = __syncthreads_count(bits != 0u);
  int sel = __popc(bits);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sel += __shfl_xor_sync(0xffffffffu, sel, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = sel;
  __syncthreads();
  if (threadIdx.x == 0) {
    w.ccount[blockIdx.x] = n;
    int t = 0;
    for (int i = 0; i < 8; ++i) t += s_red[i];
    if (stats) atomicAdd(stats + 2, (unsigned long long)t);
  }
}

__global__ void __launch_bounds__(256) batch_union_place_kernel(BatchWs w, int F, int B) {
  __shared__ int s_scan[40];
  const int blk = blockIdx.x, tid = threadIdx.x, ch = blk * 256 + tid;
  if (tid < 32) {
    int off = 0;
    for (int j = tid; j < blk; j += 32) off += w.ccount[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) off += __shfl_xor_sync(0xffffffffu, off, o);
    if (tid == 0) s_scan[36] = off;
  }
  const uint32_t bits = token_bits(w, F, B, ch);
  __syncthreads();
  const int off = s_scan[36];
  int total;
  const int pre = block_exclusive_scan(bits ? 1 : 0, s_scan, &total);
  if (bits) {
    w.ulist[off + pre] = ch;
    w.utok[off + pre] = bits;
  }
  if (tid == 0 && blk == gridDim.x - 1) w.cnt[1] = off + total;
}

// ---------------------------------------------------------------------------
// gate/up over the union channels (or every channel: dense)
// ---------------------------------------------------------------------------

constexpr int GU_THREADS = 256;  // 8 warps: gate / up x four 16-channel tiles
constexpr int GU_M = 64;         // channels per work tile
constexpr int GU_KT = 64;        // d_model elements per stage
constexpr int GU_STAGES = 3;
constexpr int GU_LDA = GU_KT + 8;
constexpr int GU_MAXE = 1024;    // union entries a CTA's run may touch (checked by the host)

struct GuSmem {
  __nv_bfloat16 a[GU_STAGES][2][GU_M][GU_LDA];     // gate, up column slices [channel][k]
  __nv_bfloat16 bhi[GU_STAGES][NB][GU_LDA], blo[GU_STAGES][NB][GU_LDA];  // x [token][k]
  int ch[GU_MAXE];                                 // channels of the run's union entries
};

// Work items (tile, ks): union entries [64 tile, 64 tile + 64) (dense:
// channels) over the d_model range ks of KS equal ranges of k tiles; the
// T KS items (T = ceil(n / 64)) are split into equal contiguous runs, one per
// CTA, and a CTA streams the k tiles of its run through one cp.async ring
// (the run's channel indices staged in shared memory first), writing each
// item's gate and up sums to gup[item][entry][token][gate|up].
__global__ void __launch_bounds__(GU_THREADS) batch_gateup_kernel(const __nv_bfloat16* __restrict__ wgu, int d,
                                                                  int F, int KS, int dense, BatchWs w) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  GuSmem& sm = *reinterpret_cast<GuSmem*>(smem_raw);
  const int n_s = dense ? F : w.cnt[1];
  const int T = (n_s + GU_M - 1) / GU_M, I = T * KS;
  const int it0 = (int)((long long)I * blockIdx.x / gridDim.x);
  const int it1 = (int)((long long)I * (blockIdx.x + 1) / gridDim.x);
  const int kper = d / GU_KT / KS;        // k tiles per item
  const int nsteps = (it1 - it0) * kper;
  if (nsteps <= 0) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kind = warp >> 2, m0 = (warp & 3) * 16;
  const int e_base = (it0 / KS) * GU_M;
  const int ne = min(GU_MAXE, ((it1 - 1) / KS + 1) * GU_M - e_base);
  for (int i = tid; i < ne; i += GU_THREADS) {
    const int e = e_base + i;
    sm.ch[i] = dense ? min(e, F - 1) : __ldg(w.ulist + min(e, n_s - 1));
  }
  __syncthreads();

  auto issue = [&](int step) {
    if (step < nsteps) {
      const int st = step % GU_STAGES, item = it0 + step / kper;
      const int el = (item / KS) * GU_M - e_base;
      const int k0 = ((item % KS) * kper + step % kper) * GU_KT;
      // 2 x 64 channels x 8 chunks, then 2 x 16 tokens x 8 chunks: 1280 copies
      for (int j = tid; j < 1280; j += GU_THREADS) {
        if (j < 1024) {
          const int kd = j >> 9, m = (j >> 3) & 63, c = j & 7;
          const size_t col = (size_t)sm.ch[el + m] * 2 * d + (size_t)kd * d + k0 + c * 8;
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
  for (int q = 0; q < GU_STAGES - 1; ++q) issue(q);
  float acc[2][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
  const int g = lane >> 2, t = lane & 3;
  for (int step = 0; step < nsteps; ++step) {
    issue(step + GU_STAGES - 1);
    cp_wait<GU_STAGES - 1>();
    __syncthreads();
    const int st = step % GU_STAGES;
#pragma unroll
    for (int k0 = 0; k0 < GU_KT; k0 += 16) {
      uint32_t a[4];
      ldsm_a(a, a_row_mk(&sm.a[st][kind][0][0], GU_LDA, m0, k0));
      mma_tokens(acc, a, &sm.bhi[st][0][0], &sm.blo[st][0][0], GU_LDA, k0);
    }
    if (step % kper == kper - 1) {
      const int item = it0 + step / kper;
      float* dst = w.gup + (size_t)item * GU_M * NB * 2;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            dst[((m0 + g + 8 * r) * NB + 8 * h + 2 * t + c) * 2 + kind] = acc[h][2 * r + c];
            acc[h][2 * r + c] = 0.f;
          }
    }
    __syncthreads();
  }
  cp_wait<0>();
}

// One thread per (union entry < roundup(n, 64), token): g and u summed over
// the KS items in order, h = act(g) u for the tokens that selected the
// channel (every token < B when dense), 0 otherwise; split into hh / hl.
__global__ void batch_gateup_finish_kernel(BatchWs w, int F, int B, int KS, int act, int dense) {
  const int n_s = dense ? F : w.cnt[1];
  const int e = blockIdx.x * (blockDim.x / NB) + threadIdx.x / NB, n = threadIdx.x % NB;
  const int Fp = (F + 63) & ~63;
  if (e >= ((n_s + 63) / 64) * 64) return;
  float h = 0.f;
  if (e < n_s && n < B && (dense || ((__ldg(w.utok + e) >> n) & 1u))) {
    const int tile = e / GU_M, m = e % GU_M;
    float gs = 0.f, us = 0.f;
    for (int ks = 0; ks < KS; ++ks) {
      const float2 v = *reinterpret_cast<const float2*>(
          w.gup + (((size_t)(tile * KS + ks) * GU_M + m) * NB + n) * 2);
      gs += v.x;
      us += v.y;
    }
    h = act_f32(gs, act) * us;
  }
  split_bf16(h, w.hh + (size_t)n * Fp + e, w.hl + (size_t)n * Fp + e);
}

// ---------------------------------------------------------------------------
// down over the union channels, then the split sum
// ---------------------------------------------------------------------------

constexpr int DN_THREADS = 256;  // 8 warps, two 16-column tiles each
constexpr int DN_M = 256;        // output columns per CTA: 512 contiguous bytes per W_down row
constexpr int DN_KT = 32;        // union entries per stage
constexpr int DN_STAGES = 4;
constexpr int DN_LDA = DN_M + 8;
constexpr int DN_LDB = DN_KT + 8;
constexpr int DN_MAXE = 4096;    // union entries a CTA's split may touch (checked by the host)

struct DnSmem {
  __nv_bfloat16 a[DN_STAGES][DN_KT][DN_LDA];        // W_down rows' column slices [entry][column]
  __nv_bfloat16 bhi[DN_STAGES][NB][DN_LDB], blo[DN_STAGES][NB][DN_LDB];  // h [token][entry]
  int ch[DN_MAXE];                                  // the split's channels
};

// Grid (d / 256, S5): CTA (cb, s) takes columns [256 cb, 256 cb + 256) and the
// entry tiles [T s / S5, T (s + 1) / S5) of the T = ceil(n / 32) tiles;
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
  for (int i = tid; i < nt * DN_KT; i += DN_THREADS) {
    const int e = t0 * DN_KT + i;
    sm.ch[i] = dense ? min(e, F - 1) : __ldg(w.ulist + min(e, n_s - 1));
  }
  __syncthreads();
  auto issue = [&](int it) {
    if (it < nt) {
      const int st = it % DN_STAGES, e0 = (t0 + it) * DN_KT;
      // 32 entries x 32 chunks, then 2 x 16 tokens x 4 chunks: 1152 copies
      for (int j = tid; j < 1152; j += DN_THREADS) {
        if (j < 1024) {
          const int k = j >> 5, c = j & 31;
          if (col0 + c * 8 < d)
            cp16(&sm.a[st][k][c * 8], wd + (size_t)sm.ch[it * DN_KT + k] * d + col0 + c * 8);
          else  // past the last column (d_model not a multiple of 256)
            *reinterpret_cast<uint4*>(&sm.a[st][k][c * 8]) = make_uint4(0u, 0u, 0u, 0u);
        } else {
          const int jj = j - 1024, lo = jj >> 6, n = (jj >> 2) & 15, c = jj & 3;
          const __nv_bfloat16* src = (lo ? w.hl : w.hh) + (size_t)n * Fp + e0 + c * 8;
          cp16(lo ? &sm.blo[st][n][c * 8] : &sm.bhi[st][n][c * 8], src);
        }
      }
    }
    cp_commit();
  };
#pragma unroll
  for (int it = 0; it < DN_STAGES - 1; ++it) issue(it);
  float acc[2][2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][h][e] = 0.f;
  for (int it = 0; it < nt; ++it) {
    issue(it + DN_STAGES - 1);
    cp_wait<DN_STAGES - 1>();
    __syncthreads();
    const int st = it % DN_STAGES;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int k0 = 0; k0 < DN_KT; k0 += 16) {
        uint32_t a[4];
        ldsm_a_trans(a, a_row_km(&sm.a[st][0][0], DN_LDA, warp * 32 + i * 16, k0));
        mma_tokens(acc[i], a, &sm.bhi[st][0][0], &sm.blo[st][0][0], DN_LDB, k0);
      }
    __syncthreads();
  }
  cp_wait<0>();
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = col0 + warp * 32 + i * 16 + g + 8 * r;
          if (col < d) w.yp[((size_t)s * NB + 8 * h + 2 * t + c) * d + col] = acc[i][h][2 * r + c];
        }
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
size_t topk_smem(int F) { return (size_t)F * 4; }
size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }
}  // namespace

void choose_batch_splits(int d, int F, int num_sms, int* s1, int* s5, int* ks) {
  const int hs = 2 * ((F + 511) / 512);  // half slices
  const int G = d / kGroup;
  *s1 = std::max(1, std::min(G, (2 * num_sms + hs - 1) / hs));
  *s5 = std::max(1, 2 * num_sms / ((d + DN_M - 1) / DN_M));
  // a split's entries must fit its channel table: at most DN_MAXE
  while ((size_t)((F + DN_KT - 1) / DN_KT + *s5 - 1) / *s5 * DN_KT > (size_t)DN_MAXE) ++*s5;
  const int nkt = (d + GU_KT - 1) / GU_KT;
  int k = std::min(8, nkt);
  while (nkt % k) --k;
  *ks = k;
}

bool batch_fits(int F, int num_sms, int ks) {
  // a gate/up run (3 num_sms CTAs) touches at most this many union entries
  const long long T = (F + GU_M - 1) / GU_M, I = T * ks, grid = 3LL * num_sms;
  return ((I + grid - 1) / grid / ks + 2) * GU_M <= GU_MAXE;
}

size_t batch_ws_bytes(int d, int F, int s1, int s5, int ks) {
  const size_t Fp = (size_t)((F + 63) & ~63), G = (size_t)d / kGroup;
  return 4 * al256((size_t)NB * d * 2) + al256((size_t)d * 4) + 2 * al256(G * 4) + al256(16) +
         al256((size_t)(d + 255) / 256 * 4) + al256((size_t)(F + 255) / 256 * 4) +
         al256((size_t)s1 * NB * 2 * F * 4) + al256((size_t)NB * F * 4) + al256((size_t)NB * F * 4) +
         2 * al256((size_t)F * 4) + al256(Fp / GU_M * ks * GU_M * NB * 2 * 4) +
         2 * al256((size_t)NB * Fp * 2) + al256((size_t)s5 * NB * d * 4);
}

void carve_batch_ws(void* base, int d, int F, int s1, int s5, int ks, BatchWs* w) {
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
  w->rcount = reinterpret_cast<int*>(take((size_t)(d + 255) / 256 * 4));
  w->ccount = reinterpret_cast<int*>(take((size_t)(F + 255) / 256 * 4));
  w->part1 = reinterpret_cast<float*>(take((size_t)s1 * NB * 2 * F * 4));
  w->scores = reinterpret_cast<float*>(take((size_t)NB * F * 4));
  w->smask = reinterpret_cast<int32_t*>(take((size_t)NB * F * 4));
  w->ulist = reinterpret_cast<int*>(take((size_t)F * 4));
  w->utok = reinterpret_cast<uint32_t*>(take((size_t)F * 4));
  w->gup = reinterpret_cast<float*>(take(Fp / GU_M * ks * GU_M * NB * 2 * 4));  // Fp / 16 tiles
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
  const int rb = (d + 255) / 256, cb = (F + 255) / 256;
  const bool per_token = !dense && B <= kBatchPerTokenStage1;
  // (per token, Stage 1 itself counts the kept rows)
  batch_prepare_count_kernel<<<rb, 256, 0, s>>>(X, B, d, L->tau, w, dense ? nullptr : L->ws.stats,
                                                per_token ? 0 : 1);
  batch_prepare_place_kernel<<<rb, 256, 0, s>>>(X, B, d, L->tau, w);
  if (per_token) {
    // each token's Stage 1, scores and mask from the per-token kernel, which
    // reads only that token's kept rows; then the union of the masks
    for (int b = 0; b < B; ++b) {
      TokenLaunch m;
      m.x = X + (size_t)b * d;
      m.stage1 = true;
      m.mode = L->mask_mode == PROX_MASK_THRESHOLD ? 3 : 1;
      m.k = L->k;
      m.tau_s = L->tau_s;
      m.select_only = true;
      m.sel_mask = w.smask + (size_t)b * F;
      cudaError_t e = launch_token(L, m, s, false);
      if (e != cudaSuccess) return e;
    }
    batch_union_count_kernel<<<cb, 256, 0, s>>>(w, F, B, L->ws.stats);
    batch_union_place_kernel<<<cb, 256, 0, s>>>(w, F, B);
  } else if (!dense) {
    batch_stage1_kernel<<<dim3(2 * ((F + 511) / 512), L->b_s1), S1_THREADS, sizeof(S1Smem), s>>>(
        L->pq, reinterpret_cast<const __half*>(L->ps), d, F, w);
    const bool thr = L->mask_mode == PROX_MASK_THRESHOLD;
    batch_score_kernel<<<dim3((F + 255) / 256, B), 256, 0, s>>>(w, F, L->b_s1, L->act, thr ? 1 : 0,
                                                                L->tau_s);
    if (!thr) batch_topk_kernel<<<B, TK_THREADS, topk_smem(F), s>>>(w, F, L->k);
    batch_union_count_kernel<<<cb, 256, 0, s>>>(w, F, B, L->ws.stats);
    batch_union_place_kernel<<<cb, 256, 0, s>>>(w, F, B);
  }
  batch_gateup_kernel<<<3 * L->num_sms, GU_THREADS, sizeof(GuSmem), s>>>(wgu, d, F, L->b_ks,
                                                                          dense ? 1 : 0, w);
  const int Fp = (F + 63) & ~63;
  batch_gateup_finish_kernel<<<Fp * NB / 256, 256, 0, s>>>(w, F, B, L->b_ks, L->act, dense ? 1 : 0);
  batch_down_kernel<<<dim3((d + DN_M - 1) / DN_M, L->b_s5), DN_THREADS, sizeof(DnSmem), s>>>(
      wd, d, F, dense ? 1 : 0, w);
  batch_reduce_kernel<<<dim3((d + 255) / 256, B), 256, 0, s>>>(w, d, B, L->b_s5, Y);
  return cudaGetLastError();
}

}  // namespace prox
