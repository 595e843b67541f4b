// Stage 1 of the Prox decode step (Prox §4.1 "Stage 1: lightweight proxy
// construction", §4.3 fused split-N proxy kernel), and the per-token top-k
// channel select (Prox App. A.6 "Per-token top-k selection").
//
// stage1_kernel -- one CTA per (column slice c, row slab r):
//   * a column slice is 512 bytes of an interleaved proxy row (16 blocks of
//     32 channels: 16 B of gate codes then 16 B of up codes per block), i.e.
//     512 channels of both proxies; each lane of a warp owns one 16-byte chunk
//     (32 channels of one branch);
//   * a row slab is `gps` whole quantisation groups (gps * 128 input rows).
//   The CTA thresholds its slab of x (|x_i| >= tau), compacts the kept rows in
//   ascending order, and its 4 warps stream those rows' chunks from HBM
//   (16-byte loads, no L1 allocation), dequantising the INT4 codes in
//   registers with fp32 (packed f32x2) arithmetic.  Codes are accumulated per
//   group and scaled once per group by the fp16 group scale.  Each CTA writes
//   a fp32 partial for its slab; the last CTA of a column slice (atomic
//   ticket, no waiting) sums the slabs in a fixed order, forms
//   score_j = |SiLU(g~_j) u~_j| and adds each score to a 2048-bin histogram of
//   its top bits -- the first level of the radix select.
//
// select_kernel -- one CTA of 1024 threads: radix select of the k-th largest
// score (fp32 bit patterns are monotone for non-negative values) in three
// levels (bits 30..20 from the histogram above, then 19..8 and 7..0 over the
// scores held in shared memory), then an ordered compaction that emits the k
// selected channels in ascending order, equal scores going to the lower index.
#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {
namespace {

constexpr int S1_NW = kStage1Warps;
constexpr int S1_NT = S1_NW * 32;
constexpr int S1_U = 8;  // rows in flight per warp

struct Stage1Args {
  const float* x;
  const uint8_t* pq;
  const __half* ps;
  float tau;
  int d, F, C, R, gps;
  float* part;
  float* scores;
  uint32_t* hist;
  uint32_t* slice_cnt;
  unsigned long long* stats;
  float* g_dbg;
  float* u_dbg;
  int32_t* slab_idx;
  int32_t* slab_cnt;
};

// Eight INT4 codes of one 32-bit word (channels 8w..8w+7 of a chunk; nibble p
// is channel 8w+p, stored as q+8) into four float2 accumulators.
// Each nibble is OR-ed into the mantissa of a float whose exponent makes the
// nibble's lowest bit worth exactly 1, so subtracting (2^e + 8) leaves q - 8
// exactly; nibbles 5..7 are first shifted down by 12 bits.
__device__ __forceinline__ void acc_word(float2* a, uint32_t w, float2 x2) {
  const uint32_t h = w >> 12;
  const float2 v0 = __fadd2_rn(make_float2(__uint_as_float((w & 0x0000000Fu) | 0x4B000000u),
                                           __uint_as_float((w & 0x000000F0u) | 0x49000000u)),
                               make_float2(-8388616.0f, -524296.0f));
  const float2 v1 = __fadd2_rn(make_float2(__uint_as_float((w & 0x00000F00u) | 0x47000000u),
                                           __uint_as_float((w & 0x0000F000u) | 0x45000000u)),
                               make_float2(-32776.0f, -2056.0f));
  const float2 v2 = __fadd2_rn(make_float2(__uint_as_float((w & 0x000F0000u) | 0x43000000u),
                                           __uint_as_float((h & 0x00000F00u) | 0x47000000u)),
                               make_float2(-136.0f, -32776.0f));
  const float2 v3 = __fadd2_rn(make_float2(__uint_as_float((h & 0x0000F000u) | 0x45000000u),
                                           __uint_as_float((h & 0x000F0000u) | 0x43000000u)),
                               make_float2(-2056.0f, -136.0f));
  a[0] = __ffma2_rn(v0, x2, a[0]);
  a[1] = __ffma2_rn(v1, x2, a[1]);
  a[2] = __ffma2_rn(v2, x2, a[2]);
  a[3] = __ffma2_rn(v3, x2, a[3]);
}

__device__ __forceinline__ void acc_chunk(float2 (&a)[16], const uint4& v, float x) {
  const float2 x2 = make_float2(x, x);
  acc_word(a + 0, v.x, x2);
  acc_word(a + 4, v.y, x2);
  acc_word(a + 8, v.z, x2);
  acc_word(a + 12, v.w, x2);
}

__global__ void __launch_bounds__(S1_NT) stage1_kernel(Stage1Args a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int c = blockIdx.x, r = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gps = a.gps, slab_rows = gps * kGroup, row0 = r * slab_rows;
  const int nchunks = a.F >> 4, nblk = a.F >> 5;
  const int chunk = c * 32 + lane;
  const bool lane_ok = chunk < nchunks;

  uint4* s_scale = reinterpret_cast<uint4*>(smem);                      // [gps][32][4]
  float* s_red = reinterpret_cast<float*>(smem + (size_t)gps * 2048);   // [NW][1024]
  int* s_row = reinterpret_cast<int*>(s_red + S1_NW * 1024);            // [slab_rows]
  float* s_xv = reinterpret_cast<float*>(s_row + slab_rows);            // [slab_rows]
  int* s_gstart = reinterpret_cast<int*>(s_xv + slab_rows);             // [gps + 1]
  int* s_scan = s_gstart + gps + 1;                                     // [33]
  int* s_flag = s_scan + 33;                                            // [1]

  // Prologue (constant weights only): this slice's fp16 scales for the slab's
  // groups, 64 bytes per lane and group.
  for (int e = tid; e < gps * 128; e += S1_NT) {
    const int gl = e >> 7, ln = (e >> 2) & 31, qd = e & 3;
    const int ch = c * 32 + ln;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (ch < nchunks) {
      const int g = (row0 / kGroup) + gl;
      const __half* src = a.ps + ((size_t)g * nblk + (ch >> 1)) * 64 + (ch & 1) * 32 + qd * 8;
      v = __ldg(reinterpret_cast<const uint4*>(src));
    }
    s_scale[(gl * 32 + ln) * 4 + qd] = v;
  }

  pdl_wait();     // x and the workspace now belong to this token
  pdl_trigger();  // let the select kernel become resident

  // Kept rows of this slab, ascending: thread t owns rows [t*gps, (t+1)*gps).
  const int rpt = slab_rows / S1_NT;
  int cnt = 0;
  for (int q = 0; q < rpt; ++q) cnt += fabsf(__ldg(a.x + row0 + tid * rpt + q)) >= a.tau;
  int total;
  int pos = block_exclusive_scan(cnt, s_scan, &total);
  for (int q = 0; q < rpt; ++q) {
    const int ri = tid * rpt + q;
    if ((ri & (kGroup - 1)) == 0) s_gstart[ri / kGroup] = pos;
    const float xv = __ldg(a.x + row0 + ri);
    if (fabsf(xv) >= a.tau) {
      s_row[pos] = row0 + ri;
      s_xv[pos] = xv;
      ++pos;
    }
  }
  if (tid == 0) s_gstart[gps] = total;
  __syncthreads();
  if (c == 0) {
    if (tid == 0) atomicAdd(a.stats, (unsigned long long)total);
    if (a.slab_idx) {
      for (int e = tid; e < total; e += S1_NT) a.slab_idx[row0 + e] = s_row[e];
      if (tid == 0) a.slab_cnt[r] = total;
    }
  }

  // Stream the kept rows' 16-byte chunks, group by group.
  float2 tot[16];
#pragma unroll
  for (int h = 0; h < 16; ++h) tot[h] = make_float2(0.f, 0.f);
  const uint8_t* colp = a.pq + (size_t)chunk * 16;
  for (int gl = 0; gl < gps; ++gl) {
    const int gs = s_gstart[gl], ge = s_gstart[gl + 1];
    float2 acc[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) acc[h] = make_float2(0.f, 0.f);
    for (int base = gs + warp; base < ge; base += S1_NW * S1_U) {
      uint4 v[S1_U];
      float xv[S1_U];
#pragma unroll
      for (int u = 0; u < S1_U; ++u) {
        const int e = base + u * S1_NW;
        const bool ok = e < ge;
        const int row = ok ? s_row[e] : 0;
        xv[u] = ok ? s_xv[e] : 0.f;
        v[u] = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
        if (ok && lane_ok) v[u] = ld_stream_v4(colp + (size_t)row * a.F);
      }
#pragma unroll
      for (int u = 0; u < S1_U; ++u) acc_chunk(acc, v[u], xv[u]);
    }
    const uint4* sc = s_scale + (gl * 32 + lane) * 4;
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const uint4 s4 = sc[qd];
      const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&sw[m]));
        tot[qd * 4 + m] = __ffma2_rn(s2, acc[qd * 4 + m], tot[qd * 4 + m]);
      }
    }
  }

  // Combine the warps (fixed order) into this CTA's partial.  Partial layout:
  // element e = j*32 + lane for channel j of the lane's chunk.
  float* red = s_red + warp * 1024;
#pragma unroll
  for (int h = 0; h < 16; ++h) {
    red[(2 * h) * 32 + lane] = tot[h].x;
    red[(2 * h + 1) * 32 + lane] = tot[h].y;
  }
  __syncthreads();
  float* dst = a.part + ((size_t)r * a.C + c) * 1024;
  for (int e = tid; e < 1024; e += S1_NT) {
    float s = s_red[e];
#pragma unroll
    for (int w = 1; w < S1_NW; ++w) s += s_red[w * 1024 + e];
    dst[e] = s;
  }

  // The last CTA of this column slice sums the slabs and scores the channels.
  __threadfence();
  __syncthreads();
  if (tid == 0) *s_flag = (atomicAdd(a.slice_cnt + c, 1u) == (unsigned)(a.R - 1));
  __syncthreads();
  if (!*s_flag) return;
  __threadfence();
  float* sum = s_red;
  for (int e = tid; e < 1024; e += S1_NT) {
    float s = 0.f;
    for (int rr = 0; rr < a.R; ++rr) s += __ldcg(a.part + ((size_t)rr * a.C + c) * 1024 + e);
    sum[e] = s;
  }
  __syncthreads();
  for (int m = tid; m < 512; m += S1_NT) {
    const int ch = c * 512 + m;
    if (ch < a.F) {
      const int blk = m >> 5, jj = m & 31;
      const float g = sum[jj * 32 + 2 * blk];
      const float u = sum[jj * 32 + 2 * blk + 1];
      const float sc = fabsf(silu_f32(g) * u);
      a.scores[ch] = sc;
      if (a.g_dbg) a.g_dbg[ch] = g;
      if (a.u_dbg) a.u_dbg[ch] = u;
      atomicAdd(a.hist + (__float_as_uint(sc) >> 20), 1u);
    }
  }
  if (tid == 0) a.slice_cnt[c] = 0u;
}

// ---------------------------------------------------------------------------

struct SelectArgs {
  const float* scores;
  uint32_t* hist;
  int F, k;
  int32_t* idx_s;
  int32_t* k_dev;
  unsigned long long* stats;
  const int32_t* slab_idx;
  const int32_t* slab_cnt;
  int R, slab_rows;
  int32_t* idx_x;
  int32_t* n_x;
};

// Among nb bins of h (counts of keys per bin, larger bin = larger key), find
// the bin holding the krem-th largest key (1-based).  Writes the bin and the
// remaining rank inside it to out[0], out[1].
__device__ void find_bin_desc(const uint32_t* h, int nb, int krem, int* scan, int* out) {
  const int nt = blockDim.x;
  const int per = (nb + nt - 1) / nt;
  const int lo = threadIdx.x * per;
  const int hi = min(lo + per, nb);
  int v = 0;
  for (int b = lo; b < hi; ++b) v += (int)h[b];
  int total;
  const int excl = block_exclusive_scan(v, scan, &total);
  int running = total - excl - v;  // keys in bins above this thread's range
  for (int b = hi - 1; b >= lo; --b) {
    const int hb = (int)h[b];
    if (running < krem && running + hb >= krem) {
      out[0] = b;
      out[1] = krem - running;
    }
    running += hb;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSelectThreads) select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t s_keys[];  // [F]
  __shared__ uint32_t s_h[4096];
  __shared__ int s_scan[33];
  __shared__ int s_sel[2];
  const int tid = threadIdx.x;
  constexpr int NT = kSelectThreads;
  const int F = a.F;

  pdl_wait();
  pdl_trigger();

  for (int e = tid; e < F; e += NT) s_keys[e] = __float_as_uint(__ldcg(a.scores + e));
  for (int b = tid; b < kHistBins; b += NT) {
    s_h[b] = __ldcg(a.hist + b);
    a.hist[b] = 0u;  // ready for the next token
  }
  __syncthreads();

  // level 1: bits 30..20
  find_bin_desc(s_h, kHistBins, a.k, s_scan, s_sel);
  const uint32_t b1 = (uint32_t)s_sel[0];
  int krem = s_sel[1];
  // level 2: bits 19..8 among keys of bin b1
  for (int b = tid; b < 4096; b += NT) s_h[b] = 0u;
  __syncthreads();
  for (int e = tid; e < F; e += NT) {
    const uint32_t key = s_keys[e];
    if ((key >> 20) == b1) atomicAdd(&s_h[(key >> 8) & 0xFFFu], 1u);
  }
  __syncthreads();
  find_bin_desc(s_h, 4096, krem, s_scan, s_sel);
  const uint32_t p2 = (b1 << 12) | (uint32_t)s_sel[0];
  krem = s_sel[1];
  // level 3: bits 7..0
  for (int b = tid; b < 256; b += NT) s_h[b] = 0u;
  __syncthreads();
  for (int e = tid; e < F; e += NT) {
    const uint32_t key = s_keys[e];
    if ((key >> 8) == p2) atomicAdd(&s_h[key & 0xFFu], 1u);
  }
  __syncthreads();
  find_bin_desc(s_h, 256, krem, s_scan, s_sel);
  const uint32_t T = (p2 << 8) | (uint32_t)s_sel[0];
  const int k_eq = s_sel[1];  // keys equal to T that are taken (lowest indices)

  // Ordered compaction: thread t owns channels [t*per, (t+1)*per).
  const int per = (F + NT - 1) / NT;
  const int lo = min(tid * per, F), hi = min(lo + per, F);
  int gt = 0, eq = 0;
  for (int e = lo; e < hi; ++e) {
    const uint32_t key = s_keys[e];
    gt += key > T;
    eq += key == T;
  }
  int tg, te;
  const int gt_before = block_exclusive_scan(gt, s_scan, &tg);
  const int eq_before = block_exclusive_scan(eq, s_scan, &te);
  int out = gt_before + min(eq_before, k_eq);
  int eq_seen = eq_before;
  for (int e = lo; e < hi; ++e) {
    const uint32_t key = s_keys[e];
    if (key > T) {
      a.idx_s[out++] = e;
    } else if (key == T) {
      if (eq_seen < k_eq) a.idx_s[out++] = e;
      ++eq_seen;
    }
  }
  if (tid == 0) {
    *a.k_dev = a.k;
    atomicAdd(a.stats + 1, 1ull);
  }

  // Debug tap: concatenate the per-slab kept-row lists into idx_x.
  if (a.idx_x != nullptr) {
    __syncthreads();
    if (tid == 0) {
      int off = 0;
      for (int r = 0; r < a.R; ++r) {
        s_h[r] = (uint32_t)off;
        off += __ldcg(a.slab_cnt + r);
      }
      s_h[a.R] = (uint32_t)off;
      if (a.n_x) *a.n_x = off;
    }
    __syncthreads();
    for (int r = 0; r < a.R; ++r) {
      const int n = (int)(s_h[r + 1] - s_h[r]);
      for (int e = tid; e < n; e += NT)
        a.idx_x[s_h[r] + e] = __ldcg(a.slab_idx + (size_t)r * a.slab_rows + e);
    }
  }
}

}  // namespace

void choose_stage1_grid(int d, int F, int num_sms, int* C, int* R, int* gps) {
  const int G = d / kGroup;
  *C = (F / 16 + 31) / 32;
  const int target = 3 * num_sms;
  int best = 1;
  long best_err = -1;
  for (int r = 1; r <= G; ++r) {
    if (G % r || G / r > kMaxGroupsPerSlab) continue;
    long err = labs((long)(*C) * r - target);
    if (best_err < 0 || err < best_err) {
      best_err = err;
      best = r;
    }
  }
  *R = best;
  *gps = G / best;
}

size_t stage1_smem_bytes(int gps) {
  return (size_t)gps * 2048 + (size_t)S1_NW * 1024 * 4 + (size_t)gps * kGroup * 8 +
         (size_t)(gps + 1 + 33 + 1) * 4;
}

size_t select_smem_bytes(int F) { return (size_t)F * 4; }

cudaError_t setup_stage1_kernels() {
  cudaError_t e = cudaFuncSetAttribute(stage1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)stage1_smem_bytes(kMaxGroupsPerSlab));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)select_smem_bytes(kMaxDff));
}

cudaError_t launch_stage1(const prox_layer* L, const float* x, const Stage1Taps& taps,
                          cudaStream_t s, bool pdl) {
  Stage1Args a;
  a.x = x;
  a.pq = L->pq;
  a.ps = reinterpret_cast<const __half*>(L->ps);
  a.tau = L->tau;
  a.d = L->d;
  a.F = L->F;
  a.C = L->C;
  a.R = L->R;
  a.gps = L->gps;
  a.part = L->ws.part;
  a.scores = L->ws.scores;
  a.hist = L->ws.hist;
  a.slice_cnt = L->ws.slice_cnt;
  a.stats = L->ws.stats;
  a.g_dbg = taps.g;
  a.u_dbg = taps.u;
  a.slab_idx = taps.slabs ? L->ws.slab_idx : nullptr;
  a.slab_cnt = L->ws.slab_cnt;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L->C, L->R, 1);
  cfg.blockDim = dim3(S1_NT, 1, 1);
  cfg.dynamicSmemBytes = L->stage1_smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stage1_kernel, a);
}

cudaError_t launch_select(const prox_layer* L, const SelectTaps& taps, cudaStream_t s,
                          bool pdl) {
  SelectArgs a;
  a.scores = L->ws.scores;
  a.hist = L->ws.hist;
  a.F = L->F;
  a.k = L->k;
  a.idx_s = L->ws.idx_s;
  a.k_dev = L->ws.k_dev;
  a.stats = L->ws.stats;
  a.slab_idx = L->ws.slab_idx;
  a.slab_cnt = L->ws.slab_cnt;
  a.R = L->R;
  a.slab_rows = L->gps * kGroup;
  a.idx_x = taps.idx_x;
  a.n_x = taps.n_x;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(kSelectThreads, 1, 1);
  cfg.dynamicSmemBytes = L->select_smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel, a);
}

}  // namespace prox
