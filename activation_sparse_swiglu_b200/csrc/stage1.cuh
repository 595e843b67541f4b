// Stage 1 of the Prox decode step (Prox §4.1 "Stage 1: lightweight proxy
// construction"; §4.3 fused split-N proxy kernel), the first phase of the
// fused per-token kernel (token.cu).
//
// Work: the set of (column slice, kept input row) pairs.  A column slice is
// 512 bytes of an interleaved proxy row (16 blocks of 32 channels, each block
// 16 B of gate codes then 16 B of up codes), i.e. 512 channels of both
// proxies; the proxy is stored slice-major, so a slice's kept rows are read in
// ascending address order.  The C * d_model (slice, row) pairs, slice-major,
// are split into equal contiguous ranges, one per CTA (a static split: a CTA's
// range lies in at most two adjacent slices).  Each CTA thresholds the rows of
// its range (|x_i| >= tau) and compacts its kept rows in order, grouped into
// segments of one slice and one quantisation group, each segment padded to a
// multiple of 8 rows (a k-tile).
//
// The product runs on the integer tensor pipe, exactly.  Each kept x_i is
// written as a fixed-point integer V_i = x_i 2^(29 - E) (E the exponent of
// the CTA's largest kept |x|, so |V_i| < 2^30; exact for every x_i within a
// factor 128 of that maximum, rounded to an integer below it) and V_i as four
// signed 8-bit digits, V_i = sum_p v_ip 256^(3 - p).  A code c = q + 8 of the
// offset-binary INT4 format becomes the signed byte 16 q with one LOP3 (the
// nibble moved to the byte's top bits and its top bit flipped).  One
// mma.sync m16n8k32 (s8 x s8 -> s32) then takes 8 kept rows x 8 code words
// of one nibble parity: B holds the rows' bytes (k = 4 t + j is row t,
// nibble pair j of the word), A the digits laid out so that output row
// m = j + 4 p sees only the k with that j, times digit p.  The 32-bit integer
// sums are exact; per segment they are combined over the digits, converted
// to fp32, scaled by the fp16 group scale and added up in segment order.
// Rows padded onto a segment have zero digits and contribute exactly zero.
//
// The 16 warps form 4 groups; group q takes a quarter of the CTA's k-tiles
// and warp v of a group the blocks 4v .. 4v+3 (128 bytes) of each of their
// rows, streamed with 16-byte cp.async copies into the warp's own ring of
// k-tile slots (no synchronisation between warps; the chunks of a row are
// placed XOR-swizzled so the tensor-pipe operand reads are conflict-free),
// together with the fp16 scales of each new segment.  Each warp's sums per
// slice are combined over the 4 groups in shared memory, in group order, and
// written channel-major as tagged words.

// After the partials are written, every CTA takes an even share of the
// channels and, for each, adds the partials of the CTAs that hold its slice
// in CTA order (deterministic), scores it, score_j = |act(g~_j) u~_j| (act
// the layer's gate activation: SiLU, or GELU for a GeGLU FFN; the signed
// value is kept too when Stage 2 runs the A3 ablation), keeps its key in
// shared memory for the selection and, for the top-k rule, counts it in the
// histograms and buckets of select.cuh (score_channels).
#pragma once
#include "select.cuh"
#include "token_args.cuh"

namespace prox {
namespace s1 {

constexpr int NW = kStage1Warps;  // consumer warps: one 32-channel block each
static_assert(NW == 16, "a 512-byte slice is 16 blocks of 32 channels");
static_assert(kTokenThreads >= (NW + 1) * 32, "the producer warp");
constexpr int SLICE = 512;        // bytes (= channels of both proxies) per column slice
constexpr int PART = 1024;        // partial values per slice: (gate, up) per channel
constexpr int KT = 8;             // rows per k-tile
constexpr int NGRP = 4;           // warp groups: group q takes a quarter of the CTA's k-tiles
constexpr int WPG = NW / NGRP;    // warps per group: warp v of a group takes blocks BPW v ...
constexpr int BPW = 16 / WPG;     // blocks per warp
constexpr int WROW = BPW * 32;    // bytes of a row slice one warp streams
constexpr int WSLOT = KT * WROW + BPW * 128;  // a warp's ring slot: 8 rows, then 4 blocks' scales
constexpr int kMaxDepth = 8;      // k-tiles in flight per warp, at most
static_assert(WSLOT % 128 == 0, "slots keep 128-byte alignment");
static_assert(kOwnMax <= kTokenThreads, "scoring takes one channel per thread");

// D += A B on the integer tensor pipe (m16n8k32, s8 x s8 -> s32).
__device__ __forceinline__ void mma_s8(int* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// The high nibbles of a code word (bytes' bits 4..7, codes c = q + 8) as
// signed bytes 16 q: keep the top nibble of each byte and flip its top bit.
__device__ __forceinline__ uint32_t codes_hi_s8(uint32_t w) {
  uint32_t r;
  asm("lop3.b32 %0, %1, 0xF0F0F0F0, 0x80808080, 0x6A;" : "=r"(r) : "r"(w));  // (w & b) ^ c
  return r;
}
// The low nibbles the same way, after moving them up by 4 bits.
__device__ __forceinline__ uint32_t codes_lo_s8(uint32_t w) { return codes_hi_s8(w << 4); }
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(a), "r"(sel));
  return r;
}


// CTA holding pair t of T pairs split over P CTAs (CTA i holds
// [floor(T i / P), floor(T (i + 1) / P))); never an empty CTA.  T * P < 2^31
// (T <= 64 * 16384, P <= 1024).
__device__ __forceinline__ int cta_of(int t, int T, int P) {
  return (int)(((unsigned)(t + 1) * (unsigned)P + (unsigned)T - 1u) / (unsigned)T) - 1;
}

// Scores the channels [F c / P, F (c + 1) / P) of CTA c (at most kOwnMax):
// a group of threads per channel adds its gate and up partials over the CTAs
// whose pair ranges cover its slice (the group's threads take interleaved CTA
// subsets, then a fixed shuffle tree: deterministic), polling each tagged
// partial until this launch's has arrived.  Thread t then takes channel
// c0 + t: it writes the score, keeps its key (the score's bits) in shared
// memory and publishes the
// signed act(g~) u~ as a tagged word.  For the top-k rule the CTA first counts
// its keys in shared-memory histograms; one thread per non-empty fine bin then
// adds the CTA's count to the global bin, whose old value places the CTA's
// keys of that bin in the bin's bucket (tagged), and the coarse counts are
// added the same way, so a global bin sees one atomic per CTA, not one per
// channel.  Every thread of the CTA calls it.
__device__ void score_channels(const TokenArgs& a, bool histogram, SelectScratch& sel, uint32_t tag,
                               uint32_t* hist, uint32_t* chist) {
  const int P = gridDim.x, cta = blockIdx.x, tid = threadIdx.x;
  const int c0 = (int)(((long long)a.F * cta) / P);
  const int c1 = (int)(((long long)a.F * (cta + 1)) / P);
  const int T = a.C * a.d;
  uint32_t* fine = select_keys(sel);  // [kScoreBins]: the CTA's counts, then its bucket offsets
  if (histogram) {  // (ordered before the counting by the barrier after the partial sums)
    for (int i = tid; i < kCoarseBins; i += blockDim.x) sel.coarse[i] = 0u;
    for (int i = tid; i < kScoreBins; i += blockDim.x) fine[i] = 0u;
  }
  {
    // g~ and u~ of the CTA's channels: tpc threads per channel (a power of two
    // <= 32, as many as the CTA has threads for), thread `part` of a channel
    // adding the partials of the CTAs i_lo + part, i_lo + part + tpc, ... in
    // order, then the group's sums by a fixed shuffle tree (deterministic).
    // Each tagged partial is polled until it carries this launch's tag.
    const int nch = c1 - c0;
    int tpc = 32;
    while (tpc > 1 && tpc * nch > (int)blockDim.x) tpc >>= 1;
    const int cl = tid / tpc, part = tid % tpc;
    float g = 0.f, u = 0.f;
    if (cl < nch) {
      const int chl = c0 + cl;
      const int c = chl / SLICE, m = chl % SLICE;
      const int e = 2 * m;  // channel m's gate and up sums in a CTA's partial row
      const int i_lo = cta_of(c * a.d, T, P);
      const int i_hi = cta_of((c + 1) * a.d - 1, T, P);
      for (int i0 = i_lo + part; i0 <= i_hi; i0 += 8 * tpc) {
        ulonglong2 v[8];
        int off[8];  // element offset of CTA i0 + q tpc's partial pair, or -1
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int i = i0 + q * tpc;
          off[q] = -1;
          v[q] = make_ulonglong2(tag_word(0u, tag), tag_word(0u, tag));
          if (i <= i_hi) {
            const unsigned tlo = (unsigned)T * (unsigned)i / (unsigned)P;
            const unsigned thi = (unsigned)T * (unsigned)(i + 1) / (unsigned)P;
            if (thi > tlo) {  // CTA i holds pairs; slice c is its first or second
              off[q] = (i * 2 + (c - (int)(tlo / (unsigned)a.d))) * PART + e;
              v[q] = ld_tag2(a.part + off[q]);
            }
          }
        }
        const long long t0 = clock64();
        for (;;) {
          bool all = true;
#pragma unroll
          for (int q = 0; q < 8; ++q) all = all && tag_ok(v[q].x, tag) && tag_ok(v[q].y, tag);
          if (all || !wait_more(t0, a.err)) break;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (off[q] >= 0 && !(tag_ok(v[q].x, tag) && tag_ok(v[q].y, tag))) v[q] = ld_tag2(a.part + off[q]);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          g += __uint_as_float((uint32_t)v[q].x);
          u += __uint_as_float((uint32_t)v[q].y);
        }
      }
    }
    for (int o = tpc >> 1; o > 0; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      u += __shfl_xor_sync(0xffffffffu, u, o);
    }
    if (cl < nch && part == 0) {
      sel.sg[cl] = g;
      sel.su[cl] = u;
    }
    __syncthreads();
  }
  const int ch = c0 + tid;
  const bool mine = ch < c1;
  uint32_t key = 0u, fb = 0u, rank = 0u;
  if (mine) {
    const float g = sel.sg[tid], u = sel.su[tid];
    stamp(a.ts, 3);
    const float sv = act_f32(g, a.act) * u;
    const float sc = fabsf(sv);
    a.scores[ch] = sc;
    st_tag(a.st64 + ch, tag_word(__float_as_uint(sv), tag));
    if (a.s_tilde) a.s_tilde[ch] = sv;
    if (a.g_dbg) a.g_dbg[ch] = g;
    if (a.u_dbg) a.u_dbg[ch] = u;
    key = __float_as_uint(sc);
    sel.own[tid] = key;

    if (histogram) {
      fb = key >> kScoreShift;
      rank = atomicAdd(&fine[fb], 1u);
      atomicAdd(&sel.coarse[key >> kCoarseShift], 1u);
    }
  }
  if (!histogram) return;
  __syncthreads();
  if (mine && rank == 0u) fine[fb] = atomicAdd(hist + fb, fine[fb]);
  for (int i = tid; i < kCoarseBins; i += blockDim.x)
    if (sel.coarse[i]) atomicAdd(chist + i, sel.coarse[i]);
  __syncthreads();
  if (mine) {
    const uint32_t slot = fine[fb] + rank;
    if (slot < (uint32_t)kBucketCap)
      st_tag2(a.bucket + ((size_t)fb * kBucketCap + slot) * 2, tag_word(key, tag), tag_word((uint32_t)ch, tag));
  }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Waits until at most n of this thread's copy groups are pending (n < kMaxDepth).
__device__ __forceinline__ void cp_async_wait_n(int n) {
  switch (n) {
    case 7: cp_async_wait<7>(); break;
    case 6: cp_async_wait<6>(); break;
    case 5: cp_async_wait<5>(); break;
    case 4: cp_async_wait<4>(); break;
    case 3: cp_async_wait<3>(); break;
    case 2: cp_async_wait<2>(); break;
    case 1: cp_async_wait<1>(); break;
    default: cp_async_wait<0>(); break;
  }
}
static_assert(kMaxDepth <= 8, "cp_async_wait_n covers depths up to 8");

// Shared memory of Stage 1 (byte offsets from the start of the dynamic
// block): the warps' rings [NW][depth][WSLOT], the groups' sums per slice
// [2][NGRP][512][2] (float), then per padded row its byte offset in the
// proxy (-1 for padding) and its digit word (byte p = digit p; stored k-tile
// interleaved so rows t and t + 4 of a k-tile are adjacent), the segment
// code of each k-tile, each segment's kept rows, the warps' largest kept
// |x|, block-scan scratch and two words.  A segment is an aligned 128-pair
// chunk of the (slice, row) pair space: one slice and one quantisation group
// (d_model is a multiple of 128); its code is sl * G + group (sl = 0, 1 the
// CTA's first or second slice; G = d_model / 128).
struct Layout {
  size_t red, off, dig, ktseg, segn, wmax, scan, misc, total;
};
// Rows of a CTA after padding: each of its at most d/128 + 2 segments adds
// at most 7.
__host__ __device__ inline int padded_rows(int lmax, int d) {
  return (lmax + 14 * (d >> 7) + 14 + KT - 1) & ~(KT - 1);
}
__host__ __device__ inline Layout layout(int depth, int lmax, int d) {
  const int lp = padded_rows(lmax, d), nseg = (d >> 7) + 2;
  Layout L;
  size_t o = (size_t)NW * depth * WSLOT;
  L.red = o;
  o += 4 * (size_t)(2 * NGRP * PART);
  L.off = o;
  o += 4 * (size_t)lp;
  L.dig = o;
  o += 4 * (size_t)lp;
  L.ktseg = o;
  o += 4 * (size_t)(lp / KT);
  L.segn = o;
  o += 4 * (size_t)nseg;
  L.wmax = o;
  o += 4 * 32;
  L.scan = o;
  o += 4 * 33;
  L.misc = o;
  o += 4 * 4;
  L.total = o;
  return L;
}
// Where padded row `pos` keeps its digit word: rows t and t + 4 of a k-tile
// side by side.
__device__ __forceinline__ int dig_index(int pos) {
  return (pos & ~7) | ((pos & 3) << 1) | ((pos >> 2) & 1);
}
// The balanced base-256 digits of the integer nearest to v (|v| < 2^30):
// v = d0 256^3 + d1 256^2 + d2 256 + d3, each d in [-128, 127], byte p = d_p.
__device__ __forceinline__ uint32_t digits_of(float v) {
  int r = __float2int_rn(v);
  const int d3 = (int)((unsigned)r << 24) >> 24;
  r = (r - d3) >> 8;
  const int d2 = (int)((unsigned)r << 24) >> 24;
  r = (r - d2) >> 8;
  const int d1 = (int)((unsigned)r << 24) >> 24;
  const int d0 = (r - d1) >> 8;
  return ((uint32_t)d0 & 255u) | (((uint32_t)d1 & 255u) << 8) | (((uint32_t)d2 & 255u) << 16) |
         ((uint32_t)d3 << 24);
}

// Stage 1 of one token: the CTA's partial sums g~, u~ of the slices its pair
// range touches go to a.part as tagged words (the tag from the launch counter
// read at the kernel's start).  Every thread of the CTA calls it: warps
// 0..NW-1 stream and multiply, the rest take part in the prologue and the
// final combine.  Returns the launch index (launch_index(counter)).
__device__ unsigned long long run(const TokenArgs& a, unsigned char* smem, unsigned long long counter) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
  const int P = gridDim.x, cta = blockIdx.x;
  const int d = a.d, G = d >> 7, depth = a.s1_depth;
  const Layout Ly = layout(depth, a.lmax, d);
  float* s_red = reinterpret_cast<float*>(smem + Ly.red);
  int* s_off = reinterpret_cast<int*>(smem + Ly.off);
  uint32_t* s_dig = reinterpret_cast<uint32_t*>(smem + Ly.dig);
  int* s_ktseg = reinterpret_cast<int*>(smem + Ly.ktseg);
  int* s_segn = reinterpret_cast<int*>(smem + Ly.segn);
  unsigned* s_wmax = reinterpret_cast<unsigned*>(smem + Ly.wmax);
  unsigned* s_scan = reinterpret_cast<unsigned*>(smem + Ly.scan);
  unsigned* s_misc = reinterpret_cast<unsigned*>(smem + Ly.misc);  // [1] k-tiles

  // ---- this CTA's pairs: [tlo, thi) of the C * d (slice, row) pairs,
  // slice-major (pair t is slice t / d, row t mod d).  The split is static:
  // it does not depend on the token. ----
  const unsigned T = (unsigned)a.C * (unsigned)d;  // T * P < 2^31
  const unsigned tlo = T * (unsigned)cta / (unsigned)P, thi = T * (unsigned)(cta + 1) / (unsigned)P;
  const int span = (int)(thi - tlo);               // <= d, since C < P
  const int cA = (int)(tlo / (unsigned)d);
  const int nsl = span > 0 && (int)((thi - 1) / (unsigned)d) > cA ? 2 : 1;  // slices the range touches
  // its segments: the aligned 128-pair chunks [128 (s0 + ls), + 128) it meets
  const int s0 = (int)(tlo >> 7);
  const int nls = span > 0 ? (int)((thi - 1) >> 7) - s0 + 1 : 0;
  // Warp w takes the segments w, w + nwarps, ...; lane l the pairs 4l .. 4l+3
  // of one: x_row for the 4 rows in one load, kept = inside the range and
  // |x| >= tau, as a 4-bit mask.
  auto seg_mask = [&](int ls, float4& xv, int& slice, int& row0) {
    const unsigned base = (unsigned)(s0 + ls) << 7;
    slice = (int)(base / (unsigned)d);
    row0 = (int)(base - (unsigned)slice * (unsigned)d);
    xv = __ldg(reinterpret_cast<const float4*>(a.x + row0) + lane);
    const float v[4] = {xv.x, xv.y, xv.z, xv.w};
    unsigned m = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const unsigned gp = base + 4u * (unsigned)lane + (unsigned)k;
      if (gp >= tlo && gp < thi && fabsf(v[k]) >= a.tau) m |= 1u << k;
    }
    return m;
  };
  // pass 1: kept rows per segment, the largest kept |x|
  unsigned mx = 0;
  for (int ls = warp; ls < nls; ls += nwarps) {
    float4 xv;
    int slice, row0;
    const unsigned m = seg_mask(ls, xv, slice, row0);
    const float v[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (m & (1u << k)) mx = max(mx, __float_as_uint(fabsf(v[k])));
    const int n = __reduce_add_sync(0xffffffffu, (unsigned)__popc(m));
    if (lane == 0) s_segn[ls] = n;
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) s_wmax[warp] = mx;
  // each warp zeroes its own entries of the groups' sums (warp v of group q:
  // channels of blocks BPW v .. BPW v + 3, both slices, both proxies)
  if (warp < NW) {
    const int q = warp / WPG, v = warp % WPG;
#pragma unroll
    for (int i = 0; i < 2 * BPW * 32 * 2 / 32; ++i) {
      const int e = i * 32 + lane;  // (slice, channel of the warp's blocks, proxy)
      const int sl = e >> 8, m = BPW * 32 * v + ((e >> 1) & 127), pr = e & 1;
      s_red[(((size_t)sl * NGRP + q) * 512 + m) * 2 + pr] = 0.f;
    }
  }
  __syncthreads();
  // E: the exponent of the largest kept |x| (clamped so every power of two
  // below stays a normal float); V = x 2^(29 - E) has |V| < 2^30.
  unsigned mxb = 0;
  for (int w = 0; w < nwarps; ++w) mxb = max(mxb, s_wmax[w]);
  const int E = max((int)(mxb >> 23) - 127, -93);
  const float vscale = __int_as_float((127 + 29 - E) << 23);
  // pass 2: each kept row at its padded position (padded rows of the earlier
  // segments + its rank in its segment), with its row slice's offset and its
  // digits; the segment's padding rows (nothing to copy, zero digits) and
  // the segment code of its k-tiles
  for (int ls = warp; ls < nls; ls += nwarps) {
    int pb = 0;
    for (int i = lane; i < ls; i += 32) pb += (s_segn[i] + KT - 1) & ~(KT - 1);
    pb = (int)__reduce_add_sync(0xffffffffu, (unsigned)pb);
    float4 xv;
    int slice, row0;
    const unsigned m = seg_mask(ls, xv, slice, row0);
    const float v[4] = {xv.x, xv.y, xv.z, xv.w};
    int incl = __popc(m);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int pos = pb + incl - __popc(m);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (m & (1u << k)) {
        s_off[pos] = (slice * d + row0 + 4 * lane + k) * SLICE;
        s_dig[dig_index(pos)] = digits_of(v[k] * vscale);
        ++pos;
      }
    const int n = s_segn[ls], padded = (n + KT - 1) & ~(KT - 1);
    for (int i = n + lane; i < padded; i += 32) {
      s_off[pb + i] = -1;
      s_dig[dig_index(pb + i)] = 0u;
    }
    const int code = (slice - cA) * G + (row0 >> 7);
    for (int i = lane; i < padded / KT; i += 32) s_ktseg[pb / KT + i] = code;
    // realised input sparsity: the kept rows counted once, in slice 0
    if (lane == 0 && slice == 0 && n > 0) atomicAdd(a.stats, (unsigned long long)n);
  }
  if (warp == 0) {
    int tot = 0;
    for (int i = lane; i < nls; i += 32) tot += (s_segn[i] + KT - 1) & ~(KT - 1);
    tot = (int)__reduce_add_sync(0xffffffffu, (unsigned)tot);
    if (lane == 0) s_misc[1] = (unsigned)tot / KT;
  }
  if (cta == 0 && (a.idx_x || a.n_x)) {
    // test taps: the token's kept rows, ascending, and their number
    const int rpt = (d + (int)blockDim.x - 1) / (int)blockDim.x;
    const int q0 = min(tid * rpt, d), q1 = min(q0 + rpt, d);
    int c = 0;
    for (int row = q0; row < q1; ++row) c += fabsf(__ldg(a.x + row)) >= a.tau;
    int n_all;
    int pos = block_exclusive_scan(c, reinterpret_cast<int*>(s_scan), &n_all);
    for (int row = q0; row < q1; ++row)
      if (fabsf(__ldg(a.x + row)) >= a.tau && a.idx_x) a.idx_x[pos++] = row;
    if (tid == 0 && a.n_x) *a.n_x = n_all;
  }
  __syncthreads();
  stamp(a.ts, 8);
  const int nkt = (int)s_misc[1];
  const float fin = __int_as_float((127 + E - 33) << 23);  // 2^(E - 33): V, and q as 16 q

  if (warp < NW) {
    const int q = warp / WPG, v = warp % WPG;
    const int k0 = (int)((long long)nkt * q / NGRP), n = (int)((long long)nkt * (q + 1) / NGRP) - k0;
    unsigned char* wring = smem + (size_t)warp * depth * WSLOT;
    const int nblk = a.F >> 5;
    const uint32_t lastw = (uint32_t)(a.F - (a.C - 1) * SLICE);  // bytes of a row of the last slice
    // ---- copies of local k-tile i into slot i % depth: lane 8 r + c copies
    // chunk c of rows r and r + 4 (16 bytes at byte 128 v + 16 c of the row
    // slice) to position c ^ 2 (r mod 4) of the row; at a segment's first
    // k-tile, lane 8 b + c also copies chunk c of block b's scales. ----
    const int cc = lane & 7, cr = lane >> 3;
    const uint32_t wbyte = (uint32_t)(v * WROW + 16 * cc);
    auto issue = [&](int i) {
      if (i < n) {
        const int kt = k0 + i;
        unsigned char* slot = wring + (size_t)(i % depth) * WSLOT;
        const int s = s_ktseg[kt];
        const int sl = s >= G ? 1 : 0;
        const uint32_t width = cA + sl == a.C - 1 ? lastw : (uint32_t)SLICE;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = cr + 4 * h;
          const int off = s_off[kt * KT + r];
          if (off >= 0 && wbyte < width) cp_async16(slot + r * WROW + 16 * (cc ^ (2 * cr)), a.pq + off + wbyte);
        }
        if (i == 0 || s != s_ktseg[kt - 1]) {
          const int B = (cA + sl) * 16 + v * BPW + cr;
          if (B < nblk)
            cp_async16(slot + KT * WROW + cr * 128 + 16 * cc,
                       a.ps + ((size_t)(s - sl * G) * nblk + B) * 64 + 8 * cc);
        }
      }
      cp_async_commit();
    };
    // ---- operands: lane (g, t) = (lane / 4, lane mod 4) ----
    const int g = lane >> 2, t = lane & 3, j = g & 3, pg = g >> 2;
    // A fragment: byte j of each register holds digit pg (a0, a2) or pg + 2
    // (a1, a3) of row t (a0, a1) or t + 4 (a2, a3); the other bytes are 0
    const uint32_t sel0 = 0x4444u ^ ((uint32_t)(pg ^ 4) << (4 * j));
    const uint32_t sel1 = 0x4444u ^ ((uint32_t)((pg + 2) ^ 4) << (4 * j));
    // weights of the digits this lane's accumulator rows carry
    const float wA = pg ? 65536.f : 16777216.f, wB = pg ? 1.f : 256.f;
    // B fragment: word g of block b in rows t and t + 4 (swizzled chunk)
    auto boff = [&](int b) { return t * WROW + 16 * ((2 * b + (g >> 2)) ^ (2 * t)) + 4 * (g & 3); };
    // scales of a lane's sums (nibbles 2j, 2j + 1 of words 2t and 2t + 1) in
    // a slot's scale area: block b, proxy t / 2, channel 16 (t mod 2) + 2j
    const int soff = KT * WROW + 64 * (t >> 1) + 32 * (t & 1) + 4 * j;
    int dl[BPW][4], dh[BPW][4];
    uint32_t sc[BPW][2];
#pragma unroll
    for (int b = 0; b < BPW; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i) dl[b][i] = dh[b][i] = 0;
    // segment end: combine the digits' rows (lanes g and g ^ 4), scale and
    // add to the group's sums of the segment's slice, s_red[sl][q][m][proxy]
    // (lanes g < 4; lanes g >= 4 hold the same values)
    auto flush = [&](int sl) {
      float* red = s_red + ((size_t)sl * NGRP + q) * 512 * 2 + (t >> 1);
#pragma unroll
      for (int b = 0; b < BPW; ++b) {
        float l0 = fmaf((float)dl[b][0], wA, (float)dl[b][2] * wB);  // word 2t,     nibble 2j
        float l1 = fmaf((float)dl[b][1], wA, (float)dl[b][3] * wB);  // word 2t + 1, nibble 2j
        float h0 = fmaf((float)dh[b][0], wA, (float)dh[b][2] * wB);  // word 2t,     nibble 2j + 1
        float h1 = fmaf((float)dh[b][1], wA, (float)dh[b][3] * wB);  // word 2t + 1, nibble 2j + 1
        l0 += __shfl_xor_sync(0xffffffffu, l0, 16);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 16);
        h0 += __shfl_xor_sync(0xffffffffu, h0, 16);
        h1 += __shfl_xor_sync(0xffffffffu, h1, 16);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&sc[b][0]));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&sc[b][1]));
        if (g < 4) {
          // channel of (word 2t + k / 2, nibble 2j + k mod 2) in the slice
          const int m0 = 32 * (BPW * v + b) + 16 * (t & 1) + 2 * j;
          red[2 * m0] = fmaf(f0.x, l0, red[2 * m0]);
          red[2 * (m0 + 1)] = fmaf(f0.y, h0, red[2 * (m0 + 1)]);
          red[2 * (m0 + 8)] = fmaf(f1.x, l1, red[2 * (m0 + 8)]);
          red[2 * (m0 + 9)] = fmaf(f1.y, h1, red[2 * (m0 + 9)]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) dl[b][i] = dh[b][i] = 0;
      }
    };
    int cur = -1;
    for (int i = 0; i < depth - 1; ++i) issue(i);
    for (int i = 0; i < n; ++i) {
      issue(i + depth - 1);
      cp_async_wait_n(depth - 1);  // this lane's copies of k-tile i have landed
      __syncwarp();                // and every lane's
      const int kt = k0 + i;
      const unsigned char* slot = wring + (size_t)(i % depth) * WSLOT;
      const int s = s_ktseg[kt];
      if (s != cur) {
        if (cur >= 0) flush(cur >= G ? 1 : 0);
        cur = s;
#pragma unroll
        for (int b = 0; b < BPW; ++b) {
          sc[b][0] = *reinterpret_cast<const uint32_t*>(slot + soff + 128 * b);
          sc[b][1] = *reinterpret_cast<const uint32_t*>(slot + soff + 128 * b + 16);
        }
      }
      const uint2 dg = *reinterpret_cast<const uint2*>(s_dig + kt * KT + 2 * t);
      const uint32_t a0 = prmt(dg.x, sel0), a1 = prmt(dg.x, sel1);
      const uint32_t a2 = prmt(dg.y, sel0), a3 = prmt(dg.y, sel1);
#pragma unroll
      for (int b = 0; b < BPW; ++b) {
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(slot + boff(b));
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(slot + boff(b) + 4 * WROW);
        mma_s8(dl[b], a0, a1, a2, a3, codes_lo_s8(w0), codes_lo_s8(w1));
        mma_s8(dh[b], a0, a1, a2, a3, codes_hi_s8(w0), codes_hi_s8(w1));
      }
      __syncwarp();  // every lane's reads of the slot come before its refill
    }
    cp_async_wait<0>();
    if (cur >= 0) flush(cur >= G ? 1 : 0);
  }
  __syncthreads();
  stamp(a.ts, 9);
  // ---- the CTA's partials: the groups' sums in group order, channel-major
  // (channel m's gate and up sums at 2m, 2m + 1) ----
  const unsigned long long index = launch_index(counter);
  const uint32_t tag = launch_tag(index);
  for (int e = tid; e < nsl * 512; e += blockDim.x) {
    const int sl = e >> 9, m = e & 511;
    float gs = 0.f, us = 0.f;
#pragma unroll
    for (int qq = 0; qq < NGRP; ++qq) {
      const float2 v2 = *reinterpret_cast<const float2*>(s_red + (((size_t)sl * NGRP + qq) * 512 + m) * 2);
      gs += v2.x;
      us += v2.y;
    }
    st_tag2(a.part + ((size_t)cta * 2 + sl) * PART + 2 * m, tag_word(__float_as_uint(gs * fin), tag),
            tag_word(__float_as_uint(us * fin), tag));
  }
  return index;
}

}  // namespace s1
}  // namespace prox
