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
// range lies in at most two adjacent slices); each CTA thresholds the rows of
// its range (|x_i| >= tau), compacts its kept pairs in order and splits them
// into equal contiguous ranges, one per warp, so every warp streams the same
// number of 512-byte row slices whatever the mask looks like.
//
// A warp streams its rows through a shared-memory ring with asynchronous
// 16-byte copies (cp.async, L2 only; each lane copies and later reads back its
// own chunk, so no barrier is needed), NB batches of four rows in flight, and
// dequantises the INT4 codes in registers with fp32 (packed f32x2)
// arithmetic, accumulating per quantisation group and scaling once per group
// by the fp16 group scale.  A batch whose rows share one slice and one group
// takes a path without any boundary checks.
//
// The warps' partial sums are combined in warp order into one partial vector
// per touched slice and written to global memory (run).  After a grid
// barrier, every CTA takes an even share of the channels and, for each, adds
// the partials of the CTAs that hold its slice in CTA order (deterministic),
// scores it, score_j = |act(g~_j) u~_j| (act the layer's gate activation:
// SiLU, or GELU for a GeGLU FFN; the signed value is kept too when Stage 2
// runs the A3 ablation), keeps its key in shared memory for the selection
// and, for the top-k rule, counts it in the histograms and buckets of
// select.cuh (score_channels).
#pragma once
#include "select.cuh"
#include "token_args.cuh"

namespace prox {
namespace s1 {

constexpr int NW = kStage1Warps;   // warps that stream rows
constexpr int NT = NW * 32;
static_assert(kMaxDModel % NT == 0, "rows per thread");
constexpr int SLICE = 512;   // bytes (= channels of both proxies) per column slice
constexpr int PART = 1024;   // partial values per slice: 32 chunks x 32 channels
constexpr int PARTP = 32 * 33;  // the same in shared memory, rows of 32 padded to 33
constexpr int U = 4;         // rows per batch
constexpr int BATCH = U * SLICE;
static_assert(kOwnMax <= kTokenThreads, "scoring takes one channel per thread");

// (w & M) | e in one instruction; e is a register (the exponents come from
// kernel parameters, so they are not folded into a second immediate).
template <uint32_t M>
__device__ __forceinline__ float andor(uint32_t w, uint32_t e) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "n"(M), "r"(e));
  return __uint_as_float(r);
}

// Eight INT4 codes of one 32-bit word (nibble p is channel 8w+p of the lane's
// chunk, stored as q+8) into four float2 accumulators.  Each nibble is OR-ed
// into the mantissa of a float whose exponent makes the nibble's lowest bit
// worth exactly 1, so subtracting (2^e + 8) leaves q exactly; nibbles 5..7
// are first shifted down by 12 bits.  This is the exponent-field construction
// of an integer as a float (the "magic number" conversion, e.g. Hacker's
// Delight, 2nd ed., §17-2, applied per nibble), with the offset of the
// codes folded into the subtracted constant.
__device__ __forceinline__ void acc_word(float2* a, uint32_t w, float2 x2, const Magic& mg) {
  const uint32_t h = w >> 12;
  const float2 v0 = __fadd2_rn(make_float2(andor<0x0000000Fu>(w, mg.e23), andor<0x000000F0u>(w, mg.e19)),
                               make_float2(-8388616.0f, -524296.0f));
  const float2 v1 = __fadd2_rn(make_float2(andor<0x00000F00u>(w, mg.e15), andor<0x0000F000u>(w, mg.e11)),
                               make_float2(-32776.0f, -2056.0f));
  const float2 v2 = __fadd2_rn(make_float2(andor<0x000F0000u>(w, mg.e7), andor<0x00000F00u>(h, mg.e15)),
                               make_float2(-136.0f, -32776.0f));
  const float2 v3 = __fadd2_rn(make_float2(andor<0x0000F000u>(h, mg.e11), andor<0x000F0000u>(h, mg.e7)),
                               make_float2(-2056.0f, -136.0f));
  a[0] = __ffma2_rn(v0, x2, a[0]);
  a[1] = __ffma2_rn(v1, x2, a[1]);
  a[2] = __ffma2_rn(v2, x2, a[2]);
  a[3] = __ffma2_rn(v3, x2, a[3]);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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
  if (histogram) {
    for (int i = tid; i < kCoarseBins; i += blockDim.x) sel.coarse[i] = 0u;
    for (int i = tid; i < kScoreBins; i += blockDim.x) fine[i] = 0u;
    __syncthreads();
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

// Shared memory: per-warp rings of NB batches, per-warp group-scaled sums,
// the CTA's kept rows, the stash of the warp that crosses a slice boundary.
template <int NB>
constexpr size_t smem_bytes(int lmax) {
  return (size_t)NW * NB * BATCH + (size_t)NW * PARTP * 4 + (size_t)lmax * 12 +
         (size_t)PARTP * 4 + (37 + kTokenThreads) * 4;
}

// The row loop of Stage 1: the CTA's partial sums of the slices its pair
// range touches go to a.part as tagged words (the tag from the launch
// counter read at the kernel's start).  Every thread of the CTA calls it;
// warps NW and above take no rows.
template <int NB>
__device__ void run(const TokenArgs& a, unsigned char* smem, unsigned long long counter) {
  constexpr int RING = NB * BATCH;  // ring bytes per warp
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = gridDim.x, cta = blockIdx.x;
  const int n16 = a.F >> 4, nblk = a.F >> 5;
  const Magic mg = a.mg;

  unsigned char* ring = smem;                                        // [NW][RING]
  float* s_tot = reinterpret_cast<float*>(smem + NW * RING);         // [NW][PARTP]
  int2* s_rx = reinterpret_cast<int2*>(s_tot + NW * PARTP);          // [lmax] (offset, x)
  int* s_key = reinterpret_cast<int*>(s_rx + a.lmax);                // [lmax] segment key
  float* s_stash = reinterpret_cast<float*>(s_key + a.lmax);         // [PARTP]
  int* s_scan = reinterpret_cast<int*>(s_stash + PARTP);             // [33]
  int* s_m = s_scan + 33;                                            // [4]
  int* s_src = s_m + 4;                                              // [kTokenThreads]

  // ---- this CTA's pairs: [tlo, thi) of the C * d (slice, row) pairs,
  // slice-major; pair p of the range is slice cA + (rA + p >= d), row
  // (rA + p) mod d.  The split is static: it does not depend on the token. ----
  const int d = a.d;
  const unsigned T = (unsigned)a.C * (unsigned)d;  // T * P < 2^31
  const unsigned tlo = T * (unsigned)cta / (unsigned)P, thi = T * (unsigned)(cta + 1) / (unsigned)P;
  const int span = (int)(thi - tlo);               // <= d, since C < P
  const int cA = (int)(tlo / (unsigned)d), rA = (int)(tlo % (unsigned)d);
  const int first = min(span, d - rA);             // pairs of the range in slice cA
  // ---- its kept pairs (|x_row| >= tau), in pair order: thread t owns pairs
  // [t*per, (t+1)*per); the two slices' counts are packed in one word ----
  const int per = (span + (int)blockDim.x - 1) / (int)blockDim.x;
  const int p0 = min(tid * per, span), p1 = min(p0 + per, span);
  float xv[4];
  unsigned cnt = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // the first four pairs (all of them while span <= 4 * blockDim.x)
    const int p = p0 + q;
    xv[q] = 0.f;
    if (p < p1) {
      const int row = rA + p < d ? rA + p : rA + p - d;
      xv[q] = __ldg(a.x + row);
      if (fabsf(xv[q]) >= a.tau) cnt += p < first ? 1u : 0x10000u;
    }
  }
  for (int p = p0 + 4; p < p1; ++p) {  // longer ranges (d > 4 * blockDim.x)
    const int row = rA + p < d ? rA + p : rA + p - d;
    if (fabsf(__ldg(a.x + row)) >= a.tau) cnt += p < first ? 1u : 0x10000u;
  }
  unsigned tot;
  const unsigned pre = block_exclusive_scan(cnt, reinterpret_cast<unsigned*>(s_scan), &tot);
  const int l_split = (int)(tot & 0xFFFFu);        // kept pairs in slice cA
  const int len = l_split + (int)(tot >> 16);      // kept pairs of the CTA
  {
    int l0 = (int)(pre & 0xFFFFu), l1 = l_split + (int)(pre >> 16);
    // the row slice's byte offset in the proxy, and its segment key (slice,
    // quantisation group), nondecreasing over the CTA's rows
    auto place = [&](int p, float v) {
      if (fabsf(v) >= a.tau) {
        const int row = rA + p < d ? rA + p : rA + p - d;
        const int sl = p < first ? 0 : 1;
        const int l = sl ? l1++ : l0++;
        s_rx[l] = make_int2(((cA + sl) * d + row) * SLICE, __float_as_int(v));
        s_key[l] = sl * 128 + (row >> 7);
      }
    };
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (p0 + q < p1) place(p0 + q, xv[q]);
    for (int p = p0 + 4; p < p1; ++p) place(p, __ldg(a.x + (rA + p < d ? rA + p : rA + p - d)));
  }
  // realised input sparsity: the kept rows counted once, in slice 0
  if (tid == 0 && cA == 0 && l_split > 0) atomicAdd(a.stats, (unsigned long long)l_split);
  if (cta == 0 && (a.idx_x || a.n_x)) {
    // test taps: the token's kept rows, ascending, and their number
    const int rpt = (d + (int)blockDim.x - 1) / (int)blockDim.x;
    const int q0 = min(tid * rpt, d), q1 = min(q0 + rpt, d);
    int c = 0;
    for (int row = q0; row < q1; ++row) c += fabsf(__ldg(a.x + row)) >= a.tau;
    int n_all;
    int pos = block_exclusive_scan(c, s_scan, &n_all);
    for (int row = q0; row < q1; ++row)
      if (fabsf(__ldg(a.x + row)) >= a.tau && a.idx_x) a.idx_x[pos++] = row;
    if (tid == 0 && a.n_x) *a.n_x = n_all;
  }
  __syncthreads();
  stamp(a.ts, 8);

  if (warp < NW) {
    // ---- this warp's local rows [wl0, wl1) ----
    const int wl0 = (int)((long long)len * warp / NW);
    const int wl1 = (int)((long long)len * (warp + 1) / NW);
    const int nbw = (wl1 - wl0 + U - 1) / U;
    unsigned char* wring = ring + warp * RING + lane * 16;
    const uint8_t* pq_lane = a.pq + lane * 16;
    float* wtot = s_tot + warp * PARTP + lane;  // element j*32 + lane (at j*33 + lane): channel j of the chunk
#pragma unroll
    for (int j = 0; j < 32; ++j) wtot[j * 33] = 0.f;
    // Only the last slice can be narrower than 512 bytes; a warp with rows there
    // checks each lane's chunk before copying it.
    const bool checked = (a.F % SLICE) != 0 && wl1 > wl0 &&
                         cA + (wl1 - 1 >= l_split ? 1 : 0) == a.C - 1;
    auto issue = [&](int j) {
      if (j < nbw) {
        unsigned char* dst = wring + (j % NB) * BATCH;
        const int l0 = wl0 + j * U;
        if (!checked && l0 + U <= wl1) {
#pragma unroll
          for (int u = 0; u < U; ++u)
            cp_async16(dst + u * SLICE, pq_lane + (uint32_t)s_rx[l0 + u].x);
        } else {
          for (int u = 0; u < U && l0 + u < wl1; ++u) {
            const int l = l0 + u;
            const int c16 = (cA + (l >= l_split ? 1 : 0)) * 32 + lane;
            if (c16 < n16) cp_async16(dst + u * SLICE, pq_lane + (uint32_t)s_rx[l].x);
          }
        }
      }
      cp_async_commit();
    };
    float2 acc[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) acc[h] = make_float2(0.f, 0.f);
    uint4 sc[4];            // fp16 scales of the current (slice, group) for this lane's chunk
    int cur_key = -1, cur_g = -1;
    float okf = 0.f;        // 1 when this lane's chunk exists in the current slice
    // group end: tot += scale * acc (tot in shared memory), acc = 0
    auto flush = [&]() {
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        const uint32_t sw[4] = {sc[qd].x, sc[qd].y, sc[qd].z, sc[qd].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int h = qd * 4 + m;
          const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&sw[m]));
          wtot[(2 * h) * 33] = fmaf(s2.x, acc[h].x, wtot[(2 * h) * 33]);
          wtot[(2 * h + 1) * 33] = fmaf(s2.y, acc[h].y, wtot[(2 * h + 1) * 33]);
          acc[h] = make_float2(0.f, 0.f);
        }
      }
    };
    auto row_fma = [&](const unsigned char* src, float xv) {
      const uint4 v = *reinterpret_cast<const uint4*>(src);
      const float2 x2 = make_float2(xv * okf, xv * okf);
      acc_word(acc + 0, v.x, x2, mg);
      acc_word(acc + 4, v.y, x2, mg);
      acc_word(acc + 8, v.z, x2, mg);
      acc_word(acc + 12, v.w, x2, mg);
    };
#pragma unroll
    for (int j = 0; j < NB - 1; ++j) issue(j);
    for (int j = 0; j < nbw; ++j) {
      issue(j + NB - 1);
      cp_async_wait<NB - 1>();  // this lane's copies of batch j have landed
      const unsigned char* src = wring + (j % NB) * BATCH;
      const int first = wl0 + j * U;
      const int last = min(first + U, wl1);
      if (last - first == U && s_key[first] == cur_key && s_key[last - 1] == cur_key) {
        // one segment: no boundary checks
#pragma unroll
        for (int u = 0; u < U; ++u)
          row_fma(src + u * SLICE, __int_as_float(s_rx[first + u].y));
      } else {
        for (int l = first; l < last; ++l) {
          const int key = s_key[l];
          if (key != cur_key) {
            if (cur_g >= 0) flush();
            if (cur_key >= 0 && (key >> 7) != (cur_key >> 7)) {
              // the warp crosses into the next slice: park the first slice's sums
#pragma unroll
              for (int j2 = 0; j2 < 32; ++j2) {
                s_stash[j2 * 33 + lane] = wtot[j2 * 33];
                wtot[j2 * 33] = 0.f;
              }
            }
            cur_key = key;
            cur_g = key & 127;
            const int c16 = (cA + (key >> 7)) * 32 + lane;
            okf = c16 < n16 ? 1.f : 0.f;
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) sc[qd] = make_uint4(0u, 0u, 0u, 0u);
            if (c16 < n16) {
              const uint4* sp = reinterpret_cast<const uint4*>(
                  a.ps + ((size_t)cur_g * nblk + (c16 >> 1)) * 64 + (c16 & 1) * 32);
#pragma unroll
              for (int qd = 0; qd < 4; ++qd) sc[qd] = __ldg(sp + qd);
            }
          }
          row_fma(src + (l - first) * SLICE, __int_as_float(s_rx[l].y));
        }
      }
    }
    cp_async_wait<0>();
    if (cur_g >= 0) flush();
  }
  __syncthreads();
  stamp(a.ts, 9);

  // ---- the CTA's partials per touched slice (warp order), then report ----
  // warp w's share: bit 0 -> its sums belong to the CTA's first slice, bit 1 ->
  // to the second, both -> it crossed (first-slice sums in the stash)
  if (tid < NW) {
    const int l0 = (int)((long long)len * tid / NW), l1 = (int)((long long)len * (tid + 1) / NW);
    s_src[tid] = l1 <= l0 ? 0 : (l1 <= l_split ? 1 : (l0 >= l_split ? 2 : 3));
  }
  __syncthreads();
  const int nsl = span > first ? 2 : 1;  // slices the CTA's pair range touches
  const uint32_t tag = launch_tag(counter);  // (the counter was loaded at the kernel's start)
  // Element e = j*32 + 2*blk + h of the sums is the gate (h = 0) or up
  // (h = 1) sum of channel m = blk*32 + j of the slice; channel m's pair is
  // stored at 2m, 2m + 1, so the scoring threads (one per channel,
  // consecutive channels) read consecutive 16-byte pairs.  One thread per
  // channel, one 16-byte store per touched slice: each warp's stores cover
  // whole sectors.
  for (int m = tid; m < PART / 2; m += blockDim.x) {
    const int ep = (m & 31) * 33 + 2 * (m >> 5);  // the gate sum in the padded layout; up at + 1
    float g0 = 0.f, u0 = 0.f, g1 = 0.f, u1 = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const int kind = s_src[w];
      const float vg = s_tot[w * PARTP + ep], vu = s_tot[w * PARTP + ep + 1];
      if (kind == 1) {
        g0 += vg;
        u0 += vu;
      }
      if (kind == 2) {
        g1 += vg;
        u1 += vu;
      }
      if (kind == 3) {
        g0 += s_stash[ep];
        u0 += s_stash[ep + 1];
        g1 += vg;
        u1 += vu;
      }
    }
    st_tag2(a.part + ((size_t)cta * 2) * PART + 2 * m, tag_word(__float_as_uint(g0), tag),
            tag_word(__float_as_uint(u0), tag));
    if (nsl == 2)
      st_tag2(a.part + ((size_t)cta * 2 + 1) * PART + 2 * m, tag_word(__float_as_uint(g1), tag),
              tag_word(__float_as_uint(u1), tag));
  }
}

}  // namespace s1
}  // namespace prox
