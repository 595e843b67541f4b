// Stage 1 of the Prox decode step (Prox §4.1 "Stage 1: lightweight proxy
// construction"; §4.3 fused split-N proxy kernel), the first phase of the
// fused per-token kernel (token.cu).
//
// Work: the set of (column slice, kept input row) pairs.  A column slice is
// 512 bytes of an interleaved proxy row (16 blocks of 32 channels, each block
// 16 B of gate codes then 16 B of up codes), i.e. 512 channels of both
// proxies.  Every CTA thresholds all of x (|x_i| >= tau) and compacts the kept
// rows in ascending order; the C * n_x pairs, slice-major, are then split into
// equal contiguous ranges, one per CTA and, inside it, one per warp, so every
// warp streams the same number of 512-byte row slices whatever the mask looks
// like.  A CTA's range lies in at most two adjacent slices.
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
// runs the A3 ablation), and -- for the top-k rule -- counts it in an
// 8192-bin histogram of the score's top bits, the first level of the radix
// select (score_channels).
#pragma once
#include "token_args.cuh"

namespace prox {
namespace s1 {

constexpr int NW = kStage1Warps;   // warps that stream rows
constexpr int NT = NW * 32;
static_assert(kMaxDModel % NT == 0, "rows per thread");
constexpr int SLICE = 512;   // bytes (= channels of both proxies) per column slice
constexpr int PART = 1024;   // partial values per slice: 32 chunks x 32 channels
constexpr int U = 4;         // rows per batch
constexpr int BATCH = U * SLICE;

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

// Scores the channels [F c / P, F (c + 1) / P) of CTA c once every CTA's
// partials are visible: thread t < the CTA's channel count takes one channel
// and adds its gate and up partials over the CTAs holding its slice, in CTA
// order.  n_x == 0: every score is 0.  Every thread of the CTA calls it.
__device__ void score_channels(const TokenArgs& a, int n_x, bool histogram) {
  const int P = gridDim.x, cta = blockIdx.x;
  const int c0 = (int)(((long long)a.F * cta) / P);
  const int c1 = (int)(((long long)a.F * (cta + 1)) / P);
  for (int ch = c0 + (int)threadIdx.x; ch < c1; ch += blockDim.x) {
    const int c = ch / SLICE, m = ch % SLICE;
    // channel m of the slice is block blk = m / 32, channel j = m % 32 of it:
    // its gate and up sums are the partial elements j*32 + 2*blk and + 1
    const int e = (m & 31) * 32 + 2 * (m >> 5);
    float g = 0.f, u = 0.f;
    if (n_x > 0) {
      const int T = a.C * n_x;
      const int i_lo = cta_of(c * n_x, T, P);
      const int i_hi = cta_of((c + 1) * n_x - 1, T, P);
      for (int i0 = i_lo; i0 <= i_hi; i0 += 8) {
        float2 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int i = i0 + q;
          v[q] = make_float2(0.f, 0.f);
          if (i <= i_hi) {
            const unsigned tlo = (unsigned)T * (unsigned)i / (unsigned)P;
            const unsigned thi = (unsigned)T * (unsigned)(i + 1) / (unsigned)P;
            if (thi > tlo) {  // CTA i holds pairs; slice c is its first or second
              const int off = (i * 2 + (c - (int)(tlo / (unsigned)n_x))) * PART;
              v[q] = __ldcg(reinterpret_cast<const float2*>(a.part + off + e));
            }
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          g += v[q].x;
          u += v[q].y;
        }
      }
    }
    const float sv = act_f32(g, a.act) * u;
    const float sc = fabsf(sv);
    a.scores[ch] = sc;
    if (a.s_tilde) a.s_tilde[ch] = sv;
    if (a.g_dbg) a.g_dbg[ch] = g;
    if (a.u_dbg) a.u_dbg[ch] = u;
    if (histogram) atomicAdd(a.hist + (__float_as_uint(sc) >> kScoreShift), 1u);
  }
}

// Shared memory: per-warp rings of NB batches, per-warp group-scaled sums,
// the CTA's kept rows, the stash of the warp that crosses a slice boundary.
template <int NB>
constexpr size_t smem_bytes(int lmax) {
  return (size_t)NW * NB * BATCH + (size_t)NW * PART * 4 + (size_t)lmax * 12 +
         (size_t)PART * 4 + (37 + kTokenThreads) * 4;
}

// The row loop of Stage 1: the CTA's partial sums of the slices it touches
// go to a.part.  Returns n_x (the kept rows of the token).  Every thread of
// the CTA calls it; warps NW and above take no rows.
template <int NB>
__device__ int run(const TokenArgs& a, unsigned char* smem) {
  constexpr int RING = NB * BATCH;  // ring bytes per warp
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = gridDim.x, cta = blockIdx.x;
  const int n16 = a.F >> 4, nblk = a.F >> 5;
  const Magic mg = a.mg;

  unsigned char* ring = smem;                                        // [NW][RING]
  float* s_tot = reinterpret_cast<float*>(smem + NW * RING);         // [NW][PART]
  int2* s_rx = reinterpret_cast<int2*>(s_tot + NW * PART);           // [lmax] (offset, x)
  int* s_key = reinterpret_cast<int*>(s_rx + a.lmax);                // [lmax] segment key
  float* s_stash = reinterpret_cast<float*>(s_key + a.lmax);         // [PART]
  int* s_scan = reinterpret_cast<int*>(s_stash + PART);              // [33]
  int* s_m = s_scan + 33;                                            // [4]
  int* s_src = s_m + 4;                                              // [kTokenThreads]

  // ---- kept rows of x, ascending: thread t < NT owns rows [t*rpt, (t+1)*rpt) ----
  const int rpt = (a.d + NT - 1) / NT;
  const int r0 = tid < NT ? tid * rpt : a.d;
  const int r1 = min(r0 + rpt, a.d);
  const bool vec = (rpt & 3) == 0;  // rows r0.. are 16-byte aligned
  auto x_at = [&](int row) -> float4 {  // rows row..row+3 (those < r1)
    if (vec) return __ldg(reinterpret_cast<const float4*>(a.x + row));
    float4 v;
    v.x = __ldg(a.x + row);
    v.y = row + 1 < r1 ? __ldg(a.x + row + 1) : 0.f;
    v.z = row + 2 < r1 ? __ldg(a.x + row + 2) : 0.f;
    v.w = row + 3 < r1 ? __ldg(a.x + row + 3) : 0.f;
    return v;
  };
  int cnt = 0;
  for (int row = r0; row < r1; row += 4) {
    const float4 v = x_at(row);
    cnt += (fabsf(v.x) >= a.tau) + (row + 1 < r1 && fabsf(v.y) >= a.tau) +
           (row + 2 < r1 && fabsf(v.z) >= a.tau) + (row + 3 < r1 && fabsf(v.w) >= a.tau);
  }
  int n_x;
  int pos = block_exclusive_scan(cnt, s_scan, &n_x);
  if (n_x == 0) {
    // nothing kept: g~ = u~ = 0 everywhere (score_channels needs no partials)
    if (cta == 0 && tid == 0) {
      if (a.n_x) *a.n_x = 0;
    }
    return 0;
  }
  const unsigned T = (unsigned)a.C * (unsigned)n_x;   // T * P < 2^31
  const unsigned tlo = T * (unsigned)cta / (unsigned)P, thi = T * (unsigned)(cta + 1) / (unsigned)P;
  const int len = (int)(thi - tlo);      // <= n_x, since C < P
  const int cA = (int)(tlo / (unsigned)n_x), pA = (int)(tlo % (unsigned)n_x);
  const int l_split = n_x - pA;          // local rows l >= l_split lie in slice cA + 1
  // local row l of this CTA is compacted position (pA + l) mod n_x
  for (int row0 = r0; row0 < r1; row0 += 4) {
    const float4 v4 = x_at(row0);
    const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int row = row0 + q;
      if (row < r1 && fabsf(vv[q]) >= a.tau) {
        int l = pos - pA;
        if (l < 0) l += n_x;
        if (l < len) {
          // the row slice's byte offset in the proxy, and its segment key
          // (slice, quantisation group), nondecreasing over the CTA's rows
          const int sl = l >= l_split ? 1 : 0;
          s_rx[l] = make_int2(row * a.F + (cA + sl) * SLICE, __float_as_int(vv[q]));
          s_key[l] = sl * 128 + (row >> 7);
        }
        if (cta == 0 && a.idx_x) a.idx_x[pos] = row;
        ++pos;
      }
    }
  }
  if (cta == 0 && tid == 0) {
    atomicAdd(a.stats, (unsigned long long)n_x);
    if (a.n_x) *a.n_x = n_x;
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
    float* wtot = s_tot + warp * PART + lane;  // element j*32 + lane: channel j of the chunk
#pragma unroll
    for (int j = 0; j < 32; ++j) wtot[j * 32] = 0.f;
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
          wtot[(2 * h) * 32] = fmaf(s2.x, acc[h].x, wtot[(2 * h) * 32]);
          wtot[(2 * h + 1) * 32] = fmaf(s2.y, acc[h].y, wtot[(2 * h + 1) * 32]);
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
                s_stash[j2 * 32 + lane] = wtot[j2 * 32];
                wtot[j2 * 32] = 0.f;
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
  const int nsl = len > l_split ? 2 : 1;
  for (int e = tid; e < PART; e += blockDim.x) {
    float p0 = 0.f, p1 = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const int kind = s_src[w];
      const float v = s_tot[w * PART + e];
      if (kind == 1) p0 += v;
      if (kind == 2) p1 += v;
      if (kind == 3) {
        p0 += s_stash[e];
        p1 += v;
      }
    }
    a.part[((size_t)cta * 2) * PART + e] = p0;
    if (nsl == 2) a.part[((size_t)cta * 2 + 1) * PART + e] = p1;
  }
  return n_x;
}

}  // namespace s1
}  // namespace prox
