// Per-token top-k channel select (Prox App. A.6 "Per-token top-k
// selection"): the k channels of largest proxy score |s~_j|, ties going to the
// lower channel index.
//
// While scoring, every CTA of the per-token kernel counts its channels' keys
// (the fp32 bit patterns of the scores, which order like the values) in two
// global histograms, a fine one over bits 30..18 (8192 bins) and a coarse one
// over bits 30..24 (128 bins, each the sum of 64 fine bins), adding per bin
// the counts it first gathered in shared memory; the fine bin's old count
// places the CTA's (key, channel) pairs of that bin in the bin's bucket.
// Every CTA then finds the exact cut itself, reading only small pieces:
//   1. the coarse histogram (512 bytes), once complete: the coarse bin
//      holding the k-th largest key;
//   2. that coarse bin's 64 fine bins: the fine bin b1 holding it and the
//      rank wanted inside b1;
//   3. b1's bucket: the candidates, ranked by (key descending, index
//      ascending), which gives the k-th largest key T and the tie cut:
//      channel j is selected iff key_j > T, or key_j == T and j <= tie cut.
// When b1 holds more keys than its bucket (many equal scores) the CTA loads
// every score and runs a radix select over them instead: a most-significant-
// digit-first select, 4 bits per level, with per-thread digit counts packed
// four to a 64-bit word (16 bits each) and summed over the CTA.
#pragma once
#include "prox_device.cuh"
#include "prox_internal.h"
#include "token_args.cuh"

namespace prox {

constexpr int kCoarseShift = 24;     // coarse histogram: key bits 30..24
constexpr int kCoarseBins = 128;
static_assert((kScoreBins >> (kCoarseShift - kScoreShift)) == kCoarseBins, "64 fine bins per coarse bin");
constexpr int kFinePerCoarse = kScoreBins / kCoarseBins;
constexpr int kOwnMax = 512;         // channels a CTA scores, at most

// Shared scratch of the selection.
struct alignas(16) SelectScratch {
  uint32_t own[kOwnMax];           // the keys of the CTA's own channels
  float sg[kOwnMax], su[kOwnMax];  // their g~ and u~ while scoring
  uint32_t coarse[kCoarseBins];    // the CTA's coarse counts while scoring
  uint32_t ck[kBucketCap];         // candidate keys
  int32_t ci[kBucketCap];          // candidate channels
  unsigned long long wsum[32][4];  // per-warp packed digit counts
  int scan[36];
  int misc[16];
};

// Bytes of the selection's shared memory for d_ff = F: the scratch, then
// room for every key (used only when the boundary bin overflows its bucket)
// or, while scoring, for the CTA's fine histogram.
__host__ __device__ constexpr size_t select_smem_bytes(int F) {
  return ((sizeof(SelectScratch) + 15) & ~(size_t)15) + (size_t)(F > kScoreBins ? F : kScoreBins) * 4;
}
__device__ __forceinline__ uint32_t* select_keys(SelectScratch& sc) {
  return reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(&sc) +
                                     ((sizeof(SelectScratch) + 15) & ~(size_t)15));
}

struct TopkCut {
  uint32_t T;   // key of the k-th largest score
  int tie_cut;  // keys equal to T are selected up to this channel
};

__device__ __forceinline__ bool selected(uint32_t key, int e, const TopkCut& cut) {
  return key > cut.T || (key == cut.T && e <= cut.tie_cut);
}

// Digit counts over the CTA: thread t's values come from its packed words
// c[4] (digit d at bits 16 (d % 4) of c[d / 4]).  Returns the 16 totals in
// tot[16] (every thread).  Totals stay below 2^16.
__device__ __forceinline__ void block_digit_counts(const unsigned long long (&c)[4],
                                                   SelectScratch& sc, int (&tot)[16]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  unsigned long long w[4] = {c[0], c[1], c[2], c[3]};
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] += __shfl_xor_sync(0xffffffffu, w[q], o);
  if (lane == 0)
#pragma unroll
    for (int q = 0; q < 4; ++q) sc.wsum[warp][q] = w[q];
  __syncthreads();
  unsigned long long s[4] = {0ull, 0ull, 0ull, 0ull};
  for (int i = 0; i < nw; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) s[q] += sc.wsum[i][q];
#pragma unroll
  for (int dgt = 0; dgt < 16; ++dgt) tot[dgt] = (int)((s[dgt >> 2] >> (16 * (dgt & 3))) & 0xFFFFull);
  __syncthreads();  // wsum may be rewritten after return
}

__device__ __forceinline__ void add_digit(unsigned long long (&c)[4], uint32_t dgt) {
  const unsigned long long inc = 1ull << (16 * (dgt & 3u));
  c[0] += (dgt >> 2) == 0 ? inc : 0ull;
  c[1] += (dgt >> 2) == 1 ? inc : 0ull;
  c[2] += (dgt >> 2) == 2 ? inc : 0ull;
  c[3] += (dgt >> 2) == 3 ? inc : 0ull;
}

// Radix select over keys spread over the threads: `items(fn)` calls
// fn(key, channel) for each of this thread's keys.  Returns the krem-th
// largest key (1-based) in *T, how many keys equal it in *n_eq, and the rank
// wanted among those in *k_eq.  Every thread calls it.
template <typename Items>
__device__ void radix_kth(Items items, int krem, SelectScratch& sc, uint32_t* T, int* n_eq,
                          int* k_eq) {
  uint32_t prefix = 0u, pmask = 0u;
  int neq = 0;
  for (int shift = 28; shift >= 0; shift -= 4) {
    unsigned long long c[4] = {0ull, 0ull, 0ull, 0ull};
    items([&](uint32_t key, int) {
      if ((key & pmask) == prefix) add_digit(c, (key >> shift) & 15u);
    });
    int tot[16];
    block_digit_counts(c, sc, tot);
    int above = 0, dsel = 0, cnt = 0;
#pragma unroll
    for (int dgt = 15; dgt >= 0; --dgt) {  // the digit holding the krem-th largest
      if (cnt == 0 && above + tot[dgt] >= krem) {
        dsel = dgt;
        cnt = tot[dgt];
      } else if (cnt == 0) {
        above += tot[dgt];
      }
    }
    krem -= above;
    neq = cnt;
    prefix |= (uint32_t)dsel << shift;
    pmask |= 15u << shift;
  }
  *T = prefix;
  *n_eq = neq;
  *k_eq = krem;
}

// The want-th smallest channel (1-based) among the keys equal to T.
template <typename Items>
__device__ int radix_tie(Items items, uint32_t T, int want, SelectScratch& sc) {
  uint32_t ip = 0u, im = 0u;
  for (int shift = 12; shift >= 0; shift -= 4) {  // channels < 2^16
    unsigned long long c[4] = {0ull, 0ull, 0ull, 0ull};
    items([&](uint32_t key, int ch) {
      if (key == T && ((uint32_t)ch & im) == ip) add_digit(c, ((uint32_t)ch >> shift) & 15u);
    });
    int tot[16];
    block_digit_counts(c, sc, tot);
    int below = 0, dsel = 0;
    bool found = false;
#pragma unroll
    for (int dgt = 0; dgt < 16; ++dgt) {
      if (!found && below + tot[dgt] >= want) {
        dsel = dgt;
        found = true;
      } else if (!found) {
        below += tot[dgt];
      }
    }
    want -= below;
    ip |= (uint32_t)dsel << shift;
    im |= 15u << shift;
  }
  return (int)ip;
}

// Warp 0's share of the cut: among nb bins (a multiple of 32, at most 128)
// read from the top (bins[nb - 1] first), the one holding the krem-th largest
// key, once the counts add up to `want` (polled: counts only grow; bounded).
// Writes its position from the top, the rank wanted inside it and its count
// to misc[m0 .. m0 + 2] (0, 1, 0 when no bin holds it); the CTA reads them
// after a barrier.
__device__ __forceinline__ void warp_find_bin_desc(const uint32_t* bins, int nb, int krem, int want,
                                                   SelectScratch& sc, int m0, int* err) {
  const int lane = threadIdx.x & 31, bpl = nb >> 5;
  const long long t0 = clock64();
  int c[4] = {0, 0, 0, 0}, sum = 0, incl = 0;
  for (;;) {
    sum = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q < bpl) {
        c[q] = (int)ld_relaxed_u32(bins + (nb - 1 - (lane * bpl + q)));
        sum += c[q];
      }
    incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int stop = __shfl_sync(0xffffffffu, incl, 31) == want;
    if (!stop && lane == 0) stop = !wait_more(t0, err);
    if (__shfl_sync(0xffffffffu, stop, 0)) break;
  }
  if (lane == 0) {
    sc.misc[m0] = 0;
    sc.misc[m0 + 1] = 1;
    sc.misc[m0 + 2] = 0;
  }
  __syncwarp();
  const int above = incl - sum;
  if (sum > 0 && above < krem && incl >= krem) {
    int acc = above;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q < bpl) {
        if (acc + c[q] >= krem) {
          sc.misc[m0] = lane * bpl + q;
          sc.misc[m0 + 1] = krem - acc;
          sc.misc[m0 + 2] = c[q];
          break;
        }
        acc += c[q];
      }
  }
}

// The exact cut of the launch; every CTA calls it once it has added its own
// counts (blockDim.x >= kCoarseBins).  1 <= k <= F.  The histograms are
// complete when the coarse counts add up to F and the fine counts under a
// coarse bin add up to its count (every count only grows), so the CTA polls
// them until they do; bucket entries and keys are tagged words.  A wait that
// runs out sets PROX_DEVERR_WAIT_TIMEOUT and goes on with what it has.
__device__ inline TopkCut select_cut(const uint32_t* hist, const uint32_t* chist,
                              const unsigned long long* bucket, const unsigned long long* st64, int F,
                              int k, SelectScratch& sc, uint32_t tag, int* err,
                              unsigned long long* ts) {
  const int tid = threadIdx.x;
  long long t0;
  // 1. the coarse bin (bins read from the top; warp 0 polls and scans them)
  if (tid < 32) warp_find_bin_desc(chist, kCoarseBins, k, F, sc, 0, err);
  __syncthreads();
  stamp(ts, 14);
  const int cb = kCoarseBins - 1 - sc.misc[0];
  const int k1 = sc.misc[1];
  const int ncb = sc.misc[2];
  // 2. its fine bins
  const int fb0 = cb * kFinePerCoarse;
  if (tid < 32) warp_find_bin_desc(hist + fb0, kFinePerCoarse, k1, ncb, sc, 3, err);
  __syncthreads();
  const uint32_t b1 = (uint32_t)(fb0 + kFinePerCoarse - 1 - sc.misc[3]);
  const int krem = sc.misc[4];
  const int n1 = sc.misc[5];
  TopkCut cut;
  if (n1 <= kBucketCap) {
    // 3. the candidates, ranked: the one with krem - 1 larger (key, ~channel)
    // composites is the cut
    if (tid < n1) {
      const unsigned long long* src = bucket + ((size_t)b1 * kBucketCap + tid) * 2;
      ulonglong2 kc = ld_tag2(src);
      t0 = clock64();
      while (!(tag_ok(kc.x, tag) && tag_ok(kc.y, tag)) && wait_more(t0, err)) kc = ld_tag2(src);
      sc.ck[tid] = (uint32_t)kc.x;
      sc.ci[tid] = (int)(uint32_t)kc.y;
    }
    if (tid == 0) {
      sc.misc[7] = 0;
      sc.misc[12] = F;
    }
    __syncthreads();
    if (tid < n1) {
      const unsigned long long c = ((unsigned long long)sc.ck[tid] << 32) | (uint32_t)~(uint32_t)sc.ci[tid];
      int rank = 0;
      for (int j = 0; j < n1; ++j)
        rank += (((unsigned long long)sc.ck[j] << 32) | (uint32_t)~(uint32_t)sc.ci[j]) > c;
      if (rank == krem - 1) {
        sc.misc[7] = (int)sc.ck[tid];
        sc.misc[12] = sc.ci[tid];
      }
    }
    __syncthreads();
    cut.T = (uint32_t)sc.misc[7];
    cut.tie_cut = sc.misc[12];
    __syncthreads();
    return cut;
  }
  // 3'. b1 overflowed its bucket (many equal scores): radix select over every
  // key (the magnitude bits of the tagged act(g~) u~), loaded into shared
  // memory
  uint32_t* sk = select_keys(sc);
  for (int e = tid; e < F; e += blockDim.x) {
    unsigned long long w = ld_tag(st64 + e);
    t0 = clock64();
    while (!tag_ok(w, tag) && wait_more(t0, err)) w = ld_tag(st64 + e);
    sk[e] = (uint32_t)w & 0x7FFFFFFFu;
  }
  __syncthreads();
  const int per = (F + (int)blockDim.x - 1) / (int)blockDim.x;
  const int j0 = min(tid * per, F), j1 = min(j0 + per, F);
  auto all = [&](auto fn) {
    for (int j = j0; j < j1; ++j) fn(sk[j], j);
  };
  int n_eq, k_eq;
  radix_kth(all, k, sc, &cut.T, &n_eq, &k_eq);
  cut.tie_cut = k_eq < n_eq ? radix_tie(all, cut.T, k_eq, sc) : F;
  return cut;
}

}  // namespace prox
