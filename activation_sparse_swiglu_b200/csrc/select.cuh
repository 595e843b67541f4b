// Per-token top-k channel select (Prox App. A.6 "Per-token top-k
// selection"): the k channels of largest proxy score |s~_j|, ties going to the
// lower channel index.
//
// select_cut -- the exact cut, computed by every CTA of the per-token kernel
// once all scores of the token are written, from the token's scores held in
// the CTA's shared memory.  Stage 1 counts the scores in an 8192-bin histogram
// of their bits 30..18 (the first radix level).  The cut is then:
//   1. the boundary bin b1 holding the k-th largest key (a scan over the
//      histogram, 32 bins per thread);
//   2. the candidates -- the keys of bin b1 -- gathered from the shared keys;
//   3. the candidates ordered by (key descending, index ascending) --
//      directly when there are few, by radix select on the remaining key bits
//      and then the index bits otherwise -- give the k-th largest key T and
//      the tie cut: channel j is selected iff key_j > T, or key_j == T and
//      j <= tie cut.
// Scores are non-negative floats, so their bit patterns order like the values.
#pragma once
#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {

constexpr int kSelectDirect = 768;   // candidates ranked directly (O(n^2))
constexpr int kSelectWorkers = 256;  // threads that scan
static_assert(kScoreBins == kSelectWorkers * 32, "32 histogram bins per worker");

// Shared scratch of select_cut; the keys of all channels follow it.
struct alignas(16) SelectScratch {
  uint32_t h[1024];                // the finer radix levels
  uint32_t ck[kSelectCand];        // candidate keys
  int32_t ci[kSelectCand];         // candidate channels
  unsigned long long c64[kSelectDirect];
  int scan[36];
  int misc[16];
};

// Bytes of the selection's shared memory for d_ff = F: the scratch, then the
// keys [F].
__host__ __device__ constexpr size_t select_smem_bytes(int F) {
  return ((sizeof(SelectScratch) + 15) & ~(size_t)15) + (size_t)F * 4;
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

// Over the candidate keys (bin b1): the gathered list, or -- when it
// overflowed -- every key of bin b1 in the shared keys (worker threads).
template <typename Fn>
__device__ __forceinline__ void for_each_cand(const uint32_t* sk, int F, bool listed, int n,
                                              const SelectScratch& sc, uint32_t b1, Fn fn) {
  if (threadIdx.x >= kSelectWorkers) return;
  if (listed) {
    for (int i = threadIdx.x; i < n; i += kSelectWorkers) fn(sc.ck[i], sc.ci[i]);
  } else {
    for (int e = threadIdx.x; e < F; e += kSelectWorkers) {
      const uint32_t key = sk[e];
      if ((key >> kScoreShift) == b1) fn(key, e);
    }
  }
}

__device__ __forceinline__ uint32_t key_of(const uint4 (&kb)[8], int j) {
  const uint4 v = kb[j >> 2];
  return (j & 3) == 0 ? v.x : (j & 3) == 1 ? v.y : (j & 3) == 2 ? v.z : v.w;
}

// Every thread of the CTA calls it (blockDim.x >= 256); sk holds the keys of
// all F channels.
__device__ TopkCut select_cut(const uint32_t* hist, const uint32_t* sk, int F, int k,
                              SelectScratch& sc) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool worker = tid < kSelectWorkers;

  // 1. boundary bin: worker t holds bins [32q, 32q+32), q = 255 - t, read
  // straight from the histogram in global memory; an exclusive scan over
  // threads counts the keys in higher bins
  {
    const int q = kSelectWorkers - 1 - tid;
    uint4 hv[8];
    int own = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      hv[j] = worker ? __ldcg(reinterpret_cast<const uint4*>(hist) + 8 * q + j)
                     : make_uint4(0u, 0u, 0u, 0u);
      own += (int)(hv[j].x + hv[j].y + hv[j].z + hv[j].w);
    }
    int total;
    const int above = block_exclusive_scan(own, sc.scan, &total);
    if (tid == 0) sc.misc[3] = 0;  // candidates gathered
    if (worker && above < k && above + own >= k) {
      int run = above;
#pragma unroll
      for (int j = 31; j >= 0; --j) {
        const int c = (int)key_of(hv, j);
        if (run < k && run + c >= k) {
          sc.misc[0] = 32 * q + j;  // b1
          sc.misc[1] = k - run;     // rank wanted inside b1 (1-based)
          sc.misc[2] = c;           // keys in b1
        }
        run += c;
      }
    }
  }
  __syncthreads();
  const uint32_t b1 = (uint32_t)sc.misc[0];
  const int krem = sc.misc[1];
  const int n1 = sc.misc[2];

  // 2. the candidates
  const bool listed = n1 <= kSelectCand;
  if (listed) {
    for (int e = tid; e < F; e += blockDim.x) {
      const uint32_t key = sk[e];
      if ((key >> kScoreShift) == b1) {
        const int slot = atomicAdd(&sc.misc[3], 1);
        if (slot < kSelectCand) {
          sc.ck[slot] = key;
          sc.ci[slot] = e;
        }
      }
    }
  }
  __syncthreads();

  // 3. the exact cut among the candidates: T and the tie cut into misc[7],
  // misc[12]
  if (listed && n1 <= kSelectDirect) {
    // The order is that of the composite key << 32 | (~index) descending, so a
    // candidate's rank is the number of larger composites.  Padding with 0
    // (below every real composite) lets the comparison loop run in blocks of
    // 8; TPC adjacent threads share a candidate.
    const int n8 = (n1 + 7) & ~7;
    for (int i = tid; i < n8; i += blockDim.x)
      sc.c64[i] = i < n1 ? ((unsigned long long)sc.ck[i] << 32) | (uint32_t)~(uint32_t)sc.ci[i] : 0ull;
    __syncthreads();
    if (worker) {
      int TPC = 1;
      while (TPC < 32 && n1 * TPC * 2 <= kSelectWorkers) TPC *= 2;
      const int per_pass = kSelectWorkers / TPC;
      for (int i0 = 0; i0 < n1; i0 += per_pass) {
        const int i = i0 + tid / TPC, sub = tid % TPC;
        const unsigned long long c = i < n1 ? sc.c64[i] : ~0ull;
        int rank = 0;
        for (int j = sub * 8; j < n8; j += TPC * 8) {
#pragma unroll
          for (int u = 0; u < 8; ++u) rank += sc.c64[j + u] > c;
        }
        for (int o = 1; o < TPC; o <<= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
        if (i < n1 && sub == 0 && rank == krem - 1) {
          sc.misc[7] = (int)sc.ck[i];
          sc.misc[12] = sc.ci[i];
        }
      }
    }
  } else {
    uint32_t* h = sc.h;
    for (int i = tid; i < 1024; i += blockDim.x) h[i] = 0u;
    __syncthreads();
    // level 2: key bits 17..8
    for_each_cand(sk, F, listed, n1, sc, b1,
                  [&](uint32_t kk, int) { atomicAdd(&h[(kk >> 8) & 0x3FFu], 1u); });
    __syncthreads();
    if (warp == 0) {
      int b2, k2, c2;
      warp_find_bin<32, false>(h, krem, &b2, &k2, &c2);
      if (lane == 0) {
        sc.misc[5] = b2;
        sc.misc[6] = k2;
      }
    }
    __syncthreads();
    const uint32_t p2 = (b1 << 10) | (uint32_t)sc.misc[5];  // key bits 30..8
    for (int i = tid; i < 1024; i += blockDim.x) h[i] = 0u;
    __syncthreads();
    // level 3: key bits 7..0
    for_each_cand(sk, F, listed, n1, sc, b1, [&](uint32_t kk, int) {
      if ((kk >> 8) == p2) atomicAdd(&h[kk & 0xFFu], 1u);
    });
    __syncthreads();
    if (warp == 0) {
      int b3, k3, c3;
      warp_find_bin<8, false>(h, sc.misc[6], &b3, &k3, &c3);
      if (lane == 0) {
        sc.misc[7] = (int)((p2 << 8) | (uint32_t)b3);
        sc.misc[8] = k3;  // keys equal to T that are taken
        sc.misc[9] = c3;  // keys equal to T
        sc.misc[12] = F;  // every key equal to T taken, unless cut below
      }
    }
    __syncthreads();
    const uint32_t T = (uint32_t)sc.misc[7];
    const int k_eq = sc.misc[8], n_eq = sc.misc[9];
    // tie cut: the k_eq-th smallest index among keys equal to T (radix on the
    // index: bits 14..7, then 6..0), i.e. the (n_eq - k_eq + 1)-th largest.
    if (k_eq < n_eq) {
      for (int i = tid; i < 1024; i += blockDim.x) h[i] = 0u;
      __syncthreads();
      for_each_cand(sk, F, listed, n1, sc, b1, [&](uint32_t kk, int ix) {
        if (kk == T) atomicAdd(&h[(ix >> 7) & 0xFFu], 1u);
      });
      __syncthreads();
      if (warp == 0) {
        int bi, ki, ci;
        warp_find_bin<8, false>(h, n_eq - k_eq + 1, &bi, &ki, &ci);
        if (lane == 0) {
          sc.misc[10] = bi;
          sc.misc[11] = ki;
        }
      }
      __syncthreads();
      const int hi7 = sc.misc[10];
      for (int i = tid; i < 1024; i += blockDim.x) h[i] = 0u;
      __syncthreads();
      for_each_cand(sk, F, listed, n1, sc, b1, [&](uint32_t kk, int ix) {
        if (kk == T && (ix >> 7) == hi7) atomicAdd(&h[ix & 0x7F], 1u);
      });
      __syncthreads();
      if (warp == 0) {
        int bl, kl, cl;
        warp_find_bin<4, false>(h, sc.misc[11], &bl, &kl, &cl);
        if (lane == 0) sc.misc[12] = (hi7 << 7) | bl;
      }
      __syncthreads();
    }
  }
  __syncthreads();
  TopkCut cut;
  cut.T = (uint32_t)sc.misc[7];
  cut.tie_cut = sc.misc[12];
  __syncthreads();  // the scratch may be reused after return
  return cut;
}

}  // namespace prox
