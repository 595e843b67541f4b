// Per-token top-k channel select (Prox App. A.6 "Per-token top-k
// selection"): the k channels of largest proxy score |s~_j|, ties going to the
// lower channel index.
//
// select_kernel -- one CTA per 256-channel slice of the scores.  Every CTA
// reads the 2048-bin histogram of score bits 30..20 built by Stage 1 and finds
// the boundary bin b1 holding the k-th largest score; it then counts the keys
// of its slice above b1 and appends the keys inside b1 (the candidates) to a
// global list.  The last CTA to finish (atomic ticket, no waiting) orders the
// candidates by (key descending, index ascending) -- directly when there are
// few, by radix select on the key bits and then the index bits otherwise --
// which gives the exact k-th largest key T and the tie cut (keys equal to T
// are taken up to that index), and publishes, per slice, the number of
// selected channels as an exclusive prefix (rank offsets).  Stage 2 turns its
// rank range into channels from those offsets.
#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {
namespace {

constexpr int SEL_NT = kSelectSlice;  // one thread per channel of a slice
constexpr int kSelectDirect = 768;    // boundary-bin size ranked directly

struct SelectArgs {
  const float* scores;
  int F, k, nsl;
  SelectState st;
  unsigned long long* stats;
};

// Over the candidate keys (bin b1): either the collected list in shared
// memory, or -- when it overflowed -- every key of the scores with bin b1.
template <typename Fn>
__device__ __forceinline__ void for_each_cand(const SelectArgs& a, bool listed, int n,
                                              const uint32_t* ck, const int32_t* ci, uint32_t b1,
                                              Fn fn) {
  if (listed) {
    for (int i = threadIdx.x; i < n; i += SEL_NT) fn(ck[i], ci[i]);
  } else {
    for (int e = threadIdx.x; e < a.F; e += SEL_NT) {
      const uint32_t key = __float_as_uint(__ldcg(a.scores + e));
      if ((key >> 20) == b1) fn(key, e);
    }
  }
}

__global__ void __launch_bounds__(SEL_NT) select_kernel(SelectArgs a) {
  __shared__ __align__(16) uint32_t s_h[kHistBins];
  __shared__ unsigned long long s_c64[kSelectDirect];
  __shared__ uint32_t s_ck[kSelectCand];
  __shared__ int32_t s_ci[kSelectCand];
  __shared__ int s_sel[kMaxSlices + 1];
  __shared__ int s_misc[16];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x;

  pdl_wait();
  pdl_trigger();

  const int e = s * SEL_NT + tid;
  const bool valid = e < a.F;
  const uint32_t key = valid ? __float_as_uint(__ldcg(a.scores + e)) : 0u;
  // the level-1 histogram (built by Stage 1) into shared memory: one round trip
  for (int i = tid; i < kHistBins / 4; i += SEL_NT)
    reinterpret_cast<uint4*>(s_h)[i] = __ldcg(reinterpret_cast<const uint4*>(a.st.hist) + i);
  __syncthreads();
  if (warp == 0) {
    int b1, krem, n1;
    warp_find_bin<kHistBins / 32, false>(s_h, a.k, &b1, &krem, &n1);
    if (lane == 0) {
      s_misc[0] = b1;
      s_misc[1] = krem;
      s_misc[2] = n1;
    }
  }
  __syncthreads();
  const uint32_t b1 = (uint32_t)s_misc[0];
  const bool above = valid && (key >> 20) > b1;
  const bool cand = valid && (key >> 20) == b1;
  const unsigned ma = __ballot_sync(0xffffffffu, above);
  const unsigned mc = __ballot_sync(0xffffffffu, cand);
  if (lane == 0) s_misc[4 + warp] = __popc(ma);
  if (mc) {  // warp-aggregated append to the global candidate list
    int base = 0;
    if (lane == 0) base = (int)atomicAdd(a.st.state + kSelCandCount, (uint32_t)__popc(mc));
    base = __shfl_sync(0xffffffffu, base, 0) + __popc(mc & ((1u << lane) - 1u));
    if (cand && base < kSelectCand) {
      a.st.cand_key[base] = key;
      a.st.cand_idx[base] = e;
    }
  }
  __syncthreads();
  if (tid == 0) {
    int g = 0;
    for (int w = 0; w < SEL_NT / 32; ++w) g += s_misc[4 + w];
    a.st.sl_gt1[s] = g;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_misc[3] = atomicAdd(a.st.state + kSelTicket, 1u) == (uint32_t)(a.nsl - 1);
  __syncthreads();
  if (!s_misc[3]) return;
  __threadfence();

  // ---------------- the last CTA: exact threshold, tie cut, rank offsets ----------------
  // Candidates are ordered by (key descending, index ascending); the one of
  // rank krem-1 is the boundary: T = its key, tie cut = its index.
  const int krem = s_misc[1];
  const int n1 = s_misc[2];
  const bool listed = n1 <= kSelectCand;
  if (listed) {
    for (int i = tid; i < n1; i += SEL_NT) {
      s_ck[i] = __ldcg(a.st.cand_key + i);
      s_ci[i] = __ldcg(a.st.cand_idx + i);
    }
  }
  for (int i = tid; i < a.nsl; i += SEL_NT) s_sel[i] = __ldcg(a.st.sl_gt1 + i);
  __syncthreads();
  uint32_t T;
  int tie_cut;
  if (listed && n1 <= kSelectDirect) {
    // Direct ranks.  The order (key descending, index ascending) is that of
    // the composite key << 32 | (~index) descending, so a candidate's rank is
    // the number of larger composites.  Padding with 0 (below every real
    // composite) lets the comparison loop run in blocks of 8.
    const int n8 = (n1 + 7) & ~7;
    for (int i = tid; i < n8; i += SEL_NT)
      s_c64[i] = i < n1 ? ((unsigned long long)s_ck[i] << 32) | (uint32_t)~(uint32_t)s_ci[i] : 0ull;
    __syncthreads();
    for (int i = tid; i < n1; i += SEL_NT) {
      const unsigned long long ci = s_c64[i];
      int rank = 0;
      for (int j = 0; j < n8; j += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) rank += s_c64[j + u] > ci;
      }
      const int ii = s_ci[i];
      if (rank < krem) atomicAdd(&s_sel[ii / kSelectSlice], 1);
      if (rank == krem - 1) {
        s_misc[7] = (int)s_ck[i];
        s_misc[12] = ii;
      }
    }
    __syncthreads();
    T = (uint32_t)s_misc[7];
    tie_cut = s_misc[12];
  } else {
    for (int i = tid; i < 1024; i += SEL_NT) s_h[i] = 0u;
    __syncthreads();
    // level 2: bits 19..10
    for_each_cand(a, listed, n1, s_ck, s_ci, b1,
                  [&](uint32_t kk, int) { atomicAdd(&s_h[(kk >> 10) & 0x3FFu], 1u); });
    __syncthreads();
    if (warp == 0) {
      int b2, k2, c2;
      warp_find_bin<32, false>(s_h, krem, &b2, &k2, &c2);
      if (lane == 0) {
        s_misc[5] = b2;
        s_misc[6] = k2;
      }
    }
    __syncthreads();
    const uint32_t p2 = (b1 << 10) | (uint32_t)s_misc[5];
    for (int i = tid; i < 1024; i += SEL_NT) s_h[i] = 0u;
    __syncthreads();
    // level 3: bits 9..0
    for_each_cand(a, listed, n1, s_ck, s_ci, b1, [&](uint32_t kk, int) {
      if ((kk >> 10) == p2) atomicAdd(&s_h[kk & 0x3FFu], 1u);
    });
    __syncthreads();
    if (warp == 0) {
      int b3, k3, c3;
      warp_find_bin<32, false>(s_h, s_misc[6], &b3, &k3, &c3);
      if (lane == 0) {
        s_misc[7] = (int)((p2 << 10) | (uint32_t)b3);
        s_misc[8] = k3;  // keys equal to T that are taken
        s_misc[9] = c3;  // keys equal to T
      }
    }
    __syncthreads();
    T = (uint32_t)s_misc[7];
    const int k_eq = s_misc[8], n_eq = s_misc[9];
    // tie cut: the k_eq-th smallest index among keys equal to T (radix on the
    // index: bits 14..7, then 6..0), i.e. the (n_eq - k_eq + 1)-th largest.
    tie_cut = a.F;
    if (k_eq < n_eq) {
      for (int i = tid; i < 1024; i += SEL_NT) s_h[i] = 0u;
      __syncthreads();
      for_each_cand(a, listed, n1, s_ck, s_ci, b1, [&](uint32_t kk, int ix) {
        if (kk == T) atomicAdd(&s_h[(ix >> 7) & 0xFFu], 1u);
      });
      __syncthreads();
      if (warp == 0) {
        int bi, ki, ci;
        warp_find_bin<8, false>(s_h, n_eq - k_eq + 1, &bi, &ki, &ci);
        if (lane == 0) {
          s_misc[10] = bi;
          s_misc[11] = ki;
        }
      }
      __syncthreads();
      const int hi7 = s_misc[10];
      for (int i = tid; i < 1024; i += SEL_NT) s_h[i] = 0u;
      __syncthreads();
      for_each_cand(a, listed, n1, s_ck, s_ci, b1, [&](uint32_t kk, int ix) {
        if (kk == T && (ix >> 7) == hi7) atomicAdd(&s_h[ix & 0x7F], 1u);
      });
      __syncthreads();
      if (warp == 0) {
        int bl, kl, cl;
        warp_find_bin<4, false>(s_h, s_misc[11], &bl, &kl, &cl);
        if (lane == 0) s_misc[12] = (hi7 << 7) | bl;
      }
      __syncthreads();
      tie_cut = s_misc[12];
    }
    // selected channels per slice: those above b1 (already counted), plus
    // candidates above T or tied at T up to the cut
    for_each_cand(a, listed, n1, s_ck, s_ci, b1, [&](uint32_t kk, int ix) {
      if (kk > T || (kk == T && ix <= tie_cut)) atomicAdd(&s_sel[ix / kSelectSlice], 1);
    });
    __syncthreads();
  }
  if (warp == 0) {
    // exclusive prefix over the slices (at most kMaxSlices)
    constexpr int PERL = kMaxSlices / 32;
    int v[PERL], sum = 0;
#pragma unroll
    for (int j = 0; j < PERL; ++j) {
      const int sl = lane * PERL + j;
      v[j] = sl < a.nsl ? s_sel[sl] : 0;
      sum += v[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nb = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += nb;
    }
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < PERL; ++j) {
      const int sl = lane * PERL + j;
      if (sl <= a.nsl) a.st.sl_off[sl] = run;
      run += v[j];
    }
    if (lane == 0) {
      a.st.state[kSelT] = T;
      a.st.state[kSelTieCut] = (uint32_t)tie_cut;
      a.st.state[kSelCandCount] = 0u;  // ready for the next token
      a.st.state[kSelTicket] = 0u;
      if (a.stats) atomicAdd(a.stats + 1, 1ull);
    }
  }
}

}  // namespace

cudaError_t launch_select(const prox_layer* L, cudaStream_t s, bool pdl) {
  SelectArgs a;
  a.scores = L->ws.scores;
  a.F = L->F;
  a.k = L->k;
  a.nsl = (L->F + kSelectSlice - 1) / kSelectSlice;
  a.st = L->ws.sel;
  a.stats = L->ws.stats;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.nsl, 1, 1);
  cfg.blockDim = dim3(SEL_NT, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel, a);
}

}  // namespace prox
