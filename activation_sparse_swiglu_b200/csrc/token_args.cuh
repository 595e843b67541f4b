// Arguments of the fused per-token kernel (token.cu) and the small device
// primitives its phases share: the grid-wide barrier and the exponent words of
// the INT4 decode.
#pragma once

#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {

// Stage-2 channel rules (TokenArgs::mode).
enum TokenMode : int {
  kModeNone = -1,      // Stage 1 only (proxy scores)
  kModeList = 0,       // a caller-given channel list
  kModeTopK = 1,       // per-token top-k of the Stage-1 scores (Prox App. A.6)
  kModeDense = 2,      // every channel (the dense baseline)
  kModeThreshold = 3,  // score >= tau_s (Prox §4.1)
};

// Exponent words for the nibble decode: 2^23, 2^19, 2^15, 2^11, 2^7.
struct Magic {
  uint32_t e23, e19, e15, e11, e7;
};

struct TokenArgs {
  const float* x;        // [d] this token's input
  float* out;            // [d] this token's output (Stage 2 modes)
  // library-owned weights
  const uint8_t* pq;     // INT4 proxy codes [C][d][512 B], gate/up interleaved per 16 B
  const __half* ps;      // fp16 scales [G][F/32][2][32]
  const uint16_t* wgu;   // bf16 channel records [F][2d]
  const uint16_t* wd;    // bf16 W_down rows [F][d]
  int d, F;
  // Stage-1 geometry
  int C;                 // 512-byte column slices of a proxy row
  int lmax;              // kept-row capacity of a CTA
  float tau;             // tau_x
  // Stage-2 geometry
  int slots, groups, max_rec;
  // what runs
  int stage1;            // 1: Stage 1 runs in this launch
  int mode;              // TokenMode
  int select_only;       // stop after the channel selection (writes sel_mask)
  int proxy_values;      // A3: s~ of Stage 1 instead of the exact s
  int act;               // gate activation (PROX_ACT_*)
  int k;                 // top-k count, or list length
  float tau_s;           // threshold mode
  const int32_t* idx;    // list mode: channels [k]
  // workspace
  float* scores;         // |act(g~) u~| [F]
  float* s_tilde;        // Stage 1 writes act(g~) u~ here when non-null [F]
  const float* s_tilde_src;  // A3 Stage 2 reads it here
  uint32_t* hist;        // [kScoreBins] fine histogram of the scores' bits 30..18
  uint32_t* chist;       // [128] coarse histogram of the scores' bits 30..24
  uint2* bucket;         // [kScoreBins][kBucketCap] (key, channel) per fine bin
  int32_t* sel_list;     // [F] CTA c's selected channels from its range's first channel on
  int32_t* sel_cnt;      // [P] CTA c's selected count
  unsigned long long* stats;
  float* part;           // Stage-1 partial sums [P][2][1024]
  float* ypart;          // Stage-2 partial output rows [P][d]
  unsigned long long* gbar;  // grid-barrier arrival counter
  int* err;              // device error word
  // taps (each may be null)
  float* g_dbg;
  float* u_dbg;
  int32_t* idx_x;
  int32_t* n_x;
  int32_t* sel_mask;     // 1/0 per channel (top-k / threshold)
  float* s_sp;           // act(g) u per selected channel
  unsigned long long* ts;  // optional phase stamps [P][kPhaseStamps]
  Magic mg;
};

// Phase stamp i of this CTA (globaltimer, ns) when stamps were asked for:
// 0 kernel entry, 1 previous kernel complete, 2 Stage-1 partials written,
// 3 partials visible (barrier), 4 channels selected, 5 partial output row
// written, 6 partial rows visible (barrier), 7 output written; 8 kept rows
// compacted, 9 Stage-1 row loop done, 10 scores of the CTA's channels written,
// 14 the histograms complete (barrier); 11 Stage-2 ring set up, 12 gate/up
// phase done; slot 13 holds the CTA's channel count, not a time.
__device__ __forceinline__ void stamp(unsigned long long* ts, int i) {
  if (ts && threadIdx.x == 0) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    ts[(size_t)blockIdx.x * kPhaseStamps + i] = t;
  }
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void red_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Grid-wide barriers of one launch whose CTAs are all resident (cooperative
// launch, one CTA per SM).  The layer's 64-bit arrival counter only grows:
// thread 0 of every CTA reads it once when the launch starts; the previous
// launch on the layer is complete by then and every barrier adds exactly
// gridDim.x arrivals, so rounding the value read down to a multiple of
// gridDim.x gives every CTA the same base even when faster CTAs have already
// arrived at the first barrier.  Barrier i of the launch is complete once the
// counter reaches base + i * expected.  A CTA's thread 0, after a bar.sync, releases the CTA's
// writes (fence) and arrives with a reduction (no round trip); it then polls
// the counter and acquires (fence) once the target is reached.  So every
// write made before the barrier by any thread of any CTA is visible to every
// thread after it.  The wait is bounded: when it runs out the CTA sets
// PROX_DEVERR_WAIT_TIMEOUT, marks itself dead (later barriers do not wait)
// and carries on, so a CTA that never arrives cannot hang the GPU; the host
// resets the counter in prox_layer_error.
struct GridSync {
  unsigned long long* ctr;
  unsigned long long base;  // thread 0: the counter when the launch started
  unsigned n;               // barriers passed so far
  bool dead;                // thread 0: a wait of this CTA ran out
};

__device__ __forceinline__ GridSync grid_sync_begin(unsigned long long* ctr) {
  GridSync g;
  g.ctr = ctr;
  if (threadIdx.x == 0) {
    const unsigned long long v = ld_relaxed_u64(ctr);
    g.base = v - v % gridDim.x;
  } else {
    g.base = 0ull;
  }
  g.n = 0;
  g.dead = false;
  return g;
}

// Every thread of the CTA calls it.
__device__ __forceinline__ void grid_barrier(GridSync& g, unsigned expected, int* err) {
  __syncthreads();
  ++g.n;
  if (threadIdx.x == 0) {
    const unsigned long long target = g.base + (unsigned long long)g.n * expected;
    fence_acq_rel_gpu();
    red_add_u64(g.ctr, 1ull);
    if (!g.dead) {
      const long long t0 = clock64();
      while (ld_relaxed_u64(g.ctr) < target) {
        __nanosleep(64);
        if (clock64() - t0 > kWaitLimitCycles) {
          atomicOr(err, PROX_DEVERR_WAIT_TIMEOUT);
          g.dead = true;
          break;
        }
      }
    }
    fence_acq_rel_gpu();
  }
  __syncthreads();
}

// Orders earlier generic-proxy accesses of this CTA's shared memory before
// later bulk-copy (async-proxy) writes to the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace prox
