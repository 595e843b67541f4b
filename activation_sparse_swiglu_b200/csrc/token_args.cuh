// Arguments of the fused per-token kernel (token.cu) and the small device
// primitives its phases share: the tagged exchange words and the phase hints.
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
  int s1_depth;          // Stage-1 k-tiles in flight per warp
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
  unsigned long long* stats;
  // exchanged between the CTAs of the launch (tagged words: payload | tag << 32)
  uint32_t* hist;        // [2][kScoreBins] fine histograms of the scores' bits 30..18
  uint32_t* chist;       // [2][kCoarseBins] coarse histograms of the scores' bits 30..24
  unsigned long long* bucket;  // [kScoreBins][kBucketCap][2] tagged (key, channel) per fine bin
  unsigned long long* st64;    // [F] tagged bits of act(g~) u~
  unsigned long long* sel_list;  // [F] tagged: CTA c's selected channels from its range's start
  unsigned long long* sel_cnt;   // [P] tagged: CTA c's selected count
  unsigned long long* part;    // [P][2][1024] tagged Stage-1 partial sums
  unsigned long long* ypart;   // [P][d] tagged Stage-2 partial output rows
  unsigned long long* gbar;    // launch counter: every CTA adds 1 when it ends
  int* err;              // device error word
  // taps (each may be null)
  float* g_dbg;
  float* u_dbg;
  int32_t* idx_x;
  int32_t* n_x;
  int32_t* sel_mask;     // 1/0 per channel (top-k / threshold)
  float* s_sp;           // act(g) u per selected channel
  unsigned long long* ts;  // optional phase stamps [P][kPhaseStamps]
};

// Phase stamp i of this CTA (the SM's clock64 cycle count) when stamps were
// asked for (a cycle count costs next to nothing; the global timer is read
// only at entry, slot 22, and exit, slot 23, with the exit cycle count in
// slot 21, to place the cycle counts on one ns time line):
// 0 kernel entry, 1 previous kernel complete, 8 kept rows compacted, 9 Stage-1
// row loop done (the CTA's partials stored), 2 phase 0 reported, 16 phase 0
// complete, 3 the partials of thread 0's channel received, 10 the CTA's
// channels scored and counted, 17 phase 1 complete, 14 the coarse histogram
// complete, 15 the top-k cut found, 18 phase 2 complete, 4 the CTA's Stage-2
// channels known, 11 Stage-2 ring set up, 12 gate/up phase done, 5 partial
// output row written, 19 phase 3 complete, 6 the partial rows of the CTA's
// columns received, 7 output written, 21 exit; slot 13 holds the CTA's
// Stage-2 channel count, not a time.
__device__ __forceinline__ void stamp(unsigned long long* ts, int i) {
  if (ts && threadIdx.x == 0) ts[(size_t)blockIdx.x * kPhaseStamps + i] = (unsigned long long)clock64();
}
__device__ __forceinline__ void stamp_timer(unsigned long long* ts, int clock_slot, int timer_slot) {
  if (ts && threadIdx.x == 0) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    ts[(size_t)blockIdx.x * kPhaseStamps + clock_slot] = (unsigned long long)clock64();
    ts[(size_t)blockIdx.x * kPhaseStamps + timer_slot] = t;
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

// Tagged words.  Everything one CTA of a launch writes for others to read is
// a 64-bit word holding a 32-bit payload and, in its high half, the launch's
// tag, stored and loaded with single 64-bit relaxed accesses (single-copy
// atomic at gpu scope).  A reader polls until the tag is the launch's: the
// payload it then holds is the one written in this launch, with no fence and
// no barrier between writer and reader.  The tag is the launch's index (the
// launch counter over the grid size, which every launch advances by exactly
// one) with the top bit set, so it is never that of zeroed memory and never
// that of the launch before.
__device__ __forceinline__ unsigned long long tag_word(uint32_t payload, uint32_t tag) {
  return ((unsigned long long)tag << 32) | payload;
}
__device__ __forceinline__ bool tag_ok(unsigned long long w, uint32_t tag) {
  return (uint32_t)(w >> 32) == tag;
}
__device__ __forceinline__ void st_tag(unsigned long long* p, unsigned long long w) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ void st_tag2(unsigned long long* p, unsigned long long w0,
                                        unsigned long long w1) {
  asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(w0), "l"(w1) : "memory");
}
__device__ __forceinline__ unsigned long long ld_tag(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ ulonglong2 ld_tag2(const unsigned long long* p) {
  ulonglong2 v;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded waiting: a poll loop calls wait_more(t0, err) after each miss; it
// sleeps briefly (the pollers must not crowd out the CTAs still streaming)
// and returns false once kWaitLimitCycles have passed since t0, after setting
// PROX_DEVERR_WAIT_TIMEOUT.  The caller then carries on with what it has.
__device__ __forceinline__ bool wait_more(long long t0, int* err) {
  __nanosleep(64);
  if (clock64() - t0 > kWaitLimitCycles) {
    atomicOr(err, PROX_DEVERR_WAIT_TIMEOUT);
    return false;
  }
  return true;
}

// Phase hints.  Each CTA adds 1 to the layer's launch counter at each of the
// kPhases phase points of every launch, whether or not the launch runs that
// phase: 0 Stage-1 partials written, 1 scores counted, 2 selection counts
// written, 3 partial output rows written.  So a launch starts with the
// counter at a multiple of kPhases * gridDim.x, its index is the counter over
// that (a CTA reading it late still sees fewer than kPhases * gridDim.x of
// this launch's additions), and phase j of the launch has been passed by
// every CTA once the counter reaches base + (j + 1) * gridDim.x.  A reader
// waits for that (one polling thread per CTA, on one word) before it reads
// what the phase wrote; the data itself is tagged, so an add that overtakes
// the writes it follows costs a re-poll, never a wrong value.  No fence.
constexpr int kPhases = 4;

// The launch's index from the launch counter read at its start: every
// earlier launch added kPhases * gridDim.x to it, and fewer than that many of
// this launch's additions can be in it.  Its tag: the index, top bit set.
__device__ __forceinline__ unsigned long long launch_index(unsigned long long counter) {
  return counter / ((unsigned long long)kPhases * gridDim.x);
}
__device__ __forceinline__ uint32_t launch_tag(unsigned long long index) {
  return (uint32_t)index | 0x80000000u;
}

struct Phases {
  unsigned long long* ctr;
  unsigned long long base;  // kPhases * gridDim.x * launch index
  int* err;
};

// Every thread of the CTA calls it, after its writes of the phase.
__device__ __forceinline__ void phase_arrive(const Phases& ph) {
  __syncthreads();
  if (threadIdx.x == 0) red_add_u64(ph.ctr, 1ull);
}

// Every thread of the CTA calls it; bounded (wait_more).
__device__ __forceinline__ void phase_wait(const Phases& ph, int j) {
  if (threadIdx.x == 0) {
    const unsigned long long target = ph.base + (unsigned long long)(j + 1) * gridDim.x;
    const long long t0 = clock64();
    while (ld_relaxed_u64(ph.ctr) < target && wait_more(t0, ph.err)) {
    }
  }
  __syncthreads();
}

// Orders earlier generic-proxy accesses of this CTA's shared memory before
// later bulk-copy (async-proxy) writes to the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace prox
