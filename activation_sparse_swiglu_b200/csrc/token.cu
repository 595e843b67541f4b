// The fused per-token kernel of the Prox decode step: one launch runs the
// whole step of one token (Prox §4.1) on all SMs, one CTA per SM:
//
//   Stage 1 (stage1.cuh): threshold x, INT4 proxy GEMV over the kept rows
//            into per-CTA partial sums, written as tagged words;
//   scores:  each CTA adds up the partials of its own share of the channels
//            (polling until each has arrived) and scores them,
//            |act(g~) u~|, counting them for the top-k rule in the
//            histograms of select.cuh;
//   Stage 2 (stage2.cuh): each CTA finds the token's exact top-k cut once
//            the histograms are complete (or applies the score threshold),
//            lists its own channels past it with their count, then takes an
//            even share of the token's ranked selection (or of a given list,
//            or of every channel for the dense baseline), streams those
//            channel records and W_down rows and writes a tagged partial
//            output row;
//   output:  CTA c adds the partial rows of its share of the columns in a
//            fixed order (deterministic).
//
// The CTAs never wait at a grid-wide barrier: whatever one CTA hands to
// another is a tagged word (token_args.cuh) that the reader polls for, and
// counts are complete when they add up to a known total.  The launch is
// cooperative (every CTA resident, so every wait ends) and programmatically
// dependent on the previous kernel in the stream: it waits for it before
// touching x or the workspace, then lets the next one launch.  Every wait is
// bounded and reports a timeout in the layer's error word; every CTA adds one
// to the layer's launch counter as it ends, which gives the next launch its
// tag and its histogram parity.
#include "prox_device.cuh"
#include "prox_internal.h"
#include "stage1.cuh"
#include "stage2.cuh"

namespace prox {
namespace {

// The CTA's share of the output: the column pairs [q0, q1) of out.  Warp w
// takes the partial rows p = w, w + W, ... (W warps), lane l the pairs
// q0 + l, q0 + l + 32, ...: a warp's loads of one row are one contiguous
// stretch, all of them in flight at once (kRowChunk rows per round) and
// polled until every tag is this launch's.  Each lane adds its rows in
// order; the warps' sums are then added in warp order (deterministic).
constexpr int kRowChunk = 9;
__device__ void reduce_output(const TokenArgs& a, uint32_t tag, unsigned char* smem) {
  const int P = gridDim.x, nq = a.d >> 1, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NW = kTokenThreads / 32;
  const int q0 = (int)(((long long)nq * blockIdx.x) / P);
  const int q1 = (int)(((long long)nq * (blockIdx.x + 1)) / P);
  const int nqc = q1 - q0;
  float2* s_sum = reinterpret_cast<float2*>(smem);  // [NW][nqc]
  for (int l = lane; l < ((nqc + 31) & ~31); l += 32) {
    const bool col = l < nqc;
    float2 acc = make_float2(0.f, 0.f);
    for (int p0 = warp; p0 < P; p0 += NW * kRowChunk) {
      ulonglong2 v[kRowChunk];
      const unsigned long long zero = tag_word(0u, tag);  // rows past P add 0
#pragma unroll
      for (int i = 0; i < kRowChunk; ++i) {
        const int p = p0 + i * NW;
        v[i] = col && p < P ? ld_tag2(a.ypart + (size_t)p * a.d + 2 * (q0 + l)) : make_ulonglong2(zero, zero);
      }
      const long long t0 = clock64();
      for (;;) {
        bool all = true;
#pragma unroll
        for (int i = 0; i < kRowChunk; ++i) all = all && tag_ok(v[i].x, tag) && tag_ok(v[i].y, tag);
        if (all || !wait_more(t0, a.err)) break;
#pragma unroll
        for (int i = 0; i < kRowChunk; ++i) {
          const int p = p0 + i * NW;
          if (col && p < P && !(tag_ok(v[i].x, tag) && tag_ok(v[i].y, tag)))
            v[i] = ld_tag2(a.ypart + (size_t)p * a.d + 2 * (q0 + l));
        }
      }
#pragma unroll
      for (int i = 0; i < kRowChunk; ++i) {
        acc.x += __uint_as_float((uint32_t)v[i].x);
        acc.y += __uint_as_float((uint32_t)v[i].y);
      }
    }
    if (col) s_sum[warp * nqc + l] = acc;
  }
  __syncthreads();
  stamp(a.ts, 6);
  for (int l = threadIdx.x; l < nqc; l += blockDim.x) {
    float2 t = s_sum[l];
    for (int w = 1; w < NW; ++w) {
      t.x += s_sum[w * nqc + l].x;
      t.y += s_sum[w * nqc + l].y;
    }
    reinterpret_cast<float2*>(a.out)[q0 + l] = t;
  }
}

template <int MAXM>
__global__ void __launch_bounds__(kTokenThreads, 1) token_kernel(TokenArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  stamp_timer(a.ts, 0, 22);
  pdl_wait();     // the previous kernel of the stream is complete: x and the workspace are ours
  pdl_trigger();  // the next kernel may launch (it waits for this one before touching anything)
  // The launch counter (every thread reads it: the dynamic shared memory
  // belongs to the phases).  Its value is first needed when Stage 1 writes
  // its partials, so the load overlaps Stage 1's start.
  const unsigned long long gv = ld_relaxed_u64(a.gbar);
  stamp(a.ts, 1);
  const bool topk = a.mode == kModeTopK;
  // the launch index (Stage 1 works it out when it first needs the tag)
  const unsigned long long e = a.stage1 ? s1::run(a, smem, gv) : launch_index(gv);
  const uint32_t tag = launch_tag(e);
  const int par = (int)(e & 1ull);
  const Phases ph{a.gbar, e * kPhases * gridDim.x, a.err};
  {
    // clear the histograms of the other parity for the next launch
    uint32_t* nh = a.hist + (size_t)(par ^ 1) * kScoreBins;
    const int b0 = (int)(((long long)kScoreBins * blockIdx.x) / gridDim.x);
    const int b1 = (int)(((long long)kScoreBins * (blockIdx.x + 1)) / gridDim.x);
    for (int i = b0 + threadIdx.x; i < b1; i += blockDim.x) nh[i] = 0u;
    if (blockIdx.x == 0 && threadIdx.x < kCoarseBins) a.chist[(par ^ 1) * kCoarseBins + threadIdx.x] = 0u;
  }
  uint32_t* hist = a.hist + (size_t)par * kScoreBins;
  uint32_t* chist = a.chist + par * kCoarseBins;
  if (a.stage1) {
    phase_arrive(ph);  // 0: partials written
    stamp(a.ts, 2);
    phase_wait(ph, 0);
    stamp(a.ts, 16);
    SelectScratch& sc = *reinterpret_cast<SelectScratch*>(smem + s2::ring_offset(a.slots, a.max_rec));
    s1::score_channels(a, topk, sc, tag, hist, chist);
    phase_arrive(ph);  // 1: scores counted
    stamp(a.ts, 10);
  } else {
    phase_arrive(ph);
    phase_arrive(ph);
  }
  bool rows = false;
  if (a.mode != kModeNone) {
    rows = s2::run<MAXM>(a, smem, tag, hist, chist, ph);  // arrives at phase 2
    stamp(a.ts, 5);
  } else {
    phase_arrive(ph);
  }
  phase_arrive(ph);  // 3: partial output rows written
  if (rows) {
    phase_wait(ph, 3);
    stamp(a.ts, 19);
    reduce_output(a, tag, smem);
    stamp(a.ts, 7);
  }
  stamp_timer(a.ts, 21, 23);
}

// Test probe of the bounded waits: one CTA adds 1 to the layer's launch
// counter and waits for a second addition that never comes.
__global__ void barrier_probe_kernel(unsigned long long* gbar, int* err) {
  const unsigned long long v = ld_relaxed_u64(gbar);
  const Phases ph{gbar, v, err};
  phase_arrive(ph);
  phase_wait(ph, 1);
}

template <int MAXM>
cudaError_t set_attr() {
  return cudaFuncSetAttribute(token_kernel<MAXM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kMaxSmemPerBlock);
}

cudaError_t launch_maxm(const cudaLaunchConfig_t& cfg, int maxm, const TokenArgs& a) {
  if (maxm <= 1) return cudaLaunchKernelEx(&cfg, token_kernel<1>, a);
  if (maxm == 2) return cudaLaunchKernelEx(&cfg, token_kernel<2>, a);
  if (maxm == 3) return cudaLaunchKernelEx(&cfg, token_kernel<3>, a);
  return cudaLaunchKernelEx(&cfg, token_kernel<4>, a);
}

}  // namespace

void choose_stage1_grid(int d, int F, int num_sms, int* C, int* lmax, int* depth) {
  *C = (F + s1::SLICE - 1) / s1::SLICE;
  // a CTA's share of the C * n_x pairs, n_x <= d
  *lmax = (int)(((long long)(*C) * d + num_sms - 1) / num_sms) + 1;
  // as many k-tiles in flight per warp as the shared memory left by the
  // tables holds, at most kMaxDepth
  const size_t tables = s1::layout(0, *lmax, d).total;
  const long long room = (long long)kMaxSmemPerBlock - (long long)tables;
  long long k = room > 0 ? room / ((long long)s1::NW * s1::WSLOT) : 0;
  if (k > s1::kMaxDepth) k = s1::kMaxDepth;
  *depth = (int)k;
}

size_t stage1_smem_bytes(int lmax, int depth, int d) { return s1::layout(depth, lmax, d).total; }

size_t stage1_part_floats(int P) { return (size_t)P * 2 * s1::PART; }

void choose_stage2(int d, int F, int num_sms, int* slots, int* groups, size_t* smem) {
  const int max_rec = (F + num_sms - 1) / num_sms + 1;
  const size_t slot_bytes = 4 * (size_t)d;  // gate + up column, or two W_down rows
  const size_t off0 = s2::ring_offset(0, max_rec) + 16 * 32 + 128;
  int s = (int)((kStage2SmemBudget - off0) / (slot_bytes + 16));
  if (s > 32) s = 32;
  if (s < 2) s = 2;
  // Consumer groups: the most groups (4, 2, 1) whose slot share is at least
  // two and whose warps hold at most 4 chunks of 8 elements per lane.
  int ng = 1;
  for (int cand : {4, 2}) {
    const int wpg = kStage2Consumers / cand;
    const int maxm = (d + wpg * 256 - 1) / (wpg * 256);
    if ((s - s % cand) / cand >= 2 && maxm <= 4) {
      ng = cand;
      break;
    }
  }
  s -= s % ng;
  *groups = ng;
  *slots = s;
  size_t region = (size_t)s * slot_bytes;
  if (region < select_smem_bytes(F)) region = select_smem_bytes(F);  // the selection's scratch and keys
  if (region < (size_t)ng * d * 4) region = (size_t)ng * d * 4;       // the groups' partial rows
  *smem = s2::ring_offset(s, max_rec) + region;
}

int stage2_maxm(int d, int groups) {
  const int wpg = kStage2Consumers / groups;
  return (d + wpg * 256 - 1) / (wpg * 256);
}

cudaError_t setup_token_kernels() {
  cudaError_t e;
  if ((e = set_attr<1>()) != cudaSuccess) return e;
  if ((e = set_attr<2>()) != cudaSuccess) return e;
  if ((e = set_attr<3>()) != cudaSuccess) return e;
  return set_attr<4>();
}

cudaError_t launch_barrier_probe(const prox_layer* L, cudaStream_t s) {
  barrier_probe_kernel<<<1, 32, 0, s>>>(L->ws.gbar, L->ws.err);
  return cudaGetLastError();
}

cudaError_t launch_token(const prox_layer* L, const TokenLaunch& m, cudaStream_t s, bool pdl) {
  TokenArgs a;
  a.x = m.x;
  a.out = m.out;
  a.pq = L->pq;
  a.ps = reinterpret_cast<const __half*>(L->ps);
  a.wgu = L->wgu;
  a.wd = L->wd;
  a.d = L->d;
  a.F = L->F;
  a.C = L->C;
  a.lmax = L->s1_lmax;
  a.s1_depth = L->s1_depth;
  a.tau = L->tau;
  a.slots = L->ring_slots;
  a.groups = L->stage2_groups;
  a.max_rec = (L->F + L->P - 1) / L->P + 1;
  a.stage1 = m.stage1 ? 1 : 0;
  a.mode = m.mode;
  a.select_only = m.select_only ? 1 : 0;
  a.proxy_values = m.proxy_values ? 1 : 0;
  a.act = L->act;
  a.k = m.k;
  a.tau_s = m.tau_s;
  a.idx = m.idx;
  a.scores = L->ws.scores;
  a.s_tilde = m.taps.s_tilde ? m.taps.s_tilde : (m.proxy_values ? L->ws.s_tilde : nullptr);
  a.hist = L->ws.hist;
  a.chist = L->ws.chist;
  a.bucket = L->ws.bucket;
  a.sel_list = L->ws.sel_list;
  a.sel_cnt = L->ws.sel_cnt;
  a.st64 = L->ws.st64;
  a.stats = L->ws.stats;
  a.part = L->ws.s1_part;
  a.ypart = L->ws.ypart;
  a.gbar = L->ws.gbar;
  a.err = L->ws.err;
  a.g_dbg = m.taps.g;
  a.u_dbg = m.taps.u;
  a.idx_x = m.taps.idx_x;
  a.n_x = m.taps.n_x;
  a.sel_mask = m.sel_mask;
  a.s_sp = m.s_sp;
  a.ts = m.phase_ns;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L->P, 1, 1);
  cfg.blockDim = dim3(kTokenThreads, 1, 1);
  cfg.dynamicSmemBytes = L->token_smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const int maxm = stage2_maxm(L->d, L->stage2_groups);
  return launch_maxm(cfg, maxm, a);
}

}  // namespace prox
