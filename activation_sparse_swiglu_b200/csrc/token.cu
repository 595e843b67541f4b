// The fused per-token kernel of the Prox decode step: one launch runs the
// whole step of one token (Prox §4.1) on all SMs, one CTA per SM, with
// grid-wide barriers between the phases instead of kernel boundaries:
//
//   Stage 1 (stage1.cuh): threshold x, INT4 proxy GEMV over the kept rows
//            into per-CTA partial sums;
//   barrier: every partial sum is written;
//   scores:  each CTA adds up the partials of its own share of the channels
//            and scores them, |act(g~) u~| (for the top-k rule counting them
//            in the histograms of select.cuh);
//   barrier: (top-k) the histograms are complete;
//   Stage 2 (stage2.cuh): each CTA finds the token's exact top-k cut (or
//            applies the score threshold) and lists its own channels past it;
//   barrier: (top-k, threshold) every CTA's list and count is written;
//            each CTA then takes an even share of the token's ranked
//            selection (or of a given list, or of every channel for the
//            dense baseline), streams those channel records and W_down rows
//            and writes a partial output row;
//   barrier: every partial row is complete;
//   output:  CTA c adds the partial rows of its share of the columns in a
//            fixed order (deterministic).
//
// The launch is cooperative (all CTAs resident, which the barriers need) and
// programmatically dependent on the previous kernel in the stream: it waits
// for it before touching x or the workspace, then lets the next one launch.
// Every wait (barrier, mbarrier) is bounded and reports a timeout in the
// layer's error word.
#include "prox_device.cuh"
#include "prox_internal.h"
#include "stage1.cuh"
#include "stage2.cuh"

namespace prox {
namespace {

template <int NB, int MAXM>
__global__ void __launch_bounds__(kTokenThreads, 1) token_kernel(TokenArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  stamp(a.ts, 0);
  pdl_wait();     // the previous kernel of the stream is complete: x and the workspace are ours
  pdl_trigger();  // the next kernel may launch (it waits for this one before touching anything)
  GridSync gs = grid_sync_begin(a.gbar);
  stamp(a.ts, 1);
  const bool topk = a.mode == kModeTopK;
  if (a.stage1) {
    s1::run<NB>(a, smem);
    stamp(a.ts, 2);
    grid_barrier(gs, gridDim.x, a.err);  // every CTA's Stage-1 partials are written
    stamp(a.ts, 3);
    SelectScratch& sc = *reinterpret_cast<SelectScratch*>(smem + s2::ring_offset(a.slots, a.max_rec));
    s1::score_channels(a, topk, sc);
    stamp(a.ts, 10);
    if (a.mode == kModeNone) return;
    if (topk) {
      grid_barrier(gs, gridDim.x, a.err);  // the histograms and buckets are complete
      stamp(a.ts, 14);
    }
  }
  if (a.mode == kModeNone) return;
  s2::run<MAXM>(a, smem, gs);
  stamp(a.ts, 5);
  grid_barrier(gs, gridDim.x, a.err);  // every partial row is written; every CTA is past the cut
  stamp(a.ts, 6);
  if (a.stage1 && topk && blockIdx.x == gridDim.x - 1) {  // ready for the next token
    for (int i = threadIdx.x; i < kScoreBins; i += blockDim.x) a.hist[i] = 0u;
    if (threadIdx.x < kCoarseBins) a.chist[threadIdx.x] = 0u;
  }
  if (a.select_only) return;

  // out[4q .. 4q+3] for the float4 columns q of this CTA: warp w sums column
  // q over the partial rows p = lane, lane + 32, ... in order (all loads in
  // flight at once), then across lanes by a fixed shuffle tree.
  const int P = gridDim.x, nq = a.d >> 2, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = (int)(((long long)nq * blockIdx.x) / P);
  const int q1 = (int)(((long long)nq * (blockIdx.x + 1)) / P);
  const float4* yp = reinterpret_cast<const float4*>(a.ypart);
  for (int q = q0 + warp; q < q1; q += kTokenThreads / 32) {
    float4 v[kMaxCtas / 32];
#pragma unroll
    for (int u = 0; u < kMaxCtas / 32; ++u) {
      const int p = lane + 32 * u;
      v[u] = p < P ? __ldcg(yp + (size_t)p * nq + q) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float4 s = v[0];
#pragma unroll
    for (int u = 1; u < kMaxCtas / 32; ++u) {
      s.x += v[u].x;
      s.y += v[u].y;
      s.z += v[u].z;
      s.w += v[u].w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s.x += __shfl_xor_sync(0xffffffffu, s.x, o);
      s.y += __shfl_xor_sync(0xffffffffu, s.y, o);
      s.z += __shfl_xor_sync(0xffffffffu, s.z, o);
      s.w += __shfl_xor_sync(0xffffffffu, s.w, o);
    }
    if (lane == 0) reinterpret_cast<float4*>(a.out)[q] = s;
  }
  stamp(a.ts, 7);
}

// Test probe of the bounded waits: one CTA arrives at the layer's grid
// barrier expecting one more arrival that never comes, so its wait runs out,
// sets PROX_DEVERR_WAIT_TIMEOUT and returns.  Nothing faults.
__global__ void barrier_probe_kernel(unsigned long long* gbar, int* err) {
  GridSync gs = grid_sync_begin(gbar);
  grid_barrier(gs, gridDim.x + 1, err);
}

template <int NB>
size_t stage1_smem(int lmax) {
  return s1::smem_bytes<NB>(lmax);
}

template <int NB, int MAXM>
cudaError_t set_attr() {
  return cudaFuncSetAttribute(token_kernel<NB, MAXM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kMaxSmemPerBlock);
}

template <int NB>
cudaError_t set_attrs_nb() {
  cudaError_t e;
  if ((e = set_attr<NB, 1>()) != cudaSuccess) return e;
  if ((e = set_attr<NB, 2>()) != cudaSuccess) return e;
  if ((e = set_attr<NB, 3>()) != cudaSuccess) return e;
  return set_attr<NB, 4>();
}

template <int NB>
cudaError_t launch_nb(const cudaLaunchConfig_t& cfg, int maxm, const TokenArgs& a) {
  if (maxm <= 1) return cudaLaunchKernelEx(&cfg, token_kernel<NB, 1>, a);
  if (maxm == 2) return cudaLaunchKernelEx(&cfg, token_kernel<NB, 2>, a);
  if (maxm == 3) return cudaLaunchKernelEx(&cfg, token_kernel<NB, 3>, a);
  return cudaLaunchKernelEx(&cfg, token_kernel<NB, 4>, a);
}

}  // namespace

void choose_stage1_grid(int d, int F, int num_sms, int* C, int* lmax, int* nb) {
  *C = (F + s1::SLICE - 1) / s1::SLICE;
  // a CTA's share of the C * n_x pairs, n_x <= d
  *lmax = (int)(((long long)(*C) * d + num_sms - 1) / num_sms) + 1;
  // four batches in flight per warp when they fit, else three, else two
  *nb = 4;
  if (s1::smem_bytes<4>(*lmax) > (size_t)kMaxSmemPerBlock) *nb = 3;
  if (s1::smem_bytes<3>(*lmax) > (size_t)kMaxSmemPerBlock) *nb = 2;
}

size_t stage1_smem_bytes(int lmax, int nb) {
  return nb == 4 ? stage1_smem<4>(lmax) : nb == 3 ? stage1_smem<3>(lmax) : stage1_smem<2>(lmax);
}

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
  if ((e = set_attrs_nb<4>()) != cudaSuccess) return e;
  if ((e = set_attrs_nb<3>()) != cudaSuccess) return e;
  return set_attrs_nb<2>();
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
  a.s_tilde_src = L->ws.s_tilde;
  a.hist = L->ws.hist;
  a.chist = L->ws.chist;
  a.bucket = L->ws.bucket;
  a.sel_list = L->ws.sel_list;
  a.sel_cnt = L->ws.sel_cnt;
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
  a.mg = Magic{0x4B000000u, 0x49000000u, 0x47000000u, 0x45000000u, 0x43000000u};

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
  if (L->s1_nb == 4) return launch_nb<4>(cfg, maxm, a);
  if (L->s1_nb == 3) return launch_nb<3>(cfg, maxm, a);
  return launch_nb<2>(cfg, maxm, a);
}

}  // namespace prox
