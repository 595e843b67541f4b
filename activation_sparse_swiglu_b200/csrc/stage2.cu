// Stage 2 of the Prox decode step (Prox §4.1 "Stage 2: exact sparse
// computation"; §4.3 fused output-sparse gate/up kernel and input-sparse
// down GEMV), and the dense SwiGLU baseline (Prox §2.1), which is the same
// kernel with every channel kept.
//
// stage2_kernel -- persistent: one CTA per SM, each CTA owning the channels
// [c0, c1) of an even split of d_ff.  In top-k mode every CTA computes the
// exact cut of the token (select.cuh: T and the tie cut, from the Stage-1
// histogram and the boundary bin's bucket) and keeps the channels of its range
// past the cut; with a given list it keeps the list's channels in its range;
// the dense baseline keeps all of them.  The uneven record counts this leaves
// are absorbed by the deep ring (each SM may stream above its average share).
// Four producer lanes stream, with 1-D bulk async copies (TMA engine) into a
// ring of 16 KB-class shared-memory slots, first the gate/up channel records of its channels (gate column then
// up column, d_model bf16 each: one copy per channel), then their W_down rows
// (two rows per slot).  Eight consumer warps take every ring item in order (so
// each mbarrier wait is for the phase right after one the waiting thread has
// already seen complete):
//   phase A: for each channel every warp forms partial dot products of its
//            share of the column with the full x (x kept in registers; fp32,
//            packed f32x2 FMAs, warp-shuffle reduction) and parks them in
//            shared memory; after the last channel the partials are summed in
//            a fixed order into g = x . W_gate[:, j], u = x . W_up[:, j] and
//            s_j = SiLU(g) u;
//   phase B: all warps accumulate y_part += s_j W_down[j, :] for the CTA's
//            channels, each thread owning 8-column groups of the output.
// Each CTA writes its fp32 partial y; reduce_kernel sums the partials in a
// fixed order (deterministic, no atomics on floats).
#include "prox_device.cuh"
#include "prox_internal.h"
#include "select.cuh"

namespace prox {
namespace {

constexpr int NCW = kStage2Consumers;
constexpr int S2_THREADS = (NCW + 1) * 32;
constexpr size_t kStage2SmemBudget = 208 * 1024;

enum Stage2Mode { kGivenList = 0, kTopK = 1, kDense = 2 };

struct Stage2Args {
  const float* x;
  const uint16_t* wgu;
  const uint16_t* wd;
  const int32_t* idx;      // kGivenList: channel list [k]
  const float* scores;     // kTopK: Stage-1 scores [F]
  const uint32_t* hist;    // kTopK: Stage-1 histogram of the scores' bits 30..20
  unsigned long long* stats;
  const uint2* bucket;     // kTopK: Stage-1 (key, channel) buckets per histogram bin
  int32_t* sel_mask;       // kTopK: 1/0 per channel (debug)
  int mode, select_only;
  int k;
  int d, F, P, slots, max_rec;
  int nprod;  // producer lanes; slots is a multiple of it
  float* ypart;
  float* s_sp;
  int* err;
  int x_ready;
};

// MAXM = ceil(d_model / 2048): 8-element chunks per thread and column.
template <int MAXM>
__global__ void __launch_bounds__(S2_THREADS, 1) stage2_kernel(Stage2Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int d = a.d, slots = a.slots;
  const uint32_t col_bytes = 2u * (uint32_t)d;     // one bf16 column / row
  const uint32_t slot_bytes = 2u * col_bytes;      // a gate/up record, or two W_down rows
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + slots;
  float* s_val = reinterpret_cast<float*>(empty + slots);        // [max_rec]
  int* s_idx = reinterpret_cast<int*>(s_val + a.max_rec);        // [max_rec]
  float* s_pg = reinterpret_cast<float*>(s_idx + a.max_rec);     // [max_rec][NCW]
  float* s_pu = s_pg + (size_t)a.max_rec * NCW;                  // [max_rec][NCW]
  int* s_lpos = reinterpret_cast<int*>(s_pu + (size_t)a.max_rec * NCW);  // [max_rec]
  size_t off = (size_t)slots * 16 + (size_t)a.max_rec * (12 + 8 * NCW);
  off = (off + 127) & ~(size_t)127;
  unsigned char* ring = smem + off;

  if (tid == 0) {
    for (int s = 0; s < slots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    fence_barrier_init();
  }
  // this thread's share of x (chunks c8 = tid + 256 m), kept in registers
  float4 xr[MAXM][2];
  if (a.x_ready && warp < NCW) {
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int e = (tid + m * NCW * 32) * 8;
      xr[m][0] = e < d ? __ldg(reinterpret_cast<const float4*>(a.x + e)) : make_float4(0, 0, 0, 0);
      xr[m][1] = e < d ? __ldg(reinterpret_cast<const float4*>(a.x + e + 4)) : make_float4(0, 0, 0, 0);
    }
  }
  __syncthreads();

  pdl_wait();
  pdl_trigger();

  if (!a.x_ready && warp < NCW) {
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int e = (tid + m * NCW * 32) * 8;
      xr[m][0] = e < d ? __ldg(reinterpret_cast<const float4*>(a.x + e)) : make_float4(0, 0, 0, 0);
      xr[m][1] = e < d ? __ldg(reinterpret_cast<const float4*>(a.x + e + 4)) : make_float4(0, 0, 0, 0);
    }
  }
  const int k = a.mode == kDense ? a.F : a.k;
  const int cta = blockIdx.x;
  int t0 = 0, n = 0;
  if (a.mode == kTopK) {
    // This CTA's channels are [c0, c1); those past the exact cut are its records.
    const int c0 = (int)(((long long)a.F * cta) / a.P);
    const int c1 = (int)(((long long)a.F * (cta + 1)) / a.P);
    SelectScratch& sc = *reinterpret_cast<SelectScratch*>(ring);
    const uint32_t key0 = c0 + tid < c1 ? __float_as_uint(__ldcg(a.scores + c0 + tid)) : 0u;
    const TopkCut cut = select_cut_cta(a.scores, a.hist, a.bucket, a.F, a.k, sc);
    for (int b = c0; b < c1; b += S2_THREADS) {
      const int e = b + tid;
      const uint32_t key =
          b == c0 ? key0 : (e < c1 ? __float_as_uint(__ldcg(a.scores + e)) : 0u);
      const bool sel = e < c1 && selected(key, e, cut);
      int total;
      const int pos = n + block_exclusive_scan(sel ? 1 : 0, sc.scan, &total);
      if (sel) s_idx[pos] = e;
      if (a.sel_mask && e < c1) a.sel_mask[e] = sel ? 1 : 0;
      n += total;
    }
    if (cta == 0 && tid == 0 && a.stats) atomicAdd(a.stats + 1, 1ull);
    __syncthreads();
  } else if (a.mode == kGivenList) {
    // Entries of the list whose channel lies in [c0, c1), in list order -- the
    // same split of the channels as the top-k step, so that a sorted list
    // reproduces it exactly.  Thread t scans entries [t*per, (t+1)*per).
    const int c0 = (int)(((long long)a.F * cta) / a.P);
    const int c1 = (int)(((long long)a.F * (cta + 1)) / a.P);
    const int per = (k + S2_THREADS - 1) / S2_THREADS;
    const int lo = min(tid * per, k), hi = min(lo + per, k);
    int cnt = 0;
    for (int i = lo; i < hi; ++i) {
      const int j = __ldcg(a.idx + i);
      if (j < 0 || j >= a.F) atomicOr(a.err, PROX_DEVERR_MASK_INDEX);
      cnt += j >= c0 && j < c1;
    }
    int total;
    int pos = block_exclusive_scan(cnt, reinterpret_cast<SelectScratch*>(ring)->scan, &total);
    for (int i = lo; i < hi; ++i) {
      const int j = __ldcg(a.idx + i);
      if (j >= c0 && j < c1) {
        if (pos < a.max_rec) {  // more only with repeated channels
          s_lpos[pos] = i;      // list position (for s_sp)
          s_idx[pos] = j;
        } else {
          atomicOr(a.err, PROX_DEVERR_MASK_INDEX);
        }
        ++pos;
      }
    }
    n = min(total, a.max_rec);
    __syncthreads();
  } else {
    t0 = (int)(((long long)k * cta) / a.P);
    n = (int)(((long long)k * (cta + 1)) / a.P) - t0;
    for (int i = tid; i < n; i += S2_THREADS) s_idx[i] = t0 + i;
    __syncthreads();
  }
  if (a.select_only) return;

  // Ring items q = 0 .. nA + nB - 1: q < n is the gate/up record of channel q;
  // q >= n holds W_down rows 2(q-n) and 2(q-n)+1.  Item q lives in slot
  // q % slots as that slot's use q / slots.
  const int nB = (n + 1) >> 1;
  const int total = n + nB;
  bool dead = false;  // set once a wait of this thread ran out
  if (warp == NCW) {
    // ---------------- producer lanes 0..nprod-1: lane l issues items q = l + j*nprod.
    // slots is a multiple of nprod, so every slot is refilled by one lane, in order.
    const int np = a.nprod;
    if (lane < np && lane < total) {
      const uint64_t pol = l2_policy_evict_first();
      int q = lane;
      int slot = q % slots;
      int use = q / slots;
      for (; q < total; q += np) {
        if (use > 0) mbar_wait(&empty[slot], (uint32_t)((use - 1) & 1), a.err, &dead);
        unsigned char* dst = ring + (size_t)slot * slot_bytes;
        if (q < n) {
          mbar_arrive_expect_tx(&full[slot], slot_bytes);
          bulk_copy_g2s(dst, a.wgu + (size_t)s_idx[q] * 2 * (size_t)d, slot_bytes, &full[slot], pol);
        } else {
          const int r0 = 2 * (q - n);
          const int nr = r0 + 1 < n ? 2 : 1;
          mbar_arrive_expect_tx(&full[slot], (uint32_t)nr * col_bytes);
          bulk_copy_g2s(dst, a.wd + (size_t)s_idx[r0] * (size_t)d, col_bytes, &full[slot], pol);
          if (nr == 2)
            bulk_copy_g2s(dst + col_bytes, a.wd + (size_t)s_idx[r0 + 1] * (size_t)d, col_bytes,
                          &full[slot], pol);
        }
        slot += np;
        while (slot >= slots) {
          slot -= slots;
          ++use;
        }
      }
      // Every issued copy must land before this CTA's shared memory is released:
      // wait for the last use of each slot this lane filled.
      for (int s2 = 0; s2 < slots; ++s2) {
        int last = -1;  // last item of this lane in slot s2
        for (int qq = s2; qq < total; qq += slots)
          if (qq % np == lane) last = qq;
        if (last >= 0) mbar_wait(&full[s2], (uint32_t)((last / slots) & 1), a.err);
      }
    }
    return;
  }

  int cs = 0;        // consumer: slot of the next item
  uint32_t cp = 0;   // and the parity of its use

  // ---------------- phase A: partial gate/up dot products ----------------
  // Records are taken RB at a time so that the 2*RB warp reductions of a batch
  // run interleaved.
  constexpr int RB = 4;
  const int rbn = slots < RB ? slots : RB;  // a batch never holds more than the ring
  for (int r0 = 0; r0 < n; r0 += rbn) {
    int sl[RB];
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      sl[b] = cs;
      if (b < rbn && r0 + b < n) {
        mbar_wait(&full[cs], cp, a.err, &dead);
        if (++cs == slots) { cs = 0; cp ^= 1u; }
      }
    }
    float g[RB], u[RB];
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      float2 ag = make_float2(0.f, 0.f), au = make_float2(0.f, 0.f);
      if (b < rbn && r0 + b < n) {
        const unsigned char* wg = ring + (size_t)sl[b] * slot_bytes;
        const unsigned char* wu = wg + col_bytes;
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
          const int e = (tid + m * NCW * 32) * 8;
          if (e < d) {
            const uint4 g4 = *reinterpret_cast<const uint4*>(wg + (size_t)e * 2);
            const uint4 u4 = *reinterpret_cast<const uint4*>(wu + (size_t)e * 2);
            const float4 xa = xr[m][0], xb = xr[m][1];
            ag = __ffma2_rn(bf16x2_to_f2(g4.x), make_float2(xa.x, xa.y), ag);
            au = __ffma2_rn(bf16x2_to_f2(u4.x), make_float2(xa.x, xa.y), au);
            ag = __ffma2_rn(bf16x2_to_f2(g4.y), make_float2(xa.z, xa.w), ag);
            au = __ffma2_rn(bf16x2_to_f2(u4.y), make_float2(xa.z, xa.w), au);
            ag = __ffma2_rn(bf16x2_to_f2(g4.z), make_float2(xb.x, xb.y), ag);
            au = __ffma2_rn(bf16x2_to_f2(u4.z), make_float2(xb.x, xb.y), au);
            ag = __ffma2_rn(bf16x2_to_f2(g4.w), make_float2(xb.z, xb.w), ag);
            au = __ffma2_rn(bf16x2_to_f2(u4.w), make_float2(xb.z, xb.w), au);
          }
        }
      }
      g[b] = ag.x + ag.y;
      u[b] = au.x + au.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        g[b] += __shfl_xor_sync(0xffffffffu, g[b], o);
        u[b] += __shfl_xor_sync(0xffffffffu, u[b], o);
      }
    }
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        if (b < rbn && r0 + b < n) {
          mbar_arrive(&empty[sl[b]], 1);
          s_pg[(r0 + b) * NCW + warp] = g[b];
          s_pu[(r0 + b) * NCW + warp] = u[b];
        }
      }
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
  for (int r = tid; r < n; r += NCW * 32) {
    float g = 0.f, u = 0.f;
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
      g += s_pg[r * NCW + w];
      u += s_pu[r * NCW + w];
    }
    const float sv = silu_f32(g) * u;
    s_val[r] = sv;
    if (a.s_sp) a.s_sp[a.mode == kGivenList ? s_lpos[r] : t0 + r] = sv;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");

  // ---------------- phase B: y_part = sum_t s_t W_down[j_t, :] ----------------
  // Items (two rows each) are taken two at a time.
  float2 acc[MAXM * 4];
#pragma unroll
  for (int i = 0; i < MAXM * 4; ++i) acc[i] = make_float2(0.f, 0.f);
  for (int rb0 = 0; rb0 < nB; rb0 += 2) {
    int sl[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      sl[b] = cs;
      if (rb0 + b < nB) {
        mbar_wait(&full[cs], cp, a.err, &dead);
        if (++cs == slots) { cs = 0; cp ^= 1u; }
      }
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int rr = 2 * rb0 + h;  // W_down row (channel slot) of this CTA
      if (rr < n) {
        const float sv = s_val[rr];
        const float2 s2 = make_float2(sv, sv);
        const unsigned char* w = ring + (size_t)sl[h >> 1] * slot_bytes + (h & 1) * col_bytes;
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
          const int e = tid * 8 + m * (NCW * 32 * 8);
          if (e < d) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(w + (size_t)e * 2);
            acc[4 * m + 0] = __ffma2_rn(bf16x2_to_f2(w4.x), s2, acc[4 * m + 0]);
            acc[4 * m + 1] = __ffma2_rn(bf16x2_to_f2(w4.y), s2, acc[4 * m + 1]);
            acc[4 * m + 2] = __ffma2_rn(bf16x2_to_f2(w4.z), s2, acc[4 * m + 2]);
            acc[4 * m + 3] = __ffma2_rn(bf16x2_to_f2(w4.w), s2, acc[4 * m + 3]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&empty[sl[0]], 1);
      if (rb0 + 1 < nB) mbar_arrive(&empty[sl[1]], 1);
    }
  }
  float* dst = a.ypart + (size_t)cta * d;
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    const int e = tid * 8 + m * (NCW * 32 * 8);
    if (e < d) {
      *reinterpret_cast<float4*>(dst + e) =
          make_float4(acc[4 * m].x, acc[4 * m].y, acc[4 * m + 1].x, acc[4 * m + 1].y);
      *reinterpret_cast<float4*>(dst + e + 4) =
          make_float4(acc[4 * m + 2].x, acc[4 * m + 2].y, acc[4 * m + 3].x, acc[4 * m + 3].y);
    }
  }
}

// out[c] = sum_p ypart[p][c]: warp w sums partials p = w, w + W, ... (all its
// loads in flight at once), then the warps' sums are added in warp order.
__global__ void __launch_bounds__(kReduceWarps * 32) reduce_kernel(const float* ypart, int P, int d,
                                                                   float* out, uint32_t* hist) {
  __shared__ float s_part[kReduceWarps][32];
  pdl_wait();
  pdl_trigger();
  // Stage 2 is complete: clear the level-1 histogram for the next token.
  if (hist && blockIdx.x == 0)
    for (int i = threadIdx.x; i < kScoreBins; i += blockDim.x) hist[i] = 0u;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (col < d) {
    for (int p0 = warp; p0 < P; p0 += 16 * kReduceWarps) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int p = p0 + u * kReduceWarps;
        v[u] = p < P ? __ldcg(ypart + (size_t)p * d + col) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) s += v[u];
    }
  }
  s_part[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && col < d) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) t += s_part[w][lane];
    out[col] = t;
  }
}

template <int M>
cudaError_t launch_stage2_t(const cudaLaunchConfig_t& cfg, const Stage2Args& a) {
  return cudaLaunchKernelEx(&cfg, stage2_kernel<M>, a);
}

template <int M>
cudaError_t set_stage2_attr() {
  return cudaFuncSetAttribute(stage2_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kStage2SmemBudget + 16 * 1024);
}

}  // namespace

void choose_stage2(int d, int F, int num_sms, int* P, int* slots, int* nprod, size_t* smem) {
  *P = num_sms;
  const int max_rec = (F + num_sms - 1) / num_sms + 1;
  size_t off = (size_t)max_rec * (12 + 8 * NCW) + 128;
  const size_t slot_bytes = 4 * (size_t)d;  // gate + up column, or two W_down rows
  int s = (int)((kStage2SmemBudget - off) / (slot_bytes + 16));
  if (s > 32) s = 32;
  if (s < 2) s = 2;
  // producer lanes: the slot count must be a multiple of them
  if (s >= 8) {
    s -= s % 4;
    *nprod = 4;
  } else {
    s -= s % 2;
    *nprod = 2;
  }
  *slots = s;
  off = (size_t)s * 16 + (size_t)max_rec * (12 + 8 * NCW);
  off = (off + 127) & ~(size_t)127;
  size_t region = (size_t)s * slot_bytes;
  if (region < sizeof(SelectScratch)) region = sizeof(SelectScratch);  // the select's scratch
  *smem = off + region;
}

cudaError_t setup_stage2_kernels() {
  cudaError_t e;
  if ((e = set_stage2_attr<1>()) != cudaSuccess) return e;
  if ((e = set_stage2_attr<2>()) != cudaSuccess) return e;
  if ((e = set_stage2_attr<3>()) != cudaSuccess) return e;
  if ((e = set_stage2_attr<4>()) != cudaSuccess) return e;
  return set_stage2_attr<8>();
}

cudaError_t launch_stage2(const prox_layer* L, const float* x, const Stage2Launch& m,
                          cudaStream_t s, bool pdl, bool x_ready) {
  Stage2Args a;
  a.x = x;
  a.wgu = L->wgu;
  a.wd = L->wd;
  a.idx = m.idx;
  a.scores = L->ws.scores;
  a.hist = L->ws.hist;
  a.stats = L->ws.stats;
  a.bucket = L->ws.bucket;
  a.sel_mask = m.sel_mask;
  a.mode = m.mode;
  a.select_only = m.select_only ? 1 : 0;
  a.k = m.k;
  a.d = L->d;
  a.F = L->F;
  a.P = L->P;
  a.slots = L->ring_slots;
  a.nprod = L->stage2_producers;
  a.max_rec = (L->F + L->P - 1) / L->P + 1;
  a.ypart = L->ws.ypart;
  a.s_sp = m.s_sp;
  a.err = L->ws.err;
  a.x_ready = x_ready ? 1 : 0;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L->P, 1, 1);
  cfg.blockDim = dim3(S2_THREADS, 1, 1);
  cfg.dynamicSmemBytes = L->stage2_smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int mm = (L->d + 2047) / 2048;
  if (mm <= 1) return launch_stage2_t<1>(cfg, a);
  if (mm == 2) return launch_stage2_t<2>(cfg, a);
  if (mm == 3) return launch_stage2_t<3>(cfg, a);
  if (mm == 4) return launch_stage2_t<4>(cfg, a);
  return launch_stage2_t<8>(cfg, a);
}

cudaError_t launch_reduce(const prox_layer* L, float* out, cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((L->d + 31) / 32, 1, 1);
  cfg.blockDim = dim3(kReduceWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, reduce_kernel, (const float*)L->ws.ypart, L->P, L->d, out,
                            L->ws.hist);
}

}  // namespace prox
