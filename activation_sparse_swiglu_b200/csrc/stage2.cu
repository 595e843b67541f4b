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
// (two rows per slot).  The consumer warps take every ring item in order (so
// each mbarrier wait is for the phase right after one the waiting thread has
// already seen complete):
//   phase A: for each channel every warp forms partial dot products of its
//            share of the column with the full x (x kept in registers; fp32,
//            packed f32x2 FMAs, warp-shuffle reduction) and parks them in
//            shared memory; after the last channel the partials are summed in
//            a fixed order into g = x . W_gate[:, j], u = x . W_up[:, j] and
//            s_j = act(g) u (the A3 ablation skips the gate/up records
//            and takes s_j = s~_j from Stage 1);
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

enum Stage2Mode { kGivenList = 0, kTopK = 1, kDense = 2, kThreshold = 3 };

struct Stage2Args {
  const float* x;
  const uint16_t* wgu;
  const uint16_t* wd;
  const int32_t* idx;      // kGivenList: channel list [k]
  const float* scores;     // kTopK: Stage-1 scores [F]
  const uint32_t* hist;    // kTopK: Stage-1 histogram of the scores' bits 30..20
  unsigned long long* stats;
  const uint2* bucket;     // kTopK: Stage-1 (key, channel) buckets per histogram bin
  int32_t* sel_mask;       // kTopK / kThreshold: 1/0 per channel (debug)
  float tau_s;             // kThreshold: channels with score >= tau_s
  int mode, select_only;
  int k;
  int d, F, P, slots, max_rec;
  int groups;  // consumer groups NG (= producer lanes); slots is a multiple of it
  float* ypart;
  float* s_sp;
  const float* s_tilde;  // proxy_values: Stage-1 act(g~) u~ [F]
  int proxy_values;      // ablation: skip the gate/up records, use s~ as s
  int act;               // gate activation (PROX_ACT_*)
  int* err;
  int x_ready;
};

// MAXM = ceil(d_model / (8 * consumer threads)): 8-element chunks per thread and column.
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
      mbar_init(&empty[s], NCW / a.groups);
    }
    fence_barrier_init();
  }
  // Consumer warps form NG groups of WPG; a group takes whole ring items, warp
  // wi of a group the elements [wi*qd, (wi+1)*qd) of each column / row
  // (qd = d / WPG), lane chunks e8 = m*32 + lane of 8 elements.
  const int NG = a.groups, WPG = NCW / NG, qd = d / WPG;
  const int grp = warp / WPG, wi = warp % WPG;
  auto elem = [&](int m) { return wi * qd + (m * 32 + lane) * 8; };
  auto elem_ok = [&](int m) { return (m * 32 + lane) * 8 < qd; };
  // this thread's x elements, kept in registers
  float4 xr[MAXM][2];
  auto load_x = [&]() {
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int e = elem(m);
      xr[m][0] = elem_ok(m) ? __ldg(reinterpret_cast<const float4*>(a.x + e)) : make_float4(0, 0, 0, 0);
      xr[m][1] = elem_ok(m) ? __ldg(reinterpret_cast<const float4*>(a.x + e + 4)) : make_float4(0, 0, 0, 0);
    }
  };
  if (a.x_ready && warp < NCW) load_x();
  __syncthreads();

  pdl_wait();
  pdl_trigger();

  if (!a.x_ready && warp < NCW) load_x();
  const int k = a.mode == kDense ? a.F : a.k;
  const int cta = blockIdx.x;
  int t0 = 0, n = 0;
  if (a.mode == kTopK || a.mode == kThreshold) {
    // This CTA's channels are [c0, c1); those past the cut are its records.
    // Top-k: the exact cut of the token; threshold (Prox §4.1): score >= tau_s,
    // i.e. key >= bits(tau_s) with every tie kept.
    const int c0 = (int)(((long long)a.F * cta) / a.P);
    const int c1 = (int)(((long long)a.F * (cta + 1)) / a.P);
    SelectScratch& sc = *reinterpret_cast<SelectScratch*>(ring);
    const uint32_t key0 = c0 + tid < c1 ? __float_as_uint(__ldcg(a.scores + c0 + tid)) : 0u;
    TopkCut cut;
    if (a.mode == kTopK) {
      cut = select_cut_cta(a.scores, a.hist, a.bucket, a.F, a.k, sc);
    } else {
      cut.T = __float_as_uint(a.tau_s);
      cut.tie_cut = a.F;
    }
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
    if (tid == 0 && a.stats && !a.select_only) {
      if (cta == 0) atomicAdd(a.stats + 1, 1ull);
      atomicAdd(a.stats + 2, (unsigned long long)n);
    }
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

  // Ring items: channel records q < n (gate column | up column), then W_down
  // row pairs (rows 2p, 2p+1).  Group g takes records g, g+NG, ... and pairs
  // g, g+NG, ...; its items, records first, use the group's own SPG slots
  // [g*SPG, (g+1)*SPG) round robin, so every slot's waiter is one group that
  // takes its uses in order.  Producer lane g fills group g's slots.
  const int nB = (n + 1) >> 1;
  const int SPG = slots / NG;
  auto group_items = [&](int g, int cnt) { return cnt > g ? (cnt - g + NG - 1) / NG : 0; };
  bool dead = false;  // set once a wait of this thread ran out
  if (warp == NCW) {
    // ---------------- producer lanes 0..NG-1 ----------------
    if (lane < NG) {
      const int g = lane;
      const uint64_t pol = l2_policy_evict_first();
      const int nA_g = a.proxy_values ? 0 : group_items(g, n), nB_g = group_items(g, nB);
      const int tot_g = nA_g + nB_g;
      for (int li = 0; li < tot_g; ++li) {
        const int slot = g * SPG + li % SPG, use = li / SPG;
        if (use > 0) mbar_wait(&empty[slot], (uint32_t)((use - 1) & 1), a.err, &dead);
        unsigned char* dst = ring + (size_t)slot * slot_bytes;
        if (li < nA_g) {
          const int r = g + li * NG;
          mbar_arrive_expect_tx(&full[slot], slot_bytes);
          bulk_copy_g2s(dst, a.wgu + (size_t)s_idx[r] * 2 * (size_t)d, slot_bytes, &full[slot], pol);
        } else {
          const int r0 = 2 * (g + (li - nA_g) * NG);
          const int nr = r0 + 1 < n ? 2 : 1;
          mbar_arrive_expect_tx(&full[slot], (uint32_t)nr * col_bytes);
          bulk_copy_g2s(dst, a.wd + (size_t)s_idx[r0] * (size_t)d, col_bytes, &full[slot], pol);
          if (nr == 2)
            bulk_copy_g2s(dst + col_bytes, a.wd + (size_t)s_idx[r0 + 1] * (size_t)d, col_bytes,
                          &full[slot], pol);
        }
      }
      // Every issued copy must land before this CTA's shared memory is released:
      // wait for the last use of each slot of the group.
      for (int j = 0; j < SPG && j < tot_g; ++j) {
        const int last = j + ((tot_g - 1 - j) / SPG) * SPG;  // last li with li % SPG == j
        mbar_wait(&full[g * SPG + j], (uint32_t)((last / SPG) & 1), a.err);
      }
    }
    return;
  }

  // ---------------- phase A: gate/up partial dot products ----------------
  // The warp's share of an item goes into registers, the slot goes back to the
  // producer, then the FMAs.
  const int nA_g = a.proxy_values ? 0 : group_items(grp, n);
  for (int li = 0; li < nA_g; ++li) {
    const int r = grp + li * NG;
    const int slot = grp * SPG + li % SPG;
    mbar_wait(&full[slot], (uint32_t)((li / SPG) & 1), a.err, &dead);
    const unsigned char* wg = ring + (size_t)slot * slot_bytes;
    const unsigned char* wu = wg + col_bytes;
    uint4 gv[MAXM], uv[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int e = elem(m);
      gv[m] = elem_ok(m) ? *reinterpret_cast<const uint4*>(wg + (size_t)e * 2) : make_uint4(0u, 0u, 0u, 0u);
      uv[m] = elem_ok(m) ? *reinterpret_cast<const uint4*>(wu + (size_t)e * 2) : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot], 1);
    float2 ag0 = make_float2(0.f, 0.f), ag1 = ag0, au0 = ag0, au1 = ag0;
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const float4 xa = xr[m][0], xb = xr[m][1];
      ag0 = __ffma2_rn(bf16x2_to_f2(gv[m].x), make_float2(xa.x, xa.y), ag0);
      au0 = __ffma2_rn(bf16x2_to_f2(uv[m].x), make_float2(xa.x, xa.y), au0);
      ag1 = __ffma2_rn(bf16x2_to_f2(gv[m].y), make_float2(xa.z, xa.w), ag1);
      au1 = __ffma2_rn(bf16x2_to_f2(uv[m].y), make_float2(xa.z, xa.w), au1);
      ag0 = __ffma2_rn(bf16x2_to_f2(gv[m].z), make_float2(xb.x, xb.y), ag0);
      au0 = __ffma2_rn(bf16x2_to_f2(uv[m].z), make_float2(xb.x, xb.y), au0);
      ag1 = __ffma2_rn(bf16x2_to_f2(gv[m].w), make_float2(xb.z, xb.w), ag1);
      au1 = __ffma2_rn(bf16x2_to_f2(uv[m].w), make_float2(xb.z, xb.w), au1);
    }
    float g = (ag0.x + ag0.y) + (ag1.x + ag1.y);
    float u = (au0.x + au0.y) + (au1.x + au1.y);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      u += __shfl_xor_sync(0xffffffffu, u, o);
    }
    if (lane == 0) {
      s_pg[r * NCW + wi] = g;
      s_pu[r * NCW + wi] = u;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
  for (int r = tid; r < n; r += NCW * 32) {
    float sv;
    if (a.proxy_values) {
      sv = __ldcg(a.s_tilde + s_idx[r]);
    } else {
      float g = 0.f, u = 0.f;
      for (int w = 0; w < WPG; ++w) {
        g += s_pg[r * NCW + w];
        u += s_pu[r * NCW + w];
      }
      sv = act_f32(g, a.act) * u;
    }
    s_val[r] = sv;
    if (a.s_sp) a.s_sp[a.mode == kGivenList ? s_lpos[r] : t0 + r] = sv;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");

  // ---------------- phase B: y_part = sum_t s_t W_down[j_t, :] ----------------
  // The group's row pairs; warp wi accumulates its columns [wi*qd, (wi+1)*qd).
  float2 acc[MAXM * 4];
#pragma unroll
  for (int i = 0; i < MAXM * 4; ++i) acc[i] = make_float2(0.f, 0.f);
  const int nB_g = group_items(grp, nB);
  for (int lb = 0; lb < nB_g; ++lb) {
    const int li = nA_g + lb;
    const int p = grp + lb * NG;  // row pair
    const int slot = grp * SPG + li % SPG;
    mbar_wait(&full[slot], (uint32_t)((li / SPG) & 1), a.err, &dead);
    const unsigned char* w = ring + (size_t)slot * slot_bytes;
    const bool two = 2 * p + 1 < n;
    uint4 wv[2][MAXM];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        const int e = elem(m);
        wv[h][m] = (elem_ok(m) && (h == 0 || two))
                       ? *reinterpret_cast<const uint4*>(w + h * col_bytes + (size_t)e * 2)
                       : make_uint4(0u, 0u, 0u, 0u);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot], 1);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float sv = (h == 0 || two) ? s_val[2 * p + h] : 0.f;
      const float2 s2 = make_float2(sv, sv);
#pragma unroll
      for (int m = 0; m < MAXM; ++m) {
        const uint4 w4 = wv[h][m];
        acc[4 * m + 0] = __ffma2_rn(bf16x2_to_f2(w4.x), s2, acc[4 * m + 0]);
        acc[4 * m + 1] = __ffma2_rn(bf16x2_to_f2(w4.y), s2, acc[4 * m + 1]);
        acc[4 * m + 2] = __ffma2_rn(bf16x2_to_f2(w4.z), s2, acc[4 * m + 2]);
        acc[4 * m + 3] = __ffma2_rn(bf16x2_to_f2(w4.w), s2, acc[4 * m + 3]);
      }
    }
  }
  // The groups' partial rows are added in group order (deterministic).  Every
  // copy has landed (each item was waited for), so the ring holds them.
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
  float* s_y = reinterpret_cast<float*>(ring);  // [NG][d]
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    if (elem_ok(m)) {
      float* dst = s_y + (size_t)grp * d + elem(m);
      *reinterpret_cast<float4*>(dst) =
          make_float4(acc[4 * m].x, acc[4 * m].y, acc[4 * m + 1].x, acc[4 * m + 1].y);
      *reinterpret_cast<float4*>(dst + 4) =
          make_float4(acc[4 * m + 2].x, acc[4 * m + 2].y, acc[4 * m + 3].x, acc[4 * m + 3].y);
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");
  float* out = a.ypart + (size_t)cta * d;
  for (int e = tid * 4; e < d; e += NCW * 32 * 4) {
    float4 v = *reinterpret_cast<const float4*>(s_y + e);
    for (int g = 1; g < NG; ++g) {
      const float4 t = *reinterpret_cast<const float4*>(s_y + (size_t)g * d + e);
      v.x += t.x;
      v.y += t.y;
      v.z += t.z;
      v.w += t.w;
    }
    *reinterpret_cast<float4*>(out + e) = v;
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

void choose_stage2(int d, int F, int num_sms, int* P, int* slots, int* groups, size_t* smem) {
  *P = num_sms;
  const int max_rec = (F + num_sms - 1) / num_sms + 1;
  size_t off = (size_t)max_rec * (12 + 8 * NCW) + 128;
  const size_t slot_bytes = 4 * (size_t)d;  // gate + up column, or two W_down rows
  int s = (int)((kStage2SmemBudget - off) / (slot_bytes + 16));
  if (s > 32) s = 32;
  if (s < 2) s = 2;
  // Consumer groups: the most groups (4, 2, 1) whose slot share is at least
  // two and whose warps hold at most 4 chunks of 8 elements per lane.
  int ng = 1;
  for (int cand : {4, 2}) {
    const int wpg = NCW / cand;
    const int maxm = (d + wpg * 256 - 1) / (wpg * 256);
    if ((s - s % cand) / cand >= 2 && maxm <= 4) {
      ng = cand;
      break;
    }
  }
  s -= s % ng;
  *groups = ng;
  *slots = s;
  off = (size_t)s * 16 + (size_t)max_rec * (12 + 8 * NCW);
  off = (off + 127) & ~(size_t)127;
  size_t region = (size_t)s * slot_bytes;
  if (region < sizeof(SelectScratch)) region = sizeof(SelectScratch);  // the select's scratch
  if (region < (size_t)ng * d * 4) region = (size_t)ng * d * 4;         // the groups' partial rows
  *smem = off + region;
}

cudaError_t setup_stage2_kernels() {
  cudaError_t e;
  if ((e = set_stage2_attr<1>()) != cudaSuccess) return e;
  if ((e = set_stage2_attr<2>()) != cudaSuccess) return e;
  if ((e = set_stage2_attr<3>()) != cudaSuccess) return e;
  return set_stage2_attr<4>();
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
  a.tau_s = m.tau_s;
  a.mode = m.mode;
  a.select_only = m.select_only ? 1 : 0;
  a.k = m.k;
  a.d = L->d;
  a.F = L->F;
  a.P = L->P;
  a.slots = L->ring_slots;
  a.groups = L->stage2_groups;
  a.max_rec = (L->F + L->P - 1) / L->P + 1;
  a.ypart = L->ws.ypart;
  a.s_sp = m.s_sp;
  a.s_tilde = L->ws.s_tilde;
  a.proxy_values = m.proxy_values ? 1 : 0;
  a.act = L->act;
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
  const int wpg = NCW / L->stage2_groups;
  const int mm = (L->d + wpg * 256 - 1) / (wpg * 256);
  if (mm <= 1) return launch_stage2_t<1>(cfg, a);
  if (mm == 2) return launch_stage2_t<2>(cfg, a);
  if (mm == 3) return launch_stage2_t<3>(cfg, a);
  return launch_stage2_t<4>(cfg, a);  // choose_stage2 keeps mm <= 4
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
