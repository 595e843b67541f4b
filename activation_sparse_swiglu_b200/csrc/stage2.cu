// Stage 2 of the Prox decode step (Prox §4.1 "Stage 2: exact sparse
// computation"; §4.3 fused output-sparse gate/up kernel and input-sparse
// down GEMV), and the dense SwiGLU baseline (Prox §2.1), which is the same
// kernel with every channel kept.
//
// stage2_kernel -- persistent: one CTA per SM, each CTA owning a contiguous,
// balanced range of the k selected channels.  A producer warp streams, with
// 1-D bulk async copies (TMA engine) into a ring of shared-memory slots, first
// the gate/up channel records of its channels (gate column then up column,
// d_model bf16 each, contiguous per channel), then their W_down rows.  Eight
// consumer warps:
//   phase A: one warp per channel computes g = x . W_gate[:, j] and
//            u = x . W_up[:, j] over the full x (fp32, packed f32x2 FMAs,
//            warp-shuffle reduction) and keeps s_j = SiLU(g) u;
//   phase B: all warps accumulate y_part += s_j W_down[j, :] for the CTA's
//            channels, each thread owning 8-column groups of the output.
// Each CTA writes its fp32 partial y; reduce_kernel sums the partials in a
// fixed order (deterministic, no atomics on floats).
#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {
namespace {

constexpr int NCW = kStage2Consumers;
constexpr int S2_THREADS = (NCW + 1) * 32;
constexpr size_t kStage2SmemBudget = 200 * 1024;

struct Stage2Args {
  const float* x;
  const uint16_t* wgu;
  const uint16_t* wd;
  const int32_t* idx;
  const int32_t* k_dev;
  int k_host;
  int d, F, P, slots, max_rec;
  float* ypart;
  float* s_sp;
  int* err;
  int x_ready;
};

__device__ __forceinline__ void load_x(float* xs, const float* x, int d, int tid, int nt) {
  for (int e = tid * 4; e < d; e += nt * 4)
    *reinterpret_cast<float4*>(xs + e) = __ldg(reinterpret_cast<const float4*>(x + e));
}

// Dot products of 8 consecutive bf16 weights (one uint4) with 8 fp32 x values.
__device__ __forceinline__ void dot8(float2 (&acc)[4], const uint4& w, const float4& xa,
                                     const float4& xb) {
  acc[0] = __ffma2_rn(bf16x2_to_f2(w.x), make_float2(xa.x, xa.y), acc[0]);
  acc[1] = __ffma2_rn(bf16x2_to_f2(w.y), make_float2(xa.z, xa.w), acc[1]);
  acc[2] = __ffma2_rn(bf16x2_to_f2(w.z), make_float2(xb.x, xb.y), acc[2]);
  acc[3] = __ffma2_rn(bf16x2_to_f2(w.w), make_float2(xb.z, xb.w), acc[3]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int MAXM>
__global__ void __launch_bounds__(S2_THREADS, 1) stage2_kernel(Stage2Args a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int d = a.d, slots = a.slots;
  const uint32_t slot_bytes = 2u * (uint32_t)d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + slots;
  float* s_val = reinterpret_cast<float*>(empty + slots);
  int* s_idx = reinterpret_cast<int*>(s_val + a.max_rec);
  size_t off = (size_t)slots * 16 + (size_t)a.max_rec * 8;
  off = (off + 15) & ~(size_t)15;
  float* xs = reinterpret_cast<float*>(smem + off);
  off += (size_t)d * 4;
  off = (off + 127) & ~(size_t)127;
  unsigned char* ring = smem + off;

  if (tid == 0) {
    for (int s = 0; s < slots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    fence_barrier_init();
  }
  if (a.x_ready) load_x(xs, a.x, d, tid, S2_THREADS);
  __syncthreads();

  pdl_wait();
  pdl_trigger();

  if (!a.x_ready) load_x(xs, a.x, d, tid, S2_THREADS);
  const int k = a.k_dev ? __ldcg(a.k_dev) : a.k_host;
  const int cta = blockIdx.x;
  const int t0 = (int)(((long long)k * cta) / a.P);
  const int t1 = (int)(((long long)k * (cta + 1)) / a.P);
  const int n = t1 - t0;
  for (int i = tid; i < n; i += S2_THREADS) {
    int j = a.idx ? __ldcg(a.idx + t0 + i) : t0 + i;
    if (j < 0 || j >= a.F) {
      atomicOr(a.err, PROX_DEVERR_MASK_INDEX);
      j = 0;
    }
    s_idx[i] = j;
  }
  __syncthreads();

  // Ring schedule.  Phase A: record r (gate column, up column) goes to slot
  // pair r % npa and is consumed by warp (r % npa) % na, so every slot pair
  // has one owning warp that consumes its uses in order.  Phase B: W_down row
  // i goes to slot i % slots and is consumed by every warp in order.  Each
  // mbarrier wait is therefore for the next phase of a barrier whose earlier
  // phases this thread has already seen complete, so parity waits cannot alias.
  bool dead = false;  // set once a wait of this thread ran out
  const int npairs = slots / 2;
  const int na = npairs < NCW ? npairs : NCW;   // phase-A consumer warps
  const int npa = na * (npairs / na);           // phase-A slot pairs in use
  // uses of slot s by phase A
  auto uses_a = [&](int slot) -> int {
    const int p = slot >> 1;
    if (p >= npa || p >= n) return 0;
    return (n - p + npa - 1) / npa;
  };
  if (warp == NCW) {
    // ---------------- producer ----------------
    if (lane == 0 && n > 0) {
      const uint64_t pol = l2_policy_evict_first();
      for (int r = 0; r < n; ++r) {
        const int p = r % npa, use = r / npa;
        const size_t rec = (size_t)s_idx[r] * 2;
        for (int h = 0; h < 2; ++h) {
          const int slot = 2 * p + h;
          if (use > 0) mbar_wait(&empty[slot], (uint32_t)((use - 1) & 1), a.err, &dead);
          mbar_arrive_expect_tx(&full[slot], slot_bytes);
          bulk_copy_g2s(ring + (size_t)slot * slot_bytes, a.wgu + (rec + h) * (size_t)d,
                        slot_bytes, &full[slot], pol);
        }
      }
      for (int i = 0; i < n; ++i) {
        const int slot = i % slots, use = uses_a(slot) + i / slots;
        if (use > 0) mbar_wait(&empty[slot], (uint32_t)((use - 1) & 1), a.err, &dead);
        mbar_arrive_expect_tx(&full[slot], slot_bytes);
        bulk_copy_g2s(ring + (size_t)slot * slot_bytes, a.wd + (size_t)s_idx[i] * (size_t)d,
                      slot_bytes, &full[slot], pol);
      }
      // Every issued copy must land before this CTA's shared memory is released.
      for (int slot = 0; slot < slots; ++slot) {
        const int uses = uses_a(slot) + (slot < n ? (n - slot + slots - 1) / slots : 0);
        if (uses > 0) mbar_wait(&full[slot], (uint32_t)((uses - 1) & 1), a.err);
      }
    }
    return;
  }

  // ---------------- phase A: gate/up, one warp per channel ----------------
  if (warp < na) {
    // npa is a multiple of na, so slot pair r % npa is always owned by warp r % na
    for (int r = warp; r < n; r += na) {
      const int p = r % npa, use = r / npa;
      const int sl0 = 2 * p, sl1 = sl0 + 1;
      mbar_wait(&full[sl0], (uint32_t)(use & 1), a.err, &dead);
      mbar_wait(&full[sl1], (uint32_t)(use & 1), a.err, &dead);
      const unsigned char* wg = ring + (size_t)sl0 * slot_bytes;
      const unsigned char* wu = ring + (size_t)sl1 * slot_bytes;
      float2 ag[4], au[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) ag[i] = au[i] = make_float2(0.f, 0.f);
      for (int e = lane * 8; e < d; e += 256) {
        const uint4 g4 = lds_v4(wg + (size_t)e * 2);
        const uint4 u4 = lds_v4(wu + (size_t)e * 2);
        const float4 xa = lds_f4(xs + e);
        const float4 xb = lds_f4(xs + e + 4);
        dot8(ag, g4, xa, xb);
        dot8(au, u4, xa, xb);
      }
      float g = (ag[0].x + ag[0].y) + (ag[1].x + ag[1].y) + (ag[2].x + ag[2].y) +
                (ag[3].x + ag[3].y);
      float u = (au[0].x + au[0].y) + (au[1].x + au[1].y) + (au[2].x + au[2].y) +
                (au[3].x + au[3].y);
      g = warp_sum(g);
      u = warp_sum(u);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[sl0], NCW);
        mbar_arrive(&empty[sl1], NCW);
        const float sv = silu_f32(g) * u;
        s_val[r] = sv;
        if (a.s_sp) a.s_sp[t0 + r] = sv;
      }
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(NCW * 32) : "memory");

  // ---------------- phase B: y_part = sum_t s_t W_down[j_t, :] ----------------
  float2 acc[MAXM * 4];
#pragma unroll
  for (int i = 0; i < MAXM * 4; ++i) acc[i] = make_float2(0.f, 0.f);
  for (int rr = 0; rr < n; ++rr) {
    const int sl = rr % slots, use = uses_a(sl) + rr / slots;
    mbar_wait(&full[sl], (uint32_t)(use & 1), a.err, &dead);
    const float sv = s_val[rr];
    const float2 s2 = make_float2(sv, sv);
    const unsigned char* w = ring + (size_t)sl * slot_bytes;
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      const int e = tid * 8 + m * (NCW * 32 * 8);
      if (e < d) {
        const uint4 w4 = lds_v4(w + (size_t)e * 2);
        acc[4 * m + 0] = __ffma2_rn(bf16x2_to_f2(w4.x), s2, acc[4 * m + 0]);
        acc[4 * m + 1] = __ffma2_rn(bf16x2_to_f2(w4.y), s2, acc[4 * m + 1]);
        acc[4 * m + 2] = __ffma2_rn(bf16x2_to_f2(w4.z), s2, acc[4 * m + 2]);
        acc[4 * m + 3] = __ffma2_rn(bf16x2_to_f2(w4.w), s2, acc[4 * m + 3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[sl], 1);
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

// out[c] = sum_p ypart[p][c], p in increasing order.
__global__ void __launch_bounds__(kReduceWarps * 32) reduce_kernel(const float* ypart, int P, int d,
                                                                   float* out) {
  __shared__ float s_part[kReduceWarps][32];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (col < d) {
    int p = warp;
    for (; p + 3 * kReduceWarps < P; p += 4 * kReduceWarps) {
      const float v0 = __ldcg(ypart + (size_t)p * d + col);
      const float v1 = __ldcg(ypart + (size_t)(p + kReduceWarps) * d + col);
      const float v2 = __ldcg(ypart + (size_t)(p + 2 * kReduceWarps) * d + col);
      const float v3 = __ldcg(ypart + (size_t)(p + 3 * kReduceWarps) * d + col);
      s += v0;
      s += v1;
      s += v2;
      s += v3;
    }
    for (; p < P; p += kReduceWarps) s += __ldcg(ypart + (size_t)p * d + col);
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

void choose_stage2(int d, int F, int num_sms, int* P, int* slots, size_t* smem) {
  *P = num_sms;
  const int max_rec = (F + num_sms - 1) / num_sms + 1;
  size_t fixed = (size_t)max_rec * 8 + 16 + (size_t)d * 4 + 128;
  const size_t slot_bytes = 2 * (size_t)d;
  int s = (int)((kStage2SmemBudget - fixed) / (slot_bytes + 16));
  if (s > 32) s = 32;
  if (s < 3) s = 3;
  *slots = s;
  size_t off = (size_t)s * 16 + (size_t)max_rec * 8;
  off = (off + 15) & ~(size_t)15;
  off += (size_t)d * 4;
  off = (off + 127) & ~(size_t)127;
  *smem = off + (size_t)s * slot_bytes;
}

cudaError_t setup_stage2_kernels() {
  cudaError_t e;
  if ((e = set_stage2_attr<1>()) != cudaSuccess) return e;
  if ((e = set_stage2_attr<2>()) != cudaSuccess) return e;
  if ((e = set_stage2_attr<3>()) != cudaSuccess) return e;
  if ((e = set_stage2_attr<4>()) != cudaSuccess) return e;
  return set_stage2_attr<8>();
}

cudaError_t launch_stage2(const prox_layer* L, const float* x, const int32_t* idx,
                          const int32_t* k_dev, int k_host, float* s_sp, cudaStream_t s,
                          bool pdl, bool x_ready) {
  Stage2Args a;
  a.x = x;
  a.wgu = L->wgu;
  a.wd = L->wd;
  a.idx = idx;
  a.k_dev = k_dev;
  a.k_host = idx ? k_host : L->F;
  a.d = L->d;
  a.F = L->F;
  a.P = L->P;
  a.slots = L->ring_slots;
  a.max_rec = (L->F + L->P - 1) / L->P + 1;
  a.ypart = L->ws.ypart;
  a.s_sp = s_sp;
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
  const int m = (L->d + 2047) / 2048;
  if (m <= 1) return launch_stage2_t<1>(cfg, a);
  if (m == 2) return launch_stage2_t<2>(cfg, a);
  if (m == 3) return launch_stage2_t<3>(cfg, a);
  if (m == 4) return launch_stage2_t<4>(cfg, a);
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
  return cudaLaunchKernelEx(&cfg, reduce_kernel, (const float*)L->ws.ypart, L->P, L->d, out);
}

}  // namespace prox
