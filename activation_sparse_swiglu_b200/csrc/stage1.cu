// Stage 1 of the Prox decode step (Prox §4.1 "Stage 1: lightweight proxy
// construction", §4.3 fused split-N proxy kernel).
//
// stage1_kernel -- one CTA per (column slice c, row slab r); the R slabs of a
// column slice form one thread-block cluster:
//   * a column slice is 512 bytes of an interleaved proxy row (16 blocks of 32
//     channels; each block is 16 B of gate codes then 16 B of up codes), i.e.
//     512 channels of both proxies; a warp reads one kept row's slice per load
//     instruction (512 contiguous bytes), a lane owning one 16-byte chunk (32
//     channels of one branch);
//   * a row slab is `gps` whole quantisation groups (gps * 128 input rows).
//   The CTA thresholds its slab of x (|x_i| >= tau) and compacts the kept rows
//   in ascending order; its 4 warps stream those rows through a per-warp
//   shared-memory ring with asynchronous 16-byte copies (cp.async, L2 only;
//   each lane copies and later reads back its own chunk, so no barrier is
//   needed), three batches of 8 rows in flight, and dequantise the INT4 codes
//   in registers with fp32 (packed f32x2) arithmetic, accumulating per group
//   and scaling once per group by the fp16 group scale.  The cluster's CTAs
//   then add their partial sums through distributed shared memory in rank
//   order (deterministic), each CTA scoring a share of the slice's channels:
//   score_j = |SiLU(g~_j) u~_j|, also added to a 2048-bin histogram of its top
//   bits -- the first level of the radix select.
//
#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {
namespace {

constexpr int S1_NW = kStage1Warps;
constexpr int S1_NT = S1_NW * 32;
constexpr int S1_SLICE = 512;   // bytes (= channels of both proxies) per column slice
constexpr int S1_CHUNKS = 32;   // 16-byte chunks per slice (one per lane)
constexpr int S1_PART = 1024;   // partial values per CTA: 32 chunks x 32 channels
constexpr int S1_U = 8;         // rows per batch
constexpr int S1_NB = 3;        // batches in flight per warp
constexpr int S1_RING = S1_NB * S1_U * S1_SLICE;  // ring bytes per warp

struct Stage1Args {
  const float* x;
  const uint8_t* pq;
  const __half* ps;
  float tau;
  int d, F, R, gps;
  float* scores;
  uint32_t* hist;
  unsigned long long* stats;
  float* g_dbg;
  float* u_dbg;
  int32_t* slab_idx;
  int32_t* slab_cnt;
};

// Eight INT4 codes of one 32-bit word (nibble p is channel 8w+p of the lane's
// chunk, stored as q+8) into four float2 accumulators.  Each nibble is OR-ed
// into the mantissa of a float whose exponent makes the nibble's lowest bit
// worth exactly 1, so subtracting (2^e + 8) leaves q - 8 exactly; nibbles 5..7
// are first shifted down by 12 bits.
__device__ __forceinline__ void acc_word(float2* a, uint32_t w, float2 x2) {
  const uint32_t h = w >> 12;
  const float2 v0 = __fadd2_rn(make_float2(__uint_as_float((w & 0x0000000Fu) | 0x4B000000u),
                                           __uint_as_float((w & 0x000000F0u) | 0x49000000u)),
                               make_float2(-8388616.0f, -524296.0f));
  const float2 v1 = __fadd2_rn(make_float2(__uint_as_float((w & 0x00000F00u) | 0x47000000u),
                                           __uint_as_float((w & 0x0000F000u) | 0x45000000u)),
                               make_float2(-32776.0f, -2056.0f));
  const float2 v2 = __fadd2_rn(make_float2(__uint_as_float((w & 0x000F0000u) | 0x43000000u),
                                           __uint_as_float((h & 0x00000F00u) | 0x47000000u)),
                               make_float2(-136.0f, -32776.0f));
  const float2 v3 = __fadd2_rn(make_float2(__uint_as_float((h & 0x0000F000u) | 0x45000000u),
                                           __uint_as_float((h & 0x000F0000u) | 0x43000000u)),
                               make_float2(-2056.0f, -136.0f));
  a[0] = __ffma2_rn(v0, x2, a[0]);
  a[1] = __ffma2_rn(v1, x2, a[1]);
  a[2] = __ffma2_rn(v2, x2, a[2]);
  a[3] = __ffma2_rn(v3, x2, a[3]);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of all CTAs of the cluster: release our shared-memory writes,
// acquire the others'.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ float ld_peer_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__global__ void __launch_bounds__(S1_NT, 4) stage1_kernel(Stage1Args a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int c = blockIdx.x, r = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cl = lane;
  const int gps = a.gps, slab_rows = gps * kGroup, row0 = r * slab_rows;
  const int n16 = a.F >> 4, nblk = a.F >> 5;
  const int c16 = c * S1_CHUNKS + cl;  // this lane's 16-byte chunk of a proxy row
  const bool lane_ok = c16 < n16;

  unsigned char* ring = smem;                                            // [NW][NB][U][512]
  float* s_red = reinterpret_cast<float*>(smem + S1_NW * S1_RING);       // [NW][1024]
  float* s_part = s_red + S1_NW * S1_PART;                               // [512]
  uint4* s_scale = reinterpret_cast<uint4*>(s_part + S1_PART);           // [gps][32][4]
  int2* s_rx = reinterpret_cast<int2*>(s_scale + gps * S1_CHUNKS * 4);   // [slab_rows]
  int* s_scan = reinterpret_cast<int*>(s_rx + slab_rows);                // [33]

  // Prologue (constant weights only): this slice's fp16 scales for the slab's
  // groups, 64 bytes per chunk and group, loaded in batches of 8.
  {
    const int n = gps * S1_CHUNKS * 4;
    for (int base = tid; base < n; base += 8 * S1_NT) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = base + u * S1_NT;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        const int gl = e / (S1_CHUNKS * 4), ck = (e >> 2) % S1_CHUNKS, qd = e & 3;
        const int cc = c * S1_CHUNKS + ck;
        if (e < n && cc < n16) {
          const int g = row0 / kGroup + gl;
          const __half* src = a.ps + ((size_t)g * nblk + (cc >> 1)) * 64 + (cc & 1) * 32 + qd * 8;
          v[u] = __ldg(reinterpret_cast<const uint4*>(src));
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = base + u * S1_NT;
        if (e < n) s_scale[e] = v[u];
      }
    }
  }

  pdl_wait();     // x and the workspace now belong to this token
  pdl_trigger();  // let Stage 2 become resident

  // Kept rows of this slab, ascending: thread t owns rows [t*rpt, (t+1)*rpt).
  const int rpt = slab_rows / S1_NT;
  const float* xs = a.x + row0 + tid * rpt;
  int cnt = 0;
  for (int i0 = 0; i0 < rpt; i0 += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = (i0 + u < rpt) ? __ldg(xs + i0 + u) : 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) cnt += (i0 + u < rpt) && (fabsf(v[u]) >= a.tau);
  }
  int total;
  int pos = block_exclusive_scan(cnt, s_scan, &total);
  for (int i = 0; i < rpt; ++i) {
    const float xv = __ldg(xs + i);
    if (fabsf(xv) >= a.tau) s_rx[pos++] = make_int2(row0 + tid * rpt + i, __float_as_int(xv));
  }
  __syncthreads();
  if (c == 0) {
    if (tid == 0) atomicAdd(a.stats, (unsigned long long)total);
    if (a.slab_idx) {
      for (int e = tid; e < total; e += S1_NT) a.slab_idx[row0 + e] = s_rx[e].x;
      if (tid == 0) a.slab_cnt[r] = total;
    }
  }

  // Warp w takes positions w, w + 4, w + 8, ... of the compacted list, in
  // batches of 8 rows through its ring (NB batches in flight).
  const int nw = total > warp ? (total - warp + S1_NW - 1) / S1_NW : 0;
  const int nbw = (nw + S1_U - 1) / S1_U;
  unsigned char* wring = ring + warp * S1_RING + lane * 16;
  const uint8_t* colp = a.pq + (size_t)(lane_ok ? c16 : 0) * 16;
  auto issue = [&](int j) {
    if (j < nbw && lane_ok) {
      unsigned char* dst = wring + (j % S1_NB) * (S1_U * S1_SLICE);
#pragma unroll
      for (int u = 0; u < S1_U; ++u) {
        const int jj = j * S1_U + u;
        if (jj < nw) cp_async16(dst + u * S1_SLICE, colp + (size_t)s_rx[warp + S1_NW * jj].x * a.F);
      }
    }
    cp_async_commit();
  };
  float2 acc[16], tot[16];
#pragma unroll
  for (int h = 0; h < 16; ++h) acc[h] = tot[h] = make_float2(0.f, 0.f);
  int cur_g = -1;
#pragma unroll
  for (int j = 0; j < S1_NB - 1; ++j) issue(j);
  for (int j = 0; j < nbw; ++j) {
    issue(j + S1_NB - 1);
    cp_async_wait<S1_NB - 1>();  // this lane's copies of batch j have landed
    const unsigned char* src = wring + (j % S1_NB) * (S1_U * S1_SLICE);
#pragma unroll
    for (int u = 0; u < S1_U; ++u) {
      const int jj = j * S1_U + u;
      if (jj < nw) {
        const int2 rx = s_rx[warp + S1_NW * jj];
        const int gl = (rx.x - row0) >> 7;
        if (gl != cur_g) {
          if (cur_g >= 0) {
            const uint4* sc = s_scale + (cur_g * S1_CHUNKS + cl) * 4;
#pragma unroll
            for (int qd = 0; qd < 4; ++qd) {
              const uint4 s4 = sc[qd];
              const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&sw[m]));
                tot[qd * 4 + m] = __ffma2_rn(s2, acc[qd * 4 + m], tot[qd * 4 + m]);
                acc[qd * 4 + m] = make_float2(0.f, 0.f);
              }
            }
          }
          cur_g = gl;
        }
        const uint4 v = lane_ok ? *reinterpret_cast<const uint4*>(src + u * S1_SLICE)
                                : make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
        const float xv = __int_as_float(rx.y);
        const float2 x2 = make_float2(xv, xv);
        acc_word(acc + 0, v.x, x2);
        acc_word(acc + 4, v.y, x2);
        acc_word(acc + 8, v.z, x2);
        acc_word(acc + 12, v.w, x2);
      }
    }
  }
  cp_async_wait<0>();
  if (cur_g >= 0) {
    const uint4* sc = s_scale + (cur_g * S1_CHUNKS + cl) * 4;
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const uint4 s4 = sc[qd];
      const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&sw[m]));
        tot[qd * 4 + m] = __ffma2_rn(s2, acc[qd * 4 + m], tot[qd * 4 + m]);
      }
    }
  }
  // Combine the warps in a fixed order.  Partial element e = j*32 + chunk for
  // channel j of a chunk.
  {
    float* red = s_red + warp * S1_PART;
#pragma unroll
    for (int h = 0; h < 16; ++h) {
      red[(2 * h) * 32 + cl] = tot[h].x;
      red[(2 * h + 1) * 32 + cl] = tot[h].y;
    }
  }
  __syncthreads();
  for (int e = tid; e < S1_PART; e += S1_NT) {
    float sum = s_red[e];
#pragma unroll
    for (int w = 1; w < S1_NW; ++w) sum += s_red[w * S1_PART + e];
    s_part[e] = sum;
  }

  // Slab partials -> channel scores: the CTA of cluster rank q scores channels
  // [q*CH, (q+1)*CH) of the slice.  TPC threads share a channel, thread
  // `sub` adding peers sub, sub+TPC, ... (all loads in flight); the TPC sums
  // are then added in a fixed order.
  cluster_sync_all();
  const uint32_t q = cluster_rank();
  const int CH = (S1_SLICE + a.R - 1) / a.R;
  const int TPC = CH * 4 <= S1_NT ? 4 : (CH * 2 <= S1_NT ? 2 : 1);
  for (int base = 0; base < CH; base += S1_NT / TPC) {
    const int mc = base + tid / TPC, sub = tid % TPC;
    const int m = (int)q * CH + mc;
    const int ch = c * S1_SLICE + m;
    const bool ok = mc < CH && m < S1_SLICE && ch < a.F;
    float g = 0.f, u = 0.f;
    if (ok) {
      const int blk = m >> 5, jj = m & 31;
      const int eg = jj * 32 + 2 * blk, eu = eg + 1;
      float vg[kMaxCluster / 1], vu[kMaxCluster / 1];
#pragma unroll
      for (int i = 0; i < kMaxCluster; ++i) {
        const int rr = sub + i * TPC;
        vg[i] = rr < a.R ? ld_peer_f32(s_part + eg, (uint32_t)rr) : 0.f;
        vu[i] = rr < a.R ? ld_peer_f32(s_part + eu, (uint32_t)rr) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kMaxCluster; ++i) {
        g += vg[i];
        u += vu[i];
      }
    }
    // lanes sub = 0..TPC-1 of a channel are adjacent: combine in a fixed order
    if (TPC >= 2) {
      g += __shfl_xor_sync(0xffffffffu, g, 1);
      u += __shfl_xor_sync(0xffffffffu, u, 1);
    }
    if (TPC >= 4) {
      g += __shfl_xor_sync(0xffffffffu, g, 2);
      u += __shfl_xor_sync(0xffffffffu, u, 2);
    }
    if (ok && sub == 0) {
      const float sc = fabsf(silu_f32(g) * u);
      a.scores[ch] = sc;
      if (a.g_dbg) a.g_dbg[ch] = g;
      if (a.u_dbg) a.u_dbg[ch] = u;
      atomicAdd(a.hist + (__float_as_uint(sc) >> 20), 1u);
    }
  }
  cluster_sync_all();  // keep our shared memory alive until the peers have read it
}

// Debug tap: concatenate the per-slab kept-row lists written by stage1_kernel
// into one ascending list idx_x (and its length n_x).
__global__ void __launch_bounds__(256) concat_slabs_kernel(const int32_t* slab_idx,
                                                           const int32_t* slab_cnt, int R,
                                                           int slab_rows, int32_t* idx_x,
                                                           int32_t* n_x) {
  __shared__ int s_off[kMaxGroupsPerSlab * 4 + 1];
  if (threadIdx.x == 0) {
    int off = 0;
    for (int r = 0; r < R; ++r) {
      s_off[r] = off;
      off += slab_cnt[r];
    }
    s_off[R] = off;
    if (n_x) *n_x = off;
  }
  __syncthreads();
  for (int r = 0; r < R; ++r) {
    const int n = s_off[r + 1] - s_off[r];
    for (int e = threadIdx.x; e < n; e += blockDim.x)
      idx_x[s_off[r] + e] = slab_idx[(size_t)r * slab_rows + e];
  }
}

}  // namespace

void choose_stage1_grid(int d, int F, int num_sms, int* C, int* R, int* gps) {
  const int G = d / kGroup;
  *C = (F + S1_SLICE - 1) / S1_SLICE;
  // The row slabs of a column slice form one cluster (at most 16 CTAs).  Take
  // the most slabs that still keep the grid within one wave of 4 CTAs per SM.
  const int cap = 4 * num_sms;
  int best = 1;
  for (int r = 1; r <= kMaxCluster && r <= G; ++r) {
    if (G % r || G / r > kMaxGroupsPerSlab) continue;
    if (r == 1 || (long)(*C) * r <= cap) best = r;
  }
  *R = best;
  *gps = G / best;
}

size_t stage1_smem_bytes(int gps) {
  return (size_t)S1_NW * S1_RING + (size_t)(S1_NW + 1) * S1_PART * 4 +
         (size_t)gps * S1_CHUNKS * 64 + (size_t)gps * kGroup * 8 + 33 * 4;
}

cudaError_t setup_stage1_kernels() {
  cudaError_t e = cudaFuncSetAttribute(stage1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)stage1_smem_bytes(kMaxGroupsPerSlab));
  if (e != cudaSuccess) return e;
  // clusters of up to 16 CTAs (a size B200 supports beyond the portable 8)
  return cudaFuncSetAttribute(stage1_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

cudaError_t launch_stage1(const prox_layer* L, const float* x, const Stage1Taps& taps,
                          cudaStream_t s, bool pdl) {
  Stage1Args a;
  a.x = x;
  a.pq = L->pq;
  a.ps = reinterpret_cast<const __half*>(L->ps);
  a.tau = L->tau;
  a.d = L->d;
  a.F = L->F;
  a.R = L->R;
  a.gps = L->gps;
  a.scores = L->ws.scores;
  a.hist = L->ws.hist;
  a.stats = L->ws.stats;
  a.g_dbg = taps.g;
  a.u_dbg = taps.u;
  a.slab_idx = taps.slabs ? L->ws.slab_idx : nullptr;
  a.slab_cnt = L->ws.slab_cnt;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L->C, L->R, 1);
  cfg.blockDim = dim3(S1_NT, 1, 1);
  cfg.dynamicSmemBytes = L->stage1_smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = (unsigned)L->R;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, stage1_kernel, a);
}

cudaError_t launch_concat_slabs(const prox_layer* L, int32_t* idx_x, int32_t* n_x,
                                cudaStream_t s) {
  concat_slabs_kernel<<<1, 256, 0, s>>>(L->ws.slab_idx, L->ws.slab_cnt, L->R, L->gps * kGroup,
                                        idx_x, n_x);
  return cudaGetLastError();
}

}  // namespace prox
