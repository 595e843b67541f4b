// Offline weight preparation (Prox §4.3 "Hardware-Aware Implementation"):
//  * pack_proxy_kernel: symmetric INT4 proxy of one [d_model, d_ff] bf16
//    matrix, groups of 128 input rows per channel, fp16 scales;
//  * interleave_proxy_kernel: gate and up codes (and scales) interleaved per
//    32-channel block, stored slice-major: the 512-byte column slice s of
//    input row i (16 blocks: 512 channels of both proxies) sits at
//    (s * d_model + i) * 512, so the kept rows of one slice are read in
//    ascending address order;
//  * gateup_records_kernel: channel-contiguous gate/up records for Stage 2.
#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {
namespace {

// One thread per (group, channel pair): two passes over the group's 128 rows.
__global__ void pack_proxy_kernel(const uint32_t* __restrict__ W, int F, uint8_t* __restrict__ codes,
                                  __half* __restrict__ scales) {
  const int half_f = F >> 1;
  const int b = blockIdx.x * blockDim.x + threadIdx.x;  // channel pair (2b, 2b+1)
  const int g = blockIdx.y;
  if (b >= half_f) return;
  const uint32_t* src = W + (size_t)g * kGroup * half_f + b;
  float amax0 = 0.f, amax1 = 0.f;
  for (int i = 0; i < kGroup; ++i) {
    const float2 w = bf16x2_to_f2(__ldg(src + (size_t)i * half_f));
    amax0 = fmaxf(amax0, fabsf(w.x));
    amax1 = fmaxf(amax1, fabsf(w.y));
  }
  // IEEE division then nearest-even to fp16.  amax has at most 8 significant
  // bits, so amax/7 is either exact or has a non-terminating binary expansion
  // of period 3 that can never sit on an fp16 rounding midpoint after the
  // fp32 rounding: the two roundings give the same fp16 as one exact rounding.
  const __half h0 = __float2half_rn(amax0 / 7.0f);
  const __half h1 = __float2half_rn(amax1 / 7.0f);
  scales[(size_t)g * F + 2 * b] = h0;
  scales[(size_t)g * F + 2 * b + 1] = h1;
  const float s0 = __half2float(h0), s1 = __half2float(h1);
  uint8_t* dst = codes + (size_t)g * kGroup * half_f + b;
  for (int i = 0; i < kGroup; ++i) {
    const float2 w = bf16x2_to_f2(__ldg(src + (size_t)i * half_f));
    int q0 = 0, q1 = 0;
    if (s0 > 0.f) q0 = min(7, max(-7, __float2int_rn(w.x / s0)));
    if (s1 > 0.f) q1 = min(7, max(-7, __float2int_rn(w.y / s1)));
    dst[(size_t)i * half_f] = (uint8_t)((q0 + 8) | ((q1 + 8) << 4));
  }
}

// pq: slice s of row i = for each of its 16 blocks of 32 channels: 16 B gate
// codes, 16 B up codes, at byte (s * d + i) * 512 (the last slice of a d_ff
// that is not a multiple of 512 is padded).  ps[g] = for each block: 32 gate
// scales, 32 up scales.
__global__ void interleave_proxy_kernel(const uint4* __restrict__ cg, const uint4* __restrict__ cu,
                                        const uint4* __restrict__ sg, const uint4* __restrict__ su,
                                        int d, int F, uint4* __restrict__ pq, uint4* __restrict__ ps) {
  const int nblk = F >> 5;
  const size_t n_code = (size_t)d * nblk;
  const size_t n_scale = (size_t)(d / kGroup) * nblk;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_code + n_scale; t += stride) {
    if (t < n_code) {
      // block b of row i (t = i * nblk + b): 16 bytes from each proxy
      const size_t i = t / nblk, b = t % nblk;
      const size_t o = (((b >> 4) * (size_t)d + i) * 16 + (b & 15)) * 2;
      pq[o] = cg[t];
      pq[o + 1] = cu[t];
    } else {
      const size_t u = t - n_code;  // (group, block): 32 halves = 4 uint4 per proxy
      for (int q = 0; q < 4; ++q) {
        ps[8 * u + q] = sg[4 * u + q];
        ps[8 * u + 4 + q] = su[4 * u + q];
      }
    }
  }
}

// wgu[j] = [W_gate[:, j] | W_up[:, j]] (bf16), via 32x32 shared-memory tiles.
__global__ void gateup_records_kernel(const uint16_t* __restrict__ Wg, const uint16_t* __restrict__ Wu,
                                      int d, int F, uint16_t* __restrict__ wgu) {
  __shared__ uint16_t tile[32][33];
  const uint16_t* W = blockIdx.z == 0 ? Wg : Wu;
  const int j0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int i = i0 + r, j = j0 + threadIdx.x;
    tile[r][threadIdx.x] = (i < d && j < F) ? W[(size_t)i * F + j] : (uint16_t)0;
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int j = j0 + r, i = i0 + threadIdx.x;
    if (j < F && i < d) wgu[((size_t)j * 2 + blockIdx.z) * d + i] = tile[threadIdx.x][r];
  }
}

}  // namespace

cudaError_t launch_pack_proxy(const uint16_t* W, int d, int F, uint8_t* codes,
                              uint16_t* scales, cudaStream_t s) {
  dim3 grid((F / 2 + 127) / 128, d / kGroup, 1);
  pack_proxy_kernel<<<grid, 128, 0, s>>>(reinterpret_cast<const uint32_t*>(W), F, codes,
                                         reinterpret_cast<__half*>(scales));
  return cudaGetLastError();
}

cudaError_t launch_interleave_proxy(const uint8_t* cg, const uint8_t* cu, const uint16_t* sg,
                                    const uint16_t* su, int d, int F, uint8_t* pq,
                                    uint16_t* ps, cudaStream_t s) {
  interleave_proxy_kernel<<<1184, 256, 0, s>>>(
      reinterpret_cast<const uint4*>(cg), reinterpret_cast<const uint4*>(cu),
      reinterpret_cast<const uint4*>(sg), reinterpret_cast<const uint4*>(su), d, F,
      reinterpret_cast<uint4*>(pq), reinterpret_cast<uint4*>(ps));
  return cudaGetLastError();
}

cudaError_t launch_gateup_records(const uint16_t* Wg, const uint16_t* Wu, int d, int F,
                                  uint16_t* wgu, cudaStream_t s) {
  dim3 grid((F + 31) / 32, (d + 31) / 32, 2);
  gateup_records_kernel<<<grid, dim3(32, 8, 1), 0, s>>>(Wg, Wu, d, F, wgu);
  return cudaGetLastError();
}

}  // namespace prox
