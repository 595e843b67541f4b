// Stage-1 threshold calibration (Prox App. A.7 "Calibration data and scale":
// the per-layer threshold is the empirical quantile of the layer's input
// magnitudes over the calibration set).
//
// Exact order statistic of |x| by a three-level radix select on the fp32 bit
// patterns of |x| (monotone for non-negative values): bits 30..20, 19..9 and
// 8..0.  Each level is one histogram kernel over all values (shared-memory
// histogram, merged with integer atomics) and one single-CTA kernel that picks
// the bin holding the wanted rank and clears the histogram.
#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {

namespace {

// scratch layout: [0, kHistBins) histogram; [kHistBins] prefix of the key
// found so far; [kHistBins+1], [kHistBins+2] remaining rank (lo, hi words).
constexpr int kPrefix = kHistBins;
constexpr int kRankLo = kHistBins + 1;
constexpr int kRankHi = kHistBins + 2;

__device__ __forceinline__ void level_params(int level, int* shift, int* nbins, int* match_shift) {
  if (level == 0) {
    *shift = 20; *nbins = 2048; *match_shift = 31;
  } else if (level == 1) {
    *shift = 9; *nbins = 2048; *match_shift = 20;
  } else {
    *shift = 0; *nbins = 512; *match_shift = 9;
  }
}

__global__ void __launch_bounds__(512) calib_hist_kernel(const float* __restrict__ X, size_t n,
                                                         int level, uint32_t* scratch) {
  __shared__ uint32_t sh[kHistBins];
  int shift, nbins, mshift;
  level_params(level, &shift, &nbins, &mshift);
  for (int b = threadIdx.x; b < nbins; b += blockDim.x) sh[b] = 0u;
  __syncthreads();
  const uint32_t prefix = level == 0 ? 0u : scratch[kPrefix];
  const uint32_t mask = (uint32_t)nbins - 1u;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint32_t key = __float_as_uint(fabsf(__ldg(X + i)));
    if (level == 0 || (key >> mshift) == prefix) atomicAdd(&sh[(key >> shift) & mask], 1u);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < nbins; b += blockDim.x)
    if (sh[b]) atomicAdd(&scratch[b], sh[b]);
}

// Picks the bin containing the remaining (0-based, ascending) rank.
__global__ void __launch_bounds__(1024) calib_select_kernel(uint32_t* scratch, int level,
                                                            float* tau_out) {
  __shared__ int s_scan[33];
  __shared__ int s_pick[2];
  int shift, nbins, mshift;
  level_params(level, &shift, &nbins, &mshift);
  const unsigned long long rank = (unsigned long long)scratch[kRankLo] |
                                  ((unsigned long long)scratch[kRankHi] << 32);
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  const int lo = min((int)threadIdx.x * per, nbins), hi = min(lo + per, nbins);
  // counts fit in 32 bits (n < 2^31 is checked on the host)
  int v = 0;
  for (int b = lo; b < hi; ++b) v += (int)scratch[b];
  int total;
  const int excl = block_exclusive_scan(v, s_scan, &total);
  unsigned long long before = (unsigned long long)excl;
  for (int b = lo; b < hi; ++b) {
    const unsigned long long hb = scratch[b];
    if (before <= rank && rank < before + hb) {
      s_pick[0] = b;
      s_pick[1] = (int)(rank - before);
    }
    before += hb;
  }
  __syncthreads();
  for (int b = lo; b < hi; ++b) scratch[b] = 0u;
  if (threadIdx.x == 0) {
    const int bits = level == 2 ? 9 : 11;
    const uint32_t prefix = level == 0 ? (uint32_t)s_pick[0]
                                       : ((scratch[kPrefix] << bits) | (uint32_t)s_pick[0]);
    scratch[kPrefix] = prefix;
    scratch[kRankLo] = (uint32_t)s_pick[1];
    scratch[kRankHi] = 0u;
    if (level == 2) *tau_out = __uint_as_float(prefix);
  }
}

__global__ void calib_init_kernel(uint32_t* scratch, unsigned long long rank) {
  for (int b = threadIdx.x; b < kHistBins; b += blockDim.x) scratch[b] = 0u;
  if (threadIdx.x == 0) {
    scratch[kPrefix] = 0u;
    scratch[kRankLo] = (uint32_t)(rank & 0xFFFFFFFFull);
    scratch[kRankHi] = (uint32_t)(rank >> 32);
  }
}

// Fixed scratch of the allocation-free calibration entry point: the histogram,
// the key prefix and the remaining rank (as in the allocated scratch), then
// room for spare words.  One per device; every call rewrites all of it.
constexpr int kStaticScratchWords = kHistBins + 8;
static __device__ __align__(256) uint32_t g_calib_scratch[kStaticScratchWords];

}  // namespace

cudaError_t calibrate_static_scratch(uint32_t** ptr) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_calib_scratch);
  *ptr = static_cast<uint32_t*>(p);
  return e;
}

cudaError_t launch_calibrate(const float* X, size_t n, unsigned long long rank,
                             uint32_t* scratch, float* tau_dev, cudaStream_t s) {
  calib_init_kernel<<<1, 1024, 0, s>>>(scratch, rank);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int blocks = (int)((n + 511) / 512);
  if (blocks > 1184) blocks = 1184;
  if (blocks < 1) blocks = 1;
  for (int level = 0; level < 3; ++level) {
    calib_hist_kernel<<<blocks, 512, 0, s>>>(X, n, level, scratch);
    calib_select_kernel<<<1, 1024, 0, s>>>(scratch, level, tau_dev);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace prox
