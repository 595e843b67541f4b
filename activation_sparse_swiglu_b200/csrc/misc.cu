// Harness kernels: unit-gain RMSNorm between stacked layers, a streaming copy
// used to measure the HBM bandwidth that rooflines are quoted against, and the
// debug compaction of a per-channel selection mask into an ascending list.
#include "prox_device.cuh"
#include "prox_internal.h"

namespace prox {
namespace {

// One CTA per row; fixed-order reduction so results are reproducible.
__global__ void __launch_bounds__(1024) rmsnorm_kernel(const float* __restrict__ y,
                                                       float* __restrict__ x, int d, float eps) {
  __shared__ float s_red[32];
  pdl_wait();
  pdl_trigger();
  const float* yr = y + (size_t)blockIdx.x * d;
  float* xr = x + (size_t)blockIdx.x * d;
  float ss = 0.f;
  for (int e = threadIdx.x; e < d; e += blockDim.x) ss = fmaf(yr[e], yr[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? s_red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) s_red[0] = v;
  }
  __syncthreads();
  const float inv = 1.0f / sqrtf(s_red[0] / (float)d + eps);
  for (int e = threadIdx.x; e < d; e += blockDim.x) xr[e] = yr[e] * inv;
}

__global__ void __launch_bounds__(256) copy_kernel(const uint4* __restrict__ src,
                                                   uint4* __restrict__ dst, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const uint4 a = ld_stream_v4(src + i);
    const uint4 b = ld_stream_v4(src + i + stride);
    const uint4 c = ld_stream_v4(src + i + 2 * stride);
    const uint4 e = ld_stream_v4(src + i + 3 * stride);
    dst[i] = a;
    dst[i + stride] = b;
    dst[i + 2 * stride] = c;
    dst[i + 3 * stride] = e;
  }
  for (; i < n; i += stride) dst[i] = ld_stream_v4(src + i);
}

// One CTA of 1024 threads: thread t owns entries [t*per, (t+1)*per).
__global__ void __launch_bounds__(1024) mask_to_list_kernel(const int32_t* __restrict__ mask,
                                                            int n, int32_t* __restrict__ list,
                                                            int32_t* count) {
  __shared__ int s_scan[33];
  const int per = (n + 1023) / 1024;
  const int lo = min((int)threadIdx.x * per, n), hi = min(lo + per, n);
  int c = 0;
  for (int i = lo; i < hi; ++i) c += mask[i] != 0;
  int total;
  int pos = block_exclusive_scan(c, s_scan, &total);
  for (int i = lo; i < hi; ++i)
    if (mask[i] != 0) list[pos++] = i;
  if (count && threadIdx.x == 0) *count = total;
}

}  // namespace

cudaError_t launch_mask_to_list(const int32_t* mask, int n, int32_t* list, int32_t* count,
                                cudaStream_t s) {
  mask_to_list_kernel<<<1, 1024, 0, s>>>(mask, n, list, count);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const float* y, float* x, int rows, int d, float eps,
                           cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows, 1, 1);
  cfg.blockDim = dim3(1024, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, rmsnorm_kernel, y, x, d, eps);
}

cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  copy_kernel<<<sms * 8, 256, 0, s>>>(reinterpret_cast<const uint4*>(src),
                                      reinterpret_cast<uint4*>(dst), bytes / 16);
  return cudaGetLastError();
}

}  // namespace prox
