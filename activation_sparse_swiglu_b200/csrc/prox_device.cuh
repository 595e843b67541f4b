// Device-side helpers shared by the Prox kernels (sm_100a only).
//
// Inline PTX for: 1-D bulk async copies (TMA engine, global -> shared) that
// complete on an mbarrier, mbarrier waits with an upper bound on their
// duration, programmatic dependent launch, and streaming loads.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "prox.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace prox {

// Upper bound for any wait on an mbarrier: about 0.1 s at B200 clocks.  A
// wait that runs out sets PROX_DEVERR_WAIT_TIMEOUT and the kernel carries on
// (later waits of the same thread give up at once), so a lost copy can never
// hang the GPU.
constexpr long long kWaitLimitCycles = 200000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- programmatic dependent launch ----------------------------------------
// pdl_wait blocks until the preceding kernel in the stream has completed and
// its writes are visible; it is a no-op when the launch had no programmatic
// dependency.  pdl_trigger lets the next kernel in the stream start its
// prologue early (it still waits in its own pdl_wait before reading our output).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
// Make mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count)
               : "memory");
}
// The waiting thread may be suspended until the phase completes, for at most
// kWaitSuspendNs per try, so a wait costs few issue slots.
constexpr uint32_t kWaitSuspendNs = 100000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(kWaitSuspendNs)
      : "memory");
  return ok != 0;
}
// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete, for at most
// kWaitLimitCycles.  Returns false (after flagging `err` and setting *dead)
// if it ran out; with *dead already set it returns false at once.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err,
                                          bool* dead = nullptr) {
  if (mbar_try_wait(bar, parity)) return true;
  if (dead && *dead) return false;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) {
      if (err) atomicOr(err, PROX_DEVERR_WAIT_TIMEOUT);
      if (dead) *dead = true;
      return false;
    }
  }
  return true;
}

// ---- bulk async copy (TMA engine), global -> this CTA's shared memory ------
// dst/src 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---- loads -------------------------------------------------------------------
// Streaming 16-byte load of read-only weights: no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 lds_v4(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ float4 lds_f4(const void* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(smem_u32(p)));
  return v;
}

// ---- bf16 pairs ----------------------------------------------------------------
// A 32-bit word holding two bf16 values (element 2m in the low half) widened
// to a float2 exactly.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// SiLU(z) = z / (1 + e^{-z}) in fp32.
__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

// Gate activations of the GLU: SiLU (SwiGLU, Prox §2.1) or GELU (GeGLU, the
// FFN family Prox §5 also sparsifies), the latter either as z Phi(z) or in the
// tanh form of Hendrycks & Gimpel, "Gaussian Error Linear Units", §2:
//   0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).
// `act` is uniform across the grid (a kernel argument), so the branch costs
// nothing.  Values follow PROX_ACT_* of prox.h.
__device__ __forceinline__ float act_f32(float z, int act) {
  if (act == 1) {
    const float c = 0.7978845608028654f;  // sqrt(2/pi)
    return 0.5f * z * (1.0f + tanhf(c * fmaf(0.044715f * z, z * z, z)));
  }
  if (act == 2) return 0.5f * z * erfcf(-z * 0.7071067811865476f);  // z Phi(z)
  return silu_f32(z);
}

// ---- block-wide scans (blockDim.x a multiple of 32, at most 1024) ---------------
// Exclusive prefix sum of `v` over the threads of the block in thread order.
// `scratch` needs 33 words of shared memory.  Returns the block total in *total.
template <typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T* scratch, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  T incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    T w = lane < nwarps ? scratch[lane] : T(0);
    T wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      T n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < nwarps) scratch[lane] = wi - w;  // exclusive warp offsets
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  const T out = scratch[warp] + incl - v;
  *total = scratch[32];
  __syncthreads();
  return out;
}

}  // namespace prox
