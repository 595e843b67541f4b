// C ABI of the Prox library: argument checks, the layer handle, and the
// stream-ordered kernel chains of the decode step.
#include <atomic>
#include <cfloat>
#include <cmath>
#include <mutex>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

#include "prox_device.cuh"
#include "prox_internal.h"

namespace {

constexpr int kMaxDevices = 64;
// Device address of the static calibration scratch per device, and the CUDA
// context it was looked up in (a device reset makes a new context, in which
// the module and its static array are loaded anew).
std::atomic<uint32_t*> g_calib_scratch_addr[kMaxDevices];
std::atomic<void*> g_calib_scratch_ctx[kMaxDevices];
std::mutex g_calib_scratch_mu;

// The current driver context, read through the runtime's driver entry-point
// table (no link-time dependency on the driver library).  nullptr if the
// entry point is unavailable.
void* current_context() {
  using Fn = int (*)(void**);
  static Fn fn = []() -> Fn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<Fn>(p);
  }();
  void* ctx = nullptr;
  if (fn && fn(&ctx) != 0) ctx = nullptr;
  return ctx;
}

// Device memory of device `dev` (device-allocated or managed)?
bool on_device(const void* p, int dev) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) && at.device == dev;
}

thread_local std::string g_last_error;

// Test-only fault injection: when positive, the allocation that brings the
// count to zero fails as if the device were out of memory.
std::atomic<int> g_alloc_countdown{0};

cudaError_t dev_alloc(void** p, size_t bytes) {
  int c = g_alloc_countdown.load();
  while (c > 0 && !g_alloc_countdown.compare_exchange_weak(c, c - 1)) {
  }
  if (c == 1) {
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  return cudaMalloc(p, bytes);
}
template <typename T>
cudaError_t dev_alloc(T** p, size_t bytes) {
  void* v = nullptr;
  const cudaError_t e = dev_alloc(&v, bytes);
  *p = static_cast<T*>(v);
  return e;
}

prox_status fail(prox_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

prox_status cuda_fail(cudaError_t e, const char* what) {
  cudaGetLastError();  // clear the sticky-free error state of the runtime
  return fail(e == cudaErrorMemoryAllocation ? PROX_ENOMEM : PROX_ECUDA, "%s: %s", what,
              cudaGetErrorString(e));
}

#define PROX_CUDA(call, what)                         \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

prox_status check_shape(int d, int F) {
  if (d <= 0 || d % prox::kGroup != 0 || d > prox::kMaxDModel)
    return fail(PROX_EINVAL, "d_model=%d must be a positive multiple of 128 and <= %d", d,
                prox::kMaxDModel);
  if (F <= 0 || F % 32 != 0 || F > prox::kMaxDff)
    return fail(PROX_EINVAL, "d_ff=%d must be a positive multiple of 32 and <= %d", F,
                prox::kMaxDff);
  return PROX_OK;
}

prox_status check_device(int* dev, int* sms) {
  PROX_CUDA(cudaGetDevice(dev), "cudaGetDevice");
  int major = 0;
  PROX_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev),
            "cudaDeviceGetAttribute");
  if (major != 10) return fail(PROX_EUNSUPPORTED, "device %d is not sm_100 (major=%d)", *dev, major);
  PROX_CUDA(cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, *dev),
            "cudaDeviceGetAttribute");
  return PROX_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

void free_layer_buffers(prox_layer* L) {
  if (L->wgu) cudaFree(L->wgu);
  if (L->wd) cudaFree(L->wd);
  if (L->pq) cudaFree(L->pq);
  if (L->ps) cudaFree(L->ps);
  if (L->ws.base) cudaFree(L->ws.base);
  L->wgu = L->wd = nullptr;
  L->pq = nullptr;
  L->ps = nullptr;
  L->ws = prox::Workspace{};
}

prox_status alloc_workspace(prox_layer* L) {
  using prox::kHostChunkTokens;
  const size_t d = L->d, F = L->F;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t o_scores = take(F * 4);
  const size_t o_st = take(F * 4);
  const size_t o_g = take(F * 4);
  const size_t o_u = take(F * 4);
  const size_t o_mask = take(F * 4);
  const size_t o_idx = take(F * 4);
  const size_t o_stats = take(24);
  const size_t o_err = take(4);
  const size_t o_xchg = off;
  const size_t o_hist = take(2 * prox::kScoreBins * 4);
  const size_t o_chist = take(2 * 128 * 4);
  const size_t o_bucket = take((size_t)prox::kScoreBins * prox::kBucketCap * 16);
  const size_t o_st64 = take(F * 8);
  const size_t o_slist = take(F * 8);
  const size_t o_scnt = take((size_t)prox::kMaxCtas * 8);
  const size_t o_s1p = take(prox::stage1_part_floats(L->P) * 8);
  const size_t o_ypart = take((size_t)L->P * d * 8);
  const size_t o_gbar = take(8);
  const size_t xchg_bytes = off - o_xchg;
  // the batched step's scratch (max_batch > 1), in the same allocation
  size_t o_batch = 0;
  if (L->max_batch > 1) {
    prox::choose_batch_splits(L->d, L->F, L->num_sms, &L->b_s1, &L->b_s5, &L->b_ks);
    if (!prox::batch_fits(L->F, L->num_sms, L->b_ks))
      return fail(PROX_EUNSUPPORTED, "d_ff=%d on %d SMs exceeds the batched step's channel table",
                  L->F, L->num_sms);
    o_batch = take(prox::batch_ws_bytes(L->d, L->F, L->b_s1, L->b_s5, L->b_ks));
  }
  const size_t o_in = take((size_t)kHostChunkTokens * d * 4);
  const size_t o_out = take((size_t)kHostChunkTokens * d * 4);
  void* base = nullptr;
  PROX_CUDA(dev_alloc(&base, off), "cudaMalloc(workspace)");
  PROX_CUDA(cudaMemset(base, 0, off), "cudaMemset(workspace)");
  char* b = static_cast<char*>(base);
  prox::Workspace& w = L->ws;
  w.base = base;
  w.bytes = off;
  w.scores = reinterpret_cast<float*>(b + o_scores);
  w.s_tilde = reinterpret_cast<float*>(b + o_st);
  w.g_dbg = reinterpret_cast<float*>(b + o_g);
  w.u_dbg = reinterpret_cast<float*>(b + o_u);
  w.hist = reinterpret_cast<uint32_t*>(b + o_hist);
  w.chist = reinterpret_cast<uint32_t*>(b + o_chist);
  w.bucket = reinterpret_cast<unsigned long long*>(b + o_bucket);
  w.st64 = reinterpret_cast<unsigned long long*>(b + o_st64);
  w.sel_list = reinterpret_cast<unsigned long long*>(b + o_slist);
  w.sel_cnt = reinterpret_cast<unsigned long long*>(b + o_scnt);
  w.xchg = b + o_xchg;
  w.xchg_bytes = xchg_bytes;
  w.sel_mask = reinterpret_cast<int32_t*>(b + o_mask);
  w.idx_s = reinterpret_cast<int32_t*>(b + o_idx);
  w.s1_part = reinterpret_cast<unsigned long long*>(b + o_s1p);
  w.ypart = reinterpret_cast<unsigned long long*>(b + o_ypart);
  w.stats = reinterpret_cast<unsigned long long*>(b + o_stats);
  w.gbar = reinterpret_cast<unsigned long long*>(b + o_gbar);
  w.err = reinterpret_cast<int*>(b + o_err);
  w.stage_in = reinterpret_cast<float*>(b + o_in);
  if (L->max_batch > 1) {
    L->bws_base = b + o_batch;
    prox::carve_batch_ws(L->bws_base, L->d, L->F, L->b_s1, L->b_s5, L->b_ks, &L->bws);
  }
  w.stage_out = reinterpret_cast<float*>(b + o_out);
  return PROX_OK;
}

// One token of the forward step under the layer's Stage-2 rule (top-k or the
// score threshold) and value source.
prox::TokenLaunch forward_launch(const prox_layer* L, const float* x, float* out) {
  prox::TokenLaunch m;
  m.x = x;
  m.out = out;
  m.stage1 = true;
  m.mode = L->mask_mode == PROX_MASK_THRESHOLD ? 3 : 1;
  m.k = L->k;
  m.tau_s = L->tau_s;
  m.proxy_values = L->stage2_source == PROX_STAGE2_PROXY_VALUES;
  return m;
}

cudaError_t enqueue_token(const prox_layer* L, const float* x, float* out, cudaStream_t s) {
  return prox::launch_token(L, forward_launch(L, x, out), s, true);
}

cudaError_t enqueue_dense(const prox_layer* L, const float* x, float* out, cudaStream_t s) {
  prox::TokenLaunch m;
  m.x = x;
  m.out = out;
  m.stage1 = false;
  m.mode = 2;
  m.k = L->F;
  return prox::launch_token(L, m, s, true);
}

prox_status check_layer(const prox_layer* L) {
  if (L == nullptr) return fail(PROX_EINVAL, "layer handle is NULL");
  int dev = -1;
  PROX_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev != L->device)
    return fail(PROX_EINVAL, "layer lives on device %d but device %d is current", L->device, dev);
  return PROX_OK;
}

}  // namespace

extern "C" {

const char* prox_version(void) { return "prox-b200 0.1 (sm_100a)"; }

size_t prox_last_error(char* msg_host, size_t n) {
  if (msg_host && n) {
    const size_t m = g_last_error.size() < n - 1 ? g_last_error.size() : n - 1;
    memcpy(msg_host, g_last_error.data(), m);
    msg_host[m] = '\0';
  }
  return g_last_error.size();
}

prox_status prox_pack_proxy(const uint16_t* W, int d_model, int d_ff, int group, uint8_t* codes,
                            uint16_t* scales, void* stream) {
  prox_status st = check_shape(d_model, d_ff);
  if (st != PROX_OK) return st;
  if (group != prox::kGroup) return fail(PROX_EINVAL, "group must be 128 (got %d)", group);
  if (!W || !codes || !scales) return fail(PROX_EINVAL, "NULL pointer");
  if (!aligned16(W) || !aligned16(codes) || !aligned16(scales))
    return fail(PROX_EINVAL, "pointers must be 16-byte aligned");
  int dev, sms;
  if ((st = check_device(&dev, &sms)) != PROX_OK) return st;
  PROX_CUDA(prox::launch_pack_proxy(W, d_model, d_ff, codes, scales, as_stream(stream)),
            "pack_proxy launch");
  return PROX_OK;
}

prox_status prox_calibrate_thresholds(const float* X_cal, int n_tok, int d_model, float s1,
                                      float* tau_host, void* stream) {
  if (!tau_host) return fail(PROX_EINVAL, "tau_host is NULL");
  if (!(s1 >= 0.f && s1 <= 1.f)) return fail(PROX_EINVAL, "s1=%g must be in [0, 1]", (double)s1);
  if (n_tok <= 0 || d_model <= 0) return fail(PROX_EINVAL, "n_tok and d_model must be positive");
  const size_t n = (size_t)n_tok * (size_t)d_model;
  if (n >= (size_t)1 << 31) return fail(PROX_EINVAL, "at most 2^31-1 calibration values");
  if (!X_cal || !aligned16(X_cal)) return fail(PROX_EINVAL, "X_cal must be a 16-byte aligned pointer");
  if (s1 == 0.f) {
    *tau_host = 0.f;
    return PROX_OK;
  }
  int dev, sms;
  prox_status st = check_device(&dev, &sms);
  if (st != PROX_OK) return st;
  unsigned long long rank = (unsigned long long)std::floor((double)s1 * (double)n);
  if (rank >= n) rank = n - 1;
  cudaStream_t s = as_stream(stream);
  void* scratch = nullptr;
  PROX_CUDA(cudaMallocAsync(&scratch, (prox::kHistBins + 4) * 4 + 16, s), "cudaMallocAsync");
  uint32_t* sc = static_cast<uint32_t*>(scratch);
  float* tau_dev = reinterpret_cast<float*>(sc + prox::kHistBins + 4);
  cudaError_t e = prox::launch_calibrate(X_cal, n, rank, sc, tau_dev, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(tau_host, tau_dev, 4, cudaMemcpyDeviceToHost, s);
  cudaFreeAsync(scratch, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "calibrate");
  return PROX_OK;
}

prox_status prox_calibrate_thresholds_noalloc(const float* X_cal, int n_tok, int d_model,
                                              float s1, float* tau_dev, void* stream) {
  if (!tau_dev || !aligned4(tau_dev)) return fail(PROX_EINVAL, "tau_dev must be a 4-byte aligned device pointer");
  if (!(s1 >= 0.f && s1 <= 1.f)) return fail(PROX_EINVAL, "s1=%g must be in [0, 1]", (double)s1);
  if (n_tok <= 0 || d_model <= 0) return fail(PROX_EINVAL, "n_tok and d_model must be positive");
  const size_t n = (size_t)n_tok * (size_t)d_model;
  if (n >= (size_t)1 << 31)
    return fail(PROX_EINVAL, "n_tok * d_model = %zu exceeds the 2^31-1 values the fixed scratch counts", n);
  if (!X_cal || !aligned16(X_cal)) return fail(PROX_EINVAL, "X_cal must be a 16-byte aligned pointer");
  int dev, sms;
  prox_status st = check_device(&dev, &sms);
  if (st != PROX_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return fail(PROX_EUNSUPPORTED, "device ordinal %d out of range", dev);
  if (!on_device(X_cal, dev) || !on_device(tau_dev, dev))
    return fail(PROX_EINVAL, "X_cal and tau_dev must be device memory of the current device %d", dev);
  // The scratch address is looked up once per device and context, with that
  // device current (it is the caller's current device here).
  void* ctx = current_context();
  uint32_t* scratch = g_calib_scratch_addr[dev].load(std::memory_order_acquire);
  if (!scratch || g_calib_scratch_ctx[dev].load(std::memory_order_acquire) != ctx) {
    std::lock_guard<std::mutex> lock(g_calib_scratch_mu);
    scratch = g_calib_scratch_addr[dev].load(std::memory_order_relaxed);
    if (!scratch || g_calib_scratch_ctx[dev].load(std::memory_order_relaxed) != ctx) {
      PROX_CUDA(prox::calibrate_static_scratch(&scratch), "cudaGetSymbolAddress(calibration scratch)");
      g_calib_scratch_ctx[dev].store(ctx, std::memory_order_release);
      g_calib_scratch_addr[dev].store(scratch, std::memory_order_release);
    }
  }
  cudaStream_t s = as_stream(stream);
  if (s1 == 0.f) {
    PROX_CUDA(cudaMemsetAsync(tau_dev, 0, 4, s), "cudaMemsetAsync(tau)");
    return PROX_OK;
  }
  unsigned long long rank = (unsigned long long)std::floor((double)s1 * (double)n);
  if (rank >= n) rank = n - 1;
  PROX_CUDA(prox::launch_calibrate(X_cal, n, rank, scratch, tau_dev, s), "calibrate launch");
  return PROX_OK;
}

// The per-token kernel's geometry for L->d x L->F over L->P SMs (one CTA
// per SM): Stage 1's slices, kept-row capacity and copy depth, Stage 2's
// ring, and the shared memory of the launch; PROX_EUNSUPPORTED when the
// device has too few or too many SMs for the shape.  Host only.
static prox_status plan_token_kernel(prox_layer* L) {
  const int sms = L->P;
  if (sms < 1 || sms > prox::kMaxCtas)
    return fail(PROX_EUNSUPPORTED, "%d SMs: the per-token kernel supports 1 to %d CTAs", sms, prox::kMaxCtas);
  if ((L->F + sms - 1) / sms > 512)
    return fail(PROX_EUNSUPPORTED, "d_ff=%d over %d SMs exceeds 512 channels per CTA", L->F, sms);
  prox::choose_stage1_grid(L->d, L->F, sms, &L->C, &L->s1_lmax, &L->s1_depth);
  if (L->s1_depth < 2)
    return fail(PROX_EUNSUPPORTED,
                "d_model=%d, d_ff=%d over %d SMs: Stage 1's row tables leave no room for two k-tiles per warp",
                L->d, L->F, sms);
  size_t s2_smem = 0;
  prox::choose_stage2(L->d, L->F, sms, &L->ring_slots, &L->stage2_groups, &s2_smem);
  const size_t s1_smem = prox::stage1_smem_bytes(L->s1_lmax, L->s1_depth, L->d);
  L->token_smem = s1_smem > s2_smem ? s1_smem : s2_smem;
  if (L->token_smem > (size_t)prox::kMaxSmemPerBlock)
    return fail(PROX_EUNSUPPORTED, "per-token kernel shared memory %zu exceeds the per-CTA limit", L->token_smem);
  return PROX_OK;
}

prox_status prox_layer_create(const uint16_t* W_gate, const uint16_t* W_up, const uint16_t* W_down,
                              int d_model, int d_ff, float tau_x, int k, int max_batch,
                              void* stream, prox_layer** out_host) {
  if (!out_host) return fail(PROX_EINVAL, "out_host is NULL");
  *out_host = nullptr;
  prox_status st = check_shape(d_model, d_ff);
  if (st != PROX_OK) return st;
  if (k < 1 || k > d_ff) return fail(PROX_EINVAL, "k=%d must be in [1, d_ff=%d]", k, d_ff);
  if (max_batch < 1) return fail(PROX_EINVAL, "max_batch must be >= 1");
  if (!(tau_x >= 0.f) || std::isinf(tau_x)) return fail(PROX_EINVAL, "tau_x must be finite and >= 0");
  if (!W_gate || !W_up || !W_down) return fail(PROX_EINVAL, "NULL weight pointer");
  if (!aligned16(W_gate) || !aligned16(W_up) || !aligned16(W_down))
    return fail(PROX_EINVAL, "weight pointers must be 16-byte aligned");
  int dev, sms;
  if ((st = check_device(&dev, &sms)) != PROX_OK) return st;

  prox_layer* L = new (std::nothrow) prox_layer();
  if (!L) return fail(PROX_ENOMEM, "host allocation failed");
  L->d = d_model;
  L->F = d_ff;
  L->G = d_model / prox::kGroup;
  L->k = k;
  L->max_batch = max_batch;
  L->tau = tau_x;
  L->device = dev;
  L->num_sms = sms;
  L->P = sms;
  if ((st = plan_token_kernel(L)) != PROX_OK) {
    delete L;
    return st;
  }

  cudaStream_t s = as_stream(stream);
  const size_t d = d_model, F = d_ff;
  uint8_t *cg = nullptr, *cu = nullptr;
  uint16_t *sg = nullptr, *su = nullptr;
  cudaError_t e = cudaSuccess;
  auto step = [&](cudaError_t r) {
    if (e == cudaSuccess) e = r;
  };
  step(prox::setup_token_kernels());
  step(prox::setup_batch_kernels());
  step(dev_alloc(&L->wgu, 2 * F * d * 2));
  step(dev_alloc(&L->wd, F * d * 2));
  step(dev_alloc(&L->pq, (size_t)L->C * d * 512));  // slice-major, last slice padded
  step(dev_alloc(&L->ps, (size_t)L->G * F * 2 * 2));
  step(dev_alloc(&cg, d * F / 2));
  step(dev_alloc(&cu, d * F / 2));
  step(dev_alloc(&sg, (size_t)L->G * F * 2));
  step(dev_alloc(&su, (size_t)L->G * F * 2));
  if (e == cudaSuccess) {
    step(prox::launch_pack_proxy(W_gate, L->d, L->F, cg, sg, s));
    step(prox::launch_pack_proxy(W_up, L->d, L->F, cu, su, s));
    step(prox::launch_interleave_proxy(cg, cu, sg, su, L->d, L->F, L->pq, L->ps, s));
    step(prox::launch_gateup_records(W_gate, W_up, L->d, L->F, L->wgu, s));
    step(cudaMemcpyAsync(L->wd, W_down, F * d * 2, cudaMemcpyDeviceToDevice, s));
    step(cudaStreamSynchronize(s));
  }
  if (cg) cudaFree(cg);
  if (cu) cudaFree(cu);
  if (sg) cudaFree(sg);
  if (su) cudaFree(su);
  if (e != cudaSuccess) {
    free_layer_buffers(L);
    delete L;
    return cuda_fail(e, "prox_layer_create");
  }
  if ((st = alloc_workspace(L)) != PROX_OK) {
    free_layer_buffers(L);
    delete L;
    return st;
  }
  *out_host = L;
  return PROX_OK;
}

prox_status prox_debug_token_geometry(int d_model, int d_ff, int num_sms, int32_t* out_host) {
  if (!out_host) return fail(PROX_EINVAL, "out_host is NULL");
  prox_status st = check_shape(d_model, d_ff);
  if (st != PROX_OK) return st;
  prox_layer L;
  L.d = d_model;
  L.F = d_ff;
  L.G = d_model / prox::kGroup;
  L.P = num_sms;
  if ((st = plan_token_kernel(&L)) != PROX_OK) return st;
  out_host[0] = L.C;
  out_host[1] = L.s1_lmax;
  out_host[2] = L.s1_depth;
  out_host[3] = L.ring_slots;
  out_host[4] = L.stage2_groups;
  out_host[5] = (int32_t)L.token_smem;
  return PROX_OK;
}

prox_status prox_debug_wait_timeout(prox_layer* L, void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  PROX_CUDA(prox::launch_barrier_probe(L, as_stream(stream)), "barrier probe launch");
  return PROX_OK;
}

prox_status prox_debug_fail_alloc(int nth) {
  if (nth < 0) return fail(PROX_EINVAL, "nth=%d must be >= 0", nth);
  g_alloc_countdown.store(nth);
  return PROX_OK;
}

prox_status prox_layer_destroy(prox_layer* L) {
  if (!L) return PROX_OK;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != L->device) cudaSetDevice(L->device);
  free_layer_buffers(L);
  if (cur != L->device) cudaSetDevice(cur);
  delete L;
  return PROX_OK;
}

prox_status prox_layer_set_tau(prox_layer* L, float tau_x) {
  if (!L) return fail(PROX_EINVAL, "layer handle is NULL");
  if (!(tau_x >= 0.f) || std::isinf(tau_x)) return fail(PROX_EINVAL, "tau_x must be finite and >= 0");
  L->tau = tau_x;
  return PROX_OK;
}

prox_status prox_layer_set_k(prox_layer* L, int k) {
  if (!L) return fail(PROX_EINVAL, "layer handle is NULL");
  if (k < 1 || k > L->F) return fail(PROX_EINVAL, "k=%d must be in [1, d_ff=%d]", k, L->F);
  L->k = k;
  return PROX_OK;
}

prox_status prox_layer_set_mask(prox_layer* L, int mode, float tau_s) {
  if (!L) return fail(PROX_EINVAL, "layer handle is NULL");
  if (mode != PROX_MASK_TOPK && mode != PROX_MASK_THRESHOLD)
    return fail(PROX_EINVAL, "mask mode %d is neither PROX_MASK_TOPK nor PROX_MASK_THRESHOLD", mode);
  if (mode == PROX_MASK_THRESHOLD && !(tau_s >= 0.f && tau_s <= FLT_MAX))
    return fail(PROX_EINVAL, "tau_s=%g must be finite and >= 0", (double)tau_s);
  L->mask_mode = mode;
  L->tau_s = mode == PROX_MASK_THRESHOLD ? tau_s : 0.f;
  return PROX_OK;
}

prox_status prox_layer_set_activation(prox_layer* L, int act) {
  if (!L) return fail(PROX_EINVAL, "layer handle is NULL");
  if (act != PROX_ACT_SILU && act != PROX_ACT_GELU_TANH && act != PROX_ACT_GELU_ERF)
    return fail(PROX_EINVAL, "activation %d is not one of PROX_ACT_*", act);
  L->act = act;
  return PROX_OK;
}

prox_status prox_layer_set_stage2(prox_layer* L, int source) {
  if (!L) return fail(PROX_EINVAL, "layer handle is NULL");
  if (source != PROX_STAGE2_EXACT && source != PROX_STAGE2_PROXY_VALUES)
    return fail(PROX_EINVAL, "Stage-2 source %d is not one of PROX_STAGE2_*", source);
  L->stage2_source = source;
  return PROX_OK;
}

prox_status prox_layer_get_info(const prox_layer* L, prox_layer_info* info) {
  if (!L || !info) return fail(PROX_EINVAL, "NULL argument");
  info->d_model = L->d;
  info->d_ff = L->F;
  info->group = prox::kGroup;
  info->k = L->k;
  info->max_batch = L->max_batch;
  info->tau_x = L->tau;
  info->stage1_col_slices = L->C;
  info->stage1_ctas = L->P;
  info->stage2_ctas = L->P;
  info->stage2_ring_slots = L->ring_slots;
  info->weight_bytes = (size_t)3 * L->F * L->d * 2;
  info->proxy_bytes = (size_t)L->d * L->F + (size_t)L->G * L->F * 4;
  info->workspace_bytes = L->ws.bytes;
  info->mask_mode = L->mask_mode;
  info->tau_s = L->tau_s;
  info->activation = L->act;
  info->stage2_source = L->stage2_source;
  return PROX_OK;
}

prox_status prox_layer_error(prox_layer* L, int32_t* word_host, void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (!word_host) return fail(PROX_EINVAL, "word_host is NULL");
  cudaStream_t s = as_stream(stream);
  int32_t v = 0;
  PROX_CUDA(cudaMemcpyAsync(&v, L->ws.err, 4, cudaMemcpyDeviceToHost, s), "read error word");
  PROX_CUDA(cudaMemsetAsync(L->ws.err, 0, 4, s), "clear error word");
  PROX_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  if (v & PROX_DEVERR_WAIT_TIMEOUT) {
    // A token whose wait ran out may have left the launch counter, the
    // histograms and the tagged exchange words mid-way: start the next token
    // clean (a counter back at 0 repeats earlier tags, so every tagged word
    // is cleared with it).
    PROX_CUDA(cudaMemsetAsync(L->ws.xchg, 0, L->ws.xchg_bytes, s), "reset exchange words");
    PROX_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  }
  *word_host = v;
  return PROX_OK;
}

prox_status prox_layer_stats(prox_layer* L, int64_t* sum_nx_host, int64_t* tokens_host,
                             int64_t* sum_sel_host, void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  cudaStream_t s = as_stream(stream);
  unsigned long long v[3] = {0, 0, 0};
  PROX_CUDA(cudaMemcpyAsync(v, L->ws.stats, 24, cudaMemcpyDeviceToHost, s), "read stats");
  PROX_CUDA(cudaMemsetAsync(L->ws.stats, 0, 24, s), "clear stats");
  PROX_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  if (sum_nx_host) *sum_nx_host = (int64_t)v[0];
  if (tokens_host) *tokens_host = (int64_t)v[1];
  if (sum_sel_host) *sum_sel_host = (int64_t)v[2];
  return PROX_OK;
}

// ---- cost model (Prox §4.2) and runtime sparsity (Prox App. A.7) ------------

prox_status prox_effective_sparsity(double s1, double s2, double alpha, double* e_host) {
  if (!e_host) return fail(PROX_EINVAL, "e_host is NULL");
  if (!(s1 >= 0.0 && s1 <= 1.0) || !(s2 >= 0.0 && s2 <= 1.0))
    return fail(PROX_EINVAL, "s1=%g and s2=%g must lie in [0, 1]", s1, s2);
  if (!(alpha >= 0.0) || std::isinf(alpha)) return fail(PROX_EINVAL, "alpha=%g must be finite and >= 0", alpha);
  *e_host = s2 - 2.0 * alpha * (1.0 - s1) / 3.0;
  return PROX_OK;
}

prox_status prox_allocate_sparsity(double e, double alpha, double s_ref, double s1_min,
                                   double s1_max, double* s1_host, double* s2_host) {
  if (!s1_host || !s2_host) return fail(PROX_EINVAL, "NULL output pointer");
  if (!std::isfinite(e)) return fail(PROX_EINVAL, "e must be finite");
  if (!(alpha > 0.0) || std::isinf(alpha)) return fail(PROX_EINVAL, "alpha=%g must be finite and > 0", alpha);
  if (!(s_ref >= 0.0 && s_ref <= 1.0)) return fail(PROX_EINVAL, "s_ref=%g must lie in [0, 1]", s_ref);
  if (!(s1_min >= 0.0 && s1_min <= s1_max && s1_max <= 1.0))
    return fail(PROX_EINVAL, "need 0 <= s1_min (%g) <= s1_max (%g) <= 1", s1_min, s1_max);
  // s2 = s_ref first; e = s2 - 2 alpha (1 - s1) / 3 then fixes s1.
  double s1 = 1.0 - 3.0 * (s_ref - e) / (2.0 * alpha);
  double s2 = s_ref;
  if (s1 < s1_min || s1 > s1_max) {
    s1 = s1 < s1_min ? s1_min : s1_max;
    s2 = e + 2.0 * alpha * (1.0 - s1) / 3.0;
    if (!(s2 >= 0.0 && s2 <= 1.0))
      return fail(PROX_EINVAL, "target e=%g is out of reach: s1 clamped to %g needs s2=%g", e, s1, s2);
  }
  *s1_host = s1;
  *s2_host = s2;
  return PROX_OK;
}

prox_status prox_runtime_sparsity(int64_t sum_nx, int64_t sum_sel, int64_t tokens, int d_model,
                                  int d_ff, double alpha, double* s1_host, double* s2_host,
                                  double* e_host) {
  if (tokens < 1 || d_model < 1 || d_ff < 1)
    return fail(PROX_EINVAL, "tokens, d_model and d_ff must be >= 1");
  if (tokens > INT64_MAX / (d_model > d_ff ? d_model : d_ff))
    return fail(PROX_EINVAL, "tokens=%lld too large", (long long)tokens);
  if (sum_nx < 0 || sum_nx > tokens * d_model || sum_sel < 0 || sum_sel > tokens * d_ff)
    return fail(PROX_EINVAL, "counts outside [0, tokens * width]");
  if (!(alpha >= 0.0) || std::isinf(alpha)) return fail(PROX_EINVAL, "alpha=%g must be finite and >= 0", alpha);
  const double s1 = 1.0 - (double)sum_nx / ((double)tokens * d_model);
  const double s2 = 1.0 - (double)sum_sel / ((double)tokens * d_ff);
  if (s1_host) *s1_host = s1;
  if (s2_host) *s2_host = s2;
  if (e_host) *e_host = s2 - 2.0 * alpha * (1.0 - s1) / 3.0;
  return PROX_OK;
}

prox_status prox_ffn_forward(const prox_layer* L, const float* x, float* out, int B,
                             void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (B < 1 || B > L->max_batch) return fail(PROX_EINVAL, "B=%d must be in [1, %d]", B, L->max_batch);
  if (!x || !out || !aligned16(x) || !aligned16(out))
    return fail(PROX_EINVAL, "x and out must be non-NULL 16-byte aligned pointers");
  if (x == out) return fail(PROX_EINVAL, "out may not alias x");
  cudaStream_t s = as_stream(stream);
  for (int b = 0; b < B; ++b) {
    cudaError_t e = enqueue_token(L, x + (size_t)b * L->d, out + (size_t)b * L->d, s);
    if (e != cudaSuccess) return cuda_fail(e, "prox_ffn_forward launch");
  }
  return PROX_OK;
}

prox_status prox_dense_ffn(const prox_layer* L, const float* x, float* out, int B, void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (B < 1 || B > L->max_batch) return fail(PROX_EINVAL, "B=%d must be in [1, %d]", B, L->max_batch);
  if (!x || !out || !aligned16(x) || !aligned16(out))
    return fail(PROX_EINVAL, "x and out must be non-NULL 16-byte aligned pointers");
  cudaStream_t s = as_stream(stream);
  for (int b = 0; b < B; ++b) {
    cudaError_t e = enqueue_dense(L, x + (size_t)b * L->d, out + (size_t)b * L->d, s);
    if (e != cudaSuccess) return cuda_fail(e, "prox_dense_ffn launch");
  }
  return PROX_OK;
}

namespace {
prox_status batch_call(const prox_layer* L, const float* x, float* out, int B, bool dense, void* stream,
                       const char* what) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (!L->bws_base) return fail(PROX_EINVAL, "%s needs a layer created with max_batch > 1", what);
  const int bmax = L->max_batch < prox::kBatchMax ? L->max_batch : prox::kBatchMax;
  if (B < 1 || B > bmax) return fail(PROX_EINVAL, "B=%d must be in [1, %d]", B, bmax);
  if (!x || !out || !aligned16(x) || !aligned16(out))
    return fail(PROX_EINVAL, "x and out must be non-NULL 16-byte aligned pointers");
  if (x == out) return fail(PROX_EINVAL, "out may not alias x");
  if (!dense && L->stage2_source != PROX_STAGE2_EXACT)
    return fail(PROX_EUNSUPPORTED, "%s computes the exact Stage 2 only", what);
  PROX_CUDA(prox::launch_batch(L, x, out, B, dense, as_stream(stream)), what);
  return PROX_OK;
}
}  // namespace

prox_status prox_ffn_forward_batch(const prox_layer* L, const float* x, float* out, int B, void* stream) {
  return batch_call(L, x, out, B, false, stream, "prox_ffn_forward_batch");
}

prox_status prox_dense_ffn_batch(const prox_layer* L, const float* x, float* out, int B, void* stream) {
  return batch_call(L, x, out, B, true, stream, "prox_dense_ffn_batch");
}

prox_status prox_batch_union_sizes(const prox_layer* L, int32_t* rows_host, int32_t* channels_host,
                                   void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (!L->bws_base) return fail(PROX_EINVAL, "the layer has no batched step (max_batch == 1)");
  if (!rows_host || !channels_host) return fail(PROX_EINVAL, "NULL output");
  int32_t v[2] = {0, 0};
  cudaStream_t s = as_stream(stream);
  PROX_CUDA(cudaMemcpyAsync(v, L->bws.cnt, 8, cudaMemcpyDeviceToHost, s), "read union sizes");
  PROX_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  *rows_host = v[0];
  *channels_host = v[1];
  return PROX_OK;
}

prox_status prox_debug_batch_masks(const prox_layer* L, int32_t* masks, int B, void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (!L->bws_base) return fail(PROX_EINVAL, "the layer has no batched step (max_batch == 1)");
  if (!masks || B < 1 || B > prox::kBatchMax) return fail(PROX_EINVAL, "masks NULL or B out of [1, 16]");
  PROX_CUDA(cudaMemcpyAsync(masks, L->bws.smask, (size_t)B * L->F * 4, cudaMemcpyDeviceToDevice,
                            as_stream(stream)),
            "copy batch masks");
  return PROX_OK;
}

prox_status prox_ffn_forward_host(prox_layer* L, const float* x_host, float* out_host, int n_tok,
                                  void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (!x_host || !out_host || n_tok < 0) return fail(PROX_EINVAL, "bad host buffers");
  cudaStream_t s = as_stream(stream);
  const size_t d = L->d;
  for (int t0 = 0; t0 < n_tok; t0 += prox::kHostChunkTokens) {
    const int n = n_tok - t0 < prox::kHostChunkTokens ? n_tok - t0 : prox::kHostChunkTokens;
    PROX_CUDA(cudaMemcpyAsync(L->ws.stage_in, x_host + t0 * d, n * d * 4,
                              cudaMemcpyHostToDevice, s),
              "H2D copy");
    for (int t = 0; t < n; ++t) {
      cudaError_t e = enqueue_token(L, L->ws.stage_in + t * d, L->ws.stage_out + t * d, s);
      if (e != cudaSuccess) return cuda_fail(e, "prox_ffn_forward_host launch");
    }
    PROX_CUDA(cudaMemcpyAsync(out_host + t0 * d, L->ws.stage_out, n * d * 4,
                              cudaMemcpyDeviceToHost, s),
              "D2H copy");
  }
  PROX_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  return PROX_OK;
}

prox_status prox_ffn_forward_profiled(const prox_layer* L, const float* x, float* out,
                                      void* const* events, uint64_t* phase_ns, void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (!events || !x || !out) return fail(PROX_EINVAL, "NULL argument");
  if (!aligned16(x) || !aligned16(out)) return fail(PROX_EINVAL, "x and out must be 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  prox::TokenLaunch m = forward_launch(L, x, out);
  m.phase_ns = reinterpret_cast<unsigned long long*>(phase_ns);
  PROX_CUDA(cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[0]), s), "cudaEventRecord");
  PROX_CUDA(prox::launch_token(L, m, s, false), "token launch");
  PROX_CUDA(cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[1]), s), "cudaEventRecord");
  return PROX_OK;
}

prox_status prox_debug_stage1(prox_layer* L, const float* x, int32_t* idx_x, int32_t* n_x,
                              float* g_tilde, float* u_tilde, int32_t* idx_s, void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (!x || !aligned16(x)) return fail(PROX_EINVAL, "x must be a 16-byte aligned pointer");
  if (idx_s && L->mask_mode != PROX_MASK_TOPK)
    return fail(PROX_EINVAL, "idx_s holds k channels under top-k only; use prox_debug_mask");
  cudaStream_t s = as_stream(stream);
  // the forward step of the token, stopped after the channel selection
  prox::TokenLaunch m = forward_launch(L, x, nullptr);
  m.taps.g = g_tilde;
  m.taps.u = u_tilde;
  m.taps.idx_x = idx_x;
  m.taps.n_x = n_x;
  m.select_only = true;
  m.sel_mask = L->ws.sel_mask;
  PROX_CUDA(prox::launch_token(L, m, s, false), "token launch");
  if (idx_s)
    PROX_CUDA(prox::launch_mask_to_list(L->ws.sel_mask, L->F, idx_s, nullptr, s),
              "mask compaction launch");
  return PROX_OK;
}

prox_status prox_debug_mask(const prox_layer* L, const float* x, int32_t* idx_s, int32_t* n_s,
                            void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (!x || !aligned16(x) || !idx_s || !n_s)
    return fail(PROX_EINVAL, "x (16-byte aligned), idx_s and n_s must be non-NULL");
  cudaStream_t s = as_stream(stream);
  prox::TokenLaunch m = forward_launch(L, x, nullptr);
  m.select_only = true;
  m.sel_mask = L->ws.sel_mask;
  PROX_CUDA(prox::launch_token(L, m, s, false), "token launch");
  PROX_CUDA(prox::launch_mask_to_list(L->ws.sel_mask, L->F, idx_s, n_s, s), "mask compaction launch");
  return PROX_OK;
}

prox_status prox_layer_proxy_scores(const prox_layer* L, const float* x, int B, float* scores,
                                    void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (B < 1) return fail(PROX_EINVAL, "B=%d must be >= 1", B);
  if (!x || !scores || !aligned16(x)) return fail(PROX_EINVAL, "x (16-byte aligned) and scores must be non-NULL");
  cudaStream_t s = as_stream(stream);
  for (int b = 0; b < B; ++b) {
    prox::TokenLaunch m;
    m.x = x + (size_t)b * L->d;
    m.stage1 = true;
    m.mode = -1;
    PROX_CUDA(prox::launch_token(L, m, s, false), "token launch");
    PROX_CUDA(cudaMemcpyAsync(scores + (size_t)b * L->F, L->ws.scores, (size_t)L->F * 4,
                              cudaMemcpyDeviceToDevice, s), "copy scores");
  }
  return PROX_OK;
}

prox_status prox_forward_with_mask(prox_layer* L, const float* x, const int32_t* idx_s, int k,
                                   float* out, float* s_sp, void* stream) {
  prox_status st = check_layer(L);
  if (st != PROX_OK) return st;
  if (k < 1 || k > L->F) return fail(PROX_EINVAL, "k=%d must be in [1, d_ff=%d]", k, L->F);
  if (!x || !out || !idx_s || !aligned16(x) || !aligned16(out))
    return fail(PROX_EINVAL, "bad pointer");
  cudaStream_t s = as_stream(stream);
  prox::TokenLaunch m;
  m.x = x;
  m.out = out;
  m.stage1 = false;
  m.mode = 0;
  m.idx = idx_s;
  m.k = k;
  m.s_sp = s_sp;
  PROX_CUDA(prox::launch_token(L, m, s, false), "token launch");
  return PROX_OK;
}

prox_status prox_rmsnorm(const float* y, float* x_out, int rows, int d, float eps, void* stream) {
  if (!y || !x_out || rows < 1 || d < 1 || !(eps >= 0.f))
    return fail(PROX_EINVAL, "bad rmsnorm arguments");
  PROX_CUDA(prox::launch_rmsnorm(y, x_out, rows, d, eps, as_stream(stream)), "rmsnorm launch");
  return PROX_OK;
}

prox_status prox_copy(const void* src, void* dst, size_t bytes, void* stream) {
  if (!src || !dst || (bytes & 15u) || !aligned16(src) || !aligned16(dst))
    return fail(PROX_EINVAL, "copy needs 16-byte aligned pointers and a multiple of 16 bytes");
  PROX_CUDA(prox::launch_copy(src, dst, bytes, as_stream(stream)), "copy launch");
  return PROX_OK;
}

}  // extern "C"
