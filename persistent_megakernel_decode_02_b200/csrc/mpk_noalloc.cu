// Final RMSNorm + LM head + greedy argmax without any device allocation.
//
// For callers that cannot allocate device memory: for instance a serving
// framework whose memory pool owns all device memory and forbids cudaMalloc /
// cudaFree (which also synchronise the device) on its decode path.  The
// scratch this computation needs (one packed (value, index) maximum and one
// arrival counter per request) lives in a file-scope __device__ array instead
// of library-allocated memory.  The caller passes every input and output
// buffer.
#include <cuda_runtime.h>

#include <cstdint>
#include <cmath>
#include <cstring>
#include <mutex>

#include "mpk.h"

namespace {

constexpr int kMaxRequests = MPK_NOALLOC_MAX_REQUESTS;
constexpr int kMaxK = MPK_NOALLOC_MAX_K;
constexpr int kThreads = 256;
constexpr int kMaxDevices = 64;

// [0, kMaxRequests): per-request maxima; [kMaxRequests, 2*kMaxRequests): arrival counters.
static __device__ __align__(256) unsigned long long g_lmhead_scratch[2 * kMaxRequests];


__device__ __forceinline__ float lo16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi16(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ unsigned long long key_of(float v, uint32_t idx) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - idx);
}

// Block (bx, r): rows [bx*V/nb, (bx+1)*V/nb) of W for request r.  One warp per
// row; the block's maximum goes to scratch[r] by atomicMax and the last block
// of request r to arrive writes the token.
__global__ void __launch_bounds__(kThreads) lmhead_argmax_noalloc_kernel(
    const float* __restrict__ x, const uint16_t* __restrict__ nw, const uint16_t* __restrict__ W, int K, int V,
    float eps, unsigned long long* scratch, int64_t* tok, float* logits) {
  extern __shared__ __align__(16) float hsm[];
  __shared__ float ss_w[kThreads / 32];
  __shared__ unsigned long long best_w[kThreads / 32];
  __shared__ int last;
  const int r = blockIdx.y, nb = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* xr = x + (size_t)r * K;
  // RMSNorm statistics in a fixed order, then h = x * rinv * w (fp32).
  float ss = 0.f;
  for (int k = threadIdx.x; k < K; k += kThreads) ss = fmaf(xr[k], xr[k], ss);
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) ss_w[warp] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < kThreads / 32; ++w) tot += ss_w[w];
  const float rinv = 1.0f / sqrtf(tot / (float)K + eps);
  for (int k = threadIdx.x; k < K; k += kThreads) {
    const float wv = __uint_as_float((uint32_t)nw[k] << 16);
    hsm[k] = xr[k] * rinv * wv;
  }
  __syncthreads();

  const int row0 = (int)((long long)blockIdx.x * V / nb), row1 = (int)((long long)(blockIdx.x + 1) * V / nb);
  unsigned long long best = 0ull;
  for (int row = row0 + warp; row < row1; row += kThreads / 32) {
    const uint16_t* wr = W + (size_t)row * K;
    float a0 = 0.f, a1 = 0.f;
    for (int e = lane * 8; e < K; e += 256) {
      const uint4 wv = __ldg(reinterpret_cast<const uint4*>(wr + e));
      const float4 h0 = *reinterpret_cast<const float4*>(hsm + e);
      const float4 h1 = *reinterpret_cast<const float4*>(hsm + e + 4);
      a0 = fmaf(lo16(wv.x), h0.x, a0); a1 = fmaf(hi16(wv.x), h0.y, a1);
      a0 = fmaf(lo16(wv.y), h0.z, a0); a1 = fmaf(hi16(wv.y), h0.w, a1);
      a0 = fmaf(lo16(wv.z), h1.x, a0); a1 = fmaf(hi16(wv.z), h1.y, a1);
      a0 = fmaf(lo16(wv.w), h1.z, a0); a1 = fmaf(hi16(wv.w), h1.w, a1);
    }
    float v = a0 + a1;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) {
      if (logits != nullptr) logits[(size_t)r * V + row] = v;
      const unsigned long long key = key_of(v, (uint32_t)row);
      best = key > best ? key : best;
    }
  }
  if (lane == 0) best_w[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long b = 0ull;
    for (int w = 0; w < kThreads / 32; ++w) b = best_w[w] > b ? best_w[w] : b;
    atomicMax(scratch + r, b);
    __threadfence();
    const unsigned long long old = atomicAdd(scratch + kMaxRequests + r, 1ull);
    last = (old + 1ull == (unsigned long long)nb);
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    const unsigned long long key = atomicAdd(scratch + r, 0ull);
    tok[r] = (int64_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
  }
}

// Address of the scratch array in the current device's context.  The symbol's
// host-side name is not a device address, so the address is looked up with
// cudaGetSymbolAddress once per device and context: a context that was torn
// down and created again (cudaDeviceReset, for instance) maps the array at a
// new address, so the cache also keeps the id of the context it came from and
// looks the address up again when the current context's id differs.
typedef int (*CtxGetCurrentFn)(void**);
typedef int (*CtxGetIdFn)(void*, unsigned long long*);

cudaError_t current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool resolved = false;
  if (!resolved) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = cudaDriverEntryPointSymbolNotFound;
    cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1);
    if (e != cudaSuccess || q1 != cudaDriverEntryPointSuccess) return e != cudaSuccess ? e : cudaErrorNotSupported;
    e = cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2);
    if (e != cudaSuccess || q2 != cudaDriverEntryPointSuccess) return e != cudaSuccess ? e : cudaErrorNotSupported;
    get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
    resolved = true;
  }
  void* ctx = nullptr;
  if (get_current(&ctx) != 0 || ctx == nullptr) return cudaErrorDeviceUninitialized;
  if (get_id(ctx, id) != 0) return cudaErrorDeviceUninitialized;
  return cudaSuccess;
}

struct ScratchEntry {
  unsigned long long ctx_id;
  unsigned long long* addr;
};
ScratchEntry g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

cudaError_t scratch_on_current_device(int dev, unsigned long long** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  // no context may be current yet (the lookup below creates the device's
  // primary context); a missing id only means "look the address up"
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id) == cudaSuccess;
  if (!have_id || g_scratch[dev].addr == nullptr || g_scratch[dev].ctx_id != id) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_lmhead_scratch);
    if (e != cudaSuccess) return e;
    e = current_context_id(&id);
    g_scratch[dev].addr = static_cast<unsigned long long*>(p);
    g_scratch[dev].ctx_id = e == cudaSuccess ? id : 0ull;
    *out = g_scratch[dev].addr;
    if (e != cudaSuccess) g_scratch[dev].addr = nullptr;  // no id to tie it to: look it up on every call
    return cudaSuccess;
  }
  *out = g_scratch[dev].addr;
  return cudaSuccess;
}

// per calling thread, so concurrent callers never see each other's message
thread_local char g_noalloc_err[256] = "";

int noalloc_fail(int code, const char* msg) {
  std::strncpy(g_noalloc_err, msg, sizeof(g_noalloc_err) - 1);
  g_noalloc_err[sizeof(g_noalloc_err) - 1] = '\0';
  return code;
}

}  // namespace

extern "C" {

MPK_API int mpk_lmhead_argmax_noalloc(const float* x, const uint16_t* norm_w, const uint16_t* w_lm,
                                      int num_requests, int K, int V, float eps, int64_t* tokens_out,
                                      float* logits_out, void* stream) {
  g_noalloc_err[0] = '\0';
  if (!x || !norm_w || !w_lm || !tokens_out) return noalloc_fail(MPK_ERR_INVALID_ARG, "NULL pointer");
  if (num_requests < 1 || num_requests > kMaxRequests)
    return noalloc_fail(MPK_ERR_INVALID_ARG, "num_requests outside 1..MPK_NOALLOC_MAX_REQUESTS");
  if (K < 8 || K % 8 != 0 || K > kMaxK)
    return noalloc_fail(MPK_ERR_SHAPE, "K must be a multiple of 8 in 8..MPK_NOALLOC_MAX_K");
  if (V < 1) return noalloc_fail(MPK_ERR_SHAPE, "V must be positive");
  if (reinterpret_cast<uintptr_t>(w_lm) % 16 != 0)
    return noalloc_fail(MPK_ERR_INVALID_ARG, "w_lm must be 16-byte aligned");
  if (!(eps > 0.f) || !(eps < INFINITY)) return noalloc_fail(MPK_ERR_INVALID_ARG, "eps must be positive and finite");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(MPK_ERR_CUDA, cudaGetErrorString(e));
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return noalloc_fail(MPK_ERR_CUDA, cudaGetErrorString(e));
  unsigned long long* scratch = nullptr;
  e = scratch_on_current_device(dev, &scratch);
  if (e != cudaSuccess) return noalloc_fail(MPK_ERR_CUDA, cudaGetErrorString(e));
  // maxima and counters must start at zero; a memset allocates nothing
  e = cudaMemsetAsync(scratch, 0, sizeof(unsigned long long) * 2 * kMaxRequests, s);
  if (e != cudaSuccess) return noalloc_fail(MPK_ERR_CUDA, cudaGetErrorString(e));
  const int nb = V < 2 * sms ? V : 2 * sms;
  const size_t smem = (size_t)K * sizeof(float);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(lmhead_argmax_noalloc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return noalloc_fail(MPK_ERR_CUDA, cudaGetErrorString(e));
  }
  lmhead_argmax_noalloc_kernel<<<dim3(nb, num_requests), kThreads, smem, s>>>(x, norm_w, w_lm, K, V, eps, scratch,
                                                                               tokens_out, logits_out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return noalloc_fail(MPK_ERR_CUDA, cudaGetErrorString(e));
  return MPK_OK;
}

MPK_API const char* mpk_noalloc_last_error(void) { return g_noalloc_err; }

}  // extern "C"
