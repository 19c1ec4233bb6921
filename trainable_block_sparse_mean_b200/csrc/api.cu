// Host-side utilities of libinfv2: parameter checks, status strings, the
// per-device kernel error word, tensor-map creation and the timeout self-test.
#include <math.h>
#include <mutex>
#include <stdio.h>
#include <stdlib.h>

#include "common.cuh"

namespace infv2 {

namespace {
__device__ int g_error_word;  // first kernel failure on this device (0 = none)

constexpr int kMaxDevices = 64;
int* g_error_ptr[kMaxDevices];
uintptr_t g_error_ctx[kMaxDevices];
int g_sm_count[kMaxDevices];
std::mutex g_mu;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}
}  // namespace

uintptr_t current_context() {
  typedef CUresult (*GetCtxFn)(CUcontext*);
  static GetCtxFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (GetCtxFn) nullptr;
    return (GetCtxFn)p;
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return 0;
  return reinterpret_cast<uintptr_t>(c);
}

int* error_word() {
  int dev = current_device();
  if (dev < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  // a cached address belongs to the context that looked it up (a device reset
  // makes a new one)
  if (!g_error_ptr[dev] || g_error_ctx[dev] != current_context()) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_error_ptr[dev] = static_cast<int*>(p);
    g_error_ctx[dev] = current_context();
  }
  return g_error_ptr[dev];
}

uint64_t wait_timeout_ns() {
  static uint64_t t = [] {
    const char* e = getenv("INFV2_WAIT_TIMEOUT_MS");
    double ms = e ? atof(e) : 2000.0;
    if (!(ms > 0)) ms = 2000.0;
    return (uint64_t)(ms * 1e6);
  }();
  return t;
}

int sm_count() {
  int dev = current_device();
  if (dev < 0) return 148;
  if (!g_sm_count[dev]) {
    int c = 0;
    cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
    g_sm_count[dev] = c > 0 ? c : 148;
  }
  return g_sm_count[dev];
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? INFV2_OK : INFV2_ERR_CUDA; }

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return (EncodeTiledFn)p;
  }();
  return fn;
}
}  // namespace

bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                  uint32_t box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box0, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {
__global__ void timeout_selftest_kernel(WaitCtx w) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(smem_u32(&bar), 0, w);  // nobody arrives
  __syncthreads();
}
// y[i] = 2^x[i] through one of the kernels' exponential forms (self-test).
__global__ void exp2_selftest_kernel(int which, const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  float2 r;
  if (which == 0) {
    r = make_float2(fast_exp2(v.x), fast_exp2(v.y));
  } else if (which == 1) {
    r = exp2_fma2(v);
  } else {
    r = exp2_cubic2(v);
  }
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}
}  // namespace

}  // namespace infv2

using namespace infv2;

extern "C" {

void infv2_default_params(infv2_params* p, int h_q, int h_kv) {
  if (!p) return;
  p->B = 64;
  p->l_c1 = 32;
  p->s_c1 = 16;
  p->pool_l = 5;
  p->pool_s = 4;
  p->n_init = 1;
  p->n_local = 2;
  p->k = 64;
  p->h_q = h_q;
  p->h_kv = h_kv;
  p->d = 128;
  p->scale = 1.0f / sqrtf(128.0f);
  p->window = 0;
  p->lse_approx = 0;
}

int infv2_check_params(const infv2_params* p) {
  if (!p) return INFV2_ERR_INVALID_ARG;
  if (p->B <= 0 || p->l_c1 <= 0 || p->s_c1 <= 0 || p->pool_l <= 0 || p->pool_s <= 0 ||
      p->n_init < 0 || p->n_local < 1 || p->k <= 0 || p->h_q <= 0 || p->h_kv <= 0 || p->d <= 0 ||
      p->window < 0 || !(p->scale > 0.0f) || !isfinite(p->scale) ||
      (p->lse_approx != 0 && p->lse_approx != 1))
    return INFV2_ERR_INVALID_ARG;
  if (p->h_q % p->h_kv != 0) return INFV2_ERR_INVALID_ARG;
  if (p->k < p->n_init + p->n_local) return INFV2_ERR_INVALID_ARG;
  if (p->window > 0 && p->n_local < (p->window + p->B - 1) / p->B + 1) return INFV2_ERR_INVALID_ARG;
  const int G = p->h_q / p->h_kv;
  if (p->d != 128 || p->B != 64 || p->l_c1 != 32 || p->s_c1 != 16 || p->pool_l != 5 ||
      p->pool_s != 4)
    return INFV2_ERR_UNSUPPORTED;
  if (!(G == 1 || G == 2 || G == 4 || G == 8 || G == 16)) return INFV2_ERR_UNSUPPORTED;
  if (p->k > 256) return INFV2_ERR_UNSUPPORTED;
  return INFV2_OK;
}

const char* infv2_status_string(int status) {
  switch (status) {
    case INFV2_OK: return "ok";
    case INFV2_ERR_INVALID_ARG: return "invalid argument";
    case INFV2_ERR_UNSUPPORTED: return "unsupported by this build's kernels";
    case INFV2_ERR_WORKSPACE: return "workspace too small";
    case INFV2_ERR_CUDA: return "CUDA error";
    case INFV2_ERR_TIMEOUT: return "kernel wait timed out";
    case INFV2_ERR_CHECK: return "device-side check failed (INFV2_CHECKS build)";
    default: return "unknown status";
  }
}

int infv2_num_kernels(const infv2_params* p, int n) {
  if (!p || n < p->l_c1 || p->s_c1 <= 0) return 0;
  return (n - p->l_c1) / p->s_c1 + 1;
}

int infv2_device_status(infv2_stream_t stream) {
  int* w = error_word();
  if (!w) return INFV2_ERR_CUDA;
  int host = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&host, w, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return INFV2_ERR_CUDA;
  if (cudaMemsetAsync(w, 0, sizeof(int), s) != cudaSuccess) return INFV2_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return INFV2_ERR_CUDA;
  return host;
}

int infv2_get_device_status(infv2_stream_t stream) { return infv2_device_status(stream); }

int infv2_selftest_exp2(int which, const float* x, float* y, int n, infv2_stream_t stream) {
  if (which < 0 || which > 2 || n < 0) return INFV2_ERR_INVALID_ARG;
  if (n == 0) return INFV2_OK;
  if (!x || !y) return INFV2_ERR_INVALID_ARG;
  const int threads = 256, pairs = (n + 1) / 2;
  exp2_selftest_kernel<<<(pairs + threads - 1) / threads, threads, 0,
                         reinterpret_cast<cudaStream_t>(stream)>>>(which, x, y, n);
  return launch_status(cudaGetLastError());
}

int infv2_selftest_timeout(int limit_us, infv2_stream_t stream) {
  if (limit_us <= 0) return INFV2_ERR_INVALID_ARG;
  WaitCtx w{error_word(), (uint64_t)limit_us * 1000ull};
  if (!w.err) return INFV2_ERR_CUDA;
  timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(w);
  return launch_status(cudaGetLastError());
}

}  // extern "C"
