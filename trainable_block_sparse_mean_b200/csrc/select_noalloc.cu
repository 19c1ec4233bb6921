// Block selection without any device allocation.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// running under a memory pool or arena it does not own, an inference engine
// whose allocator is frozen after start-up, or a plugin that only receives
// input and output pointers.  infv2_select_blocks_noalloc serves them: it runs
// the same score and selection kernels as infv2_block_scores +
// infv2_select_topk, but keeps the intermediate S^shared rows in a fixed
// device array owned by this library instead of caller memory.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it (kScratchBytes) until the process exits.  Host code cannot
// use the array's name as a device address; its address is looked up once per
// device with cudaGetSymbolAddress (on the first call made on that device,
// which therefore should come before any stream capture) and passed to the
// kernels (again whenever the device's context has changed, e.g. after a
// device reset).  All calls share the array: calls that overlap on the GPU (other
// streams, other threads) race on it and must be serialised by the caller.
// Nothing in it needs clearing: every element the selection reads is written
// earlier in the same call.
#include <mutex>

#include "internal.cuh"

namespace infv2 {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB of S^shared rows
constexpr int kMinRowsPerChunk = 128;               // one full score tile of tokens

static __device__ __align__(256) float g_noalloc_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
float* g_scratch_addr[kMaxDevices];
uintptr_t g_scratch_ctx[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up once per
// device and context: an address is only valid in the context it came from).
float* scratch_address(int* status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *status = INFV2_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev] || g_scratch_ctx[dev] != current_context()) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      *status = INFV2_ERR_CUDA;
      return nullptr;
    }
    g_scratch_addr[dev] = static_cast<float*>(p);
    g_scratch_ctx[dev] = current_context();
  }
  *status = INFV2_OK;
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace infv2

using namespace infv2;

extern "C" int infv2_select_blocks_noalloc(const infv2_params* p, const void* q, const void* kc1,
                                           int n, int q_begin, int q_len, int* idx,
                                           infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0 || q_begin < 0 || q_len < 0 || q_begin + q_len > n) return INFV2_ERR_INVALID_ARG;
  if (q_len == 0) return INFV2_OK;
  const int nc = infv2_num_kernels(p, n);
  if (!q || !idx || (nc > 0 && !kc1)) return INFV2_ERR_INVALID_ARG;
  const int ld = shared_ld(n);
  const size_t row_bytes = (size_t)p->h_kv * ld * sizeof(float);
  // the fixed array must hold the S^shared rows of at least one score tile
  if (row_bytes * kMinRowsPerChunk > kScratchBytes) return INFV2_ERR_UNSUPPORTED;
  float* scratch = scratch_address(&st);
  if (!scratch) return st;
  // whole score tiles per chunk (128 rows): no chunk ends on a partial tile
  const int chunk = (int)(kScratchBytes / row_bytes) / kMinRowsPerChunk * kMinRowsPerChunk;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t* qb = static_cast<const uint16_t*>(q);
  const uint16_t* kb = static_cast<const uint16_t*>(kc1);
  for (int q0 = q_begin; q0 < q_begin + q_len; q0 += chunk) {
    const int ql = q_begin + q_len - q0 < chunk ? q_begin + q_len - q0 : chunk;
    if (nc > 0) {
      st = launch_block_scores(p, qb, kb, n, q0, ql, scratch, ld, nullptr, cs);
      if (st != INFV2_OK) return st;
    }
    st = launch_select(p, scratch, ld, n, q0, ql, idx, (long long)n * p->k, cs);
    if (st != INFV2_OK) return st;
  }
  return INFV2_OK;
}
