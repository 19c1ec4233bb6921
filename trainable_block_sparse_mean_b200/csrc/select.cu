// Stages 3-4 kernel: one warp per (kv head, query row); see select.cuh.
#include "common.cuh"
#include "internal.cuh"
#include "select.cuh"

namespace infv2 {
namespace {

struct SelectArgs {
  const float* s_shared;  // [h_kv, q_len, ld]
  int ld, q_begin, q_len, h_kv;
  int n_init, n_local, k;
  int* idx;               // idx[g * idx_hstride + i * k + :]
  long long idx_hstride;
  int keys_per_warp;      // shared words per warp for block keys
  int* err;               // device error word (debug-build checks)
};

__global__ void __launch_bounds__(256) select_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t sm_sel[];
  const int warp = threadIdx.x >> 5;
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  if (w >= (long long)a.h_kv * a.q_len) return;
  const int g = (int)(w / a.q_len);
  const int ii = (int)(w % a.q_len);
  const int i = a.q_begin + ii;
  uint32_t* keys = sm_sel + (size_t)warp * (a.keys_per_warp + 256);
  uint32_t* hist = keys + a.keys_per_warp;
  const float* row = a.s_shared + ((size_t)g * a.q_len + ii) * (size_t)a.ld;
  int* out = a.idx + (size_t)g * a.idx_hstride + (size_t)i * a.k;
  select_row_warp(row, visible_kernels(i, 32, 16), i, a.n_init, a.n_local, a.k, keys, hist, out,
                  a.err);
}

// Top-k only, from S^cmp rows (max pooling already done by the score kernel).
__global__ void __launch_bounds__(256) select_pooled_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint32_t sm_sel[];
  const int warp = threadIdx.x >> 5;
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  if (w >= (long long)a.h_kv * a.q_len) return;
  const int g = (int)(w / a.q_len);
  const int ii = (int)(w % a.q_len);
  const int i = a.q_begin + ii;
  uint32_t* keys = sm_sel + (size_t)warp * (a.keys_per_warp + 256);
  uint32_t* hist = keys + a.keys_per_warp;
  const float* row = a.s_shared + ((size_t)g * a.q_len + ii) * (size_t)a.ld;
  int* out = a.idx + (size_t)g * a.idx_hstride + (size_t)i * a.k;
  select_row_warp_pooled(row, i, a.n_init, a.n_local, a.k, keys, hist, out, a.err);
}

template <typename Kernel>
int launch_select_rows(Kernel kernel, const infv2_params* p, const float* rows, int ld, int n,
                       int q_begin, int q_len, int* idx, long long idx_hstride, cudaStream_t st) {
  if (q_len <= 0) return INFV2_OK;
  const int n_blk = (n + 63) / 64;
  const int keys_per_warp = ((n_blk + 3) / 4) * 4;
  const int per_warp_bytes = (keys_per_warp + 256) * 4;
  int warps = 8;
  while (warps > 1 && warps * per_warp_bytes > 200 * 1024) warps >>= 1;
  if (per_warp_bytes > 200 * 1024) return INFV2_ERR_UNSUPPORTED;
  const int smem = warps * per_warp_bytes;
  if (!set_smem(kernel, smem)) return INFV2_ERR_CUDA;
  SelectArgs a{rows, ld, q_begin, q_len, p->h_kv, p->n_init, p->n_local, p->k,
               idx, idx_hstride, keys_per_warp, error_word()};
  const long long n_rows = (long long)p->h_kv * q_len;
  const long long blocks = (n_rows + warps - 1) / warps;
  kernel<<<(unsigned)blocks, warps * 32, smem, st>>>(a);
  return launch_status(cudaGetLastError());
}

}  // namespace

int launch_select(const infv2_params* p, const float* s_shared, int ld, int n, int q_begin,
                  int q_len, int* idx, long long idx_hstride, cudaStream_t st) {
  return launch_select_rows(select_kernel, p, s_shared, ld, n, q_begin, q_len, idx, idx_hstride,
                            st);
}

int launch_select_pooled(const infv2_params* p, const float* s_cmp, int ld_cmp, int n,
                         int q_begin, int q_len, int* idx, long long idx_hstride,
                         cudaStream_t st) {
  return launch_select_rows(select_pooled_kernel, p, s_cmp, ld_cmp, n, q_begin, q_len, idx,
                            idx_hstride, st);
}

}  // namespace infv2

using namespace infv2;

extern "C" int infv2_select_topk(const infv2_params* p, const float* s_shared, int ld, int n,
                                 int q_begin, int q_len, int* idx, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0 || q_begin < 0 || q_len < 0 || q_begin + q_len > n) return INFV2_ERR_INVALID_ARG;
  if (q_len == 0) return INFV2_OK;
  if (!s_shared || !idx) return INFV2_ERR_INVALID_ARG;
  if (ld < infv2_num_kernels(p, n) || ld % 4 != 0) return INFV2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(s_shared) & 15) != 0) return INFV2_ERR_INVALID_ARG;
  return launch_select(p, s_shared, ld, n, q_begin, q_len, idx, (long long)n * p->k,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int infv2_select_topk_pooled(const infv2_params* p, const float* s_cmp, int ld_cmp,
                                        int n, int q_begin, int q_len, int* idx,
                                        infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0 || q_begin < 0 || q_len < 0 || q_begin + q_len > n) return INFV2_ERR_INVALID_ARG;
  if (q_len == 0) return INFV2_OK;
  if (!s_cmp || !idx) return INFV2_ERR_INVALID_ARG;
  if (ld_cmp < (n + p->B - 1) / p->B || ld_cmp % 4 != 0) return INFV2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(s_cmp) & 15) != 0) return INFV2_ERR_INVALID_ARG;
  return launch_select_pooled(p, s_cmp, ld_cmp, n, q_begin, q_len, idx, (long long)n * p->k,
                              reinterpret_cast<cudaStream_t>(stream));
}
