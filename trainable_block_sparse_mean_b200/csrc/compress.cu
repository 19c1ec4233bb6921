// Stage 1: parameter-free compression of K into stage-1 kernels.
//
// "InfLLM-V2" paper notes, key design 3, and the MiniCPM4 "InfLLM v2" blog
// (semantic kernels): each kernel is the average of the l_C1 = 32 key vectors
// it covers, kernels overlap with stride s_C1 = 16.  The sum of 32 bf16 values
// is formed in fp64 (exact for all but pathologically spread magnitudes), the
// division by 32 is exact, and the result is rounded once to bf16 (nearest,
// ties to even).  The kernel is HBM-bound: it reads K once and writes K^C1.
#include "common.cuh"
#include "internal.cuh"
#include "kc1_mean.cuh"

namespace infv2 {
namespace {

// One thread per (kernel j, kv head g, 8-element slice c of the head dim).
__global__ void __launch_bounds__(256) compress_k_kernel(const uint16_t* __restrict__ k, int h_kv,
                                                         int nc, uint16_t* __restrict__ kc1) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)nc * h_kv * 16;
  if (tid >= total) return;
  const int c = (int)(tid & 15);
  const long long jg = tid >> 4;
  const int g = (int)(jg % h_kv);
  const int j = (int)(jg / h_kv);
  const size_t row_stride = (size_t)h_kv * 128;  // elements between consecutive tokens
  const uint16_t* src = k + (size_t)(16 * j) * row_stride + (size_t)g * 128 + c * 8;
  uint4 out = kc1_mean_slice(src, row_stride, nullptr, -1);
  *reinterpret_cast<uint4*>(kc1 + ((size_t)j * h_kv + g) * 128 + c * 8) = out;
}

}  // namespace

int launch_compress_k(const uint16_t* k, int n, int h_kv, uint16_t* kc1, cudaStream_t st) {
  const int nc = n >= 32 ? (n - 32) / 16 + 1 : 0;
  if (nc == 0) return INFV2_OK;
  const long long total = (long long)nc * h_kv * 16;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  compress_k_kernel<<<(unsigned)blocks, threads, 0, st>>>(k, h_kv, nc, kc1);
  return launch_status(cudaGetLastError());
}

}  // namespace infv2

using namespace infv2;

extern "C" int infv2_compress_k(const infv2_params* p, const void* k, int n, void* kc1,
                                infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0) return INFV2_ERR_INVALID_ARG;
  if (n >= p->l_c1 && (!k || !kc1)) return INFV2_ERR_INVALID_ARG;
  return launch_compress_k(static_cast<const uint16_t*>(k), n, p->h_kv, static_cast<uint16_t*>(kc1),
                           reinterpret_cast<cudaStream_t>(stream));
}
