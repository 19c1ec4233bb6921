// Stage 1: parameter-free compression of K into stage-1 kernels.
//
// "InfLLM-V2" paper notes, key design 3, and the MiniCPM4 "InfLLM v2" blog
// (semantic kernels): each kernel is the average of the l_C1 = 32 key vectors
// it covers, kernels overlap with stride s_C1 = 16.  The sum of 32 bf16 values
// is formed in fp64 (exact for all but pathologically spread magnitudes), the
// division by 32 is exact, and the result is rounded once to bf16 (nearest,
// ties to even).  The kernel is HBM-bound: it reads K once and writes K^C1.
// The same kernel with L = 128, S = 64 builds the coarse kernels K^C2 of the
// LSE approximation (paper notes, key design 4).
#include "common.cuh"
#include "internal.cuh"
#include "kc1_mean.cuh"

namespace infv2 {
namespace {

// Mean of L bf16 rows (one 8-element slice of the head dim), summed in fp64 in
// token order; the division by L (a power of two) is exact and the result is
// rounded once to bf16.
template <int L>
__device__ __forceinline__ uint4 kmean_slice(const uint16_t* src, size_t row_stride) {
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 4
  for (int t = 0; t < L; ++t) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + (size_t)t * row_stride));
    acc[0] += (double)bf16_lo(w.x);
    acc[1] += (double)bf16_hi(w.x);
    acc[2] += (double)bf16_lo(w.y);
    acc[3] += (double)bf16_hi(w.y);
    acc[4] += (double)bf16_lo(w.z);
    acc[5] += (double)bf16_hi(w.z);
    acc[6] += (double)bf16_lo(w.w);
    acc[7] += (double)bf16_hi(w.w);
  }
  uint16_t o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) o[e] = f64_to_bf16_rne(acc[e] * (1.0 / L));
  uint4 r;
  r.x = (uint32_t)o[0] | ((uint32_t)o[1] << 16);
  r.y = (uint32_t)o[2] | ((uint32_t)o[3] << 16);
  r.z = (uint32_t)o[4] | ((uint32_t)o[5] << 16);
  r.w = (uint32_t)o[6] | ((uint32_t)o[7] << 16);
  return r;
}

// One thread per (kernel j, kv head g, 8-element slice c of the head dim);
// kernel j covers tokens S*j .. S*j + L - 1.
template <int L, int S>
__global__ void __launch_bounds__(256) compress_k_kernel(const uint16_t* __restrict__ k, int h_kv,
                                                         int nc, uint16_t* __restrict__ kc) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)nc * h_kv * 16;
  if (tid >= total) return;
  const int c = (int)(tid & 15);
  const long long jg = tid >> 4;
  const int g = (int)(jg % h_kv);
  const int j = (int)(jg / h_kv);
  const size_t row_stride = (size_t)h_kv * 128;  // elements between consecutive tokens
  const uint16_t* src = k + (size_t)(S * j) * row_stride + (size_t)g * 128 + c * 8;
  uint4 out;
  if constexpr (L == 32)
    out = kc1_mean_slice(src, row_stride, nullptr, -1);  // the decode step's own routine
  else
    out = kmean_slice<L>(src, row_stride);
  *reinterpret_cast<uint4*>(kc + ((size_t)j * h_kv + g) * 128 + c * 8) = out;
}

template <int L, int S>
int launch_compress(const uint16_t* k, int n, int h_kv, uint16_t* kc, cudaStream_t st) {
  const int nc = n >= L ? (n - L) / S + 1 : 0;
  if (nc == 0) return INFV2_OK;
  const long long total = (long long)nc * h_kv * 16;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  compress_k_kernel<L, S><<<(unsigned)blocks, threads, 0, st>>>(k, h_kv, nc, kc);
  return launch_status(cudaGetLastError());
}

}  // namespace

int launch_compress_k(const uint16_t* k, int n, int h_kv, uint16_t* kc1, cudaStream_t st) {
  return launch_compress<32, 16>(k, n, h_kv, kc1, st);
}

int launch_compress_k2(const uint16_t* k, int n, int h_kv, uint16_t* kc2, cudaStream_t st) {
  return launch_compress<128, 64>(k, n, h_kv, kc2, st);
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

extern "C" int infv2_compress_k2(const infv2_params* p, const void* k, int n, void* kc2,
                                 infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0) return INFV2_ERR_INVALID_ARG;
  if (n >= 4 * p->l_c1 && (!k || !kc2)) return INFV2_ERR_INVALID_ARG;
  return launch_compress_k2(static_cast<const uint16_t*>(k), n, p->h_kv,
                            static_cast<uint16_t*>(kc2), reinterpret_cast<cudaStream_t>(stream));
}
