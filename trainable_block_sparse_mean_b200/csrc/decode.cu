// Single-token decode step over a batch of KV caches.
//
// MiniCPM4 "InfLLM v2" blog (query/key granularity): selection is per query
// token, so a decoding token selects its own blocks and attends to at most k*B
// keys.  The step is memory-bound (it reads K^C1 and the selected K/V once), so
// it is split over many CTAs:
//   1. append     write the new K/V row; if it completes a stage-1 kernel,
//                 write that K^C1 row (same fp64 mean as prefill compression)
//   2. logits     z = scale*log2(e) * q.K^C1 for all visible kernels, split in
//                 chunks of 256 kernels, plus each chunk's per-head (max, sum)
//   3. shared     per-head lse from the chunk partials, then
//                 S^shared[j] = sum_h exp2(z_hj - lse_h)
//   4. select     max pooling + top-k, one warp per (sequence, kv head)
//   5. attention  the block-sparse kernel over the selected blocks, with the
//                 block list split so that several CTAs share one sequence
//   6. combine    merge the splits, write O / lse, advance seqlens.
#include "attn_sparse.cuh"
#include "internal.cuh"
#include "kc1_mean.cuh"
#include "select.cuh"

namespace infv2 {
namespace {

constexpr int kChunk = 256;        // kernels per logits CTA
constexpr int kBlocksPerSplit = 8; // selected blocks per attention CTA
constexpr float kLn2 = 0.6931471805599453f;

struct DecodePlan {
  int cap_c1, zld, n_chunks, ld, n_split, G;
  size_t off_z, off_ml, off_shared, off_idx, off_po, off_pml, total;
};

DecodePlan plan_decode(const infv2_params* p, int batch, int cap) {
  DecodePlan d{};
  d.G = p->h_q / p->h_kv;
  d.cap_c1 = infv2_num_kernels(p, cap);
  d.zld = ((d.cap_c1 + 3) / 4) * 4;  // logits row pitch: 16-byte aligned rows
  d.n_chunks = (d.cap_c1 + kChunk - 1) / kChunk;
  d.ld = shared_ld(cap);
  d.n_split = (p->k + kBlocksPerSplit - 1) / kBlocksPerSplit;
  size_t off = 0;
  d.off_z = off;
  off += round256((size_t)batch * p->h_kv * d.G * (d.zld > 0 ? d.zld : 4) * 4);
  d.off_ml = off;
  off += round256((size_t)batch * p->h_kv * (d.n_chunks > 0 ? d.n_chunks : 1) * d.G * 2 * 4);
  d.off_shared = off;
  off += round256((size_t)batch * p->h_kv * d.ld * 4);
  d.off_idx = off;
  off += round256((size_t)batch * p->h_kv * p->k * 4);
  d.off_po = off;
  off += round256((size_t)batch * p->h_q * d.n_split * 128 * 4);
  d.off_pml = off;
  off += round256((size_t)batch * p->h_q * d.n_split * 2 * 4);
  d.total = off;
  return d;
}

// 1. append the new token and, if it completes a kernel, its K^C1 row.
__global__ void __launch_bounds__(128) decode_append_kernel(
    const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new, uint16_t* k_cache,
    uint16_t* v_cache, uint16_t* kc1_cache, const int* seqlens, int h_kv, int cap, int cap_c1,
    int* err) {
  const int s = blockIdx.x;
  const int L = seqlens[s];
  if (L < 0 || L >= cap) {
    if (threadIdx.x == 0) report_error(err, INFV2_ERR_INVALID_ARG);
    return;
  }
  // copy: h_kv rows of 256 B for K and for V, 16 B per thread step
  const int n16 = h_kv * 16;
  for (int x = threadIdx.x; x < 2 * n16; x += blockDim.x) {
    const int which = x / n16;  // 0: K, 1: V
    const int y = x % n16;
    const int g = y / 16, c = y % 16;
    const uint16_t* src = (which ? v_new : k_new) + ((size_t)s * h_kv + g) * 128 + c * 8;
    uint16_t* dst = (which ? v_cache : k_cache) + (((size_t)s * h_kv + g) * cap + L) * 128 + c * 8;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
  }
  const int Lp = L + 1;  // length after the append
  if (Lp >= 32 && (Lp - 32) % 16 == 0) {
    const int j = (Lp - 32) / 16;
    for (int y = threadIdx.x; y < n16; y += blockDim.x) {
      const int g = y / 16, c = y % 16;
      const uint16_t* rows = k_cache + (((size_t)s * h_kv + g) * cap + 16 * j) * 128 + c * 8;
      const uint16_t* knew = k_new + ((size_t)s * h_kv + g) * 128 + c * 8;
      const uint4 m = kc1_mean_slice(rows, 128, knew, L - 16 * j);
      *reinterpret_cast<uint4*>(kc1_cache + (((size_t)s * h_kv + g) * cap_c1 + j) * 128 + c * 8) = m;
    }
  }
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2. logits for 256 kernels of one (sequence, kv head): 4 warps x 64 kernels,
// 16 heads x 8 kernels per m16n8k16 tile, K^C1 fragments read straight from
// global memory (each row segment is used once).
__global__ void __launch_bounds__(128) decode_logits_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc1_cache, const int* seqlens,
    int h_q, int h_kv, int cap, int cap_c1, int zld, int n_chunks, float scale_log2, float* ws_z,
    float* ws_ml) {
  const int chunk = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  const int L = seqlens[s];
  if (L < 0 || L >= cap) return;
  const int nv = visible_kernels(L, 32, 16);
  const int j_chunk = chunk * kChunk;
  if (j_chunk >= nv) return;
  const int G = h_q / h_kv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  __shared__ float sm_m[4][16], sm_l[4][16];

  uint32_t qa[8][4];
  const uint16_t* qrow = q + ((size_t)s * h_q + (size_t)g * G) * 128;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int c0 = 16 * ks + 2 * tig;
    qa[ks][0] = gid < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + gid * 128 + c0)) : 0u;
    qa[ks][1] = gid + 8 < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + (gid + 8) * 128 + c0)) : 0u;
    qa[ks][2] = gid < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + gid * 128 + c0 + 8)) : 0u;
    qa[ks][3] = gid + 8 < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + (gid + 8) * 128 + c0 + 8)) : 0u;
  }
  const uint16_t* kbase = kc1_cache + ((size_t)s * h_kv + g) * cap_c1 * 128;
  float* zrow = ws_z + ((size_t)s * h_kv + g) * G * zld;
  float mx0 = -INFINITY, mx1 = -INFINITY;
  float zv[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int jn = j_chunk + warp * 64 + nt * 8;  // first kernel of this n-tile
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int jr = jn + gid;  // kernel row this lane feeds as B
    const bool rv = jr < nv;
    const uint16_t* kr = kbase + (size_t)(rv ? jr : 0) * 128;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t b0 = rv ? __ldg(reinterpret_cast<const uint32_t*>(kr + 16 * ks + 2 * tig)) : 0u;
      const uint32_t b1 = rv ? __ldg(reinterpret_cast<const uint32_t*>(kr + 16 * ks + 8 + 2 * tig)) : 0u;
      mma16816(acc, qa[ks], b0, b1);
    }
    // acc: (head gid, kernels jn+2tig, +1), (head gid+8, same kernels)
    const int j0 = jn + 2 * tig;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = j0 + (e & 1);
      zv[nt][e] = j < nv ? acc[e] * scale_log2 : -INFINITY;
    }
    mx0 = fmaxf(mx0, fmaxf(zv[nt][0], zv[nt][1]));
    mx1 = fmaxf(mx1, fmaxf(zv[nt][2], zv[nt][3]));
    if (j0 < nv) {
      if (gid < G) {
        if (j0 + 1 < nv) *reinterpret_cast<float2*>(zrow + (size_t)gid * zld + j0) = make_float2(zv[nt][0], zv[nt][1]);
        else zrow[(size_t)gid * zld + j0] = zv[nt][0];
      }
      if (gid + 8 < G) {
        if (j0 + 1 < nv) *reinterpret_cast<float2*>(zrow + (size_t)(gid + 8) * zld + j0) = make_float2(zv[nt][2], zv[nt][3]);
        else zrow[(size_t)(gid + 8) * zld + j0] = zv[nt][2];
      }
    }
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 2));
  const float r0 = mx0 == -INFINITY ? 0.f : mx0, r1 = mx1 == -INFINITY ? 0.f : mx1;
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    l0 += fast_exp2(zv[nt][0] - r0) + fast_exp2(zv[nt][1] - r0);
    l1 += fast_exp2(zv[nt][2] - r1) + fast_exp2(zv[nt][3] - r1);
  }
  l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
  l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
  l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
  l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
  if (tig == 0) {
    sm_m[warp][gid] = mx0;
    sm_m[warp][gid + 8] = mx1;
    sm_l[warp][gid] = l0;
    sm_l[warp][gid + 8] = l1;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w][h]);
    float Ls = 0.f;
    for (int w = 0; w < 4; ++w)
      if (sm_m[w][h] != -INFINITY) Ls += sm_l[w][h] * fast_exp2(sm_m[w][h] - M);
    float* ml = ws_ml + ((((size_t)s * h_kv + g) * n_chunks + chunk) * G + h) * 2;
    ml[0] = M;
    ml[1] = Ls;
  }
}

// 3. S^shared for 256 kernels of one (sequence, kv head).
__global__ void __launch_bounds__(256) decode_shared_kernel(const int* seqlens, int h_kv, int G,
                                                            int cap, int zld, int n_chunks,
                                                            int ld, const float* ws_z,
                                                            const float* ws_ml, float* ws_shared) {
  const int chunk = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  const int L = seqlens[s];
  if (L < 0 || L >= cap) return;
  const int nv = visible_kernels(L, 32, 16);
  if (chunk * kChunk >= nv) return;
  __shared__ float lse2[16];
  const int used = (nv + kChunk - 1) / kChunk;
  if (threadIdx.x < G) {
    const float* ml = ws_ml + ((size_t)s * h_kv + g) * n_chunks * G * 2;
    float M = -INFINITY;
    for (int c = 0; c < used; ++c) M = fmaxf(M, ml[(c * G + threadIdx.x) * 2]);
    float Ls = 0.f;
    for (int c = 0; c < used; ++c) {
      const float m = ml[(c * G + threadIdx.x) * 2];
      if (m != -INFINITY) Ls += ml[(c * G + threadIdx.x) * 2 + 1] * fast_exp2(m - M);
    }
    lse2[threadIdx.x] = M + __log2f(Ls);
  }
  __syncthreads();
  const int j = chunk * kChunk + threadIdx.x;
  if (j >= nv) return;
  const float* zrow = ws_z + ((size_t)s * h_kv + g) * G * zld;
  float acc = 0.f;
  for (int h = 0; h < G; ++h) acc += fast_exp2(zrow[(size_t)h * zld + j] - lse2[h]);
  ws_shared[((size_t)s * h_kv + g) * ld + j] = acc;
}

// 4. selection, one CTA of 256 threads per (sequence, kv head).
__global__ void __launch_bounds__(256) decode_select_kernel(const int* seqlens, int h_kv, int cap,
                                                            int n_init, int n_local, int k, int ld,
                                                            const float* ws_shared, int* idx,
                                                            int n_keys) {
  extern __shared__ __align__(16) uint32_t sm_sel[];
  const int s = blockIdx.x / h_kv, g = blockIdx.x % h_kv;
  const int L = seqlens[s];
  int* out = idx + ((size_t)s * h_kv + g) * k;
  if (L < 0 || L >= cap) {
    for (int x = threadIdx.x; x < k; x += blockDim.x) out[x] = -1;
    return;
  }
  select_row_cta(ws_shared + ((size_t)s * h_kv + g) * ld, visible_kernels(L, 32, 16), L, n_init,
                 n_local, k, sm_sel, sm_sel + n_keys, sm_sel + n_keys + 256, out);
}

// 6. merge the attention splits; advance seqlens.
__global__ void __launch_bounds__(256) decode_combine_kernel(int* seqlens, int h_q, int cap,
                                                             int n_split, const float* part_o,
                                                             const float* part_ml, uint16_t* o,
                                                             float* lse) {
  const int s = blockIdx.x;
  const int L = seqlens[s];
  const bool valid = L >= 0 && L < cap;
  for (int x = threadIdx.x; x < h_q * 32; x += blockDim.x) {
    const int h = x / 32, d0 = (x % 32) * 4;
    const size_t slot0 = ((size_t)s * h_q + h) * n_split;
    float M = -INFINITY;
    for (int sp = 0; sp < n_split; ++sp) M = fmaxf(M, valid ? part_ml[(slot0 + sp) * 2] : -INFINITY);
    float Ls = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
      for (int sp = 0; sp < n_split; ++sp) {
        const float m = part_ml[(slot0 + sp) * 2];
        if (m == -INFINITY) continue;
        const float sc = fast_exp2(m - M);
        Ls += part_ml[(slot0 + sp) * 2 + 1] * sc;
        const float4 v = *reinterpret_cast<const float4*>(part_o + (slot0 + sp) * 128 + d0);
        acc[0] += v.x * sc;
        acc[1] += v.y * sc;
        acc[2] += v.z * sc;
        acc[3] += v.w * sc;
      }
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    __nv_bfloat162 a0 = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
    __nv_bfloat162 a1 = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
    uint2 wv;
    wv.x = *reinterpret_cast<uint32_t*>(&a0);
    wv.y = *reinterpret_cast<uint32_t*>(&a1);
    *reinterpret_cast<uint2*>(o + ((size_t)s * h_q + h) * 128 + d0) = wv;
    if (lse && d0 == 0) lse[(size_t)s * h_q + h] = Ls > 0.f ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
  }
  __syncthreads();
  if (threadIdx.x == 0 && valid) seqlens[s] = L + 1;
}

}  // namespace
}  // namespace infv2

using namespace infv2;

extern "C" int infv2_decode_workspace_size(const infv2_params* p, int batch, int cap,
                                           size_t* bytes) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (!bytes || batch < 0 || cap < 0) return INFV2_ERR_INVALID_ARG;
  *bytes = plan_decode(p, batch, cap).total;
  return INFV2_OK;
}

extern "C" int infv2_decode(const infv2_params* p, const void* q, const void* k_new,
                            const void* v_new, void* k_cache, void* v_cache, void* kc1_cache,
                            int* seqlens, int batch, int cap, void* workspace, size_t ws_bytes,
                            int* idx_out, void* o, float* lse, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (batch < 0 || cap <= 0) return INFV2_ERR_INVALID_ARG;
  if (batch == 0) return INFV2_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !seqlens || !o) return INFV2_ERR_INVALID_ARG;
  const DecodePlan d = plan_decode(p, batch, cap);
  if (d.cap_c1 > 0 && !kc1_cache) return INFV2_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < d.total) return INFV2_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return INFV2_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* ws_z = reinterpret_cast<float*>(ws + d.off_z);
  float* ws_ml = reinterpret_cast<float*>(ws + d.off_ml);
  float* ws_shared = reinterpret_cast<float*>(ws + d.off_shared);
  int* idx = idx_out ? idx_out : reinterpret_cast<int*>(ws + d.off_idx);
  float* part_o = reinterpret_cast<float*>(ws + d.off_po);
  float* part_ml = reinterpret_cast<float*>(ws + d.off_pml);
  int* err = error_word();
  const float scale_log2 = p->scale * 1.4426950408889634f;
  uint16_t* kc = static_cast<uint16_t*>(k_cache);
  uint16_t* vc = static_cast<uint16_t*>(v_cache);
  uint16_t* kc1 = static_cast<uint16_t*>(kc1_cache);

  decode_append_kernel<<<batch, 128, 0, cs>>>(static_cast<const uint16_t*>(k_new),
                                               static_cast<const uint16_t*>(v_new), kc, vc, kc1,
                                               seqlens, p->h_kv, cap, d.cap_c1, err);
  if ((st = launch_status(cudaGetLastError())) != INFV2_OK) return st;
  if (d.n_chunks > 0) {
    dim3 grid(d.n_chunks, p->h_kv, batch);
    decode_logits_kernel<<<grid, 128, 0, cs>>>(static_cast<const uint16_t*>(q), kc1, seqlens,
                                                p->h_q, p->h_kv, cap, d.cap_c1, d.zld,
                                                d.n_chunks, scale_log2, ws_z, ws_ml);
    if ((st = launch_status(cudaGetLastError())) != INFV2_OK) return st;
    decode_shared_kernel<<<grid, 256, 0, cs>>>(seqlens, p->h_kv, d.G, cap, d.zld, d.n_chunks,
                                                d.ld, ws_z, ws_ml, ws_shared);
    if ((st = launch_status(cudaGetLastError())) != INFV2_OK) return st;
  }
  {
    const int n_keys = (((cap + 63) / 64 + 3) / 4) * 4;
    const int smem = (n_keys + 256 + 4) * 4;
    if (smem > 200 * 1024) return INFV2_ERR_UNSUPPORTED;
    if (!set_smem(decode_select_kernel, smem)) return INFV2_ERR_CUDA;
    decode_select_kernel<<<batch * p->h_kv, 256, smem, cs>>>(seqlens, p->h_kv, cap, p->n_init,
                                                              p->n_local, p->k, d.ld, ws_shared,
                                                              idx, n_keys);
    if ((st = launch_status(cudaGetLastError())) != INFV2_OK) return st;
  }
  {
    CUtensorMap tm_k, tm_v;
    const uint64_t rows = (uint64_t)batch * p->h_kv;
    if (!make_tmap_3d(&tm_k, kc, 128, cap, rows, 256, (uint64_t)cap * 256, 64, 64, 1) ||
        !make_tmap_3d(&tm_v, vc, 128, cap, rows, 256, (uint64_t)cap * 256, 64, 64, 1))
      return INFV2_ERR_CUDA;
    AttnArgs a{};
    a.n_rows = batch;
    a.h_q = p->h_q;
    a.h_kv = p->h_kv;
    a.k = p->k;
    a.idx = idx;
    a.idx_hstride = p->k;
    a.idx_rstride = (long long)p->h_kv * p->k;
    a.q = static_cast<const uint16_t*>(q);
    a.scale_log2 = scale_log2;
    a.decode = 1;
    a.seqlens = seqlens;
    a.n_split = d.n_split;
    a.blocks_per_split = kBlocksPerSplit;
    a.split_out = 1;
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.wait = wait_ctx();
    if ((st = launch_sparse_attn(tm_k, tm_v, a, cs)) != INFV2_OK) return st;
  }
  decode_combine_kernel<<<batch, 256, 0, cs>>>(seqlens, p->h_q, cap, d.n_split, part_o, part_ml,
                                                static_cast<uint16_t*>(o), lse);
  return launch_status(cudaGetLastError());
}
