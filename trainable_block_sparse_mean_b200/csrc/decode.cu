// Single-token decode step over a batch of KV caches.
//
// MiniCPM4 "InfLLM v2" blog (query/key granularity): selection is per query
// token, so a decoding token selects its own blocks and attends to at most k*B
// keys.  The step is memory-bound (it reads K^C1 and the selected K/V once) and
// runs as three kernels:
//   1. logits     (one CTA per 256 kernels of a (sequence, kv head)): the CTA
//                 of chunk 0 appends the new K/V row to the cache; the CTA whose
//                 chunk holds a kernel completed by the new token writes that
//                 K^C1 row (same fp64 mean as prefill compression); every CTA
//                 computes z = scale*log2(e) * q.K^C1 for its visible kernels
//                 (stored head-minor) and each head's (max, sum) over the chunk
//   2. select     (4 CTAs per (sequence, kv head)): per-head lse from the chunk
//                 partials, S^shared[j] = sum_h exp2(z_hj - lse_h) for the
//                 kernels of each block, max pooling into block keys; the last
//                 of the 4 CTAs runs the radix top-k over the row
//   3. attention  the block-sparse kernel over the selected blocks, the list
//                 cut into as many pieces as keep all CTAs in one wave; the
//                 last piece of a (sequence, kv head) to finish merges the
//                 pieces, writes O / lse and, for the last kv head, advances
//                 seqlens.
#include "attn_sparse.cuh"
#include "internal.cuh"
#include "kc1_mean.cuh"
#include "select.cuh"

namespace infv2 {
namespace {

constexpr int kChunk = 256;         // kernels per logits CTA
constexpr int kMaxPieces = 16;      // pieces the attention kernel's merge accepts
constexpr int kSelParts = 4;        // CTAs that build one row's block keys

struct DecodePlan {
  int cap_c1, n_chunks, n_keys, G;
  size_t off_z, off_ml, off_idx, off_po, off_pml, off_keys, off_cnt, total;
};

DecodePlan plan_decode(const infv2_params* p, int batch, int cap) {
  DecodePlan d{};
  d.G = p->h_q / p->h_kv;
  d.cap_c1 = infv2_num_kernels(p, cap);
  d.n_chunks = (d.cap_c1 + kChunk - 1) / kChunk;
  d.n_keys = (((cap + 63) / 64 + 3) / 4) * 4;
  size_t off = 0;
  d.off_z = off;  // [batch][h_kv][cap_c1][16] logits, heads padded to 16
  off += round256((size_t)batch * p->h_kv * (d.cap_c1 > 0 ? d.cap_c1 : 1) * 16 * 4);
  d.off_ml = off;  // [batch][h_kv][n_chunks][16][max, sum]
  off += round256((size_t)batch * p->h_kv * (d.n_chunks > 0 ? d.n_chunks : 1) * 16 * 2 * 4);
  d.off_idx = off;
  off += round256((size_t)batch * p->h_kv * p->k * 4);
  d.off_po = off;  // attention pieces (at most kMaxPieces per row)
  off += round256((size_t)batch * p->h_q * kMaxPieces * 128 * 4);
  d.off_pml = off;
  off += round256((size_t)batch * p->h_q * kMaxPieces * 2 * 4);
  d.off_keys = off;  // block keys of each row, built by kSelParts CTAs
  off += round256((size_t)batch * p->h_kv * d.n_keys * 4);
  d.off_cnt = off;  // attention piece counters [batch][h_kv], row counters [batch],
                    // selection part counters [batch][h_kv]
  off += round256((size_t)batch * (2 * p->h_kv + 1) * 4);
  d.total = off;
  return d;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct LogitsArgs {
  const uint16_t* q;      // [batch, h_q, 128]
  const uint16_t* k_new;  // [batch, h_kv, 128]
  const uint16_t* v_new;
  uint16_t* k_cache;      // [batch, h_kv, cap, 128]
  uint16_t* v_cache;
  uint16_t* kc1_cache;    // [batch, h_kv, cap_c1, 128]
  const int* seqlens;
  int h_q, h_kv, cap, cap_c1, n_chunks;
  float scale_log2;
  float* z;               // [batch, h_kv, cap_c1, 16]
  float* ml;              // [batch, h_kv, n_chunks, 16, 2]
  int* counters;          // [batch * h_kv] then [batch]
  int* err;
};

// 1. append + incremental K^C1 + logits for 256 kernels of one (sequence, kv
// head).  The MMA contracts over the head dim in a permuted order (both
// operands alike) so that every lane loads 16 contiguous bytes per row: for
// k-steps 2c and 2c+1 lane (gid, tig) holds dims 32c + 8tig .. 32c + 8tig + 7.
__global__ void __launch_bounds__(128) decode_logits_kernel(LogitsArgs a) {
  const int chunk = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  const int t = threadIdx.x;
  const int L = a.seqlens[s];
  if (L < 0 || L >= a.cap) {
    if (chunk == 0 && g == 0 && t == 0) report_error(a.err, INFV2_ERR_INVALID_ARG);
    return;
  }
  const size_t sg = (size_t)s * a.h_kv + g;
  if (chunk == 0) {
    // append the new token's K and V rows of this kv head; reset the
    // attention kernel's completion counters of this step
    if (t < 32) {
      const uint16_t* src = (t < 16 ? a.k_new : a.v_new) + sg * 128 + (t & 15) * 8;
      uint16_t* dst = (t < 16 ? a.k_cache : a.v_cache) + (sg * a.cap + L) * 128 + (t & 15) * 8;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
    if (t == 32) {
      const size_t B = gridDim.z;
      a.counters[sg] = 0;                                   // attention pieces
      if (g == 0) a.counters[B * a.h_kv + s] = 0;           // attention rows
      a.counters[B * (a.h_kv + 1) + sg] = 0;                // selection parts
    }
  }
  const int nv = visible_kernels(L, 32, 16);  // includes a kernel completed by token L
  const int j_chunk = chunk * kChunk;
  if (j_chunk >= nv) return;
  const int Lp = L + 1;
  const int j_new = (Lp >= 32 && (Lp - 32) % 16 == 0) ? (Lp - 32) / 16 : -1;
  if (j_new >= j_chunk && j_new < j_chunk + kChunk) {  // uniform over the CTA
    if (t < 16) {
      const uint16_t* rows = a.k_cache + (sg * a.cap + 16 * j_new) * 128 + t * 8;
      const uint16_t* knew = a.k_new + sg * 128 + t * 8;
      const uint4 m = kc1_mean_slice(rows, 128, knew, L - 16 * j_new);
      *reinterpret_cast<uint4*>(a.kc1_cache + (sg * a.cap_c1 + j_new) * 128 + t * 8) = m;
    }
    __syncthreads();  // the new K^C1 row is read below by other threads
  }
  const int G = a.h_q / a.h_kv;
  const int warp = t >> 5, lane = t & 31;
  const int gid = lane >> 2, tig = lane & 3;
  __shared__ float sm_m[4][16], sm_l[4][16];

  // Q fragments in the permuted head-dim order
  uint4 q0[4], q1[4];
  {
    const uint16_t* qrow = a.q + ((size_t)s * a.h_q + (size_t)g * G) * 128 + 8 * tig;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      q0[c] = gid < G ? __ldg(reinterpret_cast<const uint4*>(qrow + gid * 128 + 32 * c))
                      : make_uint4(0u, 0u, 0u, 0u);
      q1[c] = gid + 8 < G ? __ldg(reinterpret_cast<const uint4*>(qrow + (gid + 8) * 128 + 32 * c))
                          : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  const uint16_t* kbase = a.kc1_cache + sg * a.cap_c1 * 128 + 8 * tig;
  float* zbase = a.z + sg * a.cap_c1 * 16;
  float mx0 = -INFINITY, mx1 = -INFINITY;
  float zv[8][4];
  // the next n-tile's K^C1 rows are loaded while the current one is used
  // (L2-only loads: this kernel may have written a row)
  uint4 kn[4];
  {
    const int jr = j_chunk + warp * 64 + gid;
#pragma unroll
    for (int c = 0; c < 4; ++c)
      kn[c] = jr < nv ? __ldcg(reinterpret_cast<const uint4*>(kbase + (size_t)jr * 128 + 32 * c))
                      : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int jn = j_chunk + warp * 64 + nt * 8;  // first kernel of this n-tile
    uint4 kv[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) kv[c] = kn[c];
    if (nt + 1 < 8) {
      const int jr = jn + 8 + gid;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        kn[c] = jr < nv ? __ldcg(reinterpret_cast<const uint4*>(kbase + (size_t)jr * 128 + 32 * c))
                        : make_uint4(0u, 0u, 0u, 0u);
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      mma16816(acc, q0[c].x, q1[c].x, q0[c].y, q1[c].y, kv[c].x, kv[c].y);
      mma16816(acc, q0[c].z, q1[c].z, q0[c].w, q1[c].w, kv[c].z, kv[c].w);
    }
    // acc: (head gid, kernels jn+2tig, +1), (head gid+8, same kernels)
    const int j0 = jn + 2 * tig;
#pragma unroll
    for (int e = 0; e < 4; ++e) zv[nt][e] = (j0 + (e & 1)) < nv ? acc[e] * a.scale_log2 : -INFINITY;
    mx0 = fmaxf(mx0, fmaxf(zv[nt][0], zv[nt][1]));
    mx1 = fmaxf(mx1, fmaxf(zv[nt][2], zv[nt][3]));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = j0 + (e & 1);
      const int h = gid + ((e >> 1) << 3);
      if (j < nv && h < G) zbase[(size_t)j * 16 + h] = zv[nt][e];
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
  if (t < G) {
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w][t]);
    float Ls = 0.f;
    for (int w = 0; w < 4; ++w)
      if (sm_m[w][t] != -INFINITY) Ls += sm_l[w][t] * fast_exp2(sm_m[w][t] - M);
    float* ml = a.ml + ((sg * a.n_chunks + chunk) * 16 + t) * 2;
    ml[0] = M;
    ml[1] = Ls;
  }
}

struct SelectDecArgs {
  const int* seqlens;
  int h_kv, G, cap, cap_c1, n_chunks;
  int n_init, n_local, k;
  const float* z;
  const float* ml;
  uint32_t* keys_g;  // [batch * h_kv][n_keys]
  int* part_cnt;     // [batch * h_kv]
  int* idx;          // [batch, h_kv, k]
  int n_keys;
  int* err;          // device error word (debug-build checks)
};

// 2. selection for one (sequence, kv head), spread over kSelParts CTAs of 256
// threads: each part computes the per-head lse, S^shared[j] = sum_h
// exp2(z_hj - lse_h) for the kernels of its blocks and their max-pooled keys;
// the last part to finish runs the radix top-k over the whole row.
__global__ void __launch_bounds__(256) decode_select_kernel(SelectDecArgs a) {
  extern __shared__ __align__(16) uint32_t sm_sel[];
  __shared__ int s_last;
  uint32_t* keys = sm_sel;                            // [n_keys]
  uint32_t* hist = keys + a.n_keys;                   // [256]
  uint32_t* bcast = hist + 256;                       // [4]
  float* lse2 = reinterpret_cast<float*>(bcast + 4);  // [16]
  float* shared_s = lse2 + 16;                        // S^shared of this part's kernels
  const int part = blockIdx.x, sgi = blockIdx.y;
  const int s = sgi / a.h_kv;
  const int t = threadIdx.x;
  const int L = a.seqlens[s];
  int* out = a.idx + (size_t)sgi * a.k;
  if (L < 0 || L >= a.cap) {
    if (part == 0)
      for (int x = t; x < a.k; x += blockDim.x) out[x] = -1;
    return;
  }
  const int bi = L >> 6;
  const int n_cand = bi + 1;
  if (n_cand <= a.k) {  // every visible block
    if (part == 0)
      for (int b = t; b < a.k; b += blockDim.x) out[b] = b < n_cand ? b : -1;
    return;
  }
  const int nv = visible_kernels(L, 32, 16);
  const int used = (nv + kChunk - 1) / kChunk;
  {  // lse of each head over the chunk partials: 16 threads per head
    const int h = t >> 4, c0 = t & 15;
    const float* ml = a.ml + (size_t)sgi * a.n_chunks * 32 + h * 2;
    float M = -INFINITY;
    for (int c = c0; c < used; c += 16) M = fmaxf(M, ml[c * 32]);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
    float S = 0.f;
    for (int c = c0; c < used; c += 16) {
      const float m = ml[c * 32];
      if (m != -INFINITY) S += ml[c * 32 + 1] * fast_exp2(m - M);
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) S += __shfl_xor_sync(0xFFFFFFFFu, S, o);
    if (c0 == 0) lse2[h] = M + __log2f(S);
  }
  __syncthreads();
  float lse_r[16];
#pragma unroll
  for (int h = 0; h < 16; ++h) lse_r[h] = lse2[h];
  // this part's blocks and the kernels intersecting them
  const int per = (n_cand + kSelParts - 1) / kSelParts;
  const int b_lo = part * per;
  const int b_hi = min(n_cand, b_lo + per);
  const int j_lo = max(0, 4 * b_lo - 1);
  const int j_hi = min(nv, 4 * b_hi + 3);  // exclusive
  const float* zrow = a.z + (size_t)sgi * a.cap_c1 * 16;
  const int G = a.G;
  for (int j0 = j_lo + t; j0 < j_hi; j0 += 4 * blockDim.x) {
    float4 v[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * blockDim.x;
      const float4* zr = reinterpret_cast<const float4*>(zrow + (size_t)(j < j_hi ? j : j_lo) * 16);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        v[u][q4] = 4 * q4 < G ? __ldg(zr + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * blockDim.x;
      float sh = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float vv[4] = {v[u][q4].x, v[u][q4].y, v[u][q4].z, v[u][q4].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * q4 + e < G) sh += fast_exp2(vv[e] - lse_r[4 * q4 + e]);
      }
      if (j < j_hi) shared_s[j - j_lo] = sh;
    }
  }
  __syncthreads();
  uint32_t* kg = a.keys_g + (size_t)sgi * a.n_keys;
  for (int b = b_lo + t; b < b_hi; b += blockDim.x) {
    const bool forced = b < a.n_init || b > bi - a.n_local;
    float m = -INFINITY;
#pragma unroll
    for (int j = 4 * b - 1; j <= 4 * b + 3; ++j)
      if (j >= j_lo && j < j_hi) m = fmaxf(m, shared_s[j - j_lo]);
    kg[b] = forced ? kForcedKey : float_key(m);
  }
  __threadfence();  // this part's keys are visible before it is counted
  __syncthreads();
  if (t == 0) s_last = atomicAdd(&a.part_cnt[sgi], 1) == kSelParts - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (t == 0) {
    bcast[0] = 0xFFFFFFFFu;  // range of the competing (non-forced) keys
    bcast[1] = 0u;
  }
  __syncthreads();
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int b = t; b < n_cand; b += blockDim.x) {
    const uint32_t key = __ldcg(kg + b);
    keys[b] = key;
    if (key != kForcedKey) {
      lo = min(lo, key);
      hi = max(hi, key);
    }
  }
  lo = __reduce_min_sync(0xFFFFFFFFu, lo);
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  if ((t & 31) == 0) {
    atomicMin(&bcast[0], lo);
    atomicMax(&bcast[1], hi);
  }
  if (t == 0) a.part_cnt[sgi] = 0;
  __syncthreads();
  const uint32_t kmin = bcast[0], kmax = bcast[1];
  __syncthreads();  // bcast is reused by the digit passes
  // n_cand > k >= n_init + n_local: the init and local sets are disjoint
  select_topk_cta(keys, n_cand, a.k, hist, bcast, out, a.err, kmin, kmax, a.n_init + a.n_local);
}

}  // namespace
}  // namespace infv2

namespace infv2 {
namespace {

// Stage 5 of the decode step: split-KV block-sparse attention of the query at
// position pos[s] of each sequence; the last piece of a row writes pos + 1 to
// pos_out[s] (the advanced length, or scratch when nothing may change).
int launch_decode_attn(const infv2_params* p, const uint16_t* q, const uint16_t* kc,
                       const uint16_t* vc, const int* pos, int* pos_out, int batch, int cap,
                       const int* idx, uint8_t* ws, const DecodePlan& d, uint16_t* o, float* lse,
                       cudaStream_t cs) {
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
  a.q = q;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.decode = 1;
  a.seqlens = pos;
  a.seqlens_out = pos_out;
  a.cap = cap;
  // as many pieces per row as keep the whole step in one wave of CTAs
  int pieces = (2 * sm_count()) / (batch * p->h_kv);
  if (pieces > kMaxPieces) pieces = kMaxPieces;
  if (pieces > p->k) pieces = p->k;
  if (pieces < 1) pieces = 1;
  const int bps = (p->k + pieces - 1) / pieces;
  a.n_split = (p->k + bps - 1) / bps;
  a.blocks_per_split = bps;
  a.split_out = 1;
  a.part_o = reinterpret_cast<float*>(ws + d.off_po);
  a.part_ml = reinterpret_cast<float*>(ws + d.off_pml);
  a.counters = reinterpret_cast<int*>(ws + d.off_cnt);
  a.o = o;
  a.lse = lse;
  a.wait = wait_ctx();
  return launch_sparse_attn(tm_k, tm_v, a, cs);
}

}  // namespace
}  // namespace infv2

using namespace infv2;

extern "C" int infv2_decode_workspace_size(const infv2_params* p, int batch, int cap,
                                           size_t* bytes) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (p->lse_approx) return INFV2_ERR_UNSUPPORTED;  // the decode step scores exactly
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
  if (p->lse_approx) return INFV2_ERR_UNSUPPORTED;  // the decode step scores exactly
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
  int* idx = idx_out ? idx_out : reinterpret_cast<int*>(ws + d.off_idx);
  int* counters = reinterpret_cast<int*>(ws + d.off_cnt);
  const float scale_log2 = p->scale * 1.4426950408889634f;
  uint16_t* kc = static_cast<uint16_t*>(k_cache);
  uint16_t* vc = static_cast<uint16_t*>(v_cache);

  {
    LogitsArgs a;
    a.q = static_cast<const uint16_t*>(q);
    a.k_new = static_cast<const uint16_t*>(k_new);
    a.v_new = static_cast<const uint16_t*>(v_new);
    a.k_cache = kc;
    a.v_cache = vc;
    a.kc1_cache = static_cast<uint16_t*>(kc1_cache);
    a.seqlens = seqlens;
    a.h_q = p->h_q;
    a.h_kv = p->h_kv;
    a.cap = cap;
    a.cap_c1 = d.cap_c1;
    a.n_chunks = d.n_chunks;
    a.scale_log2 = scale_log2;
    a.z = ws_z;
    a.ml = ws_ml;
    a.counters = counters;
    a.err = error_word();
    dim3 grid(d.n_chunks > 0 ? d.n_chunks : 1, p->h_kv, batch);  // chunk 0 always appends
    decode_logits_kernel<<<grid, 128, 0, cs>>>(a);
    if ((st = launch_status(cudaGetLastError())) != INFV2_OK) return st;
  }
  {
    SelectDecArgs a;
    a.seqlens = seqlens;
    a.h_kv = p->h_kv;
    a.G = d.G;
    a.cap = cap;
    a.cap_c1 = d.cap_c1;
    a.n_chunks = d.n_chunks;
    a.n_init = p->n_init;
    a.n_local = p->n_local;
    a.k = p->k;
    a.z = ws_z;
    a.ml = ws_ml;
    a.keys_g = reinterpret_cast<uint32_t*>(ws + d.off_keys);
    a.part_cnt = counters + (size_t)batch * (p->h_kv + 1);
    a.idx = idx;
    a.n_keys = d.n_keys;
    a.err = error_word();
    const int part_kernels = 4 * ((d.n_keys + kSelParts - 1) / kSelParts) + 8;
    const int smem = (a.n_keys + 256 + 4 + 16 + part_kernels) * 4;
    if (smem > 200 * 1024) return INFV2_ERR_UNSUPPORTED;
    if (!set_smem(decode_select_kernel, smem)) return INFV2_ERR_CUDA;
    decode_select_kernel<<<dim3(kSelParts, batch * p->h_kv), 256, smem, cs>>>(a);
    if ((st = launch_status(cudaGetLastError())) != INFV2_OK) return st;
  }
  return launch_decode_attn(p, static_cast<const uint16_t*>(q), kc, vc, seqlens, seqlens, batch,
                            cap, idx, ws, d, static_cast<uint16_t*>(o), lse, cs);
}

extern "C" int infv2_decode_attn(const infv2_params* p, const void* q, const void* k_cache,
                                 const void* v_cache, const int* pos, int batch, int cap,
                                 const int* idx, void* workspace, size_t ws_bytes, void* o,
                                 float* lse, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (batch < 0 || cap <= 0) return INFV2_ERR_INVALID_ARG;
  if (batch == 0) return INFV2_OK;
  if (!q || !k_cache || !v_cache || !pos || !idx || !o) return INFV2_ERR_INVALID_ARG;
  const DecodePlan d = plan_decode(p, batch, cap);
  if (!workspace || ws_bytes < d.total) return INFV2_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return INFV2_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // the pieces' merge counters start at zero; the positions stay as given (the
  // merge writes pos + 1 into the unused selection area of the workspace)
  if (cudaMemsetAsync(ws + d.off_cnt, 0, (size_t)batch * (p->h_kv + 1) * 4, cs) != cudaSuccess)
    return INFV2_ERR_CUDA;
  return launch_decode_attn(p, static_cast<const uint16_t*>(q),
                            static_cast<const uint16_t*>(k_cache),
                            static_cast<const uint16_t*>(v_cache), pos,
                            reinterpret_cast<int*>(ws + d.off_idx), batch, cap, idx, ws, d,
                            static_cast<uint16_t*>(o), lse, cs);
}
