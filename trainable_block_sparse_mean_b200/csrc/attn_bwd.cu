// Backward of the block-sparse (or dense) causal attention, for training.
//
// arXiv summary, Appendix A: the forward returns O and the log-sum-exp so that
// the backward can recompute the softmax; the MiniCPM4 blog notes the
// selection itself is not differentiated.  With the block lists fixed and the
// FlashAttention-style definition (D = dO . O from the forward output):
//   P_t  = exp(scale q.k_t - lse),  dS_t = P_t (dO . v_t - D)
//   dq   = scale sum_t dS_t k_t,  dk_t += scale dS_t q,  dv_t += P_t dO
// over the visible tokens t of the query's blocks, per head of the group.
//
// B200 design (m16n8k16 bf16 MMAs, fp32 accumulation, TMA staging):
//   prep     D per (token, head), and a per-token row of (lse2, D) for the G
//            heads of each kv head (one 128-byte TMA copy per token later);
//            zeroes dk, dv.
//   index    (sparse lists only) the inverse of the block lists: for every
//            (kv head, block) the tokens that selected it (count, scan, fill),
//            cut into work items of at most kChunk tokens.
//   dq       one item per (kv head, token), structured like the forward kernel:
//            a TMA producer streams the token's Q, dO and its blocks' K/V
//            through a ring; four warps own 16 keys of every block each and
//            accumulate dq partials that are summed at the end.
//   dk, dv   one item per (kv head, block, chunk of its token list): the
//            block's K/V stay in shared memory while the tokens' Q and dO
//            stream through a ring; four warps own 16 keys each, accumulate
//            dk, dv in registers over the chunk and add them to the outputs
//            with vector atomics (chunks of one block land in any order, so
//            dk and dv are reproducible only up to fp32 rounding).
#include "attn_sparse.cuh"
#include "common.cuh"
#include "internal.cuh"

namespace infv2 {
namespace {

constexpr int kHalfB = 64 * 64 * 2;       // 64 rows x 64 dims of bf16 = 8 KB
constexpr int kStageB = 4 * kHalfB;       // K (2 halves) + V (2 halves) of a block
constexpr int kRowsB = 16 * 128;          // bytes of 16 head rows x 64 dims (one half)
constexpr int kTokQ = 2 * kRowsB;         // Q of a token (2 halves) = 4 KB
constexpr int kTokLd = 2 * kTokQ;         // offset of the (lse2, D) row in a token slot
constexpr int kTokSlot = 9 * 1024;        // Q, dO, (lse2, D): 8 KB + 128 B, 1024-aligned
constexpr int kChunkTok = 1024;           // tokens per dk/dv work item
constexpr int kDqStages = 2;
constexpr int kTokRing = 4;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                      uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                       uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                    uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t bf2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// (row, 16-byte chunk) inside a 64-column half stored with the 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}
// 1-D bulk copy global -> shared, completing on `bar` (16-byte aligned, size % 16 == 0)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// ------------------------------------------------------------------ prep

struct PrepArgs {
  const uint16_t* o;    // [n, h_q, 128]
  const uint16_t* d_o;  // [n, h_q, 128]
  const float* lse;     // [h_q][lse_ld], natural log
  long long lse_ld;
  int n, h_q, h_kv;
  float* ld;            // [h_kv][n][16][2]: (lse * log2 e, D) per head of the group
  float* dk;            // [n, h_kv, 128] zeroed
  float* dv;
  int* cnt;             // [n_cnt] zeroed (inverse-index counts), nullable
  int n_cnt;
};

// 16 lanes per (token, head) row: D = dO . O in fp32; zeroes dk and dv.
__global__ void __launch_bounds__(256) bwd_prep_kernel(PrepArgs a) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  const long long rows = (long long)a.n * a.h_q;
  const int G = a.h_q / a.h_kv;
  const int sub = threadIdx.x & 15;
  for (long long r = tid >> 4; r < ((rows + 1) & ~1ll); r += nthreads >> 4) {
    float acc = 0.f;
    if (r < rows) {
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(a.d_o + r * 128) + sub);
      const uint4 y = __ldg(reinterpret_cast<const uint4*>(a.o + r * 128) + sub);
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(xs[e] << 16), __uint_as_float(ys[e] << 16), acc);
        acc = fmaf(__uint_as_float(xs[e] & 0xFFFF0000u), __uint_as_float(ys[e] & 0xFFFF0000u), acc);
      }
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (r < rows && sub == 0) {
      const int i = (int)(r / a.h_q), h = (int)(r % a.h_q);
      const int g = h / G, hh = h % G;
      float* dst = a.ld + (((size_t)g * a.n + i) * 16 + hh) * 2;
      dst[0] = __ldg(a.lse + (size_t)h * a.lse_ld + i) * kLog2e;
      dst[1] = acc;
    }
  }
  const long long n4 = (long long)a.n * a.h_kv * 32;  // float4s of dk (and of dv)
  for (long long x = tid; x < n4; x += nthreads) {
    reinterpret_cast<float4*>(a.dk)[x] = make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float4*>(a.dv)[x] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (a.cnt)
    for (long long x = tid; x < a.n_cnt; x += nthreads) a.cnt[x] = 0;
}

// ------------------------------------------------------------------ index

struct IndexArgs {
  const int* idx;       // [h_kv][n][k] (row stride k, head stride idx_hstride)
  long long idx_hstride;
  int n, h_kv, k, n_blk;
  int* cnt;             // [h_kv * n_blk] tokens per (kv head, block)
  int* cursor;          // [h_kv * n_blk] fill cursors (start at the offsets)
  int* list;            // [sum of cnt] tokens, grouped by (kv head, block)
};

// Thread per (g, entry e, token i), tokens fastest, so that lanes that hold the
// same block (the initial and local blocks) share one atomic.  Entries < 0 and
// blocks past the token are skipped (they contribute nothing).
template <bool FILL>
__global__ void __launch_bounds__(256) bwd_index_kernel(IndexArgs a) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)a.h_kv * a.k * a.n;
  int key = -1, i = 0;
  if (tid < total) {
    i = (int)(tid % a.n);
    const long long ge = tid / a.n;
    const int e = (int)(ge % a.k), g = (int)(ge / a.k);
    const int b = __ldg(a.idx + (size_t)g * a.idx_hstride + (size_t)i * a.k + e);
    if (b >= 0 && b < a.n_blk && 64 * b <= i) key = g * a.n_blk + b;
  }
  const uint32_t same = __match_any_sync(0xFFFFFFFFu, key);
  if (key < 0) return;
  const int leader = __ffs(same) - 1;
  const int lane = threadIdx.x & 31;
  if (!FILL) {
    if (lane == leader) atomicAdd(a.cnt + key, __popc(same));
  } else {
    int base = 0;
    if (lane == leader) base = atomicAdd(a.cursor + key, __popc(same));
    base = __shfl_sync(same, base, leader);
    a.list[base + __popc(same & ((1u << lane) - 1u))] = i;
  }
}

// One CTA: offsets of the token lists (exclusive scan of the counts), fill
// cursors, and the work items (g, b, first position, tokens) of at most
// kChunkTok tokens.  Dense mode (no lists): block b's tokens are 64b .. n-1.
__global__ void __launch_bounds__(1024) bwd_scan_kernel(int* cnt, int* off, int* cursor, int4* items,
                                                        int* n_items, int h_kv, int n_blk, int n,
                                                        int dense) {
  __shared__ int s_warp[32];
  __shared__ int s_carry[2];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int total = h_kv * n_blk;
  if (t == 0) s_carry[0] = s_carry[1] = 0;
  __syncthreads();
  for (int base = 0; base < total; base += 1024) {
    const int x = base + t;
    int c = 0;
    if (x < total) c = dense ? n - 64 * (x % n_blk) : cnt[x];
    const int m = (c + kChunkTok - 1) / kChunkTok;  // work items of this list
    // block-wide inclusive scans of c and m (packed: both < 2^31 in practice)
    int vc = c, vm = m;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yc = __shfl_up_sync(0xFFFFFFFFu, vc, o), ym = __shfl_up_sync(0xFFFFFFFFu, vm, o);
      if (lane >= o) {
        vc += yc;
        vm += ym;
      }
    }
    if (lane == 31) s_warp[warp] = vc;
    __syncthreads();
    if (warp == 0) {
      int w = s_warp[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) w += y;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const int pre_c = (warp > 0 ? s_warp[warp - 1] : 0) + vc - c + s_carry[0];
    const int tot_c = s_warp[31];
    __syncthreads();
    if (lane == 31) s_warp[warp] = vm;
    __syncthreads();
    if (warp == 0) {
      int w = s_warp[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) w += y;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const int pre_m = (warp > 0 ? s_warp[warp - 1] : 0) + vm - m + s_carry[1];
    const int tot_m = s_warp[31];
    if (x < total) {
      off[x] = pre_c;
      if (!dense) cursor[x] = pre_c;
      const int g = x / n_blk, b = x % n_blk;
      for (int j = 0; j < m; ++j) {
        const int p0 = j * kChunkTok;
        items[pre_m + j] = make_int4(g, b, p0, min(kChunkTok, c - p0));
      }
    }
    __syncthreads();
    if (t == 0) {
      s_carry[0] += tot_c;
      s_carry[1] += tot_m;
    }
    __syncthreads();
  }
  if (t == 0) *n_items = s_carry[1];
}

// ------------------------------------------------------------------ dq

struct DqArgs {
  int n, h_q, h_kv, k;
  const int* idx;          // [h_kv][n][k] (head stride idx_hstride); nullptr = dense
  long long idx_hstride;
  float scale_log2, scale;
  const float* ld;         // [h_kv][n][16][2]
  float* dq;               // [n, h_q, 128]
  WaitCtx wait;
};

// One item = (kv head g, token i), i from the end (longest dense rows first).
__global__ void __launch_bounds__(160, 2)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  DqArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // [K/V stages][2 token slots][barriers]
  uint8_t* tok = base + kDqStages * kStageB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tok + 2 * kTokSlot);
  const uint32_t stage0 = smem_u32(base), tok0 = smem_u32(tok);
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * kDqStages;
  const uint32_t tfull0 = empty0 + 8 * kDqStages, tempty0 = tfull0 + 16, cbar = tempty0 + 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.h_q / a.h_kv;
  const long long n_items = (long long)a.h_kv * a.n;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDqStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 4);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(tfull0 + 8 * x, 1);
      mbar_init(tempty0 + 8 * x, 4);
    }
    mbar_init(cbar, 4);
    fence_mbar_init();
  }
  // head rows G..15 of the token slots are never written by TMA: keep them zero
  for (int x = threadIdx.x; x < 2 * kTokSlot / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(tok)[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      long long pc = 0, tc = 0;
      bool ok = true;
      for (long long w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++tc) {
        const int g = (int)(w / a.n), i = a.n - 1 - (int)(w % a.n);
        const int ts = (int)(tc & 1);
        if (!mbar_wait(tempty0 + 8 * ts, (uint32_t)((tc >> 1) & 1) ^ 1u, a.wait)) break;
        const uint32_t slot = tok0 + ts * kTokSlot, fb = tfull0 + 8 * ts;
        mbar_expect_tx(fb, 4 * G * 128 + 128);
        tma_load_3d(slot, &tm_q, fb, 0, g * G, i);
        tma_load_3d(slot + kRowsB, &tm_q, fb, 64, g * G, i);
        tma_load_3d(slot + kTokQ, &tm_do, fb, 0, g * G, i);
        tma_load_3d(slot + kTokQ + kRowsB, &tm_do, fb, 64, g * G, i);
        bulk_load(slot + kTokLd, a.ld + ((size_t)g * a.n + i) * 32, 128, fb);
        const int* row = a.idx ? a.idx + (size_t)g * a.idx_hstride + (size_t)i * a.k : nullptr;
        const int ne = row ? a.k : (i >> 6) + 1;
        for (int e = 0; e < ne; ++e) {
          const int b = row ? list_block(row, e, i, a.wait.err) : e;
          if (b < 0) continue;
          const int s = (int)(pc % kDqStages);
          if (!mbar_wait(empty0 + 8 * s, (uint32_t)((pc / kDqStages) & 1) ^ 1u, a.wait)) {
            ok = false;
            break;
          }
          const uint32_t dst = stage0 + s * kStageB, kf = full0 + 8 * s;
          mbar_expect_tx(kf, kStageB);
          tma_load_3d(dst, &tm_k, kf, 0, g, 64 * b);
          tma_load_3d(dst + kHalfB, &tm_k, kf, 64, g, 64 * b);
          tma_load_3d(dst + 2 * kHalfB, &tm_v, kf, 0, g, 64 * b);
          tma_load_3d(dst + 3 * kHalfB, &tm_v, kf, 64, g, 64 * b);
          ++pc;
        }
        if (!ok) break;
        {  // one stage without data: the consumers' merge buffer for this item
          const int s = (int)(pc % kDqStages);
          if (!mbar_wait(empty0 + 8 * s, (uint32_t)((pc / kDqStages) & 1) ^ 1u, a.wait)) break;
          mbar_arrive(full0 + 8 * s);
          ++pc;
        }
      }
      for (long long x = pc > kDqStages ? pc - kDqStages : 0; x < pc; ++x)
        (void)mbar_wait(full0 + 8 * (int)(x % kDqStages), (uint32_t)((x / kDqStages) & 1), a.wait);
      for (long long x = tc > 2 ? tc - 2 : 0; x < tc; ++x)
        (void)mbar_wait(tfull0 + 8 * (int)(x & 1), (uint32_t)((x >> 1) & 1), a.wait);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gid = lane >> 2, tig = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;
  const int kb = warp * 16;  // this warp's 16 keys of every block
  const float c = a.scale_log2;
  long long cc = 0, tc = 0;
  uint32_t cphase = 0;
  for (long long w = blockIdx.x; w < n_items; w += gridDim.x, ++tc) {
    const int g = (int)(w / a.n), i = a.n - 1 - (int)(w % a.n);
    const int ts = (int)(tc & 1);
    if (!mbar_wait(tfull0 + 8 * ts, (uint32_t)((tc >> 1) & 1), a.wait)) break;
    const uint32_t slot = tok0 + ts * kTokSlot;
    // Q fragments (A operand: 16 head rows x 128 dims) in registers; dO's are
    // re-read from the token slot per block, so the slot is held to the end
    uint32_t qa[8][4];
    const int qrow = rr + ((mi & 1) << 3);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      ldsm4(slot + (ks >> 2) * kRowsB + swz(qrow, (ks & 3) * 2 + (mi >> 1)), qa[ks][0], qa[ks][1],
            qa[ks][2], qa[ks][3]);
    const float* ldr = reinterpret_cast<const float*>(tok + ts * kTokSlot + kTokLd);
    // (lse2, D) of rows gid and gid + 8; rows past the group are zero rows
    const float nl0 = gid < G ? -ldr[2 * gid] : 0.f, D0 = gid < G ? ldr[2 * gid + 1] : 0.f;
    const float nl1 = gid + 8 < G ? -ldr[2 * (gid + 8)] : 0.f;
    const float D1 = gid + 8 < G ? ldr[2 * (gid + 8) + 1] : 0.f;

    float dqa[16][4];
#pragma unroll
    for (int x = 0; x < 16; ++x) dqa[x][0] = dqa[x][1] = dqa[x][2] = dqa[x][3] = 0.f;
    const int* row = a.idx ? a.idx + (size_t)g * a.idx_hstride + (size_t)i * a.k : nullptr;
    const int ne = row ? a.k : (i >> 6) + 1;
    bool ok = true;
    int chunk_b = 0;
    for (int e = 0; e < ne; ++e) {
      if ((e & 31) == 0)
        chunk_b = e + lane < ne ? (row ? list_block(row, e + lane, i, a.wait.err) : e + lane) : -1;
      const int b = __shfl_sync(0xFFFFFFFFu, chunk_b, e & 31);
      if (b < 0) continue;
      const int s = (int)(cc % kDqStages);
      if (!mbar_wait(full0 + 8 * s, (uint32_t)((cc / kDqStages) & 1), a.wait)) {
        ok = false;
        break;
      }
      const uint32_t kbase = stage0 + s * kStageB, vbase = kbase + 2 * kHalfB;
      // ---- S = Q K^T and dP = dO V^T over keys kb .. kb+15 (two n-tiles)
      float sc[2][4], sd[2][4], pc_[2][4], pd[2][4];
#pragma unroll
      for (int x = 0; x < 4; ++x) sc[0][x] = sc[1][x] = sd[0][x] = sd[1][x] = 0.f;
#pragma unroll
      for (int x = 0; x < 4; ++x) pc_[0][x] = pc_[1][x] = pd[0][x] = pd[1][x] = 0.f;
      {
        const int key = kb + rr + ((mi >> 1) << 3);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t off = swz(key, ks * 2 + (mi & 1));
          uint32_t b0, b1, b2, b3, e0, e1, e2, e3;
          ldsm4(kbase + off, b0, b1, b2, b3);
          ldsm4(kbase + kHalfB + off, e0, e1, e2, e3);
          mma(sc[0], qa[ks], b0, b1);
          mma(sc[1], qa[ks], b2, b3);
          mma(sd[0], qa[ks + 4], e0, e1);
          mma(sd[1], qa[ks + 4], e2, e3);
          uint32_t d0[4], d1[4];
          const uint32_t doff = swz(qrow, ks * 2 + (mi >> 1));
          ldsm4(slot + kTokQ + doff, d0[0], d0[1], d0[2], d0[3]);
          ldsm4(slot + kTokQ + kRowsB + doff, d1[0], d1[1], d1[2], d1[3]);
          ldsm4(vbase + off, b0, b1, b2, b3);
          ldsm4(vbase + kHalfB + off, e0, e1, e2, e3);
          mma(pc_[0], d0, b0, b1);
          mma(pc_[1], d0, b2, b3);
          mma(pd[0], d1, e0, e1);
          mma(pd[1], d1, e2, e3);
        }
      }
      // ---- P = 2^(s*c - lse2) (masked past the query), dS = P (dP - D)
      const int t0 = 64 * b + kb;
      uint32_t pa[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float ds[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const int t = t0 + nt * 8 + 2 * tig + (e2 & 1);
          const float s_ = sc[nt][e2] + sd[nt][e2];
          const float p = t <= i ? fast_exp2(fmaf(s_, c, e2 < 2 ? nl0 : nl1)) : 0.f;
          ds[e2] = p * (pc_[nt][e2] + pd[nt][e2] - (e2 < 2 ? D0 : D1));
        }
        pa[2 * nt + 0] = bf2(ds[0], ds[1]);
        pa[2 * nt + 1] = bf2(ds[2], ds[3]);
      }
      // ---- dQ += dS K (16 n-tiles of 8 dims, keys as the contraction)
      {
        const int key = kb + rr + ((mi & 1) << 3);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          const int nt = 2 * np;
          uint32_t b0, b1, b2, b3;
          ldsm4t(kbase + (nt >> 3) * kHalfB + swz(key, (nt & 7) + (mi >> 1)), b0, b1, b2, b3);
          mma(dqa[nt], pa, b0, b1);
          mma(dqa[nt + 1], pa, b2, b3);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
      ++cc;
    }
    if (!ok) break;
    // the token slot may be refilled by TMA
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(tempty0 + 8 * ts);
    // ---- sum the four warps' partials in the item's merge stage
    const int sm_ = (int)(cc % kDqStages);
    if (!mbar_wait(full0 + 8 * sm_, (uint32_t)((cc / kDqStages) & 1), a.wait)) break;
    ++cc;
    float* red = reinterpret_cast<float*>(base + sm_ * kStageB);  // [4][16][128]
    {
      float* ro = red + warp * 16 * 128;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const int col = nt * 8 + 2 * tig;
        *reinterpret_cast<float2*>(ro + gid * 128 + col) = make_float2(dqa[nt][0], dqa[nt][1]);
        *reinterpret_cast<float2*>(ro + (gid + 8) * 128 + col) = make_float2(dqa[nt][2], dqa[nt][3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    if (!mbar_wait(cbar, cphase & 1u, a.wait)) break;
    ++cphase;
    {
      const int t = threadIdx.x, rowh = t >> 3, d0 = (t & 7) * 16;
      if (rowh < G) {
        float* dst = a.dq + ((size_t)i * a.h_q + g * G + rowh) * 128 + d0;
#pragma unroll
        for (int x = 0; x < 16; x += 4) {
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(red + (q * 16 + rowh) * 128 + d0 + x);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
          }
          *reinterpret_cast<float4*>(dst + x) =
              make_float4(acc.x * a.scale, acc.y * a.scale, acc.z * a.scale, acc.w * a.scale);
        }
      }
    }
    fence_proxy_async_smem();  // the merge stage is refilled by TMA after this release
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * sm_);
  }
}

// ------------------------------------------------------------------ dk, dv

struct DkvArgs {
  int n, h_q, h_kv, n_blk;
  const int* list;         // tokens of (g, b) at list[off[g*n_blk + b] + pos]; nullptr = dense
  const int* off;
  const int4* items;       // (g, b, first position, tokens)
  const int* n_items;      // device count of items
  float scale_log2, scale;
  const float* ld;         // [h_kv][n][16][2]
  float* dk;               // [n, h_kv, 128] (accumulated)
  float* dv;
  WaitCtx wait;
};

__device__ __forceinline__ int item_token(const DkvArgs& a, const int4& it, int j) {
  return a.list ? __ldg(a.list + a.off[it.x * a.n_blk + it.y] + it.z + j) : 64 * it.y + it.z + j;
}

__global__ void __launch_bounds__(160, 2)
    bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   DkvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // [2 K/V slots][kTokRing token slots][barriers]
  uint8_t* tok = base + 2 * kStageB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tok + kTokRing * kTokSlot);
  const uint32_t kv0 = smem_u32(base), tok0 = smem_u32(tok);
  const uint32_t kvfull0 = smem_u32(bars), kvempty0 = kvfull0 + 16;
  const uint32_t tfull0 = kvempty0 + 16, tempty0 = tfull0 + 8 * kTokRing;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.h_q / a.h_kv;
  const int n_items = *reinterpret_cast<const volatile int*>(a.n_items);
  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(kvfull0 + 8 * x, 1);
      mbar_init(kvempty0 + 8 * x, 4);
    }
    for (int x = 0; x < kTokRing; ++x) {
      mbar_init(tfull0 + 8 * x, 1);
      mbar_init(tempty0 + 8 * x, 4);
    }
    fence_mbar_init();
  }
  for (int x = threadIdx.x; x < kTokRing * kTokSlot / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(tok)[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    long long ic = 0, tc = 0;
    bool ok = true;
    for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++ic) {
      const int4 it = a.items[w];
      const int g = it.x, b = it.y, cnt = it.w;
      if (lane == 0) {
        const int ks = (int)(ic & 1);
        if (mbar_wait(kvempty0 + 8 * ks, (uint32_t)((ic >> 1) & 1) ^ 1u, a.wait)) {
          const uint32_t dst = kv0 + ks * kStageB, fb = kvfull0 + 8 * ks;
          mbar_expect_tx(fb, kStageB);
          tma_load_3d(dst, &tm_k, fb, 0, g, 64 * b);
          tma_load_3d(dst + kHalfB, &tm_k, fb, 64, g, 64 * b);
          tma_load_3d(dst + 2 * kHalfB, &tm_v, fb, 0, g, 64 * b);
          tma_load_3d(dst + 3 * kHalfB, &tm_v, fb, 64, g, 64 * b);
        } else {
          ok = false;
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      for (int j0 = 0; ok && j0 < cnt; j0 += 32) {
        const int tl = j0 + lane < cnt ? item_token(a, it, j0 + lane) : 0;  // 32 tokens, one per lane
        const int m = min(32, cnt - j0);
        for (int jj = 0; jj < m; ++jj) {
          const int i = __shfl_sync(0xFFFFFFFFu, tl, jj);
          if (lane == 0 && ok) {
            const int ts = (int)(tc % kTokRing);
            if (mbar_wait(tempty0 + 8 * ts, (uint32_t)((tc / kTokRing) & 1) ^ 1u, a.wait)) {
              const uint32_t slot = tok0 + ts * kTokSlot, fb = tfull0 + 8 * ts;
              mbar_expect_tx(fb, 4 * G * 128 + 128);
              tma_load_3d(slot, &tm_q, fb, 0, g * G, i);
              tma_load_3d(slot + kRowsB, &tm_q, fb, 64, g * G, i);
              tma_load_3d(slot + kTokQ, &tm_do, fb, 0, g * G, i);
              tma_load_3d(slot + kTokQ + kRowsB, &tm_do, fb, 64, g * G, i);
              bulk_load(slot + kTokLd, a.ld + ((size_t)g * a.n + i) * 32, 128, fb);
            } else {
              ok = false;
            }
          }
          ++tc;
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      }
    }
    if (lane == 0) {
      for (long long x = tc > kTokRing ? tc - kTokRing : 0; x < tc; ++x)
        (void)mbar_wait(tfull0 + 8 * (int)(x % kTokRing), (uint32_t)((x / kTokRing) & 1), a.wait);
      for (long long x = ic > 2 ? ic - 2 : 0; x < ic; ++x)
        (void)mbar_wait(kvfull0 + 8 * (int)(x & 1), (uint32_t)((x >> 1) & 1), a.wait);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gid = lane >> 2, tig = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;
  const int kb = warp * 16;  // this warp's 16 keys of the block
  const float c = a.scale_log2;
  long long ic = 0, tc = 0;
  bool ok = true;
  for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++ic) {
    const int4 it = a.items[w];
    const int g = it.x, b = it.y, cnt = it.w;
    const int ksl = (int)(ic & 1);
    if (!mbar_wait(kvfull0 + 8 * ksl, (uint32_t)((ic >> 1) & 1), a.wait)) break;
    const uint32_t kbase = kv0 + ksl * kStageB, vbase = kbase + 2 * kHalfB;
    float dka[16][4], dva[16][4];
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      dka[x][0] = dka[x][1] = dka[x][2] = dka[x][3] = 0.f;
      dva[x][0] = dva[x][1] = dva[x][2] = dva[x][3] = 0.f;
    }
    const int key0 = 64 * b + kb + gid;  // key rows gid and gid + 8 of this warp
    int tl = 0;
    for (int j = 0; j < cnt; ++j) {
      if ((j & 31) == 0) tl = j + lane < cnt ? item_token(a, it, j + lane) : 0;
      const int i = __shfl_sync(0xFFFFFFFFu, tl, j & 31);
      const int ts = (int)(tc % kTokRing);
      if (!mbar_wait(tfull0 + 8 * ts, (uint32_t)((tc / kTokRing) & 1), a.wait)) {
        ok = false;
        break;
      }
      ++tc;
      const uint32_t qslot = tok0 + ts * kTokSlot, dslot = qslot + kTokQ;
      // (lse2, D) of the heads in this thread's columns: 2tig, 2tig+1, 8+2tig, 9+2tig
      const float* ldr = reinterpret_cast<const float*>(tok + ts * kTokSlot + kTokLd);
      float nl[2][2], Dv[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int h = nt * 8 + 2 * tig + u;
          nl[nt][u] = h < G ? -ldr[2 * h] : 0.f;
          Dv[nt][u] = h < G ? ldr[2 * h + 1] : 0.f;
        }
      // ---- S^T = K Q^T and dP^T = V dO^T: rows = this warp's keys, cols = heads
      float st[2][4], pt[2][4];
#pragma unroll
      for (int x = 0; x < 4; ++x) st[0][x] = st[1][x] = pt[0][x] = pt[1][x] = 0.f;
      {
        const int arow = kb + rr + ((mi & 1) << 3);   // A: key rows
        const int brow = rr + ((mi >> 1) << 3);       // B: head rows
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t ka[4], b0, b1, b2, b3;
          const uint32_t half = (ks >> 2);
          const uint32_t aoff = half * kHalfB + swz(arow, (ks & 3) * 2 + (mi >> 1));
          const uint32_t boff = half * kRowsB + swz(brow, (ks & 3) * 2 + (mi & 1));
          ldsm4(kbase + aoff, ka[0], ka[1], ka[2], ka[3]);
          ldsm4(qslot + boff, b0, b1, b2, b3);
          mma(st[0], ka, b0, b1);
          mma(st[1], ka, b2, b3);
          ldsm4(vbase + aoff, ka[0], ka[1], ka[2], ka[3]);
          ldsm4(dslot + boff, b0, b1, b2, b3);
          mma(pt[0], ka, b0, b1);
          mma(pt[1], ka, b2, b3);
        }
      }
      // ---- P^T (masked where the key is past the query) and dS^T
      uint32_t pa[4], sa[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float p[4], ds[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const int key = key0 + ((e2 >> 1) << 3);
          p[e2] = key <= i ? fast_exp2(fmaf(st[nt][e2], c, nl[nt][e2 & 1])) : 0.f;
          ds[e2] = p[e2] * (pt[nt][e2] - Dv[nt][e2 & 1]);
        }
        pa[2 * nt + 0] = bf2(p[0], p[1]);
        pa[2 * nt + 1] = bf2(p[2], p[3]);
        sa[2 * nt + 0] = bf2(ds[0], ds[1]);
        sa[2 * nt + 1] = bf2(ds[2], ds[3]);
      }
      // ---- dV += P^T dO and dK += dS^T Q (heads as the contraction)
      {
        const int hrow = rr + ((mi & 1) << 3);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          const int nt = 2 * np;
          const uint32_t off = (nt >> 3) * kRowsB + swz(hrow, (nt & 7) + (mi >> 1));
          uint32_t b0, b1, b2, b3;
          ldsm4t(dslot + off, b0, b1, b2, b3);
          mma(dva[nt], pa, b0, b1);
          mma(dva[nt + 1], pa, b2, b3);
          ldsm4t(qslot + off, b0, b1, b2, b3);
          mma(dka[nt], sa, b0, b1);
          mma(dka[nt + 1], sa, b2, b3);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * ts);
    }
    if (!ok) break;
    // ---- add this chunk's dk, dv of keys key0 and key0 + 8
    {
      const int k0 = key0, k1 = key0 + 8;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const int col = nt * 8 + 2 * tig;
        if (k0 < a.n) {
          const size_t o0 = ((size_t)k0 * a.h_kv + g) * 128 + col;
          atomicAdd(reinterpret_cast<float2*>(a.dk + o0), make_float2(dka[nt][0] * a.scale, dka[nt][1] * a.scale));
          atomicAdd(reinterpret_cast<float2*>(a.dv + o0), make_float2(dva[nt][0], dva[nt][1]));
        }
        if (k1 < a.n) {
          const size_t o1 = ((size_t)k1 * a.h_kv + g) * 128 + col;
          atomicAdd(reinterpret_cast<float2*>(a.dk + o1), make_float2(dka[nt][2] * a.scale, dka[nt][3] * a.scale));
          atomicAdd(reinterpret_cast<float2*>(a.dv + o1), make_float2(dva[nt][2], dva[nt][3]));
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(kvempty0 + 8 * ksl);
  }
}


struct BwdPlan {
  size_t off_ld = 0, off_cnt = 0, off_off = 0, off_cur = 0, off_list = 0, off_items = 0,
         off_nitems = 0, total = 0;
  long long max_items = 0;
  int n_blk = 0;
};

BwdPlan plan_bwd(const infv2_params* p, int n) {
  BwdPlan b;
  b.n_blk = (n + 63) / 64;
  const long long nb = (long long)p->h_kv * b.n_blk;
  // work items: sparse lists hold at most n*k entries per kv head; dense block
  // b holds n - 64b tokens
  long long dense_items = 0;
  for (int x = 0; x < b.n_blk; ++x) dense_items += (n - 64 * x + kChunkTok - 1) / kChunkTok;
  dense_items *= p->h_kv;
  const long long sparse_items = nb + ((long long)p->h_kv * n * p->k + kChunkTok - 1) / kChunkTok;
  b.max_items = dense_items > sparse_items ? dense_items : sparse_items;
  size_t off = 0;
  b.off_ld = off;
  off += round256((size_t)p->h_kv * n * 32 * 4);
  b.off_cnt = off;
  off += round256((size_t)nb * 4);
  b.off_off = off;
  off += round256((size_t)nb * 4);
  b.off_cur = off;
  off += round256((size_t)nb * 4);
  b.off_list = off;
  off += round256((size_t)p->h_kv * n * p->k * 4);
  b.off_items = off;
  off += round256((size_t)b.max_items * 16);
  b.off_nitems = off;
  off += 256;
  b.total = off;
  return b;
}

}  // namespace

int launch_attn_bwd(const infv2_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    const int* idx, long long idx_hstride, int n, const uint16_t* o,
                    const float* lse, long long lse_ld, const uint16_t* d_o, float* dq, float* dk,
                    float* dv, uint8_t* ws, cudaStream_t st) {
  if (n <= 0) return INFV2_OK;
  const BwdPlan pl = plan_bwd(p, n);
  const int G = p->h_q / p->h_kv;
  float* ld = reinterpret_cast<float*>(ws + pl.off_ld);
  int* cnt = reinterpret_cast<int*>(ws + pl.off_cnt);
  int* offs = reinterpret_cast<int*>(ws + pl.off_off);
  int* cur = reinterpret_cast<int*>(ws + pl.off_cur);
  int* list = reinterpret_cast<int*>(ws + pl.off_list);
  int4* items = reinterpret_cast<int4*>(ws + pl.off_items);
  int* n_items = reinterpret_cast<int*>(ws + pl.off_nitems);
  const int sms = sm_count();
  {
    PrepArgs a{o, d_o, lse, lse_ld, n, p->h_q, p->h_kv, ld, dk, dv, idx ? cnt : nullptr,
               p->h_kv * pl.n_blk};
    const long long want = ((long long)n * p->h_q * 16 + 255) / 256;
    const long long grid = want < 8LL * sms ? want : 8LL * sms;
    bwd_prep_kernel<<<(unsigned)(grid > 0 ? grid : 1), 256, 0, st>>>(a);
    int e = launch_status(cudaGetLastError());
    if (e != INFV2_OK) return e;
  }
  if (idx) {
    IndexArgs a{idx, idx_hstride, n, p->h_kv, p->k, pl.n_blk, cnt, cur, list};
    const long long total = (long long)p->h_kv * p->k * n;
    const unsigned grid = (unsigned)((total + 255) / 256);
    bwd_index_kernel<false><<<grid, 256, 0, st>>>(a);
    int e = launch_status(cudaGetLastError());
    if (e != INFV2_OK) return e;
    bwd_scan_kernel<<<1, 1024, 0, st>>>(cnt, offs, cur, items, n_items, p->h_kv, pl.n_blk, n, 0);
    if ((e = launch_status(cudaGetLastError())) != INFV2_OK) return e;
    bwd_index_kernel<true><<<grid, 256, 0, st>>>(a);
    if ((e = launch_status(cudaGetLastError())) != INFV2_OK) return e;
  } else {
    bwd_scan_kernel<<<1, 1024, 0, st>>>(cnt, offs, cur, items, n_items, p->h_kv, pl.n_blk, n, 1);
    int e = launch_status(cudaGetLastError());
    if (e != INFV2_OK) return e;
  }
  CUtensorMap tm_q, tm_do, tm_k, tm_v;
  if (!make_tmap_3d(&tm_q, q, 128, p->h_q, n, 256, (uint64_t)p->h_q * 256, 64, G, 1) ||
      !make_tmap_3d(&tm_do, d_o, 128, p->h_q, n, 256, (uint64_t)p->h_q * 256, 64, G, 1) ||
      !make_tmap_3d(&tm_k, k, 128, p->h_kv, n, 256, (uint64_t)p->h_kv * 256, 64, 1, 64) ||
      !make_tmap_3d(&tm_v, v, 128, p->h_kv, n, 256, (uint64_t)p->h_kv * 256, 64, 1, 64))
    return INFV2_ERR_CUDA;
  const float scale_log2 = p->scale * kLog2e;
  {
    DqArgs a{n, p->h_q, p->h_kv, p->k, idx, idx_hstride, scale_log2, p->scale, ld, dq, wait_ctx()};
    const int smem = kDqStages * kStageB + 2 * kTokSlot + 8 * (2 * kDqStages + 5) + 1024;
    if (!set_smem(bwd_dq_kernel, smem)) return INFV2_ERR_CUDA;
    const long long items_dq = (long long)p->h_kv * n;
    const long long grid = items_dq < 2LL * sms ? items_dq : 2LL * sms;
    bwd_dq_kernel<<<(unsigned)grid, 160, smem, st>>>(tm_q, tm_do, tm_k, tm_v, a);
    int e = launch_status(cudaGetLastError());
    if (e != INFV2_OK) return e;
  }
  {
    DkvArgs a{n, p->h_q, p->h_kv, pl.n_blk, idx ? list : nullptr, offs, items, n_items,
              scale_log2, p->scale, ld, dk, dv, wait_ctx()};
    const int smem = 2 * kStageB + kTokRing * kTokSlot + 8 * (4 + 2 * kTokRing) + 1024;
    if (!set_smem(bwd_dkv_kernel, smem)) return INFV2_ERR_CUDA;
    const long long grid = pl.max_items < 2LL * sms ? pl.max_items : 2LL * sms;
    bwd_dkv_kernel<<<(unsigned)(grid > 0 ? grid : 1), 160, smem, st>>>(tm_q, tm_do, tm_k, tm_v, a);
    int e = launch_status(cudaGetLastError());
    if (e != INFV2_OK) return e;
  }
  return INFV2_OK;
}

size_t attn_bwd_workspace(const infv2_params* p, int n) { return n > 0 ? plan_bwd(p, n).total : 0; }

}  // namespace infv2

using namespace infv2;

extern "C" int infv2_sparse_attn_bwd_workspace_size(const infv2_params* p, int n, size_t* bytes) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0 || !bytes) return INFV2_ERR_INVALID_ARG;
  *bytes = attn_bwd_workspace(p, n);
  return INFV2_OK;
}

extern "C" int infv2_sparse_attn_bwd(const infv2_params* p, const void* q, const void* k,
                                     const void* v, const int* idx, int n, const void* o,
                                     const float* lse, const void* d_o, float* dq, float* dk,
                                     float* dv, void* workspace, size_t ws_bytes,
                                     infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0) return INFV2_ERR_INVALID_ARG;
  if (n == 0) return INFV2_OK;
  if (!q || !k || !v || !o || !lse || !d_o || !dq || !dk || !dv) return INFV2_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < attn_bwd_workspace(p, n)) return INFV2_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return INFV2_ERR_INVALID_ARG;
  return launch_attn_bwd(p, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                         static_cast<const uint16_t*>(v), idx, (long long)n * p->k, n,
                         static_cast<const uint16_t*>(o), lse, n, static_cast<const uint16_t*>(d_o),
                         dq, dk, dv, static_cast<uint8_t*>(workspace),
                         reinterpret_cast<cudaStream_t>(stream));
}
