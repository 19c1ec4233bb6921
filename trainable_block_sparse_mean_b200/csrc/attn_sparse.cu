// Stage 5: block-sparse causal attention over the selected KV blocks.
//
// arXiv summary, Appendix A: queries are processed in parallel, each walks only
// the key/value blocks that belong to its visible-token set, and the kernel
// returns O and the log-sum-exp.  MiniCPM4 blog (query/key granularity): the
// query unit is one token, and the heads of a GQA group share its block set.
//
// Where it runs: the decode step (one query token per sequence), and prefill
// with block lists at group sizes G <= 2 or with lists longer than the
// tensor-core kernel stages ((128/G) * k > 2048 entries per tile); attn_tc.cu
// takes every other prefill shape.  A work item is one (kv head g,
// query token i): the G <= 16 query heads of the group form a 16-row tile (the
// group is the only reuse a single token's block set allows).  Each selected
// 64-token block of K and V (2 x 16 KB) is fetched by TMA into a 2-stage
// shared-memory ring by a producer warp; four consumer warps each own 16 of the
// block's 64 keys and run S = Q K^T and O += P V as m16n8k16 bf16 MMAs with
// fp32 accumulation and an online softmax, then merge their partial (max, sum,
// O) through shared memory.  Two CTAs share an SM (2 stages keep both in
// shared memory); the grid is persistent (two CTAs per SM) and walks the items
// kv head by kv head so that one head's K/V stays resident in L2.
//
// In the decode step a row is a sequence of the batch (K/V in cache layout,
// query position from seqlens), and the block list is cut so that several CTAs
// share one row; the pieces write unnormalised partial outputs, and the last
// piece of a row merges them and advances the row's length.
#include "attn_sparse.cuh"
#include "common.cuh"

namespace infv2 {
namespace {

constexpr int kStages = 2;                // 2 stages -> two CTAs fit on one SM
constexpr int kHalf = 64 * 64 * 2;        // 64 keys x 64 dims of bf16 = 8 KB
// A row's reference max is only raised when a block's max exceeds it by more
// than this (log2 units): probabilities stay below 2^8, and O, l are rescaled
// rarely.  The final normalisation makes the result independent of it.
constexpr float kRescaleSlack = 8.0f;
constexpr int kMaxSplit = 16;             // most pieces a split row may have
constexpr int kStageBytes = 4 * kHalf;    // K (2 halves) + V (2 halves)
constexpr int kQHalf = 16 * 128;          // 16 heads x 64 dims of bf16 = 2 KB
constexpr int kQSlot = 2 * kQHalf;        // one item's Q rows
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of (key, 16-byte chunk) inside one 64x64 half stored with the
// 128-byte TMA swizzle.
__device__ __forceinline__ uint32_t sw_off(int key, int chunk) {
  return (uint32_t)(key * 128 + ((chunk ^ (key & 7)) << 4));
}

struct Item {
  int g, r, sp;
};

__device__ __forceinline__ Item item_of(const AttnArgs& a, long long w) {
  Item it;
  const long long per_g = (long long)a.n_rows * a.n_split;
  it.g = (int)(w / per_g);
  const long long rem = w % per_g;
  it.r = a.row_begin + (int)(rem / a.n_split);
  it.sp = (int)(rem % a.n_split);
  return it;
}

// Entries [e_begin, e_end) of the item's block list.  Without an index array
// (dense mode) the list is every block 0 .. pos/64 and entry e is block e.
__device__ __forceinline__ void item_range(const AttnArgs& a, const Item& it, int pos,
                                           const int*& row, int& e_begin, int& e_end) {
  if (a.idx) {
    row = a.idx + (size_t)it.g * a.idx_hstride + (size_t)it.r * a.idx_rstride;
    e_begin = it.sp * a.blocks_per_split;
    e_end = min(a.k, e_begin + a.blocks_per_split);
  } else {
    row = nullptr;
    e_begin = 0;
    e_end = (pos >> 6) + 1;
  }
}

__device__ __forceinline__ int block_at(const int* row, int e, int pos, int* err) {
  return row ? list_block(row, e, pos, err) : e;
}

__global__ void __launch_bounds__(160, 2)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_last;  // split mode: this CTA merges the pieces of its (row, kv head)
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // [K/V stages][Q ring][merge buffers][barriers]; TMA destinations with the
  // 128-byte swizzle (stages, Q ring) start on 1024-byte boundaries
  uint8_t* qring = base + kStages * kStageBytes;                          // [2][2 halves][16][128 B]
  float* red_o = reinterpret_cast<float*>(qring + 2 * kQSlot);            // [4][16][128]
  float* red_m = red_o + 4 * 16 * 128;                                    // [4][16]
  float* red_l = red_m + 64;                                              // [4][16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red_l + 64);
  const uint32_t stage0 = smem_u32(base);
  const uint32_t q0 = smem_u32(qring);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * kStages;
  const uint32_t cbar = empty0 + 8 * kStages;  // consumer-group barrier
  const uint32_t qfull0 = cbar + 8;            // Q ring: 2 slots
  const uint32_t qempty0 = qfull0 + 16;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long n_items = (long long)a.h_kv * a.n_rows * a.n_split;
  const int G = a.h_q / a.h_kv;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 4);
    }
    mbar_init(cbar, 4);
    for (int x = 0; x < 2; ++x) {
      mbar_init(qfull0 + 8 * x, 1);
      mbar_init(qempty0 + 8 * x, 4);
    }
    fence_mbar_init();
  }
  // Q rows beyond the group (G < 16) are never written by TMA: keep them zero
  for (int x = threadIdx.x; x < 2 * kQSlot / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(qring)[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      long long pc = 0, qc = 0;
      bool ok = true;
      for (long long w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++qc) {
        const Item it = item_of(a, w);
        const int pos = a.decode ? __ldg(a.seqlens + it.r) : it.r;
        {  // this item's Q rows (the G heads of group g) into the Q ring
          const int qs = (int)(qc & 1);
          if (!mbar_wait(qempty0 + 8 * qs, (uint32_t)((qc >> 1) & 1) ^ 1u, a.wait)) break;
          mbar_expect_tx(qfull0 + 8 * qs, 2 * G * 128);
          tma_load_3d(q0 + qs * kQSlot, &tm_q, qfull0 + 8 * qs, 0, it.g * G, it.r);
          tma_load_3d(q0 + qs * kQSlot + kQHalf, &tm_q, qfull0 + 8 * qs, 64, it.g * G, it.r);
        }
        const int* row;
        int e0, e1;
        item_range(a, it, pos, row, e0, e1);
        for (int e = e0; e < e1; ++e) {
          const int b = block_at(row, e, pos, a.wait.err);
          if (b < 0) continue;
          const int s = (int)(pc % kStages);
          if (!mbar_wait(empty0 + 8 * s, (uint32_t)((pc / kStages) & 1) ^ 1u, a.wait)) {
            ok = false;
            break;
          }
          const uint32_t dst = stage0 + s * kStageBytes;
          const uint32_t fb = full0 + 8 * s;
          mbar_expect_tx(fb, kStageBytes);
          int c1, c2;
          if (a.decode) {
            c1 = 64 * b;
            c2 = it.r * a.h_kv + it.g;
          } else {
            c1 = it.g;
            c2 = 64 * b;
          }
          tma_load_3d(dst, &tm_k, fb, 0, c1, c2);
          tma_load_3d(dst + kHalf, &tm_k, fb, 64, c1, c2);
          tma_load_3d(dst + 2 * kHalf, &tm_v, fb, 0, c1, c2);
          tma_load_3d(dst + 3 * kHalf, &tm_v, fb, 64, c1, c2);
          ++pc;
        }
      }
      for (long long x = pc > kStages ? pc - kStages : 0; x < pc; ++x)
        (void)mbar_wait(full0 + 8 * (int)(x % kStages), (uint32_t)((x / kStages) & 1), a.wait);
      for (long long x = qc > 2 ? qc - 2 : 0; x < qc; ++x)
        (void)mbar_wait(qfull0 + 8 * (int)(x & 1), (uint32_t)((x >> 1) & 1), a.wait);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gid = lane >> 2, tig = lane & 3;
  const int kb = warp * 16;  // this warp's 16 keys of every block
  const float c = a.scale_log2;
  long long cc = 0;
  uint32_t cphase = 0;
  bool ok = true;
  long long qc = 0;
  for (long long w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++qc) {
    const Item it = item_of(a, w);
    const int pos = a.decode ? __ldg(a.seqlens + it.r) : it.r;  // query position
    // Q fragments (A operand, 16 rows = heads of the group) from the Q ring
    uint32_t qa[8][4];
    {
      const int qs = (int)(qc & 1);
      if (!mbar_wait(qfull0 + 8 * qs, (uint32_t)((qc >> 1) & 1), a.wait)) break;
      const int mi = lane >> 3, rr = lane & 7;
      const int row = rr + ((mi & 1) << 3);  // matrices: rows 0-7 / 8-15, k 0-7 / 8-15
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int chunk = (ks & 3) * 2 + (mi >> 1);
        ldsm_x4(q0 + qs * kQSlot + (ks >> 2) * kQHalf + sw_off(row, chunk), qa[ks][0], qa[ks][1],
                qa[ks][2], qa[ks][3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(qempty0 + 8 * qs);
    }
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    const int* row;
    int e0, e1;
    item_range(a, it, pos, row, e0, e1);
    int chunk_b = 0;
    for (int e = e0; e < e1; ++e) {
      if (((e - e0) & 31) == 0)  // next 32 entries of the list, one per lane
        chunk_b = e + lane < e1 ? block_at(row, e + lane, pos, a.wait.err) : -1;
      const int b = __shfl_sync(0xFFFFFFFFu, chunk_b, (e - e0) & 31);
      if (b < 0) continue;
      const int s = (int)(cc % kStages);
      if (!mbar_wait(full0 + 8 * s, (uint32_t)((cc / kStages) & 1), a.wait)) {
        ok = false;
        break;
      }
      const uint32_t kbase = stage0 + s * kStageBytes;
      const uint32_t vbase = kbase + 2 * kHalf;
      // ---- S = Q K^T for keys kb..kb+15 (two n-tiles of 8 keys); the two
      // head-dim halves accumulate separately: four independent MMA chains
      float sc[2][4], sd[2][4];
#pragma unroll
      for (int x = 0; x < 4; ++x) sc[0][x] = sc[1][x] = sd[0][x] = sd[1][x] = 0.f;
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = kb + rr + ((mi >> 1) << 3);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint32_t b0, b1, b2, b3, e0, e1, e2, e3;
          ldsm_x4(kbase + sw_off(key, ks * 2 + (mi & 1)), b0, b1, b2, b3);
          ldsm_x4(kbase + kHalf + sw_off(key, ks * 2 + (mi & 1)), e0, e1, e2, e3);
          mma16816(sc[0], qa[ks], b0, b1);
          mma16816(sc[1], qa[ks], b2, b3);
          mma16816(sd[0], qa[ks + 4], e0, e1);
          mma16816(sd[1], qa[ks + 4], e2, e3);
        }
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        sc[0][x] += sd[0][x];
        sc[1][x] += sd[1][x];
      }
      // ---- causal mask (only a block reaching past the query) and online
      // softmax with a lazily raised reference max (rows gid and gid+8).  The
      // max is taken on the unscaled scores (scale > 0) and the scale is folded
      // into the exponent argument: p = 2^(s*c - ref), one packed FMA per pair.
      const int t0 = 64 * b + kb;
      if (64 * b + 63 > pos) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int t = t0 + nt * 8 + 2 * tig + (e2 & 1);
            if (t > pos) sc[nt][e2] = -INFINITY;
          }
      }
      float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
      float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 2));
      mx0 *= c;
      mx1 *= c;
      const bool raise = mx0 > m0 + kRescaleSlack || mx1 > m1 + kRescaleSlack;
      if (__any_sync(0xFFFFFFFFu, raise)) {
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = mn0 == -INFINITY ? 1.f : fast_exp2(m0 - mn0);
        const float al1 = mn1 == -INFINITY ? 1.f : fast_exp2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          o[nt][0] *= al0;
          o[nt][1] *= al0;
          o[nt][2] *= al1;
          o[nt][3] *= al1;
        }
      }
      const float2 cpair = make_float2(c, c);
      const float2 nr0 = make_float2(m0 == -INFINITY ? 0.f : -m0, m0 == -INFINITY ? 0.f : -m0);
      const float2 nr1 = make_float2(m1 == -INFINITY ? 0.f : -m1, m1 == -INFINITY ? 0.f : -m1);
      float p[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float2 x01 = ffma2(make_float2(sc[nt][0], sc[nt][1]), cpair, nr0);
        const float2 x23 = ffma2(make_float2(sc[nt][2], sc[nt][3]), cpair, nr1);
        p[nt][0] = fast_exp2(x01.x);
        p[nt][1] = fast_exp2(x01.y);
        p[nt][2] = fast_exp2(x23.x);
        p[nt][3] = fast_exp2(x23.y);
      }
      l0 += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
      l1 += (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
      uint32_t pa[4];
      pa[0] = pack_bf16(p[0][0], p[0][1]);
      pa[1] = pack_bf16(p[0][2], p[0][3]);
      pa[2] = pack_bf16(p[1][0], p[1][1]);
      pa[3] = pack_bf16(p[1][2], p[1][3]);
      // ---- O += P V (16 n-tiles of 8 dims, two per ldmatrix.x4.trans)
      {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = kb + rr + ((mi & 1) << 3);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          const int nt = 2 * np;
          const int chunk = (nt & 7) + (mi >> 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vbase + (nt >> 3) * kHalf + sw_off(key, chunk), b0, b1, b2, b3);
          mma16816(o[nt], pa, b0, b1);
          mma16816(o[nt + 1], pa, b2, b3);
        }
      }
      // The stage was read through the generic proxy (ldmatrix) and will be
      // rewritten by TMA (async proxy): order the two before releasing it.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
      ++cc;
    }
    if (!ok) break;

    // ---- merge the four warps' partial results
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
    if (tig == 0) {
      red_m[warp * 16 + gid] = m0;
      red_m[warp * 16 + gid + 8] = m1;
      red_l[warp * 16 + gid] = l0;
      red_l[warp * 16 + gid + 8] = l1;
    }
    float* ro = red_o + warp * 16 * 128;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int col = nt * 8 + 2 * tig;
      *reinterpret_cast<float2*>(ro + gid * 128 + col) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2*>(ro + (gid + 8) * 128 + col) = make_float2(o[nt][2], o[nt][3]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    if (!mbar_wait(cbar, cphase & 1u, a.wait)) break;
    ++cphase;
    {
      const int t = threadIdx.x;  // 0..127
      const int rowh = t >> 3;    // head within the group
      const int d0 = (t & 7) * 16;
      if (rowh < G) {
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < 4; ++q) M = fmaxf(M, red_m[q * 16 + rowh]);
        float sc4[4];
        float L = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          sc4[q] = M == -INFINITY ? 0.f : fast_exp2(red_m[q * 16 + rowh] - M);
          L += red_l[q * 16 + rowh] * sc4[q];
        }
        float acc[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) acc[x] = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float* src = red_o + (q * 16 + rowh) * 128 + d0;
#pragma unroll
          for (int x = 0; x < 16; ++x) acc[x] += src[x] * sc4[q];
        }
        const int h = it.g * G + rowh;
        if (!a.split_out) {
          const float inv = L > 0.f ? 1.f / L : 0.f;
          uint4 w0, w1;
          w0.x = pack_bf16(acc[0] * inv, acc[1] * inv);
          w0.y = pack_bf16(acc[2] * inv, acc[3] * inv);
          w0.z = pack_bf16(acc[4] * inv, acc[5] * inv);
          w0.w = pack_bf16(acc[6] * inv, acc[7] * inv);
          w1.x = pack_bf16(acc[8] * inv, acc[9] * inv);
          w1.y = pack_bf16(acc[10] * inv, acc[11] * inv);
          w1.z = pack_bf16(acc[12] * inv, acc[13] * inv);
          w1.w = pack_bf16(acc[14] * inv, acc[15] * inv);
          uint16_t* dst = a.o + ((size_t)it.r * a.h_q + h) * 128 + d0;
          reinterpret_cast<uint4*>(dst)[0] = w0;
          reinterpret_cast<uint4*>(dst)[1] = w1;
          if (INFV2_CHECKS) {  // debug build: every output finite
            bool fin = true;
#pragma unroll
            for (int x = 0; x < 16; ++x) fin = fin && isfinite(acc[x] * inv);
            check(fin, a.wait.err);
          }
          if (a.lse && (t & 7) == 0)
            a.lse[(size_t)h * a.lse_ld + it.r] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
        } else {
          const size_t slot = ((size_t)it.r * a.h_q + h) * a.n_split + it.sp;
          float* dst = a.part_o + slot * 128 + d0;
#pragma unroll
          for (int x = 0; x < 16; x += 4)
            *reinterpret_cast<float4*>(dst + x) = make_float4(acc[x], acc[x + 1], acc[x + 2], acc[x + 3]);
          if ((t & 7) == 0) {
            a.part_ml[slot * 2 + 0] = M;
            a.part_ml[slot * 2 + 1] = L;
          }
        }
      }
      if (a.split_out) __threadfence();  // this piece is visible before it is counted
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    if (!mbar_wait(cbar, cphase & 1u, a.wait)) break;
    ++cphase;
    if (a.split_out) {
      // the last piece of (row, kv head) to finish merges all pieces
      if (threadIdx.x == 0) s_last = atomicAdd(&a.counters[(size_t)it.r * a.h_kv + it.g], 1) == a.n_split - 1;
      __syncwarp();
      if (lane == 0) mbar_arrive(cbar);
      if (!mbar_wait(cbar, cphase & 1u, a.wait)) break;
      ++cphase;
      if (s_last) {
        __threadfence();
        const int t = threadIdx.x;
        const int rowh = t >> 3;
        const int d0 = (t & 7) * 16;
        if (rowh < G) {
          const int h = it.g * G + rowh;
          const size_t slot0 = ((size_t)it.r * a.h_q + h) * a.n_split;
          // all pieces' (max, sum) first, independent loads in flight
          float2 mlv[kMaxSplit];
#pragma unroll
          for (int sp = 0; sp < kMaxSplit; ++sp)
            mlv[sp] = sp < a.n_split
                          ? __ldcg(reinterpret_cast<const float2*>(a.part_ml + (slot0 + sp) * 2))
                          : make_float2(-INFINITY, 0.f);
          float M = -INFINITY;
#pragma unroll
          for (int sp = 0; sp < kMaxSplit; ++sp) M = fmaxf(M, mlv[sp].x);
          float L = 0.f, acc[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) acc[x] = 0.f;
          if (M != -INFINITY) {
#pragma unroll 4
            for (int sp = 0; sp < kMaxSplit; ++sp) {
              if (sp >= a.n_split) break;
              const float sc = mlv[sp].x == -INFINITY ? 0.f : fast_exp2(mlv[sp].x - M);
              L += mlv[sp].y * sc;
              const float4* src = reinterpret_cast<const float4*>(a.part_o + (slot0 + sp) * 128 + d0);
              const float4 v0 = __ldcg(src), v1 = __ldcg(src + 1), v2 = __ldcg(src + 2),
                           v3 = __ldcg(src + 3);
              const float4 vv[4] = {v0, v1, v2, v3};
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                acc[4 * x + 0] += vv[x].x * sc;
                acc[4 * x + 1] += vv[x].y * sc;
                acc[4 * x + 2] += vv[x].z * sc;
                acc[4 * x + 3] += vv[x].w * sc;
              }
            }
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
          uint4 w0, w1;
          w0.x = pack_bf16(acc[0] * inv, acc[1] * inv);
          w0.y = pack_bf16(acc[2] * inv, acc[3] * inv);
          w0.z = pack_bf16(acc[4] * inv, acc[5] * inv);
          w0.w = pack_bf16(acc[6] * inv, acc[7] * inv);
          w1.x = pack_bf16(acc[8] * inv, acc[9] * inv);
          w1.y = pack_bf16(acc[10] * inv, acc[11] * inv);
          w1.z = pack_bf16(acc[12] * inv, acc[13] * inv);
          w1.w = pack_bf16(acc[14] * inv, acc[15] * inv);
          uint16_t* dst = a.o + ((size_t)it.r * a.h_q + h) * 128 + d0;
          reinterpret_cast<uint4*>(dst)[0] = w0;
          reinterpret_cast<uint4*>(dst)[1] = w1;
          if (INFV2_CHECKS) {  // debug build: every output finite
            bool fin = true;
#pragma unroll
            for (int x = 0; x < 16; ++x) fin = fin && isfinite(acc[x] * inv);
            check(fin, a.wait.err);
          }
          if (a.lse && (t & 7) == 0)
            a.lse[(size_t)it.r * a.h_q + h] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
        }
        if (t == 0) {
          a.counters[(size_t)it.r * a.h_kv + it.g] = 0;
          int* seq_done = a.counters + (size_t)a.n_rows * a.h_kv + it.r;
          if (atomicAdd(seq_done, 1) == a.h_kv - 1) {  // every kv head of this row merged
            *seq_done = 0;
            if (a.decode && pos >= 0 && pos < a.cap) a.seqlens_out[it.r] = pos + 1;
          }
        }
      }
    }
  }
}

}  // namespace

int launch_sparse_attn(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const AttnArgs& a,
                       cudaStream_t st) {
  const long long n_items = (long long)a.h_kv * a.n_rows * a.n_split;
  if (n_items == 0) return INFV2_OK;
  const int G = a.h_q / a.h_kv;
  CUtensorMap tm_q;  // q [rows, h_q, 128]: one item = G heads of one row
  if (!make_tmap_3d(&tm_q, a.q, 128, a.h_q, a.row_begin + a.n_rows, 256, (uint64_t)a.h_q * 256,
                    64, G, 1))
    return INFV2_ERR_CUDA;
  const int smem = kStages * kStageBytes + (4 * 16 * 128 + 128) * 4 + 2 * kQSlot +
                   8 * (2 * kStages + 1 + 4) + 1024;
  if (!set_smem(sparse_attn_kernel, smem)) return INFV2_ERR_CUDA;
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sparse_attn_kernel, 160, smem) !=
          cudaSuccess || per_sm < 1)
    per_sm = 1;
  const long long slots = (long long)per_sm * sm_count();
  const long long grid = n_items < slots ? n_items : slots;
  sparse_attn_kernel<<<(unsigned)grid, 160, smem, st>>>(tm_q, tm_k, tm_v, a);
  return launch_status(cudaGetLastError());
}

// Prefill form: K/V [n, h_kv, 128], idx [h_kv, n, k] with the given strides.
int launch_sparse_attn_rows(const infv2_params* p, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, const int* idx, long long idx_hstride, int n,
                            int r0, int r1, uint16_t* o, float* lse, long long lse_ld,
                            cudaStream_t st) {
  if (r0 < 0 || r1 > n || r0 > r1) return INFV2_ERR_INVALID_ARG;
  if (r1 == r0) return INFV2_OK;
  // tiles of 128 (token, head) rows on the tensor cores wherever the shape allows
  if (attn_tc_supports(p, idx == nullptr))
    return launch_attn_tc(p, q, k, v, idx, idx_hstride, n, r0, r1, o, lse, lse_ld, st);
  CUtensorMap tm_k, tm_v;
  if (!make_tmap_3d(&tm_k, k, 128, p->h_kv, n, 256, (uint64_t)p->h_kv * 256, 64, 1, 64) ||
      !make_tmap_3d(&tm_v, v, 128, p->h_kv, n, 256, (uint64_t)p->h_kv * 256, 64, 1, 64))
    return INFV2_ERR_CUDA;
  AttnArgs a{};
  a.n_rows = r1 - r0;
  a.row_begin = r0;
  a.h_q = p->h_q;
  a.h_kv = p->h_kv;
  a.k = p->k;
  a.idx = idx;
  a.idx_hstride = idx_hstride;
  a.idx_rstride = p->k;
  a.q = q;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.o = o;
  a.lse = lse;
  a.lse_ld = lse_ld;
  a.decode = 0;
  a.n_split = 1;
  a.blocks_per_split = p->k;
  a.split_out = 0;
  a.wait = wait_ctx();
  return launch_sparse_attn(tm_k, tm_v, a, st);
}

int launch_sparse_attn_prefill(const infv2_params* p, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const int* idx, long long idx_hstride, int n,
                               uint16_t* o, float* lse, long long lse_ld, cudaStream_t st) {
  if (n <= 0) return INFV2_OK;
  return launch_sparse_attn_rows(p, q, k, v, idx, idx_hstride, n, 0, n, o, lse, lse_ld, st);
}

}  // namespace infv2

using namespace infv2;

extern "C" int infv2_sparse_attn(const infv2_params* p, const void* q, const void* k,
                                 const void* v, const int* idx, int n, void* o, float* lse,
                                 infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0) return INFV2_ERR_INVALID_ARG;
  if (n == 0) return INFV2_OK;
  if (!q || !k || !v || !idx || !o) return INFV2_ERR_INVALID_ARG;
  return launch_sparse_attn_prefill(p, static_cast<const uint16_t*>(q),
                                    static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
                                    idx, (long long)n * p->k, n, static_cast<uint16_t*>(o), lse, n,
                                    reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int infv2_sparse_attn_rows(const infv2_params* p, const void* q, const void* k,
                                      const void* v, const int* idx, int n, int r0, int r1,
                                      void* o, float* lse, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0 || r0 < 0 || r1 > n || r0 > r1) return INFV2_ERR_INVALID_ARG;
  if (r0 == r1) return INFV2_OK;
  if (!q || !k || !v || !o) return INFV2_ERR_INVALID_ARG;
  return launch_sparse_attn_rows(p, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                 static_cast<const uint16_t*>(v), idx, idx ? (long long)n * p->k : 0,
                                 n, r0, r1, static_cast<uint16_t*>(o), lse, n,
                                 reinterpret_cast<cudaStream_t>(stream));
}

namespace infv2 {
// Dense causal attention through the same kernel with every visible block.
int launch_dense_attn_blocks(const infv2_params* p, const uint16_t* q, const uint16_t* k,
                             const uint16_t* v, int n, uint16_t* o, float* lse, long long lse_ld,
                             cudaStream_t st) {
  return launch_sparse_attn_prefill(p, q, k, v, nullptr, 0, n, o, lse, lse_ld, st);
}
}  // namespace infv2
