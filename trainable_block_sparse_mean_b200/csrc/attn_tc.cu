// Stage 5 on the fifth-generation tensor cores: block-sparse (or dense) causal
// attention over query tiles of 128 (token, head) rows.
//
// arXiv summary, Appendix A: the sparse kernel follows FlashAttention-style
// tiling while its inner loop visits only the key/value blocks a query
// selected, and it returns O together with the log-sum-exp.  MiniCPM4 blog
// (query/key granularity, top-k sharing): the query unit is one token and the
// heads of a GQA group share that token's block set.
//
// B200 design.  A tile is TQ = 128/G consecutive tokens times the G query heads
// of kv head g: 128 rows, one per TMEM lane.  Neighbouring tokens share part of
// their block sets, so a tile walks the UNION of its tokens' lists; the producer
// warp merges the lists and tags each union block with the mask of the tokens
// that chose it.  Every union block's K and V (64 keys x 128 dims each) is
// fetched once by TMA and serves all 128 rows:
//   S  = Q K^T   tcgen05 M=128 N=64 per block, K=128; A = Q in TMEM, B = K in
//                shared memory
//   softmax      four threads per row; rows whose token did not choose the block
//                get P = 0 (a warp with no such row only stores zeros)
//   O += P V     tcgen05 M=128 N=128 K=64; A = P (bf16, written over S's
//                columns) in TMEM, B = V in shared memory (MN-major)
// Shared memory therefore carries only K and V; Q, S, P and O stay in TMEM.
// Union entries go in pairs: one QK product covers two blocks (N = 128 keys),
// which is what keeps the tensor core's instruction issue, not its datapath,
// from setting the pace (a 64-key product issues at two thirds of the rate).
// The kernel is otherwise a pipeline of latencies and is organised so that no
// role waits on the one before it more than it must:
//  - K and V have separate rings of pair slots with their own producers: a K
//    slot is free again as soon as its QK product completes, a V slot once its
//    PV product does;
//  - two MMA warps: one issues the QK products, the other the PV products, so
//    that each one's barrier waits overlap the other's issue;
//  - S has two TMEM buffers of a pair each, so QK of the next pair runs while
//    the softmax of this one does;
//  - eight softmax warps, two per TMEM lane quarter, each own 16 rows (one
//    token at G = 16) through the 16-lane TMEM load/store shapes, so a row's
//    maximum and sum are reduced over four threads, and every SM sub-partition
//    has a second warp to hide latency;
//  - a row's reference max is raised only when a pair's max exceeds it by more
//    than 8 (log2 units); O is then rescaled in TMEM, so most pairs skip it;
//  - a quarter of the exponentials run on the FMA pipe (exp2_cubic2), and P is
//    rounded to bf16 with integer adds and a byte permute.
// Blocks a row did not choose add exact zeros.  The reference max of a row
// depends on the pairs its tile walks, so a row's bits are the same in any
// launch whose row range starts and ends on tile boundaries (multiples of
// 128/G tokens); other cuts agree within rounding.  Q is double-buffered in
// TMEM: the next tile's QK products start while this tile's O is read out.
// Warp roles: warp 0 merges the lists, publishes the union pairs and loads Q
// and K; warp 10 loads V; warp 1 issues the QK products and owns TMEM; warp 11
// issues the PV products; warps 2-9 copy Q into TMEM (2-5), run the softmax
// and write O and the log-sum-exp.
// Dense mode (no lists): a tile's union is every block up to its last token,
// and causality alone masks.  The grid is persistent: CTA x takes tiles x,
// x + gridDim.x, ..., ordered kv head by kv head (one head's K/V stays in L2)
// and longest rows first.
#include "attn_sparse.cuh"
#include "common.cuh"



namespace infv2 {
namespace {

constexpr int kNK = 2;                       // K ring: pair slots
constexpr int kNV = 3;                       // V ring: pair slots
constexpr int kPairBytes = 2 * 64 * 256;     // two blocks of 64 keys x 128 dims of bf16 = 32 KB
constexpr int kHalf = 64 * 128;              // 64 keys x 64 dims: one 128-byte swizzled box
constexpr int kQBytes = 128 * 256;           // 128 rows x 128 bf16
constexpr int kMetaRing = 16;                // published union pairs
constexpr int kThreads = 12 * 32;
constexpr uint32_t kColO = 0;                // TMEM columns: O [128 x 128 fp32]
constexpr uint32_t kColS = 128;              //   S / P: two buffers of a pair (128 columns)
constexpr uint32_t kColQ = 384;              //   Q: two buffers of 64 columns (128 bf16)
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleSlack = 8.0f;        // a row's reference max trails its max by <= 8
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kBars = 2 * kNK + 2 * kNV + 6 + kMetaRing + 7;

struct TcArgs {
  int row_lo, row_hi;          // query rows computed: [row_lo, row_hi)
  int tile_last, n_tiles;      // tiles tile_last - n_tiles + 1 .. tile_last
  int h_q, h_kv, k;
  const int* idx;              // block lists (g, row) at idx + g*idx_hstride + row*idx_rstride;
  long long idx_hstride, idx_rstride;  // null: dense causal attention
  float scale_log2;            // scale * log2(e)
  uint16_t* o;                 // o + (row*h_q + h)*128
  float* lse;                  // lse[h*lse_ld + row] (natural), nullable
  long long lse_ld;
  WaitCtx wait;
};

struct Tile {
  int g, i0, lo, hi;  // kv head, first token of the tile, rows [lo, hi) computed
};

template <int TQ>
__device__ __forceinline__ Tile tile_of(const TcArgs& a, long long w) {
  Tile t;
  t.g = (int)(w / a.n_tiles);
  const int tt = a.tile_last - (int)(w % a.n_tiles);
  t.i0 = tt * TQ;
  t.lo = max(t.i0, a.row_lo);
  t.hi = min(t.i0 + TQ, a.row_hi);
  return t;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two non-negative finite floats to a bf16 pair on the integer pipes: add half
// an ulp of bf16 and keep the high halves (round to nearest, ties away from
// zero; an exponential is essentially never an exact tie).
__device__ __forceinline__ uint32_t pack_bf16_int(float lo, float hi) {
  return __byte_perm(__float_as_uint(lo) + 0x8000u, __float_as_uint(hi) + 0x8000u, 0x7632);
}

// A union pair: blocks (x, z) chosen by the tokens in masks (y, w); `last`
// closes the tile.  A pair with one block carries a repeat of it with mask 0.
struct Pair {
  int4 bm;
  int last;
};

struct Smem {
  uint32_t kring, vring, q;                    // shared addresses
  uint8_t* qtile;
  int* list;
  Pair* meta;
  uint32_t k_full, k_empty, v_full, v_empty, s_full, s_free, p_full, meta_full;
  uint32_t qs_full, qs_empty, q_full, o_full, o_free, drain_qk, drain_pv;
};

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, TcArgs a) {
  constexpr int TQ = 128 / G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // [K ring][V ring][Q tile][lists][meta ring][exchange][barriers][TMEM address]
  Smem S;
  S.kring = smem_u32(base);
  S.vring = S.kring + kNK * kPairBytes;
  S.qtile = base + (kNK + kNV) * kPairBytes;
  S.q = smem_u32(S.qtile);
  S.list = reinterpret_cast<int*>(S.qtile + kQBytes);
  S.meta = reinterpret_cast<Pair*>(S.list + kTcListCap);
  uint64_t* bars = reinterpret_cast<uint64_t*>(S.meta + kMetaRing);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + kBars);
  S.k_full = smem_u32(bars);
  S.k_empty = S.k_full + 8 * kNK;
  S.v_full = S.k_empty + 8 * kNK;
  S.v_empty = S.v_full + 8 * kNV;
  S.s_full = S.v_empty + 8 * kNV;     // [2] S of a pair written by QK
  S.s_free = S.s_full + 16;           // [2] P of a pair read by PV: the S buffer is free again
  S.p_full = S.s_free + 16;           // [2] P of a pair written by the eight softmax warps
  S.meta_full = S.p_full + 16;        // [kMetaRing] union pair published
  S.qs_full = S.meta_full + 8 * kMetaRing;         // Q tile landed in shared memory
  S.qs_empty = S.qs_full + 8;         // Q tile copied out of shared memory
  S.q_full = S.qs_empty + 8;          // a tile's Q in TMEM (one phase per tile)
  S.o_full = S.q_full + 8;            // a tile's last PV done
  S.o_free = S.o_full + 8;            // a tile's O read out
  S.drain_qk = S.o_free + 8;          // MMA warps: everything they issued done
  S.drain_pv = S.drain_qk + 8;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long n_items = (long long)a.h_kv * a.n_tiles;

  if (threadIdx.x == 0) {
    for (int x = 0; x < kNK; ++x) {
      mbar_init(S.k_full + 8 * x, 1);
      mbar_init(S.k_empty + 8 * x, 1);
    }
    for (int x = 0; x < kNV; ++x) {
      mbar_init(S.v_full + 8 * x, 1);
      mbar_init(S.v_empty + 8 * x, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(S.s_full + 8 * x, 1);
      mbar_init(S.s_free + 8 * x, 1);
      mbar_init(S.p_full + 8 * x, 8);
    }
    for (int x = 0; x < kMetaRing; ++x) mbar_init(S.meta_full + 8 * x, 1);
    mbar_init(S.qs_full, 1);
    mbar_init(S.qs_empty, 4);
    mbar_init(S.q_full, 4);
    mbar_init(S.o_full, 1);
    mbar_init(S.o_free, 8);
    mbar_init(S.drain_qk, 1);
    mbar_init(S.drain_pv, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------ list merge, union pairs, Q and K
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
    }
    uint32_t kc = 0;  // union pairs published (= K pair loads issued)
    int tc = 0;       // tiles started
    bool ok = true;
    for (long long w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++tc) {
      const Tile T = tile_of<TQ>(a, w);
      if (lane == 0) {
        ok = mbar_wait(S.qs_empty, (uint32_t)(tc & 1) ^ 1u, a.wait);
        if (ok) {
          mbar_expect_tx(S.qs_full, kQBytes);
          tma_load_3d(S.q, &tm_q, S.qs_full, 0, T.g * G, T.i0);
          tma_load_3d(S.q + kQBytes / 2, &tm_q, S.qs_full, 64, T.g * G, T.i0);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      // union entries are gathered two at a time; a full pair is published
      int hb = -1;       // held first block of the next pair (-1: none)
      uint32_t hm = 0;
      auto publish = [&](int b0, uint32_t m0, int b1, uint32_t m1, int last) -> bool {
        bool good = true;
        if (lane == 0) {
          const uint32_t ks = kc % kNK, ms = kc % kMetaRing;
          good = mbar_wait(S.k_empty + 8 * ks, ((kc / kNK) & 1u) ^ 1u, a.wait);
          if (good) {
            S.meta[ms].bm = make_int4(b0, (int)m0, b1, (int)m1);
            S.meta[ms].last = last;
            mbar_arrive(S.meta_full + 8 * ms);
            // K of the pair: rows 0-63 block b0, rows 64-127 block b1, in each half
            const uint32_t dst = S.kring + ks * kPairBytes, fb = S.k_full + 8 * ks;
            mbar_expect_tx(fb, kPairBytes);
            tma_load_3d(dst, &tm_k, fb, 0, T.g, 64 * b0);
            tma_load_3d(dst + kHalf, &tm_k, fb, 0, T.g, 64 * b1);
            tma_load_3d(dst + 2 * kHalf, &tm_k, fb, 64, T.g, 64 * b0);
            tma_load_3d(dst + 3 * kHalf, &tm_k, fb, 64, T.g, 64 * b1);
          }
        }
        good = __shfl_sync(0xFFFFFFFFu, good, 0);
        if (good) ++kc;
        return good;
      };
      auto entry = [&](int b, uint32_t m) -> bool {
        if (hb < 0) {
          hb = b;
          hm = m;
          return true;
        }
        const bool good = publish(hb, hm, b, m, 0);
        hb = -1;
        return good;
      };
      // the tile's last entry closes it (an empty union runs one all-masked block)
      auto close = [&](int b, uint32_t m) -> bool {
        if (hb < 0) return publish(b, m, b, 0u, 1);
        const bool good = publish(hb, hm, b, m, 1);
        hb = -1;
        return good;
      };
      if (a.idx == nullptr) {
        const int b_hi = (T.hi - 1) >> 6;
        for (int b = 0; ok && b < b_hi; ++b) ok = entry(b, 0xFFFFFFFFu);
        if (ok) ok = close(b_hi, 0xFFFFFFFFu);
      } else {
        // stage the tile's lists (tokens outside [lo, hi) get none; blocks past
        // a token's own are dropped here, so no row takes a block it cannot see)
        const int L = TQ * a.k;
        for (int e = lane; e < L; e += 32) {
          const int tok = e / a.k;
          const int i = T.i0 + tok;
          S.list[e] = (i >= T.lo && i < T.hi)
                          ? list_block(a.idx + T.g * a.idx_hstride + (long long)i * a.idx_rstride,
                                       e - tok * a.k, i, a.wait.err)
                          : -1;
        }
        __syncwarp();
        // merge: lane j < TQ walks token j's list (entries < 0 skipped); each
        // step takes the smallest head block and the mask of the lists at it
        const int* mine = S.list + lane * a.k;
        int pos = 0;
        auto head = [&]() -> int {
          while (pos < a.k) {
            const int x = mine[pos];
            if (x >= 0) return x;
            ++pos;
          }
          return 0x7FFFFFFF;
        };
        int v = lane < TQ ? head() : 0x7FFFFFFF;
        int pb = -1;
        uint32_t pm = 0;
        for (;;) {
          const int mn = __reduce_min_sync(0xFFFFFFFFu, v);
          if (mn == 0x7FFFFFFF) break;
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, v == mn);
          if (v == mn) {
            ++pos;
            v = head();
          }
          if (pb >= 0 && !(ok = entry(pb, pm))) break;
          pb = mn;
          pm = m;
        }
        if (ok) ok = pb >= 0 ? close(pb, pm) : close(0, 0u);
        __syncwarp();  // the list buffer is rewritten for the next tile
      }
    }
    // never leave a copy in flight: wait (bounded) for the last loads to land
    if (lane == 0) {
      for (uint32_t x = kc > kNK ? kc - kNK : 0; x < kc; ++x)
        (void)mbar_wait(S.k_full + 8 * (x % kNK), (x / kNK) & 1u, a.wait);
      if (tc > 0) (void)mbar_wait(S.qs_full, (uint32_t)((tc - 1) & 1), a.wait);
    }
  } else if (warp == 10) {
    // ---------------------------------------------------------- V loads
    if (lane == 0) {
      tma_prefetch_desc(&tm_v);
      uint32_t vc = 0;
      bool ok = true;
      for (long long w = blockIdx.x; ok && w < n_items; w += gridDim.x) {
        const Tile T = tile_of<TQ>(a, w);
        for (;;) {
          const uint32_t ms = vc % kMetaRing, vs = vc % kNV;
          if (!(ok = mbar_wait(S.meta_full + 8 * ms, (vc / kMetaRing) & 1u, a.wait))) break;
          const int4 bm = S.meta[ms].bm;
          const int last = S.meta[ms].last;
          if (!(ok = mbar_wait(S.v_empty + 8 * vs, ((vc / kNV) & 1u) ^ 1u, a.wait))) break;
          // V of the pair: block b0 at [0, 16 KB) (two halves), block b1 at [16 KB, 32 KB)
          const uint32_t dst = S.vring + vs * kPairBytes, fb = S.v_full + 8 * vs;
          mbar_expect_tx(fb, kPairBytes);
          tma_load_3d(dst, &tm_v, fb, 0, T.g, 64 * bm.x);
          tma_load_3d(dst + kHalf, &tm_v, fb, 64, T.g, 64 * bm.x);
          tma_load_3d(dst + 2 * kHalf, &tm_v, fb, 0, T.g, 64 * bm.z);
          tma_load_3d(dst + 3 * kHalf, &tm_v, fb, 64, T.g, 64 * bm.z);
          ++vc;
          if (last) break;
        }
      }
      for (uint32_t x = vc > kNV ? vc - kNV : 0; x < vc; ++x)
        (void)mbar_wait(S.v_full + 8 * (x % kNV), (x / kNV) & 1u, a.wait);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- QK issuer
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
      uint32_t c = 0;  // union pairs of this CTA so far
      int tc = 0;
      bool ok = true;
      for (long long w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++tc) {
        if (!(ok = mbar_wait(S.q_full, (uint32_t)(tc & 1), a.wait))) break;
        const uint32_t qcol = kColQ + 64u * (uint32_t)(tc & 1);
        for (;;) {
          const uint32_t ks = c % kNK, sb = c & 1u;
          // K landed, and the PV product two pairs back has read this S buffer
          if (!(ok = mbar_wait2(S.k_full + 8 * ks, (c / kNK) & 1u, S.s_free + 8 * sb,
                                ((c >> 1) & 1u) ^ 1u, a.wait)))
            break;
          const int last = S.meta[c % kMetaRing].last;
          tc_fence_after();
          const uint32_t kst = S.kring + ks * kPairBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_ts(tmem + kColS + 128 * sb, tmem + qcol + 8 * kk,
                         desc_kmajor_sw128(kst + (kk >> 2) * (2 * kHalf) + (kk & 3) * 32), id_qk,
                         kk > 0 ? 1u : 0u);
          umma_commit(S.s_full + 8 * sb);
          umma_commit(S.k_empty + 8 * ks);
          ++c;
          if (last) break;
        }
      }
      // never free TMEM under a running MMA: wait (bounded) for all of them
      umma_commit(S.drain_qk);
      (void)mbar_wait(S.drain_qk, 0, a.wait);
    }
  } else if (warp == 11) {
    // ---------------------------------------------------------- PV issuer
    if (lane == 0) {
      constexpr uint32_t id_pv = idesc_bf16_f32(128, 128, false, true);
      uint32_t c = 0;
      int tc = 0;
      bool ok = true;
      for (long long w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++tc) {
        bool first = true;
        for (;;) {
          const uint32_t vs = c % kNV, sb = c & 1u;
          // P of the pair written (its meta was read by the softmax before), V landed
          if (!(ok = mbar_wait2(S.p_full + 8 * sb, (c >> 1) & 1u, S.v_full + 8 * vs,
                                (c / kNV) & 1u, a.wait)))
            break;
          // the tile's first PV overwrites O: the previous tile's O must be read out
          if (first && tc > 0 && !(ok = mbar_wait(S.o_free, (uint32_t)((tc - 1) & 1), a.wait))) break;
          const int last = S.meta[c % kMetaRing].last;
          tc_fence_after();
          const uint32_t vst = S.vring + vs * kPairBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_ts(tmem + kColO, tmem + kColS + 128 * sb + 8 * kk,
                         desc_mnmajor_sw128(vst + (kk >> 2) * (2 * kHalf) + (kk & 3) * 2048, kHalf),
                         id_pv, (first && kk == 0) ? 0u : 1u);
          umma_commit(S.v_empty + 8 * vs);
          umma_commit(S.s_free + 8 * sb);
          first = false;
          ++c;
          if (last) {
            umma_commit(S.o_full);
            break;
          }
        }
      }
      umma_commit(S.drain_pv);
      (void)mbar_wait(S.drain_pv, 0, a.wait);
    }
  } else {
    // ------------------------------------------- softmax / epilogue warps
    // Warp (q4, X) owns TMEM rows rb .. rb+15, rb = 32 q4 + 16 X (one token at
    // G = 16) for whole pairs, through the 16-lane TMEM shapes: thread t holds
    // rows rb + t/4 ("lo") and rb + t/4 + 8 ("hi"), and the four threads of a
    // row hold its columns 8j + 2(t%4) + {0, 1}.  Row maxima and sums are
    // reduced over those four threads with shuffles.
    const int q4 = warp & 3;                 // TMEM lane quarter this warp may access
    const int X = (warp - 2) >> 2;
    const int rb = q4 * 32 + 16 * X;
    const int tt = lane & 3;
    const int r_lo = rb + (lane >> 2), r_hi = r_lo + 8;
    const int tok_lo = r_lo / G, h_lo = r_lo % G, tok_hi = r_hi / G, h_hi = r_hi % G;
    const uint32_t tl = tmem + ((uint32_t)rb << 16);
    const uint32_t tq = tmem + ((uint32_t)(q4 * 32) << 16);  // 32x32b form (Q copy): quarter base
    const float cs = a.scale_log2;
    const bool dense = a.idx == nullptr;  // every block up to the row's own
    uint32_t c = 0;
    bool ok = true;

    // tile t's Q (all 32 lanes of the quarter, warps X == 0) into TMEM buffer t % 2
    auto copy_q = [&](int t) -> bool {
      // only these warps follow the Q tile's barriers: a warp that does not
      // consume a phase must not wait on it
      if (X == 0) {
        if (!mbar_wait(S.qs_full, (uint32_t)(t & 1), a.wait)) return false;
        const int r = q4 * 32 + lane;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t qv[32];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 x = *reinterpret_cast<const uint4*>(S.qtile + half * (kQBytes / 2) + r * 128 +
                                                            ((ch ^ (r & 7)) << 4));
            qv[4 * ch + 0] = x.x;
            qv[4 * ch + 1] = x.y;
            qv[4 * ch + 2] = x.z;
            qv[4 * ch + 3] = x.w;
          }
          tmem_st32(tq + kColQ + 64u * (uint32_t)(t & 1) + 32 * half, qv);
        }
        tmem_st_wait();
        fence_proxy_async_smem();  // generic reads before the next TMA write of the tile
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(S.qs_empty);
          mbar_arrive(S.q_full);
        }
      }
      return true;
    };

    int tc = 0;
    if ((long long)blockIdx.x < n_items) ok = copy_q(0);
    for (long long w = blockIdx.x; ok && w < n_items; w += gridDim.x, ++tc) {
      const Tile T = tile_of<TQ>(a, w);
      const int i_lo = T.i0 + tok_lo, i_hi = T.i0 + tok_hi;
      const bool ok_lo = i_lo >= T.lo && i_lo < T.hi, ok_hi = i_hi >= T.lo && i_hi < T.hi;
      // does a row (token tok at position i) take block b with token mask mk
      auto takes = [&](int b, uint32_t mk, int tok, int i, bool row_ok) -> bool {
        const bool ch = dense ? mk != 0u : ((mk >> (tok & 31)) & 1u) != 0u;
        return row_ok && ch && 64 * b <= i;
      };
      float m_lo = -INFINITY, m_hi = -INFINITY;  // reference maxima (log2 units)
      float l_lo = 0.f, l_hi = 0.f;              // this thread's quarter of the row sums
      bool seen_lo = false, seen_hi = false;     // the row took a block of this tile already
      for (;;) {
        const uint32_t ms = c % kMetaRing, sb = c & 1u;
        if (!(ok = mbar_wait(S.meta_full + 8 * ms, (c / kMetaRing) & 1u, a.wait))) break;
        const int4 bm = S.meta[ms].bm;
        const int last = S.meta[ms].last;
        if (!(ok = mbar_wait(S.s_full + 8 * sb, (c >> 1) & 1u, a.wait))) break;
        tc_fence_after();
        const bool a_lo = takes(bm.x, (uint32_t)bm.y, tok_lo, i_lo, ok_lo);
        const bool a_hi = takes(bm.x, (uint32_t)bm.y, tok_hi, i_hi, ok_hi);
        const bool b_lo = takes(bm.z, (uint32_t)bm.w, tok_lo, i_lo, ok_lo);
        const bool b_hi = takes(bm.z, (uint32_t)bm.w, tok_hi, i_hi, ok_hi);
        const bool anyA = __any_sync(0xFFFFFFFFu, a_lo || a_hi);
        const bool anyB = __any_sync(0xFFFFFFFFu, b_lo || b_hi);
        const uint32_t sc = tl + kColS + 128 * sb;
        uint32_t pk[32];  // P in the 16x128b.x16 layout: [2j] row lo, [2j+1] row hi
        if (anyA || anyB) {
          float va[32], vb[32];
          if (anyA) tmem_ld16x256_x8(sc, va);
          if (anyB) tmem_ld16x256_x8(sc + 64, vb);
          // causal mask (a row's own block) and the rows' maxima over the taken blocks
          float mx_lo = -INFINITY, mx_hi = -INFINITY;
          auto prep = [&](float (&v)[32], int b, bool t_lo, bool t_hi) {
            const int lim_lo = i_lo - 64 * b, lim_hi = i_hi - 64 * b;  // keys k <= lim visible
            if (lim_lo < 63 || lim_hi < 63) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int key = 8 * j + 2 * tt + e;
                  if (key > lim_lo) v[4 * j + e] = -INFINITY;
                  if (key > lim_hi) v[4 * j + 2 + e] = -INFINITY;
                }
            }
            // the 16 values of each row: eight three-operand maxima per row
            float a_lo[4], a_hi[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              a_lo[x] = fmax3(v[8 * x], v[8 * x + 1], v[8 * x + 4]);
              a_hi[x] = fmax3(v[8 * x + 2], v[8 * x + 3], v[8 * x + 6]);
            }
            float x_lo = fmax3(fmax3(a_lo[0], a_lo[1], v[5]), fmax3(a_lo[2], a_lo[3], v[13]),
                               fmax3(v[21], v[29], -INFINITY));
            float x_hi = fmax3(fmax3(a_hi[0], a_hi[1], v[7]), fmax3(a_hi[2], a_hi[3], v[15]),
                               fmax3(v[23], v[31], -INFINITY));
            if (t_lo) mx_lo = fmaxf(mx_lo, x_lo);
            if (t_hi) mx_hi = fmaxf(mx_hi, x_hi);
          };
          if (anyA) prep(va, bm.x, a_lo, a_hi);
          if (anyB) prep(vb, bm.z, b_lo, b_hi);
          mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xFFFFFFFFu, mx_lo, 1));
          mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xFFFFFFFFu, mx_lo, 2));
          mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xFFFFFFFFu, mx_hi, 1));
          mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xFFFFFFFFu, mx_hi, 2));
          mx_lo *= cs;
          mx_hi *= cs;
          // the reference max is raised only when a pair's max exceeds it by more than 8
          const bool r_lo_raise = mx_lo > m_lo + kRescaleSlack;
          const bool r_hi_raise = mx_hi > m_hi + kRescaleSlack;
          const bool resc_lo = r_lo_raise && seen_lo, resc_hi = r_hi_raise && seen_hi;
          const float mn_lo = r_lo_raise ? mx_lo : m_lo, mn_hi = r_hi_raise ? mx_hi : m_hi;
          if (__any_sync(0xFFFFFFFFu, resc_lo || resc_hi)) {
            // O must hold every earlier pair of this tile: wait for the last PV
            const uint32_t pc1 = c - 1;
            if (!(ok = mbar_wait(S.s_free + 8 * (pc1 & 1u), (pc1 >> 1) & 1u, a.wait))) break;
            tc_fence_after();
            const float al_lo = resc_lo ? fast_exp2(m_lo - mn_lo) : 1.f;
            const float al_hi = resc_hi ? fast_exp2(m_hi - mn_hi) : 1.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              float ov[32];
              tmem_ld16x256_x8(tl + kColO + 64 * half, ov);
              uint32_t ow[32];
#pragma unroll
              for (int x = 0; x < 32; ++x) ow[x] = __float_as_uint(ov[x] * ((x & 2) ? al_hi : al_lo));
              tmem_st16x256_x8(tl + kColO + 64 * half, ow);
            }
            tmem_st_wait();
            l_lo *= al_lo;
            l_hi *= al_hi;
          }
          m_lo = mn_lo;
          m_hi = mn_hi;
          // P = 2^(s*cs - m) for taken blocks (exponent -inf, i.e. 0, elsewhere)
          auto expo = [&](const float (&v)[32], bool t_lo, bool t_hi, int j0) {
            const float n_lo = t_lo ? -m_lo : -INFINITY, n_hi = t_hi ? -m_hi : -INFINITY;
            const float2 cc2 = make_float2(cs, cs);
            float2 acc_lo = make_float2(0.f, 0.f), acc_hi = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float2 e_lo = ffma2(make_float2(v[4 * j], v[4 * j + 1]), cc2, make_float2(n_lo, n_lo));
              const float2 e_hi = ffma2(make_float2(v[4 * j + 2], v[4 * j + 3]), cc2, make_float2(n_hi, n_hi));
              float2 p_lo, p_hi;
              if ((j & 3) == 1) {
                p_lo = exp2_cubic2(e_lo);
                p_hi = exp2_cubic2(e_hi);
              } else {
                p_lo = make_float2(fast_exp2(e_lo.x), fast_exp2(e_lo.y));
                p_hi = make_float2(fast_exp2(e_hi.x), fast_exp2(e_hi.y));
              }
              acc_lo = fadd2(acc_lo, p_lo);
              acc_hi = fadd2(acc_hi, p_hi);
              pk[2 * (j0 + j)] = pack_bf16_int(p_lo.x, p_lo.y);
              pk[2 * (j0 + j) + 1] = pack_bf16_int(p_hi.x, p_hi.y);
            }
            l_lo += acc_lo.x + acc_lo.y;
            l_hi += acc_hi.x + acc_hi.y;
          };
          if (anyA) {
            expo(va, a_lo, a_hi, 0);
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) pk[x] = 0u;
          }
          if (anyB) {
            expo(vb, b_lo, b_hi, 8);
          } else {
#pragma unroll
            for (int x = 16; x < 32; ++x) pk[x] = 0u;
          }
          seen_lo = seen_lo || a_lo || b_lo;
          seen_hi = seen_hi || a_hi || b_hi;
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) pk[x] = 0u;
        }
        tmem_st16x128_x16(sc, pk);  // P (bf16 pairs of keys) over the pair's first 64 S columns
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(S.p_full + 8 * sb);
        ++c;
        if (last) break;
      }
      if (!ok) break;
      // the next tile's Q goes in before this tile's epilogue, so its QK products
      // overlap the read-out of O
      if (w + gridDim.x < n_items && !(ok = copy_q(tc + 1))) break;
      // ---- epilogue: O / l and the log-sum-exp of rows lo and hi
      l_lo += __shfl_xor_sync(0xFFFFFFFFu, l_lo, 1);
      l_lo += __shfl_xor_sync(0xFFFFFFFFu, l_lo, 2);
      l_hi += __shfl_xor_sync(0xFFFFFFFFu, l_hi, 1);
      l_hi += __shfl_xor_sync(0xFFFFFFFFu, l_hi, 2);
      if (!(ok = mbar_wait(S.o_full, (uint32_t)(tc & 1), a.wait))) break;
      tc_fence_after();
      const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
      uint16_t* d_lo = a.o + ((size_t)i_lo * a.h_q + T.g * G + h_lo) * 128 + 2 * tt;
      uint16_t* d_hi = a.o + ((size_t)i_hi * a.h_q + T.g * G + h_hi) * 128 + 2 * tt;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float ov[32];
        tmem_ld16x256_x8(tl + kColO + 64 * half, ov);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int d = 64 * half + 8 * j;
          if (ok_lo)
            *reinterpret_cast<uint32_t*>(d_lo + d) = pack_bf16(ov[4 * j] * inv_lo, ov[4 * j + 1] * inv_lo);
          if (ok_hi)
            *reinterpret_cast<uint32_t*>(d_hi + d) =
                pack_bf16(ov[4 * j + 2] * inv_hi, ov[4 * j + 3] * inv_hi);
          if (INFV2_CHECKS)  // debug build: every output finite
            check((!ok_lo || (isfinite(ov[4 * j] * inv_lo) && isfinite(ov[4 * j + 1] * inv_lo))) &&
                      (!ok_hi || (isfinite(ov[4 * j + 2] * inv_hi) && isfinite(ov[4 * j + 3] * inv_hi))),
                  a.wait.err);
        }
      }
      if (tt == 0 && a.lse) {
        if (ok_lo)
          a.lse[(size_t)(T.g * G + h_lo) * a.lse_ld + i_lo] =
              l_lo > 0.f ? (m_lo + __log2f(l_lo)) * kLn2 : -INFINITY;
        if (ok_hi)
          a.lse[(size_t)(T.g * G + h_hi) * a.lse_ld + i_hi] =
              l_hi > 0.f ? (m_hi + __log2f(l_hi)) * kLn2 : -INFINITY;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(S.o_free);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

constexpr int smem_bytes() {
  return (kNK + kNV) * kPairBytes + kQBytes + kTcListCap * 4 + kMetaRing * (int)sizeof(Pair) +
         8 * kBars + 16 + 1024;
}

template <int G>
int launch_tc_g(const TcArgs& a0, const uint16_t* q, const uint16_t* k, const uint16_t* v, int n,
                cudaStream_t st) {
  constexpr int TQ = 128 / G;
  TcArgs a = a0;
  const int tile_first = a.row_lo / TQ;
  a.tile_last = (a.row_hi - 1) / TQ;
  a.n_tiles = a.tile_last - tile_first + 1;
  CUtensorMap tm_q, tm_k, tm_v;
  if (!make_tmap_3d(&tm_q, q, 128, a.h_q, n, 256, (uint64_t)a.h_q * 256, 64, G, TQ) ||
      !make_tmap_3d(&tm_k, k, 128, a.h_kv, n, 256, (uint64_t)a.h_kv * 256, 64, 1, 64) ||
      !make_tmap_3d(&tm_v, v, 128, a.h_kv, n, 256, (uint64_t)a.h_kv * 256, 64, 1, 64))
    return INFV2_ERR_CUDA;
  constexpr int smem = smem_bytes();
  if (!set_smem(attn_tc_kernel<G>, smem)) return INFV2_ERR_CUDA;
  const long long items = (long long)a.h_kv * a.n_tiles;
  const long long slots = sm_count();
  const long long grid = items < slots ? items : slots;
  attn_tc_kernel<G><<<(unsigned)grid, kThreads, smem, st>>>(tm_q, tm_k, tm_v, a);
  return launch_status(cudaGetLastError());
}

}  // namespace

bool attn_tc_supports(const infv2_params* p, bool dense) {
  const int G = p->h_q / p->h_kv;
  if (dense) return true;
  return G >= 4 && (128 / G) * p->k <= kTcListCap;
}

int launch_attn_tc(const infv2_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const int* idx, long long idx_hstride, int n, int r0, int r1, uint16_t* o,
                   float* lse, long long lse_ld, cudaStream_t st) {
  if (r0 < 0 || r1 > n || r0 > r1) return INFV2_ERR_INVALID_ARG;
  if (r1 == r0) return INFV2_OK;
  if (!attn_tc_supports(p, idx == nullptr)) return INFV2_ERR_UNSUPPORTED;
  TcArgs a{};
  a.row_lo = r0;
  a.row_hi = r1;
  a.h_q = p->h_q;
  a.h_kv = p->h_kv;
  a.k = p->k;
  a.idx = idx;
  a.idx_hstride = idx_hstride;
  a.idx_rstride = p->k;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.o = o;
  a.lse = lse;
  a.lse_ld = lse_ld;
  a.wait = wait_ctx();
  switch (p->h_q / p->h_kv) {
    case 1: return launch_tc_g<1>(a, q, k, v, n, st);
    case 2: return launch_tc_g<2>(a, q, k, v, n, st);
    case 4: return launch_tc_g<4>(a, q, k, v, n, st);
    case 8: return launch_tc_g<8>(a, q, k, v, n, st);
    case 16: return launch_tc_g<16>(a, q, k, v, n, st);
    default: return INFV2_ERR_UNSUPPORTED;
  }
}

}  // namespace infv2
