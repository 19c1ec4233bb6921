// Stage 2: fused two-pass block scores (S^C1 softmax + GQA group sum).
//
// "InfLLM-V2" paper notes, key design 4, and the arXiv summary, section 3
// ("Efficient Implementation"): S^C1 = softmax(Q K^C1^T) is never written to
// memory; the head-group sum is taken on chip.  Because the group sum and the
// online softmax do not commute, pass 1 computes each (token, head) row's
// log-sum-exp and pass 2 recomputes the logits, normalises and sums over the
// group; only S^shared (h_q/G values per token and kernel) reaches HBM.
//
// B200 design.  One CTA owns a tile of 128 (token, head) rows: TQ = 128/G
// consecutive tokens times the G heads of kv head g (all heads of a group
// share K^C1).  The Q tile (128 x 128 bf16) is loaded once by TMA and serves
// both passes; K^C1 tiles of 128 kernels stream through a 4-stage TMA ring.
//   pass 1: D[row, kernel]   = Q_tile . K^C1_tile^T   (tcgen05, M=128, N=128)
//           one TMEM lane per row -> the row's running max / sum stay in one
//           thread; lse2 (log2 domain) goes to shared memory.
//   pass 2: D[kernel, row]   = K^C1_tile . Q_tile^T   (same operands swapped)
//           one TMEM lane per kernel -> the G-head sum of exp2(z - lse2) for a
//           token is a sum over G adjacent columns inside one thread, and the
//           128 lanes store 128 consecutive floats of S^shared per token.
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer (and TMEM owner), warps
// 2-17 softmax / epilogue: four warpgroups, each owning 32 of a tile's 128
// columns (pass-1 row statistics are merged through shared memory).  A
// quarter of the exponentials run on the FMA pipe (exp2_fma) so that the MUFU
// unit is not the only pipe doing the softmax.
// Accumulators rotate through kAcc TMEM buffers of 128 columns so the next
// tiles' MMAs overlap the current tile's epilogue.
#include "common.cuh"
#include "internal.cuh"

namespace infv2 {
namespace {

constexpr int kStages = 4;
constexpr int kAcc = 2;                    // TMEM accumulators of 128 columns
constexpr int kTileBytes = 128 * 128 * 2;  // 128 rows x 128 bf16
constexpr int kEpiWarps = 16;              // four epilogue warpgroups
constexpr int kColGroups = kEpiWarps / 4;  // column groups of 128 / kColGroups columns
constexpr int kCols = 128 / kColGroups;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr float kLn2 = 0.6931471805599453f;

struct ScoreArgs {
  int q_begin, q_len, n_tiles;   // rows computed by this launch
  int o_begin, o_len;            // row range of the output buffers (row i at i - o_begin)
  int approx;                    // 1: pass 1 over the coarse kernels K^C2 (LSE approximation)
  float scale_log2;     // scale * log2(e)
  int ld;
  float* s_shared;      // [h_kv, o_len, ld]      (unpooled form)
  float* s_cmp;         // [h_kv, o_len, ld_cmp]  (pooled form: block scores)
  int ld_cmp;
  float* score_lse;     // [h_q, o_len] or null
  WaitCtx wait;
};

struct ScoreSmem {
  uint32_t q, k;        // shared addresses of the Q tile and the K^C1 ring
  uint32_t q_full, kv_full, kv_empty, acc_full, acc_empty, lse_ready;  // barriers (8 B each)
};

// POOL: instead of S^shared, write the block scores S^cmp[b] = max of S^shared
// over the kernels 4b-1 .. 4b+3 (those intersecting block b).  In pass 2 a
// TMEM lane owns one kernel, so kernels 4b .. 4b+3 are four aligned lanes of a
// warp (shuffle max) and kernel 4b-1 is the previous lane; the first lane of a
// warp takes it from the previous warp quarter (or the previous tile's last
// quarter) through shared memory: the four warps of a column group publish
// their last lane per tile and meet on a bounded mbarrier.  Tile t uses
// exchange slot t%3, read at tiles t and t+1; it is rewritten at tile t+3 only
// after the writer has passed the barrier of tile t+2, which every warp
// reaches after its reads at tile t+1.
template <int G, bool POOL>
__global__ void __launch_bounds__(kThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_k2, ScoreArgs a) {
  constexpr int TQ = 128 / G;
  constexpr int TPG = kCols / G > 0 ? kCols / G : 1;  // tokens per column group
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* s_lse2 = reinterpret_cast<float*>(base + kTileBytes * (1 + kStages));
  float* s_part = s_lse2 + 128;  // [column group][128 rows][max, sum]
  float* s_xch = s_part + kColGroups * 128 * 2;        // [3][kColGroups][4 quarters][TPG]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_xch + 3 * kColGroups * 4 * TPG + 2);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 + 2 * kStages + 2 * kAcc + kColGroups);
  ScoreSmem S;
  S.q = smem_u32(base);
  S.k = S.q + kTileBytes;
  S.q_full = smem_u32(bars);
  S.kv_full = S.q_full + 8;
  S.kv_empty = S.kv_full + 8 * kStages;
  S.acc_full = S.kv_empty + 8 * kStages;
  S.acc_empty = S.acc_full + 8 * kAcc;
  S.lse_ready = S.acc_empty + 8 * kAcc;
  const uint32_t cg_bar0 = S.lse_ready + 8;  // POOL: one barrier per column group

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int tile = a.n_tiles - 1 - (int)blockIdx.x;  // longest rows first
  const int i0 = a.q_begin + tile * TQ;
  const int i_last = min(i0 + TQ, a.q_begin + a.q_len) - 1;
  const int nv_max = visible_kernels(i_last, 32, 16);
  const int n_kt = (nv_max + 127) >> 7;  // pass-2 tiles (stage-1 kernels)
  // pass-1 tiles: the same kernels, or the coarse kernels (128 tokens at stride
  // 64) of the LSE approximation; the host sends only rows i >= 127 here
  const int n_kt1 = a.approx ? (visible_kernels(i_last, 128, 64) + 127) >> 7 : n_kt;

  if (n_kt == 0) {  // no row of this tile sees a complete kernel
    if (a.score_lse && threadIdx.x < 128) {
      const int i = i0 + (int)threadIdx.x / G;
      if (i <= i_last)
        a.score_lse[(size_t)(g * G + threadIdx.x % G) * a.o_len + (i - a.o_begin)] = -INFINITY;
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(S.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(S.kv_full + 8 * s, 1);
      mbar_init(S.kv_empty + 8 * s, 1);
    }
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(S.acc_full + 8 * b, 1);
      mbar_init(S.acc_empty + 8 * b, kEpiWarps);
    }
    mbar_init(S.lse_ready, kEpiWarps);
    if (POOL)
      for (int x = 0; x < kColGroups; ++x) mbar_init(cg_bar0 + 8 * x, 4);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), 128 * kAcc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const int total_it = n_kt1 + n_kt;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      if (a.approx) tma_prefetch_desc(&tm_k2);
      mbar_expect_tx(S.q_full, kTileBytes);
      tma_load_3d(S.q, &tm_q, S.q_full, 0, g * G, i0);
      tma_load_3d(S.q + kTileBytes / 2, &tm_q, S.q_full, 64, g * G, i0);
      int issued = 0;
      for (int it = 0; it < total_it; ++it) {
        const int s = it % kStages;
        const int jt = it < n_kt1 ? it : it - n_kt1;
        const CUtensorMap* tm = (it < n_kt1 && a.approx) ? &tm_k2 : &tm_k;
        if (!mbar_wait(S.kv_empty + 8 * s, ((it / kStages) & 1) ^ 1, a.wait)) break;
        const uint32_t dst = S.k + s * kTileBytes;
        mbar_expect_tx(S.kv_full + 8 * s, kTileBytes);
        tma_load_3d(dst, tm, S.kv_full + 8 * s, 0, g, jt * 128);
        tma_load_3d(dst + kTileBytes / 2, tm, S.kv_full + 8 * s, 64, g, jt * 128);
        issued = it + 1;
      }
      // never leave a copy in flight: wait (bounded) for the last loads to land
      (void)mbar_wait(S.q_full, 0, a.wait);
      for (int it = issued > kStages ? issued - kStages : 0; it < issued; ++it)
        (void)mbar_wait(S.kv_full + 8 * (it % kStages), (it / kStages) & 1, a.wait);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      bool ok = mbar_wait(S.q_full, 0, a.wait);
      int issued = 0;
      for (int it = 0; ok && it < total_it; ++it) {
        const int s = it % kStages;
        const int b = it % kAcc;
        if (!mbar_wait(S.kv_full + 8 * s, (it / kStages) & 1, a.wait)) break;
        if (!mbar_wait(S.acc_empty + 8 * b, ((it / kAcc) & 1) ^ 1, a.wait)) break;
        tc_fence_after();
        const uint32_t ks = S.k + s * kTileBytes;
        const uint32_t a_base = it < n_kt1 ? S.q : ks;  // pass 1: rows = Q; pass 2: rows = K^C1
        const uint32_t b_base = it < n_kt1 ? ks : S.q;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
          umma_bf16_ss(tmem + b * 128, desc_kmajor_sw128(a_base + off),
                       desc_kmajor_sw128(b_base + off), idesc, kk > 0);
        }
        umma_commit(S.kv_empty + 8 * s);
        umma_commit(S.acc_full + 8 * b);
        issued = it + 1;
      }
      // never free TMEM under a running MMA: wait (bounded) for the last commits
      for (int it = issued > kAcc ? issued - kAcc : 0; it < issued; ++it)
        (void)mbar_wait(S.acc_full + 8 * (it % kAcc), (it / kAcc) & 1, a.wait);
    }
  } else {
    // ---------------------------------------------------------- epilogue warps
    const int quarter = warp & 3;        // TMEM lanes 32*quarter .. +31
    const int cg = (warp - 2) >> 2;      // columns kCols*cg .. +kCols-1 of every tile
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + cg * kCols;
    const int tq_r = r / G;
    const int i_r = i0 + tq_r;
    // pass-1 kernel count of row r (coarse kernels in the approximation)
    const int nv_r = i_r > i_last ? 0 : (a.approx ? visible_kernels(i_r, 128, 64)
                                                  : visible_kernels(i_r, 32, 16));
    const float c = a.scale_log2;
    float vmax = -INFINITY, l = 0.f;
    float* out_g = a.s_shared + (size_t)g * a.o_len * a.ld;
    // POOL: per token of this column group, the S^cmp row and the number of
    // blocks it holds (i/B; 0 for rows past the tile's end)
    float* cmp_row[TPG];
    int cmp_lim[TPG];
    int slot = 0, slot_prev = 2;  // POOL: exchange slots of this tile and the previous one
    if constexpr (POOL) {
#pragma unroll
      for (int t = 0; t < TPG; ++t) {
        const int i = i0 + cg * TPG + t;
        const bool in = i <= i_last;
        cmp_row[t] = a.s_cmp + ((size_t)g * a.o_len + (in ? i - a.o_begin : 0)) * a.ld_cmp;
        cmp_lim[t] = in ? (i >> 6) : 0;
      }
    }
    for (int it = 0; it < total_it; ++it) {
      const int b = it % kAcc;
      if (!mbar_wait(S.acc_full + 8 * b, (it / kAcc) & 1, a.wait)) break;
      tc_fence_after();
      float v[32];
      tmem_ld32(lane_base + b * 128, v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(S.acc_empty + 8 * b);  // TMEM buffer free again
      if (it < n_kt1) {
        // pass 1: row r, kernels it*128 + kCols*cg .. +31
        const int jb = it * 128 + cg * kCols;
        if (jb + 32 > nv_r) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (jb + e >= nv_r) v[e] = -INFINITY;
        }
        // the tile max of the row's 32 values: 16 three-operand maxima
        float t3[11];
#pragma unroll
        for (int x = 0; x < 10; ++x) t3[x] = fmax3(v[3 * x], v[3 * x + 1], v[3 * x + 2]);
        t3[10] = fmaxf(v[30], v[31]);
        const float u0 = fmax3(t3[0], t3[1], t3[2]), u1 = fmax3(t3[3], t3[4], t3[5]);
        const float u2 = fmax3(t3[6], t3[7], t3[8]), u3 = fmaxf(t3[9], t3[10]);
        const float cm = fmaxf(fmax3(u0, u1, u2), u3);
        if (cm > vmax) {
          l *= fast_exp2((vmax - cm) * c);
          vmax = cm;
        }
        if (vmax != -INFINITY) {
          // packed pairs: exponent arguments and partial sums two at a time;
          // a quarter of the exponentials on the FMA pipe
          const float mneg = -vmax * c;
          const float2 cc = make_float2(c, c), mm = make_float2(mneg, mneg);
          float2 acc01 = make_float2(0.f, 0.f), acc23 = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float2 x01 = ffma2(make_float2(v[e], v[e + 1]), cc, mm);
            const float2 x23 = ffma2(make_float2(v[e + 2], v[e + 3]), cc, mm);
            acc01 = fadd2(acc01, make_float2(fast_exp2(x01.x), fast_exp2(x01.y)));
            acc23 = fadd2(acc23, (e & 4) ? exp2_fma2(x23)
                                         : make_float2(fast_exp2(x23.x), fast_exp2(x23.y)));
          }
          l += (acc01.x + acc01.y) + (acc23.x + acc23.y);
        }
        if (it == n_kt1 - 1) {
          // merge the column groups' statistics of row r
          s_part[(cg * 128 + r) * 2 + 0] = vmax;
          s_part[(cg * 128 + r) * 2 + 1] = l;
          __syncwarp();
          if (lane == 0) mbar_arrive(S.lse_ready);
          if (!mbar_wait(S.lse_ready, 0, a.wait)) break;
          if (cg == 0) {
            float M = -INFINITY;
#pragma unroll
            for (int x = 0; x < kColGroups; ++x) M = fmaxf(M, s_part[(x * 128 + r) * 2]);
            float L = 0.f;
#pragma unroll
            for (int x = 0; x < kColGroups; ++x) {
              const float mx = s_part[(x * 128 + r) * 2];
              if (mx != -INFINITY) L += s_part[(x * 128 + r) * 2 + 1] * fast_exp2((mx - M) * c);
            }
            // the approximation adds log2(s_C2 / s_C1) = 2: each coarse kernel
            // stands for four stage-1 kernels
            const float lse2 = L > 0.f ? M * c + __log2f(L) + (a.approx ? 2.0f : 0.0f) : -INFINITY;
            s_lse2[r] = -lse2;  // stored negated: pass 2 adds it
            if (a.score_lse && i_r <= i_last)
              a.score_lse[(size_t)(g * G + r % G) * a.o_len + (i_r - a.o_begin)] = lse2 * kLn2;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(S.lse_ready);
          if (!mbar_wait(S.lse_ready, 1, a.wait)) break;  // all 128 lse2 in smem
        }
      } else {
        // pass 2: kernel j = (it - n_kt1)*128 + r; this group's columns = tokens
        const int jt = it - n_kt1;
        const int j = jt * 128 + r;
        static_assert(G <= kCols, "a token's heads must fit in one column group");
        const float4* lse4 = reinterpret_cast<const float4*>(s_lse2 + cg * kCols);
        float pv[TPG];  // POOL: this kernel's S^shared per token (-inf if not visible)
#pragma unroll
        for (int t = 0; t < TPG; ++t) {
          const int tq = cg * TPG + t;
          const int i = i0 + tq;
          float ssum;
          if constexpr (G >= 4) {
            // packed pairs; heads 4*h4 .. 4*h4+3 of the token; pairs 3 and 7
            // of the token's G/2 head pairs (a quarter of G = 8, 16) take the
            // FMA-pipe exponential
            const float2 cc = make_float2(c, c);
            float2 acc01 = make_float2(0.f, 0.f), acc23 = make_float2(0.f, 0.f);
#pragma unroll
            for (int h4 = 0; h4 < G / 4; ++h4) {
              const float4 L4 = lse4[(t * G) / 4 + h4];  // broadcast read of -lse2
              const float2 x01 = ffma2(make_float2(v[t * G + 4 * h4 + 0], v[t * G + 4 * h4 + 1]), cc,
                                       make_float2(L4.x, L4.y));
              const float2 x23 = ffma2(make_float2(v[t * G + 4 * h4 + 2], v[t * G + 4 * h4 + 3]), cc,
                                       make_float2(L4.z, L4.w));
              acc01 = fadd2(acc01, make_float2(fast_exp2(x01.x), fast_exp2(x01.y)));
              acc23 = fadd2(acc23, (h4 & 1) ? exp2_fma2(x23)
                                            : make_float2(fast_exp2(x23.x), fast_exp2(x23.y)));
            }
            ssum = (acc01.x + acc01.y) + (acc23.x + acc23.y);
          } else {
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
              ps[hh] += fast_exp2(fmaf(v[t * G + hh], c, s_lse2[tq * G + hh]));
            ssum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
          }
          const bool vis = i <= i_last && j < visible_kernels(i, 32, 16);
          if constexpr (POOL) {
            pv[t] = vis ? ssum : -INFINITY;
          } else {
            if (vis) out_g[(size_t)(i - a.o_begin) * a.ld + j] = ssum;
          }
        }
        if constexpr (POOL) {
          float* xch = s_xch + ((slot * kColGroups + cg) * 4) * TPG;
          if (lane == 31)
#pragma unroll
            for (int t = 0; t < TPG; ++t) xch[quarter * TPG + t] = pv[t];
          __syncwarp();
          if (lane == 0) mbar_arrive(cg_bar0 + 8 * cg);
          if (!mbar_wait(cg_bar0 + 8 * cg, (uint32_t)(jt & 1), a.wait)) break;
          // kernel 4b-1 for lane 0: the previous quarter's last lane, or the
          // previous tile's last quarter
          const float* prv = quarter > 0 ? xch + (quarter - 1) * TPG
                                         : s_xch + ((slot_prev * kColGroups + cg) * 4 + 3) * TPG;
          slot_prev = slot;
          slot = slot == 2 ? 0 : slot + 1;
          const int b = j >> 2;
#pragma unroll
          for (int t = 0; t < TPG; ++t) {
            float prev = __shfl_up_sync(0xFFFFFFFFu, pv[t], 1);
            if (lane == 0) prev = (quarter > 0 || jt > 0) ? prv[t] : -INFINITY;
            float m4 = fmaxf(pv[t], __shfl_xor_sync(0xFFFFFFFFu, pv[t], 1));
            m4 = fmaxf(m4, __shfl_xor_sync(0xFFFFFFFFu, m4, 2));  // kernels 4b .. 4b+3
            if ((lane & 3) == 0 && b < cmp_lim[t]) cmp_row[t][b] = fmaxf(m4, prev);
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128 * kAcc);
  }
}

struct ScoreLaunch {
  const uint16_t *q, *kc1, *kc2;  // kc2: coarse kernels (approx only)
  int n, h_q, h_kv;
  int q_begin, q_len;             // rows to compute
  int o_begin, o_len;             // row range of the output buffers
  float scale;
  float* out;                     // S^shared (or S^cmp when pooled)
  int ld;
  float* score_lse;
  int approx;
};

template <int G, bool POOL>
int launch_score_g(const ScoreLaunch& L, cudaStream_t st) {
  constexpr int TQ = 128 / G;
  const int nc = L.n >= 32 ? (L.n - 32) / 16 + 1 : 0;
  CUtensorMap tm_q, tm_k, tm_k2;
  if (!make_tmap_3d(&tm_q, L.q, 128, L.h_q, L.n, 256, (uint64_t)L.h_q * 256, 64, G, TQ))
    return INFV2_ERR_CUDA;
  // K^C1 map; an empty K^C1 (nc == 0) still needs a valid map, one row is enough
  if (!make_tmap_3d(&tm_k, L.kc1, 128, L.h_kv, nc > 0 ? nc : 1, 256, (uint64_t)L.h_kv * 256, 64, 1,
                    128))
    return INFV2_ERR_CUDA;
  if (L.approx) {
    const int nc2 = num_coarse_kernels(L.n);
    if (!make_tmap_3d(&tm_k2, L.kc2, 128, L.h_kv, nc2 > 0 ? nc2 : 1, 256, (uint64_t)L.h_kv * 256,
                      64, 1, 128))
      return INFV2_ERR_CUDA;
  } else {
    tm_k2 = tm_k;  // unused
  }
  constexpr int TPG = kCols / G > 0 ? kCols / G : 1;
  const int smem = kTileBytes * (1 + kStages) + 128 * 4 + kColGroups * 128 * 2 * 4 +
                   (3 * kColGroups * 4 * TPG + 2) * 4 +
                   8 * (2 + 2 * kStages + 2 * kAcc + kColGroups) + 16 + 1024;
  if (!set_smem(score_kernel<G, POOL>, smem)) return INFV2_ERR_CUDA;
  ScoreArgs a;
  a.q_begin = L.q_begin;
  a.q_len = L.q_len;
  a.n_tiles = (L.q_len + TQ - 1) / TQ;
  a.o_begin = L.o_begin;
  a.o_len = L.o_len;
  a.approx = L.approx;
  a.scale_log2 = L.scale * 1.4426950408889634f;
  a.ld = L.ld;
  a.s_shared = POOL ? nullptr : L.out;
  a.s_cmp = POOL ? L.out : nullptr;
  a.ld_cmp = L.ld;
  a.score_lse = L.score_lse;
  a.wait = wait_ctx();
  dim3 grid(a.n_tiles, L.h_kv);
  score_kernel<G, POOL><<<grid, kThreads, smem, st>>>(tm_q, tm_k, tm_k2, a);
  return launch_status(cudaGetLastError());
}

template <bool POOL>
int launch_scores(const infv2_params* p, const ScoreLaunch& L, cudaStream_t st) {
  if (L.q_len <= 0) return INFV2_OK;
  switch (p->h_q / p->h_kv) {
    case 1: return launch_score_g<1, POOL>(L, st);
    case 2: return launch_score_g<2, POOL>(L, st);
    case 4: return launch_score_g<4, POOL>(L, st);
    case 8: return launch_score_g<8, POOL>(L, st);
    case 16: return launch_score_g<16, POOL>(L, st);
    default: return INFV2_ERR_UNSUPPORTED;
  }
}

ScoreLaunch make_launch(const infv2_params* p, const uint16_t* q, const uint16_t* kc1, int n,
                        int q_begin, int q_len, float* out, int ld, float* score_lse) {
  ScoreLaunch L;
  L.q = q;
  L.kc1 = kc1;
  L.kc2 = nullptr;
  L.n = n;
  L.h_q = p->h_q;
  L.h_kv = p->h_kv;
  L.q_begin = L.o_begin = q_begin;
  L.q_len = L.o_len = q_len;
  L.scale = p->scale;
  L.out = out;
  L.ld = ld;
  L.score_lse = score_lse;
  L.approx = 0;
  return L;
}

}  // namespace

int launch_block_scores(const infv2_params* p, const uint16_t* q, const uint16_t* kc1, int n,
                        int q_begin, int q_len, float* s_shared, int ld, float* score_lse,
                        cudaStream_t st) {
  return launch_scores<false>(p, make_launch(p, q, kc1, n, q_begin, q_len, s_shared, ld, score_lse),
                              st);
}

int launch_block_scores_approx(const infv2_params* p, const uint16_t* q, const uint16_t* kc1,
                               const uint16_t* kc2, int n, int q_begin, int q_len,
                               float* s_shared, int ld, float* score_lse, cudaStream_t st) {
  // rows that see no coarse kernel (i < 4*l_c1 - 1 = 127) keep the exact LSE
  constexpr int kFirstCoarse = 127;
  const int end = q_begin + q_len;
  ScoreLaunch L = make_launch(p, q, kc1, n, q_begin, q_len, s_shared, ld, score_lse);
  if (q_begin < kFirstCoarse) {
    L.q_len = (end < kFirstCoarse ? end : kFirstCoarse) - q_begin;
    const int st1 = launch_scores<false>(p, L, st);
    if (st1 != INFV2_OK) return st1;
  }
  if (end > kFirstCoarse) {
    L.q_begin = q_begin > kFirstCoarse ? q_begin : kFirstCoarse;
    L.q_len = end - L.q_begin;
    L.kc2 = kc2;
    L.approx = 1;
    return launch_scores<false>(p, L, st);
  }
  return INFV2_OK;
}

int launch_block_scores_pooled(const infv2_params* p, const uint16_t* q, const uint16_t* kc1,
                               int n, int q_begin, int q_len, float* s_cmp, int ld_cmp,
                               cudaStream_t st) {
  return launch_scores<true>(p, make_launch(p, q, kc1, n, q_begin, q_len, s_cmp, ld_cmp, nullptr),
                             st);
}

}  // namespace infv2

using namespace infv2;

extern "C" int infv2_block_scores(const infv2_params* p, const void* q, const void* kc1, int n,
                                  int q_begin, int q_len, float* s_shared, int ld,
                                  float* score_lse, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0 || q_begin < 0 || q_len < 0 || q_begin + q_len > n) return INFV2_ERR_INVALID_ARG;
  if (q_len == 0) return INFV2_OK;
  if (!q || !s_shared) return INFV2_ERR_INVALID_ARG;
  const int nc = infv2_num_kernels(p, n);
  if (nc > 0 && !kc1) return INFV2_ERR_INVALID_ARG;
  if (ld < nc || ld % 4 != 0) return INFV2_ERR_INVALID_ARG;
  if (nc == 0 && score_lse == nullptr) return INFV2_OK;
  const void* kc1_map = kc1 ? kc1 : q;  // any valid address when no kernel exists
  return launch_block_scores(p, static_cast<const uint16_t*>(q),
                             static_cast<const uint16_t*>(kc1_map), n, q_begin, q_len, s_shared,
                             ld, score_lse, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int infv2_block_scores_pooled(const infv2_params* p, const void* q, const void* kc1,
                                         int n, int q_begin, int q_len, float* s_cmp, int ld_cmp,
                                         infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0 || q_begin < 0 || q_len < 0 || q_begin + q_len > n) return INFV2_ERR_INVALID_ARG;
  if (q_len == 0) return INFV2_OK;
  if (!q || !s_cmp) return INFV2_ERR_INVALID_ARG;
  const int nc = infv2_num_kernels(p, n);
  if (nc > 0 && !kc1) return INFV2_ERR_INVALID_ARG;
  if (ld_cmp < (n + p->B - 1) / p->B || ld_cmp % 4 != 0) return INFV2_ERR_INVALID_ARG;
  if (nc == 0) return INFV2_OK;  // no block has a visible kernel
  return launch_block_scores_pooled(p, static_cast<const uint16_t*>(q),
                                    static_cast<const uint16_t*>(kc1), n, q_begin, q_len, s_cmp,
                                    ld_cmp, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int infv2_block_scores_approx(const infv2_params* p, const void* q, const void* kc1,
                                         const void* kc2, int n, int q_begin, int q_len,
                                         float* s_shared, int ld, float* score_lse,
                                         infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0 || q_begin < 0 || q_len < 0 || q_begin + q_len > n) return INFV2_ERR_INVALID_ARG;
  if (q_len == 0) return INFV2_OK;
  if (!q || !s_shared) return INFV2_ERR_INVALID_ARG;
  const int nc = infv2_num_kernels(p, n);
  if (nc > 0 && !kc1) return INFV2_ERR_INVALID_ARG;
  if (num_coarse_kernels(n) > 0 && q_begin + q_len > 127 && !kc2) return INFV2_ERR_INVALID_ARG;
  if (ld < nc || ld % 4 != 0) return INFV2_ERR_INVALID_ARG;
  if (nc == 0 && score_lse == nullptr) return INFV2_OK;
  const void* kc1_map = kc1 ? kc1 : q;  // any valid address when no kernel exists
  return launch_block_scores_approx(p, static_cast<const uint16_t*>(q),
                                    static_cast<const uint16_t*>(kc1_map),
                                    static_cast<const uint16_t*>(kc2), n, q_begin, q_len, s_shared,
                                    ld, score_lse, reinterpret_cast<cudaStream_t>(stream));
}
