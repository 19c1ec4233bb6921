// Stages 3-4 for one (query, kv head) row, executed by one warp: max pooling
// of S^shared into block scores and the top-k block selection.
//
// "InfLLM-V2" paper notes, key designs 2-3, and the MiniCPM4 "InfLLM v2" blog
// (semantic kernels, top-k sharing):
//   S^cmp[b] = max over the visible kernels j that intersect block b (with
//              B=64, l_C1=32, s_C1=16 these are j = 4b-1 .. 4b+3);
//   I(i)     = every block 0..i/B when there are at most k of them; otherwise
//              the init and local blocks (treated as +inf) plus the highest
//              S^cmp blocks up to k in total, equal scores to the lower block.
// The selection is an exact radix select on order-preserving 32-bit keys: up to
// four 8-bit digit passes with a per-warp shared-memory histogram narrow down
// the prefix T of the k-th largest key; blocks whose key prefix is above T are
// taken, and the blocks with prefix T in ascending block order until k are
// chosen.  The passes stop early once the bucket of the k-th key holds exactly
// the number of blocks still needed (the whole bucket is then taken, which is
// what the remaining passes would have found).
#pragma once
#include "common.cuh"

namespace infv2 {

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr uint32_t kForcedKey = 0xFFFFFFFFu;  // above every finite score and +inf
constexpr int kPoolLoads = 8;  // float4 loads in flight per lane while pooling a row

// Exact top-k of keys[0 .. n_cand) (per-warp shared memory) by one warp:
// ascending block indices written to out[0..k), padded with -1.  The n_forced
// keys equal to kForcedKey are always taken; the other keys lie in [kmin, kmax]
// and compete for the remaining k - n_forced places.  They share every bit
// above the highest bit in which kmin and kmax differ, so the digit passes
// start there (on these scores the top byte is nearly constant, and a pass
// over it would only pile every key into one bucket); each pass takes up to 8
// bits.
// The debug build (INFV2_CHECKS) checks that exactly k blocks come out (the
// radix select's invariant) and writes none past k.
__device__ __forceinline__ void topk_warp(const uint32_t* keys, int n_cand, int k, uint32_t* hist,
                                          int* __restrict__ out, int* err, uint32_t kmin,
                                          uint32_t kmax, int n_forced) {
  const int lane = (int)lane_id();
  // ---- radix select of the remaining-th largest non-forced key
  int remaining = k - n_forced;
  const uint32_t diff = kmin ^ kmax;
  int top = diff ? 32 - __clz(diff) : 0;  // bits >= top are common to every competing key
  uint32_t pmask = top >= 32 ? 0u : ~((1u << top) - 1u);
  uint32_t prefix = kmin & pmask;
  if (remaining <= 0) {  // only the forced blocks: no competing key can pass T
    top = 0;
    pmask = 0xFFFFFFFFu;
    prefix = 0xFFFFFFFFu;
  }
#pragma unroll 1
  while (top > 0) {
    const int shift = max(top - 8, 0);
    const uint32_t dm = (1u << (top - shift)) - 1u;
    for (int x = lane; x < 256; x += 32) hist[x] = 0;
    __syncwarp();
    for (int b = lane; b < n_cand; b += 32) {
      const uint32_t key = keys[b];
      if (key != kForcedKey && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dm], 1u);
    }
    __syncwarp();
    // lane L owns digits 255-8L .. 248-8L (lane 0 the largest)
    uint32_t cnt[8];
    uint32_t local = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      cnt[e] = hist[255 - 8 * lane - e];
      local += cnt[e];
    }
    uint32_t incl = local;  // inclusive scan over lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += t;
    }
    const uint32_t before = incl - local;
    const bool mine = before < (uint32_t)remaining && (uint32_t)remaining <= incl;
    uint32_t digit = 0, above = 0, dcnt = 0;
    if (mine) {
      uint32_t run = before;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (run + cnt[e] >= (uint32_t)remaining) {
          digit = 255u - 8u * lane - e;
          above = run;
          dcnt = cnt[e];
          break;
        }
        run += cnt[e];
      }
    }
    const uint32_t who = __ballot_sync(0xFFFFFFFFu, mine);
    const int src = __ffs(who) - 1;
    digit = __shfl_sync(0xFFFFFFFFu, digit, src);
    above = __shfl_sync(0xFFFFFFFFu, above, src);
    dcnt = __shfl_sync(0xFFFFFFFFu, dcnt, src);
    prefix |= digit << shift;
    pmask |= dm << shift;
    remaining -= (int)above;
    top = shift;
    __syncwarp();
    if (dcnt == (uint32_t)remaining) break;  // the whole bucket is taken
  }
  // ---- emit ascending: forced blocks and prefixes above T, then prefix T in
  // block order while needed
  const uint32_t T = prefix;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int eq_seen = 0, written = 0;
  for (int base = 0; base < n_cand; base += 32) {
    const int b = base + lane;
    const uint32_t key = b < n_cand ? keys[b] : 0u;
    const bool forced = b < n_cand && key == kForcedKey;
    const uint32_t m = key & pmask;
    const bool eq = b < n_cand && !forced && m == T;
    const uint32_t eqb = __ballot_sync(0xFFFFFFFFu, eq);
    const bool sel = forced || (b < n_cand && m > T) ||
                     (eq && eq_seen + __popc(eqb & lt_mask) < remaining);
    eq_seen += __popc(eqb);
    const uint32_t selb = __ballot_sync(0xFFFFFFFFu, sel);
    const int at = written + __popc(selb & lt_mask);
    if (sel && (!INFV2_CHECKS || at < k)) out[at] = b;
    written += __popc(selb);
  }
  check(written == k, err);
  for (int x = written + lane; x < k; x += 32) out[x] = -1;
  __syncwarp();
}

// Select for one row.  `row` holds S^shared[j] for j < nv (entries at
// j >= nv may be garbage and are never used; reads stay below 4*(bi+1)).
// `keys` is per-warp shared scratch of >= bi+1 words, `hist` 256 words.
// Writes k indices (ascending, -1 padded) to `out`.
__device__ __forceinline__ void select_row_warp(const float* __restrict__ row, int nv, int i,
                                                int n_init, int n_local, int k, uint32_t* keys,
                                                uint32_t* hist, int* __restrict__ out, int* err) {
  const int lane = (int)lane_id();
  const int bi = i >> 6;  // own block (B = 64)
  const int n_cand = bi + 1;
  if (n_cand <= k) {  // dense: every visible block
    for (int b = lane; b < k; b += 32) out[b] = b < n_cand ? b : -1;
    return;
  }
  // ---- max pooling into order keys (forced blocks get the top key);
  // kPoolLoads 512-byte row segments are loaded before any is used
  float carry = -INFINITY;  // S^shared[4*base - 1] for the next chunk's lane 0
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;  // range of the non-forced keys
  for (int base0 = 0; base0 < n_cand; base0 += 32 * kPoolLoads) {
    float4 vv[kPoolLoads];
#pragma unroll
    for (int u = 0; u < kPoolLoads; ++u) {
      const int b = base0 + 32 * u + lane;
      const int j0 = 4 * b;
      float4 v = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (b < n_cand) {
        if (j0 + 3 < nv) {
          v = __ldg(reinterpret_cast<const float4*>(row + j0));
        } else {
          if (j0 + 0 < nv) v.x = row[j0 + 0];
          if (j0 + 1 < nv) v.y = row[j0 + 1];
          if (j0 + 2 < nv) v.z = row[j0 + 2];
        }
      }
      vv[u] = v;
    }
#pragma unroll
    for (int u = 0; u < kPoolLoads; ++u) {
      const int b = base0 + 32 * u + lane;
      const float4 v = vv[u];
      // kernel 4b-1 is the previous block's last kernel (lane-1's v.w)
      float prev = __shfl_up_sync(0xFFFFFFFFu, v.w, 1);
      if (lane == 0) prev = carry;
      carry = __shfl_sync(0xFFFFFFFFu, v.w, 31);
      if (b < n_cand) {
        const float m = fmax3(fmax3(v.x, v.y, v.z), v.w, prev);
        const bool forced = b < n_init || b > bi - n_local;
        const uint32_t key = float_key(m);
        keys[b] = forced ? kForcedKey : key;
        if (!forced) {
          kmin = min(kmin, key);
          kmax = max(kmax, key);
        }
      }
    }
  }
  kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
  kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
  __syncwarp();
  // n_cand > k >= n_init + n_local: the init and local sets are disjoint
  topk_warp(keys, n_cand, k, hist, out, err, kmin, kmax, n_init + n_local);
}

// Select for one row from precomputed block scores S^cmp[b] (b < i/B; the own
// block is always local, so its entry is not read).
__device__ __forceinline__ void select_row_warp_pooled(const float* __restrict__ cmp, int i,
                                                       int n_init, int n_local, int k,
                                                       uint32_t* keys, uint32_t* hist,
                                                       int* __restrict__ out, int* err) {
  const int lane = (int)lane_id();
  const int bi = i >> 6;
  const int n_cand = bi + 1;
  if (n_cand <= k) {
    for (int b = lane; b < k; b += 32) out[b] = b < n_cand ? b : -1;
    return;
  }
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;  // range of the non-forced keys
  // kPoolLoads float4 loads (4 blocks each) in flight per lane
  for (int base = 0; base < n_cand; base += 128 * kPoolLoads) {
    float4 vv[kPoolLoads];
#pragma unroll
    for (int x = 0; x < kPoolLoads; ++x) {
      const int b0 = base + 128 * x + 4 * lane;
      if (b0 + 3 < bi) {
        vv[x] = __ldg(reinterpret_cast<const float4*>(cmp + b0));
      } else {
        vv[x].x = b0 + 0 < bi ? cmp[b0 + 0] : -INFINITY;
        vv[x].y = b0 + 1 < bi ? cmp[b0 + 1] : -INFINITY;
        vv[x].z = b0 + 2 < bi ? cmp[b0 + 2] : -INFINITY;
        vv[x].w = b0 + 3 < bi ? cmp[b0 + 3] : -INFINITY;
      }
    }
#pragma unroll
    for (int x = 0; x < kPoolLoads; ++x) {
      const int b0 = base + 128 * x + 4 * lane;
      const float v4[4] = {vv[x].x, vv[x].y, vv[x].z, vv[x].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int b = b0 + u;
        if (b < n_cand) {
          const bool forced = b < n_init || b > bi - n_local;
          const uint32_t key = float_key(v4[u]);
          keys[b] = forced ? kForcedKey : key;
          if (!forced) {
            kmin = min(kmin, key);
            kmax = max(kmax, key);
          }
        }
      }
    }
  }
  kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
  kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
  __syncwarp();
  topk_warp(keys, n_cand, k, hist, out, err, kmin, kmax, n_init + n_local);
}

// Top-k over block keys already in shared memory (keys[0..bi], forced blocks
// holding kForcedKey), by a whole CTA: the same exact radix select as
// topk_warp (passes from the first bit in which the competing keys differ,
// early stop) on a CTA-wide histogram.  kmin / kmax bound the n_forced-free
// keys.  `hist` 256 words, `bcast` 4 words (shared).  Rows with at most k
// candidates are handled by the caller.
__device__ __forceinline__ void select_topk_cta(const uint32_t* keys, int n_cand, int k,
                                                uint32_t* hist, uint32_t* bcast,
                                                int* __restrict__ out, int* err, uint32_t kmin,
                                                uint32_t kmax, int n_forced) {
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  int remaining = k - n_forced;
  const uint32_t diff = kmin ^ kmax;
  int top = diff ? 32 - __clz(diff) : 0;
  uint32_t pmask = top >= 32 ? 0u : ~((1u << top) - 1u);
  uint32_t prefix = kmin & pmask;
  if (remaining <= 0) {
    top = 0;
    pmask = 0xFFFFFFFFu;
    prefix = 0xFFFFFFFFu;
  }
#pragma unroll 1
  while (top > 0) {
    const int shift = max(top - 8, 0);
    const uint32_t dm = (1u << (top - shift)) - 1u;
    for (int x = t; x < 256; x += blockDim.x) hist[x] = 0;
    __syncthreads();
    for (int b = t; b < n_cand; b += blockDim.x) {
      const uint32_t key = keys[b];
      if (key != kForcedKey && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dm], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t cnt[8];
      uint32_t local = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        cnt[e] = hist[255 - 8 * lane - e];
        local += cnt[e];
      }
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += x;
      }
      const uint32_t before = incl - local;
      if (before < (uint32_t)remaining && (uint32_t)remaining <= incl) {
        uint32_t run = before;
        for (int e = 0; e < 8; ++e) {
          if (run + cnt[e] >= (uint32_t)remaining) {
            bcast[0] = 255u - 8u * lane - e;
            bcast[1] = run;
            bcast[2] = cnt[e];
            break;
          }
          run += cnt[e];
        }
      }
    }
    __syncthreads();
    prefix |= bcast[0] << shift;
    pmask |= dm << shift;
    remaining -= (int)bcast[1];
    const bool done = bcast[2] == (uint32_t)remaining;  // the whole bucket is taken
    top = shift;
    __syncthreads();
    if (done) break;
  }
  if (warp == 0) {
    const uint32_t T = prefix;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int eq_seen = 0, written = 0;
    for (int base = 0; base < n_cand; base += 32) {
      const int b = base + lane;
      const uint32_t key = b < n_cand ? keys[b] : 0u;
      const bool forced = b < n_cand && key == kForcedKey;
      const uint32_t m = key & pmask;
      const bool eq = b < n_cand && !forced && m == T;
      const uint32_t eqb = __ballot_sync(0xFFFFFFFFu, eq);
      const bool sel = forced || (b < n_cand && m > T) ||
                       (eq && eq_seen + __popc(eqb & lt_mask) < remaining);
      eq_seen += __popc(eqb);
      const uint32_t selb = __ballot_sync(0xFFFFFFFFu, sel);
      const int at = written + __popc(selb & lt_mask);
      if (sel && (!INFV2_CHECKS || at < k)) out[at] = b;
      written += __popc(selb);
    }
    check(written == k, err);
    for (int x = written + lane; x < k; x += 32) out[x] = -1;
  }
}

}  // namespace infv2
