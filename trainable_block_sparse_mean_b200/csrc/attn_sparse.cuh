// Arguments of the block-sparse attention kernel (prefill and decode forms).
#pragma once
#include "common.cuh"

namespace infv2 {

struct AttnArgs {
  int n_rows;              // prefill: tokens of the sequence; decode: sequences of the batch
  int row_begin;           // prefill: first query row of this launch (rows row_begin ..
                           // row_begin + n_rows - 1); decode: 0
  int h_q, h_kv, k;
  const int* idx;          // block list of (g, row): idx + g*idx_hstride + row*idx_rstride
  long long idx_hstride, idx_rstride;
  const uint16_t* q;       // q + (row*h_q + h)*128
  float scale_log2;        // scale * log2(e)
  int decode;              // 1: K/V in cache layout, query position = seqlens[row]
  const int* seqlens;
  int* seqlens_out;        // decode split mode: advanced once all of a row is merged
  int n_split, blocks_per_split;  // the block list is cut into n_split pieces
  int split_out;           // 1: write partials (part_o, part_ml) instead of o / lse
  uint16_t* o;             // o + (row*h_q + h)*128
  float* lse;              // lse[h*lse_ld + row] (natural log), nullable
  long long lse_ld;
  float* part_o;           // [row][h_q][n_split][128] unnormalised sums
  float* part_ml;          // [row][h_q][n_split][2]   (max in log2 units, sum)
  int* counters;           // split mode: [rows * h_kv] pieces done, then [rows] heads done;
                           // the last piece merges and (last head) advances seqlens
  int cap;                 // decode: cache capacity (a position >= cap is not advanced)
  WaitCtx wait;
};

int launch_sparse_attn(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const AttnArgs& a,
                       cudaStream_t st);

int launch_sparse_attn_prefill(const infv2_params* p, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const int* idx, long long idx_hstride, int n,
                               uint16_t* o, float* lse, long long lse_ld, cudaStream_t st);

// The same over query rows [r0, r1) of the n-token sequence only (q, k, v, idx,
// o and lse are the whole sequence's; rows outside the range are not touched).
int launch_sparse_attn_rows(const infv2_params* p, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, const int* idx, long long idx_hstride, int n,
                            int r0, int r1, uint16_t* o, float* lse, long long lse_ld,
                            cudaStream_t st);

}  // namespace infv2

namespace infv2 {
// Block-list entries (tokens per tile x k) that one tile of the tensor-core
// attention can stage: sparse lists need G >= 4 and (128/G)*k <= this.
constexpr int kTcListCap = 2048;

// Whether the tensor-core attention takes this shape (dense: every G).
bool attn_tc_supports(const infv2_params* p, bool dense);

// Tensor-core attention over query rows [r0, r1) of an n-token sequence:
// idx [h_kv][n][k] block lists (row stride k, kv-head stride idx_hstride), or
// null for dense causal attention.
int launch_attn_tc(const infv2_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const int* idx, long long idx_hstride, int n, int r0, int r1, uint16_t* o,
                   float* lse, long long lse_ld, cudaStream_t st);

int launch_dense_attn_blocks(const infv2_params* p, const uint16_t* q, const uint16_t* k,
                             const uint16_t* v, int n, uint16_t* o, float* lse, long long lse_ld,
                             cudaStream_t st);
}  // namespace infv2
