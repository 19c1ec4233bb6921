// Launch functions shared between the library's translation units.
#pragma once
#include "common.cuh"

namespace infv2 {

int launch_compress_k(const uint16_t* k, int n, int h_kv, uint16_t* kc1, cudaStream_t st);

// Coarse kernels of the LSE approximation: length 128, stride 64.
int launch_compress_k2(const uint16_t* k, int n, int h_kv, uint16_t* kc2, cudaStream_t st);
inline int num_coarse_kernels(int n) { return n >= 128 ? (n - 128) / 64 + 1 : 0; }

int launch_block_scores(const infv2_params* p, const uint16_t* q, const uint16_t* kc1, int n,
                        int q_begin, int q_len, float* s_shared, int ld, float* score_lse,
                        cudaStream_t st);

// Scores with the LSE approximation (pass 1 over K^C2 for rows i >= 127).
int launch_block_scores_approx(const infv2_params* p, const uint16_t* q, const uint16_t* kc1,
                               const uint16_t* kc2, int n, int q_begin, int q_len,
                               float* s_shared, int ld, float* score_lse, cudaStream_t st);

int launch_select(const infv2_params* p, const float* s_shared, int ld, int n, int q_begin,
                  int q_len, int* idx, long long idx_hstride, cudaStream_t st);

// Fused form: block scores S^cmp [h_kv, q_len, ld_cmp] straight from the score
// kernel (max pooling in its epilogue), then a top-k-only selection.
int launch_block_scores_pooled(const infv2_params* p, const uint16_t* q, const uint16_t* kc1,
                               int n, int q_begin, int q_len, float* s_cmp, int ld_cmp,
                               cudaStream_t st);

int launch_select_pooled(const infv2_params* p, const float* s_cmp, int ld_cmp, int n,
                         int q_begin, int q_len, int* idx, long long idx_hstride,
                         cudaStream_t st);

// Row pitch (floats) of S^cmp: blocks of an n-token sequence rounded to 32.
inline int cmp_ld(int n) { return (((n + 63) / 64) + 31) / 32 * 32; }

// Row pitch (floats) of S^shared for an n-token sequence: at least the kernel
// count and four kernels per block, rounded to 32 floats (128 bytes).
inline int shared_ld(int n) {
  const int nc = n >= 32 ? (n - 32) / 16 + 1 : 0;
  const int nb = (n + 63) / 64;
  int ld = nc > 4 * nb ? nc : 4 * nb;
  return ((ld + 31) / 32) * 32;
}

inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Hooks of a staged prefill (the host-buffer pipeline).  need_q(t_end) runs on
// the host before the first launch that reads packed query rows below t_end;
// done_o(t0, t1) right after the launch that completes output rows [t0, t1).
// Both may enqueue stream waits or event records; a non-zero status aborts.
struct PrefillHooks {
  int attn_parts = 1;  // attention launches per sparse sequence (row ranges)
  virtual int need_q(long long t_end) = 0;
  virtual int done_o(long long t0, long long t1) = 0;

 protected:
  ~PrefillHooks() = default;
};

// The whole layer over a packed varlen batch (infv2_prefill's body); hooks may
// be null.  Without hooks the launch sequence is exactly infv2_prefill's.
int run_prefill(const infv2_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                const int* cu_seqlens_host, int batch, void* workspace, size_t ws_bytes,
                int* idx_out, uint16_t* o, float* lse, cudaStream_t st, PrefillHooks* hooks);

}  // namespace infv2
