// Whole-layer prefill over a packed varlen batch, and the dense entry point.
//
// "InfLLM-V2" paper notes, overall framework, and the MiniCPM4 blog (semantic
// kernels): a sequence with at most k blocks (n <= k*B) takes dense causal
// attention; a longer one takes stage-1 compression, the two-pass scores, max
// pooling + selection, and block-sparse attention.  Scores are produced and
// consumed in chunks of query rows so that the S^shared buffer stays bounded.
#include "attn_sparse.cuh"
#include "internal.cuh"

namespace infv2 {
namespace {

constexpr size_t kSharedChunkBytes = size_t(1) << 30;  // S^shared buffer budget (1 GiB)

struct PrefillPlan {
  int max_sparse_n = 0;
  size_t off_kc1 = 0, off_kc2 = 0, off_shared = 0, off_idx = 0, total = 0;
  int ld = 0, chunk = 0;
};

int plan_prefill(const infv2_params* p, const int* cu, int batch, PrefillPlan* pl) {
  for (int s = 0; s < batch; ++s) {
    const int n = cu[s + 1] - cu[s];
    if (n < 0) return INFV2_ERR_INVALID_ARG;
    if (n > p->k * p->B && n > pl->max_sparse_n) pl->max_sparse_n = n;
  }
  const int n = pl->max_sparse_n;
  if (n == 0) return INFV2_OK;
  const size_t nc = (size_t)infv2_num_kernels(p, n);
  pl->ld = shared_ld(n);
  const size_t row_bytes = (size_t)p->h_kv * pl->ld * 4;
  size_t chunk = kSharedChunkBytes / row_bytes;
  chunk = (chunk / 128) * 128;
  if (chunk < 128) chunk = 128;
  if (chunk > (size_t)n) chunk = n;
  pl->chunk = (int)chunk;
  pl->off_kc1 = 0;
  pl->off_kc2 = round256(nc * p->h_kv * 128 * 2);
  const size_t nc2 = p->lse_approx ? (size_t)num_coarse_kernels(n) : 0;  // LSE approximation
  pl->off_shared = pl->off_kc2 + round256(nc2 * p->h_kv * 128 * 2);
  pl->off_idx = pl->off_shared + round256(row_bytes * chunk);
  pl->total = pl->off_idx + round256((size_t)p->h_kv * n * p->k * 4);
  return INFV2_OK;
}

}  // namespace
}  // namespace infv2

using namespace infv2;

extern "C" int infv2_dense_attn(const infv2_params* p, const void* q, const void* k, const void* v,
                                int n, void* o, float* lse, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (n < 0) return INFV2_ERR_INVALID_ARG;
  if (n == 0) return INFV2_OK;
  if (!q || !k || !v || !o) return INFV2_ERR_INVALID_ARG;
  return launch_dense_attn_blocks(p, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                  static_cast<const uint16_t*>(v), n, static_cast<uint16_t*>(o),
                                  lse, n, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int infv2_prefill_workspace_size(const infv2_params* p, const int* cu_seqlens_host,
                                            int batch, size_t* bytes) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (!cu_seqlens_host || !bytes || batch < 0) return INFV2_ERR_INVALID_ARG;
  if (batch > 0 && cu_seqlens_host[0] != 0) return INFV2_ERR_INVALID_ARG;
  PrefillPlan pl;
  st = plan_prefill(p, cu_seqlens_host, batch, &pl);
  if (st != INFV2_OK) return st;
  *bytes = pl.total;
  return INFV2_OK;
}

namespace infv2 {

int run_prefill(const infv2_params* p, const uint16_t* qb, const uint16_t* kb, const uint16_t* vb,
                const int* cu, int batch, void* workspace, size_t ws_bytes, int* idx_out,
                uint16_t* ob, float* lse, cudaStream_t cs, PrefillHooks* hooks) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (!cu || batch < 0) return INFV2_ERR_INVALID_ARG;
  if (batch == 0) return INFV2_OK;
  if (cu[0] != 0) return INFV2_ERR_INVALID_ARG;
  const long long T = cu[batch];
  if (T == 0) return INFV2_OK;
  if (!qb || !kb || !vb || !ob) return INFV2_ERR_INVALID_ARG;
  PrefillPlan pl;
  st = plan_prefill(p, cu, batch, &pl);
  if (st != INFV2_OK) return st;
  if (pl.total > 0) {
    if (!workspace || ws_bytes < pl.total) return INFV2_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return INFV2_ERR_INVALID_ARG;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* kc1 = reinterpret_cast<uint16_t*>(ws + pl.off_kc1);
  uint16_t* kc2 = reinterpret_cast<uint16_t*>(ws + pl.off_kc2);
  float* s_shared = reinterpret_cast<float*>(ws + pl.off_shared);
  int* idx_ws = reinterpret_cast<int*>(ws + pl.off_idx);
  const int parts = hooks && hooks->attn_parts > 1 ? hooks->attn_parts : 1;
  for (int s = 0; s < batch; ++s) {
    const long long off = cu[s];
    const int n = cu[s + 1] - cu[s];
    if (n == 0) continue;
    const uint16_t* qs = qb + off * p->h_q * 128;
    const uint16_t* ks = kb + off * p->h_kv * 128;
    const uint16_t* vs = vb + off * p->h_kv * 128;
    uint16_t* os = ob + off * p->h_q * 128;
    float* lses = lse ? lse + off : nullptr;
    if (n <= p->k * p->B) {
      if (hooks && (st = hooks->need_q(off + n)) != INFV2_OK) return st;
      st = launch_dense_attn_blocks(p, qs, ks, vs, n, os, lses, T, cs);
      if (st != INFV2_OK) return st;
      if (hooks && (st = hooks->done_o(off, off + n)) != INFV2_OK) return st;
      continue;
    }
    st = launch_compress_k(ks, n, p->h_kv, kc1, cs);
    if (st != INFV2_OK) return st;
    if (p->lse_approx) {
      st = launch_compress_k2(ks, n, p->h_kv, kc2, cs);
      if (st != INFV2_OK) return st;
    }
    int* idx = idx_out ? idx_out + off * p->k : idx_ws;
    const long long hstride = idx_out ? T * p->k : (long long)n * p->k;
    // attention over rows [a0, a1) as soon as their blocks are selected: one
    // launch after all score chunks, or `parts` launches interleaved with them
    int a0 = 0, part = 0;
    for (int q0 = 0; q0 < n; q0 += pl.chunk) {
      const int ql = n - q0 < pl.chunk ? n - q0 : pl.chunk;
      if (hooks && (st = hooks->need_q(off + q0 + ql)) != INFV2_OK) return st;
      st = p->lse_approx
               ? launch_block_scores_approx(p, qs, kc1, kc2, n, q0, ql, s_shared, pl.ld, nullptr, cs)
               : launch_block_scores(p, qs, kc1, n, q0, ql, s_shared, pl.ld, nullptr, cs);
      if (st != INFV2_OK) return st;
      st = launch_select(p, s_shared, pl.ld, n, q0, ql, idx, hstride, cs);
      if (st != INFV2_OK) return st;
      const int scored = q0 + ql;
      if (scored == n || (parts > 1 && scored >= (long long)n * (part + 1) / parts)) {
        st = launch_sparse_attn_rows(p, qs, ks, vs, idx, hstride, n, a0, scored, os, lses, T, cs);
        if (st != INFV2_OK) return st;
        if (hooks && (st = hooks->done_o(off + a0, off + scored)) != INFV2_OK) return st;
        a0 = scored;
        while (part < parts && scored >= (long long)n * (part + 1) / parts) ++part;
      }
    }
  }
  return INFV2_OK;
}

}  // namespace infv2

extern "C" int infv2_prefill(const infv2_params* p, const void* q, const void* k, const void* v,
                             const int* cu_seqlens_host, int batch, void* workspace,
                             size_t ws_bytes, int* idx_out, void* o, float* lse,
                             infv2_stream_t stream) {
  return run_prefill(p, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                     static_cast<const uint16_t*>(v), cu_seqlens_host, batch, workspace, ws_bytes,
                     idx_out, static_cast<uint16_t*>(o), lse, reinterpret_cast<cudaStream_t>(stream),
                     nullptr);
}
