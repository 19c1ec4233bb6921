// Varlen forms of the stage calls: the stages of a packed batch ("thd" layout),
// one launch sequence per sequence.
//
// "InfLLM-V2" paper notes, overall framework: the layer serves packed batches
// of variable-length sequences.  The lengths come as a HOST cu_seqlens array
// (as for infv2_prefill): a sequence's length sets its grids, so the host
// needs it before the first launch.  Each call walks the sequences and issues
// the same launches as the single-sequence entry point would for that
// sequence, on the packed tensors at that sequence's offsets; a sequence's
// results are therefore the single-sequence call's, bit for bit.
#include "attn_sparse.cuh"
#include "internal.cuh"

using namespace infv2;

namespace {

// cu_seqlens_host: batch + 1 non-decreasing offsets from 0 (T = cu[batch]).
int check_cu(const int* cu, int batch) {
  if (!cu || batch < 0) return INFV2_ERR_INVALID_ARG;
  if (batch > 0 && cu[0] != 0) return INFV2_ERR_INVALID_ARG;
  for (int s = 0; s < batch; ++s)
    if (cu[s + 1] < cu[s]) return INFV2_ERR_INVALID_ARG;
  return INFV2_OK;
}

int max_len(const int* cu, int batch) {
  int m = 0;
  for (int s = 0; s < batch; ++s) m = cu[s + 1] - cu[s] > m ? cu[s + 1] - cu[s] : m;
  return m;
}

}  // namespace

extern "C" int infv2_varlen_kernel_offsets(const infv2_params* p, const int* cu_seqlens_host,
                                           int batch, int* cu_kernels_host) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if ((st = check_cu(cu_seqlens_host, batch)) != INFV2_OK) return st;
  if (!cu_kernels_host) return INFV2_ERR_INVALID_ARG;
  cu_kernels_host[0] = 0;
  for (int s = 0; s < batch; ++s)
    cu_kernels_host[s + 1] =
        cu_kernels_host[s] + infv2_num_kernels(p, cu_seqlens_host[s + 1] - cu_seqlens_host[s]);
  return INFV2_OK;
}

extern "C" int infv2_compress_k_varlen(const infv2_params* p, const void* k,
                                       const int* cu_seqlens_host, int batch, void* kc1,
                                       infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if ((st = check_cu(cu_seqlens_host, batch)) != INFV2_OK) return st;
  const int* cu = cu_seqlens_host;
  const auto* kb = static_cast<const uint16_t*>(k);
  auto* cb = static_cast<uint16_t*>(kc1);
  long long ck = 0;  // K^C1 rows of the sequences before s
  for (int s = 0; s < batch; ++s) {
    const int n = cu[s + 1] - cu[s];
    const int nc = infv2_num_kernels(p, n);
    if (nc > 0) {
      if (!k || !kc1) return INFV2_ERR_INVALID_ARG;
      st = launch_compress_k(kb + (long long)cu[s] * p->h_kv * 128, n, p->h_kv,
                             cb + ck * p->h_kv * 128, reinterpret_cast<cudaStream_t>(stream));
      if (st != INFV2_OK) return st;
    }
    ck += nc;
  }
  return INFV2_OK;
}

extern "C" int infv2_block_scores_varlen(const infv2_params* p, const void* q, const void* kc1,
                                         const int* cu_seqlens_host, int batch, float* s_shared,
                                         int ld, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if ((st = check_cu(cu_seqlens_host, batch)) != INFV2_OK) return st;
  const int* cu = cu_seqlens_host;
  if (ld < infv2_num_kernels(p, max_len(cu, batch)) || ld % 4 != 0) return INFV2_ERR_INVALID_ARG;
  const auto* qb = static_cast<const uint16_t*>(q);
  const auto* cb = static_cast<const uint16_t*>(kc1);
  long long ck = 0;
  for (int s = 0; s < batch; ++s) {
    const int n = cu[s + 1] - cu[s];
    const int nc = infv2_num_kernels(p, n);
    if (nc > 0) {  // rows with no visible kernel have no scores
      if (!q || !kc1 || !s_shared) return INFV2_ERR_INVALID_ARG;
      st = launch_block_scores(p, qb + (long long)cu[s] * p->h_q * 128, cb + ck * p->h_kv * 128, n,
                               0, n, s_shared + (long long)p->h_kv * ld * cu[s], ld, nullptr,
                               reinterpret_cast<cudaStream_t>(stream));
      if (st != INFV2_OK) return st;
    }
    ck += nc;
  }
  return INFV2_OK;
}

extern "C" int infv2_select_topk_varlen(const infv2_params* p, const float* s_shared, int ld,
                                        const int* cu_seqlens_host, int batch, int* idx,
                                        infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if ((st = check_cu(cu_seqlens_host, batch)) != INFV2_OK) return st;
  const int* cu = cu_seqlens_host;
  const long long T = batch > 0 ? cu[batch] : 0;
  if (T == 0) return INFV2_OK;
  if (!s_shared || !idx) return INFV2_ERR_INVALID_ARG;
  if (ld < infv2_num_kernels(p, max_len(cu, batch)) || ld % 4 != 0) return INFV2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(s_shared) & 15) != 0) return INFV2_ERR_INVALID_ARG;
  for (int s = 0; s < batch; ++s) {
    const int n = cu[s + 1] - cu[s];
    if (n == 0) continue;
    st = launch_select(p, s_shared + (long long)p->h_kv * ld * cu[s], ld, n, 0, n,
                       idx + (long long)cu[s] * p->k, T * p->k,
                       reinterpret_cast<cudaStream_t>(stream));
    if (st != INFV2_OK) return st;
  }
  return INFV2_OK;
}

extern "C" int infv2_sparse_attn_varlen(const infv2_params* p, const void* q, const void* k,
                                        const void* v, const int* idx, const int* cu_seqlens_host,
                                        int batch, void* o, float* lse, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if ((st = check_cu(cu_seqlens_host, batch)) != INFV2_OK) return st;
  const int* cu = cu_seqlens_host;
  const long long T = batch > 0 ? cu[batch] : 0;
  if (T == 0) return INFV2_OK;
  if (!q || !k || !v || !idx || !o) return INFV2_ERR_INVALID_ARG;
  for (int s = 0; s < batch; ++s) {
    const int n = cu[s + 1] - cu[s];
    if (n == 0) continue;
    const long long off = cu[s];
    st = launch_sparse_attn_prefill(
        p, static_cast<const uint16_t*>(q) + off * p->h_q * 128,
        static_cast<const uint16_t*>(k) + off * p->h_kv * 128,
        static_cast<const uint16_t*>(v) + off * p->h_kv * 128, idx + off * p->k, T * p->k, n,
        static_cast<uint16_t*>(o) + off * p->h_q * 128, lse ? lse + off : nullptr, T,
        reinterpret_cast<cudaStream_t>(stream));
    if (st != INFV2_OK) return st;
  }
  return INFV2_OK;
}

extern "C" int infv2_dense_attn_varlen(const infv2_params* p, const void* q, const void* k,
                                       const void* v, const int* cu_seqlens_host, int batch,
                                       void* o, float* lse, infv2_stream_t stream) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if ((st = check_cu(cu_seqlens_host, batch)) != INFV2_OK) return st;
  const int* cu = cu_seqlens_host;
  const long long T = batch > 0 ? cu[batch] : 0;
  if (T == 0) return INFV2_OK;
  if (!q || !k || !v || !o) return INFV2_ERR_INVALID_ARG;
  for (int s = 0; s < batch; ++s) {
    const int n = cu[s + 1] - cu[s];
    if (n == 0) continue;
    const long long off = cu[s];
    st = launch_dense_attn_blocks(p, static_cast<const uint16_t*>(q) + off * p->h_q * 128,
                                  static_cast<const uint16_t*>(k) + off * p->h_kv * 128,
                                  static_cast<const uint16_t*>(v) + off * p->h_kv * 128, n,
                                  static_cast<uint16_t*>(o) + off * p->h_q * 128,
                                  lse ? lse + off : nullptr, T,
                                  reinterpret_cast<cudaStream_t>(stream));
    if (st != INFV2_OK) return st;
  }
  return INFV2_OK;
}
