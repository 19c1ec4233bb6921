/*
 * infv2.h -- C ABI of libinfv2.so: InfLLM-V2 dense-sparse switchable attention
 * for one causal GQA layer, hand-written for NVIDIA B200 (sm_100a).
 *
 * Method (the InfLLM-V2 paper, arXiv 2509.24663, and its public summaries):
 *   1. stage-1 compression: K^C1 = mean of K over kernels of l_C1 = B/2 tokens
 *      with stride s_C1 = B/4 (paper notes, key design 3; MiniCPM4 blog,
 *      semantic kernels);
 *   2. S^C1 = softmax(Q K^C1^T) over the causally visible kernels and the GQA
 *      group sum S^shared = sum_h S^C1(h), computed in two passes (log-sum-exp,
 *      then normalise-and-sum) so that only S^shared reaches memory (paper
 *      notes, key design 4; arXiv summary, section 3 "Efficient Implementation");
 *   3. block scores S^cmp = max pooling of S^shared over the kernels that
 *      intersect each block (l = 5, s = 4) (paper notes, key design 3; MiniCPM4
 *      blog, semantic kernels);
 *   4. selection I(i) = I_init u I_local(i) u top-k(S^cmp), one set per query
 *      token and kv head (paper notes, key design 2; MiniCPM4 blog, top-k
 *      sharing);
 *   5. block-sparse causal attention over the selected blocks, returning O and
 *      the log-sum-exp (arXiv summary, Appendix A), or dense causal attention
 *      when the sequence has at most k blocks (MiniCPM4 blog, semantic kernels).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, unless a
 *     parameter says "host".  The library allocates no device memory; scratch
 *     space is the caller's `workspace` (infv2_select_blocks_noalloc instead
 *     uses a fixed array that the library holds on each device; a pipeline
 *     handle owns host state, two streams and events).
 *   - bf16 tensors are raw 16-bit patterns (e.g. torch.bfloat16 storage);
 *     every tensor is dense, row-major, 16-byte aligned.
 *   - Token layout ("thd"): q [n, h_q, d], k and v [n, h_kv, d]; query head h
 *     belongs to kv head h / (h_q / h_kv).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and return an infv2_status for argument / launch errors.  Errors
 *     detected inside a kernel (a bounded wait that timed out) are recorded in
 *     a per-device word read by infv2_device_status().
 *   - Debug build: compiled with INFV2_CHECKS=1 (libinfv2_checks.so), the
 *     kernels also check their data-dependent indices and invariants (block
 *     lists ascending without repeats, each selected list's size, order and
 *     forced blocks, finite attention results) and record INFV2_ERR_CHECK in
 *     the same word on the first failure.  A check never traps and never
 *     changes a result; the default build compiles them out.
 *   - No call retains a pointer after it returns, except a pipeline, which
 *     keeps its workspace and the host buffers of queued batches; calls that
 *     share output or workspace memory must be ordered on the caller's
 *     streams.
 */
#ifndef INFV2_H
#define INFV2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* infv2_stream_t;

enum infv2_status {
  INFV2_OK = 0,
  INFV2_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent shape */
  INFV2_ERR_UNSUPPORTED = 2, /* valid for the method but not for this build's kernels */
  INFV2_ERR_WORKSPACE = 3,   /* workspace smaller than the *_workspace_size answer */
  INFV2_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  INFV2_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out (device word only) */
  INFV2_ERR_CHECK = 6        /* a device-side check of the INFV2_CHECKS build failed
                                (device word only; never raised by the default build) */
};

/* Method parameters.
 *   B        block size in tokens (selection and attention granularity)
 *   l_c1     stage-1 kernel length (B/2 in the paper)
 *   s_c1     stage-1 kernel stride (B/4 in the paper)
 *   pool_l   max-pool length in kernels (5): kernels intersecting a block
 *   pool_s   max-pool stride in kernels (4)
 *   n_init   initial blocks always selected
 *   n_local  local blocks always selected: {b_i - n_local + 1 .. b_i}
 *   k        total blocks selected per query, init and local included
 *   h_q, h_kv, d   query heads, kv heads, head dim
 *   scale    logit scale of both the scores and the attention (1/sqrt(d))
 *   window   sliding window (tokens) that the local blocks must cover:
 *            n_local >= ceil(window / B) + 1 is enforced (0 = no window)
 *   lse_approx  0: exact two-pass scores (default).  1: the LSE
 *            approximation (paper notes, key design 4; MiniCPM4 blog,
 *            efficient top-k): pass 1 estimates each head's log-sum-exp from
 *            coarse kernels K^C2 (l_C2 = 4 l_c1, s_C2 = 4 s_c1) as
 *            log sum_{visible c} exp(scale q . K^C2_c) + log(s_C2 / s_c1);
 *            rows that see no coarse kernel keep the exact value.  Used by
 *            infv2_prefill; infv2_decode (and its workspace query) returns
 *            INFV2_ERR_UNSUPPORTED when it is set; the stage entry points
 *            and infv2_select_blocks_noalloc do not read it (the approximate
 *            scores have their own entry, infv2_block_scores_approx).
 * This build's kernels support d = 128, B = 64, l_c1 = 32, s_c1 = 16,
 * pool_l = 5, pool_s = 4, h_q % h_kv == 0 with G = h_q/h_kv in {1,2,4,8,16},
 * k >= n_init + n_local, n_local >= 1 and k <= 256.  Other values return
 * INFV2_ERR_UNSUPPORTED. */
typedef struct infv2_params {
  int B, l_c1, s_c1, pool_l, pool_s;
  int n_init, n_local, k;
  int h_q, h_kv, d;
  float scale;
  int window;
  int lse_approx;
} infv2_params;

/* Fill *p with the paper's hyper-parameters (B=64, l_c1=32, s_c1=16, l=5,
 * s=4, n_init=1, n_local=2, k=64, d=128, scale=1/sqrt(128)) for h_q, h_kv,
 * with window 0 and the exact scores (lse_approx 0). */
void infv2_default_params(infv2_params* p, int h_q, int h_kv);

/* Validate *p against the method and this build.  Returns INFV2_OK,
 * INFV2_ERR_INVALID_ARG or INFV2_ERR_UNSUPPORTED. */
int infv2_check_params(const infv2_params* p);

/* Static text for a status code (never NULL). */
const char* infv2_status_string(int status);

/* Number of complete stage-1 kernels of an n-token sequence:
 * n >= l_c1 ? (n - l_c1) / s_c1 + 1 : 0. */
int infv2_num_kernels(const infv2_params* p, int n);

/* Read and clear this device's kernel error word (waits for `stream`).
 * Returns INFV2_OK, INFV2_ERR_TIMEOUT, INFV2_ERR_CHECK (debug build only), or
 * INFV2_ERR_CUDA if the read fails. */
int infv2_device_status(infv2_stream_t stream);

/* The same call under a second name, infv2_get_device_status. */
int infv2_get_device_status(infv2_stream_t stream);

/* Stage 1 (paper notes, key design 3): K^C1[j, g, :] = bf16 round-to-nearest-
 * even of the exact mean of K[t, g, :] over t = j*s_c1 .. j*s_c1 + l_c1 - 1.
 *   k    bf16 [n, h_kv, d]            (input)
 *   kc1  bf16 [num_kernels(n), h_kv, d] (output)
 * n = 0 or n < l_c1 writes nothing. */
int infv2_compress_k(const infv2_params* p, const void* k, int n, void* kc1,
                     infv2_stream_t stream);

/* Coarse kernels of the LSE approximation (paper notes, key design 4):
 * K^C2[c, g, :] = bf16 round-to-nearest-even of the exact mean of K[t, g, :]
 * over t = c*4*s_c1 .. c*4*s_c1 + 4*l_c1 - 1 (128 tokens at stride 64).
 *   k    bf16 [n, h_kv, d];  kc2  bf16 [num_coarse_kernels(n), h_kv, d] (output)
 * num_coarse_kernels(n) = n >= 4*l_c1 ? (n - 4*l_c1) / (4*s_c1) + 1 : 0. */
int infv2_compress_k2(const infv2_params* p, const void* k, int n, void* kc2,
                      infv2_stream_t stream);

/* Stage 2, fused two-pass scores (paper notes, key design 4; arXiv summary,
 * section 3): for query rows i in [q_begin, q_begin + q_len) of an n-token
 * sequence and kv head g, with J(i) the kernels j where j*s_c1 + l_c1 - 1 <= i,
 *   S^shared[g, i - q_begin, j] = sum_{h in group g} exp(z_hj - lse_h),
 *   z_hj = scale * q[i, h, :] . kc1[j, g, :],  lse_h = log sum_{j in J(i)} exp(z_hj).
 *   q         bf16 [n, h_q, d];  kc1  bf16 [num_kernels(n), h_kv, d]
 *   s_shared  fp32 [h_kv, q_len, ld] (output); only j < |J(i)| is written
 *   ld        row pitch in floats, >= num_kernels(n), multiple of 4
 *   score_lse fp32 [h_q, q_len] (output, nullable): lse_h (natural log),
 *             -inf for rows with no visible kernel. */
int infv2_block_scores(const infv2_params* p, const void* q, const void* kc1, int n, int q_begin,
                       int q_len, float* s_shared, int ld, float* score_lse,
                       infv2_stream_t stream);

/* infv2_block_scores with the LSE approximation: lse_h is the coarse estimate
 * of the lse_approx parameter (whatever p->lse_approx holds) for rows that see
 * a coarse kernel (i >= 4*l_c1 - 1), the exact value for the others.  Pass 1
 * then runs over the coarse kernels, a quarter as many as pass 2's.
 *   kc2  bf16 [num_coarse_kernels(n), h_kv, d] from infv2_compress_k2
 * Other arguments and outputs as infv2_block_scores (score_lse receives the
 * log-sum-exp used). */
int infv2_block_scores_approx(const infv2_params* p, const void* q, const void* kc1,
                              const void* kc2, int n, int q_begin, int q_len, float* s_shared,
                              int ld, float* score_lse, infv2_stream_t stream);

/* Stages 3-4 (paper notes, key designs 2-3; MiniCPM4 blog, semantic kernels):
 * for each row i in [q_begin, q_begin + q_len) and kv head g, block scores
 *   S^cmp[b] = max over visible kernels j intersecting block b of S^shared[j],
 * then I(i) = all of 0..i/B when that is at most k blocks, else the init and
 * local blocks plus the highest-scoring others up to k in total (equal scores:
 * lower block first).
 *   s_shared  fp32 [h_kv, q_len, ld] as written by infv2_block_scores
 *   idx       int32 [h_kv, n, k] (output): rows q_begin.. written, ascending,
 *             padded with -1. */
int infv2_select_topk(const infv2_params* p, const float* s_shared, int ld, int n, int q_begin,
                      int q_len, int* idx, infv2_stream_t stream);

/* Stages 2-3 fused (paper notes, limitations: folding max pooling and top-k
 * into the kernel is left as future work there).  Same computation as
 * infv2_block_scores followed by the max pooling of infv2_select_topk, done
 * in the score kernel's epilogue, so only the block scores reach memory:
 *   s_cmp   fp32 [h_kv, q_len, ld_cmp] (output): row (g, i - q_begin) holds
 *           S^cmp[b] for b < i/B (the blocks before the query's own block,
 *           which is always a local block); entries from i/B on are not
 *           written.  ld_cmp >= ceil(n / B) and a multiple of 4.
 * Other arguments as infv2_block_scores (no score_lse output). */
int infv2_block_scores_pooled(const infv2_params* p, const void* q, const void* kc1, int n,
                              int q_begin, int q_len, float* s_cmp, int ld_cmp,
                              infv2_stream_t stream);

/* Stage 4 alone: the top-k selection of infv2_select_topk from the block
 * scores written by infv2_block_scores_pooled (same rule, same output).
 *   s_cmp  fp32 [h_kv, q_len, ld_cmp], 16-byte aligned, ld_cmp a multiple
 *          of 4;  idx int32 [h_kv, n, k] (output). */
int infv2_select_topk_pooled(const infv2_params* p, const float* s_cmp, int ld_cmp, int n,
                             int q_begin, int q_len, int* idx, infv2_stream_t stream);

/* Stage 5, block-sparse attention (arXiv summary, Appendix A): for every
 * query i and head h of group g, softmax attention over the tokens t <= i of
 * the blocks listed in idx[g, i, :].  Entries < 0 and entries past the
 * query's own block (i / 64) add nothing and are skipped; a row left with no
 * block gets O = 0 and lse = -inf.  The lists are meant to be ascending
 * without repeats, as infv2_select_topk writes them: a repeated block would
 * count twice (the INFV2_CHECKS build reports that as INFV2_ERR_CHECK).
 *   q bf16 [n, h_q, d]; k, v bf16 [n, h_kv, d]; idx int32 [h_kv, n, k]
 *   o   bf16 [n, h_q, d] (output)
 *   lse fp32 [h_q, n] (output, nullable): natural log-sum-exp of the logits. */
int infv2_sparse_attn(const infv2_params* p, const void* q, const void* k, const void* v,
                      const int* idx, int n, void* o, float* lse, infv2_stream_t stream);

/* Stage 5 over query rows r0 .. r1-1 only (a prefill computed in row chunks:
 * the rows whose blocks have been selected so far).  Tensors are the whole
 * sequence's, as in infv2_sparse_attn; rows outside [r0, r1) of o and lse
 * are not written and rows of idx outside it are not read.  idx NULL: dense
 * causal attention (every block up to the query's own).  Only K/V rows below
 * the last block boundary at or after r1 are read.  0 <= r0 <= r1 <= n, else
 * INFV2_ERR_INVALID_ARG; r0 == r1 does nothing.  A split of [0, n) into
 * ranges whose ends are multiples of 128/G tokens (the attention's query tile;
 * G = h_q / h_kv) or n gives infv2_sparse_attn's results bit for bit; ends
 * inside a tile give results equal to within rounding (a row's probabilities
 * are rounded against a reference maximum that the other tokens of its tile
 * can move). */
int infv2_sparse_attn_rows(const infv2_params* p, const void* q, const void* k, const void* v,
                           const int* idx, int n, int r0, int r1, void* o, float* lse,
                           infv2_stream_t stream);

/* Workspace bytes that infv2_sparse_attn_bwd needs for an n-token sequence
 * (either mode: block lists or dense). */
int infv2_sparse_attn_bwd_workspace_size(const infv2_params* p, int n, size_t* bytes);

/* Backward of infv2_sparse_attn (or of the dense attention when idx is NULL)
 * for training (arXiv summary, Appendix A: the forward's log-sum-exp is kept
 * for the backward).  The block lists are fixed: the selection is not
 * differentiated.  For every query i, head h of group g and visible token t of
 * i's blocks, with P_t = exp(scale q_ih . k_t - lse[h, i]):
 *   D_ih = dO_ih . O_ih   (O = the forward output passed in)
 *   dS_t = P_t (dO_ih . v_t - D_ih)
 *   dq_ih = scale sum_t dS_t k_t;  dk_t += scale dS_t q_ih;  dv_t += P_t dO_ih
 *   q bf16 [n, h_q, d]; k, v bf16 [n, h_kv, d]; idx int32 [h_kv, n, k] or NULL
 *   o bf16 [n, h_q, d] and lse fp32 [h_q, n] (natural) from the forward
 *   d_o bf16 [n, h_q, d]
 *   dq fp32 [n, h_q, d]; dk, dv fp32 [n, h_kv, d] (outputs, overwritten)
 *   workspace: >= infv2_sparse_attn_bwd_workspace_size bytes, 256-byte aligned.
 * dk and dv are sums over many queries added in an order that varies from run
 * to run: equal inputs give results equal up to fp32 rounding. */
int infv2_sparse_attn_bwd(const infv2_params* p, const void* q, const void* k, const void* v,
                          const int* idx, int n, const void* o, const float* lse,
                          const void* d_o, float* dq, float* dk, float* dv, void* workspace,
                          size_t ws_bytes, infv2_stream_t stream);

/* Dense causal attention with the same weights (MiniCPM4 blog: sequences of
 * at most k blocks switch to dense attention).  Layouts as infv2_sparse_attn. */
int infv2_dense_attn(const infv2_params* p, const void* q, const void* k, const void* v, int n,
                     void* o, float* lse, infv2_stream_t stream);

/* ---- Varlen forms of the stage calls ----------------------------------------
 * The stage calls above on a packed batch ("thd": q [T, h_q, d], k and v
 * [T, h_kv, d], T = cu_seqlens_host[batch]); sequence s owns tokens
 * cu_seqlens_host[s] .. cu_seqlens_host[s+1]-1.  cu_seqlens_host is a HOST
 * int32 array [batch + 1], starting at 0 and non-decreasing (as for
 * infv2_prefill: each sequence's length sets its grids).  Each call issues,
 * per sequence, the launches of the single-sequence call, so a sequence's
 * results equal that call's bit for bit.  Per-sequence tensors are packed:
 *   K^C1      [sum_s nc_s, h_kv, d]: sequence s's kernels from row cu_kernels[s]
 *             (infv2_varlen_kernel_offsets), nc_s = infv2_num_kernels(p, n_s)
 *   S^shared  sequence s's [h_kv, n_s, ld] block at float offset
 *             h_kv * ld * cu_seqlens_host[s]; ld >= the largest nc_s, multiple
 *             of 4 (the whole buffer: h_kv * T * ld floats, 16-byte aligned)
 *   idx       int32 [h_kv, T, k]; o bf16 [T, h_q, d]; lse fp32 [h_q, T] (nullable)
 * Errors as for the single-sequence calls; a bad cu_seqlens_host is
 * INFV2_ERR_INVALID_ARG before any launch. */

/* cu_kernels_host[s] = sum over t < s of infv2_num_kernels(p, n_t), for
 * s = 0 .. batch (HOST int32 [batch + 1], output).  Host only. */
int infv2_varlen_kernel_offsets(const infv2_params* p, const int* cu_seqlens_host, int batch,
                                int* cu_kernels_host);
int infv2_compress_k_varlen(const infv2_params* p, const void* k, const int* cu_seqlens_host,
                            int batch, void* kc1, infv2_stream_t stream);
int infv2_block_scores_varlen(const infv2_params* p, const void* q, const void* kc1,
                              const int* cu_seqlens_host, int batch, float* s_shared, int ld,
                              infv2_stream_t stream);
int infv2_select_topk_varlen(const infv2_params* p, const float* s_shared, int ld,
                             const int* cu_seqlens_host, int batch, int* idx,
                             infv2_stream_t stream);
int infv2_sparse_attn_varlen(const infv2_params* p, const void* q, const void* k, const void* v,
                             const int* idx, const int* cu_seqlens_host, int batch, void* o,
                             float* lse, infv2_stream_t stream);
int infv2_dense_attn_varlen(const infv2_params* p, const void* q, const void* k, const void* v,
                            const int* cu_seqlens_host, int batch, void* o, float* lse,
                            infv2_stream_t stream);

/* Workspace bytes that infv2_prefill needs for this varlen batch.
 *   cu_seqlens_host  HOST int32 [batch + 1], cu_seqlens_host[0] = 0. */
int infv2_prefill_workspace_size(const infv2_params* p, const int* cu_seqlens_host, int batch,
                                 size_t* bytes);

/* The whole layer over a packed varlen batch (paper notes, overall framework:
 * dense for short sequences, sparse for long ones).  Sequence s owns tokens
 * cu_seqlens_host[s] .. cu_seqlens_host[s+1]-1 of q [T, h_q, d], k/v
 * [T, h_kv, d]; it takes dense attention if its length n <= k*B, else stages
 * 1-5.  Outputs: o bf16 [T, h_q, d]; lse fp32 [h_q, T] (nullable); idx_out
 * int32 [h_kv, T, k] (nullable; rows of dense sequences are not written).
 * workspace: device scratch of at least infv2_prefill_workspace_size bytes,
 * 256-byte aligned. */
int infv2_prefill(const infv2_params* p, const void* q, const void* k, const void* v,
                  const int* cu_seqlens_host, int batch, void* workspace, size_t ws_bytes,
                  int* idx_out, void* o, float* lse, infv2_stream_t stream);

/* ---- Prefill over HOST buffers: a two-slot copy/compute pipeline ----------
 * The same layer as infv2_prefill for a serving loop whose Q, K, V arrive in
 * host memory and whose O must return there.  A pipeline is bound to one
 * varlen shape (cu_seqlens) and one device (the current one at creation).
 * Each submit takes one of two device slots in turn:
 *   - its inputs are copied host -> device on the pipeline's input stream;
 *   - the prefill runs on the caller's compute stream;
 *   - O (and the log-sum-exp) are copied device -> host on its output stream.
 * With page-locked host buffers, batch j+1's inputs and batch j-1's output
 * cross PCIe while batch j computes; pageable buffers are accepted but their
 * copies serialise with the host.  Within a batch, K and V are copied first
 * and Q in parts of 8192 tokens; each score chunk waits only for the Q rows it
 * reads, the attention runs in row ranges between the score chunks, and each
 * finished range of O (and its log-sum-exp) is copied back while the next
 * range computes.  The results are those of infv2_prefill, bit for bit.
 * Slot reuse is ordered by events, so any number of submits may be queued.
 * The library allocates no device memory for a pipeline: the caller's
 * workspace holds the prefill workspace and both slots.  The pipeline owns
 * two CUDA streams and its events, released by infv2_pipeline_destroy.  A
 * handle is not thread-safe: one host thread at a time may call into it. */
typedef struct infv2_pipeline infv2_pipeline;

/* Device workspace bytes a pipeline for this varlen batch needs: the
 * infv2_prefill workspace plus, per slot, q, k, v, o and lse.
 * cu_seqlens_host: HOST int32 [batch + 1], cu_seqlens_host[0] = 0, batch >= 1,
 * at least one token.  Host-only; INFV2_ERR_INVALID_ARG on bad shapes. */
int infv2_pipeline_workspace_size(const infv2_params* p, const int* cu_seqlens_host, int batch,
                                  size_t* bytes);

/* Create a pipeline on the current device.
 *   workspace  device memory of at least infv2_pipeline_workspace_size bytes,
 *              256-byte aligned, owned by the caller and kept alive and
 *              untouched until infv2_pipeline_destroy returns;
 *   stream     the compute stream (the prefill kernels run there);
 *   *out       receives the handle (NULL on failure).
 * Errors: INFV2_ERR_INVALID_ARG (bad shape, NULL or misaligned workspace),
 * INFV2_ERR_WORKSPACE (too small), INFV2_ERR_CUDA (a stream or event could
 * not be created, or host memory ran out). */
int infv2_pipeline_create(const infv2_params* p, const int* cu_seqlens_host, int batch,
                          void* workspace, size_t ws_bytes, infv2_stream_t stream,
                          infv2_pipeline** out);

/* Enqueue one batch and return without waiting.
 *   q_host  HOST bf16 [T, h_q, d];  k_host, v_host  HOST bf16 [T, h_kv, d]
 *   o_host  HOST bf16 [T, h_q, d] (output)
 *   lse_host  HOST fp32 [h_q, T] (output, nullable)
 * T = cu_seqlens_host[batch] of the pipeline.  The host buffers must stay
 * allocated and the inputs unchanged, and the outputs must not be read, until
 * infv2_pipeline_sync returns (or a stream given to infv2_pipeline_join has
 * passed that point).  Errors: INFV2_ERR_INVALID_ARG (NULL pointer),
 * INFV2_ERR_CUDA (a copy, event or launch failed part-way: the pipeline then
 * refuses further submits with INFV2_ERR_CUDA and should be destroyed). */
int infv2_pipeline_submit(infv2_pipeline* pl, const void* q_host, const void* k_host,
                          const void* v_host, void* o_host, float* lse_host);

/* Order the work submitted after this call behind the work enqueued so far on
 * `stream` (all three of the pipeline's streams wait for it). */
int infv2_pipeline_wait(infv2_pipeline* pl, infv2_stream_t stream);

/* Make `stream` wait, without blocking the host, until every batch submitted
 * so far has landed in its host output buffers. */
int infv2_pipeline_join(infv2_pipeline* pl, infv2_stream_t stream);

/* Block the host until every batch submitted so far has landed in its host
 * output buffers.  INFV2_ERR_CUDA if a copy or kernel failed. */
int infv2_pipeline_sync(infv2_pipeline* pl);

/* Wait for the pipeline's streams, release them and the events, and free the
 * handle (NULL is a no-op).  The workspace may be freed afterwards. */
int infv2_pipeline_destroy(infv2_pipeline* pl);

/* Workspace bytes that infv2_decode needs. */
int infv2_decode_workspace_size(const infv2_params* p, int batch, int cap, size_t* bytes);

/* One decode step for a batch of sequences, each with its own KV cache
 * (MiniCPM4 blog, query/key granularity: one query token selects its own
 * blocks, which is what makes decoding fast).  For sequence s with L =
 * seqlens[s] cached tokens (0 <= L < cap), the step
 *   1. writes k_new[s], v_new[s] to cache position L and, when that token
 *      completes a stage-1 kernel (L + 1 >= l_c1 and (L + 1 - l_c1) % s_c1
 *      == 0), writes K^C1 of kernel (L + 1 - l_c1) / s_c1 to kc1_cache;
 *   2. computes S^shared, S^cmp and I(L) for the query at position L;
 *   3. attends over the selected tokens (dense when L + 1 <= k*B);
 *   4. increments seqlens[s].
 *   q        bf16 [batch, h_q, d];  k_new, v_new bf16 [batch, h_kv, d]
 *   k_cache, v_cache  bf16 [batch, h_kv, cap, d]
 *   kc1_cache         bf16 [batch, h_kv, num_kernels(cap), d]
 *   seqlens  int32 [batch] (device, read and incremented)
 *   o        bf16 [batch, h_q, d];  lse fp32 [batch, h_q] (nullable)
 *   idx_out  int32 [batch, h_kv, k] (nullable) */
int infv2_decode(const infv2_params* p, const void* q, const void* k_new, const void* v_new,
                 void* k_cache, void* v_cache, void* kc1_cache, int* seqlens, int batch, int cap,
                 void* workspace, size_t ws_bytes, int* idx_out, void* o, float* lse,
                 infv2_stream_t stream);

/* The attention stage of infv2_decode alone, over block lists the caller
 * gives (MiniCPM4 blog, query/key granularity: each decode query attends to
 * its own blocks; arXiv summary, Appendix A: the kernel returns O and the
 * log-sum-exp).  For sequence s, the query q[s] at position pos[s] attends to
 * the cached tokens t <= pos[s] of the blocks in idx[s, g, :] (entries < 0
 * ignored), with the split-KV kernel of the decode step.  Neither the caches
 * nor pos are written: a caller can re-run the attention on a selection it
 * holds (a verification, or a selection made elsewhere).
 *   q        bf16 [batch, h_q, d]
 *   k_cache, v_cache  bf16 [batch, h_kv, cap, d]
 *   pos      int32 [batch] (device): 0 <= pos[s] < cap
 *   idx      int32 [batch, h_kv, k]
 *   workspace: >= infv2_decode_workspace_size(p, batch, cap) bytes, 256-byte
 *            aligned (it may be the decode step's; calls that share it must be
 *            ordered on the caller's streams)
 *   o        bf16 [batch, h_q, d];  lse fp32 [batch, h_q] (nullable) */
int infv2_decode_attn(const infv2_params* p, const void* q, const void* k_cache,
                      const void* v_cache, const int* pos, int batch, int cap, const int* idx,
                      void* workspace, size_t ws_bytes, void* o, float* lse,
                      infv2_stream_t stream);

/* Block selection (the work of infv2_block_scores followed by
 * infv2_select_topk) for callers that cannot allocate device memory: code that
 * runs inside a memory arena or pool it does not own, an engine whose
 * allocator is frozen after start-up, or a plugin that only receives input and
 * output pointers.  The paper has no counterpart; this is a packaging variant.
 * The intermediate S^shared rows live in a 16 MiB array that the library
 * keeps on every GPU that loads it until the process exits; nothing is
 * allocated and no workspace is taken.  Inputs and output are as for the two
 * calls it replaces:
 *   q    bf16 [n, h_q, d];  kc1  bf16 [num_kernels(n), h_kv, d]
 *   idx  int32 [h_kv, n, k] (output): rows q_begin .. q_begin+q_len-1 written.
 * Rows are processed in chunks that fit the array.  Sizes whose S^shared rows
 * for one 128-token tile do not fit (h_kv * ld * 4 * 128 > 16 MiB, with
 * ld = max(num_kernels(n), 4*ceil(n/B)) rounded up to 32; e.g. n > 262144 at
 * h_kv = 2) return INFV2_ERR_UNSUPPORTED.  The first call on a device looks up
 * the array's device address (make it before any stream capture), and so does
 * the first call after the device's context changed (a device reset).  Every call
 * shares the array: calls that can overlap on the GPU race and must be
 * serialised by the caller. */
int infv2_select_blocks_noalloc(const infv2_params* p, const void* q, const void* kc1, int n,
                                int q_begin, int q_len, int* idx, infv2_stream_t stream);

/* Self-test of the exponentials the kernels use: y[i] = 2^x[i] by
 *   which = 0  the MUFU instruction (ex2.approx, flush to zero);
 *   which = 1  the FMA-pipe polynomial of the score kernel (degree 5, relative
 *              error below 2.3e-7; x below -127 gives 0);
 *   which = 2  the FMA-pipe cubic of the attention's probabilities (relative
 *              error below 1.1e-4 on [-126, 64]; x <= -127 gives exactly 0,
 *              x above 64 gives 2^64).
 * No counterpart in the paper: it lets a test hold each form to its bound.
 * x, y: device fp32 [n].  INFV2_ERR_INVALID_ARG for another `which`. */
int infv2_selftest_exp2(int which, const float* x, float* y, int n, infv2_stream_t stream);

/* Self-test of the bounded-wait error path: launches one kernel that waits
 * on a barrier nobody arrives at, with the given limit in microseconds; the
 * kernel gives up, records INFV2_ERR_TIMEOUT and exits normally.  Read the
 * result with infv2_device_status(). */
int infv2_selftest_timeout(int limit_us, infv2_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* INFV2_H */
