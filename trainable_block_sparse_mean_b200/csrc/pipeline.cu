// Prefill over host buffers: a two-slot copy/compute pipeline.
//
// A serving loop hands the layer host-resident Q, K, V and wants O back in
// host memory.  Each submitted batch takes one of two device slots: its inputs
// cross to the device on the pipeline's input stream, the whole prefill runs
// on the caller's compute stream, and O (and the log-sum-exp) return on the
// output stream.  With page-locked host buffers the inputs of batch j+1 and
// the output of batch j-1 travel while batch j computes.  Within a batch the
// copies are cut into parts as well: K and V first, then Q in parts of 8192
// tokens, each score chunk waiting only for the Q rows it reads; the
// attention runs in row ranges interleaved with the score chunks, and each
// finished range of O leaves while the next computes.  Slot reuse is ordered
// by events: a slot's inputs are overwritten only after the compute of the
// batch two submits earlier has read them, and its output only after that
// batch's output has left.
#include <new>
#include <vector>

#include "internal.cuh"

namespace infv2 {
namespace {

constexpr int kQPartRows = 8192;                     // tokens per host->device Q copy
constexpr size_t kOutFlushBytes = size_t(64) << 20;  // output copies coalesced up to this
constexpr int kAttnParts = 8;                        // attention row ranges per sequence

struct PipeLayout {
  size_t prefill_ws = 0;                  // workspace of infv2_prefill
  size_t q_bytes = 0, kv_bytes = 0, lse_bytes = 0;  // exact tensor sizes
  size_t slot = 0;                        // q, k, v, o, lse of one slot (256-B pieces)
  size_t total = 0;
};

int pipeline_layout(const infv2_params* p, const int* cu, int batch, PipeLayout* L) {
  int st = infv2_check_params(p);
  if (st != INFV2_OK) return st;
  if (!cu || batch <= 0 || cu[0] != 0) return INFV2_ERR_INVALID_ARG;
  size_t ws = 0;
  st = infv2_prefill_workspace_size(p, cu, batch, &ws);
  if (st != INFV2_OK) return st;
  const long long T = cu[batch];
  if (T <= 0) return INFV2_ERR_INVALID_ARG;
  L->prefill_ws = round256(ws);
  L->q_bytes = (size_t)T * p->h_q * p->d * 2;
  L->kv_bytes = (size_t)T * p->h_kv * p->d * 2;
  L->lse_bytes = (size_t)T * p->h_q * 4;
  L->slot = 2 * round256(L->q_bytes) + 2 * round256(L->kv_bytes) + round256(L->lse_bytes);
  L->total = L->prefill_ws + 2 * L->slot;
  return INFV2_OK;
}

struct Slot {
  uint16_t *q, *k, *v, *o;
  float* lse;
};

// Makes `device` current for the lifetime of the object and restores the
// caller's device afterwards.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int device) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      ok = false;
      return;
    }
    if (prev != device && cudaSetDevice(device) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

}  // namespace
}  // namespace infv2

using namespace infv2;

struct infv2_pipeline {
  infv2_params p;
  std::vector<int> cu;
  int batch = 0;
  int device = 0;
  PipeLayout L;
  uint8_t* prefill_ws = nullptr;
  Slot slot[2];
  cudaStream_t compute = nullptr;  // the caller's stream
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t in_done[2] = {nullptr, nullptr};  // K and V of the slot arrived
  std::vector<cudaEvent_t> q_done[2];            // Q part i of the slot arrived
  std::vector<cudaEvent_t> o_ready[2];           // a range of O computed (grown on demand)
  cudaEvent_t comp_done[2] = {nullptr, nullptr};
  cudaEvent_t out_done[2] = {nullptr, nullptr};
  cudaEvent_t fence = nullptr;
  bool used[2] = {false, false};
  bool failed = false;  // a submit failed part-way: its slot's queued work is unordered
  int next = 0;
  long long T = 0;
  int n_qparts = 0;
};

namespace {

void release(infv2_pipeline* pl) {
  if (pl->s_in) cudaStreamSynchronize(pl->s_in);
  if (pl->s_out) cudaStreamSynchronize(pl->s_out);
  for (int b = 0; b < 2; ++b) {
    for (cudaEvent_t e : pl->q_done[b])
      if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : pl->o_ready[b]) cudaEventDestroy(e);
    if (pl->in_done[b]) cudaEventDestroy(pl->in_done[b]);
    if (pl->comp_done[b]) cudaEventDestroy(pl->comp_done[b]);
    if (pl->out_done[b]) cudaEventDestroy(pl->out_done[b]);
  }
  if (pl->fence) cudaEventDestroy(pl->fence);
  if (pl->s_in) cudaStreamDestroy(pl->s_in);
  if (pl->s_out) cudaStreamDestroy(pl->s_out);
}

}  // namespace

extern "C" int infv2_pipeline_workspace_size(const infv2_params* p, const int* cu_seqlens_host,
                                             int batch, size_t* bytes) {
  if (!bytes) return INFV2_ERR_INVALID_ARG;
  PipeLayout L;
  const int st = pipeline_layout(p, cu_seqlens_host, batch, &L);
  if (st != INFV2_OK) return st;
  *bytes = L.total;
  return INFV2_OK;
}

extern "C" int infv2_pipeline_create(const infv2_params* p, const int* cu_seqlens_host, int batch,
                                     void* workspace, size_t ws_bytes, infv2_stream_t stream,
                                     infv2_pipeline** out) {
  if (!out) return INFV2_ERR_INVALID_ARG;
  *out = nullptr;
  PipeLayout L;
  int st = pipeline_layout(p, cu_seqlens_host, batch, &L);
  if (st != INFV2_OK) return st;
  if (!workspace) return INFV2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return INFV2_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return INFV2_ERR_WORKSPACE;
  infv2_pipeline* pl = new (std::nothrow) infv2_pipeline();
  if (!pl) return INFV2_ERR_CUDA;
  pl->p = *p;
  pl->cu.assign(cu_seqlens_host, cu_seqlens_host + batch + 1);
  pl->batch = batch;
  pl->L = L;
  pl->T = cu_seqlens_host[batch];
  pl->n_qparts = (int)((pl->T + kQPartRows - 1) / kQPartRows);
  pl->compute = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  pl->prefill_ws = ws;
  for (int b = 0; b < 2; ++b) {
    uint8_t* s = ws + L.prefill_ws + b * L.slot;
    Slot& sl = pl->slot[b];
    sl.q = reinterpret_cast<uint16_t*>(s);
    s += round256(L.q_bytes);
    sl.k = reinterpret_cast<uint16_t*>(s);
    s += round256(L.kv_bytes);
    sl.v = reinterpret_cast<uint16_t*>(s);
    s += round256(L.kv_bytes);
    sl.o = reinterpret_cast<uint16_t*>(s);
    s += round256(L.q_bytes);
    sl.lse = reinterpret_cast<float*>(s);
  }
  bool ok = cudaGetDevice(&pl->device) == cudaSuccess;
  ok = ok && cudaStreamCreateWithFlags(&pl->s_in, cudaStreamNonBlocking) == cudaSuccess;
  ok = ok && cudaStreamCreateWithFlags(&pl->s_out, cudaStreamNonBlocking) == cudaSuccess;
  for (int b = 0; b < 2 && ok; ++b) {
    pl->q_done[b].assign(pl->n_qparts, nullptr);
    for (int i = 0; i < pl->n_qparts && ok; ++i)
      ok = cudaEventCreateWithFlags(&pl->q_done[b][i], cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&pl->in_done[b], cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&pl->comp_done[b], cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&pl->out_done[b], cudaEventDisableTiming) == cudaSuccess;
  }
  ok = ok && cudaEventCreateWithFlags(&pl->fence, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    release(pl);
    delete pl;
    return INFV2_ERR_CUDA;
  }
  *out = pl;
  return INFV2_OK;
}

#define PIPE_CK(call)                                \
  do {                                               \
    if ((call) != cudaSuccess) return INFV2_ERR_CUDA; \
  } while (0)

namespace {

// The prefill's hooks for one submit: the compute stream waits for each Q part
// before the first launch that reads it, and finished ranges of O (and the
// log-sum-exp) are copied back on the output stream, coalesced up to
// kOutFlushBytes.
struct SubmitHooks final : PrefillHooks {
  infv2_pipeline* pl;
  int b;
  uint16_t* o_host;
  float* lse_host;
  int q_waited = 0;
  long long o_begin = 0, o_end = 0;  // computed output rows not yet copied back
  int n_ready = 0;                   // o_ready events used by this submit

  SubmitHooks(infv2_pipeline* pl_, int b_, void* o, float* lse)
      : pl(pl_), b(b_), o_host(static_cast<uint16_t*>(o)), lse_host(lse) {
    attn_parts = kAttnParts;
  }

  int need_q(long long t_end) override {
    while (q_waited < pl->n_qparts && (long long)q_waited * kQPartRows < t_end) {
      if (cudaStreamWaitEvent(pl->compute, pl->q_done[b][q_waited], 0) != cudaSuccess)
        return INFV2_ERR_CUDA;
      ++q_waited;
    }
    return INFV2_OK;
  }

  int done_o(long long t0, long long t1) override {
    if (t0 != o_end) {  // not contiguous with the pending range: send that first
      const int st = flush();
      if (st != INFV2_OK) return st;
      o_begin = t0;
    }
    o_end = t1;
    const size_t row_bytes = (size_t)pl->p.h_q * pl->p.d * 2;
    return (size_t)(o_end - o_begin) * row_bytes >= kOutFlushBytes ? flush() : INFV2_OK;
  }

  int flush() {
    if (o_end <= o_begin) return INFV2_OK;
    std::vector<cudaEvent_t>& ev = pl->o_ready[b];
    if (n_ready == (int)ev.size()) {
      cudaEvent_t e;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return INFV2_ERR_CUDA;
      ev.push_back(e);
    }
    cudaEvent_t e = ev[n_ready++];
    const Slot& s = pl->slot[b];
    const size_t row_bytes = (size_t)pl->p.h_q * pl->p.d * 2;
    if (cudaEventRecord(e, pl->compute) != cudaSuccess ||
        cudaStreamWaitEvent(pl->s_out, e, 0) != cudaSuccess ||
        cudaMemcpyAsync(reinterpret_cast<uint8_t*>(o_host) + o_begin * row_bytes,
                        reinterpret_cast<const uint8_t*>(s.o) + o_begin * row_bytes,
                        (size_t)(o_end - o_begin) * row_bytes, cudaMemcpyDeviceToHost,
                        pl->s_out) != cudaSuccess)
      return INFV2_ERR_CUDA;
    if (lse_host) {  // lse [h_q, T]: the range is one strip per head
      const size_t pitch = (size_t)pl->T * 4;
      if (cudaMemcpy2DAsync(lse_host + o_begin, pitch, s.lse + o_begin, pitch,
                            (size_t)(o_end - o_begin) * 4, pl->p.h_q, cudaMemcpyDeviceToHost,
                            pl->s_out) != cudaSuccess)
        return INFV2_ERR_CUDA;
    }
    o_begin = o_end;
    return INFV2_OK;
  }
};

}  // namespace

namespace {

int submit_once(infv2_pipeline* pl, const void* q_host, const void* k_host, const void* v_host,
                void* o_host, float* lse_host) {
  DeviceGuard guard(pl->device);
  if (!guard.ok) return INFV2_ERR_CUDA;
  const int b = pl->next;
  const Slot& s = pl->slot[b];
  const PipeLayout& L = pl->L;
  // inputs: after the compute of the batch two submits back has read this slot;
  // K and V first (compression and attention need all of them), then Q in parts
  if (pl->used[b]) PIPE_CK(cudaStreamWaitEvent(pl->s_in, pl->comp_done[b], 0));
  PIPE_CK(cudaMemcpyAsync(s.k, k_host, L.kv_bytes, cudaMemcpyHostToDevice, pl->s_in));
  PIPE_CK(cudaMemcpyAsync(s.v, v_host, L.kv_bytes, cudaMemcpyHostToDevice, pl->s_in));
  PIPE_CK(cudaEventRecord(pl->in_done[b], pl->s_in));
  const size_t q_row = (size_t)pl->p.h_q * pl->p.d * 2;
  for (int i = 0; i < pl->n_qparts; ++i) {
    const long long t0 = (long long)i * kQPartRows;
    const long long t1 = t0 + kQPartRows < pl->T ? t0 + kQPartRows : pl->T;
    PIPE_CK(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(s.q) + t0 * q_row,
                            static_cast<const uint8_t*>(q_host) + t0 * q_row,
                            (size_t)(t1 - t0) * q_row, cudaMemcpyHostToDevice, pl->s_in));
    PIPE_CK(cudaEventRecord(pl->q_done[b][i], pl->s_in));
  }
  // compute: after this batch's K/V arrived and the slot's previous output left
  PIPE_CK(cudaStreamWaitEvent(pl->compute, pl->in_done[b], 0));
  if (pl->used[b]) PIPE_CK(cudaStreamWaitEvent(pl->compute, pl->out_done[b], 0));
  SubmitHooks hooks(pl, b, o_host, lse_host);
  int st = run_prefill(&pl->p, s.q, s.k, s.v, pl->cu.data(), pl->batch, pl->prefill_ws,
                       L.prefill_ws, nullptr, s.o, lse_host ? s.lse : nullptr, pl->compute, &hooks);
  if (st == INFV2_OK) st = hooks.need_q(pl->T);  // every Q part before comp_done
  if (st == INFV2_OK) st = hooks.flush();
  if (st != INFV2_OK) return st;
  PIPE_CK(cudaEventRecord(pl->comp_done[b], pl->compute));
  PIPE_CK(cudaEventRecord(pl->out_done[b], pl->s_out));
  pl->used[b] = true;
  pl->next = b ^ 1;
  return INFV2_OK;
}

}  // namespace

extern "C" int infv2_pipeline_submit(infv2_pipeline* pl, const void* q_host, const void* k_host,
                                     const void* v_host, void* o_host, float* lse_host) {
  if (!pl || !q_host || !k_host || !v_host || !o_host) return INFV2_ERR_INVALID_ARG;
  // after a failed submit, the slot's events no longer order the copies and
  // kernels already queued for it, so the pipeline takes no more work
  if (pl->failed) return INFV2_ERR_CUDA;
  const int st = submit_once(pl, q_host, k_host, v_host, o_host, lse_host);
  if (st != INFV2_OK) pl->failed = true;
  return st;
}

extern "C" int infv2_pipeline_wait(infv2_pipeline* pl, infv2_stream_t stream) {
  if (!pl) return INFV2_ERR_INVALID_ARG;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return INFV2_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  PIPE_CK(cudaEventRecord(pl->fence, cs));
  PIPE_CK(cudaStreamWaitEvent(pl->s_in, pl->fence, 0));
  PIPE_CK(cudaStreamWaitEvent(pl->s_out, pl->fence, 0));
  if (cs != pl->compute) PIPE_CK(cudaStreamWaitEvent(pl->compute, pl->fence, 0));
  return INFV2_OK;
}

extern "C" int infv2_pipeline_join(infv2_pipeline* pl, infv2_stream_t stream) {
  if (!pl) return INFV2_ERR_INVALID_ARG;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return INFV2_ERR_CUDA;
  // the output stream's tail follows every submitted copy and compute
  PIPE_CK(cudaEventRecord(pl->fence, pl->s_out));
  PIPE_CK(cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(stream), pl->fence, 0));
  return INFV2_OK;
}

extern "C" int infv2_pipeline_sync(infv2_pipeline* pl) {
  if (!pl) return INFV2_ERR_INVALID_ARG;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return INFV2_ERR_CUDA;
  PIPE_CK(cudaStreamSynchronize(pl->s_out));
  return INFV2_OK;
}

extern "C" int infv2_pipeline_destroy(infv2_pipeline* pl) {
  if (!pl) return INFV2_OK;
  int st = INFV2_OK;
  {
    DeviceGuard guard(pl->device);
    if (!guard.ok) st = INFV2_ERR_CUDA;
    release(pl);
  }
  delete pl;
  return st;
}
