// Prefill over host buffers: a two-slot copy/compute pipeline.
//
// A serving loop hands the layer host-resident Q, K, V and wants O back in
// host memory.  Each submitted batch takes one of two device slots: its inputs
// cross to the device on the pipeline's input stream, the whole prefill runs
// on the caller's compute stream, and O (and the log-sum-exp) return on the
// output stream.  With page-locked host buffers the inputs of batch j+1 and
// the output of batch j-1 travel while batch j computes.  Slot reuse is
// ordered by events: a slot's inputs are overwritten only after the compute
// of the batch two submits earlier has read them, and its output only after
// that batch's output has left.
#include <new>
#include <vector>

#include "internal.cuh"

namespace infv2 {
namespace {

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
  cudaEvent_t in_done[2] = {nullptr, nullptr};
  cudaEvent_t comp_done[2] = {nullptr, nullptr};
  cudaEvent_t out_done[2] = {nullptr, nullptr};
  cudaEvent_t fence = nullptr;
  bool used[2] = {false, false};
  int next = 0;
};

namespace {

void release(infv2_pipeline* pl) {
  if (pl->s_in) cudaStreamSynchronize(pl->s_in);
  if (pl->s_out) cudaStreamSynchronize(pl->s_out);
  for (int b = 0; b < 2; ++b) {
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

extern "C" int infv2_pipeline_submit(infv2_pipeline* pl, const void* q_host, const void* k_host,
                                     const void* v_host, void* o_host, float* lse_host) {
  if (!pl || !q_host || !k_host || !v_host || !o_host) return INFV2_ERR_INVALID_ARG;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return INFV2_ERR_CUDA;
  const int b = pl->next;
  const Slot& s = pl->slot[b];
  const PipeLayout& L = pl->L;
  // inputs: after the compute of the batch two submits back has read this slot
  if (pl->used[b]) PIPE_CK(cudaStreamWaitEvent(pl->s_in, pl->comp_done[b], 0));
  PIPE_CK(cudaMemcpyAsync(s.q, q_host, L.q_bytes, cudaMemcpyHostToDevice, pl->s_in));
  PIPE_CK(cudaMemcpyAsync(s.k, k_host, L.kv_bytes, cudaMemcpyHostToDevice, pl->s_in));
  PIPE_CK(cudaMemcpyAsync(s.v, v_host, L.kv_bytes, cudaMemcpyHostToDevice, pl->s_in));
  PIPE_CK(cudaEventRecord(pl->in_done[b], pl->s_in));
  // compute: after this batch's inputs arrived and the slot's previous output left
  PIPE_CK(cudaStreamWaitEvent(pl->compute, pl->in_done[b], 0));
  if (pl->used[b]) PIPE_CK(cudaStreamWaitEvent(pl->compute, pl->out_done[b], 0));
  const int st = infv2_prefill(&pl->p, s.q, s.k, s.v, pl->cu.data(), pl->batch, pl->prefill_ws,
                               L.prefill_ws, nullptr, s.o, lse_host ? s.lse : nullptr,
                               reinterpret_cast<infv2_stream_t>(pl->compute));
  if (st != INFV2_OK) return st;
  PIPE_CK(cudaEventRecord(pl->comp_done[b], pl->compute));
  // outputs
  PIPE_CK(cudaStreamWaitEvent(pl->s_out, pl->comp_done[b], 0));
  PIPE_CK(cudaMemcpyAsync(o_host, s.o, L.q_bytes, cudaMemcpyDeviceToHost, pl->s_out));
  if (lse_host)
    PIPE_CK(cudaMemcpyAsync(lse_host, s.lse, L.lse_bytes, cudaMemcpyDeviceToHost, pl->s_out));
  PIPE_CK(cudaEventRecord(pl->out_done[b], pl->s_out));
  pl->used[b] = true;
  pl->next = b ^ 1;
  return INFV2_OK;
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
