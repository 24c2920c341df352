// Decode session: one decode step per call from host buffers to host
// buffers, with the transfers overlapped with the kernels.
//
// The session owns the device side of a decode loop: two slots of input and
// output buffers, the selection, the split partials and both workspaces.  A
// step copies its inputs host -> device on the session's upload stream,
// runs qsa_compress_append, qsa_index_topk and qsa_sparse_decode_merged on
// the compute stream, and copies o and lse
// back on the download stream.  Slots alternate, so the upload of step k+1
// and the download of step k-1 run while step k computes.  Events order the
// three streams:
//   upload (k)    waits for compute (k-2), the last reader of the slot;
//   compute (k)   waits for upload (k) and for download (k-2), the last
//                 reader of the slot's o / lse;
//   download (k)  waits for compute (k).
// This file calls only the public entry points (qsa.h); the kernels and the
// per-device error word live in qsa_api.cu.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <new>

#include "qsa.h"

struct qsa_session {
  qsa_cache cache;
  int B, T, Hq, Hkv, D, d, q_dtype, topk, S, max_blocks, max_new_tokens;
  float sm_scale;
  size_t q_bytes;  // bytes of one step's q
  cudaStream_t compute = nullptr, h2d = nullptr, d2h = nullptr;
  bool own_compute = false;
  // per slot
  int32_t *pos0[2] = {}, *cu_new[2] = {}, *ctx_lens[2] = {}, *n_sel[2] = {};
  int8_t *k_new[2] = {}, *q_idx[2] = {};
  void *q[2] = {};
  float *o[2] = {}, *lse[2] = {};
  cudaEvent_t in_ready[2] = {}, compute_done[2] = {}, out_copied[2] = {};
  // shared by the steps (used by the compute stream in order)
  int32_t *sel = nullptr;
  float *o_part = nullptr, *lse_part = nullptr;
  void *ws_topk = nullptr, *ws_dec = nullptr;
  size_t ws_topk_bytes = 0, ws_dec_bytes = 0;
  long long steps = 0;
};

namespace {

template <typename T>
bool dev_alloc(T **p, size_t bytes) {
  void *v = nullptr;
  if (cudaMalloc(&v, std::max<size_t>(bytes, 16)) != cudaSuccess) return false;
  *p = static_cast<T *>(v);
  return true;
}

void release(qsa_session *s) {
  if (!s) return;
  for (cudaStream_t st : {s->h2d, s->d2h, s->compute})
    if (st) cudaStreamSynchronize(st);
  for (int k = 0; k < 2; ++k) {
    cudaFree(s->pos0[k]);
    cudaFree(s->cu_new[k]);
    cudaFree(s->ctx_lens[k]);
    cudaFree(s->n_sel[k]);
    cudaFree(s->k_new[k]);
    cudaFree(s->q_idx[k]);
    cudaFree(s->q[k]);
    cudaFree(s->o[k]);
    cudaFree(s->lse[k]);
    if (s->in_ready[k]) cudaEventDestroy(s->in_ready[k]);
    if (s->compute_done[k]) cudaEventDestroy(s->compute_done[k]);
    if (s->out_copied[k]) cudaEventDestroy(s->out_copied[k]);
  }
  cudaFree(s->sel);
  cudaFree(s->o_part);
  cudaFree(s->lse_part);
  cudaFree(s->ws_topk);
  cudaFree(s->ws_dec);
  if (s->h2d) cudaStreamDestroy(s->h2d);
  if (s->d2h) cudaStreamDestroy(s->d2h);
  if (s->own_compute && s->compute) cudaStreamDestroy(s->compute);
  delete s;
}

}  // namespace

extern "C" {

qsa_status qsa_session_create(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                              int32_t q_dtype, int32_t topk, int32_t num_splits,
                              int32_t max_blocks, int32_t max_new_tokens, float sm_scale,
                              qsa_stream_t compute_stream, qsa_session **out) {
  if (!out) return QSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!cache || B < 1 || T < 1 || Hq < 1 || topk < 1 || num_splits < 1 || max_blocks < 1 ||
      max_new_tokens < 1 || !(sm_scale > 0.f) || !std::isfinite(sm_scale))
    return QSA_ERR_INVALID_ARG;
  if (q_dtype != QSA_F32 && q_dtype != QSA_BF16) return QSA_ERR_INVALID_ARG;
  if (cache->num_kv_heads < 1 || cache->head_dim < 1 || cache->idx_dim < 1 ||
      Hq % cache->num_kv_heads != 0)
    return QSA_ERR_INVALID_ARG;
  qsa_session *s = new (std::nothrow) qsa_session();
  if (!s) return QSA_ERR_CUDA;
  s->cache = *cache;
  s->B = B;
  s->T = T;
  s->Hq = Hq;
  s->Hkv = cache->num_kv_heads;
  s->D = cache->head_dim;
  s->d = cache->idx_dim;
  s->q_dtype = q_dtype;
  s->topk = topk;
  s->S = num_splits;
  s->max_blocks = max_blocks;
  s->max_new_tokens = max_new_tokens;
  s->sm_scale = sm_scale;
  s->q_bytes = (size_t)B * T * Hq * s->D * (q_dtype == QSA_BF16 ? 2 : 4);
  const size_t rows = (size_t)B * T * Hq;
  bool ok = true;
  if (compute_stream) {
    s->compute = reinterpret_cast<cudaStream_t>(compute_stream);
  } else {
    ok = ok && cudaStreamCreateWithFlags(&s->compute, cudaStreamNonBlocking) == cudaSuccess;
    s->own_compute = ok;
  }
  ok = ok && cudaStreamCreateWithFlags(&s->h2d, cudaStreamNonBlocking) == cudaSuccess;
  ok = ok && cudaStreamCreateWithFlags(&s->d2h, cudaStreamNonBlocking) == cudaSuccess;
  for (int k = 0; k < 2 && ok; ++k) {
    ok = ok && dev_alloc(&s->pos0[k], (size_t)B * 4) && dev_alloc(&s->cu_new[k], (size_t)(B + 1) * 4);
    ok = ok && dev_alloc(&s->ctx_lens[k], (size_t)B * 4) && dev_alloc(&s->n_sel[k], (size_t)B * 4);
    ok = ok && dev_alloc(&s->k_new[k], (size_t)max_new_tokens * s->d);
    ok = ok && dev_alloc(&s->q_idx[k], (size_t)B * s->d) && dev_alloc(&s->q[k], s->q_bytes);
    ok = ok && dev_alloc(&s->o[k], rows * s->D * 4) && dev_alloc(&s->lse[k], rows * 4);
    for (cudaEvent_t *e : {&s->in_ready[k], &s->compute_done[k], &s->out_copied[k]})
      ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  }
  ok = ok && dev_alloc(&s->sel, (size_t)B * topk * 4);
  ok = ok && dev_alloc(&s->o_part, (size_t)num_splits * rows * s->D * 4);
  ok = ok && dev_alloc(&s->lse_part, (size_t)num_splits * rows * 4);
  s->ws_topk_bytes = qsa_index_topk_workspace_bytes(B, max_blocks);
  s->ws_dec_bytes = qsa_sparse_decode_workspace_bytes(B, T, Hq, s->Hkv, s->D, topk, num_splits);
  ok = ok && s->ws_topk_bytes > 0 && s->ws_dec_bytes > 0;
  ok = ok && dev_alloc(&s->ws_topk, s->ws_topk_bytes) && dev_alloc(&s->ws_dec, s->ws_dec_bytes);
  ok = ok && cudaMemset(s->ws_dec, 0, s->ws_dec_bytes) == cudaSuccess;
  ok = ok && cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    release(s);
    return QSA_ERR_CUDA;
  }
  *out = s;
  return QSA_OK;
}

qsa_status qsa_session_step_host(qsa_session *s, const int32_t *pos0, const int32_t *cu_new,
                                 const int8_t *k_new, const int8_t *q_idx, const void *q,
                                 const int32_t *ctx_lens, const int32_t *n_sel, float *o,
                                 float *lse) {
  if (!s || !pos0 || !cu_new || !k_new || !q_idx || !q || !ctx_lens || !o || !lse)
    return QSA_ERR_INVALID_ARG;
  const int B = s->B;
  // the per-request counts of new tokens are read on the host
  if (cu_new[0] != 0) return QSA_ERR_INVALID_ARG;
  int max_new = 0;
  for (int r = 0; r < B; ++r) {
    const int n = cu_new[r + 1] - cu_new[r];
    if (n < 0) return QSA_ERR_INVALID_ARG;
    max_new = std::max(max_new, n);
  }
  const int n_new = cu_new[B];
  if (n_new > s->max_new_tokens) return QSA_ERR_INVALID_ARG;
  const int k = (int)(s->steps & 1);
  const size_t rows = (size_t)B * s->T * s->Hq;
  bool ok = true;
  // upload into slot k once the compute that last read it has finished
  ok = ok && cudaStreamWaitEvent(s->h2d, s->compute_done[k], 0) == cudaSuccess;
  auto up = [&](void *dst, const void *src, size_t bytes) {
    ok = ok && (bytes == 0 || cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s->h2d) == cudaSuccess);
  };
  up(s->pos0[k], pos0, (size_t)B * 4);
  up(s->cu_new[k], cu_new, (size_t)(B + 1) * 4);
  up(s->k_new[k], k_new, (size_t)n_new * s->d);
  up(s->q_idx[k], q_idx, (size_t)B * s->d);
  up(s->q[k], q, s->q_bytes);
  up(s->ctx_lens[k], ctx_lens, (size_t)B * 4);
  if (n_sel) up(s->n_sel[k], n_sel, (size_t)B * 4);
  ok = ok && cudaEventRecord(s->in_ready[k], s->h2d) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  // compute once the inputs are in and the slot's previous outputs are out
  if (cudaStreamWaitEvent(s->compute, s->in_ready[k], 0) != cudaSuccess ||
      cudaStreamWaitEvent(s->compute, s->out_copied[k], 0) != cudaSuccess) {
    cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  qsa_stream_t cs = reinterpret_cast<qsa_stream_t>(s->compute);
  qsa_status st = qsa_compress_append(&s->cache, B, s->pos0[k], s->cu_new[k], s->k_new[k], max_new, cs);
  if (st == QSA_OK)
    st = qsa_index_topk(&s->cache, B, s->q_idx[k], s->ctx_lens[k], n_sel ? s->n_sel[k] : nullptr,
                        s->max_blocks, s->topk, s->sel, nullptr, s->ws_topk, s->ws_topk_bytes, cs);
  if (st == QSA_OK)
    st = qsa_sparse_decode_merged(&s->cache, B, s->T, s->Hq, s->q[k], s->q_dtype, s->ctx_lens[k],
                                  s->sel, s->topk, s->sm_scale, s->S, s->o_part, s->lse_part,
                                  s->o[k], s->lse[k], s->ws_dec, s->ws_dec_bytes, cs);
  if (st != QSA_OK) return st;
  // download once the step is computed
  ok = cudaEventRecord(s->compute_done[k], s->compute) == cudaSuccess;
  ok = ok && cudaStreamWaitEvent(s->d2h, s->compute_done[k], 0) == cudaSuccess;
  ok = ok && cudaMemcpyAsync(o, s->o[k], rows * s->D * 4, cudaMemcpyDeviceToHost, s->d2h) == cudaSuccess;
  ok = ok && cudaMemcpyAsync(lse, s->lse[k], rows * 4, cudaMemcpyDeviceToHost, s->d2h) == cudaSuccess;
  ok = ok && cudaEventRecord(s->out_copied[k], s->d2h) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  ++s->steps;
  return QSA_OK;
}

qsa_status qsa_session_streams(const qsa_session *s, qsa_stream_t *h2d, qsa_stream_t *compute,
                               qsa_stream_t *d2h) {
  if (!s) return QSA_ERR_INVALID_ARG;
  if (h2d) *h2d = reinterpret_cast<qsa_stream_t>(s->h2d);
  if (compute) *compute = reinterpret_cast<qsa_stream_t>(s->compute);
  if (d2h) *d2h = reinterpret_cast<qsa_stream_t>(s->d2h);
  return QSA_OK;
}

qsa_status qsa_session_synchronize(qsa_session *s) {
  if (!s) return QSA_ERR_INVALID_ARG;
  bool ok = true;
  for (cudaStream_t st : {s->h2d, s->compute, s->d2h}) ok = ok && cudaStreamSynchronize(st) == cudaSuccess;
  return ok ? QSA_OK : QSA_ERR_CUDA;
}

qsa_status qsa_session_destroy(qsa_session *s) {
  if (!s) return QSA_ERR_INVALID_ARG;
  release(s);
  return QSA_OK;
}

}  // extern "C"
