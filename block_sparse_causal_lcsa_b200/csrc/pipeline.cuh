// Native streaming pipeline (FlashVSR summary, section 3: the model runs as
// a stream, 8 video frames = 2 latent frames at a time, with a KV cache):
// chunks arrive in host memory and their outputs return there. One submit
// queues the upload of a chunk's Q, K, V, the streaming step (ingest, select,
// attention) and the read-back of O; the uploads of chunk i+1 and the
// read-back of chunk i-1 overlap the step of chunk i. Three streams (upload,
// compute, read-back) ordered by events only; two device input sets so an
// upload never overwrites inputs a step still reads; the one O buffer is
// rewritten only after the previous read-back has finished. The pipeline owns
// its device memory and advances the caller's cache state as each step is
// queued. Included into lcsa_api.cu (one translation unit).
#pragma once

struct lcsa_pipeline {
  int dev;
  lcsa_kv_cache* kv;
  int32_t q_frames;
  lcsa_select_params sp;
  int32_t token_window;                  // token-level window of the attention (0: none)
  size_t in_bytes, o_bytes;              // one chunk's Q (= K = V) and O in bytes
  void* in[2][3];                        // device Q, K, V of the two input sets
  double* q_pool;
  int32_t* blk_idx;
  int32_t* blk_cnt;
  void* sel_ws;
  size_t sel_ws_bytes;
  void* attn_ws;
  size_t attn_ws_bytes;
  void* o;
  float* lse;
  cudaStream_t up, comp, down;
  cudaEvent_t in_ready[2], step_done[2], out_free, t0, t1;
  bool step_pending[2], out_pending, timing;
  int64_t n;
};

namespace lcsa {
namespace {

// A contiguous [B][H][T][Y][X][D] bf16 tensor descriptor.
lcsa_tensor dense_tensor(void* data, int B, int H, int T, int Y, int X, int D) {
  lcsa_tensor t{};
  t.data = data;
  t.B = B; t.H = H; t.T = T; t.Y = Y; t.X = X; t.D = D;
  t.stride_x = D;
  t.stride_y = static_cast<int64_t>(X) * D;
  t.stride_t = t.stride_y * Y;
  t.stride_h = t.stride_t * T;
  t.stride_b = t.stride_h * H;
  return t;
}

void pipeline_free(lcsa_pipeline* pl) {
  if (pl == nullptr) return;
  for (auto& set : pl->in)
    for (void* ptr : set) cudaFree(ptr);
  cudaFree(pl->q_pool); cudaFree(pl->blk_idx); cudaFree(pl->blk_cnt); cudaFree(pl->sel_ws);
  cudaFree(pl->attn_ws); cudaFree(pl->o); cudaFree(pl->lse);
  for (cudaStream_t s : {pl->up, pl->comp, pl->down})
    if (s != nullptr) cudaStreamDestroy(s);
  for (cudaEvent_t e : {pl->in_ready[0], pl->in_ready[1], pl->step_done[0], pl->step_done[1], pl->out_free,
                        pl->t0, pl->t1})
    if (e != nullptr) cudaEventDestroy(e);
  delete pl;
}

}  // namespace
}  // namespace lcsa

extern "C" {

lcsa_status lcsa_pipeline_create(lcsa_kv_cache* kv, int32_t q_frames, const lcsa_select_params* params,
                                 lcsa_pipeline** out) {
  using namespace lcsa;
  if (out == nullptr) return LCSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (params == nullptr) return LCSA_ERR_INVALID_ARG;
  lcsa_status s = check_cache(kv);
  if (s != LCSA_OK) return s;
  if (q_frames < 1 || q_frames > kv->cap_frames) return LCSA_ERR_SHAPE;
  if (params->window < 0 || params->window_mode < 0 || params->window_mode > LCSA_WINDOW_PRESERVE_TOKENS)
    return LCSA_ERR_INVALID_ARG;
  // capacity for the fullest cache state a step can see
  lcsa_kv_cache full = *kv;
  for (int b = 0; b < kv->B; ++b) {
    full.begin[b] = 0;
    full.end[b] = kv->cap_frames;
  }
  lcsa_select_params sp = *params;
  sp.kmax = lcsa_select_kmax(&full, q_frames, params);
  if (sp.kmax < 1) return LCSA_ERR_SHAPE;
  const size_t sel_ws = lcsa_select_workspace_bytes(&full, q_frames);
  if (sel_ws == 0) return LCSA_ERR_SHAPE;

  lcsa_pipeline* pl = new lcsa_pipeline{};
  if (cudaGetDevice(&pl->dev) != cudaSuccess) {
    delete pl;
    return LCSA_ERR_CUDA;
  }
  pl->kv = kv;
  pl->q_frames = q_frames;
  pl->sp = sp;
  pl->token_window = params->window_mode >= LCSA_WINDOW_TRUNCATE_TOKENS ? params->window : 0;
  const int B = kv->B, H = kv->H, Y = kv->Y, X = kv->X, D = kv->D;
  const int nQT = temporal_blocks(q_frames);
  const size_t nQB = static_cast<size_t>(nQT) * (Y / 8) * (X / 8);
  pl->in_bytes = static_cast<size_t>(B) * H * q_frames * Y * X * D * sizeof(__nv_bfloat16);
  pl->o_bytes = pl->in_bytes;
  pl->sel_ws_bytes = sel_ws;
  pl->attn_ws_bytes = lcsa_sparse_attn_fwd_workspace_bytes(D);
  bool ok = true;
  for (auto& set : pl->in)
    for (void*& ptr : set) ok = ok && cudaMalloc(&ptr, pl->in_bytes) == cudaSuccess;
  ok = ok && cudaMalloc(reinterpret_cast<void**>(&pl->q_pool), static_cast<size_t>(B) * H * nQB * D * sizeof(double)) ==
                 cudaSuccess;
  ok = ok && cudaMalloc(reinterpret_cast<void**>(&pl->blk_idx), static_cast<size_t>(B) * H * nQB * sp.kmax *
                                                                    sizeof(int32_t)) == cudaSuccess;
  ok = ok && cudaMalloc(reinterpret_cast<void**>(&pl->blk_cnt), static_cast<size_t>(B) * H * nQB * sizeof(int32_t)) ==
                 cudaSuccess;
  ok = ok && cudaMalloc(&pl->sel_ws, pl->sel_ws_bytes) == cudaSuccess;
  ok = ok && cudaMalloc(&pl->attn_ws, pl->attn_ws_bytes) == cudaSuccess;
  ok = ok && cudaMalloc(&pl->o, pl->o_bytes) == cudaSuccess;
  ok = ok && cudaMalloc(reinterpret_cast<void**>(&pl->lse), static_cast<size_t>(B) * H * q_frames * Y * X *
                                                                sizeof(float)) == cudaSuccess;
  for (cudaStream_t* st : {&pl->up, &pl->comp, &pl->down})
    ok = ok && cudaStreamCreateWithFlags(st, cudaStreamNonBlocking) == cudaSuccess;
  for (cudaEvent_t* e : {&pl->in_ready[0], &pl->in_ready[1], &pl->step_done[0], &pl->step_done[1], &pl->out_free})
    ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  ok = ok && cudaEventCreate(&pl->t0) == cudaSuccess && cudaEventCreate(&pl->t1) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    pipeline_free(pl);
    return LCSA_ERR_CUDA;
  }
  *out = pl;
  return LCSA_OK;
}

lcsa_status lcsa_pipeline_submit(lcsa_pipeline* pl, const void* q_host, const void* k_host, const void* v_host,
                                 void* o_host) {
  using namespace lcsa;
  if (pl == nullptr || q_host == nullptr || k_host == nullptr || v_host == nullptr || o_host == nullptr)
    return LCSA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != pl->dev) return LCSA_ERR_INVALID_ARG;
  const int slot = static_cast<int>(pl->n & 1);
  const lcsa_kv_cache* kv = pl->kv;
  const int B = kv->B, H = kv->H, Y = kv->Y, X = kv->X, D = kv->D, T = pl->q_frames;
  lcsa_tensor tq = dense_tensor(pl->in[slot][0], B, H, T, Y, X, D);
  lcsa_tensor tk = dense_tensor(pl->in[slot][1], B, H, T, Y, X, D);
  lcsa_tensor tv = dense_tensor(pl->in[slot][2], B, H, T, Y, X, D);
  lcsa_tensor to = dense_tensor(pl->o, B, H, T, Y, X, D);
  // upload: into the input set whose previous step has finished reading it
  if (pl->timing) {
    if (cudaEventRecord(pl->t0, pl->up) != cudaSuccess) return LCSA_ERR_CUDA;
    pl->timing = false;
  }
  if (pl->step_pending[slot] && cudaStreamWaitEvent(pl->up, pl->step_done[slot], 0) != cudaSuccess)
    return LCSA_ERR_CUDA;
  const void* src[3] = {q_host, k_host, v_host};
  for (int i = 0; i < 3; ++i)
    if (cudaMemcpyAsync(pl->in[slot][i], src[i], pl->in_bytes, cudaMemcpyHostToDevice, pl->up) != cudaSuccess)
      return LCSA_ERR_CUDA;
  if (cudaEventRecord(pl->in_ready[slot], pl->up) != cudaSuccess) return LCSA_ERR_CUDA;
  // step: once its inputs have landed and O has been read back
  if (cudaStreamWaitEvent(pl->comp, pl->in_ready[slot], 0) != cudaSuccess) return LCSA_ERR_CUDA;
  if (pl->out_pending && cudaStreamWaitEvent(pl->comp, pl->out_free, 0) != cudaSuccess) return LCSA_ERR_CUDA;
  lcsa_status s = lcsa_ingest_chunk(&tq, pl->q_pool, pl->kv, &tk, &tv, 0, pl->comp);
  if (s != LCSA_OK) return s;
  s = lcsa_select_blocks(pl->q_pool, pl->q_frames, pl->kv, &pl->sp, pl->blk_idx, pl->blk_cnt, pl->sel_ws,
                         pl->sel_ws_bytes, pl->comp);
  if (s != LCSA_OK) return s;
  s = lcsa_sparse_attn_fwd_ex(&tq, pl->kv, pl->blk_idx, pl->blk_cnt, pl->sp.kmax, pl->token_window,
                              pl->token_window > 0 ? pl->sp.window_mode : LCSA_WINDOW_TRUNCATE_TOKENS, &to, pl->lse,
                              pl->attn_ws, pl->attn_ws_bytes, pl->comp);
  if (s != LCSA_OK) return s;
  if (cudaEventRecord(pl->step_done[slot], pl->comp) != cudaSuccess) return LCSA_ERR_CUDA;
  pl->step_pending[slot] = true;
  // read-back of O
  if (cudaStreamWaitEvent(pl->down, pl->step_done[slot], 0) != cudaSuccess ||
      cudaMemcpyAsync(o_host, pl->o, pl->o_bytes, cudaMemcpyDeviceToHost, pl->down) != cudaSuccess ||
      cudaEventRecord(pl->out_free, pl->down) != cudaSuccess || cudaEventRecord(pl->t1, pl->down) != cudaSuccess)
    return LCSA_ERR_CUDA;
  pl->out_pending = true;
  ++pl->n;
  return LCSA_OK;
}

lcsa_status lcsa_pipeline_sync(lcsa_pipeline* pl) {
  if (pl == nullptr) return LCSA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(pl->up) != cudaSuccess || cudaStreamSynchronize(pl->comp) != cudaSuccess ||
      cudaStreamSynchronize(pl->down) != cudaSuccess)
    return LCSA_ERR_CUDA;
  return lcsa_last_device_error(pl->comp);
}

lcsa_status lcsa_pipeline_start_timer(lcsa_pipeline* pl) {
  if (pl == nullptr) return LCSA_ERR_INVALID_ARG;
  pl->timing = true;
  return LCSA_OK;
}

lcsa_status lcsa_pipeline_elapsed_ms(lcsa_pipeline* pl, float* ms) {
  if (pl == nullptr || ms == nullptr || pl->timing) return LCSA_ERR_INVALID_ARG;
  if (cudaEventSynchronize(pl->t1) != cudaSuccess || cudaEventElapsedTime(ms, pl->t0, pl->t1) != cudaSuccess)
    return LCSA_ERR_CUDA;
  return LCSA_OK;
}

void lcsa_pipeline_destroy(lcsa_pipeline* pl) {
  if (pl == nullptr) return;
  cudaStreamSynchronize(pl->up);
  cudaStreamSynchronize(pl->comp);
  cudaStreamSynchronize(pl->down);
  lcsa::pipeline_free(pl);
}

}  // extern "C"
