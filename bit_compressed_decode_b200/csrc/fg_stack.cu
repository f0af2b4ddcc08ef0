// fg_stack.cu -- a stack of layers whose 4-bit weight blobs live in (pinned) host memory.
//
// "FlexGen Guide: High-Throughput LLM Offloading on One GPU", sections 1 and 2: the
// weights sit in CPU memory and move to the GPU layer by layer; a loaded layer is used
// for every batch of the block before the next one.  Here two device staging buffers
// alternate: while layer l computes from buffer l%2 on the compute stream, the copy
// stream moves layer l+1's blob into the other buffer with one cudaMemcpyAsync.  Two
// events per buffer order the streams: `ready` (copy done -> compute may start) and
// `done` (compute done -> the buffer may be overwritten).
#include <stdlib.h>

#include <new>
#include <vector>

#include "fg_internal.cuh"

struct fg_stack {
  fg_layer_config cfg;
  int num_layers;
  std::vector<void *> host;
  void *staging[2];
  cudaEvent_t ready[2], done[2];
  size_t blob_bytes;
  int inject_failures;
};

namespace {

fg_status stack_run(fg_stack *st, const fg_kv_cache *kv, const fg_half *x_in, fg_half *x_out,
                    const int32_t *positions, int prompt_len, int nb, int gbs, void *workspace, size_t ws_bytes,
                    cudaStream_t cs, cudaStream_t ps) {
  if (!st || !kv) return FG_ERR_INVALID;
  const int S = nb * gbs;
  if (S == 0) return FG_OK;
  if (!workspace || !fg_aligned16(workspace) || !x_in || !x_out) return FG_ERR_INVALID;
  // workspace: two ping-pong activation buffers, then the layer's own scratch
  const size_t rows = static_cast<size_t>(S) * (prompt_len > 0 ? prompt_len : 1);
  const size_t act = ((rows * st->cfg.hidden * 2) + 255) & ~size_t(255);
  if (ws_bytes < 2 * act) return FG_ERR_WORKSPACE;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  fg_half *buf[2] = {reinterpret_cast<fg_half *>(ws), reinterpret_cast<fg_half *>(ws + act)};
  void *lws = ws + 2 * act;
  const size_t lws_bytes = ws_bytes - 2 * act;

  fg_status rc = FG_OK;
  auto prefetch = [&](int l) -> fg_status {
    const int b = l & 1;
    if (st->inject_failures > 0) {
      st->inject_failures--;
      return FG_ERR_CUDA;
    }
    fg_status r = fg_cuda_check(cudaStreamWaitEvent(ps, st->done[b], 0));
    if (r != FG_OK) return r;
    r = fg_cuda_check(cudaMemcpyAsync(st->staging[b], st->host[l], st->blob_bytes, cudaMemcpyHostToDevice, ps));
    if (r != FG_OK) return r;
    return fg_cuda_check(cudaEventRecord(st->ready[b], ps));
  };

  rc = prefetch(0);
  for (int l = 0; rc == FG_OK && l < st->num_layers; l++) {
    const int b = l & 1;
    if (l + 1 < st->num_layers && (rc = prefetch(l + 1)) != FG_OK) break;
    if ((rc = fg_cuda_check(cudaStreamWaitEvent(cs, st->ready[b], 0))) != FG_OK) break;
    fg_layer_weights w;
    if ((rc = fg_layer_weights_from_blob(&st->cfg, st->staging[b], &w)) != FG_OK) break;
    const fg_half *in = l == 0 ? x_in : buf[(l - 1) & 1];
    fg_half *out = l == st->num_layers - 1 ? x_out : buf[l & 1];
    if (prompt_len > 0)
      rc = fg_layer_prefill(&st->cfg, &w, &kv[l], in, out, positions, prompt_len, nb, gbs, lws, lws_bytes, cs);
    else
      rc = fg_layer_decode(&st->cfg, &w, &kv[l], in, out, positions, nb, gbs, lws, lws_bytes, cs);
    if (rc != FG_OK) break;
    if ((rc = fg_cuda_check(cudaEventRecord(st->done[b], cs))) != FG_OK) break;
  }
  if (rc != FG_OK) {
    // drain what was enqueued so nothing is left waiting on this stack's buffers
    cudaStreamSynchronize(ps);
    cudaStreamSynchronize(cs);
  }
  return rc;
}

}  // namespace

extern "C" fg_status fg_stack_create(const fg_layer_config *c, int num_layers, void *const *host_blobs,
                                     void *dev_staging0, void *dev_staging1, fg_stack **out) {
  if (!out) return FG_ERR_INVALID;
  *out = nullptr;
  const size_t bytes = fg_layer_blob_bytes(c);
  if (bytes == 0) return FG_ERR_UNSUPPORTED;
  if (num_layers < 1 || !host_blobs || !dev_staging0 || !dev_staging1) return FG_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(dev_staging0) & 255) || (reinterpret_cast<uintptr_t>(dev_staging1) & 255))
    return FG_ERR_INVALID;
  for (int l = 0; l < num_layers; l++)
    if (!host_blobs[l]) return FG_ERR_INVALID;
  fg_stack *st = new (std::nothrow) fg_stack;
  if (!st) return FG_ERR_INVALID;
  st->cfg = *c;
  st->num_layers = num_layers;
  st->host.assign(host_blobs, host_blobs + num_layers);
  st->staging[0] = dev_staging0;
  st->staging[1] = dev_staging1;
  st->blob_bytes = bytes;
  st->inject_failures = 0;
  for (int i = 0; i < 2; i++) {
    st->ready[i] = st->done[i] = nullptr;
  }
  for (int i = 0; i < 2; i++) {
    if (fg_cuda_check(cudaEventCreateWithFlags(&st->ready[i], cudaEventDisableTiming)) != FG_OK ||
        fg_cuda_check(cudaEventCreateWithFlags(&st->done[i], cudaEventDisableTiming)) != FG_OK) {
      fg_stack_destroy(st);
      return FG_ERR_CUDA;
    }
  }
  *out = st;
  return FG_OK;
}

extern "C" fg_status fg_stack_decode(fg_stack *st, const fg_kv_cache *kv, const fg_half *x_in, fg_half *x_out,
                                     const int32_t *positions, int num_gpu_batches, int gpu_batch_size,
                                     void *workspace, size_t workspace_bytes, void *compute_stream,
                                     void *copy_stream) {
  return stack_run(st, kv, x_in, x_out, positions, 0, num_gpu_batches, gpu_batch_size, workspace, workspace_bytes,
                   static_cast<cudaStream_t>(compute_stream), static_cast<cudaStream_t>(copy_stream));
}

extern "C" fg_status fg_stack_prefill(fg_stack *st, const fg_kv_cache *kv, const fg_half *x_in, fg_half *x_out,
                                      const int32_t *positions, int prompt_len, int num_gpu_batches,
                                      int gpu_batch_size, void *workspace, size_t workspace_bytes,
                                      void *compute_stream, void *copy_stream) {
  if (prompt_len < 1) return FG_ERR_SHAPE;
  return stack_run(st, kv, x_in, x_out, positions, prompt_len, num_gpu_batches, gpu_batch_size, workspace,
                   workspace_bytes, static_cast<cudaStream_t>(compute_stream),
                   static_cast<cudaStream_t>(copy_stream));
}

extern "C" fg_status fg_stack_inject_copy_failure(fg_stack *st, int count) {
  if (!st || count < 0) return FG_ERR_INVALID;
  st->inject_failures = count;
  return FG_OK;
}

extern "C" fg_status fg_stack_destroy(fg_stack *st) {
  if (!st) return FG_ERR_INVALID;
  for (int i = 0; i < 2; i++) {
    if (st->ready[i]) cudaEventDestroy(st->ready[i]);
    if (st->done[i]) cudaEventDestroy(st->done[i]);
  }
  delete st;
  return FG_OK;
}
