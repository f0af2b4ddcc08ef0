// fg_stack.cu -- a stack of layers whose 4-bit weight blobs live in (pinned) host memory.
//
// "FlexGen Guide: High-Throughput LLM Offloading on One GPU", sections 1 and 2: the
// weights sit in CPU memory and move to the GPU layer by layer; a loaded layer is used
// for every batch of the block before the next one.  Here two device staging buffers
// alternate: while layer l computes from buffer l%2 on the compute stream, the copy
// stream moves layer l+1's blob into the other buffer with one cudaMemcpyAsync.  Two
// events per buffer order the streams: `ready` (copy done -> compute may start) and
// `done` (compute done -> the buffer may be overwritten).  For caches larger than HBM
// (a 175B-class stack), fg_stack_decode_host_kv keeps every layer's 4-bit KV cache in
// pinned host memory too: the copy stream fills a device KV staging cache with the layer's
// cached positions next to its blob, and writes only the new token slots back after the
// layer (the pages' guide, section 2: KV cache offloaded alongside the weights).
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
  cudaEvent_t kv_back[2];  // host-KV decode: write-back from KV staging cache b done
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


bool same_geometry(const fg_kv_cache &a, const fg_kv_cache &b) {
  return a.num_seqs == b.num_seqs && a.num_heads == b.num_heads && a.head_dim == b.head_dim &&
         a.max_len == b.max_len && fg_kv_group(a.group) == fg_kv_group(b.group);
}

// Positions [p0, p1) of every (sequence, head) row of the six cache arrays, src -> dst,
// as one strided 2-D copy per array (rows of max_len slots).
fg_status kv_copy(const fg_kv_cache &dst, const fg_kv_cache &src, int p0, int p1, cudaMemcpyKind kind,
                  cudaStream_t s) {
  if (p1 <= p0) return FG_OK;
  const size_t rows = static_cast<size_t>(src.num_seqs) * src.num_heads;
  const size_t cpos = src.head_dim / 2, mpos = (src.head_dim / fg_kv_group(src.group)) * 2;  // bytes per slot
  const size_t n = static_cast<size_t>(p1 - p0);
  struct Arr {
    void *d;
    const void *s;
    size_t per;
  } arrs[6] = {{dst.k_codes, src.k_codes, cpos}, {dst.k_mins, src.k_mins, mpos}, {dst.k_scales, src.k_scales, mpos},
               {dst.v_codes, src.v_codes, cpos}, {dst.v_mins, src.v_mins, mpos}, {dst.v_scales, src.v_scales, mpos}};
  for (const Arr &x : arrs) {
    const size_t pitch = static_cast<size_t>(src.max_len) * x.per, off = static_cast<size_t>(p0) * x.per;
    fg_status r = fg_cuda_check(cudaMemcpy2DAsync(static_cast<uint8_t *>(x.d) + off, pitch,
                                                  static_cast<const uint8_t *>(x.s) + off, pitch, n * x.per, rows, kind,
                                                  s));
    if (r != FG_OK) return r;
  }
  return FG_OK;
}

// Decode with every layer's KV cache in pinned host memory: per layer, the copy stream moves
// the weight blob and positions [0, fill_len) of the cache into staging buffer l%2 (device
// KV staging cache dev_kv[l%2]), the layer runs on the staged cache, and the copy stream
// writes positions [wb_begin, wb_end) back to the host cache once the layer is done.
fg_status stack_run_host_kv(fg_stack *st, const fg_kv_cache *host_kv, const fg_kv_cache *dev_kv, int fill_len,
                            int wb_begin, int wb_end, const fg_half *x_in, fg_half *x_out, const int32_t *positions,
                            int nb, int gbs, void *workspace, size_t ws_bytes, cudaStream_t cs, cudaStream_t ps) {
  if (!st || !host_kv || !dev_kv) return FG_ERR_INVALID;
  const int S = nb * gbs;
  if (S == 0) return FG_OK;
  if (!workspace || !fg_aligned16(workspace) || !x_in || !x_out) return FG_ERR_INVALID;
  if (!same_geometry(dev_kv[0], dev_kv[1])) return FG_ERR_SHAPE;
  for (int l = 0; l < st->num_layers; l++)
    if (!same_geometry(host_kv[l], dev_kv[0])) return FG_ERR_SHAPE;
  const int maxL = dev_kv[0].max_len;
  if (fill_len < 0 || fill_len > maxL || wb_begin < 0 || wb_begin > wb_end || wb_end > maxL) return FG_ERR_INVALID;
  if (S > dev_kv[0].num_seqs) return FG_ERR_SHAPE;
  const size_t act = ((static_cast<size_t>(S) * st->cfg.hidden * 2) + 255) & ~size_t(255);
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
    if (r == FG_OK) r = fg_cuda_check(cudaStreamWaitEvent(ps, st->kv_back[b], 0));
    if (r == FG_OK)
      r = fg_cuda_check(cudaMemcpyAsync(st->staging[b], st->host[l], st->blob_bytes, cudaMemcpyHostToDevice, ps));
    if (r == FG_OK) r = kv_copy(dev_kv[b], host_kv[l], 0, fill_len, cudaMemcpyHostToDevice, ps);
    if (r == FG_OK) r = fg_cuda_check(cudaEventRecord(st->ready[b], ps));
    return r;
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
    if ((rc = fg_layer_decode(&st->cfg, &w, &dev_kv[b], in, out, positions, nb, gbs, lws, lws_bytes, cs)) != FG_OK)
      break;
    if ((rc = fg_cuda_check(cudaEventRecord(st->done[b], cs))) != FG_OK) break;
    // write the new slots back to the host cache, after the layer, on the copy stream
    if ((rc = fg_cuda_check(cudaStreamWaitEvent(ps, st->done[b], 0))) != FG_OK) break;
    if ((rc = kv_copy(host_kv[l], dev_kv[b], wb_begin, wb_end, cudaMemcpyDeviceToHost, ps)) != FG_OK) break;
    if ((rc = fg_cuda_check(cudaEventRecord(st->kv_back[b], ps))) != FG_OK) break;
  }
  // the step ends on the compute stream only once the last write-back has landed
  if (rc == FG_OK) rc = fg_cuda_check(cudaStreamWaitEvent(cs, st->kv_back[(st->num_layers - 1) & 1], 0));
  if (rc != FG_OK) {
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
    st->ready[i] = st->done[i] = st->kv_back[i] = nullptr;
  }
  for (int i = 0; i < 2; i++) {
    if (fg_cuda_check(cudaEventCreateWithFlags(&st->ready[i], cudaEventDisableTiming)) != FG_OK ||
        fg_cuda_check(cudaEventCreateWithFlags(&st->done[i], cudaEventDisableTiming)) != FG_OK ||
        fg_cuda_check(cudaEventCreateWithFlags(&st->kv_back[i], cudaEventDisableTiming)) != FG_OK) {
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

extern "C" fg_status fg_stack_decode_host_kv(fg_stack *st, const fg_kv_cache *host_kv, const fg_kv_cache *dev_kv,
                                             int fill_len, int wb_begin, int wb_end, const fg_half *x_in,
                                             fg_half *x_out, const int32_t *positions, int num_gpu_batches,
                                             int gpu_batch_size, void *workspace, size_t workspace_bytes,
                                             void *compute_stream, void *copy_stream) {
  return stack_run_host_kv(st, host_kv, dev_kv, fill_len, wb_begin, wb_end, x_in, x_out, positions, num_gpu_batches,
                           gpu_batch_size, workspace, workspace_bytes, static_cast<cudaStream_t>(compute_stream),
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
    if (st->kv_back[i]) cudaEventDestroy(st->kv_back[i]);
  }
  delete st;
  return FG_OK;
}
