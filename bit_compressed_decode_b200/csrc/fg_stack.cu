// fg_stack.cu -- a stack of layers whose 4-bit weight blobs live in (pinned) host memory.
//
// "FlexGen Guide: High-Throughput LLM Offloading on One GPU", sections 1 and 2: the
// weights sit in CPU memory and move to the GPU layer by layer; a loaded layer is used
// for every batch of the block before the next one.  Here two device staging buffers
// alternate: while layer l computes from buffer l%2 on the compute stream, the copy
// stream moves layer l+1's blob into the other buffer.  The blob moves in slices, in the
// order a layer step reads them -- its vectors, wqkv, wo, w1, w2 -- with one pair of events
// per slice and buffer: `ready` (slice copied -> the kernels that read it may run) and
// `done` (those kernels enqueued before it -> the slice may be overwritten).  So a layer's
// QKV GEMM starts once wqkv has landed while wo, w1 and w2 are still crossing the link
// (the weight loader that slices weights across batches, TightLLM abstract; the
// fine-grained offloading pipeline of PIPO, abstract).
// With one staging buffer (fg_stack_create given the same buffer twice, of
// fg_stack_one_buffer_bytes) each matrix of layer l+1 waits for layer l's kernels that read
// the same matrix: about half the staging memory.  The vectors (biases, LayerNorm parameters),
// needed first and last by a layer, alternate between the blob's vector slot and a second
// one after the blob, so layer l+1's vectors never wait for layer l's last GEMM.
// A layer whose blob the caller placed in device memory stays resident: it is read in place,
// with no copy and no staging buffer (the FlexGen guide's placement of part of the weights on
// the GPU, section 1; with 180 GB of HBM most of a 175B model's 4-bit weights fit).
// For caches larger than HBM (a 175B-class stack), fg_stack_decode_host_kv keeps every
// layer's 4-bit KV cache in pinned host memory too: the copy stream fills a device KV staging
// cache with the layer's cached positions next to its blob, and writes only the new token
// slots back after the layer (the pages' guide, section 2: KV cache offloaded alongside the
// weights).
#include <stdlib.h>

#include <new>
#include <vector>

#include "fg_internal.cuh"

struct fg_stack {
  fg_layer_config cfg;
  int num_layers;
  std::vector<void *> host;
  std::vector<char> resident;  // 1: blob l is in device memory and is read in place
  void *staging[2];
  int nbuf;  // 2: layers alternate between the two staging buffers; 1: one buffer (staging[0])
  // per staging buffer: the layer-step slice events (see fg_layer_slices; entry 2 is the
  // host-KV staging cache), and the host-KV write-back from KV staging cache b
  fg_layer_slices ev[2];
  cudaEvent_t kv_back[2];
  size_t sbegin[5], send[5];  // blob slices: vectors, wqkv, wo, w1, w2
  size_t blob_bytes;
  int inject_failures;
};

namespace {

// layer-step event index of blob slice i (vectors, wqkv, wo, w1, w2)
constexpr int kSliceEvent[5] = {0, 1, 3, 4, 5};

// The staging of layer l: buffer, its events, and where its vectors go.  One buffer: the
// matrices use staging[0] and ev[0]; the vectors of odd layers sit after the blob and use
// ev[1]'s vector events.
struct Staging {
  uint8_t *blob;
  fg_layer_slices ev;   // the events the layer step uses
  size_t vec_shift;     // added to the blob's vector offsets
  int evb;              // the ev[] entry of the matrices (and of the vectors when vec_ev < 0)
  int vec_ev;           // the ev[] entry of the vectors
};

Staging staging_of(const fg_stack *st, int l) {
  Staging g;
  if (st->nbuf == 2) {
    const int b = l & 1;
    g.blob = static_cast<uint8_t *>(st->staging[b]);
    g.ev = st->ev[b];
    g.vec_shift = 0;
    g.evb = g.vec_ev = b;
  } else {
    g.blob = static_cast<uint8_t *>(st->staging[0]);
    g.ev = st->ev[0];
    g.evb = 0;
    g.vec_ev = l & 1;
    g.ev.ready[0] = st->ev[g.vec_ev].ready[0];
    g.ev.done[0] = st->ev[g.vec_ev].done[0];
    g.vec_shift = (l & 1) ? st->blob_bytes - st->sbegin[0] : 0;
  }
  return g;
}

// Copies layer l's blob into staging buffer l % 2, slice by slice, on the copy stream: each
// slice waits until the layer that used the buffer before is done with it.  With a KV fill
// (host-KV decode), the fill goes after wqkv, before wo.
fg_status prefetch_sliced(fg_stack *st, int l, cudaStream_t ps, const fg_kv_cache *fill_dst,
                          const fg_kv_cache *fill_src, int fill_len);

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

  fg_status rc = prefetch_sliced(st, 0, ps, nullptr, nullptr, 0);
  for (int l = 0; rc == FG_OK && l < st->num_layers; l++) {
    const Staging g = staging_of(st, l);
    // two buffers: layer l+1's copies are enqueued first (they wait only for layer l-1);
    // one buffer: after layer l's kernels, whose `done` events the copies then wait for
    if (st->nbuf == 2 && l + 1 < st->num_layers && (rc = prefetch_sliced(st, l + 1, ps, nullptr, nullptr, 0)) != FG_OK)
      break;
    const bool res = st->resident[l];
    fg_layer_weights w;
    if ((rc = fg_layer_weights_from_blob(&st->cfg, res ? st->host[l] : g.blob, &w)) != FG_OK) break;
    if (!res) {
      fg_half **vecs[8] = {&w.bqkv, &w.bo, &w.b1, &w.b2, &w.ln1_g, &w.ln1_b, &w.ln2_g, &w.ln2_b};
      for (fg_half **v : vecs) *v = reinterpret_cast<fg_half *>(reinterpret_cast<uint8_t *>(*v) + g.vec_shift);
    }
    const fg_half *in = l == 0 ? x_in : buf[(l - 1) & 1];
    fg_half *out = l == st->num_layers - 1 ? x_out : buf[l & 1];
    if (prompt_len > 0) {
      // a prompt step waits for the whole blob (its chunks reuse every slice), then frees it
      for (int i = 0; i < 6 && rc == FG_OK && !res; i++)
        if (g.ev.ready[i] && i != 2) rc = fg_cuda_check(cudaStreamWaitEvent(cs, g.ev.ready[i], 0));
      if (rc == FG_OK)
        rc = fg_layer_prefill(&st->cfg, &w, &kv[l], in, out, positions, prompt_len, nb, gbs, lws, lws_bytes, cs);
      for (int i = 0; i < 6 && rc == FG_OK && !res; i++)
        if (i != 2) rc = fg_cuda_check(cudaEventRecord(g.ev.done[i], cs));
    } else if (res) {
      rc = fg_layer_decode_sliced(&st->cfg, &w, &kv[l], in, out, positions, nb, gbs, lws, lws_bytes, cs, nullptr);
    } else {
      fg_layer_slices sl = g.ev;
      sl.ready[2] = sl.done[2] = nullptr;  // the cache is resident
      rc = fg_layer_decode_sliced(&st->cfg, &w, &kv[l], in, out, positions, nb, gbs, lws, lws_bytes, cs, &sl);
    }
    if (rc == FG_OK && st->nbuf == 1 && l + 1 < st->num_layers) rc = prefetch_sliced(st, l + 1, ps, nullptr, nullptr, 0);
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
  if (st->nbuf != 2) return FG_ERR_UNSUPPORTED;  // the KV staging caches alternate with the blobs
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

  fg_status rc = prefetch_sliced(st, 0, ps, &dev_kv[0], &host_kv[0], fill_len);
  for (int l = 0; rc == FG_OK && l < st->num_layers; l++) {
    const int b = l & 1;
    if (l + 1 < st->num_layers &&
        (rc = prefetch_sliced(st, l + 1, ps, &dev_kv[(l + 1) & 1], &host_kv[l + 1], fill_len)) != FG_OK)
      break;
    const bool res = st->resident[l];
    fg_layer_weights w;
    if ((rc = fg_layer_weights_from_blob(&st->cfg, res ? st->host[l] : st->staging[b], &w)) != FG_OK) break;
    const fg_half *in = l == 0 ? x_in : buf[(l - 1) & 1];
    fg_half *out = l == st->num_layers - 1 ? x_out : buf[l & 1];
    fg_layer_slices sl = st->ev[b];
    if (res) {  // weights in place: only the KV staging cache's events
      for (int i = 0; i < 6; i++)
        if (i != 2) sl.ready[i] = sl.done[i] = nullptr;
    }
    if ((rc = fg_layer_decode_sliced(&st->cfg, &w, &dev_kv[b], in, out, positions, nb, gbs, lws, lws_bytes, cs,
                                     &sl)) != FG_OK)
      break;
    // write the new slots back to the host cache once the layer's attention is done, on the copy stream
    if ((rc = fg_cuda_check(cudaStreamWaitEvent(ps, st->ev[b].done[2], 0))) != FG_OK) break;
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

fg_status prefetch_sliced(fg_stack *st, int l, cudaStream_t ps, const fg_kv_cache *fill_dst,
                          const fg_kv_cache *fill_src, int fill_len) {
  const int b = l & 1;  // the KV staging cache and its write-back event (two buffers only)
  if (st->inject_failures > 0) {
    st->inject_failures--;
    return FG_ERR_CUDA;
  }
  const Staging g = staging_of(st, l);
  const uint8_t *src = static_cast<const uint8_t *>(st->host[l]);
  fg_layer_slices &ev = st->ev[g.evb];
  if (st->resident[l]) {  // weights in place; the layer's KV cache still goes to its staging cache
    if (!fill_dst) return FG_OK;
    fg_status r = fg_cuda_check(cudaStreamWaitEvent(ps, ev.done[2], 0));
    if (r == FG_OK) r = fg_cuda_check(cudaStreamWaitEvent(ps, st->kv_back[b], 0));
    if (r == FG_OK) r = kv_copy(*fill_dst, *fill_src, 0, fill_len, cudaMemcpyHostToDevice, ps);
    if (r == FG_OK) r = fg_cuda_check(cudaEventRecord(ev.ready[2], ps));
    return r;
  }
  for (int i = 0; i < 5; i++) {
    const int e = kSliceEvent[i];
    const size_t shift = i == 0 ? g.vec_shift : 0;
    cudaEvent_t ready = i == 0 ? st->ev[g.vec_ev].ready[0] : ev.ready[e];
    cudaEvent_t done = i == 0 ? st->ev[g.vec_ev].done[0] : ev.done[e];
    fg_status r = fg_cuda_check(cudaStreamWaitEvent(ps, done, 0));
    if (r == FG_OK)
      r = fg_cuda_check(cudaMemcpyAsync(g.blob + st->sbegin[i] + shift, src + st->sbegin[i],
                                        st->send[i] - st->sbegin[i], cudaMemcpyHostToDevice, ps));
    if (r == FG_OK) r = fg_cuda_check(cudaEventRecord(ready, ps));
    if (r != FG_OK) return r;
    if (i == 1 && fill_dst) {
      // the layer's KV cache: after the previous layer on this staging cache is done with it
      // (its attention) and has written its new slots back
      r = fg_cuda_check(cudaStreamWaitEvent(ps, ev.done[2], 0));
      if (r == FG_OK) r = fg_cuda_check(cudaStreamWaitEvent(ps, st->kv_back[b], 0));
      if (r == FG_OK) r = kv_copy(*fill_dst, *fill_src, 0, fill_len, cudaMemcpyHostToDevice, ps);
      if (r == FG_OK) r = fg_cuda_check(cudaEventRecord(ev.ready[2], ps));
      if (r != FG_OK) return r;
    }
  }
  return FG_OK;
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
  st->resident.assign(num_layers, 0);
  for (int l = 0; l < num_layers; l++) {
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, host_blobs[l]) == cudaSuccess) {
      st->resident[l] = pa.type == cudaMemoryTypeDevice;
    } else {
      cudaGetLastError();  // plain host memory on older runtimes
    }
    if (st->resident[l] && (reinterpret_cast<uintptr_t>(host_blobs[l]) & 255)) {
      delete st;
      return FG_ERR_INVALID;
    }
  }
  st->staging[0] = dev_staging0;
  st->staging[1] = dev_staging1;
  st->nbuf = dev_staging0 == dev_staging1 ? 1 : 2;
  st->blob_bytes = bytes;
  st->inject_failures = 0;
  fg_layer_blob_slices(c, st->sbegin, st->send);
  for (int i = 0; i < 2; i++) {
    st->kv_back[i] = nullptr;
    for (int e = 0; e < 6; e++) st->ev[i].ready[e] = st->ev[i].done[e] = nullptr;
  }
  for (int i = 0; i < 2; i++) {
    bool ok = fg_cuda_check(cudaEventCreateWithFlags(&st->kv_back[i], cudaEventDisableTiming)) == FG_OK;
    for (int e = 0; ok && e < 6; e++)
      ok = fg_cuda_check(cudaEventCreateWithFlags(&st->ev[i].ready[e], cudaEventDisableTiming)) == FG_OK &&
           fg_cuda_check(cudaEventCreateWithFlags(&st->ev[i].done[e], cudaEventDisableTiming)) == FG_OK;
    if (!ok) {
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
    for (int e = 0; e < 6; e++) {
      if (st->ev[i].ready[e]) cudaEventDestroy(st->ev[i].ready[e]);
      if (st->ev[i].done[e]) cudaEventDestroy(st->ev[i].done[e]);
    }
    if (st->kv_back[i]) cudaEventDestroy(st->kv_back[i]);
  }
  delete st;
  return FG_OK;
}

extern "C" size_t fg_stack_one_buffer_bytes(const fg_layer_config *c) {
  const size_t bytes = fg_layer_blob_bytes(c);
  size_t begin[5], end[5];
  if (bytes == 0 || fg_layer_blob_slices(c, begin, end) != FG_OK) return 0;
  return bytes + (end[0] - begin[0]);  // the blob, then a second slot for the vectors
}
