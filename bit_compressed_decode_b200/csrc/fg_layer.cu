// fg_layer.cu -- one OPT decoder layer over a block of GPU batches, W4 weights, KV4 cache.
//
// "FlexGen Guide: High-Throughput LLM Offloading on One GPU", section 2 (The Zig-Zag Block
// Schedule): the layer's weights are loaded once and reused by every GPU batch of the
// block.  On this GPU the reuse happens inside each GEMM: one launch covers all rows of
// the block, so every weight tile is read from HBM once per step and applied to all
// num_gpu_batches * gpu_batch_size sequences.  Section 3: weights and KV cache are 4-bit.
// Layer math (OPT, pre-LayerNorm, ReLU): see fg_layer_decode in fg.h.
#include <math.h>

#include "fg_internal.cuh"

// kernels/launchers of the other translation units
fg_status fg_layernorm_launch(const fg_half *x, int M, int h, const fg_half *gamma, const fg_half *beta, float eps,
                              fg_half *y, cudaStream_t st);
fg_status fg_linear_launch(const fg_half *x, int M, int K, const fg_qtensor *w, const fg_half *bias,
                           const fg_half *residual, int flags, int qscale_cols, float qscale, fg_half *y,
                           void *workspace, size_t ws_bytes, cudaStream_t st, bool pdl);
size_t fg_linear_ws_bytes(int M, int N, int K);
fg_status fg_kv_validate(const fg_kv_cache *kv);
fg_status fg_kv_append_launch(const fg_kv_cache *kv, const fg_half *k, const fg_half *v, int64_t ld, int rows,
                              int rows_per_seq, const int32_t *positions, cudaStream_t st, bool pdl);
fg_status fg_attention_launch(const fg_kv_cache *kv, const fg_half *q, int64_t ldq, fg_half *out, int64_t ldo,
                              int rows, int rows_per_seq, const int32_t *positions, cudaStream_t st,
                              const fg_half *k_new, const fg_half *v_new, int64_t ld_new);
size_t fg_w4a8_pair_ws_bytes(int M, int N, int K);
fg_status fg_layernorm_q8_launch(const fg_half *x, int M, int h, const fg_half *gamma, const fg_half *beta,
                                 float eps, fg_half *y, int8_t *a8, float *ascale, cudaStream_t st);

int fg_profile_begin(int slot, cudaStream_t st);
void fg_profile_end(int idx, cudaStream_t st);

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool w4a8(const fg_layer_config *c) { return c->act_bits == 8; }

bool config_ok(const fg_layer_config *c) {
  if (!c) return false;
  if (c->act_bits != 0 && c->act_bits != 16 && c->act_bits != 8) return false;
  if (c->act_bits == 8 && (fg_kv_group(c->group) != 64 || c->hidden % 128 || c->ffn % 128 || c->ffn > 65536))
    return false;
  if (c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256) return false;
  const int G = fg_kv_group(c->group);
  if (G == 0 || c->head_dim % G) return false;
  if (c->num_heads < 1 || c->hidden != c->num_heads * c->head_dim) return false;
  if (c->hidden % 128 || c->ffn % 128 || c->ffn <= 0 || c->hidden > 16384) return false;
  return true;
}

struct Matrix {
  int64_t n, k;
};

// Offsets of every array inside the layer blob (256-byte aligned).
struct BlobLayout {
  size_t off[4][4];  // [matrix][codes, mins, scales, row scales]: W4A8: codes, gmin, gstep, cscale
  size_t vec[8];     // bqkv, bo, b1, b2, ln1_g, ln1_b, ln2_g, ln2_b
  size_t total;
  Matrix mat[4];
};

BlobLayout blob_layout(const fg_layer_config *c) {
  BlobLayout L;
  const int64_t h = c->hidden, F = c->ffn;
  const int64_t G = fg_kv_group(c->group);
  L.mat[0] = {3 * h, h};
  L.mat[1] = {h, h};
  L.mat[2] = {F, h};
  L.mat[3] = {h, F};
  size_t p = 0;
  const size_t mbytes = w4a8(c) ? 1 : 2;  // per group: int8 minimum and uint8 step, or fp16 min and scale
  for (int i = 0; i < 4; i++) {
    const size_t numel = static_cast<size_t>(L.mat[i].n * L.mat[i].k);
    L.off[i][0] = p;
    p = align256(p + numel / 2);
    L.off[i][1] = p;
    p = align256(p + numel / G * mbytes);
    L.off[i][2] = p;
    p = align256(p + numel / G * mbytes);
    L.off[i][3] = p;
    if (w4a8(c)) p = align256(p + static_cast<size_t>(L.mat[i].n) * 4);
  }
  const int64_t vlen[8] = {3 * h, h, F, h, h, h, h, h};
  for (int i = 0; i < 8; i++) {
    L.vec[i] = p;
    p = align256(p + vlen[i] * 2);
  }
  L.total = p;
  return L;
}

struct WsLayout {
  size_t a, qkv, o, h1, f, a8, as, gemm, total;
};

size_t gemm_ws(const fg_layer_config *c, int rows, int N, int K) {
  return w4a8(c) ? fg_w4a8_pair_ws_bytes(rows, N, K) : fg_linear_ws_bytes(rows, N, K);
}

WsLayout ws_layout(const fg_layer_config *c, int rows) {
  WsLayout w;
  const size_t R = static_cast<size_t>(rows), h = c->hidden, F = c->ffn;
  size_t p = 0;
  w.a = p;
  p = align256(p + R * h * 2);
  w.qkv = p;
  p = align256(p + R * 3 * h * 2);
  w.o = p;
  p = align256(p + R * h * 2);
  w.h1 = p;
  p = align256(p + R * h * 2);
  w.f = p;
  p = align256(p + R * F * 2);
  w.a8 = w.as = p;  // W4A8: a product's int8 input [rows][<= F] and its row scales
  if (w4a8(c)) {
    p = align256(p + R * (F > h ? F : h));
    w.as = p;
    p = align256(p + R * 4);
  }
  w.gemm = p;
  const int N[4] = {3 * c->hidden, c->hidden, c->ffn, c->hidden}, K[4] = {c->hidden, c->hidden, c->hidden, c->ffn};
  size_t g = 0;
  for (int i = 0; i < 4; i++) {
    const size_t gi = gemm_ws(c, rows, N[i], K[i]);
    g = gi > g ? gi : g;
  }
  p = align256(p + g);
  w.total = p;
  return w;
}

bool weights_ok(const fg_layer_config *c, const fg_layer_weights *w) {
  const int64_t h = c->hidden, F = c->ffn;
  const fg_qtensor *m[4] = {&w->wqkv, &w->wo, &w->w1, &w->w2};
  const int64_t shp[4][2] = {{3 * h, h}, {h, h}, {F, h}, {h, F}};
  const int G = fg_kv_group(c->group);
  for (int i = 0; i < 4; i++) {
    if (m[i]->ndim != 2 || m[i]->dim != 1 || m[i]->bits != 4 || m[i]->group != G) return false;
    if (m[i]->shape[0] != shp[i][0] || m[i]->shape[1] != shp[i][1]) return false;
    if (!m[i]->codes || !m[i]->mins || !m[i]->scales || !fg_aligned16(m[i]->codes)) return false;
    if (w4a8(c) && (!w->cscale[i] || (reinterpret_cast<uintptr_t>(w->cscale[i]) & 3u) ||
                    (reinterpret_cast<uintptr_t>(m[i]->mins) & 1u) || (reinterpret_cast<uintptr_t>(m[i]->scales) & 1u)))
      return false;
  }
  return true;
}

}  // namespace

namespace {

fg_status slice_wait(const fg_layer_slices *sl, int i, cudaStream_t st) {
  if (!sl || !sl->ready[i]) return FG_OK;
  return fg_cuda_check(cudaStreamWaitEvent(st, sl->ready[i], 0));
}

fg_status slice_done(const fg_layer_slices *sl, int i, cudaStream_t st) {
  if (!sl || !sl->done[i]) return FG_OK;
  return fg_cuda_check(cudaEventRecord(sl->done[i], st));
}

// The layer over `rows` hidden-state rows; row r is token r % rows_per_seq of
// sequence r / rows_per_seq of `kv` (a view starting at the first sequence).
fg_status run_layer(const fg_layer_config *c, const fg_layer_weights *w, const fg_kv_cache *kv, const fg_half *x_in,
                    fg_half *x_out, const int32_t *positions, int rows, int rows_per_seq, uint8_t *ws,
                    size_t ws_bytes, cudaStream_t st, const fg_layer_slices *sl = nullptr) {
  const WsLayout L = ws_layout(c, rows);
  // the GEMMs' split-k scratch is optional: they reduce on chip when what is left is short
  if (ws_bytes < L.gemm) return FG_ERR_WORKSPACE;
  const int h = c->hidden, F = c->ffn;
  fg_half *a = reinterpret_cast<fg_half *>(ws + L.a);
  fg_half *qkv = reinterpret_cast<fg_half *>(ws + L.qkv);
  fg_half *o = reinterpret_cast<fg_half *>(ws + L.o);
  fg_half *h1 = reinterpret_cast<fg_half *>(ws + L.h1);
  fg_half *f = reinterpret_cast<fg_half *>(ws + L.f);
  void *gws = ws + L.gemm;
  const size_t gbytes = ws_bytes - L.gemm;
  const float qscale = 1.0f / sqrtf(static_cast<float>(c->head_dim));
  // Decode steps launch the GEMMs with programmatic dependent launch: a GEMM's prologue
  // (weight loads and dequantisation; the weights are fixed for the call) overlaps the
  // kernel before it.  Not for prompts, whose attention can outlast the GEMM's bounded
  // pipeline waits.
  const bool pdl = rows_per_seq == 1;
  // W4A8: each product's fp16 input is quantised to int8 per row into a8 / as first
  const bool i8 = w4a8(c);
  int8_t *a8 = reinterpret_cast<int8_t *>(ws + L.a8);
  float *as = reinterpret_cast<float *>(ws + L.as);
  const fg_qtensor *mq[4] = {&w->wqkv, &w->wo, &w->w1, &w->w2};
  fg_w4a8_weight w8[4];
  for (int i = 0; i < 4; i++) {
    w8[i].codes = const_cast<uint8_t *>(mq[i]->codes);
    w8[i].gmin = reinterpret_cast<int8_t *>(mq[i]->mins);
    w8[i].gstep = reinterpret_cast<uint8_t *>(mq[i]->scales);
    w8[i].cscale = w->cscale[i];
    w8[i].N = mq[i]->shape[0];
    w8[i].K = mq[i]->shape[1];
  }
  // the product y = epi(x W_i^T + b): W4A16 on fp16 x, or W4A8 on x quantised to int8 (profile slot qslot)
  // (qslot < 0: a8 / as already hold x's int8 form, made by the LayerNorm before it)
  auto product = [&](int i, const fg_half *x, int K, const fg_half *b, const fg_half *res, int flags, int qcols,
                     float qs, fg_half *y, int slot, int qslot) -> fg_status {
    fg_status r;
    if (!i8) {
      const int e = fg_profile_begin(slot, st);
      r = fg_linear_launch(x, rows, K, mq[i], b, res, flags, qcols, qs, y, gws, gbytes, st, pdl);
      fg_profile_end(e, st);
      return r;
    }
    int e;
    if (qslot >= 0) {
      e = fg_profile_begin(qslot, st);
      r = fg_act8_quantize(x, rows, K, a8, as, st);
      fg_profile_end(e, st);
      if (r != FG_OK) return r;
    }
    e = fg_profile_begin(slot, st);
    r = fg_linear_w4a8(a8, as, rows, K, &w8[i], b, res, flags, qcols, qs, y, gws, gbytes, st);
    fg_profile_end(e, st);
    return r;
  };
  fg_status rc;
  int ev;
#define FG_STEP(slot, call)                    \
  ev = fg_profile_begin(slot, st);             \
  if ((rc = (call)) != FG_OK) return rc;       \
  fg_profile_end(ev, st);
#define FG_SLICE(call)                   \
  if ((rc = (call)) != FG_OK) return rc;
  // a = LN1(x)
  FG_SLICE(slice_wait(sl, 0, st));
  // (W4A8: with its int8 form)
  FG_STEP(0, i8 ? fg_layernorm_q8_launch(x_in, rows, h, w->ln1_g, w->ln1_b, c->ln_eps, a, a8, as, st)
                : fg_layernorm_launch(x_in, rows, h, w->ln1_g, w->ln1_b, c->ln_eps, a, st));
  // [q k v] = a Wqkv^T + bqkv; q *= d^-1/2
  FG_SLICE(slice_wait(sl, 1, st));
  FG_SLICE(product(0, a, h, w->bqkv, nullptr, 0, h, qscale, qkv, 1, -1));
  FG_SLICE(slice_done(sl, 1, st));
  // append k, v (4-bit) at the sequences' positions, then o = softmax(q K^T) V over the
  // 4-bit cache.  When the decode attention is about one wave of (row, head) CTAs or less its
  // time is launch-bound and the append rides in it (one launch fewer: 58.6 instead of 63.7 us
  // per step at the OPT-125M block of 4 sequences); above that the separate append kernel
  // costs less than the per-CTA work it would add (a 512-sequence OPT-6.7B block: 10.7 us
  // against 18 us).  Prompt rows always append first.
  FG_SLICE(slice_wait(sl, 2, st));
  const bool fuse = rows_per_seq == 1 && static_cast<int64_t>(rows) * c->num_heads <= 4LL * fg_sm_count();
  if (fuse) {
    FG_STEP(3, fg_attention_launch(kv, qkv, 3 * h, o, h, rows, 1, positions, st, qkv + h, qkv + 2 * h, 3 * h));
  } else {
    FG_STEP(2, fg_kv_append_launch(kv, qkv + h, qkv + 2 * h, 3 * h, rows, rows_per_seq, positions, st, pdl));
    FG_STEP(3, fg_attention_launch(kv, qkv, 3 * h, o, h, rows, rows_per_seq, positions, st, nullptr, nullptr, 0));
  }
  FG_SLICE(slice_done(sl, 2, st));
  // h1 = x + o Wo^T + bo
  FG_SLICE(slice_wait(sl, 3, st));
  FG_SLICE(product(1, o, h, w->bo, x_in, FG_EPI_RESIDUAL, 0, 1.f, h1, 4, 9));
  FG_SLICE(slice_done(sl, 3, st));
  // a = LN2(h1)
  FG_STEP(5, i8 ? fg_layernorm_q8_launch(h1, rows, h, w->ln2_g, w->ln2_b, c->ln_eps, a, a8, as, st)
                : fg_layernorm_launch(h1, rows, h, w->ln2_g, w->ln2_b, c->ln_eps, a, st));
  // f = relu(a W1^T + b1)
  FG_SLICE(slice_wait(sl, 4, st));
  FG_SLICE(product(2, a, h, w->b1, nullptr, FG_EPI_RELU, 0, 1.f, f, 6, -1));
  FG_SLICE(slice_done(sl, 4, st));
  // x_out = h1 + f W2^T + b2
  FG_SLICE(slice_wait(sl, 5, st));
  FG_SLICE(product(3, f, F, w->b2, h1, FG_EPI_RESIDUAL, 0, 1.f, x_out, 7, 11));
  FG_SLICE(slice_done(sl, 5, st));
  FG_SLICE(slice_done(sl, 0, st));
#undef FG_STEP
#undef FG_SLICE
  return FG_OK;
}

fg_kv_cache kv_view(const fg_kv_cache *kv, int s0, int n) {
  fg_kv_cache v = *kv;
  const size_t slots = static_cast<size_t>(s0) * kv->num_heads * kv->max_len;
  const size_t ng = kv->head_dim / fg_kv_group(kv->group);
  v.k_codes += slots * (kv->head_dim / 2);
  v.v_codes += slots * (kv->head_dim / 2);
  v.k_mins += slots * ng;
  v.k_scales += slots * ng;
  v.v_mins += slots * ng;
  v.v_scales += slots * ng;
  v.num_seqs = n;
  return v;
}

fg_status check_common(const fg_layer_config *c, const fg_layer_weights *w, const fg_kv_cache *kv,
                       const fg_half *x_in, fg_half *x_out, const int32_t *positions, int nb, int gbs) {
  if (!config_ok(c)) return FG_ERR_UNSUPPORTED;
  if (!w || !weights_ok(c, w)) return FG_ERR_INVALID;
  fg_status rc = fg_kv_validate(kv);
  if (rc != FG_OK) return rc;
  if (kv->num_heads != c->num_heads || kv->head_dim != c->head_dim) return FG_ERR_SHAPE;
  if (fg_kv_group(kv->group) != fg_kv_group(c->group)) return FG_ERR_SHAPE;
  if (nb < 0 || gbs < 0) return FG_ERR_INVALID;
  if (static_cast<int64_t>(nb) * gbs != kv->num_seqs) return FG_ERR_SHAPE;
  if (kv->num_seqs == 0) return FG_OK;
  if (!x_in || !x_out || !positions || !fg_aligned16(x_in) || !fg_aligned16(x_out)) return FG_ERR_INVALID;
  return FG_OK;
}

}  // namespace

extern "C" size_t fg_layer_blob_bytes(const fg_layer_config *c) {
  if (!config_ok(c)) return 0;
  return blob_layout(c).total;
}

extern "C" fg_status fg_layer_weights_from_blob(const fg_layer_config *c, void *blob, fg_layer_weights *out) {
  if (!config_ok(c)) return FG_ERR_UNSUPPORTED;
  if (!blob || !out || (reinterpret_cast<uintptr_t>(blob) & 255)) return FG_ERR_INVALID;
  const BlobLayout L = blob_layout(c);
  uint8_t *b = static_cast<uint8_t *>(blob);
  fg_qtensor *m[4] = {&out->wqkv, &out->wo, &out->w1, &out->w2};
  for (int i = 0; i < 4; i++) {
    m[i]->codes = b + L.off[i][0];
    m[i]->mins = reinterpret_cast<fg_half *>(b + L.off[i][1]);
    m[i]->scales = reinterpret_cast<fg_half *>(b + L.off[i][2]);
    out->cscale[i] = w4a8(c) ? reinterpret_cast<float *>(b + L.off[i][3]) : nullptr;
    m[i]->ndim = 2;
    m[i]->shape[0] = L.mat[i].n;
    m[i]->shape[1] = L.mat[i].k;
    m[i]->shape[2] = m[i]->shape[3] = 1;
    m[i]->dim = 1;
    m[i]->bits = 4;
    m[i]->group = fg_kv_group(c->group);
  }
  fg_half **v[8] = {&out->bqkv, &out->bo, &out->b1, &out->b2, &out->ln1_g, &out->ln1_b, &out->ln2_g, &out->ln2_b};
  for (int i = 0; i < 8; i++) *v[i] = reinterpret_cast<fg_half *>(b + L.vec[i]);
  return FG_OK;
}

// The part of the layer's workspace that a call cannot do without (everything before the
// GEMMs' optional split-k scratch).
size_t fg_layer_ws_required(const fg_layer_config *c, int rows) {
  if (!c || rows <= 0 || !config_ok(c)) return 0;
  return ws_layout(c, rows).gemm;
}

extern "C" size_t fg_layer_workspace_bytes(const fg_layer_config *c, int rows) {
  if (!config_ok(c) || rows < 0) return 0;
  return ws_layout(c, rows).total;
}

extern "C" fg_status fg_layer_decode(const fg_layer_config *c, const fg_layer_weights *w, const fg_kv_cache *kv,
                                     const fg_half *x_in, fg_half *x_out, const int32_t *positions,
                                     int num_gpu_batches, int gpu_batch_size, void *workspace,
                                     size_t workspace_bytes, void *stream) {
  fg_status rc = check_common(c, w, kv, x_in, x_out, positions, num_gpu_batches, gpu_batch_size);
  if (rc != FG_OK || kv->num_seqs == 0) return rc;
  if (!workspace || !fg_aligned16(workspace)) return FG_ERR_INVALID;
  return run_layer(c, w, kv, x_in, x_out, positions, kv->num_seqs, 1, static_cast<uint8_t *>(workspace),
                   workspace_bytes, static_cast<cudaStream_t>(stream));
}

// fg_layer_decode whose weights and cache arrive in slices (see fg_layer_slices); the stack's
// sliced prefetch calls it.
fg_status fg_layer_decode_sliced(const fg_layer_config *c, const fg_layer_weights *w, const fg_kv_cache *kv,
                                 const fg_half *x_in, fg_half *x_out, const int32_t *positions, int num_gpu_batches,
                                 int gpu_batch_size, void *workspace, size_t workspace_bytes, cudaStream_t st,
                                 const fg_layer_slices *sl) {
  fg_status rc = check_common(c, w, kv, x_in, x_out, positions, num_gpu_batches, gpu_batch_size);
  if (rc != FG_OK || kv->num_seqs == 0) return rc;
  if (!workspace || !fg_aligned16(workspace)) return FG_ERR_INVALID;
  return run_layer(c, w, kv, x_in, x_out, positions, kv->num_seqs, 1, static_cast<uint8_t *>(workspace),
                   workspace_bytes, st, sl);
}

// Byte ranges of the layer blob's slices, in the order a layer step reads them: [0] the vectors,
// [1] wqkv, [2] wo, [3] w1, [4] w2 (begin[i] .. end[i]).
fg_status fg_layer_blob_slices(const fg_layer_config *c, size_t begin[5], size_t end[5]) {
  if (!config_ok(c)) return FG_ERR_UNSUPPORTED;
  const BlobLayout L = blob_layout(c);
  begin[0] = L.vec[0];
  end[0] = L.total;
  for (int i = 0; i < 4; i++) {
    begin[1 + i] = L.off[i][0];
    end[1 + i] = i < 3 ? L.off[i + 1][0] : L.vec[0];
  }
  return FG_OK;
}

extern "C" fg_status fg_layer_prefill(const fg_layer_config *c, const fg_layer_weights *w, const fg_kv_cache *kv,
                                      const fg_half *x_in, fg_half *x_out, const int32_t *positions, int prompt_len,
                                      int num_gpu_batches, int gpu_batch_size, void *workspace,
                                      size_t workspace_bytes, void *stream) {
  fg_status rc = check_common(c, w, kv, x_in, x_out, positions, num_gpu_batches, gpu_batch_size);
  if (rc != FG_OK || kv->num_seqs == 0) return rc;
  if (prompt_len < 1) return FG_ERR_SHAPE;
  if (prompt_len > kv->max_len) return FG_ERR_RANGE;
  if (!workspace || !fg_aligned16(workspace)) return FG_ERR_INVALID;
  // Process whole sequences in chunks that fit the workspace given.
  const int S = kv->num_seqs;
  int chunk = S;
  while (chunk > 0 && ws_layout(c, chunk * prompt_len).gemm > workspace_bytes) chunk = chunk > 1 ? chunk / 2 : 0;
  if (chunk == 0) return FG_ERR_WORKSPACE;
  if (static_cast<int64_t>(chunk) * prompt_len > (1 << 30)) return FG_ERR_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t h = c->hidden;
  for (int s0 = 0; s0 < S; s0 += chunk) {
    const int n = chunk < S - s0 ? chunk : S - s0;
    const fg_kv_cache sub = kv_view(kv, s0, n);
    const int64_t off = static_cast<int64_t>(s0) * prompt_len * h;
    rc = run_layer(c, w, &sub, x_in + off, x_out + off, positions + s0, n * prompt_len, prompt_len,
                   static_cast<uint8_t *>(workspace), workspace_bytes, st);
    if (rc != FG_OK) return rc;
  }
  return FG_OK;
}
