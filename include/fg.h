/*
 * fg.h -- C ABI of the B200 (sm_100a) group-wise 4-bit decode library.
 *
 * What the library computes follows these web pages:
 *   [G2] "FlexGen Guide: High-Throughput LLM Offloading on One GPU",
 *        section "2. The Zig-Zag Block Schedule" -- a loaded layer is reused for
 *        every GPU batch of a block before the next layer is loaded.
 *   [G3] same page, section "3. Group-Wise 4-Bit Quantization for Weights and KV
 *        Cache" -- weights and KV cache held as 4-bit integers with per-group
 *        scaling over contiguous groups, dequantised on the fly for FP16 compute.
 *   [G1] same page, section "1. Three-Tier Storage Hierarchy" -- weights kept in
 *        CPU memory and moved to the GPU layer by layer.
 *   [OPT] the OPT entry of the PIPO paper's reference list -- the model family
 *        (pre-LayerNorm decoder layer, multi-head attention, ReLU FFN).
 *   [Q8] the QServe W4A8KV4 entry of the same list (title only) and the
 *        "Optimizing LLM for low memory usage" page, section "Quantization and
 *        Weight Compression" (INT8 and INT4 weight formats) -- the W4A8 variant.
 *
 * The 4-bit format (the pages give no formula; this is the reading the whole
 * library and its tests use).  For every group of G consecutive fp16 values
 * x_0..x_{G-1} along the grouping dim (G = 64, or 128 where a call says so --
 * [G3] allows groups of 64 or 128), each step one IEEE fp32 operation:
 *   mn = min(x) + 0 (so -0 becomes +0);  d = max(x) - mn;
 *   scale = fp16_rn(d / 15);  if scale == 0: every code 0, stored scale +0;
 *   inv = 1 / scale;  code_i = clamp(round_half_even((x_i - mn) * inv), 0, 15);
 *   byte j of the group = code_{2j} | code_{2j+1} << 4  (even element low);
 *   min and scale are stored as fp16 in two planar arrays.
 * Dequantised value: fp16_rn(mn + code * scale), the exact value rounded once
 * (an fp16 fused multiply-add).
 *
 * Conventions for every call:
 *   - fp16 values travel as their binary16 bit patterns (fg_half).
 *   - The caller owns all memory.  Pointers named "device" must point to
 *     device memory of the current CUDA device (or memory mapped into it);
 *     the library never allocates or frees device memory.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued asynchronously; argument errors are returned before
 *     anything is launched.  Faults detected inside kernels (a cache position
 *     out of range, a pipeline wait that timed out) set a device error word
 *     that fg_sync_status() reports and clears.
 *   - Device pointers must be 16-byte aligned unless stated otherwise;
 *     a misaligned pointer returns FG_ERR_INVALID.
 *   - No call throws, exits or prints.
 */
#ifndef FG_H_
#define FG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FG_API __attribute__((visibility("default")))
#else
#define FG_API
#endif

typedef uint16_t fg_half;  /* IEEE 754 binary16 bit pattern */

typedef enum {
    FG_OK = 0,
    FG_ERR_INVALID = 1,     /* null/misaligned pointer, bad enum, negative size */
    FG_ERR_SHAPE = 2,       /* size not a multiple of the group, inconsistent dims */
    FG_ERR_UNSUPPORTED = 3, /* a code width or group size not taken, dims the kernels do not cover */
    FG_ERR_RANGE = 4,       /* a cache position outside [0, max_len) (host or device check) */
    FG_ERR_CUDA = 5,        /* a CUDA runtime call failed (launch, copy, event) */
    FG_ERR_TIMEOUT = 6,     /* a bounded wait inside a kernel gave up */
    FG_ERR_WORKSPACE = 7    /* workspace too small */
} fg_status;

/* Human-readable name of a status (static string). */
FG_API const char *fg_status_string(fg_status s);

/* Synchronises `stream`, then reads and clears the current device's error
 * word.  Returns FG_ERR_RANGE or FG_ERR_TIMEOUT if a kernel flagged one since
 * the last call, FG_ERR_CUDA if the stream reported an error, else FG_OK. */
FG_API fg_status fg_sync_status(void *stream);

/* Text of the last CUDA runtime error seen by this library on this thread. */
FG_API const char *fg_last_cuda_error(void);

/* ---------------------------------------------------------------------- */
/* Packed 4-bit tensors [G3]                                               */
/* ---------------------------------------------------------------------- */

/* A tensor of `shape` quantised in groups of `group` along `dim`.
 * codes:  uint8; bits = 4: shape with shape[dim] halved (even element in the
 *         low nibble); bits = 8: shape unchanged, one code per byte
 * mins, scales: fp16, shape with shape[dim] divided by `group`.
 * All three are row-major (C order) and caller-owned (device memory).
 * bits = 8 is the same min-max scheme with 255 steps (INT8 beside INT4 among
 * the post-training formats of the "Optimizing LLM for low memory usage"
 * page); the layer, the KV cache and fg_linear_w4a16 take 4-bit codes only. */
typedef struct {
    uint8_t *codes;
    fg_half *mins;
    fg_half *scales;
    int32_t ndim;        /* 1..4 */
    int64_t shape[4];
    int32_t dim;         /* grouping dim, 0..ndim-1 */
    int32_t bits;        /* 4 or 8 */
    int32_t group;       /* 64 or 128 */
} fg_qtensor;

/* Byte sizes of the codes array and of each of the mins/scales arrays. */
FG_API fg_status fg_qtensor_bytes(int ndim, const int64_t *shape, int dim, int bits, int group,
                           size_t *codes_bytes, size_t *meta_bytes);

/* Quantise fp16 `x` (device, row-major `shape`) along `dim` into out->codes,
 * out->mins, out->scales (device buffers set by the caller; their sizes from
 * fg_qtensor_bytes).  Fills out->ndim/shape/dim/bits/group.  x must be finite
 * (a group holding Inf or NaN gets unspecified codes).
 * Codes: with levels = 2^bits - 1, scale = fp16_rn(d / levels) for the group
 * range d, code = clamp(rint_even((x - min) * (1 / scale)), 0, levels), in the
 * fp32 steps stated at the top of this file for 4 bits (15 replaced by levels).
 * Errors: FG_ERR_SHAPE if shape[dim] % group != 0; FG_ERR_UNSUPPORTED if
 * bits is not 4 or 8, or group not 64 or 128.  [G3] */
FG_API fg_status fg_quantize(const fg_half *x, int ndim, const int64_t *shape, int dim, int bits, int group,
                      fg_qtensor *out, void *stream);

/* Dequantise q into fp16 `y` (device, row-major q->shape).  [G3] */
FG_API fg_status fg_dequantize(const fg_qtensor *q, fg_half *y, void *stream);

/* ---------------------------------------------------------------------- */
/* 4-bit KV cache of one layer [G3]                                        */
/* ---------------------------------------------------------------------- */

/* For sequence s, head h, position p the head_dim values of k (and of v) are
 * quantised in groups of G = 64 or 128 along head_dim ([G3]):
 *   k_codes  uint8 [num_seqs][num_heads][max_len][head_dim/2]
 *   k_mins, k_scales fp16 [num_seqs][num_heads][max_len][head_dim/G]
 * and the same for v.  Device memory, caller-owned.
 * Requirements: head_dim in {64, 128, 256}, a multiple of G; max_len % 64 == 0. */
typedef struct {
    uint8_t *k_codes;
    fg_half *k_mins;
    fg_half *k_scales;
    uint8_t *v_codes;
    fg_half *v_mins;
    fg_half *v_scales;
    int32_t num_seqs;
    int32_t num_heads;
    int32_t head_dim;
    int32_t max_len;
    int32_t group;       /* G: 64 or 128 (0 = 64) */
} fg_kv_cache;

/* Byte sizes of one codes array and of one mins/scales array (group 0 = 64). */
FG_API fg_status fg_kv_cache_bytes(int num_seqs, int num_heads, int head_dim, int max_len, int group,
                            size_t *codes_bytes, size_t *meta_bytes);

/* Quantise and append new k, v rows.  k, v: fp16 device rows, row r at
 * k + r*ld holding num_heads*head_dim values (head-major).  Row r belongs to
 * sequence s = r / rows_per_seq and is written at position
 * positions[s] + r % rows_per_seq (positions: int32 device [num_seqs]).
 * rows must be a multiple of rows_per_seq.  Decode: rows_per_seq = 1;
 * a prompt of P tokens: rows_per_seq = P, positions = start positions.
 * A position outside [0, max_len) is skipped and flags FG_ERR_RANGE
 * (reported by fg_sync_status).  [G3] */
FG_API fg_status fg_kv_append(const fg_kv_cache *kv, const fg_half *k, const fg_half *v, int64_t ld,
                       int rows, int rows_per_seq, const int32_t *positions, void *stream);

/* Softmax attention of query rows over the 4-bit cache.  q: fp16 device rows
 * (row stride ldq), already scaled by head_dim^-1/2; out: fp16 device rows
 * (row stride ldo).  Row r (sequence s = r / rows_per_seq) attends over
 * positions 0 .. positions[s] + r % rows_per_seq of its sequence, inclusive,
 * reading K and V from their 4-bit form.  ([G3]; attention of OPT [OPT]) */
FG_API fg_status fg_attention_decode(const fg_kv_cache *kv, const fg_half *q, int64_t ldq, fg_half *out, int64_t ldo,
                              int rows, int rows_per_seq, const int32_t *positions, void *stream);

/* One decode step's KV append and attention in one launch: for each row r
 * (sequence r, one row per sequence), k and v (fp16 device rows at
 * k + r*ldkv, v + r*ldkv, num_heads*head_dim values, head-major) are quantised
 * into the cache at position positions[r], exactly as fg_kv_append does (the
 * cache receives the same bits), and q's row then attends over positions
 * 0 .. positions[r] as fg_attention_decode does.  rows <= num_seqs.  A
 * position outside [0, max_len) appends nothing, writes zeros to the row's
 * output and flags FG_ERR_RANGE (fg_sync_status).  The k, v rows may share a
 * buffer with q (the layer passes the k and v thirds of its [q k v] rows).
 * ([G3]: the cache is written and read in its 4-bit form) */
FG_API fg_status fg_attention_decode_append(const fg_kv_cache *kv, const fg_half *q, int64_t ldq, const fg_half *k,
                                     const fg_half *v, int64_t ldkv, fg_half *out, int64_t ldo, int rows,
                                     const int32_t *positions, void *stream);

/* ---------------------------------------------------------------------- */
/* W4A16 linear layer and LayerNorm                                         */
/* ---------------------------------------------------------------------- */

enum {
    FG_EPI_RELU = 1,         /* y = max(0, .) after the bias (and q-scale) */
    FG_EPI_RESIDUAL = 2,     /* y += residual[m][n] after the activation */
    FG_GEMM_PERSISTENT = 4,  /* M > 256: take the persistent launch (see below) */
};

/* y[m][n] = epi( sum_k x[m][k] * deq(w)[n][k] + bias[n] ), fp32 accumulation,
 * fp16 output.  x: fp16 device [M][K]; w: packed along K, shape [N][K]
 * (PyTorch Linear orientation); bias: fp16 [N] or NULL; residual: fp16 [M][N]
 * (with FG_EPI_RESIDUAL); the first qscale_cols outputs of each row are
 * multiplied by qscale after the bias.  w->group 64 or 128 with K % group == 0,
 * N % 128 == 0; x, y, the
 * codes and the residual 16-byte aligned, the mins, scales and bias 2-byte
 * aligned (FG_ERR_INVALID otherwise).
 * Tensor cores dequantise W tiles in shared memory ([G3]: on-the-fly
 * dequantisation for FP16 compute).
 * Launches (see fg_linear_plan): M <= 256 runs one SM per output tile; larger M
 * runs on CTA pairs: the classic launch (one pair per tile, k-range optionally
 * split over a cluster; it stages the weights' codes and group metadata by
 * tensor copies, so it needs (K / group) % 8 == 0 and the mins and scales
 * 16-byte aligned, else the one-SM launch runs), or, with FG_GEMM_PERSISTENT in
 * flags, the persistent
 * launch (every resident pair takes an equal share of the tiles' k-iterations; a
 * tile shared between pairs is finished by the pair holding its first
 * k-segment).  The layer calls use the classic launch.
 * workspace: optional device scratch (16-byte aligned).  The classic launch's
 * split k-range adds its partial sums through the scratch when it holds
 * P = n_tiles * t_tiles * splits * tile_tokens * 256 * 4 bytes (n_tiles =
 * ceil(N / 256), t_tiles = ceil(M / tile_tokens)), else over distributed shared
 * memory.  With P + n_tiles * t_tiles * splits * 16 bytes (flags after the
 * partials) and a grid that fits the GPU in one wave, the split ranks run as
 * separate CTA pairs that meet through the flags; otherwise each tile's ranks
 * form one cluster.  All of these add the splits in the same order, so their
 * results are the same bit for bit.  The persistent launch needs fg_linear_workspace_bytes(M, N,
 * K) bytes (its shared tiles' partial sums) and falls back to the classic launch
 * with less; it adds partial sums in another order, so its results may differ
 * from the classic launch's in the last bits (each is deterministic). */
FG_API size_t fg_linear_workspace_bytes(int M, int N, int K);
/* The launches fg_linear_w4a16 makes for this shape on the current device (no
 * launch; weights in groups of 64 with 16-byte aligned metadata): the classic
 * launch's *tile_tokens = tokens per output tile (16..256 for M <= 256, or K
 * not a multiple of 512, one SM per tile; 256 or 512 for larger M, a CTA pair
 * per tile)
 * and *splits = CTAs sharing each tile's k-range (1..8 one-SM, 1..4 pair),
 * chosen by a time model of the kernels: waves of resident clusters x k-tiles
 * per CTA, plus the pipeline fill and the epilogue; *pairs = CTA pairs of the
 * persistent launch (512-token tiles) that FG_GEMM_PERSISTENT would take, 0
 * where it is not available (M <= 256, or tiles split too finely). */
FG_API fg_status fg_linear_plan(int M, int N, int K, int *tile_tokens, int *splits, int *pairs);
FG_API fg_status fg_linear_w4a16(const fg_half *x, int M, int K, const fg_qtensor *w, const fg_half *bias,
                          const fg_half *residual, int flags, int qscale_cols, float qscale,
                          fg_half *y, void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------- */
/* W4A8 linear layer: 4-bit weights, 8-bit activations, integer products   */
/* ---------------------------------------------------------------------- */
/* [Q8] The pages name W4A8 only through the QServe W4A8KV4 title in the PIPO paper's list of
 * references, and list INT8 and INT4 among post-training weight formats ("Optimizing LLM for
 * low memory usage", Quantization and Weight Compression); groups of 64 along the input
 * dimension as in [G3].  The scheme (a reading of those pages):
 *   weights [N][K], two levels: per row n, cscale = amax / 113 and w8 = clamp(round_half_even(
 *     w * (113 / amax)), -113, 113) (each one IEEE fp32 operation; amax = 0 gives cscale 0 and
 *     w8 0); per group g of 64 along k, gmin = min w8, gstep = max(1, ceil((max w8 - gmin) / 15))
 *     (1..16) and code = floor((2 (w8 - gmin) + gstep) / (2 gstep)) (0..15), two codes per byte,
 *     the even element in the low nibble.  The product's weight is gmin + code * gstep, an int8
 *     for every group (gmin + 15 gstep <= max w8 + 14 <= 127);
 *   activations [M][K]: per row t, ascale = amax / 127, a8 = clamp(round_half_even(x * (127 /
 *     amax)), -127, 127) (amax = 0: ascale 0, a8 0);
 *   y[t][n] = epi( acc * (ascale[t] * cscale[n]) + bias[n] ), acc = sum_k a8[t][k] *
 *     (gmin + code * gstep)[n][k] exact in int32 on the tensor cores (tcgen05 kind::i8), then one
 *     fp32 operation at a time: the scale product, acc * it, + bias, q-scale of the first
 *     qscale_cols outputs, ReLU (FG_EPI_RELU), + residual (FG_EPI_RESIDUAL), round to fp16. */
typedef struct {
    uint8_t *codes;   /* [N][K/2] */
    int8_t *gmin;     /* [N][K/64] */
    uint8_t *gstep;   /* [N][K/64], 1..16 (other values give unspecified results) */
    float *cscale;    /* [N] */
    int64_t N, K;
} fg_w4a8_weight;
/* Quantises fp16 weights w [N][K] (device, row-major, 16-byte aligned) into *out (device arrays
 * the caller owns, codes 16-byte aligned, cscale 4-byte aligned).  K % 64 == 0, N >= 1
 * (FG_ERR_SHAPE otherwise).  One CTA per row. */
FG_API fg_status fg_w4a8_quantize_weight(const fg_half *w, const fg_w4a8_weight *out, void *stream);
/* Quantises fp16 activations x [M][K] (device, 16-byte aligned) to a8 [M][K] (16-byte aligned)
 * and ascale [M] (fp32).  K % 64 == 0 (FG_ERR_SHAPE otherwise).  One CTA per row. */
FG_API fg_status fg_act8_quantize(const fg_half *x, int M, int K, int8_t *a8, float *ascale, void *stream);
/* The W4A8 product above: a8 [M][K] int8 and ascale [M] from fg_act8_quantize, w from
 * fg_w4a8_quantize_weight with w->K == K, bias fp16 [N] or NULL, residual fp16 [M][N].
 * K % 128 == 0 and K <= 65536 (the int32 sums stay exact), N % 128 == 0 (FG_ERR_SHAPE);
 * a8, y, the residual and the codes 16-byte aligned, gmin, gstep and bias 2-byte aligned,
 * cscale and ascale 4-byte aligned (FG_ERR_INVALID).  M <= 256: one SM per output tile of 256 features x tile_tokens tokens, the
 * k-range possibly split over a cluster whose CTAs add their int32 partials exactly.  M > 256,
 * (K / 64) % 16 == 0 and gmin, gstep 16-byte aligned: the CTA-pair launch of fg_linear_w4a16 in
 * its int8 form (256- or 512-token tiles, k-tiles of 128); its k splits add int32 partials
 * through the optional workspace (fg_linear_w4a8_workspace_bytes; the split ranks then meet
 * through flags when the grid fits one wave) or over distributed shared memory.  Integer sums are
 * exact in every launch, so the result does not depend on the plan or the scratch. */
FG_API fg_status fg_linear_w4a8(const int8_t *a8, const float *ascale, int M, int K, const fg_w4a8_weight *w,
                         const fg_half *bias, const fg_half *residual, int flags, int qscale_cols,
                         float qscale, fg_half *y, void *workspace, size_t workspace_bytes, void *stream);
/* Scratch the CTA-pair launch of fg_linear_w4a8 can use for this shape (0: none). */
FG_API size_t fg_linear_w4a8_workspace_bytes(int M, int N, int K);
/* The launch fg_linear_w4a8 makes for this shape on the current device, assuming 16-byte aligned
 * metadata (no launch): *tile_tokens (16..256 one SM per tile, 256 or 512 a CTA pair per tile) and
 * *splits (1..8, 1..4 for pairs); FG_ERR_INVALID for shapes it rejects. */
FG_API fg_status fg_linear_w4a8_plan(int M, int N, int K, int *tile_tokens, int *splits);

/* y = (x - mean) / sqrt(var + eps) * gamma + beta per row (fp32 statistics,
 * biased variance), fp16 in/out, gamma/beta fp16 [h] (NULL = 1 / 0).
 * h % 8 == 0; x, y, gamma and beta 16-byte aligned (FG_ERR_INVALID otherwise).  [OPT] */
FG_API fg_status fg_layernorm(const fg_half *x, int M, int h, const fg_half *gamma, const fg_half *beta,
                       float eps, fg_half *y, void *stream);

/* ---------------------------------------------------------------------- */
/* One OPT decoder layer over a block of GPU batches [G2][G3][OPT]         */
/* ---------------------------------------------------------------------- */

typedef struct {
    int32_t hidden;     /* h = num_heads * head_dim, multiple of 128 */
    int32_t num_heads;
    int32_t head_dim;   /* 64, 128 or 256 */
    int32_t ffn;        /* F, multiple of 128 */
    float ln_eps;       /* 1e-5 for OPT */
    int32_t group;      /* 4-bit group of the weights and the KV cache: 64 or 128 (0 = 64) [G3] */
    int32_t act_bits;   /* what the products multiply the weights with: 16 (or 0): fp16 activations,
                         * W4 weights of the format above (W4A16); 8: int8 activations, one scale
                         * per row, and weights in the W4A8 form of fg_w4a8_quantize_weight
                         * (W4A8 [Q8]; group 64, the KV cache unchanged) */
} fg_layer_config;

/* Compressed weights of one layer.  Matrices are packed along their input
 * dim (dim 1) in groups of the config's group: wqkv [3h][h] (rows: q, then k,
 * then v, each head-major), wo [h][h], w1 [F][h], w2 [h][F].  Vectors fp16:
 * bqkv [3h], bo [h], b1 [F], b2 [h], ln1_g/ln1_b/ln2_g/ln2_b [h].  All device
 * pointers.  W4A8 layers (act_bits 8): a matrix's `mins` holds its int8 group
 * minima and `scales` its uint8 group steps (fg_w4a8_weight's gmin and gstep),
 * and cscale[i] its fp32 row scales (i: wqkv, wo, w1, w2; NULL for W4A16). */
typedef struct {
    fg_qtensor wqkv, wo, w1, w2;
    fg_half *bqkv, *bo, *b1, *b2;
    fg_half *ln1_g, *ln1_b, *ln2_g, *ln2_b;
    float *cscale[4];
} fg_layer_weights;

/* Size of one layer's contiguous weight blob (every array at a 256-byte
 * aligned offset), so a layer moves host->device with one copy [G1]. */
FG_API size_t fg_layer_blob_bytes(const fg_layer_config *c);

/* Points `out` into a blob of fg_layer_blob_bytes(c) bytes at `blob`
 * (any memory; no data is touched). */
FG_API fg_status fg_layer_weights_from_blob(const fg_layer_config *c, void *blob, fg_layer_weights *out);

/* Device scratch for fg_layer_decode / fg_layer_prefill over `rows`
 * hidden-state rows (the block's sequences, or sequences * prompt length):
 * the intermediate activations, then the GEMMs' scratch (fg_linear_w4a16 /
 * fg_linear_w4a8).  The activations, each at the next 256-byte aligned
 * offset from the start, fp16 row-major: a [rows][h] (LN1, then LN2 output),
 * qkv [rows][3h], o [rows][h] (attention output), h1 [rows][h], f [rows][F]
 * (ReLU output); W4A8 layers then a8 [rows][max(h, F)] int8 and as [rows]
 * fp32 (the last product's quantised input and row scales).  After a call
 * they hold that call's values (of the last chunk of a prefill).
 * A call needs at least the activations' part and gives the GEMMs whatever
 * follows it; the GEMMs add split k-ranges on chip when it is short, with the
 * same bits. */
FG_API size_t fg_layer_workspace_bytes(const fg_layer_config *c, int rows);

/* One decode step of one layer for every sequence of a block of
 * num_gpu_batches * gpu_batch_size sequences (batch j = rows
 * [j*gpu_batch_size, (j+1)*gpu_batch_size)).  The layer's weights are loaded
 * once and reused by all batches of the block [G2]: each GEMM runs over all
 * the block's rows, so the result of a row does not depend on the batch split.
 *   x_in, x_out: fp16 device [S][h] (S = num_gpu_batches * gpu_batch_size)
 *   positions: int32 device [S], the cache position of the new token of each
 *              sequence (= number of tokens already cached).
 * Steps: a = LN1(x); [q k v] = a Wqkv^T + bqkv, q *= head_dim^-1/2;
 * append k, v to the 4-bit cache at positions; o = attention over positions
 * 0..pos; h1 = x + o Wo^T + bo; x_out = h1 + relu(LN2(h1) W1^T + b1) W2^T + b2.
 * kv->num_seqs must equal S and kv->group the config's group.  Positions are
 * not advanced by the call.  W4A8 layers (act_bits 8): each product's input
 * (a, o, LN2(h1), the ReLU output) is quantised to int8 per row first
 * (fg_act8_quantize) and multiplied with fg_linear_w4a8. */
FG_API fg_status fg_layer_decode(const fg_layer_config *c, const fg_layer_weights *w, const fg_kv_cache *kv,
                          const fg_half *x_in, fg_half *x_out, const int32_t *positions,
                          int num_gpu_batches, int gpu_batch_size,
                          void *workspace, size_t workspace_bytes, void *stream);

/* The same layer over a prompt of prompt_len tokens per sequence:
 * x_in, x_out fp16 device [S][prompt_len][h]; token t of sequence s is
 * appended at positions[s] + t and attends over 0 .. positions[s] + t. */
FG_API fg_status fg_layer_prefill(const fg_layer_config *c, const fg_layer_weights *w, const fg_kv_cache *kv,
                           const fg_half *x_in, fg_half *x_out, const int32_t *positions, int prompt_len,
                           int num_gpu_batches, int gpu_batch_size,
                           void *workspace, size_t workspace_bytes, void *stream);

/* fg_layer_decode for callers that cannot allocate device memory -- a serving
 * process that reserved all device memory up front, a host that only passes
 * pointers it already owns, or a loop that must not allocate between steps.
 * (The pages have no counterpart: this is a deployment convenience.)  The step's
 * scratch lives in a static device array of FG_NOALLOC_SCRATCH_BYTES (96 MiB)
 * that every GPU loading the library holds until the process exits; the caller
 * still passes weights, cache, inputs and outputs, as for fg_layer_decode, whose
 * computation this is, bit for bit.
 *   - Returns FG_ERR_WORKSPACE, before any launch, when the block's whole
 *     workspace, fg_layer_workspace_bytes(c, S), exceeds the array (the
 *     OPT-6.7B-shaped block of 512 sequences needs about 78 MB);
 *     FG_ERR_SHAPE when num_gpu_batches * gpu_batch_size exceeds INT_MAX.
 *   - Set-up: the first call on each device looks up the array's device
 *     address with that device current.  Under CUDA's lazy module loading (the
 *     default) that lookup is also when the array's memory is taken, and each
 *     kernel's code is loaded at its first launch.  A caller that reserves all
 *     device memory up front therefore makes one ordinary call first (one step
 *     on any block; a call with zero sequences sets up the array alone), before
 *     reserving and before any stream capture.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     nothing in it has to start at zero (each step writes what it reads).
 *     Calls whose work overlaps on the GPU (other streams, other threads)
 *     race on it: serialise them.
 *   - After that first call it allocates nothing (keep fg_profile_enable off:
 *     profiling creates events). */
#define FG_NOALLOC_SCRATCH_BYTES (96u << 20)
FG_API fg_status fg_layer_decode_noalloc(const fg_layer_config *c, const fg_layer_weights *w,
                                         const fg_kv_cache *kv, const fg_half *x_in, fg_half *x_out,
                                         const int32_t *positions, int num_gpu_batches, int gpu_batch_size,
                                         void *stream);

/* Per-kernel timing of layer calls.  While enabled, each kernel that
 * fg_layer_decode / fg_layer_prefill launch is bracketed by CUDA events on
 * the call's stream (no synchronisation added).  fg_profile_collect waits for
 * those events and writes, per kernel slot, the summed milliseconds and the
 * number of launches, then forgets them.  Slots: 0 LN1, 1 QKV GEMM, 2 KV
 * append, 3 attention, 4 out-proj GEMM, 5 LN2, 6 FC1 GEMM, 7 FC2 GEMM; W4A8
 * layers also 8..11, the activation quantisers before QKV, out-proj, FC1 and
 * FC2. */
#define FG_PROFILE_SLOTS 12
FG_API fg_status fg_profile_enable(int enable);
FG_API fg_status fg_profile_collect(float *ms, int *count, int nslots);

/* ---------------------------------------------------------------------- */
/* Layer stack with weights streamed from pinned host memory [G1][G2]      */
/* ---------------------------------------------------------------------- */

typedef struct fg_stack fg_stack;  /* opaque */

/* Prepares a stack of num_layers layers whose blobs live in host memory
 * (host_blobs[l], fg_layer_blob_bytes(c) each; pinned for overlap).  A blob
 * in device memory (256-byte aligned) keeps its layer resident: read in
 * place, no copy, no staging buffer [G1: part of the weights placed on the
 * GPU].
 * dev_staging[0..1]: two device buffers of fg_layer_blob_bytes(c) bytes that
 * the next layer is prefetched into while the current one computes.  The same
 * buffer given twice, of fg_stack_one_buffer_bytes(c) bytes, selects one
 * staging buffer: each matrix of layer l+1 is then copied once layer l's
 * kernels that read that matrix have run, and the vectors (biases, LayerNorm
 * parameters) alternate between two slots (about half the staging memory;
 * fg_stack_decode_host_kv needs two buffers and returns FG_ERR_UNSUPPORTED
 * with one).
 * Creates CUDA events only (no memory allocation).  *out is released with
 * fg_stack_destroy. */
/* Bytes of the one staging buffer of a one-buffer stack: the blob, then a second slot for the
 * vectors (0 for a configuration the library rejects). */
FG_API size_t fg_stack_one_buffer_bytes(const fg_layer_config *c);
FG_API fg_status fg_stack_create(const fg_layer_config *c, int num_layers, void *const *host_blobs,
                          void *dev_staging0, void *dev_staging1, fg_stack **out);

/* One decode step through all layers: layer l computes on compute_stream
 * from staging buffer l%2 while copy_stream copies layer l+1's blob into the
 * other buffer (events order the two).  kv: array of num_layers caches.
 * x_in/x_out/positions/block as fg_layer_decode; x_in and x_out may alias. */
FG_API fg_status fg_stack_decode(fg_stack *st, const fg_kv_cache *kv, const fg_half *x_in, fg_half *x_out,
                          const int32_t *positions, int num_gpu_batches, int gpu_batch_size,
                          void *workspace, size_t workspace_bytes, void *compute_stream, void *copy_stream);

/* As fg_stack_decode for a prompt (see fg_layer_prefill). */
FG_API fg_status fg_stack_prefill(fg_stack *st, const fg_kv_cache *kv, const fg_half *x_in, fg_half *x_out,
                           const int32_t *positions, int prompt_len, int num_gpu_batches, int gpu_batch_size,
                           void *workspace, size_t workspace_bytes, void *compute_stream, void *copy_stream);

/* One decode step with every layer's KV cache in host memory, for stacks whose
 * cache does not fit in HBM ([G1] section 2: the KV cache is offloaded with
 * the weights; [G3]: it stays in 4-bit form while it moves).
 * host_kv: array of num_layers caches in pinned host memory (same geometry).
 * dev_kv: two device caches of that geometry, used as staging: layer l runs on
 * dev_kv[l%2].  Per layer, copy_stream copies the weight blob and positions
 * [0, fill_len) of host_kv[l] into staging buffer l%2, one strided
 * cudaMemcpy2DAsync per cache array; after the layer it copies positions
 * [wb_begin, wb_end) (the slots this step appended) back to host_kv[l].
 * Events order the two streams, so the fill of layer l+1 and the write-back of
 * layer l-1 overlap the compute of layer l.  Slots past a sequence's length in
 * a staging cache may hold another layer's data; attention never reads them.
 * The write-back copies whole position slices for every sequence, so a slot in
 * [wb_begin, wb_end) that this step does not append must lie below fill_len
 * (with equal positions p: fill_len = p, wb = [p, p+1); ragged: fill_len =
 * max p + 1, wb = [min p, max p + 1)).  compute_stream waits for the last
 * write-back, so work enqueued on it afterwards sees every host cache updated.
 * Other arguments as fg_stack_decode.  Returns FG_ERR_SHAPE when the caches'
 * geometries differ or the block has more sequences than a cache,
 * FG_ERR_INVALID for fill/write-back ranges outside [0, max_len). */
FG_API fg_status fg_stack_decode_host_kv(fg_stack *st, const fg_kv_cache *host_kv, const fg_kv_cache *dev_kv,
                                  int fill_len, int wb_begin, int wb_end, const fg_half *x_in, fg_half *x_out,
                                  const int32_t *positions, int num_gpu_batches, int gpu_batch_size,
                                  void *workspace, size_t workspace_bytes, void *compute_stream,
                                  void *copy_stream);

/* Test hook of the kernels' bounded waits (failure detection without a GPU
 * fault).  The next `count` launches of the one-SM W4A16 GEMM (fg_linear_w4a16
 * with M <= 256) run with every pipeline wait limited to wait_limit_ns
 * nanoseconds (1 .. 2e9) instead of 2 s, and their dequantising warps withhold
 * their arrival on the first pipeline stage, so the tensor-core issuer's wait
 * for that stage cannot complete.  Such a launch gives up after the limit,
 * stops issuing, waits for its copies in flight, frees its tensor memory and
 * flags FG_ERR_TIMEOUT (reported by fg_sync_status); its output is
 * unspecified.  Later launches run normally. */
FG_API fg_status fg_test_gemm_stall(int count, uint64_t wait_limit_ns);

/* Test hook: the next `count` blob copies of this stack report a copy
 * failure (no copy is issued), as if cudaMemcpyAsync had failed. */
FG_API fg_status fg_stack_inject_copy_failure(fg_stack *st, int count);

FG_API fg_status fg_stack_destroy(fg_stack *st);

#ifdef __cplusplus
}
#endif
#endif /* FG_H_ */
