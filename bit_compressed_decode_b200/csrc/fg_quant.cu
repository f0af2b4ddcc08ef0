// fg_quant.cu -- group-wise 4-bit (and 8-bit) quantise (pack), dequantise and the 4-bit KV append.
//
// Format and fp32 operation order: "FlexGen Guide: High-Throughput LLM Offloading on
// One GPU", section 3 (Group-Wise 4-Bit Quantization for Weights and KV Cache), read
// as stated in fg.h.  All three kernels are HBM-bound streaming kernels: 16-byte
// coalesced loads, a group of 64 (or 128) values spread over 8 (or 16) lanes whose
// min/max is found with warp shuffles, 32-bit packed code stores, grids sized in whole
// waves of the SM count.  The KV cache always uses groups of 64 along head_dim.
#include "fg_internal.cuh"

namespace {

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

// Grid of whole waves: `per_sm` blocks per SM, capped by the work available.
unsigned grid_for(int64_t work_blocks, int per_sm) {
  int64_t g = static_cast<int64_t>(num_sms()) * per_sm;
  if (work_blocks < g) g = work_blocks;
  return static_cast<unsigned>(g < 1 ? 1 : g);
}

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }

// ------------------------------------------------------------------------------------
// K1: quantise along the last dim.  x: [ngroups][G] fp16 (as uint4 = 8 halves);
// codes: [ngroups][G/2] bytes (as uint32 = 8 codes); mins/scales [ngroups].  G/8 lanes
// per group: a warp handles 32/(G/8) groups per step and U steps per loop trip (loads
// issued first).
// ------------------------------------------------------------------------------------
constexpr int kQU = 4;

template <int G, int B>  // B: code width, 4 (two codes per byte) or 8 (one)
__global__ void __launch_bounds__(256) quantize_lastdim_kernel(const uint4 *__restrict__ x, int64_t ngroups,
                                                               uint32_t *__restrict__ codes,
                                                               __half *__restrict__ mins,
                                                               __half *__restrict__ scales) {
  constexpr int L = G / 8, GPW = 32 / L;  // lanes per group, groups per warp step
  const int lane = threadIdx.x & 31;
  const int slot = lane / L, j = lane % L;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t g0 = warp * GPW * kQU; g0 < ngroups; g0 += nwarps * GPW * kQU) {
    uint4 v[kQU];
#pragma unroll
    for (int u = 0; u < kQU; u++) {
      const int64_t g = g0 + u * GPW + slot;
      v[u] = g < ngroups ? ld_stream(x + g * L + j) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kQU; u++) {
      const int64_t g = g0 + u * GPW + slot;
      __half mn, sc;
      if constexpr (B == 8) {
        const uint2 w = quant_group8_u8<L>(v[u], mn, sc);
        if (g < ngroups) {
          reinterpret_cast<uint2 *>(codes)[g * L + j] = w;
          if (j == 0) {
            mins[g] = mn;
            scales[g] = sc;
          }
        }
      } else {
        const uint32_t w = quant_group8<L>(v[u], mn, sc);
        if (g < ngroups) {
          codes[g * L + j] = w;
          if (j == 0) {
            mins[g] = mn;
            scales[g] = sc;
          }
        }
      }
    }
  }
}

// K2: dequantise along the last dim; one thread per 8 codes (one 16-byte output).  G/8
// such chunks share a group's min and scale.
template <int G, int B>
__global__ void __launch_bounds__(256) dequantize_lastdim_kernel(const uint32_t *__restrict__ codes,
                                                                 const __half *__restrict__ mins,
                                                                 const __half *__restrict__ scales,
                                                                 int64_t nchunks, uint4 *__restrict__ y) {
  // chunk c = 8 codes: one 32-bit word (4-bit codes) or two (8-bit codes)
  auto deq = [&](int64_t c) {
    const __half2 s2 = __half2half2(scales[c / (G / 8)]), m2 = __half2half2(mins[c / (G / 8)]);
    if constexpr (B == 8) return dequant8_u8(__ldcs(reinterpret_cast<const uint2 *>(codes) + c), s2, m2);
    else return dequant8(__ldcs(codes + c), s2, m2);
  };
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if constexpr (B == 8) {
    for (; i + 3 * stride < nchunks; i += 4 * stride) {
      uint2 w[4];
      __half mn[4], sc[4];
#pragma unroll
      for (int u = 0; u < 4; u++) {
        const int64_t c = i + u * stride;
        w[u] = __ldcs(reinterpret_cast<const uint2 *>(codes) + c);
        mn[u] = mins[c / (G / 8)];
        sc[u] = scales[c / (G / 8)];
      }
#pragma unroll
      for (int u = 0; u < 4; u++) __stcs(y + i + u * stride, dequant8_u8(w[u], __half2half2(sc[u]), __half2half2(mn[u])));
    }
  } else {
    for (; i + 3 * stride < nchunks; i += 4 * stride) {
      uint32_t w[4];
      __half mn[4], sc[4];
#pragma unroll
      for (int u = 0; u < 4; u++) {
        const int64_t c = i + u * stride;
        w[u] = __ldcs(codes + c);
        mn[u] = mins[c / (G / 8)];
        sc[u] = scales[c / (G / 8)];
      }
#pragma unroll
      for (int u = 0; u < 4; u++) __stcs(y + i + u * stride, dequant8(w[u], __half2half2(sc[u]), __half2half2(mn[u])));
    }
  }
  for (; i < nchunks; i += stride) __stcs(y + i, deq(i));
}

// ------------------------------------------------------------------------------------
// Strided variants (grouping dim is not the last one): x viewed as [outer][n][inner],
// one thread per group, consecutive threads on consecutive inner positions.
// ------------------------------------------------------------------------------------
template <int G, int B>
__global__ void __launch_bounds__(256) quantize_strided_kernel(const __half *__restrict__ x, int64_t outer,
                                                               int64_t n, int64_t inner,
                                                               uint8_t *__restrict__ codes,
                                                               __half *__restrict__ mins,
                                                               __half *__restrict__ scales) {
  const int64_t ng = n / G;
  const int64_t total = outer * ng * inner;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = t % inner, g = (t / inner) % ng, o = t / (inner * ng);
    const __half *xp = x + (o * n + g * G) * inner + i;
    float v[G];
    float mn, mx;
#pragma unroll
    for (int e = 0; e < G; e++) v[e] = __half2float(xp[e * inner]);
    mn = v[0];
    mx = v[0];
#pragma unroll
    for (int e = 1; e < G; e++) {
      mn = fminf(mn, v[e]);
      mx = fmaxf(mx, v[e]);
    }
    mn = __fadd_rn(mn, 0.0f);
    const float d = __fsub_rn(mx, mn);
    constexpr int kLevels = (1 << B) - 1;
    __half sh = __float2half_rn(__fdiv_rn(d, static_cast<float>(kLevels)));
    const float s = __half2float(sh);
    uint8_t *cp = codes + (o * (n * B / 8) + g * (G * B / 8)) * inner + i;
    if (s != 0.0f) {
      const float inv = __fdiv_rn(1.0f, s);
#pragma unroll
      for (int e = 0; e < G; e += 2) {
        int c0 = min(max(__float2int_rn(__fmul_rn(__fsub_rn(v[e], mn), inv)), 0), kLevels);
        int c1 = min(max(__float2int_rn(__fmul_rn(__fsub_rn(v[e + 1], mn), inv)), 0), kLevels);
        if constexpr (B == 8) {
          cp[e * inner] = static_cast<uint8_t>(c0);
          cp[(e + 1) * inner] = static_cast<uint8_t>(c1);
        } else {
          cp[(e / 2) * inner] = static_cast<uint8_t>(c0 | (c1 << 4));
        }
      }
    } else {
      sh = __ushort_as_half(0);
#pragma unroll
      for (int e = 0; e < G * B / 8; e++) cp[e * inner] = 0;
    }
    const int64_t m = (o * ng + g) * inner + i;
    mins[m] = __float2half_rn(mn);
    scales[m] = sh;
  }
}

template <int G, int B>
__global__ void __launch_bounds__(256) dequantize_strided_kernel(const uint8_t *__restrict__ codes,
                                                                 const __half *__restrict__ mins,
                                                                 const __half *__restrict__ scales,
                                                                 int64_t outer, int64_t n, int64_t inner,
                                                                 __half *__restrict__ y) {
  if constexpr (B == 8) {  // one thread per code byte (1 element): fp16_rn(min + code * scale)
    const int64_t total = outer * n * inner;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const int64_t i = t % inner, e = (t / inner) % n, o = t / (inner * n);
      const int64_t m = (o * (n / G) + e / G) * inner + i;
      const __half c = __hsub(__ushort_as_half(static_cast<unsigned short>(0x6400u | codes[t])),
                              __ushort_as_half(0x6400));
      y[t] = __hfma(c, scales[m], mins[m]);
    }
    return;
  }
  const int64_t total = outer * (n / 2) * inner;  // one thread per code byte (2 elements)
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = t % inner, jb = (t / inner) % (n / 2), o = t / (inner * (n / 2));
    const uint32_t b = codes[t];
    const int64_t m = (o * (n / G) + (2 * jb) / G) * inner + i;
    const __half2 s2 = __half2half2(scales[m]), m2 = __half2half2(mins[m]);
    __half2 c = __hsub2(nib2_plus1024((b & 0xFu) | ((b & 0xF0u) << 12)),
                        __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
    __half2 r = __hfma2(c, s2, m2);
    y[(o * n + 2 * jb) * inner + i] = __low2half(r);
    y[(o * n + 2 * jb + 1) * inner + i] = __high2half(r);
  }
}

// ------------------------------------------------------------------------------------
// K5: append new k, v rows to the 4-bit cache.  Work unit = one G-group (64 or 128) of k or
// v of one head of one row; G/8 lanes per unit, 32/(G/8) units per warp step.
// ------------------------------------------------------------------------------------
struct KvArgs {
  uint32_t *kc, *vc;  // codes as 32-bit words
  __half *km, *ks, *vm, *vs;
  int H, d, maxL, num_seqs;
};

template <int G>
__global__ void __launch_bounds__(256) kv_append_kernel(const __half *__restrict__ k, const __half *__restrict__ v,
                                                        int64_t ld, int rows, int rows_per_seq,
                                                        const int32_t *__restrict__ positions, KvArgs a,
                                                        unsigned int *err) {
  // A warp takes one (row, head) item per step: its 2 * d/G units (k and v groups), USTEP at
  // a time in its G/8-lane slots; unit us = group * 2 + (0 for k, 1 for v).
  constexpr int L = G / 8, USTEP = 32 / L;
  // launched as a dependent of the GEMM that produces k and v (decode steps): they are read
  // only once it has completed
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int slot = lane / L, j = lane % L;
  const int ng = a.d / G;
  const int items = rows * a.H;
  const int warp = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int nwarps = static_cast<int>((static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5);
  for (int item = warp; item < items; item += nwarps) {
    const int r = item / a.H, hd = item - r * a.H;
    const int s = r / rows_per_seq;
    const int pos = positions[s] + (r - s * rows_per_seq);
    const bool in_range = pos >= 0 && pos < a.maxL;
    const int64_t slot_idx = (static_cast<int64_t>(s) * a.H + hd) * a.maxL + pos;
    for (int u0 = 0; u0 < 2 * ng; u0 += USTEP) {  // warp-uniform
      const int us = u0 + slot;
      const bool live = us < 2 * ng;
      const int which = us & 1, g = us >> 1;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (live) val = *reinterpret_cast<const uint4 *>((which ? v : k) + static_cast<int64_t>(r) * ld + hd * a.d +
                                                       g * G + j * 8);
      __half mn, sc;
      const uint32_t w = quant_group8<L>(val, mn, sc);
      if (!live) continue;
      if (!in_range) {
        if (j == 0) atomicOr(err, FG_DEVERR_RANGE);
        continue;
      }
      (which ? a.vc : a.kc)[slot_idx * (a.d / 8) + g * L + j] = w;
      if (j == 0) {
        const int64_t m = slot_idx * ng + g;
        (which ? a.vm : a.km)[m] = mn;
        (which ? a.vs : a.ks)[m] = sc;
      }
    }
  }
}

bool shape_numel(int ndim, const int64_t *shape, int64_t *numel) {
  int64_t n = 1;
  for (int i = 0; i < ndim; i++) {
    if (shape[i] < 0) return false;
    n *= shape[i];
  }
  *numel = n;
  return true;
}

}  // namespace

// ======================================================================================
// C ABI
// ======================================================================================

extern "C" fg_status fg_qtensor_bytes(int ndim, const int64_t *shape, int dim, int bits, int group,
                                      size_t *codes_bytes, size_t *meta_bytes) {
  if (!shape || ndim < 1 || ndim > 4 || dim < 0 || dim >= ndim) return FG_ERR_INVALID;
  if ((bits != 4 && bits != 8) || (group != 64 && group != 128)) return FG_ERR_UNSUPPORTED;
  int64_t numel;
  if (!shape_numel(ndim, shape, &numel)) return FG_ERR_INVALID;
  if (shape[dim] % group) return FG_ERR_SHAPE;
  if (codes_bytes) *codes_bytes = static_cast<size_t>(numel / 8 * bits);
  if (meta_bytes) *meta_bytes = static_cast<size_t>(numel / group) * 2;
  return FG_OK;
}

extern "C" fg_status fg_quantize(const fg_half *x, int ndim, const int64_t *shape, int dim, int bits, int group,
                                 fg_qtensor *out, void *stream) {
  if (!out) return FG_ERR_INVALID;
  fg_status rc = fg_qtensor_bytes(ndim, shape, dim, bits, group, nullptr, nullptr);
  if (rc != FG_OK) return rc;
  int64_t numel;
  shape_numel(ndim, shape, &numel);
  out->ndim = ndim;
  for (int i = 0; i < 4; i++) out->shape[i] = i < ndim ? shape[i] : 1;
  out->dim = dim;
  out->bits = bits;
  out->group = group;
  if (numel == 0) return FG_OK;
  if (!x || !out->codes || !out->mins || !out->scales) return FG_ERR_INVALID;
  int64_t outer = 1, inner = 1;
  for (int i = 0; i < dim; i++) outer *= shape[i];
  for (int i = dim + 1; i < ndim; i++) inner *= shape[i];
  const int64_t n = shape[dim];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (inner == 1) {
    if (!fg_aligned16(x) || !fg_aligned16(out->codes) || (reinterpret_cast<uintptr_t>(out->mins) & 1) ||
        (reinterpret_cast<uintptr_t>(out->scales) & 1))
      return FG_ERR_INVALID;
    const int64_t ngroups = numel / group;
    const int gpw = 32 / (group / 8);  // groups per warp step
    const int64_t warps_needed = (ngroups + gpw * kQU - 1) / (gpw * kQU);
    auto kern = bits == 8 ? (group == 128 ? quantize_lastdim_kernel<128, 8> : quantize_lastdim_kernel<64, 8>)
                          : (group == 128 ? quantize_lastdim_kernel<128, 4> : quantize_lastdim_kernel<64, 4>);
    kern<<<grid_for((warps_needed + 7) / 8, 8), 256, 0, st>>>(
        reinterpret_cast<const uint4 *>(x), ngroups, reinterpret_cast<uint32_t *>(out->codes),
        reinterpret_cast<__half *>(out->mins), reinterpret_cast<__half *>(out->scales));
  } else {
    if ((reinterpret_cast<uintptr_t>(x) & 1) || (reinterpret_cast<uintptr_t>(out->mins) & 1) ||
        (reinterpret_cast<uintptr_t>(out->scales) & 1))
      return FG_ERR_INVALID;
    const int64_t groups = outer * (n / group) * inner;
    auto kern = bits == 8 ? (group == 128 ? quantize_strided_kernel<128, 8> : quantize_strided_kernel<64, 8>)
                          : (group == 128 ? quantize_strided_kernel<128, 4> : quantize_strided_kernel<64, 4>);
    kern<<<grid_for((groups + 255) / 256, 8), 256, 0, st>>>(
        reinterpret_cast<const __half *>(x), outer, n, inner, out->codes, reinterpret_cast<__half *>(out->mins),
        reinterpret_cast<__half *>(out->scales));
  }
  return fg_launch_check();
}

extern "C" fg_status fg_dequantize(const fg_qtensor *q, fg_half *y, void *stream) {
  if (!q) return FG_ERR_INVALID;
  fg_status rc = fg_qtensor_bytes(q->ndim, q->shape, q->dim, q->bits, q->group, nullptr, nullptr);
  if (rc != FG_OK) return rc;
  int64_t numel;
  shape_numel(q->ndim, q->shape, &numel);
  if (numel == 0) return FG_OK;
  if (!y || !q->codes || !q->mins || !q->scales) return FG_ERR_INVALID;
  int64_t outer = 1, inner = 1;
  for (int i = 0; i < q->dim; i++) outer *= q->shape[i];
  for (int i = q->dim + 1; i < q->ndim; i++) inner *= q->shape[i];
  const int64_t n = q->shape[q->dim];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (inner == 1) {
    // chunks of 8 codes: one aligned word (4-bit codes) or two (8-bit codes)
    if (!fg_aligned16(y) || (reinterpret_cast<uintptr_t>(q->codes) & (q->bits == 8 ? 7 : 3))) return FG_ERR_INVALID;
    const int64_t nchunks = numel / 8;
    auto kern = q->bits == 8
                    ? (q->group == 128 ? dequantize_lastdim_kernel<128, 8> : dequantize_lastdim_kernel<64, 8>)
                    : (q->group == 128 ? dequantize_lastdim_kernel<128, 4> : dequantize_lastdim_kernel<64, 4>);
    kern<<<grid_for((nchunks + 255) / 256, 8), 256, 0, st>>>(
        reinterpret_cast<const uint32_t *>(q->codes), reinterpret_cast<const __half *>(q->mins),
        reinterpret_cast<const __half *>(q->scales), nchunks, reinterpret_cast<uint4 *>(y));
  } else {
    const int64_t total = outer * (n * q->bits / 8) * inner;  // one thread per code byte
    auto kern = q->bits == 8
                    ? (q->group == 128 ? dequantize_strided_kernel<128, 8> : dequantize_strided_kernel<64, 8>)
                    : (q->group == 128 ? dequantize_strided_kernel<128, 4> : dequantize_strided_kernel<64, 4>);
    kern<<<grid_for((total + 255) / 256, 8), 256, 0, st>>>(
        q->codes, reinterpret_cast<const __half *>(q->mins), reinterpret_cast<const __half *>(q->scales), outer, n,
        inner, reinterpret_cast<__half *>(y));
  }
  return fg_launch_check();
}

extern "C" fg_status fg_kv_cache_bytes(int num_seqs, int num_heads, int head_dim, int max_len, int group,
                                       size_t *codes_bytes, size_t *meta_bytes) {
  if (num_seqs < 0 || num_heads < 1 || max_len < 0) return FG_ERR_INVALID;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return FG_ERR_UNSUPPORTED;
  const int G = fg_kv_group(group);
  if (G == 0) return FG_ERR_UNSUPPORTED;
  if (max_len % 64 || head_dim % G) return FG_ERR_SHAPE;
  const size_t slots = static_cast<size_t>(num_seqs) * num_heads * max_len;
  if (codes_bytes) *codes_bytes = slots * (head_dim / 2);
  if (meta_bytes) *meta_bytes = slots * (head_dim / G) * 2;
  return FG_OK;
}

fg_status fg_kv_validate(const fg_kv_cache *kv) {
  if (!kv) return FG_ERR_INVALID;
  fg_status rc = fg_kv_cache_bytes(kv->num_seqs, kv->num_heads, kv->head_dim, kv->max_len, kv->group, nullptr,
                                   nullptr);
  if (rc != FG_OK) return rc;
  const void *p[6] = {kv->k_codes, kv->k_mins, kv->k_scales, kv->v_codes, kv->v_mins, kv->v_scales};
  for (const void *ptr : p)
    if (!ptr || !fg_aligned16(ptr)) return FG_ERR_INVALID;
  return FG_OK;
}

// pdl: launch as a programmatic dependent of the kernel before (its launch overlaps that
// kernel's tail; the kernel waits for it before reading k and v).
fg_status fg_kv_append_launch(const fg_kv_cache *kv, const fg_half *k, const fg_half *v, int64_t ld, int rows,
                              int rows_per_seq, const int32_t *positions, cudaStream_t st, bool pdl) {
  KvArgs a;
  a.kc = reinterpret_cast<uint32_t *>(kv->k_codes);
  a.vc = reinterpret_cast<uint32_t *>(kv->v_codes);
  a.km = reinterpret_cast<__half *>(kv->k_mins);
  a.ks = reinterpret_cast<__half *>(kv->k_scales);
  a.vm = reinterpret_cast<__half *>(kv->v_mins);
  a.vs = reinterpret_cast<__half *>(kv->v_scales);
  a.H = kv->num_heads;
  a.d = kv->head_dim;
  a.maxL = kv->max_len;
  a.num_seqs = kv->num_seqs;
  unsigned int *err = fg_error_word_ptr();
  if (!err) return FG_ERR_CUDA;
  const int64_t items = static_cast<int64_t>(rows) * kv->num_heads;  // one warp per (row, head)
  if (items > INT32_MAX) return FG_ERR_SHAPE;
  auto kern = fg_kv_group(kv->group) == 128 ? kv_append_kernel<128> : kv_append_kernel<64>;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid_for((items + 7) / 8, 8), 1, 1);
  lc.blockDim = dim3(256, 1, 1);
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = pdl ? 1 : 0;
  const fg_status rc = fg_cuda_check(cudaLaunchKernelEx(&lc, kern, reinterpret_cast<const __half *>(k),
                                                        reinterpret_cast<const __half *>(v), ld, rows, rows_per_seq,
                                                        positions, a, err));
  if (rc != FG_OK) return rc;
  return fg_launch_check();
}

extern "C" fg_status fg_kv_append(const fg_kv_cache *kv, const fg_half *k, const fg_half *v, int64_t ld, int rows,
                                  int rows_per_seq, const int32_t *positions, void *stream) {
  fg_status rc = fg_kv_validate(kv);
  if (rc != FG_OK) return rc;
  if (rows < 0 || rows_per_seq < 1 || rows % rows_per_seq) return FG_ERR_SHAPE;
  if (rows / rows_per_seq > kv->num_seqs) return FG_ERR_SHAPE;
  if (rows == 0) return FG_OK;
  if (!k || !v || !positions || !fg_aligned16(k) || !fg_aligned16(v)) return FG_ERR_INVALID;
  if (ld < static_cast<int64_t>(kv->num_heads) * kv->head_dim || ld % 8) return FG_ERR_SHAPE;
  return fg_kv_append_launch(kv, k, v, ld, rows, rows_per_seq, positions, static_cast<cudaStream_t>(stream), false);
}
