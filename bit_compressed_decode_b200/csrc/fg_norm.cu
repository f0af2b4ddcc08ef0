// fg_norm.cu -- LayerNorm of fp16 rows (pre-LayerNorm OPT decoder layer; model family
// from the OPT entry of the PIPO paper's reference list).  fp32 statistics: mean, then
// the biased variance of (x - mean) from the values held in registers (two passes over
// registers, one read of HBM), y = (x - mean) * rsqrt(var + eps) * gamma + beta.
#include "fg_internal.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxVec = 8;  // up to 8 x 8 halves per thread: h <= 16384

// Sum over the CTA.  red holds two slots per warp used alternately (parity), so one barrier
// per reduction suffices: a slot is rewritten only two reductions later, after the barrier
// of the reduction in between.
__device__ __forceinline__ float block_sum(float v, float *red, int parity) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[parity * (kThreads / 32) + warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; w++) t += red[parity * (kThreads / 32) + w];
  return t;
}

__device__ __forceinline__ float block_max(float v, float *red, int parity) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[parity * (kThreads / 32) + warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; w++) t = fmaxf(t, red[parity * (kThreads / 32) + w]);
  return t;
}

// round-half-even of x * inv (one fp32 multiply), clamped to [-127, 127]
__device__ __forceinline__ uint32_t q8_byte(float x, float inv) {
  int c = __float2int_rn(__fmul_rn(x, inv));
  c = c < -127 ? -127 : (c > 127 ? 127 : c);
  return static_cast<uint32_t>(c) & 0xFFu;
}

// One CTA per row; VPT 8-element vectors per thread (h = 8 * 256 * VPT at most).  Q8: the
// row's fp16 output is also quantised to int8 with one scale (the W4A8 layer's activation
// quantiser, fg_act8_quantize's arithmetic: ascale = amax / 127, codes round(y * (127 / amax)))
// into a8 / ascale, saving that kernel's launch and its read of the row.
template <int VPT, bool Q8>
__global__ void __launch_bounds__(kThreads) layernorm_kernel(const uint4 *__restrict__ x, int h,
                                                             const uint4 *__restrict__ gamma,
                                                             const uint4 *__restrict__ beta, float eps,
                                                             uint4 *__restrict__ y, uint2 *__restrict__ a8,
                                                             float *__restrict__ ascale) {
  __shared__ float red[2 * (kThreads / 32)];
  griddep_launch();  // the GEMM after this kernel may start its weight-side prologue
  const int nvec = h / 8;
  const uint4 *xr = x + static_cast<int64_t>(blockIdx.x) * nvec;
  uint4 *yr = y + static_cast<int64_t>(blockIdx.x) * nvec;
  uint4 xv[VPT], gv[VPT], bv[VPT];
#pragma unroll
  for (int i = 0; i < VPT; i++) {  // every load is issued before any reduction
    const int idx = threadIdx.x + i * kThreads;
    const bool in = idx < nvec;
    xv[i] = in ? xr[idx] : make_uint4(0, 0, 0, 0);
    gv[i] = (in && gamma) ? gamma[idx] : make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);  // 1.0
    bv[i] = (in && beta) ? beta[idx] : make_uint4(0, 0, 0, 0);
  }
  float v[VPT][8];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; i++) {
    const __half2 *h2 = reinterpret_cast<const __half2 *>(&xv[i]);
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const float2 f = __half22float2(h2[j]);
      v[i][2 * j] = f.x;
      v[i][2 * j + 1] = f.y;
      sum += f.x + f.y;
    }
  }
  const float mean = block_sum(sum, red, 0) / h;
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; i++) {
    if (threadIdx.x + i * kThreads < nvec) {
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const float d = v[i][j] - mean;
        sq += d * d;
      }
    }
  }
  const float var = block_sum(sq, red, 1) / h;
  const float rstd = rsqrtf(var + eps);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; i++) {
    const int idx = threadIdx.x + i * kThreads;
    if (idx < nvec) {
      uint4 out;
      __half2 *o2 = reinterpret_cast<__half2 *>(&out);
      const __half2 *g2 = reinterpret_cast<const __half2 *>(&gv[i]);
      const __half2 *b2 = reinterpret_cast<const __half2 *>(&bv[i]);
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const float2 g = __half22float2(g2[j]), b = __half22float2(b2[j]);
        o2[j] = __floats2half2_rn((v[i][2 * j] - mean) * rstd * g.x + b.x, (v[i][2 * j + 1] - mean) * rstd * g.y + b.y);
        if constexpr (Q8) {  // keep the fp16 outputs for the codes
          const float2 f = __half22float2(o2[j]);
          v[i][2 * j] = f.x;
          v[i][2 * j + 1] = f.y;
          amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
      yr[idx] = out;
    }
  }
  if constexpr (Q8) {
    amax = block_max(amax, red, 0);
    const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
    if (threadIdx.x == 0) ascale[blockIdx.x] = amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
    uint2 *ar = a8 + static_cast<int64_t>(blockIdx.x) * nvec;
#pragma unroll
    for (int i = 0; i < VPT; i++) {
      const int idx = threadIdx.x + i * kThreads;
      if (idx < nvec) {
        uint32_t w0 = 0, w1 = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
          w0 |= q8_byte(v[i][j], inv) << (8 * j);
          w1 |= q8_byte(v[i][4 + j], inv) << (8 * j);
        }
        ar[idx] = make_uint2(w0, w1);
      }
    }
  }
}

}  // namespace

fg_status fg_layernorm_launch(const fg_half *x, int M, int h, const fg_half *gamma, const fg_half *beta, float eps,
                              fg_half *y, cudaStream_t st) {
  if (M == 0) return FG_OK;
  const uint4 *xv = reinterpret_cast<const uint4 *>(x);
  const uint4 *gv = reinterpret_cast<const uint4 *>(gamma), *bv = reinterpret_cast<const uint4 *>(beta);
  uint4 *yv = reinterpret_cast<uint4 *>(y);
  const int vpt = (h / 8 + kThreads - 1) / kThreads;
  if (vpt <= 1) layernorm_kernel<1, false><<<M, kThreads, 0, st>>>(xv, h, gv, bv, eps, yv, nullptr, nullptr);
  else if (vpt <= 2) layernorm_kernel<2, false><<<M, kThreads, 0, st>>>(xv, h, gv, bv, eps, yv, nullptr, nullptr);
  else if (vpt <= 4) layernorm_kernel<4, false><<<M, kThreads, 0, st>>>(xv, h, gv, bv, eps, yv, nullptr, nullptr);
  else layernorm_kernel<8, false><<<M, kThreads, 0, st>>>(xv, h, gv, bv, eps, yv, nullptr, nullptr);
  return fg_launch_check();
}

// LayerNorm whose fp16 output y is also quantised to int8 per row (a8 [M][h], ascale [M]), the
// W4A8 layer's products' input: bit for bit what fg_act8_quantize makes of y.
fg_status fg_layernorm_q8_launch(const fg_half *x, int M, int h, const fg_half *gamma, const fg_half *beta,
                                 float eps, fg_half *y, int8_t *a8, float *ascale, cudaStream_t st) {
  if (M == 0) return FG_OK;
  const uint4 *xv = reinterpret_cast<const uint4 *>(x);
  const uint4 *gv = reinterpret_cast<const uint4 *>(gamma), *bv = reinterpret_cast<const uint4 *>(beta);
  uint4 *yv = reinterpret_cast<uint4 *>(y);
  uint2 *av = reinterpret_cast<uint2 *>(a8);
  const int vpt = (h / 8 + kThreads - 1) / kThreads;
  if (vpt <= 1) layernorm_kernel<1, true><<<M, kThreads, 0, st>>>(xv, h, gv, bv, eps, yv, av, ascale);
  else if (vpt <= 2) layernorm_kernel<2, true><<<M, kThreads, 0, st>>>(xv, h, gv, bv, eps, yv, av, ascale);
  else if (vpt <= 4) layernorm_kernel<4, true><<<M, kThreads, 0, st>>>(xv, h, gv, bv, eps, yv, av, ascale);
  else layernorm_kernel<8, true><<<M, kThreads, 0, st>>>(xv, h, gv, bv, eps, yv, av, ascale);
  return fg_launch_check();
}

extern "C" fg_status fg_layernorm(const fg_half *x, int M, int h, const fg_half *gamma, const fg_half *beta,
                                  float eps, fg_half *y, void *stream) {
  if (M < 0 || h <= 0) return FG_ERR_INVALID;
  if (h % 8 || h > kThreads * kMaxVec * 8) return FG_ERR_SHAPE;
  if (M == 0) return FG_OK;
  if (!x || !y || !fg_aligned16(x) || !fg_aligned16(y)) return FG_ERR_INVALID;
  if ((gamma && !fg_aligned16(gamma)) || (beta && !fg_aligned16(beta))) return FG_ERR_INVALID;
  return fg_layernorm_launch(x, M, h, gamma, beta, eps, y, static_cast<cudaStream_t>(stream));
}
