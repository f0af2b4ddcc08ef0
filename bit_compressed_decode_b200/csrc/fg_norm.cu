// fg_norm.cu -- LayerNorm of fp16 rows (pre-LayerNorm OPT decoder layer; model family
// from the OPT entry of the PIPO paper's reference list).  fp32 statistics: mean, then
// the biased variance of (x - mean) from the values held in registers (two passes over
// registers, one read of HBM), y = (x - mean) * rsqrt(var + eps) * gamma + beta.
#include "fg_internal.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxVec = 8;  // up to 8 x 8 halves per thread: h <= 16384

__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; w++) t += red[w];
  return t;
}

__global__ void __launch_bounds__(kThreads) layernorm_kernel(const uint4 *__restrict__ x, int h,
                                                             const __half *__restrict__ gamma,
                                                             const __half *__restrict__ beta, float eps,
                                                             uint4 *__restrict__ y) {
  __shared__ float red[kThreads / 32];
  const int nvec = h / 8;
  const uint4 *xr = x + static_cast<int64_t>(blockIdx.x) * nvec;
  uint4 *yr = y + static_cast<int64_t>(blockIdx.x) * nvec;
  float v[kMaxVec][8];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVec; i++) {
    const int idx = threadIdx.x + i * kThreads;
    if (idx < nvec) {
      uint4 u = xr[idx];
      const __half2 *h2 = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
      for (int j = 0; j < 4; j++) {
        float2 f = __half22float2(h2[j]);
        v[i][2 * j] = f.x;
        v[i][2 * j + 1] = f.y;
        sum += f.x + f.y;
      }
    }
  }
  const float mean = block_sum(sum, red) / h;
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVec; i++) {
    const int idx = threadIdx.x + i * kThreads;
    if (idx < nvec) {
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const float d = v[i][j] - mean;
        sq += d * d;
      }
    }
  }
  const float var = block_sum(sq, red) / h;
  const float rstd = rsqrtf(var + eps);
#pragma unroll
  for (int i = 0; i < kMaxVec; i++) {
    const int idx = threadIdx.x + i * kThreads;
    if (idx < nvec) {
      uint4 out;
      __half2 *o2 = reinterpret_cast<__half2 *>(&out);
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const int c = idx * 8 + 2 * j;
        const float g0 = gamma ? __half2float(gamma[c]) : 1.f, g1 = gamma ? __half2float(gamma[c + 1]) : 1.f;
        const float b0 = beta ? __half2float(beta[c]) : 0.f, b1 = beta ? __half2float(beta[c + 1]) : 0.f;
        o2[j] = __floats2half2_rn((v[i][2 * j] - mean) * rstd * g0 + b0, (v[i][2 * j + 1] - mean) * rstd * g1 + b1);
      }
      yr[idx] = out;
    }
  }
}

}  // namespace

fg_status fg_layernorm_launch(const fg_half *x, int M, int h, const fg_half *gamma, const fg_half *beta, float eps,
                              fg_half *y, cudaStream_t st) {
  if (M == 0) return FG_OK;
  layernorm_kernel<<<M, kThreads, 0, st>>>(reinterpret_cast<const uint4 *>(x), h,
                                           reinterpret_cast<const __half *>(gamma),
                                           reinterpret_cast<const __half *>(beta), eps, reinterpret_cast<uint4 *>(y));
  return fg_launch_check();
}

extern "C" fg_status fg_layernorm(const fg_half *x, int M, int h, const fg_half *gamma, const fg_half *beta,
                                  float eps, fg_half *y, void *stream) {
  if (M < 0 || h <= 0) return FG_ERR_INVALID;
  if (h % 8 || h > kThreads * kMaxVec * 8) return FG_ERR_SHAPE;
  if (M == 0) return FG_OK;
  if (!x || !y || !fg_aligned16(x) || !fg_aligned16(y)) return FG_ERR_INVALID;
  return fg_layernorm_launch(x, M, h, gamma, beta, eps, y, static_cast<cudaStream_t>(stream));
}
