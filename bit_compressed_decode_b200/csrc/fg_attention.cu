// fg_attention.cu -- softmax attention of query rows over the 4-bit KV cache.
//
// "FlexGen Guide: High-Throughput LLM Offloading on One GPU", section 3: the KV cache
// is held as 4-bit groups and dequantised on the fly for the attention dot products;
// the online (running max / running sum) softmax follows the tiled, IO-aware attention
// the same pages mention (dev.to guide, "Efficient Attention Implementations").
//
// One CTA (4 warps) per (query row, head).  The row's cached K/V codes and group
// metadata stream through shared memory in chunks of 64 tokens with 1-D bulk copies
// (cp.async.bulk, completion on an mbarrier), STAGES chunks in flight.  Each token
// is handled by D/32 lanes (16 code bytes = 32 dims each, half a 64-group).
// Scores use the group decomposition
//     q . k = sum_g ( min_g * sum_{d in g} q_d  +  scale_g * sum_{d in g} q_d * code_d ),
// so the per-element work is one FMA with the integer code; V is accumulated the same
// way (sum_t p_t * min_t and sum_t (p_t * scale_t) * code_t,d), all in fp32.
#include <math.h>

#include "fg_internal.cuh"

namespace {

constexpr int kChunk = 64;
constexpr int kStages = 4;
constexpr int kWarps = 4;

struct AttnArgs {
  const __half *q;
  int64_t ldq;
  __half *out;
  int64_t ldo;
  const uint8_t *kc, *vc;
  const __half *km, *ks, *vm, *vs;
  const int32_t *positions;
  int rows, rows_per_seq, H, maxL;
  unsigned int *err;
};

template <int D>
struct AttnShape {
  static constexpr int LPT = D / 32;                // lanes per token
  static constexpr int TPW = 32 / LPT;              // tokens per warp per sub-step
  static constexpr int NG = D / 64;                 // 64-groups per head
  static constexpr int SUB = kChunk / kWarps / TPW; // sub-steps per warp per chunk
  static constexpr int CODE_B = kChunk * D / 2;     // code bytes per chunk (K or V)
  static constexpr int META_B = kChunk * NG * 2;    // bytes of one metadata array per chunk
  static constexpr int STAGE_B = 2 * CODE_B + 4 * META_B;
  static constexpr int SMEM = kStages * STAGE_B;
};

// code (0..15) of nibble i of w as an fp32 value: byte-permute the nibble-holding byte
// into the low byte of 2^23 (0x4B000000), subtract 2^23.
__device__ __forceinline__ float code_f(uint32_t lo_bytes, int byte_idx) {
  const uint32_t bits = __byte_perm(lo_bytes, 0x4B000000u, 0x7540 + byte_idx);
  return __int_as_float(bits) - 8388608.0f;
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) attn_decode_kernel(const AttnArgs a) {
  using S = AttnShape<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ float red_m[kWarps], red_l[kWarps];
  __shared__ float red_o[kWarps][D];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = blockIdx.x / a.H, hd = blockIdx.x % a.H;
  const int s = r / a.rows_per_seq;
  const int L = a.positions[s] + r % a.rows_per_seq + 1;
  __half *outp = a.out + static_cast<int64_t>(r) * a.ldo + hd * D;
  if (L < 1 || L > a.maxL) {  // position outside the cache: flag and write zeros
    if (tid == 0) atomicOr(a.err, FG_DEVERR_RANGE);
    for (int i = tid; i < D; i += blockDim.x) outp[i] = __float2half_rn(0.0f);
    return;
  }
  const int nchunks = (L + kChunk - 1) / kChunk;
  const int64_t slot0 = (static_cast<int64_t>(s) * a.H + hd) * a.maxL;

  auto stage_ptr = [&](int st) { return smem + st * S::STAGE_B; };
  auto issue = [&](int c) {
    const int st = c % kStages;
    const int nt = min(kChunk, L - c * kChunk);
    const int ntr = (nt + 7) & ~7;  // whole 16-byte metadata rows; stays below max_len (multiple of 64)
    const uint32_t cb = ntr * (D / 2), mb = ntr * S::NG * 2;
    const uint32_t bar = smem_u32(&full_bar[st]);
    mbar_arrive_expect_tx(bar, 2 * cb + 4 * mb);
    const int64_t t0 = slot0 + static_cast<int64_t>(c) * kChunk;
    uint8_t *p = stage_ptr(st);
    bulk_g2s(smem_u32(p), a.kc + t0 * (D / 2), cb, bar);
    bulk_g2s(smem_u32(p + S::CODE_B), a.vc + t0 * (D / 2), cb, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 0 * S::META_B), a.km + t0 * S::NG, mb, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 1 * S::META_B), a.ks + t0 * S::NG, mb, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 2 * S::META_B), a.vm + t0 * S::NG, mb, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 3 * S::META_B), a.vs + t0 * S::NG, mb, bar);
  };

  if (tid == 0) {
    for (int i = 0; i < kStages; i++) mbar_init(smem_u32(&full_bar[i]), 1);
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (tid == 0)
    for (int c = 0; c < min(kStages, nchunks); c++) issue(c);

  // this lane's 32 query dims (scaled by log2(e) so the softmax can use exp2)
  const int p = lane % S::LPT, ts = lane / S::LPT, g = p >> 1;
  float qf[32];
  {
    const uint4 *qp = reinterpret_cast<const uint4 *>(a.q + static_cast<int64_t>(r) * a.ldq + hd * D + p * 32);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      uint4 v = qp[i];
      const __half2 *h2 = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
      for (int j = 0; j < 4; j++) {
        float2 f = __half22float2(h2[j]);
        qf[8 * i + 2 * j] = f.x * 1.4426950408889634f;
        qf[8 * i + 2 * j + 1] = f.y * 1.4426950408889634f;
      }
    }
  }
  float qsum = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i++) qsum += qf[i];
  const float Qg = qsum + __shfl_xor_sync(0xffffffffu, qsum, 1);

  float m = -INFINITY, l = 0.f, accmin = 0.f;
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; i++) acc[i] = 0.f;

  volatile int *no_abort = nullptr;
  bool ok = true;
  for (int c = 0; c < nchunks; c++) {
    const int st = c % kStages;
    if (ok && !mbar_wait_bounded(smem_u32(&full_bar[st]), (c / kStages) & 1, no_abort, a.err)) ok = false;
    if (ok) {
      const uint8_t *base = stage_ptr(st);
      const uint4 *Kc = reinterpret_cast<const uint4 *>(base);
      const uint4 *Vc = reinterpret_cast<const uint4 *>(base + S::CODE_B);
      const __half *Km = reinterpret_cast<const __half *>(base + 2 * S::CODE_B);
      const __half *Ks = Km + kChunk * S::NG;
      const __half *Vm = Ks + kChunk * S::NG;
      const __half *Vs = Vm + kChunk * S::NG;
      float sc[S::SUB];
      float cmax = -INFINITY;
#pragma unroll
      for (int u = 0; u < S::SUB; u++) {
        const int tl = warp * (kChunk / kWarps) + u * S::TPW + ts;
        const bool valid = c * kChunk + tl < L;
        const uint4 kw = Kc[tl * S::LPT + p];
        float dot = 0.f;
        const uint32_t words[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
        for (int wi = 0; wi < 4; wi++) {
          const uint32_t lo = words[wi] & 0x0F0F0F0Fu, hi = (words[wi] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
          for (int b = 0; b < 4; b++) {
            dot = fmaf(qf[8 * wi + 2 * b], code_f(lo, b), dot);
            dot = fmaf(qf[8 * wi + 2 * b + 1], code_f(hi, b), dot);
          }
        }
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        float sg = __half2float(Km[tl * S::NG + g]) * Qg + __half2float(Ks[tl * S::NG + g]) * dot;
#pragma unroll
        for (int o = 2; o < S::LPT; o <<= 1) sg += __shfl_xor_sync(0xffffffffu, sg, o);
        sc[u] = valid ? sg : -INFINITY;
        cmax = fmaxf(cmax, sc[u]);
      }
#pragma unroll
      for (int o = S::LPT; o < 32; o <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
      const float m_new = fmaxf(m, cmax);
      if (m_new != -INFINITY) {
        const float alpha = exp2f(m - m_new);  // 0 when m is -inf
        l *= alpha;
        accmin *= alpha;
#pragma unroll
        for (int i = 0; i < 32; i++) acc[i] *= alpha;
#pragma unroll
        for (int u = 0; u < S::SUB; u++) {
          const int tl = warp * (kChunk / kWarps) + u * S::TPW + ts;
          const bool valid = c * kChunk + tl < L;
          const float pt = valid ? exp2f(sc[u] - m_new) : 0.f;
          l += pt;
          const float w = valid ? pt * __half2float(Vs[tl * S::NG + g]) : 0.f;
          accmin += valid ? pt * __half2float(Vm[tl * S::NG + g]) : 0.f;
          const uint4 vw = Vc[tl * S::LPT + p];
          const uint32_t words[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
          for (int wi = 0; wi < 4; wi++) {
            const uint32_t lo = words[wi] & 0x0F0F0F0Fu, hi = (words[wi] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int b = 0; b < 4; b++) {
              acc[8 * wi + 2 * b] = fmaf(w, code_f(lo, b), acc[8 * wi + 2 * b]);
              acc[8 * wi + 2 * b + 1] = fmaf(w, code_f(hi, b), acc[8 * wi + 2 * b + 1]);
            }
          }
        }
        m = m_new;
      }
    }
    __syncthreads();  // every warp is done with stage st
    if (tid == 0 && ok && c + kStages < nchunks) issue(c + kStages);
  }

  // reduce over the token slots of the warp (lanes with equal p)
#pragma unroll
  for (int o = S::LPT; o < 32; o <<= 1) {
    l += __shfl_xor_sync(0xffffffffu, l, o);
    accmin += __shfl_xor_sync(0xffffffffu, accmin, o);
#pragma unroll
    for (int i = 0; i < 32; i++) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  }
  if (ts == 0) {
#pragma unroll
    for (int i = 0; i < 32; i++) red_o[warp][p * 32 + i] = acc[i] + accmin;
    if (p == 0) {
      red_m[warp] = m;
      red_l[warp] = l;
    }
  }
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; w++) M = fmaxf(M, red_m[w]);
  float wsc[kWarps], den = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; w++) {
    wsc[w] = red_m[w] == -INFINITY ? 0.f : exp2f(red_m[w] - M);
    den += wsc[w] * red_l[w];
  }
  const float inv = ok ? 1.0f / den : 0.f;
  for (int i = tid; i < D; i += blockDim.x) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; w++) o += wsc[w] * red_o[w][i];
    outp[i] = __float2half_rn(o * inv);
  }
}

template <int D>
fg_status launch(const AttnArgs &a, cudaStream_t st) {
  using S = AttnShape<D>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    fg_status rc = fg_cuda_check(
        cudaFuncSetAttribute(attn_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM));
    if (rc != FG_OK) return rc;
    attr_set[dev] = true;
  }
  const int64_t ctas = static_cast<int64_t>(a.rows) * a.H;
  attn_decode_kernel<D><<<static_cast<unsigned>(ctas), kWarps * 32, S::SMEM, st>>>(a);
  return fg_launch_check();
}

}  // namespace

fg_status fg_kv_validate(const fg_kv_cache *kv);

fg_status fg_attention_launch(const fg_kv_cache *kv, const fg_half *q, int64_t ldq, fg_half *out, int64_t ldo,
                              int rows, int rows_per_seq, const int32_t *positions, cudaStream_t st) {
  AttnArgs a;
  a.q = reinterpret_cast<const __half *>(q);
  a.ldq = ldq;
  a.out = reinterpret_cast<__half *>(out);
  a.ldo = ldo;
  a.kc = kv->k_codes;
  a.vc = kv->v_codes;
  a.km = reinterpret_cast<const __half *>(kv->k_mins);
  a.ks = reinterpret_cast<const __half *>(kv->k_scales);
  a.vm = reinterpret_cast<const __half *>(kv->v_mins);
  a.vs = reinterpret_cast<const __half *>(kv->v_scales);
  a.positions = positions;
  a.rows = rows;
  a.rows_per_seq = rows_per_seq;
  a.H = kv->num_heads;
  a.maxL = kv->max_len;
  a.err = fg_error_word_ptr();
  if (!a.err) return FG_ERR_CUDA;
  switch (kv->head_dim) {
    case 64: return launch<64>(a, st);
    case 128: return launch<128>(a, st);
    case 256: return launch<256>(a, st);
  }
  return FG_ERR_UNSUPPORTED;
}

extern "C" fg_status fg_attention_decode(const fg_kv_cache *kv, const fg_half *q, int64_t ldq, fg_half *out,
                                         int64_t ldo, int rows, int rows_per_seq, const int32_t *positions,
                                         void *stream) {
  fg_status rc = fg_kv_validate(kv);
  if (rc != FG_OK) return rc;
  if (rows < 0 || rows_per_seq < 1 || rows % rows_per_seq || rows / rows_per_seq > kv->num_seqs) return FG_ERR_SHAPE;
  if (rows == 0) return FG_OK;
  if (!q || !out || !positions || !fg_aligned16(q) || !fg_aligned16(out)) return FG_ERR_INVALID;
  const int64_t hD = static_cast<int64_t>(kv->num_heads) * kv->head_dim;
  if (ldq < hD || ldo < hD || ldq % 8 || ldo % 8) return FG_ERR_SHAPE;
  return fg_attention_launch(kv, q, ldq, out, ldo, rows, rows_per_seq, positions, static_cast<cudaStream_t>(stream));
}
