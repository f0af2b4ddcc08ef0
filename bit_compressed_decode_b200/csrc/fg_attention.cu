// fg_attention.cu -- softmax attention of query rows over the 4-bit KV cache.
//
// "FlexGen Guide: High-Throughput LLM Offloading on One GPU", section 3: the KV cache
// is held as 4-bit groups and dequantised on the fly for the attention dot products;
// the online (running max / running sum) softmax follows the tiled, IO-aware attention
// the same pages mention (dev.to guide, "Efficient Attention Implementations").
//
// One CTA (4 warps) per (query row, head).  The row's cached K/V codes and group
// metadata stream through shared memory in chunks of 128 tokens with 1-D bulk copies
// (cp.async.bulk, completion on an mbarrier), kStages chunks in flight; each warp takes
// 16 tokens of every 64 in a chunk (two tiles per chunk), so the per-chunk barrier, wait and
// refill are paid once per 32 tokens of a warp.
//
// Both products run on the tensor cores (mma.sync m16n8k16, fp16 operands, fp32
// accumulation) directly on the codes, through the group decomposition
//     q . k_t = sum_g ( min_tg * sum_{d in g} q_d  +  scale_tg * sum_{d in g} q_d c_td )
//     o_d     = sum_t p_t min_t,g(d)  +  sum_t (p_t scale_t,g(d)) c_td
// so the per-element work is one AND per pair of codes: a nibble left in bits 0-3 of a
// 16-bit half is the fp16 subnormal c * 2^-24, one in bits 4-7 is c * 2^-20, both exact,
// and the fp32 results are rescaled by the matching power of two.
//   scores: A = K codes (16 tokens x 16 dims per MMA), B = q (16 dims x 8 columns;
//           column n holds q on the dims of one group, zero elsewhere) -> the group sums
//           sum_{d in g} q_d c_td of every token, each group in 8/NG columns, so that every
//           lane of a quad sees all groups of its two tokens and the four lanes split the
//           per-token work;
//   output: A = V codes transposed (16 dims x 16 tokens), B = w (16 tokens x 8 columns;
//           column g is p_t * scale_tg rounded to fp16) -> row d, column g(d).
// Dims may take any order along an MMA's k dimension as long as q takes the same order
// (tokens likewise for V), which lets every lane build its operands from whole 32-bit
// words of codes.  Scores, the softmax state and every sum stay in fp32.
#include <math.h>

#include "fg_internal.cuh"

namespace {

constexpr int kChunk = 128;
constexpr int kStages = 2;
constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSlack = 2.0f;
constexpr uint32_t kLoNib = 0x000F000Fu;  // bits 0-3 of both halves: c * 2^-24
constexpr uint32_t kHiNib = 0x00F000F0u;  // bits 4-7 of both halves: c * 2^-20

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
  const __half *kn, *vn;  // decode rows: new k, v (fp16) quantised into the cache first; null: none
  int64_t ldn;
};

template <int D, int G>
struct AttnShape {
  static constexpr int NG = D / G;                  // G-groups (G = 64 or 128) per head
  static constexpr int RB = D / 2;                  // code bytes per token row
  static constexpr int KW = D / 32;                 // K code words per lane per token
  static constexpr int VW = D / 64;                 // V code words per lane per token
  static constexpr int MT = D / 16;                 // 16-dim output tiles
  static constexpr int CODE_B = kChunk * RB;        // code bytes per chunk (K or V)
  static constexpr int META_B = kChunk * NG * 2;    // bytes of one metadata array per chunk
  static constexpr int STAGE_B = 2 * CODE_B + 4 * META_B;
  static constexpr int SMEM = kStages * STAGE_B;
};

// Byte offset in a K code row of word j of lane class c (lane % 4): the dims that lane
// class feeds to the score MMAs.  Always inside one group (32 or 64 bytes).
template <int D>
__device__ __forceinline__ int kword_off(int c, int j) {
  return D == 64 ? 8 * c + 4 * j : 64 * (j >> 2) + 16 * c + 4 * (j & 3);
}

// Group held by column n of the score MMAs.  Lane (gid, c) reads columns 2c and 2c+1; the
// map puts the group(s) lane c finishes (c % 2 for NG = 2; 2 (c % 2) + {0, 1} for NG = 4)
// in those columns, the first of them in column 2c.
template <int NG>
__device__ __forceinline__ int col_group(int n) {
  return NG == 1 ? 0 : NG == 2 ? ((n >> 1) ^ n) & 1 : n & 3;
}

template <int D>
__device__ __forceinline__ void load_krow(const uint8_t *row, int c, uint32_t (&w)[D / 32]) {
  if constexpr (D == 64) {
    const uint2 v = *reinterpret_cast<const uint2 *>(row + 8 * c);
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int u = 0; u < D / 128; u++) {
      const uint4 v = *reinterpret_cast<const uint4 *>(row + 64 * u + 16 * c);
      w[4 * u] = v.x;
      w[4 * u + 1] = v.y;
      w[4 * u + 2] = v.z;
      w[4 * u + 3] = v.w;
    }
  }
}

template <int N>
__device__ __forceinline__ void load_words(const uint8_t *p, uint32_t (&w)[N]) {
  if constexpr (N == 1) {
    w[0] = *reinterpret_cast<const uint32_t *>(p);
  } else if constexpr (N == 2) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    w[0] = v.x;
    w[1] = v.y;
  } else {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    w[0] = v.x;
    w[1] = v.y;
    w[2] = v.z;
    w[3] = v.w;
  }
}

// d += A * B for one m16n8k16 tile, fp16 operands and fp32 accumulators, in the PTX
// fragment layout: a0/a1 = rows gid/gid+8 at k = 2c..2c+1, a2/a3 = the same rows at
// k = 2c+8..2c+9; b0/b1 = column gid at k = 2c..2c+1 / 2c+8..2c+9; d = rows gid, gid+8 x
// columns 2c, 2c+1 (gid = lane / 4, c = lane % 4).
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = A * B (fresh accumulators)
__device__ __forceinline__ void mma_f16_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// 2^x by the hardware approximation (relative error ~2^-22); results below 2^-126 are 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_h2(__half lo, __half hi) {
  const __half2 h = __halves2half2(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// The decode row's new k and v (D fp16 values each) in 4-bit form, held by one warp: unit us
// (group us / 2 of k for even us, of v for odd us) is quantised by G/8 lanes with the group
// quantiser the append kernel uses, so the cache receives the same bits.
template <int D, int G>
struct NewRow {
  static constexpr int NG = D / G, L = G / 8, USTEP = 32 / L, STEPS = (2 * NG + USTEP - 1) / USTEP;
  uint4 x[STEPS];
  uint32_t w[STEPS];
  __half mn[STEPS], sc[STEPS];

  __device__ __forceinline__ void load(const __half *krow, const __half *vrow, int lane) {
    const int u = lane / L, j = lane % L;
#pragma unroll
    for (int st = 0; st < STEPS; st++) {
      const int us = st * USTEP + u;
      x[st] = make_uint4(0, 0, 0, 0);
      if (us < 2 * NG) x[st] = *reinterpret_cast<const uint4 *>(((us & 1) ? vrow : krow) + (us >> 1) * G + j * 8);
    }
  }
  __device__ __forceinline__ void quantise() {  // all 32 lanes: the quantiser shuffles
#pragma unroll
    for (int st = 0; st < STEPS; st++) w[st] = quant_group8<L>(x[st], mn[st], sc[st]);
  }
  // one token row: codes as 32-bit words (D/8 per row), NG mins and scales per array
  __device__ __forceinline__ void write(uint32_t *kc, uint32_t *vc, __half *km, __half *ks, __half *vm, __half *vs,
                                        int lane) const {
    const int u = lane / L, j = lane % L;
#pragma unroll
    for (int st = 0; st < STEPS; st++) {
      const int us = st * USTEP + u;
      if (us >= 2 * NG) continue;
      const int g = us >> 1;
      ((us & 1) ? vc : kc)[g * L + j] = w[st];
      if (j == 0) {
        ((us & 1) ? vm : km)[g] = mn[st];
        ((us & 1) ? vs : ks)[g] = sc[st];
      }
    }
  }
};

// One token row (D/8 code words per array, NG mins and scales per array) copied by a warp.
template <int D, int NG>
__device__ __forceinline__ void copy_row(uint32_t *kc, uint32_t *vc, __half *km, __half *ks, __half *vm, __half *vs,
                                         const uint32_t (&codes)[2][D / 8], const __half (&meta)[4][NG], int lane) {
#pragma unroll
  for (int i = lane; i < D / 4; i += 32) (i < D / 8 ? kc[i] : vc[i - D / 8]) = codes[i / (D / 8)][i % (D / 8)];
  if (lane < 4 * NG) {
    const int arr = lane / NG, g = lane % NG;
    __half *dst = arr == 0 ? km : arr == 1 ? ks : arr == 2 ? vm : vs;
    dst[g] = meta[arr][g];
  }
}

// APP: decode rows that append their new k, v in this launch (fg_attention_decode_append);
// without it none of the append's state exists.
template <int D, int G, bool APP>
__global__ void __launch_bounds__(kWarps * 32, D <= 128 ? 5 : 3) attn_decode_kernel(const AttnArgs a) {
  using S = AttnShape<D, G>;
  constexpr int NG = S::NG, RB = S::RB, KW = S::KW, VW = S::VW, MT = S::MT;
  constexpr float kS24 = 16777216.0f, kS20 = 1048576.0f;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ float red_m[kWarps], red_l[kWarps];
  __shared__ float red_o[kWarps][D];
  // fused append: the new k, v rows (fp16, copied with the first chunk) and their 4-bit form
  constexpr int XD = APP ? D : 8, XG = APP ? NG : 1;  // (minimal arrays without the append)
  __shared__ __align__(16) __half new_x[2][XD];
  __shared__ __align__(16) uint32_t new_codes[2][XD / 8];
  __shared__ __half new_meta[4][XG];  // k min, k scale, v min, v scale
  griddep_launch();  // the output projection may start its weight-side prologue

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, c = lane & 3;
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
  auto issue = [&](int ch) {
    const int st = ch % kStages;
    const int nt = min(kChunk, L - ch * kChunk);
    const int ntr = (nt + 7) & ~7;  // whole 16-byte metadata rows; stays below max_len (multiple of 64)
    const uint32_t cb = ntr * RB, mb = ntr * NG * 2;
    const uint32_t bar = smem_u32(&full_bar[st]);
    const bool rows = APP && ch == 0;  // fused append: the new k, v rows come with chunk 0
    mbar_arrive_expect_tx(bar, 2 * cb + 4 * mb + (rows ? 4 * D : 0));
    if (rows) {
      const int64_t o = static_cast<int64_t>(r) * a.ldn + hd * D;
      bulk_g2s(smem_u32(&new_x[0][0]), a.kn + o, 2 * D, bar);
      bulk_g2s(smem_u32(&new_x[1][0]), a.vn + o, 2 * D, bar);
    }
    const int64_t t0 = slot0 + static_cast<int64_t>(ch) * kChunk;
    uint8_t *p = stage_ptr(st);
    bulk_g2s(smem_u32(p), a.kc + t0 * RB, cb, bar);
    bulk_g2s(smem_u32(p + S::CODE_B), a.vc + t0 * RB, cb, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 0 * S::META_B), a.km + t0 * NG, mb, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 1 * S::META_B), a.ks + t0 * NG, mb, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 2 * S::META_B), a.vm + t0 * NG, mb, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 3 * S::META_B), a.vs + t0 * NG, mb, bar);
  };

  if (tid == 0) {
    for (int i = 0; i < kStages; i++) mbar_init(smem_u32(&full_bar[i]), 1);
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (tid == 0)
    for (int ch = 0; ch < min(kStages, nchunks); ch++) issue(ch);
  // Fused append (decode): the new token (position L - 1, row tl of the last chunk) is read
  // only by the warp that owns its 16 tokens of the chunk's 64-token sub-tile.  When that
  // chunk has landed (the new k, v rows landed with the first chunk), the warp quantises the
  // rows, puts them in place of whatever the copy brought for that row, and stores them to
  // the cache after the loop, when no copy of this kernel still reads it.
  const int tl = (L - 1) % kChunk, app_chunk = (L - 1) / kChunk;
  const bool app_warp = APP && warp == (tl % 64) / 16;

  // ---- q as the B operand of the score MMAs, in the dim order of kword_off ----
  // Word j of lane class c holds, per 16-bit half, nibbles (bits 0-3, 4-7, 8-11, 12-15) =
  // dims 2o+{0,1,2,3} (low half) and 2o+{4,5,6,7} (high half), o = kword_off(c, j).
  // Low-nibble MMA (bits 0-3 of w and of w >> 8): k slots (2c, 2c+1) = dims (2o, 2o+4),
  // (2c+8, 2c+9) = (2o+2, 2o+6); high-nibble MMA: the same + 1.
  const __half *qrow = a.q + static_cast<int64_t>(r) * a.ldq + hd * D;
  uint32_t qlo[KW][2], qhi[KW][2];
#pragma unroll
  for (int j = 0; j < KW; j++) {
    const int o = kword_off<D>(c, j);
    if (col_group<NG>(gid) == o / (G / 2)) {
      const uint4 v = *reinterpret_cast<const uint4 *>(qrow + 2 * o);
      const __half *e = reinterpret_cast<const __half *>(&v);
      qlo[j][0] = pack_h2(e[0], e[4]);
      qlo[j][1] = pack_h2(e[2], e[6]);
      qhi[j][0] = pack_h2(e[1], e[5]);
      qhi[j][1] = pack_h2(e[3], e[7]);
    } else {
      qlo[j][0] = qlo[j][1] = qhi[j][0] = qhi[j][1] = 0u;
    }
  }
  // Lane (gid, c) finishes token gid + 8 * (c >> 1) on the groups of its column pair
  // (2c, 2c+1): g0 = (c & 1) * NG / 2 and, for NG = 4, g0 + 1; the other lane of its pair
  // (c ^ 1) holds the remaining groups.
  const int g0 = (c & 1) * (NG / 2);
  constexpr int GPL = NG == 4 ? 2 : 1;  // groups per lane
  float ql[GPL];                         // sum of q over those groups, times log2(e)
  {
    constexpr int PER = D / 32, LPG = G / PER;   // dims per lane, lanes per group
    float qs = 0.f;
#pragma unroll
    for (int i = 0; i < PER; i++) qs += __half2float(qrow[lane * PER + i]);
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
#pragma unroll
    for (int e = 0; e < GPL; e++) ql[e] = __shfl_sync(0xffffffffu, qs, (g0 + e) * LPG) * kLog2e;
  }
  const int tq = gid + 8 * (c >> 1);  // this lane's token within a warp tile

  float m = -INFINITY, l = 0.f;
  float vmin[GPL];  // sum_t p_t * min_t,g over this lane's tokens, for its groups
  float ov[MT][4];
#pragma unroll
  for (int e = 0; e < GPL; e++) vmin[e] = 0.f;
#pragma unroll
  for (int t = 0; t < MT; t++) ov[t][0] = ov[t][1] = ov[t][2] = ov[t][3] = 0.f;

  bool ok = true;
  for (int ch = 0; ch < nchunks; ch++) {
    const int st = ch % kStages;
    if (ok && !mbar_wait_bounded(smem_u32(&full_bar[st]), (ch / kStages) & 1, nullptr, a.err)) ok = false;
    if (ok) {
      const uint8_t *base = stage_ptr(st);
      const uint8_t *Kc = base, *Vc = base + S::CODE_B;
      const __half *Km = reinterpret_cast<const __half *>(base + 2 * S::CODE_B);
      const __half *Ks = Km + kChunk * NG;
      const __half *Vm = Ks + kChunk * NG;
      const __half *Vs = Vm + kChunk * NG;
      if constexpr (APP) if (app_warp && ch == app_chunk) {
        {
          NewRow<D, G> nr;
          nr.load(new_x[0], new_x[1], lane);
          nr.quantise();
          nr.write(new_codes[0], new_codes[1], new_meta[0], new_meta[1], new_meta[2], new_meta[3], lane);
        }
        __syncwarp();
        // the new row in place of the copied one; the proxy fence orders these writes before
        // the bulk copy that reuses the stage (issued after the chunk's barrier)
        uint8_t *b = stage_ptr(st);
        __half *km = reinterpret_cast<__half *>(b + 2 * S::CODE_B);
        copy_row<D, NG>(reinterpret_cast<uint32_t *>(b + tl * RB), reinterpret_cast<uint32_t *>(b + S::CODE_B + tl * RB),
                        km + tl * NG, km + kChunk * NG + tl * NG, km + 2 * kChunk * NG + tl * NG,
                        km + 3 * kChunk * NG + tl * NG, new_codes, new_meta, lane);
        fence_proxy_async_smem();
        __syncwarp();
      }
      for (int sub = 0; sub < kChunk / 64; sub++) {
      const int t0 = sub * 64 + warp * 16;  // this warp's tokens of the chunk: t0 .. t0+15
      if (ch * kChunk + t0 >= L) break;     // warp-uniform: none of them (nor later ones) visible

      // ---- group sums of q . c for tokens t0+gid and t0+gid+8 ----
      float slo[4], shi[4];
      {
        uint32_t k0[KW], k1[KW];
        load_krow<D>(Kc + (t0 + gid) * RB, c, k0);
        load_krow<D>(Kc + (t0 + gid + 8) * RB, c, k1);
#pragma unroll
        for (int j = 0; j < KW; j++) {
          const uint32_t x0 = k0[j], x1 = k1[j], y0 = x0 >> 8, y1 = x1 >> 8;
          if (j == 0) {
            mma_f16_z(slo, x0 & kLoNib, x1 & kLoNib, y0 & kLoNib, y1 & kLoNib, qlo[j][0], qlo[j][1]);
            mma_f16_z(shi, x0 & kHiNib, x1 & kHiNib, y0 & kHiNib, y1 & kHiNib, qhi[j][0], qhi[j][1]);
          } else {
            mma_f16(slo, x0 & kLoNib, x1 & kLoNib, y0 & kLoNib, y1 & kLoNib, qlo[j][0], qlo[j][1]);
            mma_f16(shi, x0 & kHiNib, x1 & kHiNib, y0 & kHiNib, y1 & kHiNib, qhi[j][0], qhi[j][1]);
          }
        }
      }
      // V codes of the tile, loaded ahead of the softmax bookkeeping
      uint32_t v0[VW], v1[VW], v2[VW], v3[VW];
      {
        const uint8_t *vrow = Vc + (t0 + c) * RB + gid * (D / 16);
        load_words<VW>(vrow, v0);
        load_words<VW>(vrow + 4 * RB, v1);
        load_words<VW>(vrow + 8 * RB, v2);
        load_words<VW>(vrow + 12 * RB, v3);
      }
      // ---- score (log2 units) of token t0+tq ----
      const bool valid = ch * kChunk + t0 + tq < L;
      float sc;
      {
        const int i0 = (t0 + tq) * NG + g0;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < GPL; e++) {
          // C element of token row tq (gid or gid+8), column 2c + e
          const bool r8 = c & 2;
          const float lo = r8 ? slo[2 + e] : slo[e], hi = r8 ? shi[2 + e] : shi[e];
          const float dot = lo * (kS24 * kLog2e) + hi * (kS20 * kLog2e);
          part += __half2float(Km[i0 + e]) * ql[e] + __half2float(Ks[i0 + e]) * dot;
        }
        if constexpr (NG > 1) part += __shfl_xor_sync(0xffffffffu, part, 1);
        sc = valid ? part : -INFINITY;
      }
      float cmax = sc;
#pragma unroll
      for (int o = 2; o < 32; o <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
      // Lazy rescaling: the reference maximum m moves only when a score exceeds it by more
      // than kSlack (log2 units), so p = 2^(s - m) <= 2^kSlack = 4 and w = p * scale stays
      // below 4 * 8734 (the largest scale of 4-bit codes of fp16 data), inside fp16.
      if (cmax > m + kSlack) {  // warp-uniform; always taken at the first valid token (m = -inf)
        const float m_new = cmax;
        const float alpha = fast_exp2(m - m_new);  // 0 when m is -inf
        l *= alpha;
#pragma unroll
        for (int e = 0; e < GPL; e++) vmin[e] *= alpha;
#pragma unroll
        for (int t = 0; t < MT; t++) {
          ov[t][0] *= alpha;
          ov[t][1] *= alpha;
          ov[t][2] *= alpha;
          ov[t][3] *= alpha;
        }
        m = m_new;
      }
      if (cmax != -INFINITY) {  // warp-uniform: some token of the tile is valid
        const float pt = fast_exp2(sc - m);  // 0 for a masked token
        l += pt;                         // each token counted by two lanes
        // w = p * V scale for this lane's (token, groups), packed as fp16 in W
        uint32_t W;
        {
          const int i0 = (t0 + tq) * NG + g0;
          float w[2];
#pragma unroll
          for (int e = 0; e < GPL; e++) {
            vmin[e] += valid ? pt * __half2float(Vm[i0 + e]) : 0.f;
            w[e] = valid ? pt * __half2float(Vs[i0 + e]) : 0.f;
          }
          W = pack_h2(w[0], w[GPL - 1]);
        }
        // ---- w as the B operand: lane (n = gid, c) holds column n at tokens c, c+4 (k slots
        //      2c, 2c+1) and c+8, c+12 (k slots 2c+8, 2c+9); w(t, n) sits in lane
        //      4 (t % 8) + 2 (t / 8) + (n / GPL) % 2, half n % GPL ----
        uint32_t wb0, wb1;
        {
          const int src = 4 * c + ((gid / GPL) & (NG > 1 ? 1 : 0));
          const uint32_t X0 = __shfl_sync(0xffffffffu, W, src), X1 = __shfl_sync(0xffffffffu, W, src + 16);
          const uint32_t X2 = __shfl_sync(0xffffffffu, W, src + 2), X3 = __shfl_sync(0xffffffffu, W, src + 18);
          const uint32_t sel = (GPL == 2 && (gid & 1)) ? 0x7632u : 0x5410u;
          wb0 = gid < NG ? __byte_perm(X0, X1, sel) : 0u;
          wb1 = gid < NG ? __byte_perm(X2, X3, sel) : 0u;
        }
        // ---- V codes as the A operand: lane (gid, c) reads its D/8 dims (bytes
        //      gid*D/16 ...) of tokens c, c+4, c+8, c+12 and pairs tokens per 16-bit half ----
#pragma unroll
        for (int j = 0; j < VW; j++) {
#pragma unroll
          for (int h = 0; h < 2; h++) {
            const uint32_t sel = h ? 0x7632u : 0x5410u;
            const uint32_t P = __byte_perm(v0[j], v1[j], sel), Q = __byte_perm(v2[j], v3[j], sel);
            const uint32_t Ps = P >> 8, Qs = Q >> 8;
            // tile 4j+2h: rows gid / gid+8 = dims gid*D/8 + 2T + 0 / + 1 (nibbles 0 / 1 of
            // the byte pair); tile 4j+2h+1: nibbles 2 / 3
            mma_f16(ov[4 * j + 2 * h], P & kLoNib, P & kHiNib, Q & kLoNib, Q & kHiNib, wb0, wb1);
            mma_f16(ov[4 * j + 2 * h + 1], Ps & kLoNib, Ps & kHiNib, Qs & kLoNib, Qs & kHiNib, wb0, wb1);
          }
        }
      }
      }
    }
    __syncthreads();  // every warp is done with stage st
    if (tid == 0 && ok && ch + kStages < nchunks) issue(ch + kStages);
  }

  if constexpr (APP) if (app_warp && ok) {  // the new row into the cache (every copy of this kernel has completed)
    const int64_t slot = slot0 + L - 1;
    copy_row<D, NG>(reinterpret_cast<uint32_t *>(const_cast<uint8_t *>(a.kc)) + slot * (D / 8),
                    reinterpret_cast<uint32_t *>(const_cast<uint8_t *>(a.vc)) + slot * (D / 8),
                    const_cast<__half *>(a.km) + slot * NG, const_cast<__half *>(a.ks) + slot * NG,
                    const_cast<__half *>(a.vm) + slot * NG, const_cast<__half *>(a.vs) + slot * NG, new_codes,
                    new_meta, lane);
  }

  // ---- per-warp totals, then combine the 4 warps ----
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  l *= 0.5f;  // every token was counted by both lanes of its pair
#pragma unroll
  for (int o = (NG > 1 ? 2 : 1); o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < GPL; e++) vmin[e] += __shfl_xor_sync(0xffffffffu, vmin[e], o);
  if constexpr (NG == 1) vmin[0] *= 0.5f;
  {
    // lane (gid, c) with c == g/2 owns dims gid*D/8 .. +D/8-1 of group g = gid*(D/8)/G:
    // column g is element (g & 1) of its accumulator pairs; the V-min total of group g sits
    // in lane (g / GPL) % 2, element g % GPL
    const int g = gid * (D / 8) / G;
    const int gl = NG > 1 ? (g / GPL) & 1 : 0;
    float vm = __shfl_sync(0xffffffffu, vmin[0], gl);
    if constexpr (GPL == 2) {
      const float vm1 = __shfl_sync(0xffffffffu, vmin[1], gl);
      vm = (g & 1) ? vm1 : vm;
    }
    if (c == g / 2) {
      const bool odd = g & 1;
      float2 *dst = reinterpret_cast<float2 *>(&red_o[warp][gid * (D / 8)]);
#pragma unroll
      for (int t = 0; t < MT; t++)
        dst[t] = make_float2((odd ? ov[t][1] : ov[t][0]) * kS24 + vm, (odd ? ov[t][3] : ov[t][2]) * kS20 + vm);
    }
  }
  if (lane == 0) {
    red_m[warp] = m;
    red_l[warp] = l;
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

template <int D, int G, bool APP>
fg_status launch_k(const AttnArgs &a, cudaStream_t st) {
  using S = AttnShape<D, G>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    fg_status rc = fg_cuda_check(
        cudaFuncSetAttribute(attn_decode_kernel<D, G, APP>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM));
    if (rc != FG_OK) return rc;
    attr_set[dev] = true;
  }
  const int64_t ctas = static_cast<int64_t>(a.rows) * a.H;
  attn_decode_kernel<D, G, APP><<<static_cast<unsigned>(ctas), kWarps * 32, S::SMEM, st>>>(a);
  return fg_launch_check();
}

template <int D, int G>
fg_status launch(const AttnArgs &a, cudaStream_t st) {
  return a.kn ? launch_k<D, G, true>(a, st) : launch_k<D, G, false>(a, st);
}

}  // namespace

fg_status fg_kv_validate(const fg_kv_cache *kv);
fg_status fg_attention_prefill_launch(const fg_kv_cache *kv, const fg_half *q, int64_t ldq, fg_half *out,
                                      int64_t ldo, int rows, int rows_per_seq, const int32_t *positions,
                                      cudaStream_t st);

// Prompt rows (rows_per_seq > 1) go to the tiled prefill kernel, which reads each K/V tile once
// for 64 query rows; decode rows, and head dims that kernel does not take, to this one.
fg_status fg_attention_launch(const fg_kv_cache *kv, const fg_half *q, int64_t ldq, fg_half *out, int64_t ldo,
                              int rows, int rows_per_seq, const int32_t *positions, cudaStream_t st,
                              const fg_half *k_new, const fg_half *v_new, int64_t ld_new) {
  if (k_new && rows_per_seq != 1) return FG_ERR_INVALID;  // the fused append is for decode rows
  if (rows_per_seq > 1) {
    const fg_status rc = fg_attention_prefill_launch(kv, q, ldq, out, ldo, rows, rows_per_seq, positions, st);
    if (rc != FG_ERR_UNSUPPORTED) return rc;
  }
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
  a.kn = reinterpret_cast<const __half *>(k_new);
  a.vn = reinterpret_cast<const __half *>(v_new);
  a.ldn = ld_new;
  const int G = fg_kv_group(kv->group);
  if (G == 64) {
    switch (kv->head_dim) {
      case 64: return launch<64, 64>(a, st);
      case 128: return launch<128, 64>(a, st);
      case 256: return launch<256, 64>(a, st);
    }
  } else if (G == 128) {
    switch (kv->head_dim) {
      case 128: return launch<128, 128>(a, st);
      case 256: return launch<256, 128>(a, st);
    }
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
  return fg_attention_launch(kv, q, ldq, out, ldo, rows, rows_per_seq, positions, static_cast<cudaStream_t>(stream),
                             nullptr, nullptr, 0);
}

extern "C" fg_status fg_attention_decode_append(const fg_kv_cache *kv, const fg_half *q, int64_t ldq,
                                                const fg_half *k, const fg_half *v, int64_t ldkv, fg_half *out,
                                                int64_t ldo, int rows, const int32_t *positions, void *stream) {
  fg_status rc = fg_kv_validate(kv);
  if (rc != FG_OK) return rc;
  if (rows < 0 || rows > kv->num_seqs) return FG_ERR_SHAPE;
  if (rows == 0) return FG_OK;
  if (!q || !out || !k || !v || !positions) return FG_ERR_INVALID;
  if (!fg_aligned16(q) || !fg_aligned16(out) || !fg_aligned16(k) || !fg_aligned16(v)) return FG_ERR_INVALID;
  const int64_t hD = static_cast<int64_t>(kv->num_heads) * kv->head_dim;
  if (ldq < hD || ldo < hD || ldkv < hD || ldq % 8 || ldo % 8 || ldkv % 8) return FG_ERR_SHAPE;
  return fg_attention_launch(kv, q, ldq, out, ldo, rows, 1, positions, static_cast<cudaStream_t>(stream), k, v, ldkv);
}
