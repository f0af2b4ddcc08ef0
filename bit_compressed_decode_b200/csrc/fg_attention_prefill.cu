// fg_attention_prefill.cu -- causal softmax attention of a prompt's query rows over the 4-bit
// KV cache, tiled so that every K/V tile is read and dequantised once for 64 query rows.
//
// "FlexGen Guide: High-Throughput LLM Offloading on One GPU", section 3: the KV cache is
// held as 4-bit groups and dequantised on the fly for FP16 compute; attention reads it in
// that form, the prompt's own tokens included (they are appended before attention).  The
// tiling follows the IO-aware attention of the dev.to guide "Optimizing LLM for low memory
// usage" (Efficient Attention Implementations): query blocks against key/value tiles with a
// running maximum and running sum per row, never forming the full score matrix.
//
// One CTA (4 warps) per (sequence, head, block of 64 prompt rows).  Per tile of 64 keys:
//   - the tile's K and V codes and their fp16 group min/scale arrive in shared memory by
//     cp.async.bulk (two stages in flight, mbarrier completion);
//   - all threads dequantise them into fp16 K and V tiles in shared memory, each value
//     round(min + code * scale) exactly as the decode path and fg_dequantize compute it;
//     keys past the block's last visible key are zeroed (their slots may hold anything);
//   - each warp multiplies its 16 query rows by the tile on the tensor cores
//     (mma.sync m16n8k16, fp16 operands from ldmatrix, fp32 accumulators), masks keys past
//     each row's position, updates the row's running max and sum, and accumulates P V with
//     P rounded to fp16 (the accumulator layout of S is the A-operand layout of P V).
// Row t of sequence s (prompt position positions[s] + t) attends over cache positions
// 0 .. positions[s] + t.  Query rows are pre-scaled by head_dim^-1/2 (the QKV epilogue).
#include <math.h>

#include "fg_internal.cuh"

namespace {

constexpr int kRows = 64;     // query rows per CTA (16 per warp)
constexpr int kKeys = 64;     // keys per tile
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int G>
struct PShape {
  static constexpr int NG = D / G;                    // G-groups (G = 64 or 128) per head row
  static constexpr int PITCH = D + 8;                 // fp16 row pitch of the Q/K/V tiles (ldmatrix: no bank conflicts)
  static constexpr int TILE_B = kKeys * PITCH * 2;    // one fp16 tile
  static constexpr int CODE_B = kKeys * D / 2;        // one tile's K (or V) codes
  static constexpr int META_B = kKeys * NG * 2;       // one tile's metadata array
  static constexpr int STAGE_B = 2 * CODE_B + 4 * META_B;
  static constexpr int SMEM = 3 * TILE_B + 2 * STAGE_B;  // Q, K, V tiles + two code stages
};

struct PrefillArgs {
  const __half *q;
  int64_t ldq;
  __half *out;
  int64_t ldo;
  const uint8_t *kc, *vc;
  const __half *km, *ks, *vm, *vs;
  const int32_t *positions;
  int num_seqs, P, H, maxL, qblocks;
  unsigned int *err;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// d += A * B, m16n8k16, fp16 operands, fp32 accumulators (PTX fragment layout).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 3) attn_prefill_kernel(const PrefillArgs a) {
  using S = PShape<D, G>;
  constexpr int NG = S::NG, PITCH = S::PITCH, KT = D / 16, NT = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[2];
  griddep_launch();

  __half *sQ = reinterpret_cast<__half *>(smem);
  __half *sK = reinterpret_cast<__half *>(smem + S::TILE_B);
  __half *sV = reinterpret_cast<__half *>(smem + 2 * S::TILE_B);
  uint8_t *stage0 = smem + 3 * S::TILE_B;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, c = lane & 3;
  // heaviest query blocks (most key tiles) first
  const int qb = a.qblocks - 1 - static_cast<int>(blockIdx.x % a.qblocks);
  const int sh = static_cast<int>(blockIdx.x / a.qblocks);
  const int s = sh / a.H, hd = sh % a.H;
  const int t0 = qb * kRows;
  const int pos0 = a.positions[s];
  const int last_row = min(t0 + kRows, a.P) - 1;           // last prompt row of this block
  const int kmax = pos0 + last_row;                         // last key any row of the block sees
  if (pos0 < 0 || kmax >= a.maxL) {                         // cache positions out of range: flag, zeros
    if (tid == 0) atomicOr(a.err, FG_DEVERR_RANGE);
    for (int i = tid; i < (last_row - t0 + 1) * D; i += kThreads) {
      const int r = t0 + i / D;
      a.out[(static_cast<int64_t>(s) * a.P + r) * a.ldo + hd * D + i % D] = __float2half_rn(0.f);
    }
    return;
  }
  const int ntiles = kmax / kKeys + 1;
  const int64_t slot0 = (static_cast<int64_t>(s) * a.H + hd) * a.maxL;

  auto issue = [&](int j) {
    uint8_t *p = stage0 + (j & 1) * S::STAGE_B;
    const uint32_t bar = smem_u32(&full_bar[j & 1]);
    mbar_arrive_expect_tx(bar, 2 * S::CODE_B + 4 * S::META_B);
    const int64_t k0 = slot0 + static_cast<int64_t>(j) * kKeys;
    bulk_g2s(smem_u32(p), a.kc + k0 * (D / 2), S::CODE_B, bar);
    bulk_g2s(smem_u32(p + S::CODE_B), a.vc + k0 * (D / 2), S::CODE_B, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 0 * S::META_B), a.km + k0 * NG, S::META_B, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 1 * S::META_B), a.ks + k0 * NG, S::META_B, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 2 * S::META_B), a.vm + k0 * NG, S::META_B, bar);
    bulk_g2s(smem_u32(p + 2 * S::CODE_B + 3 * S::META_B), a.vs + k0 * NG, S::META_B, bar);
  };

  if (tid == 0) {
    mbar_init(smem_u32(&full_bar[0]), 1);
    mbar_init(smem_u32(&full_bar[1]), 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    issue(0);
    if (ntiles > 1) issue(1);
  }

  // ---- Q block -> shared memory -> A fragments (rows past the prompt read row P-1) ----
  for (int i = tid; i < kRows * (D / 8); i += kThreads) {
    const int r = i / (D / 8), cc = i % (D / 8);
    const int t = min(t0 + r, a.P - 1);
    const uint4 v = *reinterpret_cast<const uint4 *>(a.q + (static_cast<int64_t>(s) * a.P + t) * a.ldq + hd * D + cc * 8);
    *reinterpret_cast<uint4 *>(sQ + r * PITCH + cc * 8) = v;
  }
  __syncthreads();
  uint32_t qf[KT][4];
  {
    const int r = warp * 16 + (lane & 15);
    const uint32_t base = smem_u32(sQ + r * PITCH + (lane >> 4) * 8);
#pragma unroll
    for (int kk = 0; kk < KT; kk++) ldsm_x4(base + kk * 32, qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
  }

  // this thread's two rows (gid and gid + 8 of the warp's 16) and the last key each may see
  const int row0 = t0 + warp * 16 + gid;
  const int lim0 = pos0 + min(row0, a.P - 1), lim1 = pos0 + min(row0 + 8, a.P - 1);
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; n++) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  bool ok = true;
  for (int j = 0; j < ntiles; j++) {
    // ---- dequantise tile j into sK, sV ----
    if (ok && !mbar_wait_bounded(smem_u32(&full_bar[j & 1]), (j >> 1) & 1, nullptr, a.err)) ok = false;
    if (ok) {
      const uint8_t *p = stage0 + (j & 1) * S::STAGE_B;
      const uint32_t *kcw = reinterpret_cast<const uint32_t *>(p);
      const uint32_t *vcw = reinterpret_cast<const uint32_t *>(p + S::CODE_B);
      const __half *Km = reinterpret_cast<const __half *>(p + 2 * S::CODE_B);
      const __half *Ks = Km + kKeys * NG, *Vm = Ks + kKeys * NG, *Vs = Vm + kKeys * NG;
#pragma unroll 4
      for (int u = tid; u < kKeys * (D / 8); u += kThreads) {
        const int key = u / (D / 8), w = u % (D / 8), g = w / (G / 8);
        const bool live = j * kKeys + key <= kmax;
        const int mi = key * NG + g;
        const uint4 kv = live ? dequant8(kcw[u], __half2half2(Ks[mi]), __half2half2(Km[mi])) : make_uint4(0, 0, 0, 0);
        const uint4 vv = live ? dequant8(vcw[u], __half2half2(Vs[mi]), __half2half2(Vm[mi])) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>(sK + key * PITCH + w * 8) = kv;
        *reinterpret_cast<uint4 *>(sV + key * PITCH + w * 8) = vv;
      }
    }
    __syncthreads();  // tiles ready; stage j & 1 consumed
    if (tid == 0 && ok && j + 2 < ntiles) {
      fence_proxy_async_smem();
      issue(j + 2);
    }
    if (ok) {
      // ---- S = Q K^T for 16 rows x 64 keys (8 key groups of 8) ----
      float sc[8][4];
#pragma unroll
      for (int n = 0; n < 8; n++) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int np = 0; np < 4; np++) {  // key groups 2np, 2np + 1
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const uint32_t base = smem_u32(sK + key * PITCH + ((lane >> 3) & 1) * 8);
#pragma unroll
        for (int kk = 0; kk < KT; kk++) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(base + kk * 32, b0, b1, b2, b3);
          mma16816(sc[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
          mma16816(sc[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
        }
      }
      // ---- mask, running max / sum (log2 units) ----
      float tmax0 = -INFINITY, tmax1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < 8; n++) {
        const int key = j * kKeys + n * 8 + 2 * c;
        sc[n][0] = key <= lim0 ? sc[n][0] * kLog2e : -INFINITY;
        sc[n][1] = key + 1 <= lim0 ? sc[n][1] * kLog2e : -INFINITY;
        sc[n][2] = key <= lim1 ? sc[n][2] * kLog2e : -INFINITY;
        sc[n][3] = key + 1 <= lim1 ? sc[n][3] * kLog2e : -INFINITY;
        tmax0 = fmaxf(tmax0, fmaxf(sc[n][0], sc[n][1]));
        tmax1 = fmaxf(tmax1, fmaxf(sc[n][2], sc[n][3]));
      }
      tmax0 = fmaxf(tmax0, __shfl_xor_sync(0xffffffffu, tmax0, 1));
      tmax0 = fmaxf(tmax0, __shfl_xor_sync(0xffffffffu, tmax0, 2));
      tmax1 = fmaxf(tmax1, __shfl_xor_sync(0xffffffffu, tmax1, 1));
      tmax1 = fmaxf(tmax1, __shfl_xor_sync(0xffffffffu, tmax1, 2));
      const float mn0 = fmaxf(m0, tmax0), mn1 = fmaxf(m1, tmax1);
      // a row sees key 0 in tile 0, so mn is finite from the first tile on
      const float al0 = exp2_approx(m0 - mn0), al1 = exp2_approx(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int n = 0; n < 8; n++) {
        sc[n][0] = exp2_approx(sc[n][0] - mn0);
        sc[n][1] = exp2_approx(sc[n][1] - mn0);
        sc[n][2] = exp2_approx(sc[n][2] - mn1);
        sc[n][3] = exp2_approx(sc[n][3] - mn1);
        rs0 += sc[n][0] + sc[n][1];
        rs1 += sc[n][2] + sc[n][3];
      }
      l0 = l0 * al0 + rs0;
      l1 = l1 * al1 + rs1;
#pragma unroll
      for (int n = 0; n < NT; n++) {
        o[n][0] *= al0;
        o[n][1] *= al0;
        o[n][2] *= al1;
        o[n][3] *= al1;
      }
      // ---- O += P V: P (fp16) from the S accumulators, V via transposed ldmatrix ----
#pragma unroll
      for (int kk = 0; kk < kKeys / 16; kk++) {
        const uint32_t a0 = pack_f16x2(sc[2 * kk][0], sc[2 * kk][1]);
        const uint32_t a1 = pack_f16x2(sc[2 * kk][2], sc[2 * kk][3]);
        const uint32_t a2 = pack_f16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
        const uint32_t a3 = pack_f16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
        const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const uint32_t base = smem_u32(sV + key * PITCH + (lane >> 4) * 8);
#pragma unroll
        for (int np = 0; np < NT / 2; np++) {  // dims 16 np .. 16 np + 15
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(base + np * 32, b0, b1, b2, b3);
          mma16816(o[2 * np], a0, a1, a2, a3, b0, b1);
          mma16816(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncthreads();  // every warp is done with sK, sV
  }

  if (!ok && tid == 0) {
    // a wait gave up: let the copies still in flight land before the CTA exits
    for (int j = 0; j < ntiles; j++) mbar_wait_bounded(smem_u32(&full_bar[j & 1]), (j >> 1) & 1, nullptr, nullptr);
  }

  // ---- normalise and store the rows of the prompt ----
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = ok ? 1.f / l0 : 0.f, inv1 = ok ? 1.f / l1 : 0.f;
  __half *out0 = a.out + (static_cast<int64_t>(s) * a.P + row0) * a.ldo + hd * D;
  __half *out1 = out0 + 8 * a.ldo;
#pragma unroll
  for (int n = 0; n < NT; n++) {
    const int col = n * 8 + 2 * c;
    if (row0 < a.P) *reinterpret_cast<uint32_t *>(out0 + col) = pack_f16x2(o[n][0] * inv0, o[n][1] * inv0);
    if (row0 + 8 < a.P) *reinterpret_cast<uint32_t *>(out1 + col) = pack_f16x2(o[n][2] * inv1, o[n][3] * inv1);
  }
}

template <int D, int G>
fg_status launch(const PrefillArgs &a, cudaStream_t st) {
  using S = PShape<D, G>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    fg_status rc = fg_cuda_check(
        cudaFuncSetAttribute(attn_prefill_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM));
    if (rc != FG_OK) return rc;
    attr_set[dev] = true;
  }
  const int64_t ctas = static_cast<int64_t>(a.num_seqs) * a.H * a.qblocks;
  if (ctas > INT32_MAX) return FG_ERR_SHAPE;
  attn_prefill_kernel<D, G><<<static_cast<unsigned>(ctas), kThreads, S::SMEM, st>>>(a);
  return fg_launch_check();
}

}  // namespace

// Prompt rows (rows_per_seq > 1) with head_dim 64 or 128 (groups of 64, or of 128 at head_dim
// 128); returns FG_ERR_UNSUPPORTED for other head dims (the caller then uses the row-by-row
// kernel).  q, out: row (s * P + t) holds
// sequence s, prompt token t; ldq, ldo multiples of 8.
fg_status fg_attention_prefill_launch(const fg_kv_cache *kv, const fg_half *q, int64_t ldq, fg_half *out,
                                      int64_t ldo, int rows, int rows_per_seq, const int32_t *positions,
                                      cudaStream_t st) {
  if (kv->head_dim != 64 && kv->head_dim != 128) return FG_ERR_UNSUPPORTED;
  PrefillArgs a;
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
  a.P = rows_per_seq;
  a.num_seqs = rows / rows_per_seq;
  a.H = kv->num_heads;
  a.maxL = kv->max_len;
  a.qblocks = (rows_per_seq + kRows - 1) / kRows;
  a.err = fg_error_word_ptr();
  if (!a.err) return FG_ERR_CUDA;
  const int G = fg_kv_group(kv->group);
  if (kv->head_dim == 64) return G == 64 ? launch<64, 64>(a, st) : FG_ERR_UNSUPPORTED;
  return G == 64 ? launch<128, 64>(a, st) : launch<128, 128>(a, st);
}
