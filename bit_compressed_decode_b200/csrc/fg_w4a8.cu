// fg_w4a8.cu -- W4A8 linear layer: 4-bit weights and 8-bit activations multiplied as integers on
// the 5th-generation tensor cores (tcgen05.mma kind::i8, s32 accumulators in TMEM).
//
// The pages name W4A8 through the QServe W4A8KV4 title in the PIPO paper's list of references and
// list INT8 and INT4 among the post-training weight formats ("Optimizing LLM for low memory usage",
// Quantization and Weight Compression); the groups of 64 come from the "FlexGen Guide", section 3.
// The scheme is a reading of those:
//   weights [N][K], two levels: per row, symmetric int8 with bound 113 and an fp32 scale cscale[n];
//     per group of 64 along k, the int8 values as gmin + code * gstep with 4-bit codes (nearest,
//     halves up) and an integer step 1..16.  The bound 113 keeps gmin + 15 * gstep <= 127 for every
//     group, so the weight the product uses is always an int8.
//   activations [M][K]: per row, symmetric int8 with bound 127 and an fp32 scale ascale[t];
//   y[t][n] = epi( acc[t][n] * (ascale[t] * cscale[n]) + bias[n] ), acc = sum_k a8 * w8 exact in
//     int32, the rest one fp32 operation at a time (q-scale, ReLU, residual as in the W4A16 layer).
//
// Larger blocks (M > 256, with rows of K / 64 metadata bytes that are whole 16-byte units) run on
// CTA pairs: the W4A16 pair kernel (fg_gemm.cu) in its int8 form -- the same pipeline with the
// codes widened to int8, tcgen05.mma.cta_group::2.kind::i8 and the scales applied once a sum is
// final.
//
// GEMM kernel, one SM per output tile (every other shape): 256 output features (two 128-row accumulators) x NT tokens
// x a k-range, k-tiles of 128 (two groups; one 128-byte row of int8 per feature and per token).
//   warps 0..7  thread t owns weight row n0 + t: per k-tile it loads 64 code bytes and both groups'
//               (gmin, gstep), widens 8 codes at a time to int8 -- two byte permutes, one 32-bit
//               multiply by the step (code * step <= 240: no carry between bytes) and a per-byte
//               add of gmin -- and stores 128 bytes into the 128-byte-swizzled K-major A tile;
//               afterwards the epilogue (TMEM -> registers -> fp16).
//   warp 8      TMA of the activation tile [NT tokens x 128] per k-tile.
//   warp 9      one lane issues tcgen05.mma kind::i8 (M = 128, N = NT, K = 32) per 32-byte k-step.
//   A k split forms the cluster's z dimension; the int32 partials are summed over distributed
//   shared memory (exact, so the result does not depend on the split).
// Every mbarrier wait is bounded (FG_WAIT_TIMEOUT_NS) and reports FG_ERR_TIMEOUT.
#include "fg_internal.cuh"

// the CTA-pair launch for M > 256 (fg_gemm.cu): the W4A16 pair kernel's int8 form
bool fg_w4a8_pair_eligible(int M, int K, const fg_w4a8_weight *w);
size_t fg_w4a8_pair_ws_bytes(int M, int N, int K);
void fg_w4a8_pair_plan(int M, int N, int K, int *tile_tokens, int *splits);
fg_status fg_w4a8_pair_launch(const int8_t *a8, const float *ascale, int M, int K, const fg_w4a8_weight *w,
                              const fg_half *bias, const fg_half *residual, int flags, int qscale_cols, float qscale,
                              fg_half *y, void *workspace, size_t ws_bytes, cudaStream_t st);

namespace {

constexpr int kBK = 128;   // k per tile: one 128-byte row of int8
constexpr int kGrp = 64;   // weight group along k
constexpr int kNAcc = 2;   // 128-feature accumulators per CTA
constexpr int kBM = 128 * kNAcc;
constexpr int kDeqWarps = 4 * kNAcc;
constexpr int kTmaWarp = kDeqWarps;
constexpr int kMmaWarp = kDeqWarps + 1;
constexpr int kThreads = (kDeqWarps + 2) * 32;
constexpr int kPrefetch = 2;  // k-tiles of codes in flight per dequantising thread
constexpr int kW8Bound = 113;
constexpr int kA8Bound = 127;

// Instruction descriptor: kind::i8 with signed 8-bit A and B, s32 D, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_s8_s32(int M, int N) {
  return (2u << 4)                                // D format: s32
         | (1u << 7) | (1u << 10)                 // A, B format: signed 8-bit
         | (0u << 15) | (0u << 16)                // A, B K-major
         | (static_cast<uint32_t>(N >> 3) << 17)  // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24); // M / 16
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, int8 inputs, int32 accumulation.
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

template <int NT>
struct Cfg8 {
  static constexpr int STAGES = NT >= 256 ? 3 : 4;
  static constexpr int A_BYTES = 128 * 128;  // one accumulator's A tile: 128 rows x 128 B
  static constexpr int B_BYTES = NT * 128;   // activation tile: NT rows x 128 B
  static constexpr int STAGE = kNAcc * A_BYTES + B_BYTES;
  static constexpr int SMEM = STAGES * STAGE + 1024;  // + alignment slack
  static constexpr int COLS = kNAcc * NT < 32 ? 32 : kNAcc * NT;
  static constexpr uint32_t IDESC = umma_idesc_s8_s32(128, NT);
};

struct Args8 {
  const uint8_t *wc;       // codes [N][K/2]
  const int8_t *gmin;      // [N][K/64]
  const uint8_t *gstep;    // [N][K/64]
  const float *cscale;     // [N]
  const float *ascale;     // [M]
  const __half *bias;      // [N] or null
  const __half *res;       // [M][N] or null
  __half *y;               // [M][N]
  int M, N, K;
  int relu, qcols;
  float qscale;
  int splits;
  unsigned int *err;
};

// 8 codes of one word (element 2j in the low nibble of byte j) -> the 8 int8 weights
// gmin + code * step in element order, as two words: each byte formed in offset binary,
// code * step + (gmin + 128) in [15, 255] (no carry between bytes), then its top bit flipped.
// off4 = (gmin + 128) replicated into the 4 bytes.
__device__ __forceinline__ uint2 widen8(uint32_t w, uint32_t step, uint32_t off4) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t e0 = __byte_perm(lo, hi, 0x5140), e1 = __byte_perm(lo, hi, 0x7362);
  return make_uint2((e0 * step + off4) ^ 0x80808080u, (e1 * step + off4) ^ 0x80808080u);
}

// acc -> fp32 scale, bias, q-scale, ReLU, residual: one IEEE fp32 operation each
__device__ __forceinline__ float epilogue8(int acc, float cs, float bias, float res, int n, const Args8 &a) {
  float v = __fmul_rn(__int2float_rn(acc), cs);
  v = __fadd_rn(v, bias);
  if (n < a.qcols) v = __fmul_rn(v, a.qscale);
  if (a.relu) v = fmaxf(v, 0.f);
  return __fadd_rn(v, res);
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) w4a8_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                                                                const Args8 a) {
  using C = Cfg8<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_a[C::STAGES], full_b[C::STAGES], empty[C::STAGES], accum_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kBM, t0 = blockIdx.y * NT, split = blockIdx.z;
  const int ktiles = a.K / kBK;
  const int kt0 = static_cast<int>((static_cast<int64_t>(split) * ktiles) / a.splits);
  const int kt1 = static_cast<int>((static_cast<int64_t>(split + 1) * ktiles) / a.splits);
  const int nk = kt1 - kt0;
  volatile int *abortp = &abort_flag;

  auto a_tile = [&](int st, int acc) { return smem + st * C::STAGE + acc * C::A_BYTES; };
  auto b_tile = [&](int st) { return smem + st * C::STAGE + kNAcc * C::A_BYTES; };

  if (tid == 0) {
    for (int i = 0; i < C::STAGES; i++) {
      mbar_init(smem_u32(&full_a[i]), kDeqWarps);
      mbar_init(smem_u32(&full_b[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    mbar_init(smem_u32(&accum_bar), 1);
    abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&tmem_slot), C::COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp < kDeqWarps) {
    // ---------------- widen the 4-bit codes to int8: one weight row per thread ----------------
    const int row = tid;  // 0..255
    const int n = n0 + row;
    const bool live = n < a.N;
    const int acc = row >> 7, r = row & 127;
    const int ng = a.K / kGrp;
    const uint4 *crow = reinterpret_cast<const uint4 *>(a.wc + static_cast<int64_t>(live ? n : 0) * (a.K / 2));
    const uint16_t *mrow = reinterpret_cast<const uint16_t *>(a.gmin + static_cast<int64_t>(live ? n : 0) * ng);
    const uint16_t *srow = reinterpret_cast<const uint16_t *>(a.gstep + static_cast<int64_t>(live ? n : 0) * ng);
    uint4 cb[kPrefetch][4];
    uint16_t mb[kPrefetch], sb[kPrefetch];
#pragma unroll
    for (int j = 0; j < kPrefetch; j++) {
      if (j < nk && live) {
        const int kt = kt0 + j;
#pragma unroll
        for (int u = 0; u < 4; u++) cb[j][u] = crow[kt * 4 + u];
        mb[j] = mrow[kt];
        sb[j] = srow[kt];
      } else {
#pragma unroll
        for (int u = 0; u < 4; u++) cb[j][u] = make_uint4(0, 0, 0, 0);
        mb[j] = sb[j] = 0;
      }
    }
    bool go = true;
    for (int i0 = 0; go && i0 < nk; i0 += kPrefetch) {
#pragma unroll
      for (int j = 0; j < kPrefetch; j++) {
        const int i = i0 + j;
        if (!go || i >= nk) break;
        const int st = i % C::STAGES;
        const uint4 c0 = cb[j][0], c1 = cb[j][1], c2 = cb[j][2], c3 = cb[j][3];
        const uint32_t m2 = mb[j], s2 = sb[j];
        if (i + kPrefetch < nk && live) {
          const int kt = kt0 + i + kPrefetch;
#pragma unroll
          for (int u = 0; u < 4; u++) cb[j][u] = crow[kt * 4 + u];
          mb[j] = mrow[kt];
          sb[j] = srow[kt];
        }
        if (i >= C::STAGES &&
            !mbar_wait_bounded(smem_u32(&empty[st]), ((i / C::STAGES) - 1) & 1, abortp, a.err)) {
          go = false;
          break;
        }
        // group 2kt in the low byte of m2/s2, group 2kt+1 in the high byte
        const uint32_t min_lo = ((m2 & 0xFFu) ^ 0x80u) * 0x01010101u, min_hi = ((m2 >> 8) ^ 0x80u) * 0x01010101u;  // gmin + 128
        const uint32_t step_lo = s2 & 0xFFu, step_hi = s2 >> 8;
        uint8_t *at = a_tile(st, acc);
        const uint32_t words[16] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w,
                                    c2.x, c2.y, c2.z, c2.w, c3.x, c3.y, c3.z, c3.w};
#pragma unroll
        for (int c = 0; c < 8; c++) {  // 16-byte chunk c: elements 16c..16c+15, code words 2c, 2c+1
          const uint32_t mn4 = c < 4 ? min_lo : min_hi, stp = c < 4 ? step_lo : step_hi;
          const uint2 p = widen8(words[2 * c], stp, mn4), q = widen8(words[2 * c + 1], stp, mn4);
          const uint4 v = live ? make_uint4(p.x, p.y, q.x, q.y) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(at + sw128_offset(r, c)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&full_a[st]));
      }
    }
  } else if (warp == kTmaWarp) {
    // ---------------- TMA producer for the activation tiles ----------------
    if (lane == 0) {
      prefetch_tmap(&amap);
      int issued = 0;
      for (int i = 0; i < nk; i++) {
        const int st = i % C::STAGES;
        if (i >= C::STAGES && !mbar_wait_bounded(smem_u32(&empty[st]), ((i / C::STAGES) - 1) & 1, abortp, a.err))
          break;
        const uint32_t bar = smem_u32(&full_b[st]);
        mbar_arrive_expect_tx(bar, C::B_BYTES);
        tma_load_2d(smem_u32(b_tile(st)), &amap, (kt0 + i) * kBK, t0, bar);
        issued = i + 1;
      }
      if (*abortp) {  // let copies still in flight land before the CTA exits
        for (int j = issued > C::STAGES ? issued - C::STAGES : 0; j < issued; j++)
          mbar_wait_bounded(smem_u32(&full_b[j % C::STAGES]), (j / C::STAGES) & 1, nullptr, nullptr);
      }
    }
  } else {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      for (int i = 0; i < nk; i++) {
        const int st = i % C::STAGES;
        const uint32_t par = (i / C::STAGES) & 1;
        if (!mbar_wait_bounded(smem_u32(&full_a[st]), par, abortp, a.err)) break;
        if (!mbar_wait_bounded(smem_u32(&full_b[st]), par, abortp, a.err)) break;
        tc_fence_after();
        const uint32_t bbase = smem_u32(b_tile(st));
#pragma unroll
        for (int kk = 0; kk < kBK / 32; kk++) {  // 32 int8 = 32 bytes per MMA
          const uint64_t bdesc = umma_desc_sw128(bbase + kk * 32);
#pragma unroll
          for (int acc = 0; acc < kNAcc; acc++) {
            const uint64_t adesc = umma_desc_sw128(smem_u32(a_tile(st, acc)) + kk * 32);
            umma_i8(tmem + acc * NT, adesc, bdesc, C::IDESC, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(smem_u32(&empty[st]));
      }
      umma_commit(smem_u32(&accum_bar));  // also tracks completion if the loop stopped early
    }
  }

  // ---------------- epilogue: TMEM -> registers -> global ----------------
  constexpr int kChunks = NT >= 32 ? NT / 32 : 1;
  constexpr int kCW = NT >= 32 ? 32 : NT;
  bool ready = false;
  if (warp < kDeqWarps) {
    ready = mbar_wait_bounded(smem_u32(&accum_bar), 0, nullptr, a.err) && !*abortp;
    tc_fence_after();
  }
  const int acc = (warp & 7) >> 2, q = warp & 3;
  const int n = n0 + acc * 128 + q * 32 + lane;
  const bool nlive = n < a.N;
  auto load_chunk = [&](int ch, uint32_t (&v)[32]) {
    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * NT + ch * kCW;
    if constexpr (NT >= 32) {
      tmem_ld_32x32b_x32(taddr, v);
    } else {
      tmem_ld_32x32b_x16(taddr, v);
    }
    tmem_wait_ld();
  };
  if (a.splits == 1) {
    if (warp < kDeqWarps) {
      const float bias = (a.bias && nlive) ? __half2float(a.bias[n]) : 0.f;
      const float cscale = nlive ? a.cscale[n] : 0.f;
      for (int ch = 0; ch < kChunks; ch++) {
        uint32_t v[32];
        load_chunk(ch, v);
        if (!ready || !nlive) continue;
        float res[kCW];
#pragma unroll
        for (int j = 0; j < kCW; j++) {
          const int m = t0 + ch * kCW + j;
          res[j] = (a.res && m < a.M) ? __half2float(a.res[static_cast<int64_t>(m) * a.N + n]) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < kCW; j++) {
          const int m = t0 + ch * kCW + j;
          if (m < a.M) {
            const float cs = __fmul_rn(a.ascale[m], cscale);
            a.y[static_cast<int64_t>(m) * a.N + n] =
                __float2half_rn(epilogue8(static_cast<int>(v[j]), cs, bias, res[j], n, a));
          }
        }
      }
    }
  } else {
    // Cluster reduction of the k-split partial sums (int32, exact).  Chunks are staged kRound at
    // a time in the idle pipeline buffers as [chunk][column][feature]; chunk ch is finished by
    // cluster rank ch % splits.  Every thread of every CTA takes the same cluster barriers.
    constexpr int kChunkBytes = kCW * kBM * 4;
    constexpr int kRound = (C::STAGES * C::STAGE) / kChunkBytes < kChunks ? (C::STAGES * C::STAGE) / kChunkBytes
                                                                           : kChunks;
    static_assert(kRound >= 1, "reduction buffer");
    const uint32_t rank = cluster_ctarank();
    uint32_t *buf = reinterpret_cast<uint32_t *>(smem);
    const int feat = tid;
    for (int r0 = 0; r0 < kChunks; r0 += kRound) {
      if (warp < kDeqWarps) {
        for (int i = 0; i < kRound && r0 + i < kChunks; i++) {
          uint32_t v[32];
          load_chunk(r0 + i, v);
          uint32_t *cbuf = buf + i * (kCW * kBM);
          const int f = acc * 128 + q * 32 + lane;
#pragma unroll
          for (int j = 0; j < kCW; j++) cbuf[j * kBM + f] = v[j];
        }
      }
      __syncwarp();
      cluster_sync_all();
      if (warp < kDeqWarps && ready) {
        const int nn = n0 + feat;
        const bool live = nn < a.N;
        const float rbias = (a.bias && live) ? __half2float(a.bias[nn]) : 0.f;
        const float cscale = live ? a.cscale[nn] : 0.f;
        for (int i = 0; i < kRound && r0 + i < kChunks; i++) {
          const int ch = r0 + i;
          if (ch % a.splits != static_cast<int>(rank)) continue;
          const uint32_t base = smem_u32(buf + i * (kCW * kBM) + feat);
          for (int j = 0; j < kCW; j++) {
            int sum = 0;
            for (int sp = 0; sp < a.splits; sp++) sum += static_cast<int>(ld_shared_cluster_u32(mapa_shared(base + j * kBM * 4, sp)));
            const int m = t0 + ch * kCW + j;
            if (m < a.M && live) {
              const float res = a.res ? __half2float(a.res[static_cast<int64_t>(m) * a.N + nn]) : 0.f;
              const float cs = __fmul_rn(a.ascale[m], cscale);
              a.y[static_cast<int64_t>(m) * a.N + nn] = __float2half_rn(epilogue8(sum, cs, rbias, res, nn, a));
            }
          }
        }
      }
      __syncwarp();
      cluster_sync_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::COLS);
  }
}

// ------------------------------------------------------------------------------------
// quantisers
// ------------------------------------------------------------------------------------

// max over the CTA of a non-negative value (every thread gets it); `red` holds one slot per warp
template <int THREADS>
__device__ __forceinline__ float cta_max(float v, float *red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = 0.f;
#pragma unroll
  for (int w = 0; w < THREADS / 32; w++) m = fmaxf(m, red[w]);
  __syncthreads();
  return m;
}

__device__ __forceinline__ float absmax8(const uint4 &v, float m) {
  const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
  for (int j = 0; j < 4; j++) {
    const float2 f = __half22float2(h[j]);
    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
  }
  return m;
}

// round-half-even of x * inv (one fp32 multiply), clamped to [-bound, bound]
__device__ __forceinline__ int q8(float x, float inv, int bound) {
  const int c = __float2int_rn(__fmul_rn(x, inv));
  return c < -bound ? -bound : (c > bound ? bound : c);
}

// Activations: one CTA per row of K values (K % 8 == 0); ascale = amax / 127, codes
// round(x * (127 / amax)).
constexpr int kActThreads = 256;
__global__ void __launch_bounds__(kActThreads) act8_quant_kernel(const __half *x, int K, int8_t *a8, float *ascale) {
  __shared__ float red[kActThreads / 32];
  const int64_t t = blockIdx.x;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + t * K);
  const int nv = K / 8;
  float m = 0.f;
  for (int i = threadIdx.x; i < nv; i += kActThreads) m = absmax8(xr[i], m);
  const float amax = cta_max<kActThreads>(m, red);
  const float inv = amax > 0.f ? __fdiv_rn(static_cast<float>(kA8Bound), amax) : 0.f;
  if (threadIdx.x == 0) ascale[t] = amax > 0.f ? __fdiv_rn(amax, static_cast<float>(kA8Bound)) : 0.f;
  uint2 *out = reinterpret_cast<uint2 *>(a8 + t * K);
  for (int i = threadIdx.x; i < nv; i += kActThreads) {
    const uint4 v = xr[i];
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const float2 f = __half22float2(h[j]);
      const uint32_t b0 = static_cast<uint8_t>(q8(f.x, inv, kA8Bound)), b1 = static_cast<uint8_t>(q8(f.y, inv, kA8Bound));
      w[j >> 1] |= (b0 | (b1 << 8)) << ((j & 1) * 16);
    }
    out[i] = make_uint2(w[0], w[1]);
  }
}

// The same with the row held in registers (V 16-byte vectors per thread): one read of x.
template <int V>
__global__ void __launch_bounds__(kActThreads) act8_quant_reg_kernel(const __half *x, int K, int8_t *a8,
                                                                     float *ascale) {
  __shared__ float red[kActThreads / 32];
  const int64_t t = blockIdx.x;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + t * K);
  const int nv = K / 8;
  uint4 v[V];
  float m = 0.f;
#pragma unroll
  for (int u = 0; u < V; u++) {
    const int i = threadIdx.x + u * kActThreads;
    v[u] = i < nv ? xr[i] : make_uint4(0, 0, 0, 0);
    m = absmax8(v[u], m);
  }
  const float amax = cta_max<kActThreads>(m, red);
  const float inv = amax > 0.f ? __fdiv_rn(static_cast<float>(kA8Bound), amax) : 0.f;
  if (threadIdx.x == 0) ascale[t] = amax > 0.f ? __fdiv_rn(amax, static_cast<float>(kA8Bound)) : 0.f;
  uint2 *out = reinterpret_cast<uint2 *>(a8 + t * K);
#pragma unroll
  for (int u = 0; u < V; u++) {
    const int i = threadIdx.x + u * kActThreads;
    if (i >= nv) break;
    const __half2 *h = reinterpret_cast<const __half2 *>(&v[u]);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const float2 f = __half22float2(h[j]);
      const uint32_t b0 = static_cast<uint8_t>(q8(f.x, inv, kA8Bound)), b1 = static_cast<uint8_t>(q8(f.y, inv, kA8Bound));
      w[j >> 1] |= (b0 | (b1 << 8)) << ((j & 1) * 16);
    }
    out[i] = make_uint2(w[0], w[1]);
  }
}

// Weights: one CTA per row of K values (K % 64 == 0).  Level 1 as for the activations with bound
// 113; level 2 per group of 64: mn, mx of the int8 values, step = max(1, ceil((mx - mn) / 15)),
// code = floor((2 (w8 - mn) + step) / (2 step)).
constexpr int kWThreads = 128;
__global__ void __launch_bounds__(kWThreads) w4a8_quant_weight_kernel(const __half *w, int K, uint8_t *codes,
                                                                      int8_t *gmin, uint8_t *gstep, float *cscale) {
  __shared__ float red[kWThreads / 32];
  const int64_t n = blockIdx.x;
  const __half *row = w + n * K;
  const uint4 *wr = reinterpret_cast<const uint4 *>(row);
  float m = 0.f;
  for (int i = threadIdx.x; i < K / 8; i += kWThreads) m = absmax8(wr[i], m);
  const float amax = cta_max<kWThreads>(m, red);
  const float inv = amax > 0.f ? __fdiv_rn(static_cast<float>(kW8Bound), amax) : 0.f;
  if (threadIdx.x == 0) cscale[n] = amax > 0.f ? __fdiv_rn(amax, static_cast<float>(kW8Bound)) : 0.f;
  const int ng = K / kGrp;
  for (int g = threadIdx.x; g < ng; g += kWThreads) {
    const uint4 *gp = wr + g * (kGrp / 8);
    int mn = kW8Bound, mx = -kW8Bound;
#pragma unroll
    for (int u = 0; u < kGrp / 8; u++) {
      const uint4 v = gp[u];
      const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const float2 f = __half22float2(h[j]);
        const int a = q8(f.x, inv, kW8Bound), b = q8(f.y, inv, kW8Bound);
        mn = min(mn, min(a, b));
        mx = max(mx, max(a, b));
      }
    }
    int step = (mx - mn + 14) / 15;
    step = step < 1 ? 1 : step;
    const int two = 2 * step;
    uint32_t packed[kGrp / 8];
#pragma unroll
    for (int u = 0; u < kGrp / 8; u++) {  // 8 elements -> one 32-bit word of codes
      const uint4 v = gp[u];
      const __half2 *h = reinterpret_cast<const __half2 *>(&v);
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const float2 f = __half22float2(h[j]);
        const uint32_t c0 = static_cast<uint32_t>((2 * (q8(f.x, inv, kW8Bound) - mn) + step) / two);
        const uint32_t c1 = static_cast<uint32_t>((2 * (q8(f.y, inv, kW8Bound) - mn) + step) / two);
        word |= (c0 | (c1 << 4)) << (8 * j);
      }
      packed[u] = word;
    }
    uint4 *cp = reinterpret_cast<uint4 *>(codes + n * (K / 2) + g * (kGrp / 2));
    cp[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    cp[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    gmin[n * ng + g] = static_cast<int8_t>(mn);
    gstep[n * ng + g] = static_cast<uint8_t>(step);
  }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn8() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

struct Plan8 {
  int nt, n_tiles, t_tiles, splits;
};

// Token tile from M; the k-range is split over the CTAs of a cluster only to fill the SMs:
// minimise waves x k-tiles per CTA, with a small charge per extra split.
Plan8 make_plan8(int M, int N, int K) {
  Plan8 p;
  p.nt = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
  p.n_tiles = (N + kBM - 1) / kBM;
  p.t_tiles = (M + p.nt - 1) / p.nt;
  const int ktiles = K / kBK;
  const int base = p.n_tiles * p.t_tiles;
  const int nsm = fg_sm_count();
  double best = 1e30;
  p.splits = 1;
  for (int s = 1; s <= 8; s++) {
    if (s > 1 && ktiles / s < 4) break;
    const int waves = (base * s + nsm - 1) / nsm;
    const double cost = static_cast<double>(waves) * ((ktiles + s - 1) / s) * (1.0 + 0.05 * (s - 1));
    if (cost < best - 1e-9) {
      best = cost;
      p.splits = s;
    }
  }
  return p;
}

template <int NT>
fg_status launch8(const CUtensorMap &map, const Args8 &a, const Plan8 &p, cudaStream_t st) {
  using C = Cfg8<NT>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    fg_status rc = fg_cuda_check(
        cudaFuncSetAttribute(w4a8_gemm_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    if (rc != FG_OK) return rc;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(p.n_tiles, p.t_tiles, p.splits);
  lc.blockDim = dim3(kThreads, 1, 1);
  lc.dynamicSmemBytes = C::SMEM;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = p.splits;
  lc.attrs = attr;
  lc.numAttrs = 1;
  fg_status rc = fg_cuda_check(cudaLaunchKernelEx(&lc, w4a8_gemm_kernel<NT>, map, a));
  if (rc != FG_OK) return rc;
  return fg_launch_check();
}

bool w4a8_shape_ok(const fg_w4a8_weight *w) {
  return w && w->N > 0 && w->K > 0 && w->K % kGrp == 0 && w->N <= (1 << 30) && w->K <= (1 << 30);
}

}  // namespace

extern "C" fg_status fg_w4a8_quantize_weight(const fg_half *w, const fg_w4a8_weight *out, void *stream) {
  if (!out) return FG_ERR_INVALID;
  if (!w4a8_shape_ok(out)) return FG_ERR_SHAPE;
  if (!w || !out->codes || !out->gmin || !out->gstep || !out->cscale) return FG_ERR_INVALID;
  if (!fg_aligned16(w) || !fg_aligned16(out->codes) || (reinterpret_cast<uintptr_t>(out->cscale) & 3u))
    return FG_ERR_INVALID;
  if (out->N > 0x7FFFFFFF) return FG_ERR_SHAPE;
  w4a8_quant_weight_kernel<<<static_cast<unsigned>(out->N), kWThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __half *>(w), static_cast<int>(out->K), out->codes, out->gmin, out->gstep, out->cscale);
  return fg_launch_check();
}

extern "C" fg_status fg_act8_quantize(const fg_half *x, int M, int K, int8_t *a8, float *ascale, void *stream) {
  if (M < 0 || K <= 0) return FG_ERR_INVALID;
  if (K % kGrp) return FG_ERR_SHAPE;
  if (M == 0) return FG_OK;
  if (!x || !a8 || !ascale || !fg_aligned16(x) || !fg_aligned16(a8) || (reinterpret_cast<uintptr_t>(ascale) & 3u))
    return FG_ERR_INVALID;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __half *xh = reinterpret_cast<const __half *>(x);
  const int per = (K / 8 + kActThreads - 1) / kActThreads;  // 16-byte vectors per thread
  if (per <= 1)
    act8_quant_reg_kernel<1><<<M, kActThreads, 0, st>>>(xh, K, a8, ascale);
  else if (per <= 2)
    act8_quant_reg_kernel<2><<<M, kActThreads, 0, st>>>(xh, K, a8, ascale);
  else if (per <= 4)
    act8_quant_reg_kernel<4><<<M, kActThreads, 0, st>>>(xh, K, a8, ascale);
  else if (per <= 8)
    act8_quant_reg_kernel<8><<<M, kActThreads, 0, st>>>(xh, K, a8, ascale);
  else if (per <= 16)
    act8_quant_reg_kernel<16><<<M, kActThreads, 0, st>>>(xh, K, a8, ascale);
  else  // rows above 32768 values: two passes (the second from cache)
    act8_quant_kernel<<<M, kActThreads, 0, st>>>(xh, K, a8, ascale);
  return fg_launch_check();
}

extern "C" fg_status fg_linear_w4a8_plan(int M, int N, int K, int *tile_tokens, int *splits) {
  if (!tile_tokens || !splits || M <= 0 || N <= 0 || N % 128 || K <= 0 || K % kBK) return FG_ERR_INVALID;
  if (M > 256 && (K / kGrp) % 16 == 0) {
    fg_w4a8_pair_plan(M, N, K, tile_tokens, splits);
    return FG_OK;
  }
  const Plan8 p = make_plan8(M, N, K);
  *tile_tokens = p.nt;
  *splits = p.splits;
  return FG_OK;
}

extern "C" size_t fg_linear_w4a8_workspace_bytes(int M, int N, int K) {
  if (M <= 256 || N <= 0 || K <= 0 || K % kBK || (K / kGrp) % 16) return 0;
  return fg_w4a8_pair_ws_bytes(M, N, K);
}

extern "C" fg_status fg_linear_w4a8(const int8_t *a8, const float *ascale, int M, int K, const fg_w4a8_weight *w,
                                    const fg_half *bias, const fg_half *residual, int flags, int qscale_cols,
                                    float qscale, fg_half *y, void *workspace, size_t workspace_bytes,
                                    void *stream) {
  if (!w || M < 0 || K <= 0) return FG_ERR_INVALID;
  if (!w4a8_shape_ok(w) || w->K != K || K % kBK || K > 65536 || w->N % 128) return FG_ERR_SHAPE;
  if (flags & ~(FG_EPI_RELU | FG_EPI_RESIDUAL)) return FG_ERR_INVALID;
  if (M == 0) return FG_OK;
  if (!a8 || !ascale || !y || !w->codes || !w->gmin || !w->gstep || !w->cscale) return FG_ERR_INVALID;
  if (!fg_aligned16(a8) || !fg_aligned16(y) || !fg_aligned16(w->codes) ||
      (reinterpret_cast<uintptr_t>(w->gmin) & 1u) || (reinterpret_cast<uintptr_t>(w->gstep) & 1u) ||
      (reinterpret_cast<uintptr_t>(w->cscale) & 3u) || (reinterpret_cast<uintptr_t>(ascale) & 3u) ||
      (reinterpret_cast<uintptr_t>(bias) & 1u))
    return FG_ERR_INVALID;
  if ((flags & FG_EPI_RESIDUAL) && (!residual || !fg_aligned16(residual))) return FG_ERR_INVALID;
  if (fg_w4a8_pair_eligible(M, K, w))
    return fg_w4a8_pair_launch(a8, ascale, M, K, w, bias, residual, flags, qscale_cols, qscale, y, workspace,
                               workspace_bytes, static_cast<cudaStream_t>(stream));
  const int N = static_cast<int>(w->N);
  const Plan8 p = make_plan8(M, N, K);
  EncodeTiledFn enc = encode_fn8();
  if (!enc) return FG_ERR_CUDA;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {kBK, static_cast<cuuint32_t>(p.nt)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(a8), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return FG_ERR_INVALID;
  Args8 a;
  a.wc = w->codes;
  a.gmin = w->gmin;
  a.gstep = w->gstep;
  a.cscale = w->cscale;
  a.ascale = ascale;
  a.bias = reinterpret_cast<const __half *>(bias);
  a.res = (flags & FG_EPI_RESIDUAL) ? reinterpret_cast<const __half *>(residual) : nullptr;
  a.y = reinterpret_cast<__half *>(y);
  a.M = M;
  a.N = N;
  a.K = K;
  a.relu = (flags & FG_EPI_RELU) ? 1 : 0;
  a.qcols = qscale_cols;
  a.qscale = qscale;
  a.splits = p.splits;
  a.err = fg_error_word_ptr();
  if (!a.err) return FG_ERR_CUDA;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (p.nt) {
    case 16: return launch8<16>(map, a, p, st);
    case 32: return launch8<32>(map, a, p, st);
    case 64: return launch8<64>(map, a, p, st);
    case 128: return launch8<128>(map, a, p, st);
    default: return launch8<256>(map, a, p, st);
  }
}
