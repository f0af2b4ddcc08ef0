// fg_gemm.cu -- W4A16 linear layer on the 5th-generation tensor cores (tcgen05/TMEM).
//
// y[m][n] = epi( sum_k x[m][k] * deq(W)[n][k] + b[n] ),  W packed 4-bit along k.
//
// "FlexGen Guide: High-Throughput LLM Offloading on One GPU", section 3: weights stay
// in 4-bit form and are dequantised on the fly so the tensor cores compute in FP16.
// Here the dequantisation target is shared memory, in the tensor cores' operand layout:
//
// One-SM kernel (M <= 256 tokens; the CTA-pair kernel for larger M is described further down):
//   CTA tile: 256 output features (two 128-row MMA accumulators) x NT tokens x a k-range.
//   warps 0..7   dequantise: thread t owns weight row n0+t; per 64-wide k-tile it loads
//                32 code bytes + the group's fp16 min/scale (a group covers one k-tile, or
//                two with groups of 128; prefetched 3 tiles ahead),
//                expands them with fp16 FMAs (exactly round(min + code*scale)) and stores
//                128 bytes into the 128-byte-swizzled K-major A tile; then the epilogue.
//   warp 8       TMA: the x tile [NT tokens x 64] (128-byte swizzle) per k-tile.
//   warp 9       one lane issues tcgen05.mma (M=128, N=NT, K=16, fp16 in, fp32 in TMEM),
//                A = dequantised W tile, B = x tile, and commits each stage back.
//   The accumulators D[feature][token] live in TMEM (2*NT columns); the epilogue reads
//   them with tcgen05.ld, adds bias / q-scale / ReLU / residual and stores fp16.
//   When the k-range is split, the splits of one output tile run as one thread-block
//   cluster: each CTA copies its partial accumulator, 32 token columns at a time, into
//   its own shared memory, and the owner of each 32-column chunk adds the partials of
//   all CTAs of the cluster over distributed shared memory in cluster-rank order
//   (deterministic) before the epilogue -- this kernel's partial sums never go through
//   global memory.
// Both kernels may be launched with programmatic dependent launch: they read only weights
// before griddep_wait(), and activations, residual, outputs and scratch after it.
// Every mbarrier wait is bounded (FG_WAIT_TIMEOUT_NS) and reports FG_ERR_TIMEOUT.
#include <stdio.h>

#include <atomic>

#include "fg_internal.cuh"

// the persistent stream-K launch (fg_gemm_streamk.cu)
int fg_streamk_pairs();
size_t fg_streamk_scratch_bytes(int pairs);
fg_status fg_streamk_launch(const CUtensorMap &map, const uint8_t *wc, const __half *wm, const __half *wsc, int gshift,
                            const __half *bias, const __half *res, int relu, int qcols, float qscale, __half *y,
                            int M, int N, int K, int pairs, void *scratch, unsigned int *err, cudaStream_t st,
                            bool pdl);

namespace {

constexpr int kBK = 64;                      // k-tile = one quantisation group
constexpr int kNAcc = 2;                     // accumulators (128 features each) per CTA
constexpr int kBM = 128 * kNAcc;             // features per CTA
constexpr int kDeqWarps = 4 * kNAcc;         // dequant / epilogue warps
constexpr int kTmaWarp = kDeqWarps;
constexpr int kMmaWarp = kDeqWarps + 1;
constexpr int kThreads = (kDeqWarps + 2) * 32;
constexpr int kPrefetch = 3;                 // k-tiles of codes in flight per dequant thread

template <int NT>
struct Cfg {
  static constexpr int STAGES = NT >= 256 ? 3 : 4;
  static constexpr int A_BYTES = 128 * 128;  // one accumulator's A tile: 128 rows x 128 B
  static constexpr int B_BYTES = NT * 128;   // x tile: NT rows x 128 B
  static constexpr int STAGE = kNAcc * A_BYTES + B_BYTES;
  static constexpr int SMEM = STAGES * STAGE + 1024;  // + alignment slack
  static constexpr int COLS = kNAcc * NT < 32 ? 32 : kNAcc * NT;
  static constexpr uint32_t IDESC = umma_idesc_f16_f32(128, NT);
};

struct GemmArgs {
  const uint8_t *wc;   // codes [N][K/2]
  const __half *wm;    // mins  [N][K/64]
  const __half *ws;    // scales[N][K/64]
  const __half *bias;  // [N] or null
  const __half *res;   // [M][N] or null
  __half *y;           // [M][N]
  int M, N, K;
  int relu, qcols;
  float qscale;
  int splits;
  int gshift;          // log2(group / 64): the weights' min/scale cover 1 (group 64) or 2 (128) k-tiles
  float *part;         // pair kernel, k split: fp32 partial sums through global memory, or null
  unsigned long long *flags;  // with part: the split ranks are separate clusters (one wave) that
                              // publish their partials with these [tile][rank][CTA half] flags
  unsigned long long epoch;   // the launch's flag value
  unsigned int *err;
  const float *ascale; // W4A8 pair kernel: per-token activation scales [M]
  const float *cscale; // W4A8 pair kernel: per-row weight scales [N]
  uint64_t wait_ns;    // one-SM kernel: limit of every pipeline wait (FG_WAIT_TIMEOUT_NS unless a test shortens it)
  int stall;           // one-SM kernel, test hook: the dequantising warps withhold their first-stage arrival
};

// ((acc + bias) * qscale if n < qcols) -> ReLU if set -> + residual (0 when unused).
__device__ __forceinline__ float epilogue(float v, float bias, float res, int n, const GemmArgs &a) {
  v += bias;
  if (n < a.qcols) v *= a.qscale;
  if (a.relu) v = fmaxf(v, 0.f);
  return v + res;
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1) w4a16_gemm_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                 const GemmArgs a) {
  using C = Cfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_a[C::STAGES], full_b[C::STAGES], empty[C::STAGES], accum_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  griddep_launch();
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
    // ---------------- dequantise producer: one weight row per thread ----------------
    const int row = tid;  // 0..255
    const int n = n0 + row;
    const bool live = n < a.N;
    const int acc = row >> 7, r = row & 127;
    const uint4 *crow = reinterpret_cast<const uint4 *>(a.wc + static_cast<int64_t>(live ? n : 0) * (a.K / 2));
    const __half *mrow = a.wm + static_cast<int64_t>(live ? n : 0) * ((a.K / kBK) >> a.gshift);
    const __half *srow = a.ws + static_cast<int64_t>(live ? n : 0) * ((a.K / kBK) >> a.gshift);
    uint4 cb[kPrefetch][2];
    __half mb[kPrefetch], sb[kPrefetch];
#pragma unroll
    for (int j = 0; j < kPrefetch; j++) {
      if (j < nk && live) {
        const int kt = kt0 + j;
        cb[j][0] = crow[kt * 2];
        cb[j][1] = crow[kt * 2 + 1];
        mb[j] = mrow[kt >> a.gshift];
        sb[j] = srow[kt >> a.gshift];
      } else {
        cb[j][0] = cb[j][1] = make_uint4(0, 0, 0, 0);
        mb[j] = sb[j] = __ushort_as_half(0);
      }
    }
    // ring of prefetched codes indexed statically (unrolled by the prefetch depth): a slot
    // is consumed in place and refilled kPrefetch k-tiles ahead, so no register holding a
    // load in flight is ever moved (a move would wait for its load)
    bool go = true;
    for (int i0 = 0; go && i0 < nk; i0 += kPrefetch) {
#pragma unroll
      for (int j = 0; j < kPrefetch; j++) {
        const int i = i0 + j;
        if (!go || i >= nk) break;
        const int st = i % C::STAGES;
        const uint4 c0 = cb[j][0], c1 = cb[j][1];
        const __half m0 = mb[j], s0 = sb[j];
        if (i + kPrefetch < nk && live) {
          const int kt = kt0 + i + kPrefetch;
          cb[j][0] = crow[kt * 2];
          cb[j][1] = crow[kt * 2 + 1];
          mb[j] = mrow[kt >> a.gshift];
          sb[j] = srow[kt >> a.gshift];
        }
        if (i >= C::STAGES &&
            !mbar_wait_bounded(smem_u32(&empty[st]), ((i / C::STAGES) - 1) & 1, abortp, a.err, a.wait_ns)) {
          go = false;
          break;
        }
        const __half2 s2 = __half2half2(s0), m2 = __half2half2(m0);
        uint8_t *at = a_tile(st, acc);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int c = 0; c < 8; c++) {
          const uint4 v = live ? dequant8(words[c], s2, m2) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(at + sw128_offset(r, c)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && !(a.stall && i == 0)) mbar_arrive(smem_u32(&full_a[st]));
      }
    }
  } else if (warp == kTmaWarp) {
    // ---------------- TMA producer for the x tiles ----------------
    if (lane == 0) {
      prefetch_tmap(&xmap);
      griddep_wait();  // x comes from the previous kernel
      int issued = 0;
      for (int i = 0; i < nk; i++) {
        const int st = i % C::STAGES;
        if (i >= C::STAGES &&
            !mbar_wait_bounded(smem_u32(&empty[st]), ((i / C::STAGES) - 1) & 1, abortp, a.err, a.wait_ns))
          break;
        const uint32_t bar = smem_u32(&full_b[st]);
        mbar_arrive_expect_tx(bar, C::B_BYTES);
        tma_load_2d(smem_u32(b_tile(st)), &xmap, (kt0 + i) * kBK, t0, bar);
        issued = i + 1;
      }
      if (*abortp) {  // let copies still in flight land before the CTA exits
        for (int j = issued > C::STAGES ? issued - C::STAGES : 0; j < issued; j++)
          mbar_wait_bounded(smem_u32(&full_b[j % C::STAGES]), (j / C::STAGES) & 1, nullptr, nullptr, a.wait_ns);
      }
    }
  } else {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      for (int i = 0; i < nk; i++) {
        const int st = i % C::STAGES;
        const uint32_t par = (i / C::STAGES) & 1;
        if (!mbar_wait_bounded(smem_u32(&full_a[st]), par, abortp, a.err, a.wait_ns)) break;
        if (!mbar_wait_bounded(smem_u32(&full_b[st]), par, abortp, a.err, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t bbase = smem_u32(b_tile(st));
#pragma unroll
        for (int kk = 0; kk < kBK / 16; kk++) {
          const uint64_t bdesc = umma_desc_sw128(bbase + kk * 32);
#pragma unroll
          for (int acc = 0; acc < kNAcc; acc++) {
            const uint64_t adesc = umma_desc_sw128(smem_u32(a_tile(st, acc)) + kk * 32);
            umma_f16(tmem + acc * NT, adesc, bdesc, C::IDESC, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(smem_u32(&empty[st]));
      }
      umma_commit(smem_u32(&accum_bar));  // also tracks completion if the loop stopped early
    }
  }

  // ---------------- epilogue: TMEM -> registers -> global ----------------
  constexpr int kChunks = NT >= 32 ? NT / 32 : 1;  // 32-column chunks of the accumulator
  constexpr int kCW = NT >= 32 ? 32 : NT;          // columns per chunk
  griddep_wait();  // residual and outputs: after the previous kernel has finished
  bool ready = false;
  if (warp < kDeqWarps) {
    ready = mbar_wait_bounded(smem_u32(&accum_bar), 0, nullptr, a.err, a.wait_ns) && !*abortp;
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
      tmem_ld_32x32b_x16(taddr, v);  // NT == 16: this accumulator's 16 columns only
    }
    tmem_wait_ld();
  };
  if (a.splits == 1) {
    if (warp < kDeqWarps) {
      const float bias = (a.bias && nlive) ? __half2float(a.bias[n]) : 0.f;
      for (int ch = 0; ch < kChunks; ch++) {
        uint32_t v[32];
        load_chunk(ch, v);
        if (!ready || !nlive) continue;
        float res[kCW];
#pragma unroll
        for (int j = 0; j < kCW; j++) {  // every residual load is issued before any store
          const int m = t0 + ch * kCW + j;
          res[j] = (a.res && m < a.M) ? __half2float(a.res[static_cast<int64_t>(m) * a.N + n]) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < kCW; j++) {
          const int m = t0 + ch * kCW + j;
          if (m < a.M)
            a.y[static_cast<int64_t>(m) * a.N + n] = __float2half_rn(epilogue(__uint_as_float(v[j]), bias, res[j], n, a));
        }
      }
    }
  } else {
    // Cluster reduction of the k-split partial sums.  Chunks are staged kRound at a time
    // in the (now idle) pipeline buffers as [chunk][column][feature] fp32; chunk ch is
    // reduced by cluster rank ch % splits.  Every thread of every CTA takes the same
    // cluster barriers.
    constexpr int kChunkBytes = kCW * kBM * 4;
    constexpr int kRound = (C::STAGES * C::STAGE) / kChunkBytes < kChunks ? (C::STAGES * C::STAGE) / kChunkBytes
                                                                           : kChunks;
    static_assert(kRound >= 1, "reduction buffer");
    const uint32_t rank = cluster_ctarank();
    float *buf = reinterpret_cast<float *>(smem);
    const int feat = tid;  // reducer thread -> feature row of the tile (epilogue warps only)
    for (int r0 = 0; r0 < kChunks; r0 += kRound) {
      if (warp < kDeqWarps) {
        for (int i = 0; i < kRound && r0 + i < kChunks; i++) {
          uint32_t v[32];
          load_chunk(r0 + i, v);
          float *cb = buf + i * (kCW * kBM);
          const int f = acc * 128 + q * 32 + lane;
#pragma unroll
          for (int j = 0; j < kCW; j++) cb[j * kBM + f] = __uint_as_float(v[j]);
        }
      }
      __syncwarp();
      cluster_sync_all();
      if (warp < kDeqWarps && ready) {
        const int nn = n0 + feat;
        const float rbias = (a.bias && nn < a.N) ? __half2float(a.bias[nn]) : 0.f;
        for (int i = 0; i < kRound && r0 + i < kChunks; i++) {
          const int ch = r0 + i;
          if (ch % a.splits != static_cast<int>(rank)) continue;
          const uint32_t base = smem_u32(buf + i * (kCW * kBM) + feat);
          constexpr int kU = kCW < 8 ? kCW : 8;
          for (int j0 = 0; j0 < kCW; j0 += kU) {
            float sum[kU];
#pragma unroll
            for (int u = 0; u < kU; u++) sum[u] = 0.f;
#pragma unroll
            for (int sp = 0; sp < 8; sp++) {  // cluster-rank order: deterministic
              if (sp < a.splits) {
                const uint32_t rb = mapa_shared(base + j0 * kBM * 4, sp);
#pragma unroll
                for (int u = 0; u < kU; u++) sum[u] += ld_shared_cluster_f32(rb + u * kBM * 4);
              }
            }
            float res[kU];
#pragma unroll
            for (int u = 0; u < kU; u++) {
              const int m = t0 + ch * kCW + j0 + u;
              res[u] = (a.res && m < a.M && nn < a.N) ? __half2float(a.res[static_cast<int64_t>(m) * a.N + nn]) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kU; u++) {
              const int m = t0 + ch * kCW + j0 + u;
              if (m < a.M && nn < a.N)
                a.y[static_cast<int64_t>(m) * a.N + nn] = __float2half_rn(epilogue(sum[u], rbias, res[u], nn, a));
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
// Pair kernel: one tcgen05.mma.cta_group::2 spans two SMs.
//
//   CTA pair (cluster ranks 2p, 2p+1): 256 output features x NTT * 256 tokens (NTT = 2, or
//   1 for smaller tiles) x a k-range.  Each CTA dequantises its own 128 weight rows (the
//   MMA's A = 256 rows is split by rows) and loads its halves of the NTT 256-token x tiles
//   (B is split by columns: tokens tile*256 + half*128 ...).  The even CTA issues NTT M=256,
//   N=256 MMAs per 16-wide k-step, one per token tile, into TMEM columns [tile*256, +256) of
//   BOTH CTAs (each holds its 128 feature rows).  Per SM and k-tile at NTT = 2: 128
//   dequantised rows (half of the single-SM kernel's rows per flop) and ~112 KB of
//   shared-memory traffic for 8 MFLOP.
//   warps 0..7   dequantise (thread: row tid % 128, k half tid / 128), then the epilogue
//                (warp: TMEM lane quarter warp % 4, token tile warp / 4);
//   warp 8       lane 0: TMA of this CTA's x halves, completing on the even CTA's barrier;
//                lane 1: TMA of this CTA's packed weights: the codes of each k-tile (128 rows x
//                32 B, a 24 KB ring running ahead of the dequant warps) and the fp16 group mins
//                and scales, 8 group columns at a time (two buffers) -- one tensor copy each
//                instead of a scattered 16-byte and two 2-byte loads per thread and k-tile.  A
//                code slot is released once its codes have been used, after a proxy fence (the
//                tensor copy that refills it must not overtake the generic-proxy reads);
//   warp 9       even CTA: the MMA issuer; odd CTA: forwards "A half ready" to the even
//                CTA (a 16-byte bulk copy completing on its barrier); TMEM allocation.
//   Split k-ranges of one pair tile form the cluster's z dimension (cluster 2 x 1 x splits);
//   partial sums are reduced in z-rank order through a global scratch (L2) when the caller
//   gives one, else over distributed shared memory.
// ------------------------------------------------------------------------------------

constexpr int kPairA = 128 * 128;              // this CTA's A tile: 128 rows x 128 B
constexpr int kPairBHalf = 128 * 128;          // this CTA's half of one token tile: 128 tokens x 128 B
constexpr int kPairRing = 192 * 1024;          // pipeline ring (both tile sizes)
constexpr int kPairCodeStages = 6;             // k-tiles of codes staged ahead
constexpr int kPairCodeBytes = 128 * 32;       // one k-tile of this CTA's codes: 128 rows x 32 B
constexpr int kPairMetaBytes = 128 * 8 * 2;    // 8 group columns of mins (or scales) x 128 rows
constexpr int kPairCodeOff = kPairRing;
constexpr int kPairMetaOff = kPairCodeOff + kPairCodeStages * kPairCodeBytes;  // 2 buffers x (mins, scales)
constexpr int kPairSmem = kPairMetaOff + 4 * kPairMetaBytes + 1024;            // + alignment slack
static_assert(kPairSmem <= 227 * 1024 - 1024, "shared memory of the pair kernel");
// NTT 256-token MMA tiles per pair tile: 2 (512 tokens, the A tile feeds two MMAs per k
// step) or 1 (256 tokens: half the partial sums when the k-range is split, twice the
// dequantisation per flop)
template <int NTT>
struct PairCfg {
  static constexpr int kTok = 256 * NTT;               // tokens per pair tile
  static constexpr int kStage = kPairA + NTT * kPairBHalf;
  static constexpr int kStages = kPairRing / kStage;   // 4 or 6
  static constexpr int kCols = 256 * NTT;              // TMEM columns (fp32 accumulators)
  static constexpr int kChunks = kCols / 32;           // 32-token epilogue chunks
  static_assert(kStages * kStage == kPairRing, "ring");
};
constexpr uint32_t kPairIdesc = umma_idesc_f16_f32(256, 256);
// Instruction descriptor of the W4A8 form: kind::i8, signed 8-bit A and B, s32 D, K-major.
constexpr uint32_t kPairIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(256 >> 3) << 17) |
                                  (static_cast<uint32_t>(256 >> 4) << 24);
// The two operand widths of the pair kernel.  W4A16: fp16 operands, k-tiles of 64 (one group),
// 32 code bytes per row and k-tile, fp16 mins and scales 8 group columns per tensor copy.  W4A8:
// int8 operands, k-tiles of 128 (two groups, the same 128-byte rows), 64 code bytes per row and
// k-tile, int8 minima and uint8 steps 16 group columns per tensor copy.  Both stage 24 KB of codes
// and 2 KB per metadata buffer.
template <bool I8>
struct PairW {
  static constexpr int kK = I8 ? 128 : 64;
  static constexpr int kCodeRow = I8 ? 64 : 32;
  static constexpr int kCodeBytes = 128 * kCodeRow;
  static constexpr int kCodeStages = (kPairCodeStages * kPairCodeBytes) / kCodeBytes;
  static constexpr int kMetaCols = I8 ? 16 : 8;
  static_assert(kCodeStages * kCodeBytes == kPairCodeStages * kPairCodeBytes, "code ring");
  static_assert(kMetaCols * 128 * (I8 ? 1 : 2) == kPairMetaBytes, "metadata buffer");
};

// D (+)= A * B^T over the pair, int8 operands, int32 accumulation.
__device__ __forceinline__ void umma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 8 codes of one word (element 2j in the low nibble of byte j) -> the 8 int8 weights
// gmin + code * step in element order, as two words.  Each byte is formed in offset binary,
// code * step + (gmin + 128), which lies in [15, 255] (the weight lies in [-113, 127]), so one
// 32-bit multiply-add makes four bytes with no carry between them; flipping each byte's top bit
// turns w + 128 into the two's-complement w.  off4 = (gmin + 128) replicated into the 4 bytes.
__device__ __forceinline__ uint2 widen8_i8(uint32_t w, uint32_t step, uint32_t off4) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t e0 = __byte_perm(lo, hi, 0x5140), e1 = __byte_perm(lo, hi, 0x7362);
  return make_uint2((e0 * step + off4) ^ 0x80808080u, (e1 * step + off4) ^ 0x80808080u);
}
// warps 0..7 dequant + epilogue, 8 TMA, 9 MMA issuer (even CTA) or "A half ready"
// forwarder (odd CTA), and TMEM allocation.  Ten warps leave room for ~168 registers per
// thread (the register file is split over the four schedulers).
constexpr int kPairThreads = (kDeqWarps + 2) * 32;

template <bool I8>
struct PairAcc {
  using T = float;
};
template <>
struct PairAcc<true> {
  using T = int;
};

// The pair kernel's body for both operand widths (I8: the W4A8 form, whose cmap, mmap and smap
// cover the codes, the int8 group minima and the uint8 group steps).
template <int NTT, bool I8>
__device__ __forceinline__ void gemm_pair_body(const CUtensorMap &xmap, const CUtensorMap &cmap,
                                               const CUtensorMap &mmap, const CUtensorMap &smap, const GemmArgs &a) {
  using C = PairCfg<NTT>;
  using W = PairW<I8>;
  constexpr int kPairStages = C::kStages, kPairStage = C::kStage, kPairTok = C::kTok, kPairCols = C::kCols;
  constexpr int kCS = W::kCodeStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // full (even CTA): the stage is ready -- its 8 dequant warps arrive, its TMA thread
  // arrives expecting the x bytes of both CTAs plus the 16 bytes of the odd CTA's "A half
  // done" token (one wait per stage for the MMA thread, whose issue rate bounds the
  // kernel); a_half (odd CTA): its 8 dequant warps are done; empty: the pair's MMAs are
  // done with the stage.  The odd CTA signals with a 16-byte bulk copy into the even CTA
  // rather than a remote arrive: a remote mbarrier arrive took over a microsecond to land,
  // the bulk copy's completion a few hundred nanoseconds.
  __shared__ __align__(8) uint64_t full[kPairStages], a_half[kPairStages], empty[kPairStages], accum_bar;
  __shared__ __align__(16) uint32_t token_src[4], token_sink[kPairStages][4];
  __shared__ __align__(8) uint64_t recv_bar;  // split-k epilogue: this rank's received partials
  // staged weights: code_full (TMA) / code_empty (the 8 dequant warps have read the slot);
  // meta_full / meta_empty likewise for the two metadata buffers
  __shared__ __align__(8) uint64_t code_full[kPairCodeStages], code_empty[kPairCodeStages], meta_full[2], meta_empty[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  griddep_launch();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t lead = crank & ~1u;
  const bool leader = crank == lead;
  const int half = static_cast<int>(crank & 1u);
  const int n0 = blockIdx.x * 128;  // this CTA's 128 weight rows
  const int t0 = blockIdx.y * kPairTok, split = blockIdx.z;
  const int ktiles = a.K / W::kK;
  const int kt0 = static_cast<int>((static_cast<int64_t>(split) * ktiles) / a.splits);
  const int kt1 = static_cast<int>((static_cast<int64_t>(split + 1) * ktiles) / a.splits);
  const int nk = kt1 - kt0;
  volatile int *abortp = &abort_flag;
  const uint16_t pair_mask = static_cast<uint16_t>(3u << lead);

  auto a_tile = [&](int st) { return smem + st * kPairStage; };
  auto b_tile = [&](int st, int tile) { return smem + st * kPairStage + kPairA + tile * kPairBHalf; };

  if (tid == 0) {
    for (int i = 0; i < kPairStages; i++) {
      mbar_init(smem_u32(&full[i]), kDeqWarps + 1);  // 8 local warps + TMA (odd CTA: tx bytes)
      mbar_init(smem_u32(&a_half[i]), kDeqWarps);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    mbar_init(smem_u32(&accum_bar), 1);
    mbar_init(smem_u32(&recv_bar), 1);
    for (int i = 0; i < kCS; i++) {
      mbar_init(smem_u32(&code_full[i]), 1);
      mbar_init(smem_u32(&code_empty[i]), kDeqWarps);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(smem_u32(&meta_full[i]), 1);
      mbar_init(smem_u32(&meta_empty[i]), kDeqWarps);
    }
    abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_u32(&tmem_slot), kPairCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // metadata column group (8 group columns) of k-tile kt, relative to the first one of the range
  const int sj0 = (kt0 >> a.gshift) >> 3;
  auto meta_unit = [&](int kt) { return ((kt >> a.gshift) >> 3) - sj0; };
  if (warp < kDeqWarps) {
    // ---------------- dequantise producer: row tid % 128, k half tid / 128 ----------------
    const int row = tid & 127, hk = tid >> 7;
    const bool live = n0 + row < a.N;
    int cur_u = -1;
    // leader: arrive on its own full barrier; odd CTA: on a_half, forwarded by warp 9
    const uint32_t done_bar0 = smem_u32(leader ? &full[0] : &a_half[0]);
    for (int i = 0; i < nk; i++) {
      const int st = i % kPairStages, cs = i % kCS;
      if (!mbar_wait_bounded(smem_u32(&code_full[cs]), (i / kCS) & 1, abortp, a.err)) break;
      const uint8_t *cp = smem + kPairCodeOff + cs * W::kCodeBytes + row * W::kCodeRow + hk * (W::kCodeRow / 2);
      const uint4 c0 = *reinterpret_cast<const uint4 *>(cp);
      const uint4 c1 = I8 ? *reinterpret_cast<const uint4 *>(cp + 16) : make_uint4(0, 0, 0, 0);
      const int mi = (kt0 + i) >> a.gshift, u = meta_unit(kt0 + i);
      if (u != cur_u) {  // warp-uniform
        if (cur_u >= 0 && lane == 0) mbar_arrive(smem_u32(&meta_empty[cur_u & 1]));  // read by every lane above
        if (!mbar_wait_bounded(smem_u32(&meta_full[u & 1]), (u >> 1) & 1, abortp, a.err)) break;
        cur_u = u;
      }
      const uint8_t *mbase = smem + kPairMetaOff + (u & 1) * 2 * kPairMetaBytes;
      if (i >= kPairStages &&
          !mbar_wait_bounded(smem_u32(&empty[st]), ((i / kPairStages) - 1) & 1, abortp, a.err))
        break;
      uint8_t *at = a_tile(st);
      if constexpr (I8) {
        // this thread's 64 k values are group 2 kt + hk: column (2 kt + hk) mod 16 of the unit
        const int col = 2 * ((kt0 + i) & 7) + hk;
        const uint32_t off4 = ((static_cast<uint32_t>(mbase[row * 16 + col]) ^ 0x80u)) * 0x01010101u;  // gmin + 128
        const uint32_t step = mbase[kPairMetaBytes + row * 16 + col];
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int c = 0; c < 4; c++) {  // chunk 4 hk + c: k values 16c..16c+15 of the thread's 64
          const uint2 p = widen8_i8(words[2 * c], step, off4), r = widen8_i8(words[2 * c + 1], step, off4);
          const uint4 v = live ? make_uint4(p.x, p.y, r.x, r.y) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(at + sw128_offset(row, 4 * hk + c)) = v;
        }
      } else {
        const __half *mb = reinterpret_cast<const __half *>(mbase);
        const __half m0 = mb[row * 8 + (mi & 7)], s0 = mb[kPairMetaBytes / 2 + row * 8 + (mi & 7)];
        const __half2 s2 = __half2half2(s0), m2 = __half2half2(m0);
        const uint32_t words[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
        for (int c = 0; c < 4; c++) {
          const uint4 v = live ? dequant8(words[c], s2, m2) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(at + sw128_offset(row, 4 * hk + c)) = v;
        }
      }
      // The code slot is released only now: the codes have been used (so read), and the proxy
      // fence orders these generic-proxy reads before the tensor copy that refills the slot.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(done_bar0 + st * 8);
        mbar_arrive(smem_u32(&code_empty[cs]));
      }
    }
  } else if (warp == kTmaWarp) {
    // ---------------- TMA producers ----------------
    // lane 0: this CTA's halves of the token tiles of x, stage by stage;  lane 1: this CTA's
    // packed weights -- the codes of each k-tile into the code ring, the group metadata a column
    // group at a time into its two buffers -- as far ahead as the dequant warps release slots.
    // On separate lanes a code slot the dequant warps still hold never delays an x copy.
    if (lane == 0) {
      prefetch_tmap(&xmap);
      griddep_wait();  // x comes from the previous kernel
      for (int i = 0; i < nk; i++) {
        const int st = i % kPairStages;
        if (i >= kPairStages &&
            !mbar_wait_bounded(smem_u32(&empty[st]), ((i / kPairStages) - 1) & 1, abortp, a.err))
          break;
        const uint32_t fb = mapa_shared(smem_u32(&full[st]), lead);
        if (leader) mbar_arrive_expect_tx(smem_u32(&full[st]), 2 * NTT * kPairBHalf + 16);  // x of both CTAs + token
#pragma unroll
        for (int tile = 0; tile < NTT; tile++)
          tma_load_2d_pair(smem_u32(b_tile(st, tile)), &xmap, (kt0 + i) * W::kK, t0 + tile * 256 + half * 128, fb);
      }
    } else if (lane == 1) {
      // the weights are fixed for the call: no dependency wait
      prefetch_tmap(&cmap);
      prefetch_tmap(&mmap);
      prefetch_tmap(&smap);
      int um = 0;
      for (int jc = 0; jc < nk; jc++) {
        if (meta_unit(kt0 + jc) == um) {  // the first k-tile of a metadata column group
          if (um >= 2 && !mbar_wait_bounded(smem_u32(&meta_empty[um & 1]), ((um >> 1) - 1) & 1, abortp, a.err))
            break;
          const uint32_t mbar = smem_u32(&meta_full[um & 1]);
          uint8_t *mb = smem + kPairMetaOff + (um & 1) * 2 * kPairMetaBytes;
          mbar_arrive_expect_tx(mbar, 2 * kPairMetaBytes);
          tma_load_2d(smem_u32(mb), &mmap, (sj0 + um) * W::kMetaCols, n0, mbar);
          tma_load_2d(smem_u32(mb + kPairMetaBytes), &smap, (sj0 + um) * W::kMetaCols, n0, mbar);
          um++;
        }
        const int cs = jc % kCS;
        if (jc >= kCS && !mbar_wait_bounded(smem_u32(&code_empty[cs]), ((jc / kCS) - 1) & 1, abortp, a.err))
          break;
        const uint32_t cbar = smem_u32(&code_full[cs]);
        mbar_arrive_expect_tx(cbar, W::kCodeBytes);
        tma_load_2d(smem_u32(smem + kPairCodeOff + cs * W::kCodeBytes), &cmap, (kt0 + jc) * W::kCodeRow, n0, cbar);
      }
    }
  } else if (!leader) {
    // ---------------- odd CTA: forward "A half ready" to the even CTA ----------------
    // Warp 9 forwards every stage; the bulk copy does not hold the thread.  Ordering: the
    // dequant warps' proxy fence and release (a_half), this thread's acquire, then the bulk
    // copy whose completion the even CTA acquires at cluster scope before its MMAs read
    // this CTA's A half.
    if (warp == kMmaWarp && lane == 0) {
      for (int i = 0; i < nk; i++) {
        const int st = i % kPairStages;
        if (!mbar_wait_bounded(smem_u32(&a_half[st]), (i / kPairStages) & 1, abortp, a.err)) break;
        bulk_s2s_cluster(mapa_shared(smem_u32(&token_sink[st][0]), lead), smem_u32(&token_src[0]), 16,
                         mapa_shared(smem_u32(&full[st]), lead));
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer (even CTA) ----------------
    // Kept lean: one wait, 8 MMAs and one commit per stage, descriptors precomputed (the
    // 14-bit start-address field advances by 2 per 32-byte k step without carrying).
    if (lane == 0) {
      const uint64_t adesc0 = umma_desc_sw128(smem_u32(a_tile(0)));
      const uint64_t bdesc0 = umma_desc_sw128(smem_u32(b_tile(0, 0)));
      constexpr uint64_t kStageStep = kPairStage >> 4, kTileStep = kPairBHalf >> 4;
      for (int i = 0; i < nk; i++) {
        const int st = i % kPairStages;
        if (!mbar_poll_bounded<true>(smem_u32(&full[st]), (i / kPairStages) & 1, abortp, a.err)) break;
        tc_fence_after();
        const uint64_t ad = adesc0 + st * kStageStep, bd = bdesc0 + st * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 4; kk++) {  // 32-byte k steps: 16 fp16 or 32 int8 values
#pragma unroll
          for (int tile = 0; tile < NTT; tile++) {
            if constexpr (I8)
              umma_i8_pair(tmem + tile * 256, ad + 2 * kk, bd + tile * kTileStep + 2 * kk, kPairIdescI8,
                           (i > 0 || kk > 0) ? 1u : 0u);
            else
              umma_f16_pair(tmem + tile * 256, ad + 2 * kk, bd + tile * kTileStep + 2 * kk, kPairIdesc,
                            (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit_pair(smem_u32(&empty[st]), pair_mask);
      }
      umma_commit_pair(smem_u32(&accum_bar), pair_mask);  // also tracks completion if the loop stopped early
    }
  }

  // ---------------- epilogue: TMEM -> shared memory -> global ----------------
  // The 128 x 512 fp32 accumulator is transposed through the idle ring buffers so that every
  // thread writes 8 consecutive features (16-byte stores covering whole 256-byte row
  // segments of y).  Without a residual or a k split, bias, q-scale and ReLU are applied
  // straight out of TMEM (a thread holds one feature) and only fp16 is staged; otherwise
  // fp32 chunks of [32 tokens][128 features] are staged kRound at a time and chunk ch is
  // finished by z rank ch % splits, which sums it over the cluster's z ranks in rank order
  // (deterministic) before the epilogue.  All threads of all CTAs take the same barriers.
  griddep_wait();  // residual, outputs and scratch: after the previous kernel has finished
  bool ready = false;
  if (warp < kDeqWarps) {
    ready = mbar_wait_bounded_cluster(smem_u32(&accum_bar), 0, nullptr, a.err) && !*abortp;
    tc_fence_after();
  }
  // Accumulator values travel as 32-bit words: fp32 (W4A16) or s32 sums (W4A8), which k-split
  // partials add exactly; a W4A8 value becomes the fp32 product acc * (ascale[m] * cscale[n]),
  // one IEEE operation each, only once it is final.
  using Acc = typename PairAcc<I8>::T;
  auto acc_of = [](float word) -> Acc {
    if constexpr (I8) return __float_as_int(word); else return word;
  };
  auto fin = [&](Acc v, int m, float csc) -> float {
    if constexpr (I8) return __fmul_rn(__int2float_rn(v), __fmul_rn(a.ascale[m], csc)); else return v;
  };
  const int q = warp & 3, etile = (warp >> 2) & 1;
  // finishing thread: 8 features f8 .. f8+7, tokens mj0 + 16 it of a 32-token chunk
  const int f8 = (tid & 15) * 8, mj0 = (tid >> 4) & 15;
  const int nb = n0 + f8;
  if (a.splits == 1 && !a.res) {
    __half *hbuf = reinterpret_cast<__half *>(smem);  // [chunks][32 tokens][128 features]
    if (warp < kDeqWarps) {
      const int n = n0 + q * 32 + lane;
      const float bias = (a.bias && n < a.N) ? __half2float(a.bias[n]) : 0.f;
      const float qs = n < a.qcols ? a.qscale : 1.f;
      const float csc = (I8 && n < a.N) ? a.cscale[n] : 0.f;
      for (int c8 = 0; c8 < C::kChunks / 2; c8++) {
        const int ch = etile * (C::kChunks / 2) + c8;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + ch * 32, v);
        // W4A8: lane j loads the scale of token j of the chunk; the warp shares them (every lane
        // of these warps runs this loop)
        const int ml = t0 + ch * 32 + lane;
        const float as_l = I8 ? a.ascale[ml < a.M ? ml : a.M - 1] : 0.f;
        tmem_wait_ld();
        __half *cb = hbuf + ch * (32 * 128) + q * 32 + lane;
#pragma unroll
        for (int j = 0; j < 32; j++) {
          float y;
          if constexpr (I8)
            y = (__fmul_rn(__int2float_rn(static_cast<int>(v[j])), __fmul_rn(__shfl_sync(0xffffffffu, as_l, j), csc)) +
                 bias) * qs;
          else
            y = (__uint_as_float(v[j]) + bias) * qs;
          if (a.relu) y = fmaxf(y, 0.f);
          cb[j * 128] = __float2half_rn(y);
        }
      }
    }
    __syncthreads();
    if (warp < kDeqWarps && ready && nb < a.N) {
#pragma unroll 4
      for (int ch = 0; ch < kPairCols / 32; ch++) {
#pragma unroll
        for (int it = 0; it < 2; it++) {
          const int mj = mj0 + 16 * it, m = t0 + ch * 32 + mj;
          const uint4 ov = *reinterpret_cast<const uint4 *>(hbuf + ch * (32 * 128) + mj * 128 + f8);
          if (m < a.M) *reinterpret_cast<uint4 *>(a.y + static_cast<int64_t>(m) * a.N + nb) = ov;
        }
      }
    }
    __syncthreads();
  } else if (a.splits == 1) {
    // residual, no k split: fp32 chunks staged kRound at a time, finished by this CTA
    constexpr int kChunkFloats = 32 * 128;
    constexpr int kRound = kPairRing / (kChunkFloats * 4);  // 12 chunks of the 16
    constexpr int kChunks = kPairCols / 32;
    float *buf = reinterpret_cast<float *>(smem);
    float bias[8], csc8[8];
#pragma unroll
    for (int u = 0; u < 8; u++) {
      bias[u] = (a.bias && warp < kDeqWarps && nb < a.N) ? __half2float(a.bias[nb + u]) : 0.f;
      csc8[u] = (I8 && warp < kDeqWarps && nb < a.N) ? a.cscale[nb + u] : 0.f;
    }
    for (int r0 = 0; r0 < kChunks; r0 += kRound) {
      if (warp < kDeqWarps) {
        // warps q and q + 4 share TMEM lanes 32q..32q+31 and take alternate chunks
        for (int ch = r0 + etile; ch < r0 + kRound && ch < kChunks; ch += 2) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + ch * 32, v);
          tmem_wait_ld();
          float *cbuf = buf + (ch - r0) * kChunkFloats;
#pragma unroll
          for (int j = 0; j < 32; j++) cbuf[j * 128 + q * 32 + lane] = __uint_as_float(v[j]);
        }
      }
      __syncthreads();
      if (warp < kDeqWarps && ready && nb < a.N) {
        for (int ch = r0; ch < r0 + kRound && ch < kChunks; ch++) {
          const float *own = buf + (ch - r0) * kChunkFloats + mj0 * 128 + f8;
          uint4 rv[2];
#pragma unroll
          for (int it = 0; it < 2; it++) {
            const int m = t0 + ch * 32 + mj0 + 16 * it;
            rv[it] = (a.res && m < a.M) ? *reinterpret_cast<const uint4 *>(a.res + static_cast<int64_t>(m) * a.N + nb)
                                        : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int it = 0; it < 2; it++) {
            const int m = t0 + ch * 32 + mj0 + 16 * it;
            if (m >= a.M) continue;
            const float4 p0 = *reinterpret_cast<const float4 *>(own + it * 16 * 128);
            const float4 p1 = *reinterpret_cast<const float4 *>(own + it * 16 * 128 + 4);
            const float acc[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            const __half *rh = reinterpret_cast<const __half *>(&rv[it]);
            uint4 ov;
            __half *oh = reinterpret_cast<__half *>(&ov);
#pragma unroll
            for (int u = 0; u < 8; u++)
              oh[u] = __float2half_rn(epilogue(fin(acc_of(acc[u]), m, csc8[u]), bias[u], __half2float(rh[u]), nb + u, a));
            *reinterpret_cast<uint4 *>(a.y + static_cast<int64_t>(m) * a.N + nb) = ov;
          }
        }
      }
      __syncthreads();
    }
  } else if (a.part) {
    // k split, partial sums through global memory (they stay in L2): every z rank stores its
    // fp32 partial [512 tokens][its 128 features] straight from TMEM -- a warp writes 128
    // contiguous bytes per token -- the cluster synchronises (release / acquire at cluster
    // scope orders these stores for the other ranks' loads), and the owner of each 32-token
    // chunk (chunk % splits) adds the splits' partials in z-rank order, as the on-chip
    // reduction below does, and finishes the chunk.  One barrier instead of a chain of
    // rounds of distributed-shared-memory copies.
    constexpr int kChunks = kPairCols / 32;
    const int S = a.splits, zrank = static_cast<int>(blockIdx.z);
    constexpr int64_t kTileFloats = static_cast<int64_t>(kPairTok) * 256;
    const int64_t tile = static_cast<int64_t>(blockIdx.y) * (gridDim.x / 2) + blockIdx.x / 2;
    const float *tilep = a.part + tile * S * kTileFloats;
    if (warp < kDeqWarps && ready) {
      float *mine = const_cast<float *>(tilep) + zrank * kTileFloats + half * 128 + q * 32 + lane;
      for (int c8 = 0; c8 < kChunks / 2; c8++) {
        const int ch = etile * (kChunks / 2) + c8;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + ch * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j++) mine[static_cast<int64_t>(ch * 32 + j) * 256] = __uint_as_float(v[j]);
      }
    }
    __threadfence();
    if (a.flags) {
      // The split ranks are separate clusters, all resident (the launch takes this form only
      // when the grid is one wave): publish this CTA's partial, then wait for the other ranks'
      // partials of the same tile half (bounded; a timeout flags FG_ERR_TIMEOUT and skips the sum).
      __syncthreads();
      unsigned long long *fl = a.flags + tile * S * 2 + half;  // [tile][rank][half]
      if (tid == 0) {
        st_release_u64(fl + 2 * zrank, a.epoch);
        for (int z = 0; z < S && !*abortp; z++) {
          if (z == zrank) continue;
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_u64(fl + 2 * z) != a.epoch) {
            if (globaltimer_ns() - t0 > FG_WAIT_TIMEOUT_NS) {
              atomicOr(a.err, FG_DEVERR_TIMEOUT);
              *abortp = 1;
              break;
            }
            __nanosleep(64);
          }
        }
      }
      __syncthreads();
      ready = ready && !*abortp;
    } else {
      cluster_sync_all();
    }
    if (warp < kDeqWarps && ready && nb < a.N) {
      float bias[8], csc8[8];
#pragma unroll
      for (int u = 0; u < 8; u++) {
        bias[u] = a.bias ? __half2float(a.bias[nb + u]) : 0.f;
        csc8[u] = I8 ? a.cscale[nb + u] : 0.f;
      }
      const float *col = tilep + half * 128 + f8;
      for (int ch = zrank; ch < kChunks; ch += S) {
        uint4 rv[2];
        Acc acc[2][8];
#pragma unroll
        for (int it = 0; it < 2; it++) {
          const int m = t0 + ch * 32 + mj0 + 16 * it;
          rv[it] = (a.res && m < a.M) ? *reinterpret_cast<const uint4 *>(a.res + static_cast<int64_t>(m) * a.N + nb)
                                      : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int u = 0; u < 8; u++) acc[it][u] = 0;
        }
#pragma unroll
        for (int z = 0; z < 4; z++) {  // z-rank order
          if (z >= S) break;
#pragma unroll
          for (int it = 0; it < 2; it++) {
            const float *src = col + z * kTileFloats + static_cast<int64_t>(ch * 32 + mj0 + 16 * it) * 256;
            const float4 p0 = __ldcg(reinterpret_cast<const float4 *>(src));
            const float4 p1 = __ldcg(reinterpret_cast<const float4 *>(src + 4));
            acc[it][0] += acc_of(p0.x); acc[it][1] += acc_of(p0.y); acc[it][2] += acc_of(p0.z);
            acc[it][3] += acc_of(p0.w); acc[it][4] += acc_of(p1.x); acc[it][5] += acc_of(p1.y);
            acc[it][6] += acc_of(p1.z); acc[it][7] += acc_of(p1.w);
          }
        }
#pragma unroll
        for (int it = 0; it < 2; it++) {
          const int m = t0 + ch * 32 + mj0 + 16 * it;
          if (m >= a.M) continue;
          const __half *rh = reinterpret_cast<const __half *>(&rv[it]);
          uint4 ov;
          __half *oh = reinterpret_cast<__half *>(&ov);
#pragma unroll
          for (int u = 0; u < 8; u++)
            oh[u] = __float2half_rn(epilogue(fin(acc[it][u], m, csc8[u]), bias[u], __half2float(rh[u]), nb + u, a));
          *reinterpret_cast<uint4 *>(a.y + static_cast<int64_t>(m) * a.N + nb) = ov;
        }
      }
    }
  } else {
    // k split over the cluster's z ranks.  Per round of kR chunks every rank stages its fp32
    // partial of each chunk, then pushes the chunks it does not own into the owner's receive
    // slots with bulk copies (completion counted on the owner's recv_bar); the owner sums
    // its own partial and the received ones in z-rank order (deterministic) and finishes.
    constexpr int kChunkFloats = 32 * 128;
    constexpr int kChunkBytes = kChunkFloats * 4;
    constexpr int kR = 6;                                        // chunks per round
    constexpr int kSlots = kPairRing / kChunkBytes - kR;         // receive slots: 6
    constexpr int kChunks = kPairCols / 32;
    constexpr int kOwnMax = 3;                                   // chunks of a round one rank owns (splits >= 2)
    static_assert(kSlots >= 6, "a rank owns at most 2 chunks x 3 senders or 3 chunks x 1 sender per round");
    const int S = a.splits, zrank = static_cast<int>(crank >> 1);
    float *sendb = reinterpret_cast<float *>(smem);              // [kR] chunks
    float *recvb = sendb + kR * kChunkFloats;                    // [kSlots] chunks
    float bias[8], csc8[8];
#pragma unroll
    for (int u = 0; u < 8; u++) {
      bias[u] = (a.bias && warp < kDeqWarps && nb < a.N) ? __half2float(a.bias[nb + u]) : 0.f;
      csc8[u] = (I8 && warp < kDeqWarps && nb < a.N) ? a.cscale[nb + u] : 0.f;
    }
    auto first_owned = [&](int owner, int r0) { return r0 + ((owner - r0 % S) + S) % S; };
    int round = 0;
    for (int r0 = 0; r0 < kChunks; r0 += kR, round++) {
      const int rend = min(r0 + kR, kChunks);
      const int f0 = first_owned(zrank, r0);
      const int nown = f0 < rend ? (rend - 1 - f0) / S + 1 : 0;
      if (warp < kDeqWarps) {
        for (int ch = r0 + etile; ch < rend; ch += 2) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + ch * 32, v);
          tmem_wait_ld();
          float *cbuf = sendb + (ch - r0) * kChunkFloats;
#pragma unroll
          for (int j = 0; j < 32; j++) cbuf[j * 128 + q * 32 + lane] = __uint_as_float(v[j]);
        }
        fence_proxy_async_smem();  // the staged partials are read by bulk copies
      }
      if (tid == 0) mbar_arrive_expect_tx(smem_u32(&recv_bar), static_cast<uint32_t>(nown * (S - 1) * kChunkBytes));
      __syncwarp();
      cluster_sync_all();  // staged everywhere; every receiver's slots free and its barrier armed
      if (tid == 0) {
        for (int ch = r0; ch < rend; ch++) {
          const int owner = ch % S;
          if (owner == zrank) continue;
          const int j = (ch - first_owned(owner, r0)) / S;
          const int slot = j * (S - 1) + (zrank < owner ? zrank : zrank - 1);
          const uint32_t dst = (crank & 1u) + 2u * static_cast<uint32_t>(owner);
          bulk_s2s_cluster(mapa_shared(smem_u32(recvb + slot * kChunkFloats), dst),
                           smem_u32(sendb + (ch - r0) * kChunkFloats), kChunkBytes, mapa_shared(smem_u32(&recv_bar), dst));
        }
      }
      if (warp < kDeqWarps) {
        const bool got = mbar_wait_bounded(smem_u32(&recv_bar), round & 1, nullptr, a.err);
        if (got && ready && nb < a.N) {
          uint4 resv[kOwnMax][2];
#pragma unroll
          for (int j = 0; j < kOwnMax; j++) {
            const int ch = f0 + j * S;
#pragma unroll
            for (int it = 0; it < 2; it++) {
              const int m = t0 + ch * 32 + mj0 + 16 * it;
              resv[j][it] = (a.res && j < nown && m < a.M)
                                ? *reinterpret_cast<const uint4 *>(a.res + static_cast<int64_t>(m) * a.N + nb)
                                : make_uint4(0, 0, 0, 0);
            }
          }
#pragma unroll
          for (int j = 0; j < kOwnMax; j++) {
            if (j >= nown) continue;
            const int ch = f0 + j * S;
#pragma unroll
            for (int it = 0; it < 2; it++) {
              const int m = t0 + ch * 32 + mj0 + 16 * it;
              if (m >= a.M) continue;
              const int eoff = (mj0 + 16 * it) * 128 + f8;
              Acc acc[8];
#pragma unroll
              for (int u = 0; u < 8; u++) acc[u] = 0;
              for (int z = 0; z < S; z++) {  // z-rank order
                const float *src = z == zrank ? sendb + (ch - r0) * kChunkFloats + eoff
                                              : recvb + (j * (S - 1) + (z < zrank ? z : z - 1)) * kChunkFloats + eoff;
                const float4 p0 = *reinterpret_cast<const float4 *>(src);
                const float4 p1 = *reinterpret_cast<const float4 *>(src + 4);
                acc[0] += acc_of(p0.x); acc[1] += acc_of(p0.y); acc[2] += acc_of(p0.z); acc[3] += acc_of(p0.w);
                acc[4] += acc_of(p1.x); acc[5] += acc_of(p1.y); acc[6] += acc_of(p1.z); acc[7] += acc_of(p1.w);
              }
              const __half *rh = reinterpret_cast<const __half *>(&resv[j][it]);
              uint4 ov;
              __half *oh = reinterpret_cast<__half *>(&ov);
#pragma unroll
              for (int u = 0; u < 8; u++)
                oh[u] = __float2half_rn(epilogue(fin(acc[u], m, csc8[u]), bias[u], __half2float(rh[u]), nb + u, a));
              *reinterpret_cast<uint4 *>(a.y + static_cast<int64_t>(m) * a.N + nb) = ov;
            }
          }
        }
      }
      __syncwarp();
      cluster_sync_all();  // every push has landed: send buffers and slots can be reused
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's TMEM and shared memory are no longer in use
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kPairCols);
  }
}

template <int NTT>
__global__ void __launch_bounds__(kPairThreads, 1) w4a16_gemm_pair_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                      const __grid_constant__ CUtensorMap cmap,
                                                                      const __grid_constant__ CUtensorMap mmap,
                                                                      const __grid_constant__ CUtensorMap smap,
                                                                      const GemmArgs a) {
  gemm_pair_body<NTT, false>(xmap, cmap, mmap, smap, a);
}

// W4A8: xmap covers the int8 activations, cmap the codes, mmap the int8 group minima, smap the
// uint8 group steps; a.ascale and a.cscale the per-token and per-row fp32 scales.
template <int NTT>
__global__ void __launch_bounds__(kPairThreads, 1) w4a8_gemm_pair_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                     const __grid_constant__ CUtensorMap cmap,
                                                                     const __grid_constant__ CUtensorMap mmap,
                                                                     const __grid_constant__ CUtensorMap smap,
                                                                     const GemmArgs a) {
  gemm_pair_body<NTT, true>(xmap, cmap, mmap, smap, a);
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

int sm_count() {
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

int pick_nt(int M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128) return 128;
  return 256;
}

struct Plan {
  int nt, n_tiles, t_tiles, splits;
  double cost;  // pair kernel: modelled microseconds
  int pairs;    // > 0: the persistent stream-K launch over this many CTA pairs is faster
};

// Split the k-range over the CTAs of a cluster only to fill the SMs: minimise
// waves * k-tiles per CTA, with a small charge per extra split for the cluster reduction.
Plan make_plan(int M, int N, int K) {
  Plan p;
  p.pairs = 0;
  p.cost = 0.0;
  p.nt = pick_nt(M);
  p.n_tiles = (N + kBM - 1) / kBM;
  p.t_tiles = (M + p.nt - 1) / p.nt;
  const int ktiles = K / kBK;
  const int base = p.n_tiles * p.t_tiles;
  const int nsm = sm_count();
  double best = 1e30;
  p.splits = 1;
  for (int s = 1; s <= 8; s++) {
    if (s > 1 && ktiles / s < 8) break;
    const int waves = (base * s + nsm - 1) / nsm;
    const double cost = static_cast<double>(waves) * ((ktiles + s - 1) / s) * (1.0 + 0.05 * (s - 1));
    if (cost < best - 1e-9) {
      best = cost;
      p.splits = s;
    }
  }
  return p;
}

// pdl: launch with programmatic stream serialisation -- the kernel's prologue (barriers,
// TMEM, weight loads and their dequantisation) may overlap the previous kernel, which the
// kernel waits for before it touches activations, residual or outputs.  Only for callers
// whose weights the previous kernel cannot be writing.
template <int NT>
fg_status launch_nt(const CUtensorMap &map, const GemmArgs &a, const Plan &p, cudaStream_t st, bool pdl) {
  using C = Cfg<NT>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    fg_status rc = fg_cuda_check(
        cudaFuncSetAttribute(w4a16_gemm_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    if (rc != FG_OK) return rc;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(p.n_tiles, p.t_tiles, p.splits);
  lc.blockDim = dim3(kThreads, 1, 1);
  lc.dynamicSmemBytes = C::SMEM;
  lc.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = p.splits;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = pdl ? 2 : 1;
  fg_status rc = fg_cuda_check(cudaLaunchKernelEx(&lc, w4a16_gemm_kernel<NT>, map, a));
  if (rc != FG_OK) return rc;
  return fg_launch_check();
}


// ---- pair kernel planning ----

template <int NTT, bool I8 = false>
fg_status pair_attr_once() {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    fg_status rc = fg_cuda_check(cudaFuncSetAttribute(I8 ? w4a8_gemm_pair_kernel<NTT> : w4a16_gemm_pair_kernel<NTT>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem));
    if (rc != FG_OK) return rc;
    attr_set[dev] = true;
  }
  return FG_OK;
}

// Pair-kernel clusters (2 x 1 x splits CTAs) that can be resident at once; 0 when such a
// cluster does not fit on the device.
template <int NTT>
int pair_clusters_resident(int splits) {
  static int cache[64][5];
  static bool known[64][5] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || splits < 1 || splits > 4) return 0;
  // the occupancy query needs the kernel's shared-memory attribute; a failed query is not cached
  if (pair_attr_once<NTT>() != FG_OK) return 0;
  if (!known[dev][splits]) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(2, 1, splits);
    lc.blockDim = dim3(kPairThreads, 1, 1);
    lc.dynamicSmemBytes = kPairSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = splits;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, w4a16_gemm_pair_kernel<NTT>, &lc) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cache[dev][splits] = n > 0 ? n : 0;
    known[dev][splits] = true;
  }
  return cache[dev][splits];
}

// Tile size (256 or 512 tokens) and k splits (the cluster's z dimension, at most 4) by a
// time model in microseconds, measured on B200 for this kernel: a k-tile takes about
// 0.70 us at 512 tokens and 0.63 us at 256 (half the MMA work, the same dequantisation
// and pipeline hand-offs); each wave pays its pipeline fill (~5 us) and the epilogue, whose
// partial sums grow with the tile and the number of splits.
Plan make_pair_plan(int M, int N, int K, int kb = kBK) {
  Plan p;
  p.n_tiles = (N + 255) / 256;  // CTA pairs along the features
  p.nt = 512;
  p.splits = 1;
  const int ktiles = K / kb;  // k-tiles of 64 (fp16 operands) or 128 (int8: the same bytes per k-tile)
  double best = 1e30;
  for (int ntt = 2; ntt >= 1; ntt--) {
    const int tok = 256 * ntt;
    const int t_tiles = (M + tok - 1) / tok;
    const int clusters = p.n_tiles * t_tiles;
    const double ktime = ntt == 2 ? 0.70 : 0.63;
    const int one = ntt == 2 ? pair_clusters_resident<2>(1) : pair_clusters_resident<1>(1);
    for (int s = 1; s <= 4; s++) {
      if (s > 1 && ktiles / s < 8) break;
      const int resident = ntt == 2 ? pair_clusters_resident<2>(s) : pair_clusters_resident<1>(s);
      if (resident == 0) continue;
      // a split grid that fits one wave of single-pair clusters runs its ranks as separate
      // clusters (given the scratch fg_linear_workspace_bytes asks for): one wave
      const int waves = (s > 1 && clusters * s <= one) ? 1 : (clusters + resident - 1) / resident;
      const double epi = 3.0 * ntt + (s > 1 ? 4.0 * ntt + 1.0 * s : 0.0);
      const double cost = waves * (((ktiles + s - 1) / s) * ktime + 5.0 + epi);
      if (cost < best - 1e-9) {
        best = cost;
        p.nt = tok;
        p.splits = s;
      }
    }
  }
  p.t_tiles = (M + p.nt - 1) / p.nt;
  p.cost = best;
  // The persistent stream-K launch (every resident pair takes an equal share of the (tile,
  // k-tile) iterations of 512-token tiles) runs only when a caller asks for it
  // (FG_GEMM_PERSISTENT): measured on the decode shapes it is still 1.5-2.6x slower than this
  // classic launch, so the time model does not choose it.  It needs every tile split into at
  // most 13 segments (the staging buffers of a split tile's partials).
  p.pairs = 0;
  const int sk = fg_streamk_pairs();
  if (sk > 0) {
    const int64_t iters = static_cast<int64_t>(p.n_tiles) * ((M + 511) / 512) * ktiles;
    const int P = static_cast<int>(iters < sk ? iters : sk);
    const int64_t per = (iters + P - 1) / P;
    const int64_t segs = per >= ktiles ? 2 : (ktiles + per - 1) / per + 1;  // most segments of a tile
    if (segs - 1 <= 12) p.pairs = sk;
  }
  return p;
}

template <int NTT, bool I8 = false>
fg_status launch_pair_nt(const CUtensorMap (&maps)[4], const GemmArgs &a, const Plan &p, cudaStream_t st, bool pdl) {
  fg_status rc = pair_attr_once<NTT, I8>();
  if (rc != FG_OK) return rc;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * p.n_tiles, p.t_tiles, p.splits);
  lc.blockDim = dim3(kPairThreads, 1, 1);
  lc.dynamicSmemBytes = kPairSmem;
  lc.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = a.flags ? 1 : p.splits;  // split ranks: one cluster, or flags
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = pdl ? 2 : 1;
  rc = fg_cuda_check(cudaLaunchKernelEx(&lc, I8 ? w4a8_gemm_pair_kernel<NTT> : w4a16_gemm_pair_kernel<NTT>, maps[0],
                                        maps[1], maps[2], maps[3], a));
  if (rc != FG_OK) return rc;
  return fg_launch_check();
}

fg_status launch_pair(const CUtensorMap (&maps)[4], const GemmArgs &a, const Plan &p, cudaStream_t st, bool pdl) {
  return p.nt == 256 ? launch_pair_nt<1>(maps, a, p, st, pdl) : launch_pair_nt<2>(maps, a, p, st, pdl);
}

// Test hook state (fg_test_gemm_stall): launches of the one-SM kernel still to stall, and
// their wait limit.
std::atomic<int> g_stall_count{0};
// Launch counter behind the split-rank flags' values (tagged apart from the stream-K kernel's).
std::atomic<unsigned long long> g_split_epoch{0};
std::atomic<uint64_t> g_stall_wait_ns{FG_WAIT_TIMEOUT_NS};

}  // namespace

// Optional scratch of the pair kernel's k split: one fp32 partial [tile tokens][256 features]
// per split of every pair tile.  Without it the partials are reduced inside the cluster.
static size_t pair_part_bytes(const Plan &p) {
  return p.splits < 2 ? 0 : static_cast<size_t>(p.n_tiles) * p.t_tiles * p.splits * p.nt * 256 * sizeof(float);
}
// ... and the flags of the split ranks run as separate clusters: [tile][rank][CTA half]
static size_t pair_flag_bytes(const Plan &p) {
  return p.splits < 2 ? 0 : static_cast<size_t>(p.n_tiles) * p.t_tiles * p.splits * 2 * sizeof(unsigned long long);
}

size_t fg_linear_ws_bytes(int M, int N, int K) {
  if (M <= 256 || N <= 0 || K <= 0 || K % kBK) return 0;
  const Plan p = make_pair_plan(M, N, K);
  const size_t classic = pair_part_bytes(p) + pair_flag_bytes(p), sk = p.pairs > 0 ? fg_streamk_scratch_bytes(p.pairs) : 0;
  return classic > sk ? classic : sk;
}

fg_status fg_linear_launch(const fg_half *x, int M, int K, const fg_qtensor *w, const fg_half *bias,
                           const fg_half *residual, int flags, int qscale_cols, float qscale, fg_half *y,
                           void *workspace, size_t ws_bytes, cudaStream_t st, bool pdl) {
  const int N = static_cast<int>(w->shape[0]);
  if (M == 0) return FG_OK;
  const int G = w->group == 128 ? 128 : 64;
  // M > 256: CTA pairs.  The classic pair kernel stages the group metadata by tensor copies of
  // 8 group columns, so a row of K/G fp16 values must be whole 16-byte units and the arrays
  // 16-byte aligned; otherwise (and for M <= 256) the one-SM kernel runs.
  const bool big = M > 256;
  const Plan pp = big ? make_pair_plan(M, N, K) : Plan{};
  const bool sk = big && (flags & FG_GEMM_PERSISTENT) && pp.pairs > 0 && workspace && fg_aligned16(workspace) &&
                  ws_bytes >= fg_streamk_scratch_bytes(pp.pairs);
  const bool pair = big && !sk && (K / G) % 8 == 0 && fg_aligned16(w->mins) && fg_aligned16(w->scales);
  const Plan p = (sk || pair) ? pp : make_plan(M, N, K);
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FG_ERR_CUDA;
  CUtensorMap maps[4];  // x, and for the classic pair kernel the codes, mins and scales
  CUtensorMap &map = maps[0];
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {kBK, static_cast<cuuint32_t>((sk || pair) ? 128 : p.nt)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<fg_half *>(x), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return FG_ERR_INVALID;
  if (pair) {
    // codes [N][K/2] bytes, box 32 B (one k-tile) x 128 rows; mins, scales [N][K/G] fp16,
    // box 8 columns x 128 rows
    const cuuint64_t cdims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
    const cuuint64_t cstr[1] = {static_cast<cuuint64_t>(K / 2)};
    const cuuint32_t cbox[2] = {32, 128};
    cr = enc(&maps[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w->codes), cdims, cstr, cbox, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return FG_ERR_INVALID;
    const cuuint64_t mdims[2] = {static_cast<cuuint64_t>(K / G), static_cast<cuuint64_t>(N)};
    const cuuint64_t mstr[1] = {static_cast<cuuint64_t>(K / G) * 2};
    const cuuint32_t mbox[2] = {8, 128};
    const void *meta[2] = {w->mins, w->scales};
    for (int j = 0; j < 2; j++) {
      cr = enc(&maps[2 + j], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(meta[j]), mdims, mstr, mbox, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (cr != CUDA_SUCCESS) return FG_ERR_INVALID;
    }
  }
  GemmArgs a;
  a.wc = w->codes;
  a.wm = reinterpret_cast<const __half *>(w->mins);
  a.ws = reinterpret_cast<const __half *>(w->scales);
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
  a.gshift = w->group == 128 ? 1 : 0;
  a.part = nullptr;
  a.flags = nullptr;
  a.epoch = 0;
  if (pair && p.splits > 1 && workspace && fg_aligned16(workspace) && ws_bytes >= pair_part_bytes(p)) {
    a.part = static_cast<float *>(workspace);
    // With room for the flags and the whole grid resident at once (clusters of one pair), the
    // split ranks run as separate clusters and meet through the flags: no cluster of 2 x splits
    // CTAs, which the GPCs may not hold in one wave.
    const int one = p.nt == 256 ? pair_clusters_resident<1>(1) : pair_clusters_resident<2>(1);
    if (ws_bytes >= pair_part_bytes(p) + pair_flag_bytes(p) && p.n_tiles * p.t_tiles * p.splits <= one) {
      a.flags = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) + pair_part_bytes(p));
      a.epoch = 0xF6A4000000000000ull | (g_split_epoch.fetch_add(1) + 1);
    }
  }
  a.ascale = nullptr;
  a.cscale = nullptr;
  a.err = fg_error_word_ptr();
  if (!a.err) return FG_ERR_CUDA;
  a.wait_ns = FG_WAIT_TIMEOUT_NS;
  a.stall = 0;
  if (sk)
    return fg_streamk_launch(map, a.wc, a.wm, a.ws, a.gshift, a.bias, a.res, a.relu, a.qcols, a.qscale, a.y, M, N, K,
                             p.pairs, workspace, a.err, st, pdl);
  if (pair) return launch_pair(maps, a, p, st, pdl);
  int left = g_stall_count.load();
  while (left > 0 && !g_stall_count.compare_exchange_weak(left, left - 1)) {
  }
  if (left > 0) {
    a.stall = 1;
    a.wait_ns = g_stall_wait_ns.load();
  }
  switch (p.nt) {
    case 16: return launch_nt<16>(map, a, p, st, pdl);
    case 32: return launch_nt<32>(map, a, p, st, pdl);
    case 64: return launch_nt<64>(map, a, p, st, pdl);
    case 128: return launch_nt<128>(map, a, p, st, pdl);
    default: return launch_nt<256>(map, a, p, st, pdl);
  }
}

extern "C" size_t fg_linear_workspace_bytes(int M, int N, int K) { return fg_linear_ws_bytes(M, N, K); }

extern "C" fg_status fg_test_gemm_stall(int count, uint64_t wait_limit_ns) {
  if (count < 0 || wait_limit_ns == 0 || wait_limit_ns > FG_WAIT_TIMEOUT_NS) return FG_ERR_INVALID;
  g_stall_wait_ns.store(wait_limit_ns);
  g_stall_count.store(count);
  return FG_OK;
}

extern "C" fg_status fg_linear_plan(int M, int N, int K, int *tile_tokens, int *splits, int *pairs) {
  if (!tile_tokens || !splits || !pairs || M <= 0 || N <= 0 || K <= 0 || K % kBK || N % 128) return FG_ERR_INVALID;
  Plan p;
  if (M > 256) {
    p = make_pair_plan(M, N, K);
    if ((K / 64) % 8) {  // the classic launch for groups of 64 runs one SM per tile here
      const int pairs = p.pairs;
      p = make_plan(M, N, K);
      p.pairs = pairs;
    }
  } else {
    p = make_plan(M, N, K);
    p.pairs = 0;
  }
  *tile_tokens = p.nt;
  *splits = p.splits;
  *pairs = p.pairs;
  return FG_OK;
}

extern "C" fg_status fg_linear_w4a16(const fg_half *x, int M, int K, const fg_qtensor *w, const fg_half *bias,
                                     const fg_half *residual, int flags, int qscale_cols, float qscale, fg_half *y,
                                     void *workspace, size_t workspace_bytes, void *stream) {
  if (!w || M < 0 || K <= 0) return FG_ERR_INVALID;
  if (w->bits != 4 || (w->group != 64 && w->group != 128)) return FG_ERR_UNSUPPORTED;
  if (w->ndim != 2 || w->dim != 1 || w->shape[1] != K) return FG_ERR_SHAPE;
  const int64_t N = w->shape[0];
  if (K % w->group || N <= 0 || N % 128 || N > (1 << 30)) return FG_ERR_SHAPE;
  if (flags & ~(FG_EPI_RELU | FG_EPI_RESIDUAL | FG_GEMM_PERSISTENT)) return FG_ERR_INVALID;
  if (M == 0) return FG_OK;
  if (!x || !y || !w->codes || !w->mins || !w->scales) return FG_ERR_INVALID;
  if (!fg_aligned16(x) || !fg_aligned16(y) || !fg_aligned16(w->codes)) return FG_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(bias) & 1u) || (reinterpret_cast<uintptr_t>(w->mins) & 1u) ||
      (reinterpret_cast<uintptr_t>(w->scales) & 1u))
    return FG_ERR_INVALID;
  if ((flags & FG_EPI_RESIDUAL) && (!residual || !fg_aligned16(residual))) return FG_ERR_INVALID;
  // weights may come from the kernel just before (fg_quantize): no overlap with it
  return fg_linear_launch(x, M, K, w, bias, residual, flags, qscale_cols, qscale, y, workspace, workspace_bytes,
                          static_cast<cudaStream_t>(stream), false);
}

// ---- W4A8 on CTA pairs (fg_w4a8.cu takes this launch for M > 256) ----
// The W4A16 pair launch's planner (k-tiles of 128) and k-split modes: with the scratch of
// fg_w4a8_pair_ws_bytes the ranks' s32 partials go through it (flags when the grid is one wave),
// else over distributed shared memory; the sums are exact in every mode.  The group metadata
// arrive by tensor copies of 16 group columns: rows of K / 64 bytes must be whole 16-byte units.
bool fg_w4a8_pair_eligible(int M, int K, const fg_w4a8_weight *w) {
  return M > 256 && (K / 64) % 16 == 0 && fg_aligned16(w->gmin) && fg_aligned16(w->gstep);
}

size_t fg_w4a8_pair_ws_bytes(int M, int N, int K) {
  if (M <= 256 || N <= 0 || K <= 0 || K % 128) return 0;
  const Plan p = make_pair_plan(M, N, K, 128);
  return pair_part_bytes(p) + pair_flag_bytes(p);
}

void fg_w4a8_pair_plan(int M, int N, int K, int *tile_tokens, int *splits) {
  const Plan p = make_pair_plan(M, N, K, 128);
  *tile_tokens = p.nt;
  *splits = p.splits;
}

fg_status fg_w4a8_pair_launch(const int8_t *a8, const float *ascale, int M, int K, const fg_w4a8_weight *w,
                              const fg_half *bias, const fg_half *residual, int flags, int qscale_cols, float qscale,
                              fg_half *y, void *workspace, size_t ws_bytes, cudaStream_t st) {
  const int N = static_cast<int>(w->N);
  const Plan p = make_pair_plan(M, N, K, 128);
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FG_ERR_CUDA;
  CUtensorMap maps[4];  // activations, codes, group minima, group steps
  const cuuint32_t estr[2] = {1, 1};
  const cuuint64_t xdims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t xstr[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t xbox[2] = {128, 128};
  CUresult cr = enc(&maps[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(a8), xdims, xstr, xbox, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return FG_ERR_INVALID;
  const cuuint64_t cdims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
  const cuuint64_t cstr[1] = {static_cast<cuuint64_t>(K / 2)};
  const cuuint32_t cbox[2] = {64, 128};
  cr = enc(&maps[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w->codes, cdims, cstr, cbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return FG_ERR_INVALID;
  const cuuint64_t mdims[2] = {static_cast<cuuint64_t>(K / 64), static_cast<cuuint64_t>(N)};
  const cuuint64_t mstr[1] = {static_cast<cuuint64_t>(K / 64)};
  const cuuint32_t mbox[2] = {16, 128};
  void *meta[2] = {w->gmin, w->gstep};
  for (int j = 0; j < 2; j++) {
    cr = enc(&maps[2 + j], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, meta[j], mdims, mstr, mbox, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return FG_ERR_INVALID;
  }
  GemmArgs a;
  a.wc = w->codes;
  a.wm = nullptr;
  a.ws = nullptr;
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
  a.gshift = 0;
  a.part = nullptr;
  a.flags = nullptr;
  a.epoch = 0;
  if (p.splits > 1 && workspace && fg_aligned16(workspace) && ws_bytes >= pair_part_bytes(p)) {
    a.part = static_cast<float *>(workspace);
    const int one = p.nt == 256 ? pair_clusters_resident<1>(1) : pair_clusters_resident<2>(1);
    if (ws_bytes >= pair_part_bytes(p) + pair_flag_bytes(p) && p.n_tiles * p.t_tiles * p.splits <= one) {
      a.flags = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) + pair_part_bytes(p));
      a.epoch = 0xF6A4000000000000ull | (g_split_epoch.fetch_add(1) + 1);
    }
  }
  a.ascale = ascale;
  a.cscale = w->cscale;
  a.err = fg_error_word_ptr();
  if (!a.err) return FG_ERR_CUDA;
  a.wait_ns = FG_WAIT_TIMEOUT_NS;
  a.stall = 0;
  return p.nt == 256 ? launch_pair_nt<1, true>(maps, a, p, st, false) : launch_pair_nt<2, true>(maps, a, p, st, false);
}
