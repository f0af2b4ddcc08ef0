// fg_gemm_streamk.cu -- persistent W4A16 GEMM on CTA pairs with a stream-K schedule.
//
// y[m][n] = epi( sum_k x[m][k] * deq(W)[n][k] + b[n] ), W packed 4-bit along k ("FlexGen
// Guide: High-Throughput LLM Offloading on One GPU", section 3: weights stay 4-bit and are
// dequantised on the fly so the tensor cores compute in FP16).
//
// Work: pair tiles of 256 output features x 512 tokens (two M=256 x N=256 tcgen05 MMAs per
// 16-wide k step, cta_group::2), each over K/64 k-tiles.  The (tile, k-tile) iterations,
// tile-major, are cut into one contiguous range per CTA pair of the grid (one pair per two SMs,
// all resident), so every pair does the same number of k-tiles whatever the tile count -- the
// decode GEMMs have 16 to 64 pair tiles for 74 pairs.  A pair's range is a sequence of units
// (one tile's k-range each); a unit that covers a whole tile is finished directly, a tile split
// between pairs is finished by the pair holding its first k-segment: the other pairs store
// their fp32 partial sums in their slot of the caller's scratch and publish them with a flag
// tagged by the launch's epoch; the finishing pair adds them to its own, in k order (the same
// bits on every run), then applies the epilogue.  A split tile's first segment is the last unit
// of its pair's range and its other segments the first units of the next pairs' ranges, so the
// partials are normally in place before they are needed; the wait for them is bounded.
//
// Warp roles per CTA (448 threads):
//   warps 0..7   dequantise this CTA's 128 weight rows per k-tile into the ring (as the classic
//                pair kernel), running ahead across unit boundaries;
//   warp 8       TMA of this CTA's halves of the x tiles;
//   warp 9       even CTA: the MMA issuer; odd CTA: forwards "A half ready"; TMEM allocation;
//   warps 10..13 epilogue: drain the 512 accumulator columns from TMEM in two halves of 256
//                (one per token tile), releasing each half as soon as it is read, so the next
//                unit's MMAs start while the epilogue still stores.
// Epilogue stores go straight from registers to global memory: a warp writes 32 consecutive
// features of one token per instruction (64 B of fp16 or 128 B of fp32).
// Every wait is bounded (FG_WAIT_TIMEOUT_NS) and reports FG_ERR_TIMEOUT.
#include <atomic>

#include "fg_internal.cuh"

namespace {

constexpr int kBK = 64;
constexpr int kDeqWarps = 8;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kEpiWarp0 = 10;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
constexpr int kA = 128 * 128;              // this CTA's A tile: 128 rows x 128 B
constexpr int kBHalf = 128 * 128;          // this CTA's half of one token tile: 128 tokens x 128 B
constexpr int kNTT = 2;                    // 256-token MMA tiles per pair tile
constexpr int kTok = 256 * kNTT;           // tokens per pair tile
constexpr int kStage = kA + kNTT * kBHalf;
constexpr int kStages = 4;
constexpr int kRing = kStages * kStage;    // 192 KB
constexpr int kOutChunk = 32 * 128 * 4;    // one 32-token chunk of this CTA's 128 features, fp32: 16 KB
constexpr int kSmem = kRing + 2 * kOutChunk + 1024;  // ring + double-buffered output staging + alignment
constexpr int kCols = 256 * kNTT;          // TMEM columns
constexpr int kPrefetch = 4;
constexpr uint32_t kIdesc = umma_idesc_f16_f32(256, 256);
constexpr int64_t kSlotFloats = static_cast<int64_t>(kTok) * 256;  // one pair's fp32 partial
constexpr int kRedChunk = 32 * 128 * 4;    // one 32-token chunk of one CTA's partial: 16 KB
constexpr int kRedBufs = kRing / kRedChunk;  // 12 staging buffers in the (then idle) ring
static_assert(kRing == 192 * 1024, "ring");

struct SkArgs {
  const uint8_t *wc;   // codes [N][K/2]
  const __half *wm;    // mins  [N][K/G]
  const __half *ws;    // scales[N][K/G]
  const __half *bias;  // [N] or null
  const __half *res;   // [M][N] or null
  __half *y;           // [M][N]
  int M, N, K;
  int relu, qcols;
  float qscale;
  int gshift;          // log2(group / 64)
  int nf;              // feature pairs: ceil(N / 256)
  int KT;              // k-tiles: K / 64
  int64_t iters;       // tiles * KT
  int P;               // CTA pairs in the grid
  float *part;         // [P][2 CTA halves][512 tokens][128 features] fp32 partial slots
  unsigned long long *flags;  // [P][2]: epoch once slot p's half h is stored
  unsigned long long epoch;
  unsigned int *err;
};

__device__ __forceinline__ int64_t range_begin(const SkArgs &a, int p) { return static_cast<int64_t>(p) * a.iters / a.P; }

// Barrier among the epilogue warps only (named barrier 1; the non-aligned form, so a lane that
// polled alone may arrive apart from its warp).
__device__ __forceinline__ void epi_sync() { asm volatile("barrier.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); }

// Bounded wait for an mbarrier phase completed by this CTA's bulk copies, sleeping between tests.
__device__ __forceinline__ bool wait_sleeping_cta(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                  unsigned int *err) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > FG_WAIT_TIMEOUT_NS) {
      *abort_flag = 1;
      atomicOr(err, FG_DEVERR_TIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// Bounded wait for an mbarrier phase (acquire at cluster scope) that sleeps between tests, for
// warps with nothing else to do while the mainloop runs: they leave the issue slots to the
// producers.  Gives up on the CTA's abort flag or after FG_WAIT_TIMEOUT_NS.
__device__ __forceinline__ bool wait_sleeping(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                              unsigned int *err) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test_wait_cluster(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > FG_WAIT_TIMEOUT_NS) {
      *abort_flag = 1;
      atomicOr(err, FG_DEVERR_TIMEOUT);
      return false;
    }
    __nanosleep(256);
  }
  return true;
}


__global__ void __launch_bounds__(kThreads, 1) w4a16_gemm_streamk_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                        const SkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // full (even CTA): stage ready (8 dequant warps + TMA arrive with the x bytes of both CTAs
  // and the odd CTA's 16-byte "A half done" token); a_half (odd CTA): its dequant warps are
  // done; empty: the pair's MMAs are done with the stage; accum_full: a unit's accumulation
  // is complete (both CTAs); tmem_empty[h] (even CTA): both CTAs' epilogue warps have read
  // accumulator half h; drain: the MMA issuer's final commit.
  __shared__ __align__(8) uint64_t full[kStages], a_half[kStages], empty[kStages], accum_full, tmem_empty[2], drain;
  __shared__ __align__(8) uint64_t red_bar[kRedBufs];  // staged partial chunks of a split tile's other segments
  __shared__ __align__(16) uint32_t token_src[4], token_sink[kStages][4];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  griddep_launch();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t lead = crank & ~1u;
  const bool leader = crank == lead;
  const int half = static_cast<int>(crank & 1u);
  const int p = blockIdx.x >> 1;
  const int64_t it0 = range_begin(a, p), it1 = range_begin(a, p + 1);
  const int nit = static_cast<int>(it1 - it0);
  volatile int *abortp = &abort_flag;
  const uint16_t pair_mask = static_cast<uint16_t>(3u << lead);
  auto a_tile = [&](int st) { return smem + st * kStage; };
  auto b_tile = [&](int st, int t) { return smem + st * kStage + kA + t * kBHalf; };

  if (tid == 0) {
    for (int i = 0; i < kStages; i++) {
      mbar_init(smem_u32(&full[i]), kDeqWarps + 1);
      mbar_init(smem_u32(&a_half[i]), kDeqWarps);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    mbar_init(smem_u32(&accum_full), 1);
    mbar_init(smem_u32(&tmem_empty[0]), 2 * kEpiWarps);
    mbar_init(smem_u32(&tmem_empty[1]), 2 * kEpiWarps);
    mbar_init(smem_u32(&drain), 1);
    for (int i = 0; i < kRedBufs; i++) mbar_init(smem_u32(&red_bar[i]), 1);
    abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_u32(&tmem_slot), kCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp < kDeqWarps) {
    // ---------------- dequantise: row tid % 128, k half tid / 128, every iteration ----------------
    const int row = tid & 127, hk = tid >> 7;
    const int gstride = (a.K / kBK) >> a.gshift;
    // position (tile, k-tile) of the next fetch, advanced without divisions
    int ftile = static_cast<int>(it0 / a.KT), fkt = static_cast<int>(it0 % a.KT);
    const uint4 *crow = nullptr;
    const __half *mrow = nullptr, *srow = nullptr;
    bool live = false;
    auto set_row = [&]() {
      const int n = (ftile % a.nf) * 256 + half * 128 + row;
      live = n < a.N;
      crow = reinterpret_cast<const uint4 *>(a.wc + static_cast<int64_t>(live ? n : 0) * (a.K / 2));
      mrow = a.wm + static_cast<int64_t>(live ? n : 0) * gstride;
      srow = a.ws + static_cast<int64_t>(live ? n : 0) * gstride;
    };
    set_row();
    auto fetch = [&](uint4 &cb, __half &mb, __half &sb) {
      if (live) {
        cb = crow[fkt * 2 + hk];
        mb = mrow[fkt >> a.gshift];
        sb = srow[fkt >> a.gshift];
      } else {
        cb = make_uint4(0, 0, 0, 0);
        mb = sb = __ushort_as_half(0);
      }
      if (++fkt == a.KT) {
        fkt = 0;
        ftile++;
        set_row();
      }
    };
    uint4 cb[kPrefetch];
    __half mb[kPrefetch], sb[kPrefetch];
#pragma unroll
    for (int j = 0; j < kPrefetch; j++) {
      if (j < nit) {
        fetch(cb[j], mb[j], sb[j]);
      } else {
        cb[j] = make_uint4(0, 0, 0, 0);
        mb[j] = sb[j] = __ushort_as_half(0);
      }
    }
    const uint32_t done_bar0 = smem_u32(leader ? &full[0] : &a_half[0]);
    // statically indexed ring of prefetched codes (see the classic pair kernel): a slot is
    // consumed in place and refilled kPrefetch iterations ahead
    bool go = true;
    for (int i0 = 0; go && i0 < nit; i0 += kPrefetch) {
#pragma unroll
      for (int j = 0; j < kPrefetch; j++) {
        const int i = i0 + j;
        if (!go || i >= nit) break;
        const int st = i % kStages;
        const uint4 c0 = cb[j];
        const __half m0 = mb[j], s0 = sb[j];
        if (i + kPrefetch < nit) fetch(cb[j], mb[j], sb[j]);
        if (i >= kStages && !mbar_wait_bounded(smem_u32(&empty[st]), ((i / kStages) - 1) & 1, abortp, a.err)) {
          go = false;
          break;
        }
        const __half2 s2 = __half2half2(s0), m2 = __half2half2(m0);
        uint8_t *at = a_tile(st);
        const uint32_t words[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
        for (int c = 0; c < 4; c++) *reinterpret_cast<uint4 *>(at + sw128_offset(row, 4 * hk + c)) = dequant8(words[c], s2, m2);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(done_bar0 + st * 8);
      }
    }
  } else if (warp == kTmaWarp) {
    // ---------------- TMA: this CTA's halves of the two token tiles, every iteration ----------------
    if (lane == 0) {
      prefetch_tmap(&xmap);
      griddep_wait();  // x comes from the previous kernel
      int tile = static_cast<int>(it0 / a.KT), kt = static_cast<int>(it0 % a.KT);
      for (int i = 0; i < nit; i++, kt++) {
        if (kt == a.KT) {
          kt = 0;
          tile++;
        }
        const int st = i % kStages;
        if (i >= kStages && !mbar_wait_bounded(smem_u32(&empty[st]), ((i / kStages) - 1) & 1, abortp, a.err)) break;
        const int tok0 = (tile / a.nf) * kTok;
        const uint32_t fb = mapa_shared(smem_u32(&full[st]), lead);
        if (leader) mbar_arrive_expect_tx(smem_u32(&full[st]), 2 * kNTT * kBHalf + 16);
#pragma unroll
        for (int t = 0; t < kNTT; t++) tma_load_2d_pair(smem_u32(b_tile(st, t)), &xmap, kt * kBK, tok0 + t * 256 + half * 128, fb);
      }
    }
  } else if (warp == kMmaWarp) {
    if (!leader) {
      // ---------------- odd CTA: forward "A half ready" to the even CTA ----------------
      if (lane == 0) {
        for (int i = 0; i < nit; i++) {
          const int st = i % kStages;
          if (!mbar_wait_bounded(smem_u32(&a_half[st]), (i / kStages) & 1, abortp, a.err)) break;
          bulk_s2s_cluster(mapa_shared(smem_u32(&token_sink[st][0]), lead), smem_u32(&token_src[0]), 16,
                           mapa_shared(smem_u32(&full[st]), lead));
        }
      }
    } else if (lane == 0) {
      // ---------------- MMA issuer (even CTA) ----------------
      const uint64_t adesc0 = umma_desc_sw128(smem_u32(a_tile(0)));
      const uint64_t bdesc0 = umma_desc_sw128(smem_u32(b_tile(0, 0)));
      constexpr uint64_t kStageStep = kStage >> 4, kTileStep = kBHalf >> 4;
      int i = 0, u = 0;
      bool ok = true;
      for (int64_t it = it0; ok && it < it1; u++) {
        const int kb = static_cast<int>(it % a.KT);
        const int len = static_cast<int>(a.KT - kb < it1 - it ? a.KT - kb : it1 - it);
        for (int j = 0; j < len; j++, i++) {
          const int st = i % kStages;
          if (!mbar_poll_bounded<true>(smem_u32(&full[st]), (i / kStages) & 1, abortp, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = adesc0 + st * kStageStep, bd = bdesc0 + st * kStageStep;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; kk++) {
#pragma unroll
            for (int t = 0; t < kNTT; t++) {
              if (j == 0 && kk == 0 && u > 0) {
                // accumulator half t of the previous unit must have been read by both CTAs
                if (!mbar_poll_bounded<true>(smem_u32(&tmem_empty[t]), (u - 1) & 1, abortp, a.err)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
              }
              umma_f16_pair(tmem + t * 256, ad + 2 * kk, bd + t * kTileStep + 2 * kk, kIdesc, (j > 0 || kk > 0) ? 1u : 0u);
            }
            if (!ok) break;
          }
          if (!ok) break;
          umma_commit_pair(smem_u32(&empty[st]), pair_mask);
        }
        if (!ok) break;
        umma_commit_pair(smem_u32(&accum_full), pair_mask);
        it += len;
      }
      // every MMA issued so far has completed before TMEM is released
      umma_commit_pair(smem_u32(&drain), static_cast<uint16_t>(1u << crank));
      mbar_wait_bounded(smem_u32(&drain), 0, nullptr, a.err);
    }
  } else {
    // ---------------- epilogue warps: one unit at a time ----------------
    const int q4 = warp & 3;                       // TMEM lane quarter
    const int fl = q4 * 32 + lane;                 // feature row within this CTA's 128
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t te0 = mapa_shared(smem_u32(&tmem_empty[0]), lead);
    // scratch slots, flags, residual and outputs: only after the previous kernel has finished
    // (consecutive GEMMs of a layer share the scratch and may overlap under dependent launch)
    griddep_wait();
    int u = 0;
    for (int64_t it = it0; it < it1; u++) {
      const int tile = static_cast<int>(it / a.KT);
      const int kb = static_cast<int>(it % a.KT);
      const int len = static_cast<int>(a.KT - kb < it1 - it ? a.KT - kb : it1 - it);
      it += len;
      const bool whole = kb == 0 && len == a.KT, first = kb == 0;
      const int n = (tile % a.nf) * 256 + half * 128 + fl;
      const int tok0 = (tile / a.nf) * kTok;
      const bool nlive = n < a.N;
      bool ready = wait_sleeping(smem_u32(&accum_full), u & 1, abortp, a.err);
      tc_fence_after();
      // a split tile's first segment: wait until the pairs holding its other segments have
      // stored them (pairs p+1 .. q_last, whose ranges start inside this tile)
      int q_last = p;
      if (first && !whole) {
        const int64_t tile_end = static_cast<int64_t>(tile + 1) * a.KT;
        while (q_last + 1 < a.P && range_begin(a, q_last + 1) < tile_end) q_last++;
        if (warp == kEpiWarp0 && lane == 0 && ready) {
          for (int q = p + 1; q <= q_last && ready; q++) {
            const unsigned long long *f = a.flags + 2 * q + half;
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_u64(f) != a.epoch) {
              if (*abortp || globaltimer_ns() - t0 > FG_WAIT_TIMEOUT_NS) {
                *abortp = 1;
                atomicOr(a.err, FG_DEVERR_TIMEOUT);
                ready = false;
                break;
              }
              __nanosleep(128);
            }
          }
        }
        __syncwarp();
        epi_sync();
        ready = ready && !*abortp;
      }
      const float bias = (a.bias && nlive) ? __half2float(a.bias[n]) : 0.f;
      // this CTA's half of pair q's partial slot: [512 tokens][128 features]
      auto slot = [&](int q) { return a.part + static_cast<int64_t>(q * 2 + half) * kTok * 128; };
      float *mine = slot(p) + fl;
      // A split tile's first segment is always its pair's last unit (its range ends inside the
      // tile), so the pipeline ring is idle: the other segments' partials of each 32-token chunk
      // (16 KB contiguous per segment) are staged there by bulk copies, D chunks ahead.
      const int nq = q_last - p;
      const bool staged = first && !whole && nq <= kRedBufs;
      const int D = staged ? kRedBufs / nq : 1;
      auto issue_chunk = [&](int c) {
        const int b = c % D;
        const uint32_t bar = smem_u32(&red_bar[b]);
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nq * kRedChunk));
        for (int qi = 0; qi < nq; qi++)
          bulk_g2s(smem_u32(smem + (b * nq + qi) * kRedChunk), slot(p + 1 + qi) + c * 32 * 128, kRedChunk, bar);
      };
      if (staged && warp == kEpiWarp0 && lane == 0 && ready) {
        fence_proxy_async_smem();
        for (int c = 0; c < D && c < 2 * 8; c++) issue_chunk(c);
      }
      const int te = (warp - kEpiWarp0) * 32 + lane;   // epilogue thread 0..127
      const int n0 = (tile % a.nf) * 256 + half * 128;  // this CTA's first feature (N % 128 == 0)
      float qs = 1.f;
      if (n < a.qcols) qs = a.qscale;
      for (int t = 0; t < kNTT; t++) {
#pragma unroll 1
        for (int c32 = 0; c32 < 8; c32++) {
          const int c = t * 8 + c32;
          float *ost = reinterpret_cast<float *>(smem + kRing + (c & 1) * kOutChunk);  // [32 tokens][128]
          uint32_t v[32];
          tmem_ld_32x32b_x32(lane_base + t * 256 + c32 * 32, v);
          tmem_wait_ld();
          const int ml = t * 256 + c32 * 32;   // first token of the chunk within the tile
          float acc[32];
#pragma unroll
          for (int j = 0; j < 32; j++) acc[j] = __uint_as_float(v[j]);
          if (first && staged) {
            // the other segments, in k order, from the staged chunk
            if (ready && wait_sleeping_cta(smem_u32(&red_bar[c % D]), (c / D) & 1, abortp, a.err)) {
              for (int qi = 0; qi < nq; qi++) {
                const float *buf = reinterpret_cast<const float *>(smem + ((c % D) * nq + qi) * kRedChunk) + fl;
#pragma unroll
                for (int j = 0; j < 32; j++) acc[j] += buf[j * 128];
              }
            } else {
              ready = false;
            }
          } else if (first && !whole && ready) {
            for (int q = p + 1; q <= q_last; q++) {  // the other segments, in k order
              const float *src = slot(q) + fl;
#pragma unroll
              for (int j = 0; j < 32; j++) acc[j] += __ldcg(src + static_cast<int64_t>(ml + j) * 128);
            }
          }
          // stage the chunk: the raw partial sum of a later segment, or the output before its
          // residual (bias, q-scale, ReLU applied per feature)
#pragma unroll
          for (int j = 0; j < 32; j++) {
            float y = acc[j];
            if (first) {
              y = (y + bias) * qs;
              if (a.relu) y = fmaxf(y, 0.f);
            }
            ost[j * 128 + fl] = y;
          }
          // every epilogue thread has staged chunk c (and is done with its staged partials)
          epi_sync();
          if (staged && warp == kEpiWarp0 && lane == 0 && c + D < 2 * 8 && !*abortp) {
            fence_proxy_async_smem();
            issue_chunk(c + D);
          }
          if (ready) {
            if (!first) {
              // 16 KB contiguous in this pair's slot: 8 passes of 16 bytes per thread
#pragma unroll
              for (int i = 0; i < 8; i++) {
                const int e = i * 128 + te;
                *reinterpret_cast<float4 *>(mine - fl + static_cast<int64_t>(ml + (e >> 5)) * 128 + (e & 31) * 4) =
                    reinterpret_cast<const float4 *>(ost)[e];
              }
            } else if (n0 < a.N) {
              // 8 features of one token per thread and pass (16-byte stores, residual added here)
#pragma unroll
              for (int i = 0; i < 4; i++) {
                const int e = i * 128 + te, tok = e >> 4, f8 = (e & 15) * 8;
                const int m = tok0 + ml + tok;
                if (m >= a.M) continue;
                const float4 p0 = *reinterpret_cast<const float4 *>(ost + tok * 128 + f8);
                const float4 p1 = *reinterpret_cast<const float4 *>(ost + tok * 128 + f8 + 4);
                const float w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                __half *yp = a.y + static_cast<int64_t>(m) * a.N + n0 + f8;
                uint4 rv = make_uint4(0, 0, 0, 0);
                if (a.res) rv = *reinterpret_cast<const uint4 *>(a.res + static_cast<int64_t>(m) * a.N + n0 + f8);
                const __half *rh = reinterpret_cast<const __half *>(&rv);
                uint4 ov;
                __half *oh = reinterpret_cast<__half *>(&ov);
#pragma unroll
                for (int u = 0; u < 8; u++) oh[u] = __float2half_rn(w[u] + __half2float(rh[u]));
                *reinterpret_cast<uint4 *>(yp) = ov;
              }
            }
          }
        }
        // accumulator half t has been read: the next unit's MMAs may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader) mbar_arrive(smem_u32(&tmem_empty[t]));
          else mbar_arrive_cluster(te0 + t * 8);
        }
      }
      if (!first) {
        // publish the partial: every epilogue thread's stores, then the flag.  Every epilogue
        // thread takes every unit's barriers (an abort only skips loads and stores).
        __threadfence();
        epi_sync();
        if (warp == kEpiWarp0 && lane == 0 && !*abortp) st_release_u64(a.flags + 2 * p + half, a.epoch);
      }
    }
  }

  // copies issued before an abort land within microseconds: give them that long
  if (*abortp && (warp == kTmaWarp || warp == kMmaWarp) && lane == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 50000) {
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's TMEM and shared memory are no longer in use
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kCols);
  }
}

std::atomic<unsigned long long> g_epoch{0};

bool attr_done[64] = {false};

fg_status set_attr() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    fg_status rc = fg_cuda_check(
        cudaFuncSetAttribute(w4a16_gemm_streamk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem));
    if (rc != FG_OK) return rc;
    attr_done[dev] = true;
  }
  return FG_OK;
}

}  // namespace

// CTA pairs of this kernel that can be resident at once on the current device (0 if unknown).
int fg_streamk_pairs() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 0;
  if (!cache[dev]) {
    if (set_attr() != FG_OK) return 0;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(2, 1, 1);
    lc.blockDim = dim3(kThreads, 1, 1);
    lc.dynamicSmemBytes = kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, w4a16_gemm_streamk_kernel, &lc) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cache[dev] = n > 0 ? n : 0;
  }
  return cache[dev];
}

// Scratch of a stream-K launch over `pairs` CTA pairs: the partial slots, then the flags.
size_t fg_streamk_scratch_bytes(int pairs) {
  return static_cast<size_t>(pairs) * kSlotFloats * sizeof(float) + static_cast<size_t>(pairs) * 2 * 8;
}

// The stream-K launch: x through `map` (box 64 x 128 tokens, 128-byte swizzle), `pairs` CTA
// pairs, scratch of fg_streamk_scratch_bytes(pairs) bytes (16-byte aligned).
fg_status fg_streamk_launch(const CUtensorMap &map, const uint8_t *wc, const __half *wm, const __half *wsc, int gshift,
                            const __half *bias, const __half *res, int relu, int qcols, float qscale, __half *y,
                            int M, int N, int K, int pairs, void *scratch, unsigned int *err, cudaStream_t st,
                            bool pdl) {
  fg_status rc = set_attr();
  if (rc != FG_OK) return rc;
  SkArgs a;
  a.wc = wc;
  a.wm = wm;
  a.ws = wsc;
  a.bias = bias;
  a.res = res;
  a.y = y;
  a.M = M;
  a.N = N;
  a.K = K;
  a.relu = relu;
  a.qcols = qcols;
  a.qscale = qscale;
  a.gshift = gshift;
  a.nf = (N + 255) / 256;
  a.KT = K / kBK;
  a.iters = static_cast<int64_t>(a.nf) * ((M + kTok - 1) / kTok) * a.KT;
  a.P = static_cast<int>(pairs < a.iters ? pairs : a.iters);
  a.part = static_cast<float *>(scratch);
  a.flags = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(scratch) +
                                                   static_cast<size_t>(pairs) * kSlotFloats * sizeof(float));
  // flags hold a value no earlier launch wrote: a fixed high tag and a per-process count
  a.epoch = 0xF6A3000000000000ull | (g_epoch.fetch_add(1) + 1);
  a.err = err;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * a.P, 1, 1);
  lc.blockDim = dim3(kThreads, 1, 1);
  lc.dynamicSmemBytes = kSmem;
  lc.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = pdl ? 2 : 1;
  rc = fg_cuda_check(cudaLaunchKernelEx(&lc, w4a16_gemm_streamk_kernel, map, a));
  if (rc != FG_OK) return rc;
  return fg_launch_check();
}
