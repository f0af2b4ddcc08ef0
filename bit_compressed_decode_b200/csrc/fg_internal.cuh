// fg_internal.cuh -- shared device/host helpers of the sm_100a library.
// Inline PTX for mbarriers, bulk/tensor copies (TMA) and the 5th-generation
// tensor-core instructions (tcgen05), plus bounded waits that report through
// the device error word instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fg.h"

// Bits of the device error word.
#define FG_DEVERR_RANGE 1u
#define FG_DEVERR_TIMEOUT 2u

// Every pipeline wait gives up after this many nanoseconds of device time.
#define FG_WAIT_TIMEOUT_NS 2000000000ull

// Host helpers (fg_status.cu).
unsigned int *fg_error_word_ptr();  // device address of this device's error word (nullptr on failure)
int fg_sm_count();                  // streaming multiprocessors of the current device (148 if unknown)
size_t fg_layer_ws_required(const fg_layer_config *c, int rows);  // workspace a layer call cannot do without
fg_status fg_cuda_check(cudaError_t e);  // records the error text, maps to FG_ERR_CUDA
fg_status fg_launch_check();             // cudaGetLastError after a launch

static inline bool fg_aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Events of a layer step whose weights (and cache) arrive in slices (the stack's sliced
// prefetch): `ready` events the step waits for before the kernels that read a slice, `done`
// events it records once the kernels that read a slice have been enqueued.  Any may be null.
//   ready: [0] vectors (biases, LayerNorm parameters) before LN1, [1] wqkv before the QKV GEMM,
//          [2] the KV cache before the KV append, [3] wo, [4] w1, [5] w2 before their GEMMs.
//   done:  [1] after the QKV GEMM, [2] after attention (the cache), [3] after the output
//          projection, [4] after FC1, [0] and [5] after FC2 (its bias is the last vector read).
struct fg_layer_slices {
  cudaEvent_t ready[6];
  cudaEvent_t done[6];
};
fg_status fg_layer_decode_sliced(const fg_layer_config *c, const fg_layer_weights *w, const fg_kv_cache *kv,
                                 const fg_half *x_in, fg_half *x_out, const int32_t *positions, int num_gpu_batches,
                                 int gpu_batch_size, void *workspace, size_t workspace_bytes, cudaStream_t st,
                                 const fg_layer_slices *sl);
fg_status fg_layer_blob_slices(const fg_layer_config *c, size_t begin[5], size_t end[5]);

// The 4-bit group of a KV cache or layer config: 0 selects 64; 64 and 128 as given; 0 for any
// other value (unsupported).
static inline int fg_kv_group(int group) { return group == 0 ? 64 : (group == 64 || group == 128) ? group : 0; }

// --------------------------------------------------------------------------------------
// device helpers
// --------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Flags in global memory that CTAs of one grid, all resident, exchange (release / acquire at
// GPU scope).
__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of an mbarrier.  Gives up (returns false) when the
// shared abort flag is raised by another thread or after limit_ns nanoseconds
// (FG_WAIT_TIMEOUT_NS unless a test shortens it), in which case it raises the abort
// flag and the device error word.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                  unsigned int *err, uint64_t limit_ns = FG_WAIT_TIMEOUT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort_flag && *abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      if (abort_flag) *abort_flag = 1;
      if (err) atomicOr(err, FG_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 2-D tiled tensor copy global -> shared (no multicast).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- thread-block clusters / distributed shared memory --------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of every CTA in the cluster arrives (release) and waits (acquire).
// Programmatic dependent launch.  A kernel launched with the programmatic-serialisation
// attribute may start while the previous kernel in its stream is still running;
// griddep_wait() blocks until that kernel has completed and its memory is visible, so it
// must precede every read of data the previous kernel produced and every write the previous
// kernel could still be reading.  griddep_launch() lets the next such kernel be scheduled
// once every CTA of this grid has issued it (without it: once this grid completes).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// ---- tcgen05 (5th-gen tensor cores, TMEM accumulators) -------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, fp16 inputs, fp32 accumulation.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T: A read from tensor memory (row m in lane m,
// k along columns, two fp16 per 32-bit column), fp32 accumulation.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers: thread i writes lane (base+i).
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Arrive on an mbarrier once every previously issued tcgen05.mma of this thread has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base+i), columns col..col+31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Non-blocking phase test (no suspension), acquire at CTA or cluster scope.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait by polling, for a thread that has its warp to itself and must react to the
// phase change at once (try_wait may suspend the thread past the completion).
template <bool kCluster>
__device__ __forceinline__ bool mbar_poll_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                  unsigned int *err) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; it++) {
    if (kCluster ? mbar_test_wait_cluster(bar, parity) : mbar_test_wait(bar, parity)) return true;
    if ((it & 63u) == 63u) {
      if (abort_flag && *abort_flag) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > FG_WAIT_TIMEOUT_NS) {
        if (abort_flag) *abort_flag = 1;
        if (err) atomicOr(err, FG_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

// ---- CTA pairs (cta_group::2): one MMA spans the tensor cores of two SMs --------------
// The pair is two CTAs of a cluster with ranks 2p and 2p+1; the even CTA issues the MMAs.
// A (M = 256) is split by rows (128 per CTA), B by columns (N/2 per CTA), and each CTA's
// TMEM holds its 128 rows of D over all N columns.

// Issued by the same warp in both CTAs of the pair, with the same shared-memory slot.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (+)= A * B^T over the pair; descriptors name this CTA's halves (same offsets in both).
__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at the same offset in every CTA of `cta_mask` when all
// previously issued pair MMAs of this thread have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(cta_mask)
      : "memory");
}

// 2-D tiled copy global -> this CTA's shared memory, completion counted on an mbarrier that
// may sit in the peer CTA of the pair (shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

// 1-D bulk copy from this CTA's shared memory to shared memory of a CTA of the cluster,
// completion counted (complete_tx) on an mbarrier in that CTA (both addresses and the size
// multiples of 16 bytes; shared::cluster addresses for dst and the barrier).
__device__ __forceinline__ void bulk_s2s_cluster(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                                 uint32_t bar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(src), "r"(bytes), "r"(bar_cluster)
               : "memory");
}

// Arrive (release at cluster scope) on an mbarrier given by its shared::cluster address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// try_wait with acquire at cluster scope (arrivals may come from the peer CTA).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded_cluster(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                          unsigned int *err) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (abort_flag && *abort_flag) return false;
    if (globaltimer_ns() - t0 > FG_WAIT_TIMEOUT_NS) {
      if (abort_flag) *abort_flag = 1;
      if (err) atomicOr(err, FG_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// Shared-memory matrix descriptor of a K-major operand tile laid out in the
// 128-byte swizzle pattern: rows of 128 bytes, 8-row (1024-byte) atoms stacked
// along M/N (stride 1024 bytes), atom base 1024-byte aligned.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1u) << 16;                     // leading byte offset (unused for swizzled K-major)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;             // stride byte offset: 8 rows * 128 B
  d |= static_cast<uint64_t>(1u) << 46;                     // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2u) << 61;                     // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16 with fp16 A and B, fp32 D, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_f16_f32(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (0u << 7) | (0u << 10)                    // A, B format: f16
         | (0u << 15) | (0u << 16)                   // A, B K-major
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// ---- 4-bit group helpers shared by the quantise kernels --------------------------------

// fp16 value of 1024 + n for a nibble n in bits 0..3 and 16..19 of `bits` (magic-number
// conversion: 0x6400 is 1024.0 in binary16 and the nibble fills the low mantissa bits).
__device__ __forceinline__ __half2 nib2_plus1024(uint32_t bits) {
  uint32_t v = (bits & 0x000F000Fu) | 0x64006400u;
  return *reinterpret_cast<__half2 *>(&v);
}

// Dequantise 8 codes of one 32-bit word (element 2j in the low nibble of byte j)
// into 8 fp16 values in element order: round_to_fp16(min + code * scale), exactly
// rounded once (hfma2).  Each pair (e_2j, e_2j+1) is gathered with one byte
// permute (byte j of w -> bits 0..7, byte j of w>>4 -> bits 16..23); the mask in
// nib2_plus1024 keeps the low nibble of each half.
__device__ __forceinline__ uint4 dequant8(uint32_t w, __half2 scale2, __half2 min2) {
  const __half2 k1024 = __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400));
  const uint32_t s = w >> 4;
  __half2 c01 = __hsub2(nib2_plus1024(__byte_perm(w, s, 0x0400)), k1024);
  __half2 c23 = __hsub2(nib2_plus1024(__byte_perm(w, s, 0x0501)), k1024);
  __half2 c45 = __hsub2(nib2_plus1024(__byte_perm(w, s, 0x0602)), k1024);
  __half2 c67 = __hsub2(nib2_plus1024(__byte_perm(w, s, 0x0703)), k1024);
  __half2 y01 = __hfma2(c01, scale2, min2);
  __half2 y23 = __hfma2(c23, scale2, min2);
  __half2 y45 = __hfma2(c45, scale2, min2);
  __half2 y67 = __hfma2(c67, scale2, min2);
  uint4 r;
  r.x = *reinterpret_cast<uint32_t *>(&y01);
  r.y = *reinterpret_cast<uint32_t *>(&y23);
  r.z = *reinterpret_cast<uint32_t *>(&y45);
  r.w = *reinterpret_cast<uint32_t *>(&y67);
  return r;
}

// 8-bit form of quant_group8: the same group min/max, scale = fp16(RN(d / 255)) (the IEEE
// division), the same reciprocal and rounding, codes clamped to 255, one byte per code: the
// lane's 8 codes as two words (byte k of word w = code 4w + k).  All 32 lanes must call it.
template <int LANES = 8>
__device__ __forceinline__ uint2 quant_group8_u8(const uint4 v, __half &min_h, __half &scale_h);

// RN(d / 15) for finite d >= 0: d * RN(1/15) corrected by one fused multiply-add on the
// exact residual d - 15 q0 (Markstein's correction step, P. Markstein, IBM J. Res. Dev. 34,
// 1990).  Equal to the correctly rounded quotient for every non-negative finite float
// (checked exhaustively against __fdiv_rn on B200).
__device__ __forceinline__ float div15_rn(float d) {
  const float c = 0.0666666701436042785644531250f;  // RN(1/15)
  const float q0 = __fmul_rn(d, c);
  const float r = __fmaf_rn(-15.0f, q0, d);
  return __fmaf_rn(r, c, q0);
}

// RN(1 / s) for s a positive finite fp16 value widened to fp32: one Newton-Raphson step with
// a fused multiply-add on the hardware reciprocal approximation (Markstein, same reference).
// Equal to the correctly rounded reciprocal for every such s (checked exhaustively against
// __fdiv_rn on B200).
__device__ __forceinline__ float rcp_rn_f16val(float s) {
  float r0;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(s));
  const float e = __fmaf_rn(-s, r0, 1.0f);
  return __fmaf_rn(e, r0, r0);
}

// Insert the low 4 bits of v into w at bit position pos.
__device__ __forceinline__ uint32_t bfi4(uint32_t v, uint32_t w, uint32_t pos) {
  uint32_t r;
  asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(r) : "r"(v), "r"(w), "r"(pos));
  return r;
}

// Cooperative quantisation of one group of 8 * LANES fp16 values (64 or 128) held by
// LANES consecutive lanes (lane j of them holds elements 8j..8j+7 in v).  Steps and fp32 operation
// order as stated in fg.h: min/max over the group, mn += 0, d = mx - mn,
// scale = fp16_rn(d/15), inv = 1/scale, code = clamp(rint((x - mn) * inv), 0, 15).
// Min and max are taken on the fp16 values (exact, as on their fp32 widenings), carried
// between lanes as the pair {min, -max}; rint is the fp32 addition of 1.5 * 2^23 (the
// nearest integer, ties to even, lands in the low mantissa bits; the quotient lies in
// [0, 30] because the scale is rounded to fp16).  Inputs must be finite.
// Returns this lane's 8 codes packed into one 32-bit word (element 8j+2i in the low
// nibble of byte i) and the group's fp16 min and scale.  All 32 lanes of the warp
// must call it together.
template <int LANES = 8>  // lanes sharing one group: 8 (group of 64) or 16 (group of 128)
__device__ __forceinline__ uint32_t quant_group8(const uint4 v, __half &min_h, __half &scale_h) {
  const __half2 *h2 = reinterpret_cast<const __half2 *>(&v);
  const __half2 lo = __hmin2(__hmin2(h2[0], h2[1]), __hmin2(h2[2], h2[3]));
  const __half2 hi = __hmax2(__hmax2(h2[0], h2[1]), __hmax2(h2[2], h2[3]));
  // {min, -max} of this lane's 8 values
  __half2 mm = __halves2half2(__hmin(__low2half(lo), __high2half(lo)),
                              __hneg(__hmax(__low2half(hi), __high2half(hi))));
#pragma unroll
  for (int o = 1; o < LANES; o <<= 1) {
    const uint32_t u = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<const uint32_t *>(&mm), o);
    mm = __hmin2(mm, *reinterpret_cast<const __half2 *>(&u));
  }
  float mn = __low2float(mm);
  const float mx = -__high2float(mm);
  mn = __fadd_rn(mn, 0.0f);
  const float d = __fsub_rn(mx, mn);
  __half sh = __float2half_rn(div15_rn(d));
  const float s = __half2float(sh);
  uint32_t word = 0;
  if (s != 0.0f) {
    const float inv = rcp_rn_f16val(s);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const float2 f = __half22float2(h2[i]);
      const float r0 = __fadd_rn(__fmul_rn(__fsub_rn(f.x, mn), inv), 12582912.0f);
      const float r1 = __fadd_rn(__fmul_rn(__fsub_rn(f.y, mn), inv), 12582912.0f);
      word = bfi4(min(__float_as_uint(r0), 0x4B40000Fu), word, 8 * i);
      word = bfi4(min(__float_as_uint(r1), 0x4B40000Fu), word, 8 * i + 4);
    }
  } else {
    sh = __ushort_as_half(0);
  }
  min_h = __float2half_rn(mn);
  scale_h = sh;
  return word;
}

template <int LANES>
__device__ __forceinline__ uint2 quant_group8_u8(const uint4 v, __half &min_h, __half &scale_h) {
  const __half2 *h2 = reinterpret_cast<const __half2 *>(&v);
  const __half2 lo = __hmin2(__hmin2(h2[0], h2[1]), __hmin2(h2[2], h2[3]));
  const __half2 hi = __hmax2(__hmax2(h2[0], h2[1]), __hmax2(h2[2], h2[3]));
  __half2 mm = __halves2half2(__hmin(__low2half(lo), __high2half(lo)),
                              __hneg(__hmax(__low2half(hi), __high2half(hi))));
#pragma unroll
  for (int o = 1; o < LANES; o <<= 1) {
    const uint32_t u = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<const uint32_t *>(&mm), o);
    mm = __hmin2(mm, *reinterpret_cast<const __half2 *>(&u));
  }
  float mn = __low2float(mm);
  const float mx = -__high2float(mm);
  mn = __fadd_rn(mn, 0.0f);
  const float d = __fsub_rn(mx, mn);
  __half sh = __float2half_rn(__fdiv_rn(d, 255.0f));
  const float s = __half2float(sh);
  uint32_t w[2] = {0u, 0u};
  if (s != 0.0f) {
    const float inv = rcp_rn_f16val(s);
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const float2 f = __half22float2(h2[i]);
      const float r0 = __fadd_rn(__fmul_rn(__fsub_rn(f.x, mn), inv), 12582912.0f);
      const float r1 = __fadd_rn(__fmul_rn(__fsub_rn(f.y, mn), inv), 12582912.0f);
      const uint32_t c0 = min(__float_as_uint(r0), 0x4B4000FFu) & 0xFFu;
      const uint32_t c1 = min(__float_as_uint(r1), 0x4B4000FFu) & 0xFFu;
      w[i >> 1] |= (c0 | (c1 << 8)) << (16 * (i & 1));
    }
  } else {
    sh = __ushort_as_half(0);
  }
  min_h = __float2half_rn(mn);
  scale_h = sh;
  return make_uint2(w[0], w[1]);
}

// Eight 8-bit codes (two words, byte k of word w = code 4w + k) -> eight fp16 values
// fp16_rn(min + code * scale): a byte placed under the exponent bits 0x64 is the fp16 value
// 1024 + code (exact), less 1024 is the code, and one half-precision FMA rounds once.
__device__ __forceinline__ uint4 dequant8_u8(uint2 w, __half2 scale2, __half2 min2) {
  const __half2 k1024 = __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400));
  uint4 r;
  uint32_t *o = reinterpret_cast<uint32_t *>(&r);
  const uint32_t words[2] = {w.x, w.y};
#pragma unroll
  for (int i = 0; i < 2; i++) {
    const uint32_t a = __byte_perm(words[i], 0x6464u, 0x5140), b = __byte_perm(words[i], 0x6464u, 0x5342);
    const __half2 ca = __hsub2(*reinterpret_cast<const __half2 *>(&a), k1024);
    const __half2 cb = __hsub2(*reinterpret_cast<const __half2 *>(&b), k1024);
    const __half2 ya = __hfma2(ca, scale2, min2), yb = __hfma2(cb, scale2, min2);
    o[2 * i] = *reinterpret_cast<const uint32_t *>(&ya);
    o[2 * i + 1] = *reinterpret_cast<const uint32_t *>(&yb);
  }
  return r;
}
