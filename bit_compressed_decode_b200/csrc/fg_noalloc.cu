// fg_noalloc.cu -- fg_layer_decode for callers that cannot allocate device memory.
//
// Some callers can't call cudaMalloc when they decode: a serving process that reserved
// all device memory up front for weights and KV cache (so any further allocation fails),
// an allocator-less host that only hands the library pointers it already owns, or code
// that must not allocate between steps for latency reasons.  For them this file keeps
// the layer's scratch (the intermediate activations of one decode step) in a file-scope
// device array of fixed size, which every GPU that loads the library holds until the
// process exits.  The computation is exactly fg_layer_decode's.  Under CUDA's lazy module
// loading the array's memory is taken when this file's module is loaded, which the first
// address lookup below triggers: callers make one call before they reserve device memory.
#include <limits.h>

#include <mutex>

#include "fg_internal.cuh"

namespace {

static __device__ __align__(256) uint8_t fg_noalloc_scratch[FG_NOALLOC_SCRATCH_BYTES];

std::mutex g_setup_mu;
void *g_scratch_addr[64] = {nullptr};

// Device address of this device's scratch array.  Set up once per device, with that
// device current; in host code the array's name only stands in for the symbol.
fg_status scratch_address(void **out) {
  int dev = 0;
  fg_status rc = fg_cuda_check(cudaGetDevice(&dev));
  if (rc != FG_OK) return rc;
  if (dev < 0 || dev >= 64) return FG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    rc = fg_cuda_check(cudaGetSymbolAddress(&p, fg_noalloc_scratch));
    if (rc != FG_OK) return rc;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FG_OK;
}

}  // namespace

extern "C" fg_status fg_layer_decode_noalloc(const fg_layer_config *c, const fg_layer_weights *w,
                                             const fg_kv_cache *kv, const fg_half *x_in, fg_half *x_out,
                                             const int32_t *positions, int num_gpu_batches, int gpu_batch_size,
                                             void *stream) {
  if (num_gpu_batches < 0 || gpu_batch_size < 0) return FG_ERR_INVALID;
  const int64_t rows = static_cast<int64_t>(num_gpu_batches) * gpu_batch_size;
  if (rows > INT_MAX) return FG_ERR_SHAPE;
  // the whole layer workspace must fit (activations and the GEMMs' scratch), so the GEMMs take
  // the same launches as fg_layer_decode given its full workspace: the same bits
  if (rows > 0 && fg_layer_ws_required(c, static_cast<int>(rows)) == 0) return FG_ERR_UNSUPPORTED;
  if (fg_layer_workspace_bytes(c, static_cast<int>(rows)) > FG_NOALLOC_SCRATCH_BYTES) return FG_ERR_WORKSPACE;
  void *scratch = nullptr;
  fg_status rc = scratch_address(&scratch);
  if (rc != FG_OK) return rc;
  return fg_layer_decode(c, w, kv, x_in, x_out, positions, num_gpu_batches, gpu_batch_size, scratch,
                         FG_NOALLOC_SCRATCH_BYTES, stream);
}
