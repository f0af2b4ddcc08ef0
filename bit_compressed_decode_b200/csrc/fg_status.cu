// fg_status.cu -- device error word, CUDA error mapping, fg_sync_status.
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "fg_internal.cuh"

// One error word per device (every device that loads the library holds its own
// copy of this variable).  Kernels atomicOr FG_DEVERR_* bits into it.
__device__ unsigned int fg_device_error_word;

static thread_local char g_last_cuda_error[256];

fg_status fg_cuda_check(cudaError_t e) {
  if (e == cudaSuccess) return FG_OK;
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return FG_ERR_CUDA;
}

fg_status fg_launch_check() { return fg_cuda_check(cudaGetLastError()); }

// Per-device cache of the error word's address.  Threads that race on a first call each look
// the address up (the same value) and store it; readers see either null or that value.
unsigned int *fg_error_word_ptr() {
  static std::atomic<unsigned int *> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  unsigned int *p = cache[dev].load(std::memory_order_acquire);
  if (!p) {
    void *q = nullptr;
    if (fg_cuda_check(cudaGetSymbolAddress(&q, fg_device_error_word)) != FG_OK) return nullptr;
    p = static_cast<unsigned int *>(q);
    cache[dev].store(p, std::memory_order_release);
  }
  return p;
}

extern "C" const char *fg_last_cuda_error(void) { return g_last_cuda_error; }

extern "C" const char *fg_status_string(fg_status s) {
  switch (s) {
    case FG_OK: return "FG_OK";
    case FG_ERR_INVALID: return "FG_ERR_INVALID";
    case FG_ERR_SHAPE: return "FG_ERR_SHAPE";
    case FG_ERR_UNSUPPORTED: return "FG_ERR_UNSUPPORTED";
    case FG_ERR_RANGE: return "FG_ERR_RANGE";
    case FG_ERR_CUDA: return "FG_ERR_CUDA";
    case FG_ERR_TIMEOUT: return "FG_ERR_TIMEOUT";
    case FG_ERR_WORKSPACE: return "FG_ERR_WORKSPACE";
  }
  return "FG_ERR_UNKNOWN";
}

int fg_sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load();
  if (!n) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n);
  }
  return n;
}

extern "C" fg_status fg_sync_status(void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fg_status rc = fg_cuda_check(cudaStreamSynchronize(st));
  if (rc != FG_OK) return rc;
  unsigned int *p = fg_error_word_ptr();
  if (!p) return FG_ERR_CUDA;
  unsigned int word = 0;
  rc = fg_cuda_check(cudaMemcpyFromSymbol(&word, fg_device_error_word, sizeof(word)));
  if (rc != FG_OK) return rc;
  if (word) {
    const unsigned int zero = 0;
    rc = fg_cuda_check(cudaMemcpyToSymbol(fg_device_error_word, &zero, sizeof(zero)));
    if (rc != FG_OK) return rc;
  }
  if (word & FG_DEVERR_TIMEOUT) return FG_ERR_TIMEOUT;
  if (word & FG_DEVERR_RANGE) return FG_ERR_RANGE;
  return FG_OK;
}
