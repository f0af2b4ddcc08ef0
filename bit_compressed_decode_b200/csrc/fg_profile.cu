// fg_profile.cu -- optional per-kernel timing of layer calls with CUDA events.
//
// While enabled, every kernel launched by fg_layer_decode / fg_layer_prefill is bracketed
// by CUDA events recorded on the launching stream (no synchronisation is added).
// fg_profile_collect synchronises on those events and returns the summed durations per
// kernel slot.  Events are created on demand (no device memory is allocated).
#include <mutex>
#include <vector>

#include "fg_internal.cuh"

namespace {

struct Record {
  int slot;
  cudaEvent_t start, stop;
};

std::mutex g_mu;
bool g_enabled = false;
std::vector<Record> g_records;
std::vector<cudaEvent_t> g_free;

cudaEvent_t take_event() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

bool fg_profile_on() { return g_enabled; }

// Returns a record index (or -1) after recording its start event on `st`.
int fg_profile_begin(int slot, cudaStream_t st) {
  if (!g_enabled) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  Record r{slot, take_event(), take_event()};
  if (!r.start || !r.stop || cudaEventRecord(r.start, st) != cudaSuccess) return -1;
  g_records.push_back(r);
  return static_cast<int>(g_records.size()) - 1;
}

void fg_profile_end(int idx, cudaStream_t st) {
  if (idx < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (idx < static_cast<int>(g_records.size())) cudaEventRecord(g_records[idx].stop, st);
}

extern "C" fg_status fg_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_enabled = enable != 0;
  return FG_OK;
}

extern "C" fg_status fg_profile_collect(float *ms, int *count, int nslots) {
  if (!ms || !count || nslots < 1) return FG_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int i = 0; i < nslots; i++) {
    ms[i] = 0.f;
    count[i] = 0;
  }
  fg_status rc = FG_OK;
  for (const Record &r : g_records) {
    float t = 0.f;
    if (rc == FG_OK) rc = fg_cuda_check(cudaEventSynchronize(r.stop));
    if (rc == FG_OK) rc = fg_cuda_check(cudaEventElapsedTime(&t, r.start, r.stop));
    if (rc == FG_OK && r.slot >= 0 && r.slot < nslots) {
      ms[r.slot] += t;
      count[r.slot] += 1;
    }
    g_free.push_back(r.start);
    g_free.push_back(r.stop);
  }
  g_records.clear();
  return rc;
}
