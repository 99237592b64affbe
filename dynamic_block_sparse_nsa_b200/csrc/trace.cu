// Kernel trace: optional CUDA-event brackets around every launch, so a caller
// can read per-kernel device time of a multi-kernel call (used by the
// benchmark to time the dominant kernel inside the timed region).
#include <vector>

#include "internal.h"

namespace nsa {
namespace {

struct Rec {
  const char* name;
  cudaEvent_t start, stop;
};

std::vector<Rec> g_recs;
int g_count = 0;
bool g_on = false;

void destroy_all() {
  for (Rec& r : g_recs) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  g_recs.clear();
}

}  // namespace

void trace_begin(const char* name, cudaStream_t stream) {
  if (!g_on) return;
  if (g_count < (int)g_recs.size()) {
    g_recs[g_count].name = name;
    cudaEventRecord(g_recs[g_count].start, stream);
  }
}

void trace_end(cudaStream_t stream) {
  if (!g_on) return;
  if (g_count < (int)g_recs.size()) cudaEventRecord(g_recs[g_count].stop, stream);
  ++g_count;
}

}  // namespace nsa

using namespace nsa;

extern "C" {

nsa_status nsa_trace_enable(int on, int capacity) {
  g_on = false;
  g_count = 0;
  destroy_all();
  if (!on) return NSA_OK;
  if (capacity < 0) return NSA_ERR_INVALID_ARGUMENT;
  g_recs.resize(capacity);
  for (Rec& r : g_recs) {
    r.name = "";
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) {
      g_recs.clear();
      return NSA_ERR_CUDA;
    }
  }
  g_on = true;
  return NSA_OK;
}

int nsa_trace_count(void) { return g_count; }

nsa_status nsa_trace_get(int i, const char** name, float* ms) {
  if (i < 0 || i >= g_count || i >= (int)g_recs.size() || !name || !ms)
    return NSA_ERR_INVALID_ARGUMENT;
  if (cudaEventSynchronize(g_recs[i].stop) != cudaSuccess) return NSA_ERR_CUDA;
  *name = g_recs[i].name;
  return cudaEventElapsedTime(ms, g_recs[i].start, g_recs[i].stop) == cudaSuccess ? NSA_OK
                                                                                 : NSA_ERR_CUDA;
}

}  // extern "C"
