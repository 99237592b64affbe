// Kernel trace: optional CUDA-event brackets around every launch, so a caller
// can read per-kernel device time of a multi-kernel call (used by the
// benchmark to time the dominant kernel inside the timed region).
#include <cstring>
#include <string>
#include <vector>

#include "internal.h"

namespace nsa {
namespace {

struct Rec {
  const char* name;
  cudaEvent_t start, stop;
};

std::vector<Rec> g_recs;
int g_count = 0;   // launches seen
int g_timed = 0;   // launches bracketed
bool g_on = false;
bool g_cur = false;  // the launch in progress is being timed
std::string g_filter;

void destroy_all() {
  for (Rec& r : g_recs) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  g_recs.clear();
}

}  // namespace

// During stream capture the events become event-record nodes of the graph
// (external records), so a replayed graph is timed kernel by kernel too.
static void record(cudaEvent_t e, cudaStream_t stream) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(stream, &st);
  if (st == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, stream, cudaEventRecordExternal);
  else
    cudaEventRecord(e, stream);
}

void trace_begin(const char* name, cudaStream_t stream) {
  g_cur = false;
  if (!g_on) return;
  if (!g_filter.empty() && std::strncmp(name, g_filter.c_str(), g_filter.size()) != 0) return;
  if (g_timed < (int)g_recs.size()) {
    g_recs[g_timed].name = name;
    record(g_recs[g_timed].start, stream);
    g_cur = true;
  }
}

void trace_end(cudaStream_t stream) {
  if (!g_on) return;
  if (g_cur) {
    record(g_recs[g_timed].stop, stream);
    ++g_timed;
    g_cur = false;
  }
  ++g_count;
}

}  // namespace nsa

using namespace nsa;

extern "C" {

nsa_status nsa_trace_set_filter(const char* prefix) {
  g_filter = prefix ? prefix : "";
  return NSA_OK;
}

nsa_status nsa_trace_enable(int on, int capacity) {
  g_on = false;
  g_count = 0;
  g_timed = 0;
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

int nsa_trace_timed(void) { return g_timed; }

nsa_status nsa_trace_get(int i, const char** name, float* ms) {
  if (i < 0 || i >= g_timed || i >= (int)g_recs.size() || !name || !ms)
    return NSA_ERR_INVALID_ARGUMENT;
  if (cudaEventSynchronize(g_recs[i].stop) != cudaSuccess) return NSA_ERR_CUDA;
  *name = g_recs[i].name;
  return cudaEventElapsedTime(ms, g_recs[i].start, g_recs[i].stop) == cudaSuccess ? NSA_OK
                                                                                 : NSA_ERR_CUDA;
}

}  // extern "C"
