// Per-launch CUDA-event recorder behind ffn_nvfp4_profile_begin/_end.
#include <string.h>

#include <vector>

#include "ffn_nvfp4.h"
#include "profile.h"

namespace ffn {
namespace {

struct Mark {
  const char* name;
  cudaEvent_t start, stop;
};

struct Recorder {
  bool active = false;
  std::vector<Mark> marks;
  std::vector<cudaEvent_t> pool;  // events reused across recordings
  size_t used = 0;
  cudaEvent_t take() {
    if (used == pool.size()) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
      pool.push_back(e);
    }
    return pool[used++];
  }
};

thread_local Recorder rec;

}  // namespace

bool profiling() { return rec.active; }

// While the stream is being captured into a CUDA graph the events become
// event-record nodes of the graph, so they time each replay on the device.
static void prof_record(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else
    cudaEventRecord(e, s);
}

void prof_mark_start(cudaStream_t s, const char* name) {
  Mark m{name, rec.take(), rec.take()};
  if (m.start && m.stop) {
    prof_record(m.start, s);
    rec.marks.push_back(m);
  }
}

void prof_mark_stop(cudaStream_t s) {
  if (!rec.marks.empty()) prof_record(rec.marks.back().stop, s);
}

}  // namespace ffn

extern "C" {

ffn_status ffn_nvfp4_profile_begin(void) {
  ffn::rec.marks.clear();
  ffn::rec.used = 0;
  ffn::rec.active = true;
  return FFN_OK;
}

ffn_status ffn_nvfp4_profile_end(ffn_kernel_time* out, int capacity, int* count) {
  ffn::rec.active = false;
  if (!count || capacity < 0 || (capacity > 0 && !out)) return FFN_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return FFN_ERR_CUDA;
  }
  int n = 0;
  for (const auto& m : ffn::rec.marks) {
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, m.start, m.stop) != cudaSuccess) {
      cudaGetLastError();
      return FFN_ERR_CUDA;
    }
    int i = 0;
    while (i < n && strcmp(out[i].name, m.name) != 0) ++i;
    if (i == n) {
      if (n == capacity) return FFN_ERR_INVALID_ARG;
      out[n].name = m.name;
      out[n].launches = 0;
      out[n].total_ms = 0.0;
      ++n;
    }
    out[i].launches += 1;
    out[i].total_ms += ms;
  }
  *count = n;
  ffn::rec.marks.clear();
  ffn::rec.used = 0;
  return FFN_OK;
}

}  // extern "C"
