// Opt-in per-launch timing: while a recording is open on the calling thread,
// every kernel launch the library makes is bracketed by a pair of CUDA events
// on its stream (ffn_nvfp4_profile_begin / _end in the C ABI).
#pragma once

#include <cuda_runtime.h>

namespace ffn {

bool profiling();
void prof_mark_start(cudaStream_t s, const char* name);
void prof_mark_stop(cudaStream_t s);

struct ProfScope {
  cudaStream_t s;
  bool on;
  ProfScope(cudaStream_t st, const char* name) : s(st), on(profiling()) {
    if (on) prof_mark_start(s, name);
  }
  ~ProfScope() {
    if (on) prof_mark_stop(s);
  }
};

}  // namespace ffn
