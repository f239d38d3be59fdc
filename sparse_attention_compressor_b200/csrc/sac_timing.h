// Internal hooks of the optional per-kernel timer (see sac_timing_begin in include/sac.h).
#pragma once

#include <cuda_runtime.h>

namespace sac {

// Records a start event on `st` if timing is enabled; returns a slot (-1 when disabled) and the
// stop event to record after the launch.
int timer_start(const char* name, cudaStream_t st, cudaEvent_t* stop_out);
void timer_stop(int slot, cudaEvent_t stop, cudaStream_t st);

// Brackets one launch: `f()` issues the kernel on `st` and returns its launch status.
template <class F>
cudaError_t timed(const char* name, cudaStream_t st, F&& f) {
  cudaEvent_t stop = nullptr;
  int slot = timer_start(name, st, &stop);
  cudaError_t e = f();
  timer_stop(slot, stop, st);
  return e;
}

}  // namespace sac
