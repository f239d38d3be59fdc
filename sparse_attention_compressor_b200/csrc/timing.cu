// Optional per-kernel timing: while enabled, every kernel launch of the library is bracketed by a
// pair of CUDA events recorded on the launch's own stream; sac_timing_end() waits for them and
// returns launches and total device time per kernel name. Launches captured into a CUDA graph
// carry their events into the graph, and sac_timing_end() then reports the graph's latest replay.
#include <mutex>
#include <string>
#include <vector>

#include "sac.h"
#include "sac_timing.h"

namespace sac {
namespace {

struct Pending {
  int slot;
  cudaEvent_t start, stop;
};

struct TimerState {
  std::mutex mu;
  bool on = false;
  std::vector<std::string> names;
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> free_events;
};

TimerState& state() {
  static TimerState s;
  return s;
}

cudaEvent_t take_event(TimerState& s) {
  if (!s.free_events.empty()) {
    cudaEvent_t e = s.free_events.back();
    s.free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Inside a CUDA-graph capture an ordinary event record only marks a dependency; an external
// record becomes an event node of the graph, timestamped on every replay.
void record(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  else
    cudaEventRecord(e, st);
}

}  // namespace

int timer_start(const char* name, cudaStream_t st, cudaEvent_t* stop_out) {
  TimerState& s = state();
  std::lock_guard<std::mutex> lk(s.mu);
  if (!s.on) return -1;
  int slot = -1;
  for (size_t i = 0; i < s.names.size(); ++i)
    if (s.names[i] == name) slot = (int)i;
  if (slot < 0) {
    s.names.emplace_back(name);
    slot = (int)s.names.size() - 1;
  }
  Pending p{slot, take_event(s), take_event(s)};
  record(p.start, st);
  *stop_out = p.stop;
  s.pending.push_back(p);
  return slot;
}

void timer_stop(int slot, cudaEvent_t stop, cudaStream_t st) {
  if (slot < 0) return;
  record(stop, st);
}

}  // namespace sac

extern "C" {

int sac_timing_begin(void) {
  sac::TimerState& s = sac::state();
  std::lock_guard<std::mutex> lk(s.mu);
  for (auto& p : s.pending) {
    s.free_events.push_back(p.start);
    s.free_events.push_back(p.stop);
  }
  s.pending.clear();
  s.names.clear();
  s.on = true;
  return SAC_OK;
}

int sac_timing_end(sac_kernel_time* out, int max_entries) {
  sac::TimerState& s = sac::state();
  std::lock_guard<std::mutex> lk(s.mu);
  s.on = false;
  std::vector<double> ms(s.names.size(), 0.0);
  std::vector<int> n(s.names.size(), 0);
  for (auto& p : s.pending) {
    float t = 0.f;
    if (cudaEventSynchronize(p.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, p.start, p.stop) != cudaSuccess)
      return SAC_ERR_LAUNCH;
    ms[p.slot] += t;
    n[p.slot] += 1;
    s.free_events.push_back(p.start);
    s.free_events.push_back(p.stop);
  }
  s.pending.clear();
  int count = (int)s.names.size();
  for (int i = 0; i < count && i < max_entries; ++i) {
    std::snprintf(out[i].name, sizeof(out[i].name), "%s", s.names[i].c_str());
    out[i].launches = n[i];
    out[i].total_ms = ms[i];
  }
  return count;
}

}  // extern "C"
