// Per-kernel CUDA-event timing registry (see profile.h). Single-threaded use:
// enable, run, read, from one host thread.
#include "../../include/kata.h"
#include "profile.h"

#include <string.h>

#include <mutex>
#include <vector>

namespace kata {
namespace {

constexpr int kMaxKernels = 32;
constexpr int kMaxPending = 1 << 14;

struct Slot {
  const char *name;
  long long launches;
  double total_ms;
};

struct Pending {
  int slot;
  cudaEvent_t start, end;
};

struct Registry {
  std::mutex mu;
  bool enabled = false;
  Slot slots[kMaxKernels];
  int n_slots = 0;
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> free_events;
  bool overflow = false;

  cudaEvent_t get_event() {
    if (!free_events.empty()) {
      cudaEvent_t e = free_events.back();
      free_events.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }

  int slot_of(const char *name) {
    for (int i = 0; i < n_slots; ++i)
      if (strcmp(slots[i].name, name) == 0) return i;
    if (n_slots == kMaxKernels) return -1;
    slots[n_slots] = Slot{name, 0, 0.0};
    return n_slots++;
  }

  // Waits for and folds every pending pair into the totals.
  bool drain() {
    bool ok = true;
    for (auto &p : pending) {
      float ms = 0.f;
      if (cudaEventSynchronize(p.end) != cudaSuccess ||
          cudaEventElapsedTime(&ms, p.start, p.end) != cudaSuccess) {
        ok = false;
      } else {
        slots[p.slot].launches += 1;
        slots[p.slot].total_ms += ms;
      }
      free_events.push_back(p.start);
      free_events.push_back(p.end);
    }
    pending.clear();
    return ok;
  }
};

Registry &reg() {
  static Registry r;
  return r;
}

}  // namespace

bool profile_enabled() { return reg().enabled; }

int profile_begin(const char *name, cudaStream_t stream) {
  Registry &r = reg();
  if (!r.enabled) return -1;
  std::lock_guard<std::mutex> lk(r.mu);
  if ((int)r.pending.size() >= kMaxPending) r.drain();
  const int slot = r.slot_of(name);
  if (slot < 0) {
    r.overflow = true;
    return -1;
  }
  Pending p{slot, r.get_event(), r.get_event()};
  if (!p.start || !p.end || cudaEventRecord(p.start, stream) != cudaSuccess) {
    r.overflow = true;
    return -1;
  }
  r.pending.push_back(p);
  return (int)r.pending.size() - 1;
}

void profile_end(int ticket, cudaStream_t stream) {
  if (ticket < 0) return;
  Registry &r = reg();
  std::lock_guard<std::mutex> lk(r.mu);
  if (ticket < (int)r.pending.size()) cudaEventRecord(r.pending[ticket].end, stream);
}

}  // namespace kata

using namespace kata;

extern "C" {

kata_status_t kata_profile_enable(int enable) {
  Registry &r = reg();
  std::lock_guard<std::mutex> lk(r.mu);
  bool ok = r.drain();
  r.n_slots = 0;
  r.overflow = false;
  r.enabled = enable != 0;
  return ok ? KATA_OK : KATA_ERR_CUDA;
}

int kata_profile_count(void) {
  Registry &r = reg();
  std::lock_guard<std::mutex> lk(r.mu);
  r.drain();
  return r.n_slots;
}

kata_status_t kata_profile_get(int index, const char **name, long long *launches,
                               double *total_ms) {
  Registry &r = reg();
  std::lock_guard<std::mutex> lk(r.mu);
  if (!r.drain()) return KATA_ERR_CUDA;
  if (index < 0 || index >= r.n_slots || !name || !launches || !total_ms)
    return KATA_ERR_INVALID_ARGUMENT;
  *name = r.slots[index].name;
  *launches = r.slots[index].launches;
  *total_ms = r.slots[index].total_ms;
  return KATA_OK;
}

}  // extern "C"
