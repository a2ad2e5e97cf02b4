// Optional per-kernel timing with CUDA events (off by default). When enabled
// through kata_profile_enable, every kernel launch of the library is
// bracketed by two events recorded on its stream; kata_profile_get then
// reports launches and total device time per kernel name.
#pragma once

#include <cuda_runtime.h>

namespace kata {

bool profile_enabled();
// Records the start event; returns a ticket (or -1 when profiling is off).
int profile_begin(const char *name, cudaStream_t stream);
void profile_end(int ticket, cudaStream_t stream);

struct ProfileScope {
  int ticket;
  cudaStream_t stream;
  ProfileScope(const char *name, cudaStream_t s) : ticket(profile_begin(name, s)), stream(s) {}
  ~ProfileScope() { profile_end(ticket, stream); }
};

}  // namespace kata
