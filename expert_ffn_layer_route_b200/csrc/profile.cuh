// Optional per-kernel device timing.  When enabled (moe_profile_enable), every
// kernel the library launches is bracketed by two CUDA events recorded on the
// stream it is launched on; moe_profile_collect waits for them and returns
// launches and total milliseconds per kernel name.
#pragma once

#include <cuda_runtime.h>

namespace moe {

bool profile_on();
// Record the start of `name` on `st`; returns a token for profile_end (or -1).
int profile_begin(const char* name, cudaStream_t st);
void profile_end(int token, cudaStream_t st);

struct ProfScope {
  int tok;
  cudaStream_t st;
  ProfScope(const char* name, cudaStream_t s) : tok(profile_on() ? profile_begin(name, s) : -1), st(s) {}
  ~ProfScope() {
    if (tok >= 0) profile_end(tok, st);
  }
};

}  // namespace moe
