// pa_fallback.h -- the switch that makes two launchers take their fallback kernels.
#ifndef PA_FALLBACK_H_
#define PA_FALLBACK_H_

#include <stdlib.h>

namespace pa {

// PA_FALLBACK_KERNELS=1 in the environment makes the launchers take the kernels they
// fall back to when a kernel's build does not have the register count its setmaxnreg
// split assumes (the E4M3 shared-prefix decode on mma.sync, the chunked prefill on
// one 128-row tile per CTA), so that tests can run those paths.  Read at each call.
inline bool fallback_kernels_forced() {
  const char* e = getenv("PA_FALLBACK_KERNELS");
  return e != nullptr && e[0] == '1';
}

}  // namespace pa

#endif  // PA_FALLBACK_H_
