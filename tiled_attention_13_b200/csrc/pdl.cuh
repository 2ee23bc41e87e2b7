// pdl.cuh -- programmatic dependent launch on sm_100.
//
// A kernel launched with programmatic stream serialization may start while
// the previous kernel in the stream is still running.  pdl_wait() blocks
// until that kernel has completed and its writes are visible; every thread
// calls it before its first global access of data another kernel may touch.
// pdl_launch_dependents() lets the next such kernel launch early (its CTAs
// take SMs as this grid's CTAs exit and wait in pdl_wait()).  Without the
// launch attribute both are no-ops in effect.
#pragma once

namespace fa {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace fa
