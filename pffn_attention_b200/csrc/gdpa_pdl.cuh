// gdpa_pdl.cuh -- programmatic dependent launch between the schedule kernel
// and the attention kernel that reads its results.
#pragma once

namespace gdpa {

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the kernel before it in the stream still
// runs; griddep_wait() returns once that kernel has completed and its memory
// writes are visible (a no-op for a kernel launched the ordinary way).
// griddep_launch_dependents() lets the next such kernel start early.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace gdpa
