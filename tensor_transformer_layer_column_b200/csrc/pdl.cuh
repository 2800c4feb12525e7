// Device side of programmatic dependent launch (shared by the kernels).
#pragma once

namespace tp {

// Programmatic dependent launch.  A kernel launched by launch_pdl may be
// scheduled while the kernel before it on the stream is still finishing
// (once every CTA of that kernel has called grid_dep_launch or exited), so
// its launch and set-up overlap the tail of the previous one.  Every such
// kernel calls grid_dep_wait, in every thread, before its first access to
// global memory: the wait returns once the previous grid has completed and
// its writes are visible (immediately when launched without the attribute).
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace tp
