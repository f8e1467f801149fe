// launch_dep.cuh -- programmatic dependent launch (sm_90 and later) for the
// kernels that follow another kernel of the same call on a stream.
#pragma once

namespace fa {

// Programmatic dependent launch: the grid launched after this one with
// programmatic stream serialisation may start once every CTA of this grid
// has executed launch_dependents (or exited); it must wait (grid_dep_wait)
// before reading anything this grid writes.  Both are no-ops for a grid
// launched without that attribute.
__device__ __forceinline__ void grid_dep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace fa
