// Programmatic dependent launch for the memory-bound kernels (KV append,
// key rotation, hybrid state delta and scan), launched with programmatic
// stream serialisation: grid_dep_wait() returns once the grids this one
// depends on have completed and their writes are visible (at once for a
// plain launch); grid_dep_launch() then lets the next grid on the stream be
// scheduled while this one runs.  Each such kernel calls both first, before
// touching global memory.
#pragma once

namespace vattn {
namespace pdl {

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace pdl
}  // namespace vattn
