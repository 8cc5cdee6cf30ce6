// pdl.cuh -- device side of programmatic dependent launch (the host side is
// launch_pdl in tw_internal.h).
#pragma once
#include "tw_common.cuh"

namespace tw {

// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialization attribute may be scheduled before the previous kernel
// on its stream has finished; pdl_wait blocks until that kernel has completed
// and its memory operations are visible (it returns at once for a kernel
// launched normally), so it comes before the kernel's first global access.
// pdl_launch_next lets the next such kernel be scheduled; that kernel still
// waits for this one's completion in its own pdl_wait.
TW_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
TW_DEV void pdl_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace tw
