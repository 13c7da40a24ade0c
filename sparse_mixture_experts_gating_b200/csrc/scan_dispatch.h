// Scan and dispatch of the routing in one launch (routing.cu).
#pragma once

#include "internal.h"

namespace moe {

// True when every thread of the fused kernel sums at most a short run of the
// router's per-block histogram entries (few experts times router blocks).
bool scan_dispatch_fits(const RoutingArgs& a);

// Expert totals and offsets, slot ranks, the scan's tables and statistics, and
// the row copies into the expert-sorted buffer, for batches of more than one
// router block; replaces launch_scan + launch_dispatch.
cudaError_t launch_scan_dispatch(const RoutingArgs& a, cudaStream_t s);

}  // namespace moe
