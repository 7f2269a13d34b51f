// Pieces of the C ABI's implementation that more than one source file uses.
#pragma once

#include <cuda_runtime.h>

#include <vector>

#include "../../include/cbv.h"
#include "plan.h"

namespace cbv {

// Sets the text cbv_last_error_message() returns.
void set_last_error(const char* msg);

// The tile schedules of one ring forward call and the workspace bytes they need.
struct RingFwdLayout {
  Plan fused;
  std::vector<Plan> steps;
  size_t bytes = 0;
};

// Checks a ring forward call's arguments (the status and message cbv_zigzag_ring_fwd would
// return) and plans it.  On success *L holds the schedule and its workspace size.
int ring_fwd_plan(const cbv_ring_args* a, RingFwdLayout* L);
// Runs a planned ring forward with `workspace` (at least L.bytes, 256-byte aligned) as scratch;
// a->workspace is not used.
// wait_limit_ns and withhold_loads are the forward kernel's diagnostics (FwdParams); 0 for a normal call.
int ring_fwd_run(const cbv_ring_args* a, const RingFwdLayout& L, void* workspace, cudaStream_t s,
                 uint64_t wait_limit_ns = 0, int withhold_loads = 0);

}  // namespace cbv
