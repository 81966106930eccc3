// scan.h — host launcher of the segment scan (scan.cu).
#pragma once
#include <cuda_runtime.h>

#include "linattn.h"

namespace la {

void count_launches(int n);  // process-wide kernel launch counter (la_launch_count)

// Exclusive decayed prefix over the n_seg segment states of each of BH heads,
// in place in ws_state; state-in (mode INOUT) seeds the scan, the final state
// goes to state_S/state_z (mode OUT/INOUT) and to `total` when non-null.
la_status launch_segment_scan(float *ws_state, const float *ws_A, long BH, int n_seg, int D,
                              int mode, float *state_S, float *state_z, float *total,
                              cudaStream_t st, bool pdl = false);

}  // namespace la
