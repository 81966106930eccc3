// scan.h — host launcher of the segment scan (scan.cu).
#pragma once
#include <cuda_runtime.h>

#include "linattn.h"

namespace la {

void count_launches(int n);  // process-wide kernel launch counter (la_launch_count)

// Exclusive decayed prefix over the segment states of each of BH heads, in
// place in ws_state: afterwards segment s (s < n_seg) holds the state entering
// it.  Only the first n_dx segments (n_seg - 1 or n_seg) carry a contribution
// (dX_s, A_s); the last one has none when the output pass forms the final
// state itself.  State-in (mode INOUT) seeds the scan; when n_dx == n_seg the
// final state goes to state_S/state_z (mode OUT/INOUT) and to `total` when
// non-null.
// total_A (non-null): receives each head's product of the first n_dx segment
// factors.
la_status launch_segment_scan(float *ws_state, const float *ws_A, long BH, int n_seg, int n_dx, int D,
                              int mode, float *state_S, float *state_z, float *total,
                              cudaStream_t st, bool pdl = false, float *total_A = nullptr);

// Entry state of shard r of a sequence split over shards (see
// state_combine_kernel in scan.cu).
la_status launch_state_combine(const float *S_all, const float *z_all, const float *A_all, int r, long BH, int D,
                               const float *S_in, const float *z_in, float *S_out, float *z_out, cudaStream_t st);

}  // namespace la
