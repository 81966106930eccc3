// noalloc.cu — la_prefill_causal_noalloc: the causal prefill for callers that
// cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: a plugin hosted by another
// runtime that owns all device memory, or a process that forbids allocation
// after start-up (a fixed-budget server, a real-time deployment).  For them
// this entry point runs the same prefill kernels with their scratch (the
// per-segment states joined by the prefix scan) placed in a fixed array in the
// library's own device memory instead of a caller-provided workspace.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds LA_NOALLOC_SCRATCH_BYTES of it until the process exits.  Host
// code cannot use the variable's name as a device address (on the host it is
// only a stand-in symbol), so each call looks the device address up with
// cudaGetSymbolAddress, with the call's device current.  The lookup allocates
// nothing; repeating it on every call keeps the address right if the caller
// has torn down and recreated the device's primary context in between.
#include "linattn.h"
#include <cuda_runtime.h>

static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array on the current device, or nullptr if
// the lookup fails.
void *scratch_for_current_device() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    return p;
}

}  // namespace

extern "C" la_status la_prefill_causal_noalloc(const void *q, const void *k, const void *v,
                                               la_dtype in_dtype, const float *decay, int B,
                                               int H, int T, int d_k, int d_v, float eps,
                                               int chunk, float *state_S, float *state_z,
                                               la_state_mode mode, void *out, la_dtype out_dtype,
                                               void *stream) {
    if (B > 0 && H > 0 && T > 0 &&
        la_prefill_workspace_size(B, H, T, d_k, d_v, chunk) > (size_t)LA_NOALLOC_SCRATCH_BYTES)
        return LA_ERR_UNSUPPORTED;
    void *scratch = scratch_for_current_device();
    if (!scratch) return LA_ERR_CUDA;   // device address lookup failed
    return la_prefill_causal(q, k, v, in_dtype, decay, B, H, T, d_k, d_v, eps, chunk, state_S,
                             state_z, mode, out, out_dtype, scratch,
                             (size_t)LA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" la_status la_noalloc_status(int *waiter, void *stream) {
    void *scratch = scratch_for_current_device();
    if (!scratch) return LA_ERR_CUDA;
    return la_workspace_status(scratch, waiter, stream);
}
