// errors.h — per-thread record of the last CUDA failure behind LA_ERR_CUDA,
// readable through la_last_error_string().
#pragma once
#include <cuda_runtime.h>

#include "linattn.h"

namespace la {

// Records "where: <CUDA error text>" and returns LA_ERR_CUDA.
la_status cuda_fail(const char *where, cudaError_t e);
// Records a message (for non-runtime failures) and returns LA_ERR_CUDA.
la_status cuda_fail_msg(const char *where, const char *msg);
// LA_OK if e is cudaSuccess, else cuda_fail(where, e).
inline la_status cuda_check(const char *where, cudaError_t e) {
    return e == cudaSuccess ? LA_OK : cuda_fail(where, e);
}

// Records caller event i of `events` (an array of cudaEvent_t, or null) on st.
inline la_status record_event(void *const *events, int i, cudaStream_t st) {
    if (events == nullptr || events[i] == nullptr) return LA_OK;
    return cuda_check("event record", cudaEventRecord((cudaEvent_t)events[i], st));
}

}  // namespace la
