// tc_launch.h — host entry points of the tcgen05 (tensor-core) kernels.
#pragma once
#include <cuda_runtime.h>

#include "linattn.h"

namespace la {

struct TcCausalArgs {
    const void *q, *k, *v;
    const float *decay;
    const float *gain;     // per-token gain on the new term, or null
    int mlstm;             // identity feature map, max(|den|, 1) read-out
    int flash;             // the FLASH chunk form (identity map, relu(score / s)^2, no normaliser)
    float inv_s;           // FLASH: 1 / s
    bool summary;          // state pass + scan only: the total contribution to state_S/state_z (mode OUT)
    float *sum_A;          // summary: each head's decay product [BH]
    void *out;
    la_dtype in_dtype, out_dtype;
    float *ws_state, *ws_A;
    int *status;           // the call's status word [2] in the workspace (cleared by the caller)
    unsigned long long wait_ns;   // limit of every bounded device-side wait
    float *state_S, *state_z;
    la_state_mode mode;
    long BH;
    int T, D, chunk, seg_len, n_seg;
    float eps;
    void *const *events;   // 4 cudaEvent_t recorded around K1, K2, K3, or null
};

struct TcNoncausalArgs {
    const void *q, *k, *v;
    void *out;
    la_dtype in_dtype, out_dtype;
    float *ws_state, *ws_A, *ws_total;
    uint8_t *ws_bimg;             // d 32 tensor-core path: [BH][6144] the heads' read-out operand images
    int *status;                  // the call's status word [2] (cleared by the caller)
    unsigned long long wait_ns;
    float *state_S, *state_z;
    la_state_mode mode;
    long BH;
    int Lq, Lk, D, seg_len, n_seg;
    float eps;
};

void count_launches(int n);  // process-wide kernel launch counter (la_launch_count)

bool tc_supported(la_dtype in_dtype, int D, int chunk, bool has_decay);
bool tc_noncausal_supported(la_dtype in_dtype, int D);
la_status tc_causal(const TcCausalArgs &a, cudaStream_t st);
la_status tc_noncausal(const TcNoncausalArgs &a, cudaStream_t st);

}  // namespace la
