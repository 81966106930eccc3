// scan.cu — K2, the decayed exclusive prefix scan over segment states,
// shared by the CUDA-core and tensor-core paths.
#include "common.cuh"
#include "errors.h"
#include "scan.h"

namespace la {

// K2: decayed exclusive prefix scan over the segments of each head, in place
// (this form: many segments per head).
// Segment s maps X -> A_s X + dX_s; entering segment s the state is
//   S_in(s) = A_{s-1} S_in(s-1) + dX_{s-1},  S_in(0) = state-in or 0,
// and the final state is S_in(n_seg).  A block takes 32 state elements of one
// head; a 32-segment x 32-element tile is staged through shared memory so
// global accesses stay coalesced, and each warp scans one element across the
// 32 segments of the tile with shuffles (lanes = segments).  Segments from
// n_dx on contribute nothing (A = 1, dX = 0).
// grid (ceil((D*D + D) / 32), BH), 256 threads.
__global__ void __launch_bounds__(256) segment_scan_kernel(float *ws_state, const float *ws_A,
                                                           int n_seg, int n_dx, int E, int dS,
                                                           const float *state_in_S,
                                                           const float *state_in_z,
                                                           float *state_out_S, float *state_out_z,
                                                           float *total, float *total_A) {
    __shared__ float tile[32][33];
    __shared__ float Atile[32];
    pdl_wait();   // the segment states of the state pass
    const int bh = blockIdx.y, e0 = blockIdx.x * 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *ws = ws_state + (size_t)bh * n_seg * E;
    const float *Ah = ws_A + (size_t)bh * n_seg;

    // carries of this warp's four elements (e0 + warp + 8 m), replicated in all lanes
    float carry[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int e = e0 + warp + 8 * m;
        float c = 0.f;
        if (e < E) {
            if (e < dS) { if (state_in_S) c = state_in_S[(size_t)bh * dS + e]; }
            else if (state_in_z) c = state_in_z[(size_t)bh * (E - dS) + (e - dS)];
        }
        carry[m] = c;
    }
    for (int s0 = 0; s0 < n_seg; s0 += 32) {
        __syncthreads();
        for (int i = warp; i < 32; i += 8) {
            const int s = s0 + i, e = e0 + lane;
            tile[i][lane] = (s < n_dx && e < E) ? ws[(size_t)s * E + e] : 0.f;
        }
        if (tid < 32) Atile[tid] = (s0 + tid < n_dx) ? Ah[s0 + tid] : 1.f;
        __syncthreads();
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int el = warp + 8 * m;
            float a = Atile[lane], x = tile[lane][el];
            warp_affine_scan(a, x, lane);
            float pa = __shfl_up_sync(0xffffffffu, a, 1);
            float px = __shfl_up_sync(0xffffffffu, x, 1);
            if (lane == 0) { pa = 1.f; px = 0.f; }
            tile[lane][el] = fmaf(pa, carry[m], px);
            const float a31 = __shfl_sync(0xffffffffu, a, 31);
            const float x31 = __shfl_sync(0xffffffffu, x, 31);
            carry[m] = fmaf(a31, carry[m], x31);
        }
        __syncthreads();
        for (int i = warp; i < 32; i += 8) {
            const int s = s0 + i, e = e0 + lane;
            if (s < n_seg && e < E) ws[(size_t)s * E + e] = tile[i][lane];
        }
    }
    if (total_A && blockIdx.x == 0 && threadIdx.x == 0) {   // the head's total decay product
        float A = 1.f;
        for (int i = 0; i < n_dx; ++i) A *= Ah[i];
        total_A[bh] = A;
    }
    if (lane == 0 && n_dx == n_seg) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int e = e0 + warp + 8 * m;
            if (e >= E) continue;
            if (total) total[(size_t)bh * E + e] = carry[m];
            if (e < dS) { if (state_out_S) state_out_S[(size_t)bh * dS + e] = carry[m]; }
            else if (state_out_z) state_out_z[(size_t)bh * (E - dS) + (e - dS)] = carry[m];
        }
    }
    pdl_trigger();
}


// K2 for few segments per head (the common case): one thread per four
// consecutive state elements walks the head's segments in order.  Its loads
// for the first eight segments are issued before the block waits for the
// segment factors A_s (staged in shared memory), so both latencies overlap,
// and a grid of 16-byte accesses fits in one wave at the usual head counts.
// E (= D*D + D) and D*D are multiples of 4 for every supported head dim, and
// the workspace and state pointers are 16-byte aligned.
// grid (ceil(E / 1024), BH), 256 threads.
constexpr int kSeqScanMaxSeg = 64;
constexpr int kSeqScanBatch = 8;
__device__ __forceinline__ float4 fma4(float a, const float4 &c, const float4 &x) {
    return make_float4(fmaf(a, c.x, x.x), fmaf(a, c.y, x.y), fmaf(a, c.z, x.z), fmaf(a, c.w, x.w));
}
__global__ void __launch_bounds__(256) segment_scan_seq_kernel(float *ws_state, const float *ws_A,
                                                               int n_seg, int n_dx, int E, int dS,
                                                               const float *state_in_S,
                                                               const float *state_in_z,
                                                               float *state_out_S, float *state_out_z,
                                                               float *total, float *total_A) {
    __shared__ float Ash[kSeqScanMaxSeg];
    pdl_wait();   // the segment states of the state pass
    const int bh = blockIdx.y;
    const int e = (blockIdx.x * 256 + threadIdx.x) * 4;
    const bool live = e < E;
    float4 *ws = reinterpret_cast<float4 *>(ws_state + (size_t)bh * n_seg * E + (live ? e : 0));
    const size_t E4 = (size_t)E / 4;   // segment stride in float4
    float4 x[kSeqScanBatch];
#pragma unroll
    for (int i = 0; i < kSeqScanBatch; ++i)
        x[i] = (live && i < n_dx) ? ws[i * E4] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 carry = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live) {
        if (e < dS) { if (state_in_S) carry = *reinterpret_cast<const float4 *>(state_in_S + (size_t)bh * dS + e); }
        else if (state_in_z) carry = *reinterpret_cast<const float4 *>(state_in_z + (size_t)bh * (E - dS) + (e - dS));
    }
    if (threadIdx.x < n_dx) Ash[threadIdx.x] = ws_A[(size_t)bh * n_seg + threadIdx.x];
    __syncthreads();
    if (total_A && blockIdx.x == 0 && threadIdx.x == 0) {   // the head's total decay product
        float A = 1.f;
        for (int i = 0; i < n_dx; ++i) A *= Ash[i];
        total_A[bh] = A;
    }
    if (!live) return;
#pragma unroll 1
    for (int s0 = 0; s0 < n_seg; s0 += kSeqScanBatch) {
        if (s0 > 0) {
#pragma unroll
            for (int i = 0; i < kSeqScanBatch; ++i)
                if (s0 + i < n_dx) x[i] = ws[(size_t)(s0 + i) * E4];
        }
#pragma unroll
        for (int i = 0; i < kSeqScanBatch; ++i) {
            if (s0 + i < n_seg) {
                ws[(size_t)(s0 + i) * E4] = carry;   // state entering segment s0 + i
                if (s0 + i < n_dx) carry = fma4(Ash[s0 + i], carry, x[i]);
            }
        }
    }
    if (n_dx != n_seg) {   // the output pass forms the final state
        pdl_trigger();
        return;
    }
    if (total) *reinterpret_cast<float4 *>(total + (size_t)bh * E + e) = carry;
    if (e < dS) { if (state_out_S) *reinterpret_cast<float4 *>(state_out_S + (size_t)bh * dS + e) = carry; }
    else if (state_out_z) *reinterpret_cast<float4 *>(state_out_z + (size_t)bh * (E - dS) + (e - dS)) = carry;
    pdl_trigger();
}

la_status launch_segment_scan(float *ws_state, const float *ws_A, long BH, int n_seg, int n_dx, int D,
                              int mode, float *state_S, float *state_z, float *total,
                              cudaStream_t st, bool pdl, float *total_A) {
    const int E = D * D + D;
    const float *sin_S = mode == LA_STATE_INOUT ? state_S : nullptr;
    const float *sin_z = mode == LA_STATE_INOUT ? state_z : nullptr;
    float *sout_S = mode != LA_STATE_NONE ? state_S : nullptr;
    float *sout_z = mode != LA_STATE_NONE ? state_z : nullptr;
    // with pdl, the scan may start launching while the state pass finishes
    // (it waits for that pass's results before reading them)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t err;
    if (n_seg <= kSeqScanMaxSeg && E % 4 == 0 && D % 4 == 0) {   // float4 groups stay inside S or z
        cfg.gridDim = dim3((E / 4 + 255) / 256, (unsigned)BH);
        err = cudaLaunchKernelEx(&cfg, segment_scan_seq_kernel, ws_state, ws_A, n_seg, n_dx, E, D * D, sin_S, sin_z,
                                 sout_S, sout_z, total, total_A);
    } else {
        cfg.gridDim = dim3((E + 31) / 32, (unsigned)BH);
        err = cudaLaunchKernelEx(&cfg, segment_scan_kernel, ws_state, ws_A, n_seg, n_dx, E, D * D, sin_S, sin_z,
                                 sout_S, sout_z, total, total_A);
    }
    count_launches(1);
    if (err != cudaSuccess) return cuda_fail("segment_scan launch", err);
    return cuda_check("segment_scan launch", cudaGetLastError());
}

// Entry state of shard r of a sequence split over R shards (in order): the
// shards' summaries (dS_i, dz_i, A_i) fold as X_{i+1} = A_i X_i + dX_i from
// X_0 = state-in (or 0); shard r starts from X_r.  One thread per element of
// a head's state; layouts [R][BH][D*D] (S), [R][BH][D] (z), [R][BH] (A).
__global__ void __launch_bounds__(256) state_combine_kernel(const float *S_all, const float *z_all,
                                                            const float *A_all, int r, long BH, int D,
                                                            const float *S_in, const float *z_in, float *S_out,
                                                            float *z_out) {
    const int E = D * D + D;
    const long bh = blockIdx.y;
    const int e = blockIdx.x * 256 + threadIdx.x;
    if (e >= E) return;
    const bool isS = e < D * D;
    const int ez = e - D * D;
    float x = 0.f;
    if (isS) { if (S_in) x = S_in[bh * D * D + e]; }
    else if (z_in) x = z_in[bh * D + ez];
    for (int i = 0; i < r; ++i) {
        const float dx = isS ? S_all[((size_t)i * BH + bh) * D * D + e] : z_all[((size_t)i * BH + bh) * D + ez];
        x = fmaf(A_all[(size_t)i * BH + bh], x, dx);
    }
    if (isS) S_out[bh * D * D + e] = x;
    else z_out[bh * D + ez] = x;
}

la_status launch_state_combine(const float *S_all, const float *z_all, const float *A_all, int r, long BH, int D,
                               const float *S_in, const float *z_in, float *S_out, float *z_out, cudaStream_t st) {
    const int E = D * D + D;
    state_combine_kernel<<<dim3((E + 255) / 256, (unsigned)BH), 256, 0, st>>>(S_all, z_all, A_all, r, BH, D, S_in,
                                                                               z_in, S_out, z_out);
    count_launches(1);
    return cuda_check("state_combine launch", cudaGetLastError());
}

}  // namespace la
