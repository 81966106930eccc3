// nc32_kernels.cuh — the non-causal form at head dimension 32 on the CUDA
// cores ("Linear Attention" knowledge-base page, section 3, non-causal sketch:
// S = phi(K)^T V, z = sum_j phi(k_j), out_i = phi(q_i)^T S / (phi(q_i)^T z + eps)).
//
// At d = 32 the per-token contraction is 32 x 32, too narrow for the
// tensor-core shapes (M >= 64) and small enough that the work is bound by
// memory traffic.  Both kernels give each lane of a warp one column of the
// 32 x 32 state, so that a whole row of phi(k) or phi(q) is one broadcast
// read of shared memory and 32 fused multiply-adds per lane.
#pragma once
#include "common.cuh"

namespace la {

constexpr int kNc32Warps = 8;
constexpr int kNc32Batch = 8;   // keys staged per warp per step

// Per-segment partial state over keys [s*seg_len, min(Lk, (s+1)*seg_len)).
// grid (n_seg, BH), 256 threads; writes ws_state[bh][seg] = (S, z) and
// ws_A[bh][seg] = 1 (no decay), the layout the segment scan consumes.
template <typename InT>
__global__ void __launch_bounds__(kNc32Warps * 32)
nc32_state_kernel(const InT *__restrict__ k, const InT *__restrict__ v, int Lk, int seg_len,
                  int n_seg, float *__restrict__ ws_state, float *__restrict__ ws_A) {
    __shared__ float fk[kNc32Warps][kNc32Batch][32];
    __shared__ float red[kNc32Warps][33][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg = blockIdx.x, bh = blockIdx.y;
    const long j0 = (long)seg * seg_len, j1 = min((long)Lk, j0 + seg_len);
    const InT *K = k + (size_t)bh * Lk * 32;
    const InT *V = v + (size_t)bh * Lk * 32;
    float S[32];   // column `lane` of this warp's partial state
#pragma unroll
    for (int a = 0; a < 32; ++a) S[a] = 0.f;
    float z = 0.f;  // z[lane]
    for (long jb = j0 + (long)warp * kNc32Batch; jb < j1; jb += (long)kNc32Warps * kNc32Batch) {
        float vb[kNc32Batch];
#pragma unroll
        for (int t = 0; t < kNc32Batch; ++t) {
            const long j = jb + t;
            float kf = 0.f, vf = 0.f;
            if (j < j1) {
                kf = phi_precise(to_f32(K[(size_t)j * 32 + lane]));
                vf = to_f32(V[(size_t)j * 32 + lane]);
            }
            fk[warp][t][lane] = kf;
            vb[t] = vf;
            z += kf;
        }
        __syncwarp();
#pragma unroll
        for (int t = 0; t < kNc32Batch; ++t) {
            const float4 *row = reinterpret_cast<const float4 *>(fk[warp][t]);
#pragma unroll
            for (int a4 = 0; a4 < 8; ++a4) {
                const float4 f = row[a4];
                S[4 * a4 + 0] = fmaf(f.x, vb[t], S[4 * a4 + 0]);
                S[4 * a4 + 1] = fmaf(f.y, vb[t], S[4 * a4 + 1]);
                S[4 * a4 + 2] = fmaf(f.z, vb[t], S[4 * a4 + 2]);
                S[4 * a4 + 3] = fmaf(f.w, vb[t], S[4 * a4 + 3]);
            }
        }
        __syncwarp();
    }
    // reduce the warps' partials (fixed order: deterministic)
#pragma unroll
    for (int a = 0; a < 32; ++a) red[warp][a][lane] = S[a];
    red[warp][32][lane] = z;
    __syncthreads();
    float *dst = ws_state + ((size_t)bh * n_seg + seg) * (32 * 32 + 32);
    for (int e = threadIdx.x; e < 33 * 32; e += kNc32Warps * 32) {
        const int a = e / 32, b = e % 32;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kNc32Warps; ++w) acc += red[w][a][b];
        dst[e] = acc;   // rows 0..31 are S[a][b]; row 32 is z[b]
    }
    if (threadIdx.x == 0) ws_A[(size_t)bh * n_seg + seg] = 1.f;
}

constexpr int kNc32Queries = 32 * kNc32Warps;   // queries per CTA (one 32-query block per warp)

// out_i = phi(q_i)^T S / (phi(q_i)^T z + eps) with the head's total (S, z).
// grid (ceil(Lq / 256), BH), 256 threads.
template <typename InT, typename OutT>
__global__ void __launch_bounds__(kNc32Warps * 32)
nc32_readout_kernel(const InT *__restrict__ q, int Lq, const float *__restrict__ total, float eps,
                    OutT *__restrict__ out) {
    __shared__ float fq[kNc32Warps][32][33];
    __shared__ float dens[kNc32Warps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const float *tot = total + (size_t)bh * (32 * 32 + 32);
    float Sc[32], zr[32];
#pragma unroll
    for (int a = 0; a < 32; ++a) {
        Sc[a] = tot[a * 32 + lane];   // column `lane` of S
        zr[a] = tot[32 * 32 + a];     // z (every lane)
    }
    const long i0 = (long)blockIdx.x * kNc32Queries + (long)warp * 32;
    if (i0 >= Lq) return;
    const InT *Q = q + (size_t)bh * Lq * 32;
    OutT *O = out + (size_t)bh * Lq * 32;
    const int nq = (int)min(32L, (long)Lq - i0);
    // stage phi(q) of the block's 32 queries (row i in fq[warp][i][.])
    for (int i = 0; i < 32; ++i)
        fq[warp][i][lane] = (i < nq) ? phi_precise(to_f32(Q[(size_t)(i0 + i) * 32 + lane])) : 0.f;
    __syncwarp();
    // lane i: denominator of query i
    {
        float d = 0.f;
#pragma unroll
        for (int a = 0; a < 32; ++a) d = fmaf(fq[warp][lane][a], zr[a], d);
        dens[warp][lane] = d + eps;
    }
    __syncwarp();
    // lane b: numerators of column b for the 32 queries
    for (int i = 0; i < nq; ++i) {
        float num = 0.f;
#pragma unroll
        for (int a = 0; a < 32; ++a) num = fmaf(fq[warp][i][a], Sc[a], num);
        O[(size_t)(i0 + i) * 32 + lane] = from_f32<OutT>(num / dens[warp][i]);
    }
}

}  // namespace la
