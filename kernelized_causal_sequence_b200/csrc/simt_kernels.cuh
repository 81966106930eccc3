// simt_kernels.cuh — CUDA-core (fp32 FMA) kernels of the chunked causal form,
// the non-causal read-out and the segment scan.
//
// These carry the fp32-input path, whose 1e-4 parity target rules out the
// tf32 tensor-core format (10-bit mantissa).  They implement the same
// segment / chunk decomposition as the tensor-core kernels:
//
//   tokens of one head = segments of `seg_len` tokens = chunks of `chunk` tokens
//   K1 segment_state : per segment, dS = sum_j w_j phi(k_j) v_j^T,
//                      dz = sum_j w_j phi(k_j), A = prod a over the segment,
//                      w_j = prod_{l>j, l in segment} a_l
//   K2 segment_scan  : exclusive decayed prefix over segments (see
//                      segment_scan_kernel), plus the final state
//   K3 chunk_output  : per segment, walk the chunks with the carried (S, z):
//                      exact masked products inside the chunk plus the
//                      decayed inter-chunk term, then the state update.
//
// The decay is handled in log space inside a chunk: L_j = sum_{l<=j} log a_l
// (chunk-local, inclusive), so every weight is exp(L_i - L_j) <= 1 with a
// non-positive exponent (no overflow for any a in (0, 1]).
#pragma once
#include "common.cuh"

namespace la {

struct SimtParams {
    const void *q, *k, *v;
    const float *decay;     // [BH, T] or nullptr
    const float *gain;      // [BH, T] or nullptr: gain b_t on token t's new term (causal only)
    int mlstm;              // causal only: identity feature map, read-out / max(|den|, 1)
    void *out;
    float *ws_state;        // [BH, n_seg, D*D + D]
    float *ws_A;            // [BH, n_seg]
    float *ws_total;        // [BH, D*D + D] (non-causal) or nullptr
    float *state_S, *state_z;
    int mode;               // la_state_mode
    int BH, T, Lq, chunk, seg_len, n_seg;
    float eps;
    void *const *events;    // host only: 4 cudaEvent_t recorded around K1, K2, K3, or null
    float *sum_A;           // host only: shard summary (no output pass), each head's decay product
};

constexpr int kSimtThreads = 256;
constexpr int kSub = 32;

// This thread's elements of rows [r0, r0 + kSub) of a [*, D] matrix (rows at
// or beyond r0 + rn read as 0), converted to fp32.  The loads are all issued
// before any is used, so a tile costs one memory round trip.
constexpr int simt_per_thread(int D) { return kSub * D / kSimtThreads; }
template <typename InT, int D>
__device__ __forceinline__ void simt_load_rows(const InT *base, long r0, int rn,
                                               float (&x)[simt_per_thread(D)]) {
#pragma unroll
    for (int u = 0; u < simt_per_thread(D); ++u) {
        const int idx = threadIdx.x + u * kSimtThreads, j = idx / D, a = idx % D;
        x[u] = (j < rn) ? to_f32(base[(size_t)(r0 + j) * D + a]) : 0.f;
    }
}

// Chunk-local inclusive cumulative sum of log a (warp 0 only).
__device__ __forceinline__ void chunk_log_cumsum(const float *a, int n, float *Lc) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        float carry = 0.f;
        for (int j0 = 0; j0 < n; j0 += 32) {
            const int j = j0 + lane;
            float x = (j < n) ? logf(a[j]) : 0.f;
            x = warp_sum_scan(x, lane) + carry;
            if (j < n) Lc[j] = x;
            carry = __shfl_sync(0xffffffffu, x, 31);
        }
    }
}

template <int D> __host__ __device__ constexpr size_t simt_state_smem() {
    return sizeof(float) * (2 * kSub * D + 128);
}

// K1: per-segment state contribution.  grid (n_seg, BH), 256 threads.
template <typename InT, int D>
__global__ void __launch_bounds__(kSimtThreads) simt_segment_state_kernel(SimtParams p, int T_keys) {
    constexpr int TR = D / 16;
    extern __shared__ float smem[];
    float *fk = smem;              // [kSub][D]
    float *vv = fk + kSub * D;     // [kSub][D]
    float *Lc = vv + kSub * D;     // [128]
    const int seg = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    const long t_begin = (long)seg * p.seg_len;
    const long t_end = min((long)T_keys, t_begin + p.seg_len);
    const InT *K = (const InT *)p.k + (size_t)bh * T_keys * D;
    const InT *V = (const InT *)p.v + (size_t)bh * T_keys * D;
    const float *A = p.decay ? p.decay + (size_t)bh * T_keys : nullptr;
    const float *Gk = p.gain ? p.gain + (size_t)bh * T_keys : nullptr;   // per-token gains

    float acc[TR][TR];
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
        for (int c = 0; c < TR; ++c) acc[r][c] = 0.f;
    float zacc = 0.f, Aseg = 1.f;

    for (long c0 = t_begin; c0 < t_end; c0 += p.chunk) {
        const int n = (int)min((long)p.chunk, t_end - c0);
        float Lend = 0.f;
        if (A) {
            __syncthreads();
            chunk_log_cumsum(A + c0, n, Lc);
            __syncthreads();
            Lend = Lc[n - 1];
            const float g = expf(Lend);
#pragma unroll
            for (int r = 0; r < TR; ++r)
#pragma unroll
                for (int c = 0; c < TR; ++c) acc[r][c] *= g;
            zacc *= g;
            Aseg *= g;
        }
        for (int j0 = 0; j0 < n; j0 += kSub) {
            {
                float kx[simt_per_thread(D)], vx[simt_per_thread(D)];
                simt_load_rows<InT, D>(K, c0 + j0, n - j0, kx);
                simt_load_rows<InT, D>(V, c0 + j0, n - j0, vx);
#pragma unroll
                for (int u = 0; u < simt_per_thread(D); ++u) {
                    const int idx = tid + u * kSimtThreads, j = idx / D;
                    float f = 0.f;
                    if (j0 + j < n) {
                        f = p.mlstm ? kx[u] : phi_precise(kx[u]);
                        if (A) f *= expf(Lend - Lc[j0 + j]);
                        if (Gk) f *= Gk[c0 + j0 + j];
                    }
                    fk[idx] = f;
                    vv[idx] = vx[u];
                }
            }
            __syncthreads();
            for (int j = 0; j < kSub; ++j) {
                float ar[TR], bc[TR];
#pragma unroll
                for (int r = 0; r < TR; ++r) ar[r] = fk[j * D + ty * TR + r];
#pragma unroll
                for (int c = 0; c < TR; ++c) bc[c] = vv[j * D + tx * TR + c];
#pragma unroll
                for (int r = 0; r < TR; ++r)
#pragma unroll
                    for (int c = 0; c < TR; ++c) acc[r][c] = fmaf(ar[r], bc[c], acc[r][c]);
            }
            if (tid < D)
                for (int j = 0; j < kSub; ++j) zacc += fk[j * D + tid];
            __syncthreads();
        }
    }
    float *dst = p.ws_state + ((size_t)bh * p.n_seg + seg) * (D * D + D);
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
        for (int c = 0; c < TR; ++c) dst[(ty * TR + r) * D + tx * TR + c] = acc[r][c];
    if (tid < D) dst[D * D + tid] = zacc;
    if (tid == 0) p.ws_A[(size_t)bh * p.n_seg + seg] = Aseg;
    __syncthreads();
    pdl_trigger();   // this segment's state is written: the scan may launch
}

template <int D> __host__ __device__ constexpr size_t simt_output_smem() {
    return sizeof(float) * (D * D + D + 2 * kSub * (D + 1) + kSub * D + kSub * (kSub + 1) + 128);
}

// K3: chunked causal output.  grid (n_seg, BH), 256 threads.
template <typename InT, typename OutT, int D>
__global__ void __launch_bounds__(kSimtThreads) simt_chunk_output_kernel(SimtParams p) {
    constexpr int TR = D / 16;
    constexpr int CPT = D / 8;  // output columns per thread (32 rows x 8 column groups)
    // phi(q) and phi(k) rows are padded to D + 1 floats: the scores loop reads
    // 32 different key rows at the same column in one warp, and the inter-term
    // loop 4 different query rows, which would otherwise share a bank
    constexpr int RS = D + 1;
    extern __shared__ float smem[];
    float *S = smem;                    // [D][D]
    float *z = S + D * D;               // [D]
    float *fq = z + D;                  // [kSub][D + 1]
    float *fk = fq + kSub * RS;         // [kSub][D + 1]
    float *vv = fk + kSub * RS;         // [kSub][D]
    float *P = vv + kSub * D;           // [kSub][kSub + 1]
    float *Lc = P + kSub * (kSub + 1);  // [128]
    const int seg = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    const int row = tid / 8, cg = tid % 8;
    const long t_begin = (long)seg * p.seg_len;
    const long t_end = min((long)p.T, t_begin + p.seg_len);
    const InT *Q = (const InT *)p.q + (size_t)bh * p.T * D;
    const InT *K = (const InT *)p.k + (size_t)bh * p.T * D;
    const InT *V = (const InT *)p.v + (size_t)bh * p.T * D;
    OutT *O = (OutT *)p.out + (size_t)bh * p.T * D;
    const float *A = p.decay ? p.decay + (size_t)bh * p.T : nullptr;
    const float *Gk = p.gain ? p.gain + (size_t)bh * p.T : nullptr;   // per-token gains

    const float *st = p.ws_state + ((size_t)bh * p.n_seg + seg) * (D * D + D);
    pdl_wait();   // the segment scan's output
    for (int i = tid; i < D * D + D; i += kSimtThreads) S[i] = st[i];
    __syncthreads();

    for (long c0 = t_begin; c0 < t_end; c0 += p.chunk) {
        const int n = (int)min((long)p.chunk, t_end - c0);
        if (A) chunk_log_cumsum(A + c0, n, Lc);
        __syncthreads();
        for (int q0 = 0; q0 < n; q0 += kSub) {
            {
                float qx[simt_per_thread(D)];
                simt_load_rows<InT, D>(Q, c0 + q0, n - q0, qx);
#pragma unroll
                for (int u = 0; u < simt_per_thread(D); ++u) {
                    const int idx = tid + u * kSimtThreads, j = idx / D, a = idx % D;
                    fq[j * RS + a] = (q0 + j < n) ? (p.mlstm ? qx[u] : phi_precise(qx[u])) : 0.f;
                }
            }
            __syncthreads();
            const int il = q0 + row;
            float acc[CPT], den;
            {
                // inter-chunk term with the carried state, decayed by the
                // product of a over the chunk's tokens up to and including i
                const float g = A ? expf(Lc[min(il, n - 1)]) : 1.f;
                float s[CPT];
#pragma unroll
                for (int c = 0; c < CPT; ++c) s[c] = 0.f;
                float dz = 0.f;
                for (int a = 0; a < D; ++a) {
                    const float f = fq[row * RS + a];
                    dz = fmaf(f, z[a], dz);
#pragma unroll
                    for (int c = 0; c < CPT; ++c) s[c] = fmaf(f, S[a * D + cg * CPT + c], s[c]);
                }
#pragma unroll
                for (int c = 0; c < CPT; ++c) acc[c] = g * s[c];
                den = g * dz;
            }
            for (int k0 = 0; k0 <= q0; k0 += kSub) {
                {
                    float kx[simt_per_thread(D)], vx[simt_per_thread(D)];
                    simt_load_rows<InT, D>(K, c0 + k0, n - k0, kx);
                    simt_load_rows<InT, D>(V, c0 + k0, n - k0, vx);
#pragma unroll
                    for (int u = 0; u < simt_per_thread(D); ++u) {
                        const int idx = tid + u * kSimtThreads, j = idx / D, a = idx % D;
                        fk[j * RS + a] =
                            (k0 + j < n) ? (p.mlstm ? kx[u] : phi_precise(kx[u])) * (Gk ? Gk[c0 + k0 + j] : 1.f) : 0.f;
                        vv[idx] = vx[u];
                    }
                }
                __syncthreads();
                for (int e = tid; e < kSub * kSub; e += kSimtThreads) {
                    const int i = e / kSub, j = e % kSub;
                    const int gi = q0 + i, gj = k0 + j;
                    float sc = 0.f;
                    if (gj <= gi && gi < n) {
                        // four independent partial sums (a dependent chain of D FMAs
                        // would serialise on their latency)
                        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                        for (int a = 0; a < D; a += 4) {
#pragma unroll
                            for (int u = 0; u < 4; ++u) s4[u] = fmaf(fq[i * RS + a + u], fk[j * RS + a + u], s4[u]);
                        }
                        sc = (s4[0] + s4[1]) + (s4[2] + s4[3]);
                        if (A) sc *= expf(Lc[gi] - Lc[gj]);
                    }
                    P[i * (kSub + 1) + j] = sc;
                }
                __syncthreads();
                for (int j = 0; j < kSub; ++j) {
                    const float pij = P[row * (kSub + 1) + j];
                    den += pij;
#pragma unroll
                    for (int c = 0; c < CPT; ++c) acc[c] = fmaf(pij, vv[j * D + cg * CPT + c], acc[c]);
                }
                __syncthreads();
            }
            if (il < n) {
                const float dn = p.mlstm ? fmaxf(fabsf(den), 1.f) : den + p.eps;
                OutT *o = O + (size_t)(c0 + il) * D + cg * CPT;
#pragma unroll
                for (int c = 0; c < CPT; ++c) o[c] = from_f32<OutT>(acc[c] / dn);
            }
        }
        // the state after the segment's last chunk is never read (the scan
        // forms the segment-entry states and the final state)
        if (c0 + p.chunk >= t_end) break;
        // state update over the chunk's keys
        const float Lend = A ? Lc[n - 1] : 0.f;
        float sreg[TR][TR];
        {
            const float g = A ? expf(Lend) : 1.f;
#pragma unroll
            for (int r = 0; r < TR; ++r)
#pragma unroll
                for (int c = 0; c < TR; ++c) sreg[r][c] = g * S[(ty * TR + r) * D + tx * TR + c];
        }
        float zreg = 0.f;
        if (tid < D) zreg = (A ? expf(Lend) : 1.f) * z[tid];
        for (int k0 = 0; k0 < n; k0 += kSub) {
            __syncthreads();
            {
                float kx[simt_per_thread(D)], vx[simt_per_thread(D)];
                simt_load_rows<InT, D>(K, c0 + k0, n - k0, kx);
                simt_load_rows<InT, D>(V, c0 + k0, n - k0, vx);
#pragma unroll
                for (int u = 0; u < simt_per_thread(D); ++u) {
                    const int idx = tid + u * kSimtThreads, j = idx / D, a = idx % D;
                    float f = 0.f;
                    if (k0 + j < n) {
                        f = p.mlstm ? kx[u] : phi_precise(kx[u]);
                        if (A) f *= expf(Lend - Lc[k0 + j]);
                        if (Gk) f *= Gk[c0 + k0 + j];
                    }
                    fk[j * RS + a] = f;
                    vv[idx] = vx[u];
                }
            }
            __syncthreads();
            for (int j = 0; j < kSub; ++j) {
                float ar[TR], bc[TR];
#pragma unroll
                for (int r = 0; r < TR; ++r) ar[r] = fk[j * RS + ty * TR + r];
#pragma unroll
                for (int c = 0; c < TR; ++c) bc[c] = vv[j * D + tx * TR + c];
#pragma unroll
                for (int r = 0; r < TR; ++r)
#pragma unroll
                    for (int c = 0; c < TR; ++c) sreg[r][c] = fmaf(ar[r], bc[c], sreg[r][c]);
            }
            if (tid < D)
                for (int j = 0; j < kSub; ++j) zreg += fk[j * RS + tid];
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < TR; ++r)
#pragma unroll
            for (int c = 0; c < TR; ++c) S[(ty * TR + r) * D + tx * TR + c] = sreg[r][c];
        if (tid < D) z[tid] = zreg;
        __syncthreads();
    }
}

template <int D> __host__ __device__ constexpr size_t simt_readout_smem() {
    return sizeof(float) * (D * D + D + kSub * (D + 1));
}

constexpr int kReadoutQueries = 128;

// Non-causal read-out: out_i = phi(q_i)^T S / (phi(q_i)^T z + eps) with the
// head's total (S, z).  grid (ceil(Lq / 128), BH), 256 threads.
template <typename InT, typename OutT, int D>
__global__ void __launch_bounds__(kSimtThreads) simt_noncausal_readout_kernel(SimtParams p) {
    constexpr int CPT = D / 8;
    extern __shared__ float smem[];
    float *S = smem;          // [D][D]
    float *z = S + D * D;     // [D]
    float *fq = z + D;        // [kSub][D + 1] (padded: 4 query rows per warp)
    constexpr int RS = D + 1;
    const int bh = blockIdx.y, tid = threadIdx.x;
    const int row = tid / 8, cg = tid % 8;
    const float *tot = p.ws_total + (size_t)bh * (D * D + D);
    pdl_wait();   // the segment scan's head totals
    for (int i = tid; i < D * D + D; i += kSimtThreads) S[i] = tot[i];
    const InT *Q = (const InT *)p.q + (size_t)bh * p.Lq * D;
    OutT *O = (OutT *)p.out + (size_t)bh * p.Lq * D;
    const int qb = blockIdx.x * kReadoutQueries;
    const int qe = min(p.Lq, qb + kReadoutQueries);
    for (int q0 = qb; q0 < qe; q0 += kSub) {
        __syncthreads();
        {
            float qx[simt_per_thread(D)];
            simt_load_rows<InT, D>(Q, q0, qe - q0, qx);
#pragma unroll
            for (int u = 0; u < simt_per_thread(D); ++u) {
                const int idx = tid + u * kSimtThreads, j = idx / D, a = idx % D;
                fq[j * RS + a] = (q0 + j < qe) ? phi_precise(qx[u]) : 0.f;
            }
        }
        __syncthreads();
        float s[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) s[c] = 0.f;
        float dz = 0.f;
        for (int a = 0; a < D; ++a) {
            const float f = fq[row * RS + a];
            dz = fmaf(f, z[a], dz);
#pragma unroll
            for (int c = 0; c < CPT; ++c) s[c] = fmaf(f, S[a * D + cg * CPT + c], s[c]);
        }
        if (q0 + row < qe) {
            const float dn = dz + p.eps;
            OutT *o = O + (size_t)(q0 + row) * D + cg * CPT;
#pragma unroll
            for (int c = 0; c < CPT; ++c) o[c] = from_f32<OutT>(s[c] / dn);
        }
    }
}

}  // namespace la
