// nc32_kernels.cuh — the non-causal form at head dimension 32 on the CUDA
// cores ("Linear Attention" knowledge-base page, section 3, non-causal sketch:
// S = phi(K)^T V, z = sum_j phi(k_j), out_i = phi(q_i)^T S / (phi(q_i)^T z + eps)).
//
// At d = 32 the per-token contraction is 32 x 32, too narrow for the
// tensor-core shapes (M >= 64), and the work is bound by memory traffic and
// FMA issue.  Both kernels stage tiles of 128 rows through shared memory with
// 16-byte coalesced loads (the next tile's loads are in flight while the
// current one is used) and give every thread a 4 x 4 block of outputs, so each
// pair of shared-memory loads feeds 16 fused multiply-adds.
#pragma once
#include "common.cuh"

namespace la {

constexpr int kNc32Threads = 256;
constexpr int kNc32Tile = 128;   // rows (keys or queries) per shared-memory tile

// 16-byte chunks of one [kNc32Tile][32] tile that each thread loads.
template <typename InT> struct Nc32Io {
    static constexpr int ELEMS = 16 / (int)sizeof(InT);            // elements per chunk
    static constexpr int CPR = 32 / ELEMS;                          // chunks per row
    static constexpr int NLD = kNc32Tile * CPR / kNc32Threads;      // chunks per thread
};

template <typename InT>
__device__ __forceinline__ void nc32_unpack(const uint4 &u, float (&x)[Nc32Io<InT>::ELEMS]);
template <> __device__ __forceinline__ void nc32_unpack<float>(const uint4 &u, float (&x)[4]) {
    x[0] = __uint_as_float(u.x); x[1] = __uint_as_float(u.y);
    x[2] = __uint_as_float(u.z); x[3] = __uint_as_float(u.w);
}
template <> __device__ __forceinline__ void nc32_unpack<bf16>(const uint4 &u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
template <> __device__ __forceinline__ void nc32_unpack<f16>(const uint4 &u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// Loads this thread's chunks of rows [r0, r0 + kNc32Tile) of a [*, 32] matrix
// (rows >= r1 read as zero).
template <typename InT>
__device__ __forceinline__ void nc32_load_tile(const InT *__restrict__ base, long r0, long r1,
                                               uint4 (&raw)[Nc32Io<InT>::NLD]) {
    using I = Nc32Io<InT>;
#pragma unroll
    for (int i = 0; i < I::NLD; ++i) {
        const int u = threadIdx.x + kNc32Threads * i;
        const long r = r0 + u / I::CPR;
        raw[i] = (r < r1) ? *reinterpret_cast<const uint4 *>(base + r * 32 + (u % I::CPR) * I::ELEMS)
                          : make_uint4(0u, 0u, 0u, 0u);
    }
}

// Per-segment partial state over keys [s*seg_len, min(Lk, (s+1)*seg_len)).
// Thread t owns rows a0..a0+3 and columns b0..b0+3 of S (a0 = 4*((t%64)/8),
// b0 = 4*(t%8)) for the keys of one quarter of each tile (t/64); z is summed
// per tile by each warp over 16 rows (lane = feature).  The partials are
// added at the end in a fixed order (deterministic).
// grid (n_seg, BH), 256 threads; writes ws_state[bh][seg] = (S, z) and
// ws_A[bh][seg] = 1 (no decay), the layout the segment scan consumes.
template <typename InT>
__global__ void __launch_bounds__(kNc32Threads, 4)
nc32_state_kernel(const InT *__restrict__ k, const InT *__restrict__ v, int Lk, int seg_len,
                  int n_seg, float *__restrict__ ws_state, float *__restrict__ ws_A) {
    using I = Nc32Io<InT>;
    // phi(k) rows, v rows; after the last tile the same memory holds the
    // per-quarter partial (S, z) for the final sum
    __shared__ __align__(16) float sm[2 * kNc32Tile * 32];
    float(*fk)[32] = reinterpret_cast<float(*)[32]>(sm);
    float(*vv)[32] = reinterpret_cast<float(*)[32]>(sm + kNc32Tile * 32);
    float(*red)[32][32] = reinterpret_cast<float(*)[32][32]>(sm);
    float(*redz)[32] = reinterpret_cast<float(*)[32]>(sm + 4 * 32 * 32);
    static_assert(4 * 32 * 32 + 8 * 32 <= 2 * kNc32Tile * 32, "reduction fits the tile buffers");
    const int t = threadIdx.x, kg = t >> 6, a0 = ((t & 63) >> 3) * 4, b0 = (t & 7) * 4;
    const int warp = t >> 5, lane = t & 31;
    const int seg = blockIdx.x, bh = blockIdx.y;
    const long j0 = (long)seg * seg_len, j1 = min((long)Lk, j0 + seg_len);
    const InT *K = k + (size_t)bh * Lk * 32;
    const InT *V = v + (size_t)bh * Lk * 32;
    float acc[4][4] = {}, zpart = 0.f;   // zpart: z[lane] over this warp's rows of each tile
    uint4 rk[I::NLD], rv[I::NLD];
    nc32_load_tile<InT>(K, j0, j1, rk);
    nc32_load_tile<InT>(V, j0, j1, rv);
#pragma unroll 1
    for (long jt = j0; jt < j1; jt += kNc32Tile) {
        __syncthreads();   // the previous tile has been used
#pragma unroll
        for (int i = 0; i < I::NLD; ++i) {
            const int u = t + kNc32Threads * i, row = u / I::CPR, col = (u % I::CPR) * I::ELEMS;
            const bool valid = jt + row < j1;
            float x[I::ELEMS], y[I::ELEMS];
            nc32_unpack<InT>(rk[i], x);
            nc32_unpack<InT>(rv[i], y);
#pragma unroll
            for (int e = 0; e < I::ELEMS; e += 4) {
                *reinterpret_cast<float4 *>(&fk[row][col + e]) =
                    valid ? make_float4(phi_precise(x[e]), phi_precise(x[e + 1]), phi_precise(x[e + 2]),
                                        phi_precise(x[e + 3]))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4 *>(&vv[row][col + e]) = make_float4(y[e], y[e + 1], y[e + 2], y[e + 3]);
            }
        }
        __syncthreads();
        if (jt + kNc32Tile < j1) {   // next tile in flight while this one is used
            nc32_load_tile<InT>(K, jt + kNc32Tile, j1, rk);
            nc32_load_tile<InT>(V, jt + kNc32Tile, j1, rv);
        }
#pragma unroll 4
        for (int jj = 0; jj < kNc32Tile / 4; ++jj) {
            const int j = kg * (kNc32Tile / 4) + jj;
            const float4 f = *reinterpret_cast<const float4 *>(&fk[j][a0]);
            const float4 w = *reinterpret_cast<const float4 *>(&vv[j][b0]);
            const float fa[4] = {f.x, f.y, f.z, f.w}, wb[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(fa[r], wb[c], acc[r][c]);
        }
#pragma unroll 4
        for (int jj = 0; jj < kNc32Tile / 8; ++jj) zpart += fk[warp * (kNc32Tile / 8) + jj][lane];
    }
    // add the four key quarters (fixed order)
    __syncthreads();   // the tile buffers are reused
#pragma unroll
    for (int r = 0; r < 4; ++r)
        *reinterpret_cast<float4 *>(&red[kg][a0 + r][b0]) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    redz[warp][lane] = zpart;
    __syncthreads();
    float *dst = ws_state + ((size_t)bh * n_seg + seg) * (32 * 32 + 32);
    for (int e = t; e < 32 * 32; e += kNc32Threads) {
        const int a = e / 32, b = e % 32;
        dst[e] = ((red[0][a][b] + red[1][a][b]) + red[2][a][b]) + red[3][a][b];
    }
    if (t < 32) {
        float zs = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) zs += redz[w][t];
        dst[32 * 32 + t] = zs;
    }
    if (t == 0) ws_A[(size_t)bh * n_seg + seg] = 1.f;
    __syncthreads();
    pdl_trigger();   // this segment's state is written: the scan may launch
}


template <typename OutT> __device__ __forceinline__ void nc32_store4(OutT *dst, float o0, float o1, float o2, float o3);
template <> __device__ __forceinline__ void nc32_store4<float>(float *dst, float o0, float o1, float o2, float o3) {
    *reinterpret_cast<float4 *>(dst) = make_float4(o0, o1, o2, o3);
}
template <> __device__ __forceinline__ void nc32_store4<bf16>(bf16 *dst, float o0, float o1, float o2, float o3) {
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(o0, o1), p1 = __floats2bfloat162_rn(o2, o3);
    *reinterpret_cast<uint2 *>(dst) =
        make_uint2(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1));
}
template <> __device__ __forceinline__ void nc32_store4<f16>(f16 *dst, float o0, float o1, float o2, float o3) {
    const __half2 p0 = __floats2half2_rn(o0, o1), p1 = __floats2half2_rn(o2, o3);
    *reinterpret_cast<uint2 *>(dst) =
        make_uint2(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1));
}

// out_i = phi(q_i)^T S / (phi(q_i)^T z + eps) with the head's total (S, z).
// phi(q) of a 128-query tile is staged transposed, [feature][query], with the
// query index XOR-swizzled by 8 x (the feature's 8-column block) so the
// transposing stores of a warp hit 32 different banks; thread t owns queries
// i0..i0+3 (i0 = 4*(t/8)) and columns b0..b0+3 (b0 = 4*(t%8)) of each tile.
// The denominators of a tile are formed once per query (threads 0..127)
// before the product loop.  grid (ceil(Lq / (128 * tiles_per_cta)), BH),
// 256 threads.
template <typename InT, typename OutT>
__global__ void __launch_bounds__(kNc32Threads, 4)
nc32_readout_kernel(const InT *__restrict__ q, int Lq, int tiles_per_cta, const float *__restrict__ total,
                    float eps, OutT *__restrict__ out) {
    using I = Nc32Io<InT>;
    __shared__ __align__(16) float Ssm[32][32];
    __shared__ float zsm[32];
    __shared__ __align__(16) float fq[32][kNc32Tile];
    __shared__ float inv_den[kNc32Tile];
    const int t = threadIdx.x, i0 = (t >> 3) * 4, b0 = (t & 7) * 4;
    const int bh = blockIdx.y;
    const float *tot = total + (size_t)bh * (32 * 32 + 32);
    pdl_wait();   // the segment scan's head totals
    for (int e = t; e < 32 * 32; e += kNc32Threads) Ssm[e / 32][e % 32] = tot[e];
    if (t < 32) zsm[t] = tot[32 * 32 + t];
    const long span = (long)tiles_per_cta * kNc32Tile;
    const long q0 = (long)blockIdx.x * span, q1 = min((long)Lq, q0 + span);
    const InT *Q = q + (size_t)bh * Lq * 32;
    OutT *O = out + (size_t)bh * Lq * 32;
    uint4 rq[I::NLD];
    if (q0 < q1) nc32_load_tile<InT>(Q, q0, q1, rq);
#pragma unroll 1
    for (long it = q0; it < q1; it += kNc32Tile) {
        __syncthreads();   // S staged; the previous tile has been used
#pragma unroll
        for (int i = 0; i < I::NLD; ++i) {
            const int u = t + kNc32Threads * i, row = u / I::CPR, col = (u % I::CPR) * I::ELEMS;
            float x[I::ELEMS];
            nc32_unpack<InT>(rq[i], x);
#pragma unroll
            for (int e = 0; e < I::ELEMS; ++e) {
                const int c = col + e;
                fq[c][row ^ ((c >> 3) << 3)] = phi_precise(x[e]);
            }
        }
        __syncthreads();
        if (it + kNc32Tile < q1) nc32_load_tile<InT>(Q, it + kNc32Tile, q1, rq);
        if (t < kNc32Tile) {   // denominator of query t of the tile
            float d = 0.f;
#pragma unroll 8
            for (int a = 0; a < 32; ++a) d = fmaf(fq[a][t ^ ((a >> 3) << 3)], zsm[a], d);
            inv_den[t] = 1.f / (d + eps);
        }
        float acc[4][4] = {};
#pragma unroll 8
        for (int a = 0; a < 32; ++a) {
            const float4 f = *reinterpret_cast<const float4 *>(&fq[a][i0 ^ ((a >> 3) << 3)]);
            const float4 s = *reinterpret_cast<const float4 *>(&Ssm[a][b0]);
            const float fr[4] = {f.x, f.y, f.z, f.w}, sc[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(fr[r], sc[c], acc[r][c]);
        }
        __syncthreads();   // inv_den of this tile
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const long i = it + i0 + r;
            if (i < q1) {
                const float inv = inv_den[i0 + r];
                nc32_store4<OutT>(O + i * 32 + b0, acc[r][0] * inv, acc[r][1] * inv, acc[r][2] * inv,
                                  acc[r][3] * inv);
            }
        }
    }
}

}  // namespace la
