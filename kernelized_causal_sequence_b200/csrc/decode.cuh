// decode.cuh — the constant-state decode step (knowledge-base page, section 2
// "Causal recurrence"; concept card "Implementation sketch" with the optional
// scalar decay and, for the gated form, a gain b on the new term — the RFA
// gate is a = g, b = 1 - g):
//                 S <- a S + b phi(k) v^T,  z <- a z + b phi(k),
//                 out = phi(q)^T S / (phi(q)^T z + eps);
// the mLSTM read-out takes phi = identity and divides by max(|q^T z|, 1).
//
// Memory-bound: each head's fp32 state (d_k x d_v + d_k) is read once and
// written once; q, k, v and out are a few hundred bytes.  One CTA per head;
// each thread owns a float4 column group of the state and strides over its
// rows, so every warp moves whole 512-byte rows with 16-byte accesses, and
// the update and the read-out share the single pass over S.
#pragma once
#include "common.cuh"

namespace la {

constexpr int kDecodeThreads = 256;

// 8 CTAs per SM (at most 32 registers a thread): a decode step of 1024 heads
// (B64 H16) is then one wave on 148 SMs; at 40 registers only 6 fit and the
// last 136 heads ran as a second, mostly idle wave
template <typename InT, typename OutT, int D>
__global__ void __launch_bounds__(kDecodeThreads, 8)
decode_step_kernel(const InT *__restrict__ q, const InT *__restrict__ k, const InT *__restrict__ v,
                   const float *__restrict__ decay, const float *__restrict__ gain, int mlstm,
                   float eps, float *__restrict__ S,
                   float *__restrict__ z, OutT *__restrict__ out) {
    constexpr int CG = D / 4;                     // float4 column groups per row
    constexpr int RSTEP = kDecodeThreads / CG;    // rows handled concurrently
    __shared__ float fk[D], fq[D];
    __shared__ float4 red[RSTEP][CG];
    __shared__ float den_part[kDecodeThreads / 32];
    const int bh = blockIdx.x, tid = threadIdx.x;
    // launched with programmatic stream serialisation: the next kernel may be
    // scheduled now; this one waits for the previous kernel (which may have
    // written q, k, v or the state) before reading anything
    pdl_trigger();
    pdl_wait();
    const float a = decay ? decay[bh] : 1.f;
    const float b = gain ? gain[bh] : 1.f;
    if (tid < D) {
        const float kx = to_f32(k[(size_t)bh * D + tid]), qx = to_f32(q[(size_t)bh * D + tid]);
        fk[tid] = b * (mlstm ? kx : phi_fast(kx));
        fq[tid] = mlstm ? qx : phi_fast(qx);
    }
    const int cg = tid % CG, r0 = tid / CG;
    float4 vv;
    {
        const InT *vp = v + (size_t)bh * D + cg * 4;
        vv = make_float4(to_f32(vp[0]), to_f32(vp[1]), to_f32(vp[2]), to_f32(vp[3]));
    }
    __syncthreads();
    // normaliser: z <- a z + phi(k); den = phi(q) . z
    float dpart = 0.f;
    if (tid < D) {
        float *zp = z + (size_t)bh * D + tid;
        const float zn = fmaf(a, *zp, fk[tid]);
        *zp = zn;
        dpart = fq[tid] * zn;
    }
    dpart = warp_sum(dpart);
    if ((tid & 31) == 0) den_part[tid >> 5] = dpart;
    // state rows: S[r] <- a S[r] + phi(k)_r v ; num += phi(q)_r S[r]
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 *Sp = reinterpret_cast<float4 *>(S + (size_t)bh * D * D) + cg;
#pragma unroll 2   // (4 spills under the 32-register bound and measured slower)
    for (int r = r0; r < D; r += RSTEP) {
        float4 s = Sp[(size_t)r * CG];
        const float f = fk[r], g = fq[r];
        s.x = fmaf(a, s.x, f * vv.x);
        s.y = fmaf(a, s.y, f * vv.y);
        s.z = fmaf(a, s.z, f * vv.z);
        s.w = fmaf(a, s.w, f * vv.w);
        Sp[(size_t)r * CG] = s;
        num.x = fmaf(g, s.x, num.x);
        num.y = fmaf(g, s.y, num.y);
        num.z = fmaf(g, s.z, num.z);
        num.w = fmaf(g, s.w, num.w);
    }
    red[r0][cg] = num;
    __syncthreads();
    if (tid < CG) {
        float4 t = red[0][tid];
        for (int i = 1; i < RSTEP; ++i) {
            const float4 u = red[i][tid];
            t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
        }
        float den = 0.f;
        for (int w = 0; w < kDecodeThreads / 32; ++w) den += den_part[w];
        den = mlstm ? fmaxf(fabsf(den), 1.f) : den + eps;
        OutT *o = out + (size_t)bh * D + tid * 4;
        o[0] = from_f32<OutT>(t.x / den);
        o[1] = from_f32<OutT>(t.y / den);
        o[2] = from_f32<OutT>(t.z / den);
        o[3] = from_f32<OutT>(t.w / den);
    }
}

}  // namespace la
