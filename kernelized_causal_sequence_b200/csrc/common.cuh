// common.cuh — element conversions, the feature map and small device helpers
// shared by the library's kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace la {

using bf16 = __nv_bfloat16;
using f16 = __half;

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<bf16>(bf16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f32<f16>(f16 x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ f16 from_f32<f16>(float x) { return __float2half_rn(x); }

// 2^x with the hardware approximation instruction (relative error ~2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// log2(x) with the hardware approximation instruction.
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;

// Programmatic dependent launch: pdl_wait blocks until the grids this one was
// launched after have completed and their memory is visible (it returns at
// once for a normal launch); pdl_trigger lets a dependent grid start launching
// once every CTA of this grid has triggered or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// phi(x) = elu(x) + 1 (alpha = 1): x + 1 for x > 0, and e^x for x <= 0, which
// equals (e^x - 1) + 1 without the cancellation.  ("Transformers are RNNs"
// feature map, as given on the knowledge-base page, section 2, "Choice of phi".)
// The fp32-input path uses the library expf; the 16-bit paths, whose operands
// are rounded to bf16 anyway, take e^x = 2^(x log2 e) on the ex2 unit.
__device__ __forceinline__ float phi_precise(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float phi_fast(float x) {
    const float e = ex2_approx(x * kLog2e);
    return x > 0.f ? x + 1.f : e;
}

// Inclusive warp scan of the pair operator (a1, x1) o (a2, x2) = (a1 a2, a2 x1 + x2),
// which composes the affine maps X -> a X + x of consecutive segments.
__device__ __forceinline__ void warp_affine_scan(float &a, float &x, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        float a_up = __shfl_up_sync(0xffffffffu, a, off);
        float x_up = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) {
            x = fmaf(a, x_up, x);
            a = a * a_up;
        }
    }
}

// Inclusive warp sum scan.
__device__ __forceinline__ float warp_sum_scan(float x, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        float up = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += up;
    }
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

}  // namespace la
