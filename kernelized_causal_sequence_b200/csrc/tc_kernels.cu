// tc_kernels.cu — host side of the tcgen05 prefill: tensor maps, launch
// configuration and the K1 (state build) -> K2 (scan) -> K3 (chunk output)
// sequence on the caller's stream.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "errors.h"
#include "scan.h"
#include "tc_launch.h"
#include "tc_prefill.cuh"

namespace la {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D map over a [BH][T][D] tensor; box = 128 bytes of columns x C rows x 1
// head, 128-byte swizzle, zero fill (loads) / clipping (stores) beyond T.
bool make_map(CUtensorMap *m, const void *base, la_dtype dt, long BH, int T, int D, int C) {
    auto enc = encode_fn();
    if (!enc) return false;
    const int es = dt == LA_F32 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)T * D * es};
    cuuint32_t box[3] = {(cuuint32_t)(128 / es), (cuuint32_t)C, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType t = dt == LA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                  : dt == LA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    CUresult r = enc(m, t, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int C, int D, bool DECAY, int MODE, typename InT, typename OutT>
la_status launch_tc(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                    const CUtensorMap &mo, const tc::TcParams &p, long BH, int n_ctas_x, cudaStream_t st,
                    bool pdl = false) {
    using G = tc::Cfg<C, D, DECAY, MODE>;
    auto kern = tc::tc_prefill_kernel<C, D, DECAY, MODE, InT, OutT>;
    la_status e = cuda_check("tensor-core kernel smem attribute",
                             cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES));
    if (e != LA_OK) return e;
    // with pdl the kernel may start launching while the previous one (the
    // segment scan) finishes; it waits for that kernel before reading its output
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(n_ctas_x, (unsigned)BH);
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = G::SMEM_BYTES;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, p);
    count_launches(1);
    if (err != cudaSuccess) return cuda_fail("tensor-core kernel launch", err);
    return cuda_check("tensor-core kernel launch", cudaGetLastError());
}

template <int C, int D, bool DECAY, typename InT, typename OutT>
la_status run_causal(const TcCausalArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, a.in_dtype, a.BH, a.T, D, C) || !make_map(&mk, a.k, a.in_dtype, a.BH, a.T, D, C) ||
        !make_map(&mv, a.v, a.in_dtype, a.BH, a.T, D, C) ||
        !make_map(&mo, a.out, a.out_dtype, a.BH, a.T, D, C == 128 ? 32 : 16))   // per-warp row blocks
        return cuda_fail_msg("cuTensorMapEncodeTiled", "tensor map encoding failed");
    tc::TcParams p;
    p.decay = a.decay;
    p.gain = a.gain;
    p.mlstm = a.mlstm;
    p.out = a.out;
    p.ws_state = a.ws_state;
    p.ws_A = a.ws_A;
    // the last segment's output pass forms the final state, so the state pass
    // and the scan skip that segment's contribution
    const int n_k1 = a.n_seg - 1;
    p.fin_S = a.mode != LA_STATE_NONE ? a.state_S : nullptr;
    p.fin_z = a.mode != LA_STATE_NONE ? a.state_z : nullptr;
    p.status = a.status;
    p.T = a.T;
    p.seg_len = a.seg_len;
    p.n_seg = a.n_seg;
    p.eps = a.eps;
    la_status e0 = cuda_check("status memset", cudaMemsetAsync(a.status, 0, sizeof(int), st));
    if (e0 != LA_OK) return e0;
    la_status s = record_event(a.events, 0, st);
    if (s != LA_OK) return s;
    // K1: per-segment state contributions of segments 0 .. n_seg-2.  A
    // segment's contribution does not depend on the chunk, so K1 always walks
    // it in 128-token tiles (fewer, longer pipeline steps); segments are whole
    // 64-token chunks and the last tile of a segment may be a half tile.
    if (n_k1 == 0) {
        s = LA_OK;
    } else if constexpr (C == 64) {
        CUtensorMap mk1, mv1;
        if (!make_map(&mk1, a.k, a.in_dtype, a.BH, a.T, D, 128) || !make_map(&mv1, a.v, a.in_dtype, a.BH, a.T, D, 128))
            return cuda_fail_msg("cuTensorMapEncodeTiled", "tensor map encoding failed");
        s = launch_tc<128, D, DECAY, tc::kStateOnly, InT, float>(mq, mk1, mv1, mo, p, a.BH, n_k1, st);
    } else {
        s = launch_tc<C, D, DECAY, tc::kStateOnly, InT, float>(mq, mk, mv, mo, p, a.BH, n_k1, st);
    }
    if (s != LA_OK) return s;
    if ((s = record_event(a.events, 1, st)) != LA_OK) return s;
    // K2: decayed exclusive scan over segments (+ state in/out)
    // (programmatic dependent launches: each kernel's launch overlaps the end of
    // the previous one; events between the passes, when asked for, serialise them)
    const bool pdl = a.events == nullptr;
    s = launch_segment_scan(a.ws_state, a.ws_A, a.BH, a.n_seg, n_k1, D, a.mode, a.state_S, a.state_z,
                            nullptr, st, pdl && n_k1 > 0);
    if (s != LA_OK) return s;
    if ((s = record_event(a.events, 2, st)) != LA_OK) return s;
    // K3: chunked output from the segment-entry states
    s = launch_tc<C, D, DECAY, tc::kOutput, InT, OutT>(mq, mk, mv, mo, p, a.BH, a.n_seg, st, pdl);
    if (s != LA_OK) return s;
    return record_event(a.events, 3, st);
}

template <typename InT, typename OutT>
la_status dispatch_cd(const TcCausalArgs &a, cudaStream_t st) {
    // a gain or the mLSTM form runs the decay kernels (the gain's weights share
    // the decay's log2 form; without decay a = 1)
    const bool dec = a.decay != nullptr || a.gain != nullptr || a.mlstm;
    if (a.D == 128) {
        if (a.chunk == 128)
            return dec ? run_causal<128, 128, true, InT, OutT>(a, st) : run_causal<128, 128, false, InT, OutT>(a, st);
        return dec ? run_causal<64, 128, true, InT, OutT>(a, st) : run_causal<64, 128, false, InT, OutT>(a, st);
    }
    if (a.D == 64) {
        if (a.chunk == 128)
            return dec ? run_causal<128, 64, true, InT, OutT>(a, st) : run_causal<128, 64, false, InT, OutT>(a, st);
        return dec ? run_causal<64, 64, true, InT, OutT>(a, st) : run_causal<64, 64, false, InT, OutT>(a, st);
    }
    return LA_ERR_UNSUPPORTED;
}

}  // namespace

bool tc_supported(la_dtype in_dtype, int D, int chunk, bool has_decay) {
    if (in_dtype != LA_BF16 && in_dtype != LA_F16) return false;
    if (D != 64 && D != 128) return false;
    if (chunk != 64 && chunk != 128) return false;
    (void)has_decay;
    return true;
}

bool tc_noncausal_supported(la_dtype, int) { return false; }

la_status tc_causal(const TcCausalArgs &a, cudaStream_t st) {
    if (a.in_dtype == LA_BF16) {
        if (a.out_dtype == LA_BF16) return dispatch_cd<bf16, bf16>(a, st);
        return dispatch_cd<bf16, float>(a, st);
    }
    if (a.in_dtype == LA_F16) {
        if (a.out_dtype == LA_F16) return dispatch_cd<f16, f16>(a, st);
        return dispatch_cd<f16, float>(a, st);
    }
    return LA_ERR_UNSUPPORTED;
}

la_status tc_noncausal(const TcNoncausalArgs &, cudaStream_t) { return LA_ERR_UNSUPPORTED; }

}  // namespace la
