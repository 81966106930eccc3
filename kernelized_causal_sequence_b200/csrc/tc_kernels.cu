// tc_kernels.cu — host side of the tcgen05 prefill: tensor maps, launch
// configuration and the K1 (state build) -> K2 (scan) -> K3 (chunk output)
// sequence on the caller's stream.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "errors.h"
#include "scan.h"
#include "nc_tc.cuh"
#include "plan.h"
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

// 3-D map over a [BH][L][D] tensor with an explicit box (D columns x rows x
// heads) and swizzle; zero fill (loads) / clipping (stores) outside the tensor.
bool make_map_box(CUtensorMap *m, const void *base, la_dtype dt, long BH, long L, int D, int rows, int heads,
                  CUtensorMapSwizzle sw) {
    auto enc = encode_fn();
    if (!enc) return false;
    const int es = dt == LA_F32 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)L * D * es};
    cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)rows, (cuuint32_t)heads};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType t = dt == LA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                  : dt == LA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    CUresult r = enc(m, t, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D map over a [BH][L][D] tensor with a box of `cols` columns x rows x 1
// head and the given swizzle.
bool make_map_cols(CUtensorMap *m, const void *base, la_dtype dt, long BH, long L, int D, int cols, int rows,
                   CUtensorMapSwizzle sw) {
    auto enc = encode_fn();
    if (!enc) return false;
    const int es = dt == LA_F32 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)L * D * es};
    cuuint32_t box[3] = {(cuuint32_t)cols, (cuuint32_t)rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType t = dt == LA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                  : dt == LA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    CUresult r = enc(m, t, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int C, int D, int FORM, int MODE, typename InT, typename OutT>
la_status launch_tc(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                    const CUtensorMap &mo, const tc::TcParams &p, long BH, int n_ctas_x, cudaStream_t st,
                    bool pdl = false) {
    using G = tc::Cfg<C, D, FORM != 0, MODE>;
    auto kern = tc::tc_prefill_kernel<C, D, FORM, MODE, InT, OutT>;
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

// FORM: 0 no decay, 1 decay (gated, mLSTM), 2 FLASH (whose state-only pass is
// the decay form's: the same weights of 1 and identity feature map)
template <int C, int D, int FORM, typename InT, typename OutT>
la_status run_causal(const TcCausalArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, a.in_dtype, a.BH, a.T, D, C) || !make_map(&mk, a.k, a.in_dtype, a.BH, a.T, D, C) ||
        !make_map(&mv, a.v, a.in_dtype, a.BH, a.T, D, C) ||
        // per-warp row blocks of 32 columns (64-byte rows, 16-bit outputs) or 128 bytes (fp32)
        !make_map_cols(&mo, a.out, a.out_dtype, a.BH, a.T, D, 32, C == 128 ? 32 : 16,
                       a.out_dtype == LA_F32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
        return cuda_fail_msg("cuTensorMapEncodeTiled", "tensor map encoding failed");
    tc::TcParams p;
    p.decay = a.decay;
    p.gain = a.gain;
    p.mlstm = a.mlstm;
    p.out = a.out;
    p.ws_state = a.ws_state;
    p.ws_A = a.ws_A;
    // the last segment's output pass forms the final state, so the state pass
    // and the scan skip that segment's contribution; a summary (no output
    // pass) takes every segment
    const int n_k1 = a.summary ? a.n_seg : a.n_seg - 1;
    p.fin_S = a.mode != LA_STATE_NONE ? a.state_S : nullptr;
    p.fin_z = a.mode != LA_STATE_NONE ? a.state_z : nullptr;
    p.status = a.status;
    p.wait_ns = a.wait_ns;
    p.flash = a.flash;
    p.inv_s = a.inv_s;
    p.T = a.T;
    p.seg_len = a.seg_len;
    p.n_seg = a.n_seg;
    p.eps = a.eps;
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
        s = launch_tc<128, D, (FORM != 0 ? 1 : 0), tc::kStateOnly, InT, float>(mq, mk1, mv1, mo, p, a.BH, n_k1, st);
    } else {
        s = launch_tc<C, D, (FORM != 0 ? 1 : 0), tc::kStateOnly, InT, float>(mq, mk, mv, mo, p, a.BH, n_k1, st);
    }
    if (s != LA_OK) return s;
    if ((s = record_event(a.events, 1, st)) != LA_OK) return s;
    // K2: decayed exclusive scan over segments (+ state in/out)
    // (programmatic dependent launches: each kernel's launch overlaps the end of
    // the previous one; events between the passes, when asked for, serialise them)
    const bool pdl = a.events == nullptr;
    s = launch_segment_scan(a.ws_state, a.ws_A, a.BH, a.n_seg, n_k1, D, a.mode, a.state_S, a.state_z,
                            nullptr, st, pdl && n_k1 > 0, a.summary ? a.sum_A : nullptr);
    if (s != LA_OK) return s;
    if (a.summary) return record_event(a.events, 3, st);
    if ((s = record_event(a.events, 2, st)) != LA_OK) return s;
    // K3: chunked output from the segment-entry states
    s = launch_tc<C, D, FORM, tc::kOutput, InT, OutT>(mq, mk, mv, mo, p, a.BH, a.n_seg, st, pdl);
    if (s != LA_OK) return s;
    return record_event(a.events, 3, st);
}

template <typename InT, typename OutT>
la_status dispatch_cd(const TcCausalArgs &a, cudaStream_t st) {
    // a gain or the mLSTM form runs the decay kernels (the gain's weights share
    // the decay's log2 form; without decay a = 1); FLASH its own output pass
    const int form = a.flash ? 2 : (a.decay != nullptr || a.gain != nullptr || a.mlstm) ? 1 : 0;
#define LA_FORMS(C, D)                                                   \
    switch (form) {                                                      \
        case 0: return run_causal<C, D, 0, InT, OutT>(a, st);            \
        case 1: return run_causal<C, D, 1, InT, OutT>(a, st);            \
        default: return run_causal<C, D, 2, InT, OutT>(a, st);           \
    }
    if (a.D == 128) {
        if (a.chunk == 128) { LA_FORMS(128, 128) }
        LA_FORMS(64, 128)
    }
    if (a.D == 64) {
        if (a.chunk == 128) { LA_FORMS(128, 64) }
        LA_FORMS(64, 64)
    }
#undef LA_FORMS
    return LA_ERR_UNSUPPORTED;
}

// Non-causal form at head dim 32: the state kernel (per group of 4 heads and
// key segment) and the read-out kernel, chained by programmatic dependent
// launch.  With no queries the segment scan forms the state output instead.
// Launches kern with programmatic stream serialisation when pdl is set.
template <typename... KArgs, typename... Args>
la_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                     const char *what, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, args...);
    count_launches(1);
    if (err != cudaSuccess) return cuda_fail(what, err);
    return cuda_check(what, cudaGetLastError());
}

// Non-causal form at head dim 32: the state kernel (per group of 4 heads and
// key segment), the combine kernel (per head: totals, state-out, read-out
// operands) and the read-out kernel, chained by programmatic dependent launch.
template <typename InT, typename OutT>
la_status run_noncausal32(const TcNoncausalArgs &a, cudaStream_t st) {
    using namespace nctc;
    const bool keys = a.Lk > 0;
    const bool inout = a.mode == LA_STATE_INOUT;
    la_status s = LA_OK;
    if (keys) {
        CUtensorMap mk, mv;
        if (!make_map_box(&mk, a.k, a.in_dtype, a.BH, a.Lk, kD, kSRows, kHP, CU_TENSOR_MAP_SWIZZLE_64B) ||
            !make_map_box(&mv, a.v, a.in_dtype, a.BH, a.Lk, kD, kSRows, kHP, CU_TENSOR_MAP_SWIZZLE_64B))
            return cuda_fail_msg("cuTensorMapEncodeTiled", "tensor map encoding failed");
        NcStateParams sp;
        sp.ws_state = a.ws_state;
        sp.status = a.status;
        sp.wait_ns = a.wait_ns;
        sp.BH = (int)a.BH;
        sp.Lk = a.Lk;
        sp.n_seg = a.n_seg;
        auto kern = nc_state_kernel<InT>;
        s = cuda_check("non-causal state smem attribute",
                       cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SCfg::SMEM_BYTES));
        if (s != LA_OK) return s;
        // the largest shared-memory carveout, so that a read-out CTA fits beside a state CTA
        s = cuda_check("non-causal state carveout",
                       cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                            (int)cudaSharedmemCarveoutMaxShared));
        if (s != LA_OK) return s;
        s = launch_pdl(kern, dim3((unsigned)a.n_seg, (unsigned)((a.BH + kHP - 1) / kHP)), dim3(SCfg::THREADS),
                       SCfg::SMEM_BYTES, st, false, "non-causal state launch", mk, mv, sp);
        if (s != LA_OK) return s;
    }
    if (a.Lq == 0 && a.mode == LA_STATE_NONE) return LA_OK;
    NcCombineParams cp;
    cp.ws_state = a.ws_state;
    cp.ws_bimg = a.Lq > 0 ? a.ws_bimg : nullptr;
    cp.state_in_S = inout ? a.state_S : nullptr;
    cp.state_in_z = inout ? a.state_z : nullptr;
    cp.state_out_S = a.mode != LA_STATE_NONE ? a.state_S : nullptr;
    cp.state_out_z = a.mode != LA_STATE_NONE ? a.state_z : nullptr;
    cp.n_seg = keys ? a.n_seg : 0;
    s = launch_pdl(nc_combine_kernel, dim3((unsigned)a.BH), dim3(kCombineThreads), 0, st, keys,
                   "non-causal combine launch", cp);
    if (s != LA_OK || a.Lq == 0) return s;
    CUtensorMap mq, mo;
    if (!make_map_box(&mq, a.q, a.in_dtype, a.BH, a.Lq, kD, kRows, 1, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_box(&mo, a.out, a.out_dtype, a.BH, a.Lq, kD, 32, 1,
                      a.out_dtype == LA_F32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
        return cuda_fail_msg("cuTensorMapEncodeTiled", "tensor map encoding failed");
    NcReadParams rp;
    rp.ws_bimg = a.ws_bimg;
    rp.status = a.status;
    rp.wait_ns = a.wait_ns;
    rp.BH = (int)a.BH;
    rp.Lq = a.Lq;
    rp.n_seg = keys ? a.n_seg : 0;
    rp.tiles_per_head = (a.Lq + kRows - 1) / kRows;
    rp.total_tiles = a.BH * rp.tiles_per_head;
    rp.eps = a.eps;
    auto kern = nc_readout_kernel<InT, OutT>;
    constexpr int SM = RCfg<OutT>::SMEM_BYTES;
    s = cuda_check("non-causal read-out smem attribute",
                   cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM));
    if (s != LA_OK) return s;
    s = cuda_check("non-causal read-out carveout",
                   cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                        (int)cudaSharedmemCarveoutMaxShared));
    if (s != LA_OK) return s;
    const long grid = rp.total_tiles < kNumSMs ? rp.total_tiles : kNumSMs;
    // its set-up and query loads overlap the combine kernel
    return launch_pdl(kern, dim3((unsigned)grid), dim3(RCfg<OutT>::THREADS), SM, st, true,
                      "non-causal read-out launch", mq, mo, rp);
}

}  // namespace

bool tc_supported(la_dtype in_dtype, int D, int chunk, bool has_decay) {
    if (in_dtype != LA_BF16 && in_dtype != LA_F16) return false;
    if (D != 64 && D != 128) return false;
    if (chunk != 64 && chunk != 128) return false;
    (void)has_decay;
    return true;
}

bool tc_noncausal_supported(la_dtype in_dtype, int D) {
    return (in_dtype == LA_BF16 || in_dtype == LA_F16) && D == 32;
}

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

la_status tc_noncausal(const TcNoncausalArgs &a, cudaStream_t st) {
    if (a.D != 32) return LA_ERR_UNSUPPORTED;
    if (a.in_dtype == LA_BF16) {
        if (a.out_dtype == LA_BF16) return run_noncausal32<bf16, bf16>(a, st);
        return run_noncausal32<bf16, float>(a, st);
    }
    if (a.in_dtype == LA_F16) {
        if (a.out_dtype == LA_F16) return run_noncausal32<f16, f16>(a, st);
        return run_noncausal32<f16, float>(a, st);
    }
    return LA_ERR_UNSUPPORTED;
}

}  // namespace la
