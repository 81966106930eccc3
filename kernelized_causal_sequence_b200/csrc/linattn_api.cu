// linattn_api.cu — the C ABI declared in include/linattn.h: argument checks,
// the segment plan, workspace layout and kernel dispatch.  Every entry point
// validates on the host first and launches nothing on error.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "linattn.h"
#include "common.cuh"
#include "decode.cuh"
#include "nc32_kernels.cuh"
#include "errors.h"
#include "plan.h"
#include "scan.h"
#include "simt_kernels.cuh"
#include "tc_launch.h"

using namespace la;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }
inline bool dtype_ok(la_dtype t) { return t == LA_F32 || t == LA_BF16 || t == LA_F16; }

// Workspace layout of the segment-scan paths:
//   [status word: 2 ints, 256 bytes][ws_state: BH * n_seg * (D*D + D) fp32]
//   [ws_A: BH * n_seg fp32][ws_total: BH * (D*D + D) fp32, non-causal only]
// The status word sits at offset 0 so that la_workspace_status can read it
// without knowing the sizes of the call.
struct WsLayout {
    size_t status_off, state_off, A_off, total_off, bytes;
};

// (non-causal: the totals region also holds, at head dim 32, the tensor-core
// read-out's operand images of 6144 bytes per head)
constexpr size_t kBimgBytes = 6144;
WsLayout ws_layout(long BH, int n_seg, int D, bool with_total) {
    WsLayout w;
    const size_t E = (size_t)D * D + D;
    w.status_off = 0;
    w.state_off = kAlign;
    w.A_off = align_up(w.state_off + sizeof(float) * (size_t)BH * n_seg * E);
    w.total_off = align_up(w.A_off + sizeof(float) * (size_t)BH * n_seg);
    size_t per_head = sizeof(float) * E;
    if (D == 32 && per_head < kBimgBytes) per_head = kBimgBytes;
    w.bytes = with_total ? align_up(w.total_off + per_head * (size_t)BH) : w.total_off;
    return w;
}

// Limit of every bounded device-side wait of the calls that follow
// (la_set_wait_limit_ns), process-wide.
std::atomic<unsigned long long> g_wait_ns{2000000000ull};

// Clears the call's status word (2 ints at the start of the workspace).
la_status clear_status(void *workspace, cudaStream_t st) {
    return cuda_check("status memset", cudaMemsetAsync(workspace, 0, 2 * sizeof(int), st));
}

// Per-(kernel, device) opt-in to large dynamic shared memory.
template <typename K> cudaError_t allow_smem(K kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}


}  // namespace

namespace la {
std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

thread_local char g_last_error[256] = "";
la_status cuda_fail_msg(const char *where, const char *msg) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, msg);
    return LA_ERR_CUDA;
}
la_status cuda_fail(const char *where, cudaError_t e) {
    return cuda_fail_msg(where, cudaGetErrorString(e));
}
}  // namespace la

namespace {

// Launches kern, with programmatic stream serialisation when pdl is set (the
// kernel may start launching while the previous kernel in the stream ends; it
// must call pdl_wait before reading that kernel's output).
template <typename... KArgs, typename... Args>
la_status launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
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
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    count_launches(1);
    if (e != cudaSuccess) return cuda_fail(what, e);
    return cuda_check(what, cudaGetLastError());
}

// ---------------------------------------------------------------- SIMT path
template <typename InT, typename OutT, int D>
la_status simt_causal(SimtParams p, cudaStream_t st) {
    if (record_event(p.events, 0, st) != LA_OK) return LA_ERR_CUDA;
    {
        auto k1 = simt_segment_state_kernel<InT, D>;
        const size_t sm = simt_state_smem<D>();
        la_status e = cuda_check("segment_state smem attribute", allow_smem(k1, sm));
        if (e != LA_OK) return e;
        k1<<<dim3(p.n_seg, p.BH), kSimtThreads, sm, st>>>(p, p.T);
    }
    count_launches(1);
    la_status e = cuda_check("segment_state launch", cudaGetLastError());
    if (e != LA_OK) return e;
    if (record_event(p.events, 1, st) != LA_OK) return LA_ERR_CUDA;
    const bool pdl = p.events == nullptr;   // events between the passes serialise them
    if (launch_segment_scan(p.ws_state, p.ws_A, p.BH, p.n_seg, p.n_seg, D, p.mode, p.state_S, p.state_z,
                            nullptr, st, pdl, p.sum_A) != LA_OK)
        return LA_ERR_CUDA;
    if (p.sum_A) return record_event(p.events, 3, st);   // shard summary: no output pass
    if (record_event(p.events, 2, st) != LA_OK) return LA_ERR_CUDA;
    {
        auto k3 = simt_chunk_output_kernel<InT, OutT, D>;
        const size_t sm = simt_output_smem<D>();
        e = cuda_check("chunk_output smem attribute", allow_smem(k3, sm));
        if (e != LA_OK) return e;
        e = launch_ex(k3, dim3(p.n_seg, p.BH), dim3(kSimtThreads), sm, st, pdl, "chunk_output launch", p);
        if (e != LA_OK) return e;
    }
    return record_event(p.events, 3, st);
}

template <typename InT, typename OutT, int D>
la_status simt_noncausal(SimtParams p, int Lk, cudaStream_t st) {
    {
        auto k1 = simt_segment_state_kernel<InT, D>;
        const size_t sm = simt_state_smem<D>();
        la_status e = cuda_check("segment_state smem attribute", allow_smem(k1, sm));
        if (e != LA_OK) return e;
        k1<<<dim3(p.n_seg, p.BH), kSimtThreads, sm, st>>>(p, Lk);
    }
    count_launches(1);
    la_status e = cuda_check("segment_state launch", cudaGetLastError());
    if (e != LA_OK) return e;
    if (launch_segment_scan(p.ws_state, p.ws_A, p.BH, p.n_seg, p.n_seg, D, p.mode, p.state_S, p.state_z,
                            p.ws_total, st, true) != LA_OK)
        return LA_ERR_CUDA;
    if (p.Lq > 0) {
        auto k3 = simt_noncausal_readout_kernel<InT, OutT, D>;
        const size_t sm = simt_readout_smem<D>();
        e = cuda_check("readout smem attribute", allow_smem(k3, sm));
        if (e != LA_OK) return e;
        e = launch_ex(k3, dim3((p.Lq + kReadoutQueries - 1) / kReadoutQueries, p.BH), dim3(kSimtThreads), sm, st,
                      true, "readout launch", p);
    }
    return e;
}

// Dispatch over (in dtype, out dtype, head dim) for a functor template F.
template <template <typename, typename, int> class F, typename... Args>
la_status dispatch3(la_dtype in, la_dtype out, int D, Args... args) {
#define LA_DISPATCH_D(IT, OT)                                       \
    switch (D) {                                                    \
        case 32: return F<IT, OT, 32>::run(args...);                \
        case 64: return F<IT, OT, 64>::run(args...);                \
        case 128: return F<IT, OT, 128>::run(args...);              \
        default: return LA_ERR_UNSUPPORTED;                         \
    }
    if (in == LA_F32) { LA_DISPATCH_D(float, float) }
    if (in == LA_BF16) {
        if (out == LA_BF16) { LA_DISPATCH_D(bf16, bf16) }
        LA_DISPATCH_D(bf16, float)
    }
    if (in == LA_F16) {
        if (out == LA_F16) { LA_DISPATCH_D(f16, f16) }
        LA_DISPATCH_D(f16, float)
    }
#undef LA_DISPATCH_D
    return LA_ERR_UNSUPPORTED;
}

template <typename IT, typename OT, int D> struct SimtCausalF {
    static la_status run(SimtParams p, cudaStream_t st) { return simt_causal<IT, OT, D>(p, st); }
};
// Head dim 32: register-blocked CUDA-core state and read-out kernels (nc32_kernels.cuh).
template <typename InT, typename OutT>
la_status nc32_noncausal(SimtParams p, int Lk, cudaStream_t st) {
    nc32_state_kernel<InT><<<dim3(p.n_seg, p.BH), kNc32Threads, 0, st>>>(
        (const InT *)p.k, (const InT *)p.v, Lk, p.seg_len, p.n_seg, p.ws_state, p.ws_A);
    count_launches(1);
    la_status e = cuda_check("nc32 state launch", cudaGetLastError());
    if (e != LA_OK) return e;
    e = launch_segment_scan(p.ws_state, p.ws_A, p.BH, p.n_seg, p.n_seg, 32, p.mode, p.state_S, p.state_z,
                            p.ws_total, st, true);
    if (e != LA_OK) return e;
    if (p.Lq > 0) {
        const int tpc = nc32_tiles_per_cta(p.BH, p.Lq);
        const long span = (long)tpc * kNc32Tile;
        e = launch_ex(nc32_readout_kernel<InT, OutT>, dim3((unsigned)((p.Lq + span - 1) / span), p.BH),
                      dim3(kNc32Threads), 0, st, true, "nc32 read-out launch", (const InT *)p.q, p.Lq, tpc,
                      (const float *)p.ws_total, p.eps, (OutT *)p.out);
    }
    return e;
}

template <typename IT, typename OT, int D> struct SimtNoncausalF {
    static la_status run(SimtParams p, int Lk, cudaStream_t st) {
        if constexpr (D == 32) return nc32_noncausal<IT, OT>(p, Lk, st);
        else return simt_noncausal<IT, OT, D>(p, Lk, st);
    }
};
template <typename IT, typename OT, int D> struct DecodeF {
    static la_status run(const void *q, const void *k, const void *v, const float *decay, const float *gain,
                         int mlstm, float eps, float *S, float *z, void *out, long BH, cudaStream_t st) {
        // programmatic dependent launch: the step may be scheduled while the
        // previous kernel in the stream drains; it waits for that kernel's
        // completion (griddepcontrol.wait) before its first global access
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3((unsigned)BH);
        cfg.blockDim = dim3(kDecodeThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t err = cudaLaunchKernelEx(&cfg, decode_step_kernel<IT, OT, D>, (const IT *)q,
                                                   (const IT *)k, (const IT *)v, decay, gain, mlstm, eps, S, z,
                                                   (OT *)out);
        count_launches(1);
        if (err != cudaSuccess) return cuda_fail("decode_step launch", err);
        return cuda_check("decode_step launch", cudaGetLastError());
    }
};

// Shared host-side checks.  Returns LA_OK when the call may proceed.
la_status check_common(la_dtype in, la_dtype out, int d_k, int d_v, float eps) {
    if (!dtype_ok(in) || !dtype_ok(out)) return LA_ERR_INVALID_ARG;
    if (!(std::isfinite(eps) && eps >= 0.f)) return LA_ERR_INVALID_ARG;
    if (d_k <= 0 || d_v <= 0) return LA_ERR_INVALID_ARG;
    if (d_k != d_v || !dim_ok(d_k)) return LA_ERR_UNSUPPORTED;
    if (!(out == in || out == LA_F32)) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

la_status check_state(la_state_mode mode, const float *S, const float *z) {
    if (mode != LA_STATE_NONE && mode != LA_STATE_OUT && mode != LA_STATE_INOUT)
        return LA_ERR_INVALID_ARG;
    if (mode != LA_STATE_NONE && (!S || !z || !aligned16(S) || !aligned16(z)))
        return LA_ERR_INVALID_ARG;
    return LA_OK;
}

// The causal prefill behind every prefill entry point: decay and gain are
// optional per-token [BH, T] arrays, mlstm selects the identity feature map
// and the max(|den|, 1) read-out, events optional (4 cudaEvent_t).
la_status prefill_impl(const void *q, const void *k, const void *v, la_dtype in_dtype, const float *decay,
                       const float *gain, int mlstm, int B, int H, int T, int d_k, int d_v, float eps, int chunk,
                       float *state_S, float *state_z, la_state_mode mode, void *out, la_dtype out_dtype,
                       void *workspace, size_t workspace_bytes, void *stream, void *const *events,
                       int flash = 0, float inv_s = 1.f, float *sum_A = nullptr) {
    // sum_A non-null: the shard summary (state pass + scan, no output pass):
    // state_S/state_z receive the total contribution, sum_A the decay product
    la_status s = check_common(in_dtype, out_dtype, d_k, d_v, eps);
    if (s != LA_OK) return s;
    if (B < 0 || H < 0 || T < 0) return LA_ERR_INVALID_ARG;
    if (chunk != 64 && chunk != 128) return LA_ERR_UNSUPPORTED;
    if (flash && !tc_supported(in_dtype, d_k, chunk, false)) return LA_ERR_UNSUPPORTED;
    if ((s = check_state(mode, state_S, state_z)) != LA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    const long BH = (long)B * H;
    if (BH == 0) return LA_OK;
    const bool summary = sum_A != nullptr;
    if (T == 0 && summary) {
        // nothing to summarise: (0, 0) and a decay product of 1, from the scan over no segments
        if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < kAlign)
            return LA_ERR_INVALID_ARG;
        la_status e = clear_status(workspace, st);
        if (e != LA_OK) return e;
        return launch_segment_scan(nullptr, nullptr, BH, 0, 0, d_k, LA_STATE_OUT, state_S, state_z, nullptr, st,
                                   false, sum_A);
    }
    if (T == 0) {
        if (mode == LA_STATE_OUT) {
            la_status e = cuda_check("state memset", cudaMemsetAsync(state_S, 0, sizeof(float) * BH * d_k * d_v, st));
            if (e == LA_OK) e = cuda_check("state memset", cudaMemsetAsync(state_z, 0, sizeof(float) * BH * d_k, st));
            if (e != LA_OK) return e;
        }
        return LA_OK;
    }
    if (summary) {   // no queries, no output: the maps of the unused operands point at the keys
        q = k;
        out = const_cast<void *>(k);
        out_dtype = in_dtype;
    }
    if (!q || !k || !v || !out) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    if (summary && !aligned16(sum_A)) return LA_ERR_INVALID_ARG;
    if (decay && !aligned16(decay)) return LA_ERR_INVALID_ARG;
    if (gain && !aligned16(gain)) return LA_ERR_INVALID_ARG;
    if (BH > 65535L) return LA_ERR_UNSUPPORTED;   // heads run along grid y
    const Plan pl = make_plan(BH, T, chunk, d_k);
    const WsLayout wl = ws_layout(BH, pl.n_seg, d_k, false);
    if (!workspace || workspace_bytes < wl.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return LA_ERR_INVALID_ARG;
    char *ws = (char *)workspace;
    if ((s = clear_status(ws, st)) != LA_OK) return s;

    if (tc_supported(in_dtype, d_k, chunk, decay != nullptr)) {
        TcCausalArgs a;
        a.q = q; a.k = k; a.v = v; a.decay = decay; a.gain = gain; a.mlstm = mlstm; a.out = out;
        a.flash = flash; a.inv_s = inv_s;
        a.summary = summary; a.sum_A = sum_A;
        a.in_dtype = in_dtype; a.out_dtype = out_dtype;
        a.ws_state = (float *)(ws + wl.state_off);
        a.ws_A = (float *)(ws + wl.A_off);
        a.status = (int *)(ws + wl.status_off);
        a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
        a.state_S = state_S; a.state_z = state_z; a.mode = mode;
        a.BH = BH; a.T = T; a.D = d_k; a.chunk = chunk; a.seg_len = pl.seg_len;
        a.n_seg = pl.n_seg; a.eps = eps;
        a.events = events;
        return tc_causal(a, st);
    }
    SimtParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q; p.k = k; p.v = v; p.decay = decay; p.gain = gain; p.mlstm = mlstm; p.out = out;
    p.ws_state = (float *)(ws + wl.state_off);
    p.ws_A = (float *)(ws + wl.A_off);
    p.ws_total = nullptr;
    p.state_S = state_S; p.state_z = state_z; p.mode = mode;
    p.BH = (int)BH; p.T = T; p.Lq = T; p.chunk = chunk; p.seg_len = pl.seg_len; p.n_seg = pl.n_seg;
    p.eps = eps;
    p.events = events;
    p.sum_A = sum_A;
    return dispatch3<SimtCausalF>(in_dtype, out_dtype, d_k, p, st);
}

// Every decode entry point: gain optional, mlstm as for the prefill.
la_status decode_impl(const void *q, const void *k, const void *v, la_dtype in_dtype, const float *decay,
                      const float *gain, int mlstm, int B, int H, int d_k, int d_v, float eps, float *state_S,
                      float *state_z, void *out, la_dtype out_dtype, void *stream) {
    la_status s = check_common(in_dtype, out_dtype, d_k, d_v, eps);
    if (s != LA_OK) return s;
    if (B < 0 || H < 0) return LA_ERR_INVALID_ARG;
    const long BH = (long)B * H;
    if (BH == 0) return LA_OK;
    if (!q || !k || !v || !out || !state_S || !state_z) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        !aligned16(state_S) || !aligned16(state_z) || (decay && !aligned16(decay)) ||
        (gain && !aligned16(gain)))
        return LA_ERR_INVALID_ARG;
    if (BH > 0x7fffffffL) return LA_ERR_UNSUPPORTED;
    return dispatch3<DecodeF>(in_dtype, out_dtype, d_k, q, k, v, decay, gain, mlstm, eps, state_S, state_z,
                              out, BH, (cudaStream_t)stream);
}

}  // namespace

extern "C" {

uint64_t la_launch_count(void) { return la::g_launches.load(std::memory_order_relaxed); }

uint64_t la_set_wait_limit_ns(uint64_t ns) { return g_wait_ns.exchange(ns); }

la_status la_workspace_status(const void *workspace, int *waiter, void *stream) {
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return LA_ERR_INVALID_ARG;
    int host[2] = {0, 0};
    cudaStream_t st = (cudaStream_t)stream;
    la_status e = cuda_check("status read", cudaMemcpyAsync(host, workspace, sizeof(host), cudaMemcpyDeviceToHost, st));
    if (e == LA_OK) e = cuda_check("status read", cudaStreamSynchronize(st));
    if (e != LA_OK) return e;
    if (waiter) *waiter = host[1];
    return (la_status)host[0];
}

const char *la_last_error_string(void) { return la::g_last_error; }

const char *la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "LA_OK: success";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: unsupported size, chunk or dtype";
        case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA runtime or launch error";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT: bounded device wait expired";
        default: return "unknown la_status";
    }
}

la_status la_prefill_plan(int B, int H, int T, int d_k, int chunk, int *n_seg, int *seg_len) {
    if (B < 0 || H < 0 || T < 0 || d_k <= 0 || !n_seg || !seg_len || (chunk != 64 && chunk != 128))
        return LA_ERR_INVALID_ARG;
    const Plan pl = make_plan((long)B * H, T > 0 ? T : 1, chunk, d_k);
    *n_seg = pl.n_seg;
    *seg_len = pl.seg_len;
    return LA_OK;
}

int la_prefill_path(la_dtype in_dtype, int d_k, int d_v, int chunk, int has_decay) {
    if (!dtype_ok(in_dtype) || d_k != d_v || !dim_ok(d_k) || (chunk != 64 && chunk != 128))
        return -1;
    return tc_supported(in_dtype, d_k, chunk, has_decay != 0) ? 1 : 0;
}

size_t la_prefill_workspace_size(int B, int H, int T, int d_k, int d_v, int chunk) {
    if (B <= 0 || H <= 0 || T <= 0 || d_k != d_v || !dim_ok(d_k) || (chunk != 64 && chunk != 128))
        return 0;
    const long BH = (long)B * H;
    const Plan pl = make_plan(BH, T, chunk, d_k);
    return ws_layout(BH, pl.n_seg, d_k, false).bytes;
}

size_t la_noncausal_workspace_size(int B, int H, int Lk, int d_k, int d_v) {
    if (B <= 0 || H <= 0 || Lk < 0 || d_k != d_v || !dim_ok(d_k)) return 0;
    const long BH = (long)B * H;
    // enough for either path (the dtype is not an argument here)
    const Plan pl = make_nc_plan(BH, Lk, d_k);
    int n_seg = pl.n_seg;
    if (d_k == 32) {
        const Plan pt = make_nc_tc_plan(BH, Lk);
        if (pt.n_seg > n_seg) n_seg = pt.n_seg;
    }
    return ws_layout(BH, n_seg, d_k, true).bytes;
}

la_status la_prefill_causal(const void *q, const void *k, const void *v, la_dtype in_dtype,
                            const float *decay, int B, int H, int T, int d_k, int d_v, float eps,
                            int chunk, float *state_S, float *state_z, la_state_mode mode,
                            void *out, la_dtype out_dtype, void *workspace,
                            size_t workspace_bytes, void *stream) {
    return la_prefill_causal_ev(q, k, v, in_dtype, decay, B, H, T, d_k, d_v, eps, chunk, state_S,
                                state_z, mode, out, out_dtype, workspace, workspace_bytes, stream,
                                nullptr);
}

la_status la_prefill_causal_ev(const void *q, const void *k, const void *v, la_dtype in_dtype,
                               const float *decay, int B, int H, int T, int d_k, int d_v, float eps,
                               int chunk, float *state_S, float *state_z, la_state_mode mode,
                               void *out, la_dtype out_dtype, void *workspace,
                               size_t workspace_bytes, void *stream, void *const *events) {
    return prefill_impl(q, k, v, in_dtype, decay, nullptr, 0, B, H, T, d_k, d_v, eps, chunk, state_S, state_z,
                        mode, out, out_dtype, workspace, workspace_bytes, stream, events);
}

la_status la_prefill_causal_gated(const void *q, const void *k, const void *v, la_dtype in_dtype,
                                  const float *decay, const float *gain, int B, int H, int T, int d_k,
                                  int d_v, float eps, int chunk, float *state_S, float *state_z,
                                  la_state_mode mode, void *out, la_dtype out_dtype, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    return prefill_impl(q, k, v, in_dtype, decay, gain, 0, B, H, T, d_k, d_v, eps, chunk, state_S, state_z,
                        mode, out, out_dtype, workspace, workspace_bytes, stream, nullptr);
}

la_status la_prefill_causal_mlstm(const void *q, const void *k, const void *v, la_dtype in_dtype,
                                  const float *forget, const float *input_gate, int B, int H, int T,
                                  int d_k, int d_v, int chunk, float *state_S, float *state_z,
                                  la_state_mode mode, void *out, la_dtype out_dtype, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    return prefill_impl(q, k, v, in_dtype, forget, input_gate, 1, B, H, T, d_k, d_v, 0.f, chunk, state_S,
                        state_z, mode, out, out_dtype, workspace, workspace_bytes, stream, nullptr);
}

la_status la_prefill_causal_summary(const void *k, const void *v, la_dtype in_dtype, const float *decay,
                                    const float *gain, int B, int H, int T, int d_k, int d_v, int chunk,
                                    float *sum_S, float *sum_z, float *sum_A, void *workspace,
                                    size_t workspace_bytes, void *stream) {
    if (!sum_A || !sum_S || !sum_z) return LA_ERR_INVALID_ARG;
    return prefill_impl(nullptr, k, v, in_dtype, decay, gain, 0, B, H, T, d_k, d_v, 0.f, chunk, sum_S, sum_z,
                        LA_STATE_OUT, nullptr, in_dtype, workspace, workspace_bytes, stream, nullptr, 0, 1.f,
                        sum_A);
}

la_status la_state_combine(const float *S_all, const float *z_all, const float *A_all, int R, int r, int B,
                           int H, int d_k, int d_v, const float *S_in, const float *z_in, float *S_out,
                           float *z_out, void *stream) {
    if (B < 0 || H < 0 || R < 1 || r < 0 || r >= R || d_k <= 0 || d_v <= 0) return LA_ERR_INVALID_ARG;
    if (d_k != d_v || !dim_ok(d_k)) return LA_ERR_UNSUPPORTED;
    const long BH = (long)B * H;
    if (BH == 0) return LA_OK;
    if (BH > 65535L) return LA_ERR_UNSUPPORTED;
    if (!S_out || !z_out || (r > 0 && (!S_all || !z_all || !A_all)) || ((S_in == nullptr) != (z_in == nullptr)))
        return LA_ERR_INVALID_ARG;
    return launch_state_combine(S_all, z_all, A_all, r, BH, d_k, S_in, z_in, S_out, z_out, (cudaStream_t)stream);
}

la_status la_prefill_causal_flash(const void *q, const void *k, const void *v, la_dtype in_dtype, int B, int H,
                                  int T, int d_k, int d_v, int chunk, int scaled, float *state_S, float *state_z,
                                  la_state_mode mode, void *out, la_dtype out_dtype, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    if (scaled != 0 && scaled != 1) return LA_ERR_INVALID_ARG;
    const float inv_s = scaled ? 1.f / (float)chunk : 1.f;   // chunk is 64 or 128: exact
    return prefill_impl(q, k, v, in_dtype, nullptr, nullptr, 0, B, H, T, d_k, d_v, 0.f, chunk, state_S, state_z,
                        mode, out, out_dtype, workspace, workspace_bytes, stream, nullptr, 1, inv_s);
}

la_status la_forward_noncausal(const void *q, const void *k, const void *v, la_dtype in_dtype,
                               const float *decay, int B, int H, int Lq, int Lk, int d_k, int d_v,
                               float eps, float *state_S, float *state_z, la_state_mode mode,
                               void *out, la_dtype out_dtype, void *workspace,
                               size_t workspace_bytes, void *stream) {
    la_status s = check_common(in_dtype, out_dtype, d_k, d_v, eps);
    if (s != LA_OK) return s;
    if (B < 0 || H < 0 || Lq < 0 || Lk < 0) return LA_ERR_INVALID_ARG;
    if (decay) return LA_ERR_UNSUPPORTED;
    if ((s = check_state(mode, state_S, state_z)) != LA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    const long BH = (long)B * H;
    if (BH == 0) return LA_OK;
    if (Lq > 0 && (!q || !out || !aligned16(q) || !aligned16(out))) return LA_ERR_INVALID_ARG;
    if (Lk > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return LA_ERR_INVALID_ARG;
    if (BH > 65535L) return LA_ERR_UNSUPPORTED;   // heads run along grid y
    const bool tc = tc_noncausal_supported(in_dtype, d_k);
    const Plan pl = tc ? make_nc_tc_plan(BH, Lk) : make_nc_plan(BH, Lk, d_k);
    const WsLayout wl = ws_layout(BH, pl.n_seg, d_k, true);
    if (!workspace || workspace_bytes < wl.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return LA_ERR_INVALID_ARG;
    char *ws = (char *)workspace;
    if ((s = clear_status(ws, st)) != LA_OK) return s;

    if (tc) {
        TcNoncausalArgs a;
        a.q = q; a.k = k; a.v = v; a.out = out;
        a.in_dtype = in_dtype; a.out_dtype = out_dtype;
        a.ws_state = (float *)(ws + wl.state_off);
        a.ws_A = (float *)(ws + wl.A_off);
        a.ws_total = (float *)(ws + wl.total_off);
        a.ws_bimg = (uint8_t *)(ws + wl.total_off);
        a.status = (int *)(ws + wl.status_off);
        a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
        a.state_S = state_S; a.state_z = state_z; a.mode = mode;
        a.BH = BH; a.Lq = Lq; a.Lk = Lk; a.D = d_k; a.seg_len = pl.seg_len; a.n_seg = pl.n_seg;
        a.eps = eps;
        return tc_noncausal(a, st);
    }
    SimtParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q; p.k = k; p.v = v; p.decay = nullptr; p.out = out;
    p.ws_state = (float *)(ws + wl.state_off);
    p.ws_A = (float *)(ws + wl.A_off);
    p.ws_total = (float *)(ws + wl.total_off);
    p.state_S = state_S; p.state_z = state_z; p.mode = mode;
    p.BH = (int)BH; p.T = Lk; p.Lq = Lq; p.chunk = pl.chunk; p.seg_len = pl.seg_len;
    p.n_seg = pl.n_seg; p.eps = eps;
    return dispatch3<SimtNoncausalF>(in_dtype, out_dtype, d_k, p, Lk, st);
}

la_status la_decode_step_gated(const void *q, const void *k, const void *v, la_dtype in_dtype,
                               const float *decay, const float *gain, int B, int H, int d_k, int d_v,
                               float eps, float *state_S, float *state_z, void *out, la_dtype out_dtype,
                               void *stream) {
    return decode_impl(q, k, v, in_dtype, decay, gain, 0, B, H, d_k, d_v, eps, state_S, state_z, out, out_dtype,
                       stream);
}

la_status la_decode_step_mlstm(const void *q, const void *k, const void *v, la_dtype in_dtype,
                               const float *forget, const float *input_gate, int B, int H, int d_k,
                               int d_v, float *state_S, float *state_z, void *out, la_dtype out_dtype,
                               void *stream) {
    return decode_impl(q, k, v, in_dtype, forget, input_gate, 1, B, H, d_k, d_v, 0.f, state_S, state_z, out,
                       out_dtype, stream);
}

la_status la_decode_step(const void *q, const void *k, const void *v, la_dtype in_dtype,
                         const float *decay, int B, int H, int d_k, int d_v, float eps,
                         float *state_S, float *state_z, void *out, la_dtype out_dtype,
                         void *stream) {
    return decode_impl(q, k, v, in_dtype, decay, nullptr, 0, B, H, d_k, d_v, eps, state_S, state_z, out,
                       out_dtype, stream);
}

}  // extern "C"
