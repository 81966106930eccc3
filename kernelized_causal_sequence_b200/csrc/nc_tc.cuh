// nc_tc.cuh — tcgen05 tensor-core kernels of the non-causal form at head
// dimension 32 (16-bit inputs; tensor-core operands in the input's type for
// the state pass and in bf16 for the read-out; fp32 accumulation):
//
//   S = phi(K)^T V,  z = phi(K)^T 1,  out_i = phi(q_i)^T S / (phi(q_i)^T z + eps)
//
// ("Linear Attention" knowledge-base page, section 3, non-causal sketch: the
// key-value summary is formed once and every query reads it; the linear-
// attention lesson's developer snippet, step 1, the regrouping
// (phi(Q) phi(K)^T) V = phi(Q) (phi(K)^T V).)
//
// Three kernels, chained by programmatic dependent launch:
//
// nc_state_kernel — one CTA per (group of 4 heads, key segment), the key
//   tiles split evenly over the segments.  The 4 heads' [64 keys x 32] K and
//   V tiles arrive by TMA (4 stages; 64-byte swizzle, one slab per head);
//   eight warps apply phi(K) in place in the input's type (rows past the
//   segment zeroed), so the MMA reads phi(K) and V as they are (bf16 or fp16
//   operands).  With the 4 heads' feature columns stacked along M (MN-major
//   A, the next head's slab one 32-element block further), one M=128, N=128
//   MMA per 16 keys accumulates phi(K_g)^T V_h for every head pair (g, h) of
//   the group; the diagonal 32 x 32 blocks are the heads' states, the rest
//   is discarded (d = 32 is below the tensor core's M >= 64, and the extra
//   products are free beside the memory traffic).  A second MMA against a
//   ones operand gives z.  Each CTA writes its heads' partial (S, z) to the
//   workspace.
//
// nc_combine_kernel — per head: the partials summed in segment order
//   (deterministic) plus the state-in; writes the state-out and the head's
//   read-out operands: S and z as a bf16 hi + lo pair of K-major [48][32]
//   images (rows 0-31 the columns of S, row 32 z), so the read-out keeps
//   about 16 mantissa bits of the state.
//
// nc_readout_kernel — a persistent pass over 128-query tiles (every CTA a
//   contiguous range of (head, tile) pairs).  Its set-up and first query
//   loads overlap the state kernel (the largest shared-memory carveout lets
//   a read-out CTA sit beside a state CTA).  After waiting for the combine
//   kernel (griddepcontrol.wait) the query producer brings each head's
//   operand images (6 KB) in by one bulk copy, into one of two buffers by
//   the head's parity, ahead of the head's first tile.  Per tile: phi(Q) is
//   formed in place in the query tile (one thread per query row), which then
//   serves as the K-major A operand; four M=128, N=48, K=16 MMAs form
//   [phi(q) S | phi(q) z] in one of four TMEM accumulators, and the epilogue
//   divides, stages the rows swizzled and stores them by TMA (rows past Lq
//   clipped).
//
// Every wait is bounded (tc_ptx.cuh); on expiry the CTA raises the call's
// status word (LA_ERR_TIMEOUT), drains its copies and products and exits.
#pragma once
#include <type_traits>

#include "common.cuh"
#include "tc_prefill.cuh"
#include "tc_ptx.cuh"

namespace la {
namespace nctc {

using namespace la::tc;

constexpr int kD = 32;               // head dimension of these kernels
constexpr int kHP = 4;               // heads per state CTA: M = 4 x 32 = 128
constexpr int kRows = 128;           // queries per read-out tile
constexpr int kSRows = 64;           // keys per state tile
constexpr int kRowBytes = kD * 2;    // one 16-bit row of 32 features
constexpr int kE = kD * kD + kD;     // floats of one (S, z) state

constexpr int kBN = 48;                       // rows of the read-out's B operand: 32 of S, 1 of z, 15 unused
constexpr int kBop = kBN * kD * 2;            // bytes of one [48][32] bf16 operand
constexpr int kBimg = 2 * kBop;               // the hi and lo operands of one head: 6 KB

// Byte offset of element (n, k) of a K-major no-swizzle [48][32] operand:
// core matrices (8 rows x 8 k) of 128 bytes, 4 along K (128 bytes apart),
// groups of 8 rows 512 bytes apart.
__device__ __forceinline__ int bop_off(int n, int k) {
    return (n >> 3) * 512 + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

struct NcStateParams {
    float *ws_state;                 // [BH][n_seg][kE] partial states
    int *status;                     // the call's status word [2]
    unsigned long long wait_ns;
    int BH, Lk, n_seg;               // segment s: key tiles [s * tiles / n_seg, (s + 1) * tiles / n_seg)
};

struct SCfg {
    static constexpr int HEAD_TILE = kSRows * kRowBytes;  // 4 KB: one head's [64][32] tile
    static constexpr int TILE = kHP * HEAD_TILE;          // 16 KB: the group's 4 slabs
    static constexpr int STAGE = 2 * TILE;                // K, then V
    static constexpr int NST = 4;                         // 128 KB of keys and values in flight
    static constexpr int OFF_KV = 0;
    static constexpr int OFF_ONES = NST * STAGE;          // ones operand [16][64]
    static constexpr int ONES = 16 * kSRows * 2;
    static constexpr int OFF_BAR = OFF_ONES + ONES;
    static constexpr int B_FULL = 0, B_EMPTY = NST, B_PHI = 2 * NST, B_DONE = 3 * NST, B_DRAIN = B_DONE + 1;
    static constexpr int NBAR = B_DRAIN + 1;
    static constexpr int OFF_TMEMADDR = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEMADDR + 4;
    static constexpr int SMEM_BYTES = OFF_ABORT + 4 + 1024;   // + alignment slack
    static constexpr int T_S = 0, T_Z = 128, TMEM_COLS = 256;
    static constexpr int THREADS = 320;   // warp 0 TMA, warp 1 MMA, warps 2-9 phi and epilogue
    static constexpr int PHI_THREADS = 256;
    static_assert(STAGE % 1024 == 0 && HEAD_TILE % 512 == 0 && OFF_ONES % 16 == 0, "layout");
};

// phi on a packed pair of fp16 values, in fp16: max(x, 0) + 2^(min(x, 0) log2 e)
// (x + 1 for x > 0, e^x for x <= 0), the exponential on the packed fp16 ex2
// unit.  The exponent's fp16 rounding (2^-11 relative) moves e^x by under
// 0.2% for |x| <= 3, below the tolerance of 16-bit inputs.
__device__ __forceinline__ uint32_t phi_f16x2(uint32_t x2) {
    constexpr uint32_t kLog2eH2 = 0x3DC53DC5u;   // log2(e) rounded to fp16, twice
    uint32_t m, p, e, r;
    asm("min.f16x2 %0, %1, %2;" : "=r"(m) : "r"(x2), "r"(0u));
    asm("max.f16x2 %0, %1, %2;" : "=r"(p) : "r"(x2), "r"(0u));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(m) : "r"(m), "r"(kLog2eH2));
    asm("ex2.approx.f16x2 %0, %1;" : "=r"(e) : "r"(m));
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(p), "r"(e));
    return r;
}

// phi in place on the [4 heads][64 rows][64 B] K tile (rows >= nvalid
// zeroed), in the input's own 16-bit type: the state MMA then reads phi(K)
// and V as they are (bf16 x bf16 or fp16 x fp16), and V needs no conversion.
// Thread tw (0..NT-1) takes the 16-byte chunks u = tw + NT i: the swizzle only
// permutes chunks inside a 64-byte row, so chunk u lies in row (u / 4) % 64
// whatever its position.
template <typename InT, int NT>
__device__ __forceinline__ void phi_key_tile(uint8_t *kt, int tw, int nvalid) {
    constexpr int NCH = SCfg::TILE / 16;        // 1024 chunks
    constexpr int PER = NCH / NT;
    constexpr int BATCH = PER < 8 ? PER : 8;
#pragma unroll 1
    for (int i0 = 0; i0 < PER; i0 += BATCH) {
        uint4 raw[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) raw[i] = reinterpret_cast<const uint4 *>(kt)[tw + NT * (i0 + i)];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int u = tw + NT * (i0 + i);
            const bool valid = ((u >> 2) & (kSRows - 1)) < nvalid;
            uint4 f;
            if constexpr (std::is_same<InT, bf16>::value)
                f = phi_bf16x8(raw[i]);
            else
                f = make_uint4(phi_f16x2(raw[i].x), phi_f16x2(raw[i].y), phi_f16x2(raw[i].z), phi_f16x2(raw[i].w));
            if (!valid) f = make_uint4(0u, 0u, 0u, 0u);
            reinterpret_cast<uint4 *>(kt)[u] = f;
        }
    }
}

// grid (n_seg, ceil(BH / 4)), 320 threads.
template <typename InT>
__global__ void __launch_bounds__(SCfg::THREADS, 1)
nc_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                NcStateParams p) {
    using G = SCfg;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + G::OFF_BAR);
    uint32_t *tmem_addr_smem = reinterpret_cast<uint32_t *>(smem + G::OFF_TMEMADDR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + G::OFF_ABORT);
    const AbortCtx ab{abort_flag, p.status, p.wait_ns};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg = blockIdx.x, grp = blockIdx.y;
    const long n_tiles = ((long)p.Lk + kSRows - 1) / kSRows;
    const long j0 = seg * n_tiles / p.n_seg * kSRows;
    const long j1 = min((long)p.Lk, (seg + 1) * n_tiles / p.n_seg * kSRows);
    const int ntiles = (int)((j1 - j0 + kSRows - 1) / kSRows);

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < G::NST; ++s) {
            mbar_init(&bar[G::B_FULL + s], 1);
            mbar_init(&bar[G::B_EMPTY + s], 1);
            mbar_init(&bar[G::B_PHI + s], G::PHI_THREADS / 32);
        }
        mbar_init(&bar[G::B_DONE], 1);
        mbar_init(&bar[G::B_DRAIN], 1);
        fence_mbar_init();
    }
    {   // ones operand in the MMA's operand type
        const uint32_t one2 = std::is_same<InT, f16>::value ? 0x3C003C00u : 0x3F803F80u;   // 1.0 pairs
        uint32_t *ones = reinterpret_cast<uint32_t *>(smem + G::OFF_ONES);
        for (int i = threadIdx.x; i < G::ONES / 4; i += G::THREADS) ones[i] = one2;
        fence_proxy_async_smem();
    }
    if (warp == 1) tmem_alloc(tmem_addr_smem, G::TMEM_COLS);
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_addr_smem;
    if ((smem_u32(smem) & 1023u) != 0) raise_abort(ab, 99, kStatusLayout);
    // the read-out kernel may be scheduled now: its set-up and query loads do
    // not depend on this grid, and it waits for this grid before reading the
    // partial states
    pdl_trigger();

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0 && !*abort_flag) {
            int issued[G::NST] = {};
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % G::NST, use = t / G::NST;
                if (use > 0 && !mbar_wait(&bar[G::B_EMPTY + s], (use - 1) & 1, ab, 1)) break;
                uint8_t *kd = smem + G::OFF_KV + s * G::STAGE;
                mbar_expect_tx(&bar[G::B_FULL + s], 2 * G::TILE);
                const int y = (int)(j0 + (long)t * kSRows), z = grp * kHP;
                tma_load_3d(kd, &tm_k, &bar[G::B_FULL + s], 0, y, z);
                tma_load_3d(kd + G::TILE, &tm_v, &bar[G::B_FULL + s], 0, y, z);
                issued[s] = use + 1;
            }
            if (*abort_flag) {
                volatile int never = 0;
                AbortCtx timed{&never, nullptr, kDrainLimitNs};
                for (int s = 0; s < G::NST; ++s)
                    if (issued[s] > 0) mbar_wait(&bar[G::B_FULL + s], (issued[s] - 1) & 1, timed, 0);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0 && !*abort_flag) {
            constexpr bool F16 = std::is_same<InT, f16>::value;
            constexpr uint32_t ID_S = F16 ? idesc_f16(128, 128, true, true) : idesc_bf16(128, 128, true, true);
            constexpr uint32_t ID_Z = F16 ? idesc_f16(128, 16, true, false) : idesc_bf16(128, 16, true, false);
            const uint32_t sb = smem_u32(smem);
            const uint64_t dOnes = sdesc_nosw(sb + G::OFF_ONES, 128, (kSRows / 8) * 128);
            bool done = true;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % G::NST;
                if (!mbar_wait(&bar[G::B_PHI + s], (t / G::NST) & 1, ab, 3)) { done = false; break; }
                tc_fence_after();
                const uint32_t kt = sb + G::OFF_KV + s * G::STAGE;
                // MN-major operands: 4 head slabs of 32 columns (lbo = one slab),
                // 8-row groups 512 bytes apart; 16 keys = 1024 bytes per K step
                const uint64_t dK = sdesc_sw64(kt, G::HEAD_TILE, 512);
                const uint64_t dV = sdesc_sw64(kt + G::TILE, G::HEAD_TILE, 512);
#pragma unroll
                for (int kk = 0; kk < kSRows / 16; ++kk)
                    mma_ss(tmem + G::T_S, dK + (uint64_t)((kk * 1024) >> 4), dV + (uint64_t)((kk * 1024) >> 4), ID_S,
                           (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < kSRows / 16; ++kk)
                    mma_ss(tmem + G::T_Z, dK + (uint64_t)((kk * 1024) >> 4), dOnes + (uint64_t)((kk * 256) >> 4), ID_Z,
                           (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bar[G::B_EMPTY + s]);
            }
            if (done) mma_commit(&bar[G::B_DONE]);
            volatile int never = 0;
            AbortCtx timed{&never, nullptr, kDrainLimitNs};
            mma_commit(&bar[G::B_DRAIN]);
            mbar_wait(&bar[G::B_DRAIN], 0, timed, 0);
        }
    } else {
        // ================= warps 2-9: phi(K), then the partial state out
        const int tw = threadIdx.x - 64;
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            const int s = t % G::NST;
            if (!mbar_wait(&bar[G::B_FULL + s], (t / G::NST) & 1, ab, 4)) { ok = false; break; }
            const long y0 = j0 + (long)t * kSRows;
            const int nvalid = (int)min((long)kSRows, j1 - y0);
            uint8_t *kt = smem + G::OFF_KV + s * G::STAGE;
            phi_key_tile<InT, G::PHI_THREADS>(kt, tw, nvalid);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G::B_PHI + s]);
        }
        // the CTA's partial (S, z) of each of its heads -> the workspace
        if (ok && ntiles > 0 && mbar_wait(&bar[G::B_DONE], 0, ab, 5)) {
            tc_fence_after();
            // TMEM lane quarter q = head q of the group; lane = feature a; warps
            // 2-5 take columns 0-15 of the head's diagonal block (and z), warps
            // 6-9 columns 16-31
            const int q = warp & 3, a = lane, half = warp >= 6 ? 1 : 0;
            const long bh = (long)grp * kHP + q;
            const uint32_t lane_base = (uint32_t)(q * 32) << 16;
            uint32_t u[16], zb = 0;
            tmem_ld16(tmem + lane_base + G::T_S + q * 32 + half * 16, u);
            if (!half) tmem_ld1(tmem + lane_base + G::T_Z, zb);
            tmem_ld_wait();
            if (bh < p.BH && !*abort_flag) {
                float *dst = p.ws_state + ((size_t)bh * p.n_seg + seg) * kE;
                float4 *d4 = reinterpret_cast<float4 *>(dst + a * kD + half * 16);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    d4[i] = make_float4(__uint_as_float(u[4 * i]), __uint_as_float(u[4 * i + 1]),
                                        __uint_as_float(u[4 * i + 2]), __uint_as_float(u[4 * i + 3]));
                if (!half) dst[kD * kD + a] = __uint_as_float(zb);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, G::TMEM_COLS);
    }
}

// --------------------------------------------------------------------------
// nc_combine_kernel — each head's total: the sum of its partial states in
// segment order (deterministic) plus the state-in; writes the state-out and
// the read-out's B operand images (bf16 hi and lo, K-major [48][32]: rows
// 0-31 the columns of S, row 32 z; rows 33-47 are not written and only reach
// output columns the read-out never reads).  One CTA per head, one thread
// per 4 consecutive state elements; each thread's loads for up to 16
// segments are issued before any is used.  With no keys (n_seg = 0) the total is the
// state-in or zeros.  grid (BH), kE / 4 = 264 threads.
struct NcCombineParams {
    const float *ws_state;           // [BH][n_seg][kE]
    uint8_t *ws_bimg;                // [BH][kBimg]
    const float *state_in_S, *state_in_z;   // or null
    float *state_out_S, *state_out_z;       // or null
    int n_seg;
};
constexpr int kCombineThreads = kE / 4;
__global__ void __launch_bounds__(kCombineThreads) nc_combine_kernel(NcCombineParams p) {
    const int g = threadIdx.x;
    const long bh = blockIdx.x;
    // the read-out kernel may be scheduled now (its set-up and query loads do
    // not depend on this grid; it waits for this grid before reading the images)
    pdl_trigger();
    pdl_wait();   // the state kernel's partials
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.state_in_S)
        acc = g < kD * kD / 4 ? reinterpret_cast<const float4 *>(p.state_in_S + (size_t)bh * kD * kD)[g]
                              : reinterpret_cast<const float4 *>(p.state_in_z + (size_t)bh * kD)[g - kD * kD / 4];
    const float4 *src = reinterpret_cast<const float4 *>(p.ws_state + (size_t)bh * p.n_seg * kE) + g;
    for (int s0 = 0; s0 < p.n_seg; s0 += 16) {
        float4 x[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            x[j] = s0 + j < p.n_seg ? src[(size_t)(s0 + j) * (kE / 4)] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            acc.x += x[j].x;
            acc.y += x[j].y;
            acc.z += x[j].z;
            acc.w += x[j].w;
        }
    }
    if (p.state_out_S) {
        if (g < kD * kD / 4) reinterpret_cast<float4 *>(p.state_out_S + (size_t)bh * kD * kD)[g] = acc;
        else reinterpret_cast<float4 *>(p.state_out_z + (size_t)bh * kD)[g - kD * kD / 4] = acc;
    }
    if (p.ws_bimg) {
        uint8_t *img = p.ws_bimg + (size_t)bh * kBimg;
        const float v4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // S[k][nn] -> element (nn, k); z[k] -> element (32, k)
            const int e = 4 * g + j;
            const int nn = e < kD * kD ? e % kD : kD;
            const int k = e < kD * kD ? e / kD : e - kD * kD;
            const bf16 hi = __float2bfloat16_rn(v4[j]);
            *reinterpret_cast<bf16 *>(img + bop_off(nn, k)) = hi;
            *reinterpret_cast<bf16 *>(img + kBop + bop_off(nn, k)) = __float2bfloat16_rn(v4[j] - __bfloat162float(hi));
        }
    }
}

// --------------------------------------------------------------------------
struct NcReadParams {
    const uint8_t *ws_bimg;          // [BH][kBimg] the heads' B operand images (the combine kernel's)
    int *status;
    unsigned long long wait_ns;
    int BH, Lq, n_seg, tiles_per_head;
    long total_tiles;                // BH * tiles_per_head
    float eps;
};

template <typename OutT> struct RCfg {
    static constexpr int QT = kRows * kRowBytes;            // 8 KB query tile (phi(Q) in place: the A operand)
    static constexpr int NQ = 5;                            // query tiles in flight
    static constexpr int ND = 4;                            // TMEM accumulators [128 x 48] in flight
    static constexpr int OFF_Q = 0;
    static constexpr int STG_WARP = 4096;                   // one warp's 32 output rows (<= 128 B each)
    static constexpr int OFF_STG = NQ * QT;                 // 2 buffers x 4 warps
    static constexpr int OFF_B = OFF_STG + 2 * 4 * STG_WARP;
    static constexpr int BN = kBN;                          // B operand rows: 32 of S, 1 of z, 15 unused
    static constexpr int BOP = kBop;                        // 3 KB
    static constexpr int OFF_BAR = OFF_B + 2 * kBimg;       // two heads' operands (hi, lo), by head parity
    static constexpr int B_QFULL = 0, B_PHI = NQ, B_QEMPTY = 2 * NQ, B_DFULL = 3 * NQ, B_DEMPTY = B_DFULL + ND,
                         B_BFREE = B_DEMPTY + ND, B_BLOAD = B_BFREE + 2, B_DRAIN = B_BLOAD + 2,
                         NBAR = B_DRAIN + 1;
    static constexpr int OFF_TMEMADDR = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEMADDR + 4;
    static constexpr int SMEM_BYTES = OFF_ABORT + 4 + 1024;
    static constexpr int T_DSTRIDE = 64, TMEM_COLS = 256;   // accumulator a at columns 64 a .. 64 a + 47
    static constexpr int THREADS = 320;   // warp 0 TMA, 1 MMA, 2-5 phi(Q), 6-9 epilogue
    static constexpr int ROWB = kD * (int)sizeof(OutT);     // output row bytes: 128 (fp32) or 64
    static_assert(OFF_STG % 1024 == 0 && OFF_B % 16 == 0 && ND * T_DSTRIDE <= TMEM_COLS, "layout");
};

// 16-byte chunk c of output row r in a warp's staging rows, swizzled as the
// output tensor map (128-byte rows: 128-byte swizzle; 64-byte rows: 64-byte).
template <int ROWB> __device__ __forceinline__ int stg_off(int r, int c) {
    if constexpr (ROWB == 128) return r * 128 + ((c ^ (r & 7)) << 4);
    else return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}

// grid (G), 320 threads; CTA b takes the flattened (head, tile) range
// [b * total / G, (b + 1) * total / G).
template <typename InT, typename OutT>
__global__ void __launch_bounds__(RCfg<OutT>::THREADS, 1)
nc_readout_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                  NcReadParams p) {
    using G = RCfg<OutT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + G::OFF_BAR);
    uint32_t *tmem_addr_smem = reinterpret_cast<uint32_t *>(smem + G::OFF_TMEMADDR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + G::OFF_ABORT);
    const AbortCtx ab{abort_flag, p.status, p.wait_ns};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long f0 = (long)blockIdx.x * p.total_tiles / gridDim.x;
    const long f1 = (long)(blockIdx.x + 1) * p.total_tiles / gridDim.x;
    const int n = (int)(f1 - f0);
    const int tph = p.tiles_per_head;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < G::NQ; ++s) {
            mbar_init(&bar[G::B_QFULL + s], 1);
            mbar_init(&bar[G::B_PHI + s], 4);
            mbar_init(&bar[G::B_QEMPTY + s], 1);
        }
        for (int a = 0; a < G::ND; ++a) {
            mbar_init(&bar[G::B_DFULL + a], 1);
            mbar_init(&bar[G::B_DEMPTY + a], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar[G::B_BFREE + b], 1);
            mbar_init(&bar[G::B_BLOAD + b], 1);
        }
        mbar_init(&bar[G::B_DRAIN], 1);
        fence_mbar_init();
    }
    {   // B operands start zeroed (rows 33-47 stay zero)
        uint32_t *b = reinterpret_cast<uint32_t *>(smem + G::OFF_B);
        for (int i = threadIdx.x; i < 2 * kBimg / 4; i += G::THREADS) b[i] = 0u;
    }
    if (warp == 1) tmem_alloc(tmem_addr_smem, G::TMEM_COLS);
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_addr_smem;
    if ((smem_u32(smem) & 1023u) != 0) raise_abort(ab, 99, kStatusLayout);

    if (warp == 0) {
        // ================= TMA producer: query tiles (independent of the state kernel), and
        // each head's operand images (the combine kernel's) into the buffer of the head's parity
        if (lane == 0 && !*abort_flag) {
            int issued[G::NQ] = {}, issued_b[2] = {};
            const int head0 = (int)(f0 / tph);
            int next_img = 0;   // images issued so far (head index within this CTA's range)
            bool ok = true;
            // images of the heads up to index h: after the combine kernel (griddepcontrol.wait),
            // each into its buffer once the MMAs of the head two before are complete
            auto images_upto = [&](int h) {
                for (; ok && next_img <= h; ++next_img) {
                    const int b = next_img & 1;
                    if (next_img == 0) pdl_wait();
                    if (next_img >= 2 && !mbar_wait(&bar[G::B_BFREE + b], ((next_img >> 1) - 1) & 1, ab, 4)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&bar[G::B_BLOAD + b], kBimg);
                    bulk_load(smem + G::OFF_B + b * kBimg, p.ws_bimg + (size_t)(head0 + next_img) * kBimg, kBimg,
                              &bar[G::B_BLOAD + b]);
                    issued_b[b] = (next_img >> 1) + 1;
                }
            };
            for (int i = 0; ok && i < n; ++i) {
                const int s = i % G::NQ, use = i / G::NQ;
                if (use > 0 && !mbar_wait(&bar[G::B_QEMPTY + s], (use - 1) & 1, ab, 1)) break;
                const long f = f0 + i;
                const int bh = (int)(f / tph), t = (int)(f % tph);
                mbar_expect_tx(&bar[G::B_QFULL + s], G::QT);
                tma_load_3d(smem + G::OFF_Q + s * G::QT, &tm_q, &bar[G::B_QFULL + s], 0, t * kRows, bh);
                issued[s] = use + 1;
                // once the first stages are filled: the images of the heads loaded so far
                if (i >= G::NQ - 1 || i == n - 1) images_upto(bh - head0);
            }
            if (*abort_flag) {
                volatile int never = 0;
                AbortCtx timed{&never, nullptr, kDrainLimitNs};
                for (int s = 0; s < G::NQ; ++s)
                    if (issued[s] > 0) mbar_wait(&bar[G::B_QFULL + s], (issued[s] - 1) & 1, timed, 0);
                for (int b = 0; b < 2; ++b)
                    if (issued_b[b] > 0) mbar_wait(&bar[G::B_BLOAD + b], (issued_b[b] - 1) & 1, timed, 0);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0 && !*abort_flag) {
            constexpr uint32_t ID = idesc_bf16(128, G::BN, false, false);
            const uint32_t sb = smem_u32(smem);
            int cur = -1, hc = -1;
            for (int i = 0; i < n; ++i) {
                const int s = i % G::NQ, a = i % G::ND;
                const int bh = (int)((f0 + i) / tph);
                if (!mbar_wait(&bar[G::B_PHI + s], (i / G::NQ) & 1, ab, 2)) break;
                if (i >= G::ND && !mbar_wait(&bar[G::B_DEMPTY + a], ((i / G::ND) - 1) & 1, ab, 3)) break;
                if (bh != cur) {
                    // the previous head's operand buffer is free once its MMAs are complete
                    if (hc >= 0) mma_commit(&bar[G::B_BFREE + (hc & 1)]);
                    cur = bh;
                    ++hc;
                    if (!mbar_wait(&bar[G::B_BLOAD + (hc & 1)], (hc >> 1) & 1, ab, 6)) break;
                }
                tc_fence_after();
                const uint64_t dBhi = sdesc_nosw(sb + G::OFF_B + (hc & 1) * kBimg, 128, 512);
                const uint64_t dBlo = sdesc_nosw(sb + G::OFF_B + (hc & 1) * kBimg + G::BOP, 128, 512);
                // A = phi(Q) in place in the query stage: K-major, 64-byte swizzle,
                // 8-row groups 512 bytes apart; a K step of 16 is 32 bytes
                const uint64_t dA = sdesc_sw64(sb + G::OFF_Q + s * G::QT, 16, 512);
                const uint32_t d = tmem + a * G::T_DSTRIDE;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    mma_ss(d, dA + (uint64_t)((kk * 32) >> 4), dBhi + (uint64_t)((kk * 256) >> 4), ID,
                           kk > 0 ? 1u : 0u);
                    mma_ss(d, dA + (uint64_t)((kk * 32) >> 4), dBlo + (uint64_t)((kk * 256) >> 4), ID, 1u);
                }
                mma_commit(&bar[G::B_DFULL + a]);
                mma_commit(&bar[G::B_QEMPTY + s]);   // the query stage may be reloaded
            }
            volatile int never = 0;
            AbortCtx timed{&never, nullptr, kDrainLimitNs};
            mma_commit(&bar[G::B_DRAIN]);
            mbar_wait(&bar[G::B_DRAIN], 0, timed, 0);
        }
    } else if (warp < 6) {
        // ================= phi(Q) in place (warps 2-5, one thread per query row)
        const int q = warp & 3, r = q * 32 + lane;
        for (int i = 0; i < n; ++i) {
            const int s = i % G::NQ;
            if (!mbar_wait(&bar[G::B_QFULL + s], (i / G::NQ) & 1, ab, 5)) break;
            uint8_t *qs = smem + G::OFF_Q + s * G::QT;
            uint4 raw[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                raw[c] = *reinterpret_cast<const uint4 *>(qs + r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 f;
                if constexpr (std::is_same<InT, bf16>::value) {
                    f = phi_bf16x8(raw[c]);
                } else {
                    float x[8];
                    unpack8<InT>(raw[c], x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = phi_fast(x[e]);
                    f = pack8_bf16(x);
                }
                *reinterpret_cast<uint4 *>(qs + r * 64 + ((c ^ ((r >> 1) & 3)) << 4)) = f;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G::B_PHI + s]);
        }
    } else {
        // ================= epilogue (warps 6-9): divide, stage, store
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        for (int i = 0; i < n; ++i) {
            const int a = i % G::ND;
            const long f = f0 + i;
            const int bh = (int)(f / tph), t = (int)(f % tph);
            if (!mbar_wait(&bar[G::B_DFULL + a], (i / G::ND) & 1, ab, 7)) break;
            tc_fence_after();
            uint32_t u[32], ud;
            const uint32_t d = tmem + lane_base + a * G::T_DSTRIDE;
            tmem_ld32(d, u);
            tmem_ld1(d + kD, ud);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G::B_DEMPTY + a]);
            const float inv = 1.f / (__uint_as_float(ud) + p.eps);
            uint8_t *stg = smem + G::OFF_STG + ((i & 1) * 4 + (warp - 6)) * G::STG_WARP;
            // this warp's store of two tiles ago must have read its staging rows
            if (lane == 0) bulk_wait_read1();
            __syncwarp();
            if constexpr (sizeof(OutT) == 4) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<float4 *>(stg + stg_off<128>(lane, c)) =
                        make_float4(__uint_as_float(u[4 * c]) * inv, __uint_as_float(u[4 * c + 1]) * inv,
                                    __uint_as_float(u[4 * c + 2]) * inv, __uint_as_float(u[4 * c + 3]) * inv);
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(u[8 * c + e]) * inv;
                    uint4 w;
                    if constexpr (std::is_same<OutT, bf16>::value) w = pack8_bf16(x);
                    else
                        w = make_uint4(pack_f16x2(x[0], x[1]), pack_f16x2(x[2], x[3]), pack_f16x2(x[4], x[5]),
                                       pack_f16x2(x[6], x[7]));
                    *reinterpret_cast<uint4 *>(stg + stg_off<64>(lane, c)) = w;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(&tm_o, stg, 0, t * kRows + q * 32, bh);
                bulk_commit();
            }
        }
        if (lane == 0) bulk_wait0();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, G::TMEM_COLS);
    }
}

}  // namespace nctc
}  // namespace la
