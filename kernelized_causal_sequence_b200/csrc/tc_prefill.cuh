// tc_prefill.cuh — tcgen05 tensor-core kernels of the chunked causal form
// (bf16/fp16 inputs, bf16 tensor-core operands, fp32 accumulation and state).
//
// One CTA owns one segment of one head and walks its chunks of C tokens.
// Per chunk (C tokens, head dim D), with the state (S, z) entering the chunk:
//
//   MMA1  scores = phi(Q) phi(K)^T                      (C x C,  K = D)
//   MMA2  O      = phi(Q) S                            (C x D,  K = D)   inter-chunk term
//   MMAd  den    = phi(Q) z                            (C x 16, K = D)
//   MMA3  S     += (w o phi(K))^T V                    (D x D,  K = C)   state update
//   MMAz  z     += (w o phi(K))^T 1                    (D x 16, K = C)
//   MMA4  O     += P V,  P = scores o mask o decay     (C x D,  K = C)   exact intra-chunk part
//   out   = O / (den_inter + rowsum(P) + eps)
//
// ("Linear Attention" knowledge-base page, section 2 and section 3 sketches;
// the linear-attention lesson's "Implementation reality": quadratic inside a
// chunk, the state carried across chunks; the concept card's SSD variant for
// the scalar decay.)  With decay, w_j = prod_{l>j in chunk} a_l, the mask is
// exp(L_i - L_j) for j <= i (L = chunk-local inclusive cumsum of log a), the
// inter term of row i is scaled by exp(L_i), and the state is rescaled by the
// chunk's total decay before each update.
//
// Warp roles (320 threads):
//   warps 0-3  epilogue: scores -> P (mask, decay, row sums), output division
//              and store.  Warp w reads TMEM lanes 32w..32w+31.
//   warp  4    TMA producer (one elected thread).
//   warp  5    TMEM allocator and MMA issuer (one elected thread).
//   warps 6-9  feature map phi on the staged tiles, decay cumsum, and the
//              state epilogue (TMEM S -> bf16 operand, decay rescale).
//
// Every wait is bounded (see tc_ptx.cuh); on expiry the CTA raises its abort
// flag and the status word, drains its copies and MMAs, frees TMEM, returns.
#pragma once
#include <type_traits>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace la {
namespace tc {

enum Mode { kStateOnly = 0, kOutput = 1 };

constexpr int kThreads = 320;
constexpr int kEpiWarp0 = 0, kTmaWarp = 4, kMmaWarp = 5, kPhiWarp0 = 6;

constexpr int tmem_alloc_cols(int used) {
    return used <= 32 ? 32 : used <= 64 ? 64 : used <= 128 ? 128 : used <= 256 ? 256 : 512;
}

template <int C_, int D_, bool DECAY_, int MODE_> struct Cfg {
    static constexpr int C = C_, D = D_;
    static constexpr bool DECAY = DECAY_;
    static constexpr bool OUT = MODE_ == kOutput;
    static constexpr int KB = D / 64;              // 64-column (128-byte) boxes per row
    static constexpr int BOXB = C * 128;           // bytes of one [C][64] bf16 box
    static constexpr int TILE = C * D * 2;         // bytes of one [C][D] bf16 tile
    static constexpr bool QT = OUT && C == 128;    // phi(Q) held in TMEM
    static constexpr bool PT = OUT && C == 128;    // P held in TMEM
    static constexpr bool SPLIT = OUT && DECAY;    // separate inter / intra accumulators
    static constexpr int NKV = 2;                  // K/V stages
    static constexpr int NQ = OUT ? (QT ? 1 : 2) : 0;
    static constexpr int ROWS_PER_WARP = (C == 128) ? 32 : 16;   // M=64 uses lanes 0-15

    // ---- shared memory (offsets from a 1024-byte aligned base)
    static constexpr int KV_STAGE = 2 * TILE + (DECAY ? TILE : 0);  // K, V, (w o phi(K))
    static constexpr int OFF_KV = 0;
    static constexpr int OFF_Q = OFF_KV + NKV * KV_STAGE;
    static constexpr int OFF_SBF = OFF_Q + NQ * TILE;                // S as bf16 MMA operand
    static constexpr int SBF = OUT ? D * D * 2 : 0;
    static constexpr int OFF_P = OFF_SBF + SBF;
    static constexpr int PB = (OUT && !PT) ? C * C * 2 : 0;
    static constexpr int OFF_ZB = OFF_P + PB;                        // z as MMA operand [16][D]
    static constexpr int ZB = OUT ? 16 * D * 2 : 0;
    static constexpr int OFF_ONES = OFF_ZB + ZB;                     // ones operand [16][C]
    static constexpr int ONES = 16 * C * 2;
    static constexpr int OFF_F = OFF_ONES + ONES;                    // fp32 scratch
    static constexpr int F_L = 0;                                    // [NKV][C] log-decay cumsum
    static constexpr int F_G = F_L + (DECAY ? NKV * C : 0);          // [NKV] chunk decay
    static constexpr int F_END = F_G + NKV;
    static constexpr int OFF_BAR = (OFF_F + F_END * 4 + 7) / 8 * 8;
    // barrier indices
    static constexpr int B_KV_FULL = 0, B_KV_EMPTY = B_KV_FULL + NKV, B_PHI = B_KV_EMPTY + NKV;
    static constexpr int B_Q_FULL = B_PHI + NKV, B_Q_EMPTY = B_Q_FULL + 2;
    static constexpr int B_QT_EMPTY = B_Q_EMPTY + 2, B_SC_FULL = B_QT_EMPTY + 1;
    static constexpr int B_P_READY = B_SC_FULL + 1, B_MMA4 = B_P_READY + 1;
    static constexpr int B_O_FULL = B_MMA4 + 1, B_O_EMPTY = B_O_FULL + 1;
    static constexpr int B_DS_FULL = B_O_EMPTY + 1, B_S_READY = B_DS_FULL + 1;
    static constexpr int B_DRAIN = B_S_READY + 1, NBAR = B_DRAIN + 1;
    static constexpr int OFF_TMEMADDR = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEMADDR + 4;
    static constexpr int OFF_END = OFF_ABORT + 4;
    static constexpr int SMEM_BYTES = OFF_END + 1024;   // + alignment slack

    // ---- TMEM columns
    static constexpr int T_SC = 0;
    static constexpr int T_O = OUT ? C : 0;
    static constexpr int T_O2 = T_O + (OUT ? D : 0);
    static constexpr int T_S = T_O2 + (SPLIT ? D : 0);
    static constexpr int T_Z = T_S + D;
    static constexpr int T_DEN = T_Z + 16;
    static constexpr int T_Q = T_DEN + (OUT ? 16 : 0);
    static constexpr int T_USED = T_Q + (QT ? D / 2 : 0);
    static constexpr int TMEM_COLS = tmem_alloc_cols(T_USED);

    static_assert(D == 64 || D == 128, "tensor-core path: D in {64, 128}");
    static_assert(C == 64 || C == 128, "tensor-core path: chunk in {64, 128}");
    static_assert(!(C == 128 && DECAY && OUT), "chunk 128 with decay exceeds TMEM");
    static_assert(T_USED <= 512, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct TcParams {
    const float *decay;   // [BH, T] or null
    void *out;            // [BH, T, D]
    float *ws_state;      // [BH, n_seg, D*D + D]
    float *ws_A;          // [BH, n_seg]
    int *status;          // status word (0 = ok)
    int T, seg_len, n_seg;
    float eps;
};

template <typename OutT> __device__ __forceinline__ void store_row32(OutT *dst, const float (&o)[32]);
template <> __device__ __forceinline__ void store_row32<float>(float *dst, const float (&o)[32]) {
    float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
    for (int i = 0; i < 8; ++i) d4[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}
template <> __device__ __forceinline__ void store_row32<bf16>(bf16 *dst, const float (&o)[32]) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        d4[i] = make_uint4(pack_bf16x2(o[8 * i], o[8 * i + 1]), pack_bf16x2(o[8 * i + 2], o[8 * i + 3]),
                           pack_bf16x2(o[8 * i + 4], o[8 * i + 5]), pack_bf16x2(o[8 * i + 6], o[8 * i + 7]));
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
template <> __device__ __forceinline__ void store_row32<f16>(f16 *dst, const float (&o)[32]) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        d4[i] = make_uint4(pack_f16x2(o[8 * i], o[8 * i + 1]), pack_f16x2(o[8 * i + 2], o[8 * i + 3]),
                           pack_f16x2(o[8 * i + 4], o[8 * i + 5]), pack_f16x2(o[8 * i + 6], o[8 * i + 7]));
}

// Unpack 8 input elements (one 16-byte chunk) to fp32.
template <typename InT> __device__ __forceinline__ void unpack8(const uint4 &u, float (&x)[8]);
template <> __device__ __forceinline__ void unpack8<bf16>(const uint4 &u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) { x[2 * i] = bf16lo(w[i]); x[2 * i + 1] = bf16hi(w[i]); }
}
template <> __device__ __forceinline__ void unpack8<f16>(const uint4 &u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
        const float2 f = __half22float2(h);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&x)[8]) {
    return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                      pack_bf16x2(x[6], x[7]));
}

// ---------------------------------------------------------------------------
template <int C, int D, bool DECAY, int MODE, typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
tc_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, TcParams p) {
    using G = Cfg<C, D, DECAY, MODE>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + G::OFF_BAR);
    uint32_t *tmem_addr_smem = reinterpret_cast<uint32_t *>(smem + G::OFF_TMEMADDR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + G::OFF_ABORT);
    float *Fsm = reinterpret_cast<float *>(smem + G::OFF_F);
    const AbortCtx ab{abort_flag, p.status};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg = blockIdx.x, bh = blockIdx.y;
    const long t_begin = (long)seg * p.seg_len;
    const long t_end = min((long)p.T, t_begin + p.seg_len);
    const int nch = (int)((t_end - t_begin + C - 1) / C);

    // ---------------- set-up
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < G::NKV; ++s) {
            mbar_init(&bar[G::B_KV_FULL + s], 1);
            mbar_init(&bar[G::B_KV_EMPTY + s], 1);
            mbar_init(&bar[G::B_PHI + s], 4);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar[G::B_Q_FULL + s], 1);
            mbar_init(&bar[G::B_Q_EMPTY + s], G::QT ? 4 : 1);
        }
        mbar_init(&bar[G::B_QT_EMPTY], 1);
        mbar_init(&bar[G::B_SC_FULL], 1);
        mbar_init(&bar[G::B_P_READY], 4);
        mbar_init(&bar[G::B_MMA4], 1);
        mbar_init(&bar[G::B_O_FULL], 1);
        mbar_init(&bar[G::B_O_EMPTY], 4);
        mbar_init(&bar[G::B_DS_FULL], 1);
        mbar_init(&bar[G::B_S_READY], 4);
        mbar_init(&bar[G::B_DRAIN], 1);
        fence_mbar_init();
    }
    // constant operands: all-ones [16][C] and (OUT) a zeroed z operand [16][D]
    {
        uint32_t *ones = reinterpret_cast<uint32_t *>(smem + G::OFF_ONES);
        for (int i = threadIdx.x; i < G::ONES / 4; i += kThreads) ones[i] = 0x3F803F80u;
        if constexpr (G::OUT) {
            uint32_t *zb = reinterpret_cast<uint32_t *>(smem + G::OFF_ZB);
            for (int i = threadIdx.x; i < G::ZB / 4; i += kThreads) zb[i] = 0u;
        }
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_addr_smem, G::TMEM_COLS);
    if (warp == kTmaWarp && lane == 0) {
        if constexpr (G::OUT) prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_addr_smem;
    if ((smem_u32(smem) & 1023u) != 0) raise_abort(ab, 16);  // layout assumption violated

    if (warp == kTmaWarp) {
        // ================= TMA producer
        if (lane == 0 && !*abort_flag) {
            int issued_kv[G::NKV] = {}, issued_q[2] = {};
            for (int c = 0; c < nch; ++c) {
                const int s = c % G::NKV;
                const int y = (int)(t_begin + (long)c * C);
                if constexpr (G::OUT) {
                    const int sq = G::QT ? 0 : (c & 1);
                    const int use = G::QT ? c : (c >> 1);
                    if (use > 0 && !mbar_wait(&bar[G::B_Q_EMPTY + sq], (use - 1) & 1, ab, 1)) break;
                    uint8_t *qd = smem + G::OFF_Q + sq * G::TILE;
                    mbar_expect_tx(&bar[G::B_Q_FULL + sq], G::TILE);
#pragma unroll
                    for (int b = 0; b < G::KB; ++b)
                        tma_load_3d(qd + b * G::BOXB, &tm_q, &bar[G::B_Q_FULL + sq], 64 * b, y, bh);
                    issued_q[sq] = use + 1;
                }
                const int use = c / G::NKV;
                if (use > 0 && !mbar_wait(&bar[G::B_KV_EMPTY + s], (use - 1) & 1, ab, 2)) break;
                uint8_t *kd = smem + G::OFF_KV + s * G::KV_STAGE;
                mbar_expect_tx(&bar[G::B_KV_FULL + s], 2 * G::TILE);
#pragma unroll
                for (int b = 0; b < G::KB; ++b) {
                    tma_load_3d(kd + b * G::BOXB, &tm_k, &bar[G::B_KV_FULL + s], 64 * b, y, bh);
                    tma_load_3d(kd + G::TILE + b * G::BOXB, &tm_v, &bar[G::B_KV_FULL + s], 64 * b, y, bh);
                }
                issued_kv[s] = use + 1;
            }
            if (*abort_flag) {
                // drain copies still in flight before the CTA may exit
                AbortCtx drain{abort_flag, nullptr};
                volatile int never = 0;
                AbortCtx timed{&never, nullptr};
                for (int s = 0; s < G::NKV; ++s)
                    if (issued_kv[s] > 0) mbar_wait(&bar[G::B_KV_FULL + s], (issued_kv[s] - 1) & 1, timed, 0);
                for (int s = 0; s < 2; ++s)
                    if (issued_q[s] > 0) mbar_wait(&bar[G::B_Q_FULL + s], (issued_q[s] - 1) & 1, timed, 0);
                (void)drain;
            }
        }
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer
        if (lane == 0 && !*abort_flag) {
            constexpr uint32_t ID_SC = idesc_bf16(C, C, false, false);
            constexpr uint32_t ID_INT = idesc_bf16(C, D, false, true);
            constexpr uint32_t ID_DEN = idesc_bf16(C, 16, false, false);
            constexpr uint32_t ID_DS = idesc_bf16(D, D, true, true);
            constexpr uint32_t ID_DZ = idesc_bf16(D, 16, true, false);
            constexpr uint32_t ID_PV = idesc_bf16(C, D, false, true);
            const uint32_t sb = smem_u32(smem);
            for (int c = 0; c < nch; ++c) {
                const int s = c % G::NKV;
                const uint32_t kt = sb + G::OFF_KV + s * G::KV_STAGE;   // phi(K)
                const uint32_t vt = kt + G::TILE;                        // V
                const uint32_t at = DECAY ? kt + 2 * G::TILE : kt;       // state-update A operand
                if (!mbar_wait(&bar[G::B_PHI + s], (c / G::NKV) & 1, ab, 3)) break;
                tc_fence_after();
                if constexpr (G::OUT) {
                    const uint32_t qt = sb + G::OFF_Q + (G::QT ? 0 : (c & 1)) * G::TILE;  // phi(Q) (smem)
                    // MMA1: scores = phi(Q) phi(K)^T (scores buffer free once MMA4 of c-1 is done)
                    if (c > 0 && !mbar_wait(&bar[G::B_MMA4], (c - 1) & 1, ab, 4)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = (kk >> 2) * G::BOXB + (kk & 3) * 32;
                        const uint64_t bdesc = sdesc_sw128(kt + koff, 16, 1024);
                        if constexpr (G::QT)
                            mma_ts(tmem + G::T_SC, tmem + G::T_Q + kk * 8, bdesc, ID_SC, kk > 0);
                        else
                            mma_ss(tmem + G::T_SC, sdesc_sw128(qt + koff, 16, 1024), bdesc, ID_SC, kk > 0);
                    }
                    mma_commit(&bar[G::B_SC_FULL]);
                    // MMA2 + MMAd: inter term and its denominator with the state entering c
                    if (!mbar_wait(&bar[G::B_S_READY], c & 1, ab, 5)) break;
                    if (c > 0 && !mbar_wait(&bar[G::B_O_EMPTY], (c - 1) & 1, ab, 6)) break;
                    tc_fence_after();
                    const uint32_t sbf = sb + G::OFF_SBF, zb = sb + G::OFF_ZB;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t bS = sdesc_sw128(sbf + kk * 2048, D * 128, 1024);
                        const uint64_t bZ = [&] {
                            const uint32_t a = zb + kk * 256;
                            return (uint64_t)((a >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) |
                                   ((uint64_t)(((D / 8) * 128) >> 4) << 32) | (1ull << 46);
                        }();
                        if constexpr (G::QT) {
                            mma_ts(tmem + G::T_O, tmem + G::T_Q + kk * 8, bS, ID_INT, kk > 0);
                            mma_ts(tmem + G::T_DEN, tmem + G::T_Q + kk * 8, bZ, ID_DEN, kk > 0);
                        } else {
                            const uint32_t koff = (kk >> 2) * G::BOXB + (kk & 3) * 32;
                            const uint64_t aQ = sdesc_sw128(qt + koff, 16, 1024);
                            mma_ss(tmem + G::T_O, aQ, bS, ID_INT, kk > 0);
                            mma_ss(tmem + G::T_DEN, aQ, bZ, ID_DEN, kk > 0);
                        }
                    }
                    if constexpr (G::QT) mma_commit(&bar[G::B_QT_EMPTY]);
                    else mma_commit(&bar[G::B_Q_EMPTY + (c & 1)]);
                } else {
                    if ((c == 0 || DECAY) && !mbar_wait(&bar[G::B_S_READY], c & 1, ab, 5)) break;
                    tc_fence_after();
                }
                // MMA3 + MMAz: state update with this chunk's keys and values
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t aK = sdesc_sw128(at + kk * 2048, G::BOXB, 1024);
                    const uint64_t bV = sdesc_sw128(vt + kk * 2048, G::BOXB, 1024);
                    const uint32_t oa = sb + G::OFF_ONES + kk * 256;
                    const uint64_t b1 = (uint64_t)((oa >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) |
                                        ((uint64_t)(((C / 8) * 128) >> 4) << 32) | (1ull << 46);
                    mma_ss(tmem + G::T_S, aK, bV, ID_DS, 1);
                    mma_ss(tmem + G::T_Z, aK, b1, ID_DZ, 1);
                }
                if (G::OUT || DECAY || c == nch - 1) mma_commit(&bar[G::B_DS_FULL]);
                if constexpr (G::OUT) {
                    // MMA4: exact intra-chunk product with the masked, decayed scores
                    if (!mbar_wait(&bar[G::B_P_READY], c & 1, ab, 7)) break;
                    tc_fence_after();
                    const uint32_t dst = tmem + (G::SPLIT ? G::T_O2 : G::T_O);
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk) {
                        const uint64_t bV = sdesc_sw128(vt + kk * 2048, G::BOXB, 1024);
                        if constexpr (G::PT)
                            mma_ts(dst, tmem + G::T_SC + kk * 8, bV, ID_PV, G::SPLIT ? (kk > 0) : 1);
                        else
                            mma_ss(dst, sdesc_sw128(sb + G::OFF_P + kk * 32, 16, 1024), bV, ID_PV,
                                   G::SPLIT ? (kk > 0) : 1);
                    }
                    mma_commit(&bar[G::B_MMA4]);
                    mma_commit(&bar[G::B_O_FULL]);
                }
                mma_commit(&bar[G::B_KV_EMPTY + s]);
            }
            // drain: every MMA issued by this thread has completed
            volatile int never = 0;
            AbortCtx timed{&never, nullptr};
            mma_commit(&bar[G::B_DRAIN]);
            mbar_wait(&bar[G::B_DRAIN], 0, timed, 0);
        }
    } else if (warp >= kPhiWarp0) {
        // ================= feature map, decay, state epilogue (warps 6-9)
        const int tw = threadIdx.x - kPhiWarp0 * 32;        // 0..127
        const int q = warp & 3;                              // TMEM lane quarter
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        float Aseg = 1.f;  // product of chunk decays (state-only mode)
        bool ok = true;

        // phi on one staged chunk; returns false on abort
        auto phi_chunk = [&](int c) -> bool {
            const int s = c % G::NKV;
            const long t0 = t_begin + (long)c * C;
            const int n = (int)min((long)C, t_end - t0);
            if (!mbar_wait(&bar[G::B_KV_FULL + s], (c / G::NKV) & 1, ab, 8)) return false;
            float *L = Fsm + G::F_L + s * C;
            if constexpr (DECAY) {
                if (tw < 32) {
                    const float *a = p.decay + (size_t)bh * p.T + t0;
                    float carry = 0.f;
                    for (int j0 = 0; j0 < C; j0 += 32) {
                        const int j = j0 + lane;
                        float x = (j < n) ? logf(a[j]) : 0.f;
                        x = warp_sum_scan(x, lane) + carry;
                        L[j] = x;   // rows >= n repeat the chunk total (never used)
                        carry = __shfl_sync(0xffffffffu, x, 31);
                    }
                    if (lane == 0) {
                        const float g = expf(carry);
                        Fsm[G::F_G + s] = g;
                        Aseg *= g;
                    }
                }
                named_bar_sync(1, 128);
            }
            uint8_t *kt = smem + G::OFF_KV + s * G::KV_STAGE;
            // K: phi in place (rows >= n zeroed); with decay also w o phi(K)
            {
                const int lc = tw & 7;
                constexpr int PH = 128 / (8 * G::KB);
                const int b = (tw >> 3) % G::KB, ph = tw / (8 * G::KB);
                const float Lend = DECAY ? L[n - 1] : 0.f;
                for (int r = ph; r < C; r += PH) {
                    const uint32_t off = b * G::BOXB + sw128_off(r, lc);
                    uint4 *src = reinterpret_cast<uint4 *>(kt + off);
                    float x[8];
                    unpack8<InT>(*src, x);
                    const bool valid = r < n;
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = valid ? phi_fast(x[e]) : 0.f;
                    *src = pack8_bf16(x);
                    if constexpr (DECAY) {
                        const float w = valid ? __expf(Lend - L[r]) : 0.f;
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] *= w;
                        *reinterpret_cast<uint4 *>(kt + 2 * G::TILE + off) = pack8_bf16(x);
                    }
                    if constexpr (sizeof(InT) == 2 && !std::is_same<InT, bf16>::value) {
                        // fp16 values -> bf16 operands
                        uint4 *vs = reinterpret_cast<uint4 *>(kt + G::TILE + off);
                        float y[8];
                        unpack8<InT>(*vs, y);
                        *vs = pack8_bf16(y);
                    }
                }
            }
            if constexpr (G::OUT) {
                const int sq = G::QT ? 0 : (c & 1);
                const int use = G::QT ? c : (c >> 1);
                if (!mbar_wait(&bar[G::B_Q_FULL + sq], use & 1, ab, 9)) return false;
                uint8_t *qs = smem + G::OFF_Q + sq * G::TILE;
                if constexpr (G::QT) {
                    // row i = 32q + lane: phi(q_i) -> TMEM (A operand, bf16 pairs)
                    if (c > 0 && !mbar_wait(&bar[G::B_QT_EMPTY], (c - 1) & 1, ab, 10)) return false;
                    tc_fence_after();
                    const int r = q * 32 + lane;
                    uint32_t packed[D / 2];
#pragma unroll
                    for (int b = 0; b < G::KB; ++b)
#pragma unroll
                        for (int lc = 0; lc < 8; ++lc) {
                            float x[8];
                            unpack8<InT>(*reinterpret_cast<const uint4 *>(qs + b * G::BOXB + sw128_off(r, lc)), x);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                packed[b * 32 + lc * 4 + e] = pack_bf16x2(phi_fast(x[2 * e]), phi_fast(x[2 * e + 1]));
                        }
                    // raw Q slot may be refilled
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar[G::B_Q_EMPTY]);
#pragma unroll
                    for (int h = 0; h < D / 64; ++h) {
                        uint32_t chunk32[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) chunk32[i] = packed[h * 32 + i];
                        tmem_st32(tmem + lane_base + G::T_Q + h * 32, chunk32);
                    }
                    tmem_st_wait();
                } else {
                    const int lc = tw & 7;
                    constexpr int PH = 128 / (8 * G::KB);
                    const int b = (tw >> 3) % G::KB, ph = tw / (8 * G::KB);
                    for (int r = ph; r < C; r += PH) {
                        uint4 *src = reinterpret_cast<uint4 *>(qs + b * G::BOXB + sw128_off(r, lc));
                        float x[8];
                        unpack8<InT>(*src, x);
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] = phi_fast(x[e]);
                        *src = pack8_bf16(x);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G::B_PHI + s]);
            return true;
        };

        // state rows owned by this thread: TMEM lane quarter q, rows of the
        // M = D accumulator (D = 64: lanes 0-15 of each quarter)
        constexpr int SROWS = (D == 128) ? 32 : 16;
        const bool srow_ok = lane < SROWS;
        const int a_row = q * SROWS + lane;   // state row (feature index)

        auto write_state_operands = [&](const float *srow, int col0, float zval) {
            // S row a (32 values from column col0) -> bf16 MN-major operand
            uint8_t *sbf = smem + G::OFF_SBF + (col0 / 64) * (D * 128);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = srow[8 * m + e];
                const int lcol = ((col0 % 64) / 8) + m;
                *reinterpret_cast<uint4 *>(sbf + sw128_off(a_row, lcol)) = pack8_bf16(x);
            }
            (void)zval;
        };

        if (nch > 0) ok = phi_chunk(0);
        // ---- segment start: state entering the segment -> TMEM (and operands)
        if (ok) {
            tc_fence_after();
            const float g0 = DECAY ? Fsm[G::F_G + 0] : 1.f;
            const float *st = p.ws_state + ((size_t)bh * p.n_seg + seg) * (D * D + D);
            {
#pragma unroll
                for (int cb = 0; cb < D / 32; ++cb) {
                    float vals[32];
                    uint32_t u[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        vals[i] = (G::OUT && srow_ok) ? st[(size_t)a_row * D + cb * 32 + i] : 0.f;
                        u[i] = __float_as_uint(vals[i] * g0);
                    }
                    tmem_st32(tmem + lane_base + G::T_S + cb * 32, u);
                    if constexpr (G::OUT) if (srow_ok) write_state_operands(vals, cb * 32, 0.f);
                }
                const float zin = (G::OUT && srow_ok) ? st[(size_t)D * D + a_row] : 0.f;
                uint32_t uz[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) uz[i] = __float_as_uint(zin * g0);
                asm volatile(
                    "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                    ::"r"(tmem + lane_base + G::T_Z), "r"(uz[0]), "r"(uz[1]), "r"(uz[2]), "r"(uz[3]), "r"(uz[4]),
                      "r"(uz[5]), "r"(uz[6]), "r"(uz[7]), "r"(uz[8]), "r"(uz[9]), "r"(uz[10]), "r"(uz[11]),
                      "r"(uz[12]), "r"(uz[13]), "r"(uz[14]), "r"(uz[15]) : "memory");
                if constexpr (G::OUT) {
                    if (srow_ok) {
                        // z operand: row n = 0 of the [16][D] K-major no-swizzle layout
                        bf16 *zb = reinterpret_cast<bf16 *>(smem + G::OFF_ZB);
                        zb[(a_row / 8) * 64 + (a_row % 8)] = __float2bfloat16_rn(zin);
                    }
                }
                tmem_st_wait();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G::B_S_READY]);
        }

        for (int c = 0; ok && c < nch; ++c) {
            if (c + 1 < nch) { if (!(ok = phi_chunk(c + 1))) break; }
            const bool need = G::OUT || DECAY || c == nch - 1;
            if (!need) continue;
            if (!mbar_wait(&bar[G::B_DS_FULL], (G::OUT || DECAY) ? (c & 1) : 0, ab, 11)) { ok = false; break; }
            tc_fence_after();
            const bool last = c == nch - 1;
            const float gnext = (DECAY && !last) ? Fsm[G::F_G + ((c + 1) % G::NKV)] : 1.f;
            if (last && !G::OUT) {
                // state-only mode: write the segment's (dS, dz, A) to the workspace
                float *dst = p.ws_state + ((size_t)bh * p.n_seg + seg) * (D * D + D);
#pragma unroll
                for (int cb = 0; cb < D / 32; ++cb) {
                    uint32_t u[32];
                    tmem_ld32(tmem + lane_base + G::T_S + cb * 32, u);
                    tmem_ld_wait();
                    if (srow_ok) {
                        float4 *d4 = reinterpret_cast<float4 *>(dst + (size_t)a_row * D + cb * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            d4[i] = make_float4(__uint_as_float(u[4 * i]), __uint_as_float(u[4 * i + 1]),
                                                __uint_as_float(u[4 * i + 2]), __uint_as_float(u[4 * i + 3]));
                    }
                }
                uint32_t u[32];
                tmem_ld32(tmem + lane_base + G::T_Z, u);
                tmem_ld_wait();
                if (srow_ok) dst[(size_t)D * D + a_row] = __uint_as_float(u[0]);
                if (tw == 0) p.ws_A[(size_t)bh * p.n_seg + seg] = Aseg;
                break;
            }
            if (last && G::OUT) break;   // the final state of a segment is produced by the scan
            // state entering chunk c+1: bf16 operands, and (decay) rescale in TMEM
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t u[32];
                tmem_ld32(tmem + lane_base + G::T_S + cb * 32, u);
                tmem_ld_wait();
                float vals[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) vals[i] = __uint_as_float(u[i]);
                if constexpr (G::OUT) if (srow_ok) write_state_operands(vals, cb * 32, 0.f);
                if constexpr (DECAY) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(vals[i] * gnext);
                    tmem_st32(tmem + lane_base + G::T_S + cb * 32, u);
                }
            }
            {
                uint32_t u[32];
                tmem_ld32(tmem + lane_base + G::T_Z, u);
                tmem_ld_wait();
                const float zc = __uint_as_float(u[0]);
                if constexpr (G::OUT) {
                    if (srow_ok) {
                        bf16 *zb = reinterpret_cast<bf16 *>(smem + G::OFF_ZB);
                        zb[(a_row / 8) * 64 + (a_row % 8)] = __float2bfloat16_rn(zc);
                    }
                }
                if constexpr (DECAY) {
                    uint32_t uz[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) uz[i] = __float_as_uint(zc * gnext);
                    asm volatile(
                        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                        ::"r"(tmem + lane_base + G::T_Z), "r"(uz[0]), "r"(uz[1]), "r"(uz[2]), "r"(uz[3]), "r"(uz[4]),
                          "r"(uz[5]), "r"(uz[6]), "r"(uz[7]), "r"(uz[8]), "r"(uz[9]), "r"(uz[10]), "r"(uz[11]),
                          "r"(uz[12]), "r"(uz[13]), "r"(uz[14]), "r"(uz[15]) : "memory");
                }
            }
            if constexpr (DECAY) tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G::B_S_READY]);
        }
    } else if constexpr (G::OUT) {
        // ================= epilogue (warps 0-3)
        const int q = warp;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const bool rvalid_lane = lane < G::ROWS_PER_WARP;
        const int i = q * G::ROWS_PER_WARP + lane;   // row of the chunk held by this thread
        OutT *O = reinterpret_cast<OutT *>(p.out) + (size_t)bh * p.T * D;
        for (int c = 0; c < nch; ++c) {
            const int s = c % G::NKV;
            const long t0 = t_begin + (long)c * C;
            const int n = (int)min((long)C, t_end - t0);
            if (!mbar_wait(&bar[G::B_PHI + s], (c / G::NKV) & 1, ab, 12)) break;
            if (!mbar_wait(&bar[G::B_SC_FULL], c & 1, ab, 13)) break;
            tc_fence_after();
            const float *L = Fsm + G::F_L + s * C;
            const float Li = (DECAY && rvalid_lane) ? L[min(i, C - 1)] : 0.f;
            float rowsum = 0.f;
#pragma unroll
            for (int cb = 0; cb < C / 32; ++cb) {
                uint32_t u[32];
                tmem_ld32(tmem + lane_base + G::T_SC + cb * 32, u);
                tmem_ld_wait();
                float pv[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int j = cb * 32 + k;
                    float v = (j <= i) ? __uint_as_float(u[k]) : 0.f;
                    if constexpr (DECAY) v = (j <= i) ? v * __expf(Li - L[j]) : 0.f;
                    pv[k] = v;
                    rowsum += v;
                }
                if constexpr (G::PT) {
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(pv[2 * k], pv[2 * k + 1]);
                    tmem_st16(tmem + lane_base + G::T_SC + cb * 16, pk);
                } else if (rvalid_lane) {
                    uint8_t *pr = smem + G::OFF_P;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] = pv[8 * m + e];
                        *reinterpret_cast<uint4 *>(pr + sw128_off(i, cb * 4 + m)) = pack8_bf16(x);
                    }
                }
            }
            if constexpr (G::PT) tmem_st_wait();
            else fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G::B_P_READY]);
            const float gi = DECAY ? __expf(Li) : 1.f;

            if (!mbar_wait(&bar[G::B_O_FULL], c & 1, ab, 14)) break;
            tc_fence_after();
            float den;
            {
                uint32_t u[32];
                tmem_ld32(tmem + lane_base + G::T_DEN, u);   // columns beyond 16 unused
                tmem_ld_wait();
                den = gi * __uint_as_float(u[0]) + rowsum + p.eps;
            }
            const float inv = 1.f / den;
            const bool store = rvalid_lane && i < n;
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t u[32];
                tmem_ld32(tmem + lane_base + G::T_O + cb * 32, u);
                tmem_ld_wait();
                float o[32];
                if constexpr (G::SPLIT) {
                    uint32_t u2[32];
                    tmem_ld32(tmem + lane_base + G::T_O2 + cb * 32, u2);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        o[k] = (gi * __uint_as_float(u[k]) + __uint_as_float(u2[k])) * inv;
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = __uint_as_float(u[k]) * inv;
                }
                if (store) store_row32<OutT>(O + (size_t)(t0 + i) * D + cb * 32, o);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G::B_O_EMPTY]);
        }
    }

    // ---------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, G::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace la
