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
//   MMAz  z     += (w o phi(K))^T 1                    (D x 16, K = C)   ones operand
//   MMA4  O     += P V,  P = scores o mask o decay     (C x D,  K = C)   exact intra-chunk part
//   out   = O / (den_inter + rowsum(P) + eps)
//
// ("Linear Attention" knowledge-base page, section 2 and section 3 sketches;
// the linear-attention lesson's "Implementation reality": quadratic inside a
// chunk, the state carried across chunks; the concept card's SSD variant for
// the scalar decay.)  With decay, w_j = prod_{l>j in chunk} a_l, the mask is
// 2^(L_i - L_j) for j <= i (L = chunk-local inclusive cumsum of log2 a), the
// inter term of row i is scaled by 2^(L_i), and the state is rescaled by the
// chunk's total decay before each update.  MMA1 reads the plain phi(Q) and
// phi(K); once it has, the rows of phi(K) are rescaled in place by w_j for
// MMA3/MMAz, so no second K tile is needed.  At chunk 128 the rows of phi(Q)
// are likewise rescaled by 2^(L_i) for MMA2/MMAd and one accumulator holds
// the inter and intra terms; at chunk 64 the inter term has an accumulator of
// its own and the output epilogue applies 2^(L_i) to it.
//
// The decay instantiations also serve two forms of the concept card:
// - a per-token gain b_j on the new term (the RFA gate's 1 - g): it folds
//   into the key-side log weights, Lk_j = L_j - log2 b_j, which the mask,
//   w o phi(K) and the state pass read in place of L;
// - the mLSTM read-out (flag mlstm): phi = identity and
//   out = O / max(|den|, 1).
// Their z operand of MMAd carries a hi and a lo bf16 row, so that a cancelling
// q.z keeps about 16 mantissa bits.  The state-only pass covers every segment
// but a head's last; the output pass of that segment writes the final state.
//
// Warp roles (480 threads; at most four warps share a scheduler, which caps
// registers at 128 per thread):
//   warps 0-3    epilogue: scores -> P (mask, decay, row sums), output division
//                and store.  Warp w reads TMEM lanes 32w..32w+31; at chunk 64
//                (M = 64 products, rows in lanes 0-15 of each quarter) threads
//                0-15 and 16-31 take the two column halves of the same 16 rows.
//                In the state-only pass: the second half of phi(K).  Without
//                decay at chunk 128 the P epilogue runs on warps 6-9 instead.
//   warp  4      TMA producer (one elected thread).
//   warp  5      TMEM allocator and MMA issuer (one elected thread).
//   warps 6-9    phi(Q) (into TMEM for chunk 128; with decay at chunk 128
//                then rescaled by 2^(L_i)) and the state epilogue (TMEM S ->
//                bf16 operand, decay rescale).
//   warps 10-13  decay cumsum and phi(K) (then w o phi(K) in place).
//   warp  14     TMA producer of the query tiles (output mode).
//
// Every wait is bounded (see tc_ptx.cuh); on expiry the CTA raises its abort
// flag and the call's status word (LA_ERR_TIMEOUT and the id of the wait),
// drains its copies and MMAs, frees TMEM and returns.
#pragma once
#include <type_traits>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace la {
namespace tc {

enum Mode { kStateOnly = 0, kOutput = 1 };

constexpr int kThreads = 480;
constexpr int kEpiWarp0 = 0, kTmaWarp = 4, kMmaWarp = 5, kPhiWarp0 = 6, kKWarp0 = 10, kQTmaWarp = 14;

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
    // With decay the inter term of row i is scaled by 2^(L_i): phi(Q) rows are
    // rescaled in place once MMA1 has read them, so one accumulator holds
    // inter + intra; likewise phi(K) becomes w o phi(K) in place for MMA3.
    static constexpr bool QS = OUT && DECAY;
    // Decay forms at chunk 64: the inter term and its normaliser are formed
    // from the plain phi(Q) in an accumulator of their own, and the output
    // epilogue applies 2^(L_i) in fp32 (inter * 2^(L_i) + intra), instead of
    // rescaling the phi(Q) tile in place after MMA1: the query warps are spared
    // that pass and MMA2 need not wait for it.  (Chunk 128 has no TMEM left for
    // the second accumulator and rescales phi(Q) in place.)
    static constexpr bool QSEP = QS && C == 64;
    static constexpr bool QW = QS && !QSEP;       // phi(Q) rescaled in place after MMA1
    // Output pass, no decay, chunk 128: the P epilogue (scores -> P, row sums)
    // runs on the state-epilogue warps, whose other work is light here, so the
    // output warps only read out O and the intra-chunk product of chunk c does
    // not wait for the read-out of chunk c - 1.  The row sums reach the output
    // warps through TMEM (two columns, by chunk parity).
    static constexpr bool PW = OUT && !DECAY && C == 128;
    // K/V stages: two in output mode (shared memory is full); the state-only
    // pass has room for more, which hides the load latency of its short chunks
    static constexpr int KV_BYTES = 2 * C * D * 2;
    static constexpr int NKV = OUT ? 2 : (KV_BYTES <= 48 * 1024 ? 4 : 3);
    static constexpr int NQ = OUT ? (QT ? 1 : 2) : 0;
    static constexpr int ROWS_PER_WARP = (C == 128) ? 32 : 16;   // M=64 uses lanes 0-15

    // ---- shared memory (offsets from a 1024-byte aligned base)
    static constexpr int KV_STAGE = 2 * TILE;                        // K (phi(K) in place), V
    static constexpr int OFF_KV = 0;
    static constexpr int OFF_Q = OFF_KV + NKV * KV_STAGE;
    static constexpr int OFF_SBF = OFF_Q + NQ * TILE;                // S as bf16 MMA operand
    static constexpr int SBF = OUT ? D * D * 2 : 0;
    static constexpr int OFF_P = OFF_SBF + SBF;
    static constexpr int PB = (OUT && !PT) ? C * C * 2 : 0;
    static constexpr int OFF_ZB = OFF_P + PB;                        // z as MMA operand [16][D]
    static constexpr int ZB = OUT ? 16 * D * 2 : 0;
    static constexpr int OFF_ONES = OFF_ZB + ZB;                     // ones operand [16][C] of MMAz
    static constexpr int ONES = 16 * C * 2;
    static constexpr int OFF_STG = (OFF_ONES + ONES + 1023) / 1024 * 1024;   // output staging, 4 warps x [R][128 B]
    static constexpr int STG = OUT ? 4 * ROWS_PER_WARP * 128 : 0;
    static constexpr int OFF_F = OFF_STG + STG;                      // fp32 scratch
    static constexpr int F_L = 0;                                    // [NKV][C] log2-decay cumsum
    // [NKV][C] key-side log2 weights L_j - log2 b_j when a per-token gain b is given
    static constexpr int F_LK = F_L + (DECAY ? NKV * C : 0);
    static constexpr int F_G = F_LK + (DECAY ? NKV * C : 0);         // [NKV] chunk decay
    static constexpr int F_LE = F_G + NKV;                           // [NKV] log2 weight origin
    static constexpr int F_END = F_LE + NKV;
    static constexpr int OFF_BAR = (OFF_F + F_END * 4 + 7) / 8 * 8;
    // barrier indices
    static constexpr int B_KV_FULL = 0, B_KV_EMPTY = B_KV_FULL + NKV, B_PHI = B_KV_EMPTY + NKV;
    static constexpr int B_Q_FULL = B_PHI + NKV, B_Q_EMPTY = B_Q_FULL + 2;
    static constexpr int B_QT_EMPTY = B_Q_EMPTY + 2, B_SC_FULL = B_QT_EMPTY + 1;
    static constexpr int B_P_READY = B_SC_FULL + 1, B_MMA4 = B_P_READY + 1;
    static constexpr int B_O_FULL = B_MMA4 + 1, B_O_EMPTY = B_O_FULL + 1;
    static constexpr int B_DS_FULL = B_O_EMPTY + 1, B_S_READY = B_DS_FULL + 1;
    static constexpr int B_DRAIN = B_S_READY + 1, B_KW_READY = B_DRAIN + 1, B_QS_READY = B_KW_READY + 1;
    static constexpr int B_L_READY = B_QS_READY + 1;
    static constexpr int B_V_EMPTY = B_L_READY + NKV;   // V of a stage consumed (K: B_KV_EMPTY)
    static constexpr int NBAR = B_V_EMPTY + NKV;
    static constexpr int OFF_TMEMADDR = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEMADDR + 4;
    static constexpr int OFF_END = OFF_ABORT + 4;
    static constexpr int SMEM_BYTES = OFF_END + 1024;   // + alignment slack

    // ---- TMEM columns
    static constexpr int T_SC = 0;
    static constexpr int T_O = OUT ? C : 0;
    static constexpr int T_OI = T_O + D;                      // QSEP: the inter term (D columns)
    static constexpr int T_S = T_O + (OUT ? D : 0) + (QSEP ? D : 0);
    static constexpr int T_Z = T_S + D;                       // z (column 0; MMAz accumulator)
    static constexpr int T_DEN = T_Z + 16;                    // phi(Q) z of the carried state
    static constexpr int T_Q = T_DEN + (OUT ? 16 : 0);
    static constexpr int T_RS = T_Q + (QT ? D / 2 : 0);      // row sums of P (PW), two columns
    static constexpr int T_USED = T_RS + (PW ? 2 : 0);
    static constexpr int TMEM_COLS = tmem_alloc_cols(T_USED);

    static_assert(D == 64 || D == 128, "tensor-core path: D in {64, 128}");
    static_assert(C == 64 || C == 128, "tensor-core path: chunk in {64, 128}");

    static_assert(T_USED <= 512, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(OFF_ONES % 16 == 0, "no-swizzle operand alignment");
    static_assert(OFF_STG % 1024 == 0 && OFF_SBF % 1024 == 0 && OFF_P % 1024 == 0 && OFF_ZB % 16 == 0 &&
                  OFF_Q % 1024 == 0 && KV_STAGE % 1024 == 0, "swizzled tiles need 1024-byte alignment");
};

struct TcParams {
    const float *decay;   // [BH, T] or null
    const float *gain;    // [BH, T] or null: per-token gain b_t >= 0 on the new term
    void *out;            // [BH, T, D]
    float *ws_state;      // [BH, n_seg, D*D + D]
    float *ws_A;          // [BH, n_seg]
    float *fin_S;         // [BH, D, D] or null: output mode writes the final state
    float *fin_z;         // [BH, D]      from the last segment (the scan does not)
    int *status;          // status word [2]: code (0 = ok), id of the first wait that gave up
    int T, seg_len, n_seg;
    float eps;
    int mlstm;            // 1: identity feature map and the max(|den|, 1) read-out (decay kernels only)
    unsigned long long wait_ns;   // limit of every working wait
    int flash;            // 1: the FLASH chunk form (identity feature map; kernels of form 2 and
                          //    the decay form's state-only pass)
    float inv_s;          // FLASH: 1 / the score and summary scale (1 or 1 / chunk)
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

// The state (S, z) held in TMEM (rows = feature index, one row per thread)
// to fp32 global memory: S row-major [D][D], z [D].  Out of line: it runs
// once per CTA and keeps the chunk loop's code small.
template <int D>
__device__ __noinline__ void write_final_state(uint32_t t_s, uint32_t t_z, float *S, float *z, int a_row,
                                               bool row_ok) {
    uint32_t zbits;
    tmem_ld1(t_z, zbits);
#pragma unroll 1
    for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t u[32];
        tmem_ld32(t_s + cb * 32, u);
        tmem_ld_wait();
        if (row_ok) {
            float4 *d4 = reinterpret_cast<float4 *>(S + (size_t)a_row * D + cb * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                d4[i] = make_float4(__uint_as_float(u[4 * i]), __uint_as_float(u[4 * i + 1]),
                                    __uint_as_float(u[4 * i + 2]), __uint_as_float(u[4 * i + 3]));
        }
    }
    if (row_ok) z[a_row] = __uint_as_float(zbits);
}

// z (row a of the normaliser) as the B operand of MMAd, K-major without
// swizzle, [16][D] bf16: row n = 0 holds bf16(z) and row n = 1 bf16(z -
// bf16(z)), so column 0 + column 1 of the product is phi(q).z to about 16
// mantissa bits (with the identity feature map q.z can cancel, and one bf16
// rounding of z would be amplified by it; without it the normaliser of a long
// prefill still keeps its precision).  Element (n, a) sits at
// (a / 8) * 64 + 8 n + a % 8.
template <bool HILO>
__device__ __forceinline__ void write_z_operand(bf16 *zb, int a, float z) {
    const bf16 hi = __float2bfloat16_rn(z);
    zb[(a / 8) * 64 + (a % 8)] = hi;
    if constexpr (HILO) zb[(a / 8) * 64 + 8 + (a % 8)] = __float2bfloat16_rn(z - __bfloat162float(hi));
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

// phi on a packed pair of bf16 values: phi(x) = max(x, 0) + e^(min(x, 0))
// (x + 1 for x > 0, e^x for x <= 0).  min/max/add run on the pair; e^m is
// taken as 2^(m log2 e) on the fp32 ex2 unit (measured faster here than the
// packed bf16x2 ex2) and rounded once to bf16.  For x > 0 the result is
// x + 1 rounded once to bf16.
__device__ __forceinline__ uint32_t phi_bf16x2(uint32_t x2) {
    uint32_t m, pz, r;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(x2), "r"(0u));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(pz) : "r"(x2), "r"(0u));
    const float e0 = ex2_approx(__uint_as_float(m << 16) * kLog2e);
    const float e1 = ex2_approx(__uint_as_float(m & 0xFFFF0000u) * kLog2e);
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(pz), "r"(pack_bf16x2(e0, e1)));
    return r;
}
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint4 phi_bf16x8(const uint4 &u) {
    return make_uint4(phi_bf16x2(u.x), phi_bf16x2(u.y), phi_bf16x2(u.z), phi_bf16x2(u.w));
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&x)[8]) {
    return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                      pack_bf16x2(x[6], x[7]));
}


// S row `a` (32 fp32 values from column col0) -> the bf16 MN-major operand
// [D/64 column blocks][D rows][128 bytes], 128-byte swizzled.
template <int D>
__device__ __forceinline__ void write_state_row(uint8_t *sbf, int a, int col0, const float (&vals)[32]) {
    uint8_t *blk = sbf + (col0 / 64) * (D * 128);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = vals[8 * m + e];
        *reinterpret_cast<uint4 *>(blk + sw128_off(a, ((col0 % 64) / 8) + m)) = pack8_bf16(x);
    }
}

// phi applied in place to a staged [C][D] tile (KB boxes of [C][128 B]),
// rows >= n zeroed.  With WEIGHT each row is also multiplied by
// w_r = 2^(Lend - L_r) (the state-only pass: the key's decay to the segment
// end); with FP16 inputs the V tile is converted to bf16.
// Thread tw (0..127) owns one 16-byte column chunk of one box on every PH-th
// row; with PH a multiple of 8 its swizzled chunk position is the same on
// all its rows, and all loads of a batch are issued before any arithmetic.
// The tile's rows are split into NPART equal parts; this call does parts
// [PB, PE) (the two warpgroups of the state-only pass each take half).
// With ident the feature map is the identity (the mLSTM read-out): rows are
// only weighted, zeroed past n and converted to bf16.
template <typename InT, int C, int D, bool WEIGHT, bool CONVERT_V, int PB = 0, int PE = 1, int NPART = 1>
__device__ __forceinline__ void phi_tile(uint8_t *tile, uint8_t *vt, int tw, int n, const float *L, float Lend,
                                         bool ident = false) {
    constexpr int KB = D / 64, BOXB = C * 128;
    constexpr int PH = 128 / (8 * KB);
    constexpr int NIT = C / PH;
    constexpr int IPART = NIT / NPART;
    // two rows per batch: the loop body stays small (this kernel's warp roles
    // compete for the instruction cache; measured faster than 4 or 8)
    constexpr int BATCH = IPART < 2 ? IPART : 2;
    static_assert(NIT % NPART == 0 && IPART % BATCH == 0, "row split");
    const int lc = tw & 7, b = (tw >> 3) % KB, ph = tw / (8 * KB);
    const uint32_t base = b * BOXB + ph * 128 + ((lc ^ (ph & 7)) << 4);
#pragma unroll 1
    for (int i0 = PB * IPART; i0 < PE * IPART; i0 += BATCH) {
        uint4 raw[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) raw[i] = *reinterpret_cast<const uint4 *>(tile + base + (i0 + i) * PH * 128);
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int r = ph + (i0 + i) * PH;
            const uint32_t off = base + (i0 + i) * PH * 128;
            const bool valid = r < n;
            if constexpr (std::is_same<InT, bf16>::value) {
                uint4 f = ident ? raw[i] : phi_bf16x8(raw[i]);
                if (!valid) f = make_uint4(0u, 0u, 0u, 0u);
                if constexpr (WEIGHT) {
                    const float w = valid ? ex2_approx(Lend - L[r]) : 0.f;
                    const uint32_t w2 = pack_bf16x2(w, w);
                    f = make_uint4(mul_bf16x2(f.x, w2), mul_bf16x2(f.y, w2), mul_bf16x2(f.z, w2),
                                   mul_bf16x2(f.w, w2));
                }
                *reinterpret_cast<uint4 *>(tile + off) = f;
            } else {
                float x[8];
                unpack8<InT>(raw[i], x);
                const float w = WEIGHT ? (valid ? ex2_approx(Lend - L[r]) : 0.f) : 1.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = valid ? (ident ? x[e] : phi_fast(x[e])) * w : 0.f;
                *reinterpret_cast<uint4 *>(tile + off) = pack8_bf16(x);
            }
        }
        if constexpr (CONVERT_V) {
            uint4 rv[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i) rv[i] = *reinterpret_cast<const uint4 *>(vt + base + (i0 + i) * PH * 128);
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                float y[8];
                unpack8<InT>(rv[i], y);
                *reinterpret_cast<uint4 *>(vt + base + (i0 + i) * PH * 128) = pack8_bf16(y);
            }
        }
    }
}

// Multiplies the rows of a staged bf16 [C][D] tile in place: row r by
// 2^(Lend - L_r) (KEYS: w o phi(K) for the state update, chunk-relative) or by
// 2^(L_r) (queries: the decay of the carried state at query r).  Same thread
// mapping as phi_tile, all rows, thread tw = 0..127.
template <int C, int D, bool KEYS>
__device__ __forceinline__ void scale_rows(uint8_t *tile, int tw, const float *L, float Lend) {
    constexpr int KB = D / 64, BOXB = C * 128;
    constexpr int PH = 128 / (8 * KB);
    constexpr int NIT = C / PH;
    constexpr int BATCH = NIT < 8 ? NIT : 8;
    const int lc = tw & 7, b = (tw >> 3) % KB, ph = tw / (8 * KB);
    const uint32_t base = b * BOXB + ph * 128 + ((lc ^ (ph & 7)) << 4);
#pragma unroll 1
    for (int i0 = 0; i0 < NIT; i0 += BATCH) {
        uint4 raw[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) raw[i] = *reinterpret_cast<const uint4 *>(tile + base + (i0 + i) * PH * 128);
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int r = ph + (i0 + i) * PH;
            const float w = ex2_approx(KEYS ? Lend - L[r] : L[r]);
            const uint32_t w2 = pack_bf16x2(w, w);
            const uint4 f = raw[i];
            *reinterpret_cast<uint4 *>(tile + base + (i0 + i) * PH * 128) =
                make_uint4(mul_bf16x2(f.x, w2), mul_bf16x2(f.y, w2), mul_bf16x2(f.z, w2), mul_bf16x2(f.w, w2));
        }
    }
}

// The chunk handled at step c: output mode walks the segment forwards (the
// state is carried), the state-only pass walks it backwards so that the
// decay from each key to the segment's end is known when its chunk is read.
template <bool OUT> __device__ __forceinline__ int chunk_at(int c, int nch) { return OUT ? c : nch - 1 - c; }

// Decay cumsum of chunk c by one warp: L_j (chunk-local inclusive cumsum of
// log2 a) to shared memory, the chunk decay g = 2^(L_end) and the weight
// origin; arrives on l_ready.  With a per-token gain b (which scales key j's
// new term), the key-side weights use Lk_j = L_j - log2 b_j instead of L_j:
// every weight a key receives, 2^(x - L_j), becomes b_j 2^(x - L_j)
// (b_j = 0 gives Lk_j = +inf and the weight 0).  Without decay (gain only)
// a = 1.  The decays (and gains) of chunk c were loaded into registers
// during chunk c-1; the loads of the next chunk start here so their latency
// is hidden.  The caller has waited until the stage's L slot is free.
template <int C, int D, bool DECAY, int MODE>
__device__ __forceinline__ void decay_cumsum(uint64_t *bar, float *Fsm, const TcParams &p, long t_begin,
                                             long t_end, int bh, int c, int nch, int lane, float &Aseg,
                                             float (&apre)[C / 32], float (&bpre)[C / 32], float &lam) {
    using G = Cfg<C, D, DECAY, MODE>;
    const int s = c % G::NKV;
    const long t0 = t_begin + (long)chunk_at<G::OUT>(c, nch) * C;
    const int n = (int)min((long)C, t_end - t0);
    float *L = Fsm + G::F_L + s * C;
    const bool has_a = p.decay != nullptr, has_b = p.gain != nullptr;
    const float *a = has_a ? p.decay + (size_t)bh * p.T + t0 : nullptr;
    const float *bg = has_b ? p.gain + (size_t)bh * p.T + t0 : nullptr;
    float cur[C / 32], bcur[C / 32];
#pragma unroll
    for (int h = 0; h < C / 32; ++h) {
        const int j = h * 32 + lane;
        cur[h] = (c == 0) ? ((has_a && j < n) ? a[j] : 1.f) : apre[h];
        bcur[h] = (c == 0) ? ((has_b && j < n) ? bg[j] : 1.f) : bpre[h];
    }
    if (c + 1 < nch) {
        const long t1 = t_begin + (long)chunk_at<G::OUT>(c + 1, nch) * C;
        const int n1 = (int)min((long)C, t_end - t1);
        const float *a1 = has_a ? p.decay + (size_t)bh * p.T + t1 : nullptr;
        const float *b1 = has_b ? p.gain + (size_t)bh * p.T + t1 : nullptr;
#pragma unroll
        for (int h = 0; h < C / 32; ++h) {
            const int j = h * 32 + lane;
            apre[h] = (has_a && j < n1) ? a1[j] : 1.f;
            bpre[h] = (has_b && j < n1) ? b1[j] : 1.f;
        }
    }
    float carry = 0.f;
#pragma unroll
    for (int h = 0; h < C / 32; ++h) {
        const int j = h * 32 + lane;
        float x = (j < n) ? lg2_approx(cur[h]) : 0.f;   // log2 units
        x = warp_sum_scan(x, lane) + carry;
        L[j] = x;   // rows >= n repeat the chunk total (never used)
        if (has_b) Fsm[G::F_LK + s * C + j] = x - lg2_approx(bcur[h]);
        carry = __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) {
        const float g = ex2_approx(carry);
        Fsm[G::F_G + s] = g;
        Aseg *= g;
        // weights w_j = 2^(origin - L_j): the chunk's end in output mode; in
        // state-only mode the segment's end (lam = log2 decay of the chunks
        // after this one, all processed already)
        Fsm[G::F_LE + s] = G::OUT ? carry : carry + lam;
        lam += carry;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar[G::B_L_READY + s]);
}

// Key-side log2 weights of stage s: L, or L - log2 b with a gain.
template <int C, int D, bool DECAY, int MODE>
__device__ __forceinline__ const float *key_log_weights(const float *Fsm, const TcParams &p, int s) {
    using G = Cfg<C, D, DECAY, MODE>;
    return Fsm + (p.gain ? G::F_LK : G::F_L) + s * C;
}

// Keys of chunk c (K warpgroup, thread index tk = 0..127): phi(K) in place (in
// output mode all key rows, in state-only mode the first half, weighted by
// the decay to the segment end; warps 0-3 take the rest); in output mode
// with decay, warp 0 then forms the chunk's decay cumsum.
// Arrives on phi_done.  Returns false if the CTA is aborting.
template <int C, int D, bool DECAY, int MODE, typename InT>
__device__ __forceinline__ bool k_stage(uint8_t *smem, uint64_t *bar, float *Fsm, const AbortCtx ab,
                                        const TcParams &p, long t_begin, long t_end, int bh, int c,
                                        int nch, int tk, float &Aseg, float (&apre)[C / 32],
                                        float (&bpre)[C / 32], float &lam) {
    using G = Cfg<C, D, DECAY, MODE>;
    const int lane = tk & 31;
    const int s = c % G::NKV;
    const long t0 = t_begin + (long)chunk_at<G::OUT>(c, nch) * C;
    const int n = (int)min((long)C, t_end - t0);
    if (!mbar_wait(&bar[G::B_KV_FULL + s], (c / G::NKV) & 1, ab, 8)) return false;
    const float *Lk = key_log_weights<C, D, DECAY, MODE>(Fsm, p, s);
    // state-only mode: the weights need the decay cumsum, which the idle phi(Q)
    // warps compute ahead of the key warps
    if constexpr (DECAY && !G::OUT)
        if (!mbar_wait(&bar[G::B_L_READY + s], (c / G::NKV) & 1, ab, 29)) return false;
    uint8_t *kt = smem + G::OFF_KV + s * G::KV_STAGE;
    constexpr bool CONV = !std::is_same<InT, bf16>::value;
    const float Lend = DECAY ? Fsm[G::F_LE + s] : 0.f;
    // output mode: plain phi(K) (MMA1 needs it; the decay weights are applied
    // in place after MMA1, see k_weight); state-only: w o phi(K) directly
    if constexpr (G::OUT)
        phi_tile<InT, C, D, false, CONV, 0, 1, 1>(kt, kt + G::TILE, tk, n, Lk, Lend, DECAY && (p.mlstm || p.flash));
    else
        phi_tile<InT, C, D, DECAY, CONV, 0, 2, 4>(kt, kt + G::TILE, tk, n, Lk, Lend, DECAY && (p.mlstm || p.flash));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar[G::B_PHI + s]);
    // output mode: phi(K) did not need the decays; the cumsum follows it (warp 0)
    if constexpr (DECAY && G::OUT)
        if (tk < 32)
            decay_cumsum<C, D, DECAY, MODE>(bar, Fsm, p, t_begin, t_end, bh, c, nch, lane, Aseg, apre, bpre, lam);
    return true;
}

// Queries of chunk c (phi warpgroup, output mode, tw = 0..127): phi(Q) into
// TMEM as the A operand (chunk 128: row r = 32q + lane, the thread's TMEM lane)
// or in place in shared memory (chunk 64).  Arrives on phi_done.
template <int C, int D, bool DECAY, int MODE, typename InT>
__device__ __forceinline__ bool q_stage(uint8_t *smem, uint64_t *bar, const AbortCtx ab, uint32_t tmem,
                                        int c, int tw, bool ident) {
    using G = Cfg<C, D, DECAY, MODE>;
    const int lane = tw & 31, q = (kPhiWarp0 + (tw >> 5)) & 3;
    const int s = c % G::NKV;
    const int sq = G::QT ? 0 : (c & 1);
    const int use = G::QT ? c : (c >> 1);
    if (!mbar_wait(&bar[G::B_Q_FULL + sq], use & 1, ab, 9)) return false;
    uint8_t *qs = smem + G::OFF_Q + sq * G::TILE;
    if constexpr (G::QT) {
        const int r = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
#pragma unroll 1
        for (int b = 0; b < G::KB; ++b) {
            uint4 raw[8];
#pragma unroll
            for (int lc = 0; lc < 8; ++lc)
                raw[lc] = *reinterpret_cast<const uint4 *>(qs + b * G::BOXB + sw128_off(r, lc));
            uint32_t packed[32];
#pragma unroll
            for (int lc = 0; lc < 8; ++lc) {
                if constexpr (std::is_same<InT, bf16>::value) {
                    const uint4 f = ident ? raw[lc] : phi_bf16x8(raw[lc]);
                    packed[lc * 4 + 0] = f.x;
                    packed[lc * 4 + 1] = f.y;
                    packed[lc * 4 + 2] = f.z;
                    packed[lc * 4 + 3] = f.w;
                } else {
                    float x[8];
                    unpack8<InT>(raw[lc], x);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        packed[lc * 4 + e] = ident ? pack_bf16x2(x[2 * e], x[2 * e + 1])
                                                   : pack_bf16x2(phi_fast(x[2 * e]), phi_fast(x[2 * e + 1]));
                }
            }
            if (b == G::KB - 1) {
                // this warp's reads of the raw Q slot are done
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[G::B_Q_EMPTY]);
            }
            if (b == 0) {
                if (c > 0 && !mbar_wait(&bar[G::B_QT_EMPTY], (c - 1) & 1, ab, 10)) return false;
                tc_fence_after();
            }
            tmem_st32(tmem + lane_base + G::T_Q + b * 32, packed);
        }
        tmem_st_wait();
    } else {
        phi_tile<InT, C, D, false, false>(qs, nullptr, tw, C, nullptr, 0.f, ident);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar[G::B_PHI + s]);
    return true;
}

// Output mode with decay, keys of chunk c once MMA1 has read phi(K): the tile
// becomes w o phi(K) in place (w_j = 2^(L_end - L_j)) for MMA3; arrives on
// kw_ready.  False if aborting.
template <int C, int D, bool DECAY, int MODE>
__device__ __forceinline__ bool k_weight(uint8_t *smem, uint64_t *bar, float *Fsm, const TcParams &p,
                                         const AbortCtx ab, int c, int tk) {
    using G = Cfg<C, D, DECAY, MODE>;
    const int s = c % G::NKV;
    if (!mbar_wait(&bar[G::B_SC_FULL], c & 1, ab, 21)) return false;
    if (!mbar_wait(&bar[G::B_L_READY + s], (c / G::NKV) & 1, ab, 30)) return false;
    scale_rows<C, D, true>(smem + G::OFF_KV + s * G::KV_STAGE, tk, key_log_weights<C, D, DECAY, MODE>(Fsm, p, s),
                           Fsm[G::F_LE + s]);
    fence_proxy_async_smem();
    __syncwarp();
    if ((tk & 31) == 0) mbar_arrive(&bar[G::B_KW_READY]);
    return true;
}

// Output mode with decay, queries of chunk c once MMA1 has read phi(Q): row i
// is scaled by 2^(L_i) (the decay of the carried state at query i) for MMA2
// and MMAd — in TMEM (chunk 128: this thread's row) or in shared memory
// (chunk 64).  Arrives on qs_ready.  False if aborting.
template <int C, int D, bool DECAY, int MODE>
__device__ __forceinline__ bool q_weight(uint8_t *smem, uint64_t *bar, float *Fsm, const AbortCtx ab,
                                         uint32_t tmem, int c, int tw) {
    using G = Cfg<C, D, DECAY, MODE>;
    const int lane = tw & 31, q = (kPhiWarp0 + (tw >> 5)) & 3;
    const int s = c % G::NKV;
    if (!mbar_wait(&bar[G::B_SC_FULL], c & 1, ab, 22)) return false;
    if (!mbar_wait(&bar[G::B_L_READY + s], (c / G::NKV) & 1, ab, 23)) return false;
    const float *L = Fsm + G::F_L + s * C;
    tc_fence_after();
    if constexpr (G::QT) {
        const int r = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float w = ex2_approx(L[r]);
        const uint32_t w2 = pack_bf16x2(w, w);
#pragma unroll 1
        for (int b = 0; b < G::KB; ++b) {
            uint32_t u[32];
            tmem_ld32(tmem + lane_base + G::T_Q + b * 32, u);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) u[k] = mul_bf16x2(u[k], w2);
            tmem_st32(tmem + lane_base + G::T_Q + b * 32, u);
        }
        tmem_st_wait();
    } else {
        scale_rows<C, D, false>(smem + G::OFF_Q + (c & 1) * G::TILE, tw, L, 0.f);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar[G::B_QS_READY]);
    return true;
}

// State-only mode: second half of the key rows of chunk c, done by warps
// 0-3 (thread index et = 0..127); arrives on phi_done.  False if aborting.
template <int C, int D, bool DECAY, int MODE, typename InT>
__device__ __forceinline__ bool phi_keys_second_half(uint8_t *smem, uint64_t *bar, float *Fsm,
                                                     const TcParams &p, const AbortCtx ab, long t_begin,
                                                     long t_end, int c, int nch, int et) {
    using G = Cfg<C, D, DECAY, MODE>;
    const int s = c % G::NKV;
    const long t0 = t_begin + (long)chunk_at<G::OUT>(c, nch) * C;
    const int n = (int)min((long)C, t_end - t0);
    if (!mbar_wait(&bar[G::B_KV_FULL + s], (c / G::NKV) & 1, ab, 15)) return false;
    const float *L = key_log_weights<C, D, DECAY, MODE>(Fsm, p, s);
    if constexpr (DECAY)
        if (!mbar_wait(&bar[G::B_L_READY + s], (c / G::NKV) & 1, ab, 16)) return false;
    uint8_t *kt = smem + G::OFF_KV + s * G::KV_STAGE;
    constexpr bool CONV = !std::is_same<InT, bf16>::value;
    phi_tile<InT, C, D, DECAY, CONV, 2, 4, 4>(kt, kt + G::TILE, et, n, L, DECAY ? Fsm[G::F_LE + s] : 0.f,
                                              DECAY && (p.mlstm || p.flash));
    fence_proxy_async_smem();
    __syncwarp();
    if ((et & 31) == 0) mbar_arrive(&bar[G::B_PHI + s]);
    return true;
}

// ---------------------------------------------------------------------------
// FORM: 0 = no decay, 1 = decay (also the gated and mLSTM forms), 2 = the
// FLASH chunk form (the decay form's machinery with a = 1 and the identity
// feature map; scores -> relu(score / s)^2 inside the chunk, the carried
// summaries read as S / s, no normaliser).
// Scores -> P of chunk c for the TMEM lane quarter q (this warp's rows): the
// mask (and decay, or FLASH's squared ReLU), P packed to bf16 (TMEM for chunk
// 128, shared memory for chunk 64) and the row sums; arrives on p_ready.
// With RS_TMEM the row sum also goes to TMEM column T_RS + (c & 1), for an
// output epilogue run by other warps.  False if aborting.
template <int C, int D, int FORM, int MODE, bool RS_TMEM>
__device__ __forceinline__ bool p_epilogue(uint8_t *smem, uint64_t *bar, float *Fsm, const TcParams &p,
                                           const AbortCtx ab, uint32_t tmem, int c, int q, int lane,
                                           float &rowsum, float &li_out) {
    constexpr bool DECAY = FORM != 0;
    constexpr bool FLASH = FORM == 2;
    using G = Cfg<C, D, DECAY, MODE>;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    // HS (chunk 64): threads 0-15 and 16-31 hold the low and high 16 columns
    // of each 32-column block of the same row
    constexpr bool HS = G::ROWS_PER_WARP == 16;
    constexpr int NV = HS ? 16 : 32;                          // values per thread per block
    const int hc = HS ? (lane >> 4) * 16 : 0;                 // this thread's column offset in a block
    const int i = q * G::ROWS_PER_WARP + (HS ? (lane & 15) : lane);   // row of the chunk held by this thread
    const int s = c % G::NKV;
    rowsum = 0.f;
    if (!mbar_wait(&bar[G::B_PHI + s], (c / G::NKV) & 1, ab, 12)) return false;
    if (!mbar_wait(&bar[G::B_SC_FULL], c & 1, ab, 13)) return false;
    if (DECAY && !mbar_wait(&bar[G::B_L_READY + s], (c / G::NKV) & 1, ab, 28)) return false;
    tc_fence_after();
    const float *L = Fsm + G::F_L + s * C;
    const float *Lk = key_log_weights<C, D, DECAY, MODE>(Fsm, p, s);   // key side (gain folded in)
    const float Li = DECAY ? L[i] : 0.f;
    li_out = Li;
    // scores -> P, one 32-column block per TMEM round trip (small code;
    // measured faster than two).  For this warp's rows [r0, r0 + R) a
    // block lies fully below the diagonal (no mask), fully above it
    // (P = 0, scores not read) or on it.
    const int r0 = q * G::ROWS_PER_WARP, r1 = r0 + G::ROWS_PER_WARP - 1;
#pragma unroll 1
    for (int cb0 = 0; cb0 < C / 32; cb0 += 1) {
        uint32_t u[1][NV];
        bool live[1];
#pragma unroll
        for (int h = 0; h < 1; ++h) {
            live[h] = (cb0 + h) * 32 <= r1;
            if (live[h]) {
                if constexpr (HS) tmem_ld16x2<16>(tmem + lane_base + G::T_SC + (cb0 + h) * 32, u[h]);
                else tmem_ld32(tmem + lane_base + G::T_SC + (cb0 + h) * 32, u[h]);
            }
        }
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 1; ++h) {
            const int cb = cb0 + h;
            uint32_t pk[NV / 2];
            if (!live[h]) {
#pragma unroll
                for (int k = 0; k < NV / 2; ++k) pk[k] = 0u;
            } else {
                const bool full = cb * 32 + 31 < r0;   // every j < every row of the warp
#pragma unroll
                for (int k = 0; k < NV / 2; ++k) {
                    const int j = cb * 32 + hc + 2 * k;
                    float v0 = __uint_as_float(u[h][2 * k]), v1 = __uint_as_float(u[h][2 * k + 1]);
                    if constexpr (FLASH) {
                        // exact squared-ReLU weight of the chunk form
                        v0 = fmaxf(v0 * p.inv_s, 0.f);
                        v1 = fmaxf(v1 * p.inv_s, 0.f);
                        v0 *= v0;
                        v1 *= v1;
                    } else if constexpr (DECAY) {
                        v0 *= ex2_approx(Li - Lk[j]);
                        v1 *= ex2_approx(Li - Lk[j + 1]);
                    }
                    v0 = (full || j <= i) ? v0 : 0.f;
                    v1 = (full || j + 1 <= i) ? v1 : 0.f;
                    rowsum += v0 + v1;
                    pk[k] = pack_bf16x2(v0, v1);
                }
            }
            if constexpr (G::PT) {
                tmem_st16(tmem + lane_base + G::T_SC + cb * 16, pk);
            } else {
                uint8_t *pr = smem + G::OFF_P;
#pragma unroll
                for (int m = 0; m < NV / 8; ++m)
                    *reinterpret_cast<uint4 *>(pr + sw128_off(i, cb * 4 + hc / 8 + m)) =
                        make_uint4(pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
            }
        }
    }
    if constexpr (HS) rowsum += __shfl_xor_sync(0xffffffffu, rowsum, 16);   // both column halves
    if constexpr (G::PT) tmem_st_wait();
    else fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if constexpr (RS_TMEM) {
        // the row sum for the output epilogue, in a TMEM column by chunk parity
        tmem_st1(tmem + lane_base + G::T_RS + (c & 1), __float_as_uint(rowsum));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
    }
    if (lane == 0) mbar_arrive(&bar[G::B_P_READY]);
    return true;
}

template <int C, int D, int FORM, int MODE, typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
tc_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  TcParams p) {
    constexpr bool DECAY = FORM != 0;
    constexpr bool FLASH = FORM == 2;
    using G = Cfg<C, D, DECAY, MODE>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + G::OFF_BAR);
    uint32_t *tmem_addr_smem = reinterpret_cast<uint32_t *>(smem + G::OFF_TMEMADDR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + G::OFF_ABORT);
    float *Fsm = reinterpret_cast<float *>(smem + G::OFF_F);
    const AbortCtx ab{abort_flag, p.status, p.wait_ns};

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
            mbar_init(&bar[G::B_V_EMPTY + s], 1);
            mbar_init(&bar[G::B_PHI + s], 8);   // key warps + (query warps | warps 0-3)
            mbar_init(&bar[G::B_L_READY + s], 1);
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
        mbar_init(&bar[G::B_KW_READY], 4);   // key warps
        mbar_init(&bar[G::B_QS_READY], 4);   // query warps
        fence_mbar_init();
    }
    // (output mode) the z operand [16][D] starts zeroed: only its row 0 is used;
    // the ones operand of MMAz is all ones (every column of its result is z)
    {
        if constexpr (G::OUT) {
            uint32_t *zb = reinterpret_cast<uint32_t *>(smem + G::OFF_ZB);
            for (int i = threadIdx.x; i < G::ZB / 4; i += kThreads) zb[i] = 0u;
        }
        uint32_t *ones = reinterpret_cast<uint32_t *>(smem + G::OFF_ONES);
        for (int i = threadIdx.x; i < G::ONES / 4; i += kThreads) ones[i] = 0x3F803F80u;   // bf16 1.0 pairs
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_addr_smem, G::TMEM_COLS);
    if (warp == kTmaWarp && lane == 0) {
        if constexpr (G::OUT) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_o);
        }
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_addr_smem;
    if ((smem_u32(smem) & 1023u) != 0) raise_abort(ab, 99, kStatusLayout);  // layout assumption violated

    if (warp == kQTmaWarp) {
        // ================= TMA producer of the query tiles (output mode): its
        // own thread, so that a query slot that frees late does not hold back
        // the key and value loads
        if constexpr (G::OUT) {
            if (lane == 0 && !*abort_flag) {
                int issued_q[2] = {};
                for (int c = 0; c < nch; ++c) {
                    const int y = (int)(t_begin + (long)c * C);
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
                if (*abort_flag) {
                    volatile int never = 0;
                    AbortCtx timed{&never, nullptr, kDrainLimitNs};
                    for (int s = 0; s < 2; ++s)
                        if (issued_q[s] > 0) mbar_wait(&bar[G::B_Q_FULL + s], (issued_q[s] - 1) & 1, timed, 0);
                }
            }
        }
    } else if (warp == kTmaWarp) {
        // ================= TMA producer of the key and value tiles: a stage's
        // K is reloaded once its last reader (MMA3/MMAz) is done, its V once
        // MMA4 is; one full barrier counts both
        if (lane == 0 && !*abort_flag) {
            int issued_kv[G::NKV] = {};
            for (int c = 0; c < nch; ++c) {
                const int s = c % G::NKV;
                const int y = (int)(t_begin + (long)chunk_at<G::OUT>(c, nch) * C);
                const int use = c / G::NKV;
                if (use > 0 && !mbar_wait(&bar[G::B_KV_EMPTY + s], (use - 1) & 1, ab, 2)) break;
                uint8_t *kd = smem + G::OFF_KV + s * G::KV_STAGE;
                mbar_expect_tx(&bar[G::B_KV_FULL + s], 2 * G::TILE);
                issued_kv[s] = use + 1;
#pragma unroll
                for (int b = 0; b < G::KB; ++b)
                    tma_load_3d(kd + b * G::BOXB, &tm_k, &bar[G::B_KV_FULL + s], 64 * b, y, bh);
                if (use > 0 && !mbar_wait(&bar[G::B_V_EMPTY + s], (use - 1) & 1, ab, 26)) break;
#pragma unroll
                for (int b = 0; b < G::KB; ++b)
                    tma_load_3d(kd + G::TILE + b * G::BOXB, &tm_v, &bar[G::B_KV_FULL + s], 64 * b, y, bh);
            }
            if (*abort_flag) {
                // drain copies still in flight before the CTA may exit (a stage
                // whose V was never issued completes no phase: its wait gives up
                // after the fixed bound)
                volatile int never = 0;
                AbortCtx timed{&never, nullptr, kDrainLimitNs};
                for (int s = 0; s < G::NKV; ++s)
                    if (issued_kv[s] > 0) mbar_wait(&bar[G::B_KV_FULL + s], (issued_kv[s] - 1) & 1, timed, 0);
            }
        }
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer
        if (lane == 0 && !*abort_flag) {
            constexpr uint32_t ID_SC = idesc_bf16(C, C, false, false);
            constexpr uint32_t ID_INT = idesc_bf16(C, D, false, true);
            constexpr uint32_t ID_DEN = idesc_bf16(C, 16, false, false);
            constexpr uint32_t ID_DS = idesc_bf16(D, D, true, true);
            constexpr uint32_t ID_PV = idesc_bf16(C, D, false, true);
            constexpr uint32_t ID_Z = idesc_bf16(D, 16, true, false);
            const uint32_t sb = smem_u32(smem);
            // Base descriptors; a K-step advances the start address field
            // (address >> 4 in the low 14 bits, which never carries here:
            // shared memory is < 256 KB), so descriptor + (offset >> 4).
            auto nosw = [](uint32_t addr, uint32_t sbo) -> uint64_t {   // no-swizzle K-major
                return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) |
                       ((uint64_t)(sbo >> 4) << 32) | (1ull << 46);
            };
            const uint64_t dS0 = sdesc_sw128(sb + G::OFF_SBF, D * 128, 1024);   // S (MN-major)
            const uint64_t dZ0 = nosw(sb + G::OFF_ZB, (D / 8) * 128);           // z [16][D]
            const uint64_t dP0 = sdesc_sw128(sb + G::OFF_P, 16, 1024);          // P (K-major, smem)
            const uint64_t dOnes = nosw(sb + G::OFF_ONES, (C / 8) * 128);       // ones [16][C]
            for (int c = 0; c < nch; ++c) {
                const int s = c % G::NKV;
                const uint32_t kt = sb + G::OFF_KV + s * G::KV_STAGE;   // phi(K)
                const uint64_t dKk = sdesc_sw128(kt, 16, 1024);                        // phi(K), K-major
                const uint64_t dKm = sdesc_sw128(kt, G::BOXB, 1024);                   // (w o) phi(K), MN-major
                const uint64_t dVm = sdesc_sw128(kt + G::TILE, G::BOXB, 1024);         // V, MN-major
                if (!mbar_wait(&bar[G::B_PHI + s], (c / G::NKV) & 1, ab, 3)) break;
                tc_fence_after();
                if constexpr (G::OUT && !DECAY) {
                    // No decay: the state update (MMA3, MMAz) is issued right after
                    // the scores, ahead of the inter term, so it runs while the
                    // previous chunk's output is still being read out of the O
                    // accumulator.  The state epilogue then waits for MMA2/MMAd as
                    // well (DS_FULL is committed after them): it rewrites the
                    // operands they read.
                    const uint64_t dQk = sdesc_sw128(sb + G::OFF_Q + (G::QT ? 0 : (c & 1)) * G::TILE, 16, 1024);
                    // MMA1: scores = phi(Q) phi(K)^T (scores buffer free once MMA4 of c-1 is done)
                    if (c > 0 && !mbar_wait(&bar[G::B_MMA4], (c - 1) & 1, ab, 4)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = ((kk >> 2) * G::BOXB + (kk & 3) * 32) >> 4;
                        if constexpr (G::QT)
                            mma_ts(tmem + G::T_SC, tmem + G::T_Q + kk * 8, dKk + koff, ID_SC, kk > 0);
                        else
                            mma_ss(tmem + G::T_SC, dQk + koff, dKk + koff, ID_SC, kk > 0);
                    }
                    mma_commit(&bar[G::B_SC_FULL]);
                    // MMA3 + MMAz: the state epilogue of c-1 has read the accumulators
                    if (!mbar_wait(&bar[G::B_S_READY], c & 1, ab, 5)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_ss(tmem + G::T_S, dKm + (uint64_t)((kk * 2048) >> 4),
                               dVm + (uint64_t)((kk * 2048) >> 4), ID_DS, 1);
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_ss(tmem + G::T_Z, dKm + (uint64_t)((kk * 2048) >> 4),
                               dOnes + (uint64_t)((kk * 256) >> 4), ID_Z, 1);
                    mma_commit(&bar[G::B_KV_EMPTY + s]);   // the keys' last readers are issued
                    // MMA2 + MMAd: O is free once the output of c-1 has been read
                    if (c > 0 && !mbar_wait(&bar[G::B_O_EMPTY], (c - 1) & 1, ab, 6)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t bS = dS0 + (uint64_t)((kk * 2048) >> 4);
                        const uint64_t bZ = dZ0 + (uint64_t)((kk * 256) >> 4);
                        if constexpr (G::QT) {
                            mma_ts(tmem + G::T_O, tmem + G::T_Q + kk * 8, bS, ID_INT, kk > 0);
                            mma_ts(tmem + G::T_DEN, tmem + G::T_Q + kk * 8, bZ, ID_DEN, kk > 0);
                        } else {
                            const uint64_t aQ = dQk + (uint64_t)(((kk >> 2) * G::BOXB + (kk & 3) * 32) >> 4);
                            mma_ss(tmem + G::T_O, aQ, bS, ID_INT, kk > 0);
                            mma_ss(tmem + G::T_DEN, aQ, bZ, ID_DEN, kk > 0);
                        }
                    }
                    if constexpr (G::QT) mma_commit(&bar[G::B_QT_EMPTY]);
                    else mma_commit(&bar[G::B_Q_EMPTY + (c & 1)]);
                    mma_commit(&bar[G::B_DS_FULL]);
                    // MMA4: exact intra-chunk product with the masked scores
                    if (!mbar_wait(&bar[G::B_P_READY], c & 1, ab, 7)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk) {
                        const uint64_t bV = dVm + (uint64_t)((kk * 2048) >> 4);
                        if constexpr (G::PT)
                            mma_ts(tmem + G::T_O, tmem + G::T_SC + kk * 8, bV, ID_PV, 1u);
                        else
                            mma_ss(tmem + G::T_O, dP0 + (uint64_t)((kk * 32) >> 4), bV, ID_PV, 1u);
                    }
                    mma_commit(&bar[G::B_MMA4]);
                    mma_commit(&bar[G::B_O_FULL]);
                    mma_commit(&bar[G::B_V_EMPTY + s]);
                    continue;
                }
                if constexpr (G::OUT) {
                    const uint64_t dQk = sdesc_sw128(sb + G::OFF_Q + (G::QT ? 0 : (c & 1)) * G::TILE, 16, 1024);
                    // MMA1: scores = phi(Q) phi(K)^T (scores buffer free once MMA4 of c-1 is done)
                    if (c > 0 && !mbar_wait(&bar[G::B_MMA4], (c - 1) & 1, ab, 4)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = ((kk >> 2) * G::BOXB + (kk & 3) * 32) >> 4;
                        if constexpr (G::QT)
                            mma_ts(tmem + G::T_SC, tmem + G::T_Q + kk * 8, dKk + koff, ID_SC, kk > 0);
                        else
                            mma_ss(tmem + G::T_SC, dQk + koff, dKk + koff, ID_SC, kk > 0);
                    }
                    mma_commit(&bar[G::B_SC_FULL]);
                    // MMA2 + MMAd: inter term and its denominator with the state entering c
                    // (with decay: from the 2^(L_i)-scaled phi(Q))
                    if (!mbar_wait(&bar[G::B_S_READY], c & 1, ab, 5)) break;
                    if (c > 0 && !mbar_wait(&bar[G::B_O_EMPTY], (c - 1) & 1, ab, 6)) break;
                    if (G::QW && !mbar_wait(&bar[G::B_QS_READY], c & 1, ab, 24)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t bS = dS0 + (uint64_t)((kk * 2048) >> 4);
                        const uint64_t bZ = dZ0 + (uint64_t)((kk * 256) >> 4);
                        if constexpr (G::QT) {
                            mma_ts(tmem + G::T_O, tmem + G::T_Q + kk * 8, bS, ID_INT, kk > 0);
                            mma_ts(tmem + G::T_DEN, tmem + G::T_Q + kk * 8, bZ, ID_DEN, kk > 0);
                        } else {
                            const uint64_t aQ = dQk + (uint64_t)(((kk >> 2) * G::BOXB + (kk & 3) * 32) >> 4);
                            mma_ss(tmem + (G::QSEP ? G::T_OI : G::T_O), aQ, bS, ID_INT, kk > 0);
                            mma_ss(tmem + G::T_DEN, aQ, bZ, ID_DEN, kk > 0);
                        }
                    }
                    if constexpr (G::QT) mma_commit(&bar[G::B_QT_EMPTY]);
                    else mma_commit(&bar[G::B_Q_EMPTY + (c & 1)]);
                } else {
                    if (c == 0 && !mbar_wait(&bar[G::B_S_READY], 0, ab, 5)) break;
                    tc_fence_after();
                }
                // MMA3 + MMAz: state update with this chunk's keys and values
                if (G::QS) {
                    if (!mbar_wait(&bar[G::B_KW_READY], c & 1, ab, 25)) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_ss(tmem + G::T_S, dKm + (uint64_t)((kk * 2048) >> 4),
                           dVm + (uint64_t)((kk * 2048) >> 4), ID_DS, 1);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_ss(tmem + G::T_Z, dKm + (uint64_t)((kk * 2048) >> 4),
                           dOnes + (uint64_t)((kk * 256) >> 4), ID_Z, 1);
                if (G::OUT || c == nch - 1) mma_commit(&bar[G::B_DS_FULL]);
                if constexpr (G::OUT) {
                    // MMA4: exact intra-chunk product with the masked, decayed scores
                    if (!mbar_wait(&bar[G::B_P_READY], c & 1, ab, 7)) break;
                    tc_fence_after();
                    // O (+)= P V  (QSEP: O = P V, the inter term has its own accumulator)
                    const uint32_t dst = tmem + G::T_O;
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk) {
                        const uint64_t bV = dVm + (uint64_t)((kk * 2048) >> 4);
                        const uint32_t acc = (G::QSEP && kk == 0) ? 0u : 1u;
                        if constexpr (G::PT)
                            mma_ts(dst, tmem + G::T_SC + kk * 8, bV, ID_PV, acc);
                        else
                            mma_ss(dst, dP0 + (uint64_t)((kk * 32) >> 4), bV, ID_PV, acc);
                    }
                    mma_commit(&bar[G::B_MMA4]);
                    mma_commit(&bar[G::B_O_FULL]);
                }
                mma_commit(&bar[G::B_KV_EMPTY + s]);
                mma_commit(&bar[G::B_V_EMPTY + s]);
            }
            // drain: every MMA issued by this thread has completed
            volatile int never = 0;
            AbortCtx timed{&never, nullptr, kDrainLimitNs};
            mma_commit(&bar[G::B_DRAIN]);
            mbar_wait(&bar[G::B_DRAIN], 0, timed, 0);
        }
    } else if (warp >= kKWarp0 && warp < kKWarp0 + 4) {
        // ================= keys: decay cumsum and phi(K) (warps 10-13)
        const int tk = threadIdx.x - kKWarp0 * 32;   // 0..127
        float Aseg = 1.f;                            // product of chunk decays (state-only mode)
        float apre[C / 32], bpre[C / 32];            // decays and gains of the next chunk (warp kKWarp0)
#pragma unroll
        for (int h = 0; h < C / 32; ++h) apre[h] = bpre[h] = 1.f;
        float lam = 0.f;   // log2 decay of the chunks already processed (state-only mode)
        bool ok = true;
        for (int c = 0; ok && c < nch; ++c) {
            ok = k_stage<C, D, DECAY, MODE, InT>(smem, bar, Fsm, ab, p, t_begin, t_end, bh, c, nch, tk, Aseg,
                                                 apre, bpre, lam);
            if constexpr (G::QS) if (ok) ok = k_weight<C, D, DECAY, MODE>(smem, bar, Fsm, p, ab, c, tk);
        }
    } else if (warp >= kPhiWarp0) {
        // ================= phi(Q) and the state epilogue (warps 6-9)
        const int tw = threadIdx.x - kPhiWarp0 * 32;        // 0..127
        const int q = warp & 3;                              // TMEM lane quarter
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        bool ok = true;

        // state rows owned by this thread: TMEM lane quarter q, rows of the
        // M = D accumulator (D = 64: lanes 0-15 of each quarter)
        constexpr int SROWS = (D == 128) ? 32 : 16;
        const bool srow_ok = lane < SROWS;
        const int a_row = q * SROWS + lane;   // state row (feature index)

        if constexpr (G::OUT)
            if (nch > 0) ok = q_stage<C, D, DECAY, MODE, InT>(smem, bar, ab, tmem, 0, tw, DECAY && (p.mlstm || p.flash));
        // ---- segment start: state entering the segment -> TMEM (and operands)
        if (ok && nch > 0) {
            float g0 = 1.f;   // decay of chunk 0 (the state is rescaled before its update)
            if constexpr (DECAY && G::OUT) {
                ok = mbar_wait(&bar[G::B_L_READY + 0], 0, ab, 17);
                g0 = Fsm[G::F_G + 0];
            }
            tc_fence_after();
            // (output mode may have been launched before the segment scan ended)
            if constexpr (G::OUT) pdl_wait();
            const float *st = p.ws_state + ((size_t)bh * p.n_seg + seg) * (D * D + D);
            if (ok) {
#pragma unroll 1
                for (int cb = 0; cb < D / 32; ++cb) {
                    float vals[32];
                    uint32_t u[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        vals[i] = (G::OUT && srow_ok) ? st[(size_t)a_row * D + cb * 32 + i] : 0.f;
                        u[i] = __float_as_uint(vals[i] * g0);
                        if constexpr (FLASH) vals[i] *= p.inv_s;   // operand: the summaries over s
                    }
                    tmem_st32(tmem + lane_base + G::T_S + cb * 32, u);
                    if constexpr (G::OUT) if (srow_ok) write_state_row<D>(smem + G::OFF_SBF, a_row, cb * 32, vals);
                }
                const float zin = (G::OUT && srow_ok) ? st[(size_t)D * D + a_row] : 0.f;
                tmem_st1(tmem + lane_base + G::T_Z, __float_as_uint(zin * g0));
                if constexpr (G::OUT) {
                    if (srow_ok) {
                        // z operand: row n = 0 of the [16][D] K-major no-swizzle layout
                        bf16 *zb = reinterpret_cast<bf16 *>(smem + G::OFF_ZB);
                        write_z_operand<true>(zb, a_row, zin);
                    }
                }
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[G::B_S_READY]);
            }
        }

        if constexpr (!G::OUT) {
            // state-only mode with decay: warp 0 forms every chunk's decay cumsum
            // ahead of the key warps.  Chunk c's L slot is free once both key
            // warpgroups have finished the feature map of chunk c - NKV (its
            // phi_done), so the cumsum does not wait for the chunk's data.
            float Aseg = 1.f;   // product of the chunk decays (the segment's A)
            if constexpr (DECAY) {
                if (tw < 32) {
                    float apre[C / 32], bpre[C / 32];
#pragma unroll
                    for (int h = 0; h < C / 32; ++h) apre[h] = bpre[h] = 1.f;
                    float lam = 0.f;
                    for (int c = 0; ok && c < nch; ++c) {
                        if (c >= G::NKV &&
                            !mbar_wait(&bar[G::B_PHI + c % G::NKV], ((c - G::NKV) / G::NKV) & 1, ab, 31)) {
                            ok = false;
                            break;
                        }
                        decay_cumsum<C, D, DECAY, MODE>(bar, Fsm, p, t_begin, t_end, bh, c, nch, lane, Aseg, apre,
                                                        bpre, lam);
                    }
                }
            }
            if (tw == 0 && ok && nch > 0) p.ws_A[(size_t)bh * p.n_seg + seg] = Aseg;
            // state-only mode: write the segment's (dS, dz) to the workspace
            if (ok && nch > 0 && mbar_wait(&bar[G::B_DS_FULL], 0, ab, 11)) {
                tc_fence_after();
                float *dst = p.ws_state + ((size_t)bh * p.n_seg + seg) * (D * D + D);
                uint32_t zbits;
                tmem_ld1(tmem + lane_base + G::T_Z, zbits);
#pragma unroll 1
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
                if (srow_ok) dst[(size_t)D * D + a_row] = __uint_as_float(zbits);
            }
        } else {
            for (int c = 0; ok && c < nch; ++c) {
                if constexpr (G::PW) {
                    float rs;
                    float li_unused;
                    ok = p_epilogue<C, D, FORM, MODE, true>(smem, bar, Fsm, p, ab, tmem, c, q, lane, rs, li_unused);
                    if (!ok) break;
                }
                if constexpr (G::QW) {
                    ok = q_weight<C, D, DECAY, MODE>(smem, bar, Fsm, ab, tmem, c, tw);
                    if (!ok) break;
                }
                if (c + 1 < nch) {
                    ok = q_stage<C, D, DECAY, MODE, InT>(smem, bar, ab, tmem, c + 1, tw, DECAY && (p.mlstm || p.flash));
                    if (!ok) break;
                }
                if (c == nch - 1) {
                    // the state after a segment's last chunk is read only as the
                    // final state, which the last segment writes out
                    if (p.fin_S && seg == p.n_seg - 1 && mbar_wait(&bar[G::B_DS_FULL], c & 1, ab, 19)) {
                        tc_fence_after();
                        write_final_state<D>(tmem + lane_base + G::T_S, tmem + lane_base + G::T_Z,
                                             p.fin_S + (size_t)bh * D * D, p.fin_z + (size_t)bh * D, a_row,
                                             srow_ok);
                    }
                    break;
                }
                if (!mbar_wait(&bar[G::B_DS_FULL], c & 1, ab, 11)) { ok = false; break; }
                float gnext = 1.f;   // decay of chunk c+1
                if constexpr (DECAY) {
                    const int s1 = (c + 1) % G::NKV;
                    if (!mbar_wait(&bar[G::B_L_READY + s1], ((c + 1) / G::NKV) & 1, ab, 18)) { ok = false; break; }
                    gnext = Fsm[G::F_G + s1];
                }
                tc_fence_after();
                uint32_t zbits;   // z of this thread's state row entering chunk c+1
                tmem_ld1(tmem + lane_base + G::T_Z, zbits);
                // state entering chunk c+1: bf16 operands, and (decay) rescale in TMEM
#pragma unroll 1
                for (int cb = 0; cb < D / 32; ++cb) {
                    uint32_t u[32];
                    tmem_ld32(tmem + lane_base + G::T_S + cb * 32, u);
                    tmem_ld_wait();
                    float vals[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) vals[i] = __uint_as_float(u[i]);
                    if constexpr (FLASH) {
                        // the read-out sees the summaries over s; TMEM keeps the raw sum
#pragma unroll
                        for (int i = 0; i < 32; ++i) vals[i] *= p.inv_s;
                    }
                    if (srow_ok) write_state_row<D>(smem + G::OFF_SBF, a_row, cb * 32, vals);
                    if constexpr (DECAY && !FLASH) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(vals[i] * gnext);
                        tmem_st32(tmem + lane_base + G::T_S + cb * 32, u);
                    }
                }
                if (srow_ok) {
                    bf16 *zb = reinterpret_cast<bf16 *>(smem + G::OFF_ZB);
                    write_z_operand<true>(zb, a_row, __uint_as_float(zbits));
                }
                if constexpr (DECAY && !FLASH) {
                    tmem_st1(tmem + lane_base + G::T_Z, __float_as_uint(__uint_as_float(zbits) * gnext));
                    tmem_st_wait();
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar[G::B_S_READY]);
            }
        }
    } else if constexpr (!G::OUT) {
        // ================= warps 0-3 in state-only mode: second half of phi(K)
        for (int c = 0; c < nch; ++c)
            if (!phi_keys_second_half<C, D, DECAY, MODE, InT>(smem, bar, Fsm, p, ab, t_begin, t_end, c, nch,
                                                              threadIdx.x))
                break;
    } else {
        // ================= epilogue (warps 0-3): scores -> P, output division and store
        const int q = warp;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        // HS (chunk 64, rows in lanes 0-15 of the warp's quarter): thread t
        // holds row t & 15 and the columns [16 (t >> 4), + 16) of each
        // 32-column group; otherwise thread t holds row t and all 32 columns
        constexpr bool HS = G::ROWS_PER_WARP == 16;
        constexpr int NV = HS ? 16 : 32;
        const int r = HS ? (lane & 15) : lane;    // this thread's row in the warp's rows
        const int hm = HS ? (lane >> 4) : 0;      // its column half (16-byte chunks 2hm.. / 4hm..)
        for (int c = 0; c < nch; ++c) {
            const int s = c % G::NKV;
            const long t0 = t_begin + (long)c * C;
            float rowsum = 0.f, Li = 0.f;
            if constexpr (!G::PW) {
                if (!p_epilogue<C, D, FORM, MODE, false>(smem, bar, Fsm, p, ab, tmem, c, q, lane, rowsum, Li)) break;
            }
            // QSEP: the decay of the carried state at this row, applied to the inter term here
            const float wq = G::QSEP ? ex2_approx(Li) : 1.f;

            if (!mbar_wait(&bar[G::B_O_FULL], c & 1, ab, 14)) break;
            tc_fence_after();
            if constexpr (G::PW) {
                uint32_t rsb;
                tmem_ld1(tmem + lane_base + G::T_RS + (c & 1), rsb);
                tmem_ld_wait();
                rowsum = __uint_as_float(rsb);
            }
            // output: 32 columns per TMEM round trip, scaled, converted and
            // written swizzled to this warp's staging rows, then stored by TMA
            // (each warp stores its own rows; rows beyond T are clipped).  The
            // O accumulator is released after its last TMEM read, before the
            // last group is converted and stored.  16-bit outputs: one
            // 32-column box (64-byte rows) per group, two staging buffers per
            // warp, so a box waits only for the store two boxes back; fp32:
            // one 128-byte-wide box per group, one buffer.
            constexpr bool NARROW = sizeof(OutT) == 2;
            uint8_t *stg_w = smem + G::OFF_STG + q * (G::ROWS_PER_WARP * 128);   // this warp's 4 KB (2 KB)
            float inv = 0.f;
#pragma unroll 1
            for (int g = 0; g < D / 32; ++g) {
                float o[NV];
                {
                    uint32_t u[NV], ud = 0u, ud_lo = 0u;
                    if (g == 0) {
                        tmem_ld1(tmem + lane_base + G::T_DEN, ud);
                        tmem_ld1(tmem + lane_base + G::T_DEN + 1, ud_lo);   // phi(q).z_lo
                    }
                    uint32_t ui[NV];
                    if constexpr (HS) {
                        tmem_ld16x2<16>(tmem + lane_base + G::T_O + g * 32, u);
                        if constexpr (G::QSEP) tmem_ld16x2<16>(tmem + lane_base + G::T_OI + g * 32, ui);
                    } else {
                        tmem_ld32(tmem + lane_base + G::T_O + g * 32, u);
                        if constexpr (G::QSEP) tmem_ld32(tmem + lane_base + G::T_OI + g * 32, ui);
                    }
                    tmem_ld_wait();
                    if constexpr (HS) {
                        // the denominator terms sit in lane r's row (read by threads 0-15)
                        if (g == 0) {
                            ud = __shfl_sync(0xffffffffu, ud, r);
                            ud_lo = __shfl_sync(0xffffffffu, ud_lo, r);
                        }
                    }
                    if constexpr (G::QSEP) {
                        // O = 2^(L_i) inter + intra
#pragma unroll
                        for (int k = 0; k < NV; ++k)
                            u[k] = __float_as_uint(fmaf(wq, __uint_as_float(ui[k]), __uint_as_float(u[k])));
                    }
                    if (g == D / 32 - 1) {
                        // every TMEM read of O is complete: the next chunk's MMA2 may overwrite it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bar[G::B_O_EMPTY]);
                    }
                    // denominator: (decayed) phi(q).z of the carried state + row sum of P + eps
                    if (g == 0) {
                        if constexpr (FLASH) {
                            inv = 1.f;   // no normaliser
                        } else if constexpr (DECAY) {
                            // (QSEP: the carried-state part from the plain phi(Q), scaled here)
                            const float den = wq * (__uint_as_float(ud) + __uint_as_float(ud_lo)) + rowsum;
                            // mLSTM read-out: divide by max(|den|, 1)
                            inv = p.mlstm ? 1.f / fmaxf(fabsf(den), 1.f) : 1.f / (den + p.eps);
                        } else {
                            inv = 1.f / ((__uint_as_float(ud) + __uint_as_float(ud_lo)) + rowsum + p.eps);
                        }
                    }
#pragma unroll
                    for (int k = 0; k < NV; ++k) o[k] = __uint_as_float(u[k]) * inv;
                }
                if constexpr (NARROW) {
                    // buffer (c * D/32 + g) & 1 of this warp: [R][64 B], 64-byte swizzle
                    const int nb = c * (D / 32) + g;
                    uint8_t *stg = stg_w + (nb & 1) * (G::ROWS_PER_WARP * 64);
                    if (lane == 0) bulk_wait_read1();   // the store that last used this buffer has read it
                    __syncwarp();
#pragma unroll
                    for (int mm = 0; mm < NV / 8; ++mm) {
                        const int m = (NV / 8) * hm + mm;   // 16-byte chunk of the 64-byte row
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[e] = o[8 * mm + e];
                        uint4 w;
                        if constexpr (std::is_same<OutT, bf16>::value) w = pack8_bf16(x);
                        else
                            w = make_uint4(pack_f16x2(x[0], x[1]), pack_f16x2(x[2], x[3]),
                                           pack_f16x2(x[4], x[5]), pack_f16x2(x[6], x[7]));
                        *reinterpret_cast<uint4 *>(stg + r * 64 + ((m ^ ((r >> 1) & 3)) << 4)) = w;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&tm_o, stg, g * 32, (int)t0 + q * G::ROWS_PER_WARP, bh);
                        bulk_commit();
                    }
                } else {
                    // this warp's previous store must have read its staging rows
                    if (lane == 0) bulk_wait_read0();
                    __syncwarp();
#pragma unroll
                    for (int mm = 0; mm < NV / 4; ++mm)
                        *reinterpret_cast<float4 *>(stg_w + sw128_off(r, (NV / 4) * hm + mm)) =
                            make_float4(o[4 * mm], o[4 * mm + 1], o[4 * mm + 2], o[4 * mm + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&tm_o, stg_w, g * 32, (int)t0 + q * G::ROWS_PER_WARP, bh);
                        bulk_commit();
                    }
                }
            }
        }
    }

    // ---------------- teardown
    if constexpr (G::OUT) {
        if (warp < 4 && lane == 0) bulk_wait0();   // output stores complete
    }
    tc_fence_before();
    __syncthreads();
    // the CTA's work is done (state-only: its segment state is written), so a
    // dependent grid may start launching; it waits for this grid's completion
    // before it reads anything this grid wrote
    pdl_trigger();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, G::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace la
