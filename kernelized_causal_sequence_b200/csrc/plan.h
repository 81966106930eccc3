// plan.h — how a head's tokens are cut into segments of whole chunks.
//
// Segments run on different SMs and are joined by the decayed prefix scan
// over their states, so the plan trades parallelism (enough segments to fill
// the 148 SMs) against scan traffic (each segment costs one fp32 state of
// D*D + D floats written, scanned and read back).
#pragma once

namespace la {

constexpr int kNumSMs = 148;           // B200
constexpr int kNoncausalChunk = 128;   // key block of the non-causal state build

struct Plan {
    int chunk;    // tokens per chunk
    int seg_len;  // tokens per segment (a multiple of chunk)
    int n_seg;    // segments per head
};

// Segments per head.  Each segment is one CTA (one per SM), so the critical
// path is (waves of CTAs) x (chunks per segment): choose the segment count
// that minimises it, preferring fewer segments (less scan traffic) on ties.
// Segments are kept at least `min_chunks` long so the per-segment state
// (D*D + D fp32 written, scanned, read back) stays a small fraction of the
// segment's own input bytes.
inline Plan make_plan(long BH, long T, int chunk, int D) {
    Plan p;
    p.chunk = chunk;
    const long n_chunks = (T + chunk - 1) / chunk;
    // >= 4*D tokens per segment, unless the whole problem has fewer chunks than
    // two waves of SMs (then latency, not scan traffic, is what matters)
    long min_chunks = ((long)D * 4 + chunk - 1) / chunk;
    if (BH * n_chunks < 2L * kNumSMs) min_chunks = 1;
    if (min_chunks < 1) min_chunks = 1;
    long max_segs = n_chunks / min_chunks;
    if (max_segs < 1) max_segs = 1;
    if (max_segs > 4096) max_segs = 4096;
    long best_segs = 1, best_cost = -1;
    for (long segs = 1; segs <= max_segs; ++segs) {
        const long G = (n_chunks + segs - 1) / segs;
        const long real = (n_chunks + G - 1) / G;
        const long waves = (BH * real + kNumSMs - 1) / kNumSMs;
        const long cost = waves * (G + 2);   // ~2 chunks of per-CTA fill, set-up and drain
        if (best_cost < 0 || cost < best_cost) { best_cost = cost; best_segs = segs; }
    }
    const long G = (n_chunks + best_segs - 1) / best_segs;
    p.seg_len = (int)(G * chunk);
    p.n_seg = (int)((n_chunks + G - 1) / G);
    return p;
}

// Key segments of the non-causal form.  At head dim 32 the CUDA-core state
// kernel runs several CTAs per SM, so aim for ~4 CTAs per SM over all heads,
// with segments of at least 64 keys; other head dims use the chunk plan.
inline Plan make_nc_plan(long BH, long Lk, int D) {
    if (D != 32) return make_plan(BH, Lk > 0 ? Lk : 1, kNoncausalChunk, D);
    Plan p;
    p.chunk = 64;
    const long L = Lk > 0 ? Lk : 1;
    long segs = (4L * kNumSMs + BH - 1) / BH;
    const long max_segs = (L + 63) / 64;
    if (segs > max_segs) segs = max_segs;
    if (segs < 1) segs = 1;
    long seg_len = (L + segs - 1) / segs;
    seg_len = (seg_len + 63) / 64 * 64;
    p.seg_len = (int)seg_len;
    p.n_seg = (int)((L + seg_len - 1) / seg_len);
    return p;
}

}  // namespace la
