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

// Segments per head: enough CTAs for two per SM across all heads, but no
// segment shorter than `min_tokens` unless the head itself is shorter.
inline Plan make_plan(long BH, long T, int chunk, int D) {
    Plan p;
    p.chunk = chunk;
    const long n_chunks = (T + chunk - 1) / chunk;
    const long want_ctas = 2L * kNumSMs;
    long segs = (want_ctas + BH - 1) / BH;
    // keep the scan traffic (4 passes over D*D fp32 per segment) below ~1/8
    // of the segment's own q/k/v/o bytes (~8*D bytes per token at 16 bits)
    long min_tokens = (long)D * 16;
    if (min_tokens < chunk) min_tokens = chunk;
    long min_chunks = (min_tokens + chunk - 1) / chunk;
    long max_segs = n_chunks / min_chunks;
    if (max_segs < 1) max_segs = 1;
    if (segs > max_segs) segs = max_segs;
    if (segs < 1) segs = 1;
    long G = (n_chunks + segs - 1) / segs;
    p.seg_len = (int)(G * chunk);
    p.n_seg = (int)((n_chunks + G - 1) / G);
    return p;
}

}  // namespace la
