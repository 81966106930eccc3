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

// Key segments of the non-causal form.  At head dimension 32 the CUDA-core
// state kernel fits four 256-thread CTAs per SM, so the plan fills one wave
// of 4 x 148 CTAs over all heads, with segments of whole 128-key tiles;
// other head dims use the chunk plan.
constexpr int kNc32CtasPerSm = 4;
constexpr int kNc32TileRows = 128;
inline Plan make_nc_plan(long BH, long Lk, int D) {
    if (D != 32) return make_plan(BH, Lk > 0 ? Lk : 1, kNoncausalChunk, D);
    Plan p;
    p.chunk = kNc32TileRows;
    const long L = Lk > 0 ? Lk : 1;
    long segs = (long)kNc32CtasPerSm * kNumSMs / (BH > 0 ? BH : 1);
    if (segs < 1) segs = 1;
    long seg_len = (L + segs - 1) / segs;
    seg_len = (seg_len + kNc32TileRows - 1) / kNc32TileRows * kNc32TileRows;
    p.seg_len = (int)seg_len;
    p.n_seg = (int)((L + seg_len - 1) / seg_len);
    return p;
}

// Key segments of the tensor-core non-causal form (head dimension 32): one
// CTA per (group of 4 heads, segment of whole 64-key tiles), the segment
// count chosen so that all CTAs fit in one wave on the SMs.  The kernel splits
// the tiles evenly: segment s takes tiles [s * tiles / n_seg, (s + 1) * tiles
// / n_seg) (seg_len is the longest segment).
constexpr int kNcTcHeads = 4;
constexpr int kNcTcKeyTile = 64;
inline Plan make_nc_tc_plan(long BH, long Lk) {
    Plan p;
    p.chunk = kNcTcKeyTile;
    const long groups = (BH + kNcTcHeads - 1) / kNcTcHeads;
    const long tiles = Lk > 0 ? (Lk + kNcTcKeyTile - 1) / kNcTcKeyTile : 1;
    long segs = kNumSMs / (groups > 0 ? groups : 1);
    if (segs < 1) segs = 1;
    if (segs > tiles) segs = tiles;
    const long per = (tiles + segs - 1) / segs;
    p.seg_len = (int)(per * kNcTcKeyTile);
    p.n_seg = (int)segs;
    return p;
}

// Query tiles per read-out CTA at head dimension 32: one wave of
// 4 x 148 CTAs over all heads.
inline int nc32_tiles_per_cta(long BH, long Lq) {
    const long tiles = (Lq + kNc32TileRows - 1) / kNc32TileRows;
    const long slots = (long)kNc32CtasPerSm * kNumSMs;
    long t = (tiles * BH + slots - 1) / slots;
    return (int)(t < 1 ? 1 : t);
}

}  // namespace la
