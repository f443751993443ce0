// ew_bias.cuh -- per-warp classification of the relative attention bias over a block of scores.
//
// rab^{p,t} (Meta HSTU blog, section 3.2) is rab_pos[pidx(i, j)] + rab_time[tb(i, j)]
// with pidx = clamp(pos_j - pos_i, -(P-1), P-1) + (P-1) and tb = min(nb-1,
// bit_length(|ts_i - ts_j|)).  Inside one warp's block of a score tile the two
// terms are often constant, or simple:
//   position:  constant when every pos_j - pos_i is clamped to the same end;
//              otherwise a function of j - i alone when positions are indices
//              (causal rows, or MTGR blocks without candidates), so one row of
//              2*32+... values per warp (the "diagonal row") holds it -- with the
//              causal mask folded in as a huge negative bias, SiLU(-inf) = 0;
//   time:      constant when bucket(min |dt|) == bucket(max |dt|); one threshold
//              when the two differ by one bucket; else a 32-bit bit length when
//              every |dt| of the block is below 2^31.
// The elementwise loops are specialised on these modes; blocks that fit none of
// them (int64-wide time spans, MTGR candidate rows, the last partial key tile)
// use the element-by-element rules of hstu_rules.cuh.
#pragma once
#include <stdint.h>

#include "hstu_rules.cuh"

namespace hstu {

// kPosUniform: one position index for the block; kPosDiag: index from j - i (a
// diagonal row of biases); kPosCol: every row of the block sits at one position
// (M-FALCON candidates), so the index depends on the column alone.
enum PosMode { kPosUniform = 0, kPosDiag = 1, kPosCol = 2 };
enum TimeMode { kTimeUniform = 0, kTimeTwo = 1, kTimeBits = 2 };

// Masked scores get this bias: z ~ -1e30, tanh(z/2) = -1 exactly, SiLU = 0 and SiLU' = 0.
constexpr float kMaskedHalfBias = -5.0e29f;

struct TimeClass {
    int mode;          // TimeMode, or -1 when no 32-bit form exists
    int tb_lo, tb_hi;  // buckets of the smallest and largest |dt|
    uint32_t thr;      // kTimeTwo: |dt| >= thr  <=>  bucket == tb_hi
};

// Blocks with rows' times in [rmin, rmax] and columns' times in [cmin, cmax].
__device__ __forceinline__ TimeClass classify_time(int64_t rmin, int64_t rmax, int64_t cmin,
                                                   int64_t cmax, int nb) {
    TimeClass t;
    uint64_t lo;
    if (rmin > cmax) lo = abs_diff_u64(rmin, cmax);
    else if (cmin > rmax) lo = abs_diff_u64(cmin, rmax);
    else lo = 0;
    const uint64_t hi = max(abs_diff_u64(rmax, cmin), abs_diff_u64(cmax, rmin));
    t.tb_lo = time_bucket_of_delta(lo, nb);
    t.tb_hi = time_bucket_of_delta(hi, nb);
    t.thr = 0;
    if (t.tb_lo == t.tb_hi) {
        t.mode = kTimeUniform;
    } else if (hi >= (1ull << 31)) {
        t.mode = -1;
    } else if (t.tb_hi == t.tb_lo + 1) {
        t.mode = kTimeTwo;
        t.thr = 1u << (t.tb_hi - 1);        // bit_length(x) >= tb_hi  <=>  x >= 2^(tb_hi-1)
    } else {
        t.mode = kTimeBits;
    }
    return t;
}

// Bucket of a 32-bit |dt| (< 2^31).
__device__ __forceinline__ int time_bucket_u32(uint32_t x, int nbm1) {
    return min(32 - __clz((int)x), nbm1);
}

}  // namespace hstu
