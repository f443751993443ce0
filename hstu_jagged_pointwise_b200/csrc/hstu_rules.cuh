// hstu_rules.cuh -- integer rules of jagged HSTU attention, as device functions.
//
// Every kernel (forward, backward, M-FALCON, the debug hook) takes its mask,
// relative-position index and time bucket from these functions, so the debug
// hook's output is exactly what the fused kernels use.
//
//   rab^{p,t} (Meta HSTU blog, section 3.2): a relative position bias plus a
//   time bias.  pidx = clamp(pos_j - pos_i, -(P-1), P-1) + (P-1);
//   bucket = min(nb-1, bit_length(|ts_i - ts_j|)).
//   MTGR dynamic mixed mask (MTGR deep-dive, section 2; MTGR arXiv report,
//   section 3.1): static tokens bidirectional, real-time causal, candidates
//   see themselves plus non-candidates with a strictly earlier timestamp.
//   Full-sequence M-FALCON (HSTU blog, section 4.2): [history ; candidates] in
//   one row, history causal, every candidate sees all history and itself (no
//   timestamp filter); it is the MTGR layout with no static part.
#pragma once
#include <stdint.h>

#define HSTU_KIND_CAUSAL 0
#define HSTU_KIND_MTGR 1
#define HSTU_KIND_MFALCON 2
#define HSTU_KIND_MFSEQ 3

namespace hstu {

// Segment sizes of row b: S static tokens, R real-time / history tokens, the rest candidates.
__device__ __forceinline__ void segment_sizes(int kind, const int32_t* n_static, const int32_t* n_rt, int b,
                                              int L, int* S, int* R) {
    if (kind == HSTU_KIND_MTGR) {
        *S = n_static[b];
        *R = n_rt[b];
    } else if (kind == HSTU_KIND_MFSEQ) {
        *S = 0;
        *R = n_rt[b];
    } else {
        *S = L;
        *R = 0;
    }
}

// 0 static, 1 real-time, 2 candidate (MTGR rows); causal rows are all "static-causal".
__device__ __forceinline__ int token_class(int i, int S, int R) {
    return i < S ? 0 : (i < S + R ? 1 : 2);
}

// Position used by rab_pos.  MTGR candidates share the slot right after the history.
__device__ __forceinline__ int token_pos(int kind, int i, int S, int R) {
    return ((kind == HSTU_KIND_MTGR || kind == HSTU_KIND_MFSEQ) && i >= S + R) ? S + R : i;
}

__device__ __forceinline__ int pos_index(int pos_i, int pos_j, int P) {
    int dp = pos_j - pos_i;
    dp = max(dp, -(P - 1));
    dp = min(dp, P - 1);
    return dp + (P - 1);
}

// |a - b| of two int64 values without overflow.
__device__ __forceinline__ uint64_t abs_diff_u64(int64_t a, int64_t b) {
    return a >= b ? (uint64_t)a - (uint64_t)b : (uint64_t)b - (uint64_t)a;
}

// Bit length of |ts_i - ts_j| capped at nb-1 (bit_length(0) = 0).
__device__ __forceinline__ int time_bucket_of_delta(uint64_t d, int nb) {
    int bl = 64 - __clzll((long long)d);
    return min(bl, nb - 1);
}

__device__ __forceinline__ int time_bucket(int64_t ti, int64_t tj, int nb) {
    return time_bucket_of_delta(abs_diff_u64(ti, tj), nb);
}

// Mask of causal, MTGR and full-sequence M-FALCON rows (i, j local to the sequence).
__device__ __forceinline__ bool visible(int kind, int i, int j, int S, int R, int64_t ts_i,
                                        int64_t ts_j) {
    if (kind == HSTU_KIND_CAUSAL) return j <= i;
    int ci = token_class(i, S, R), cj = token_class(j, S, R);
    if (ci == 0) return cj == 0;
    if (ci == 1) return cj == 0 || (cj == 1 && j <= i);
    return j == i || (cj != 2 && (kind == HSTU_KIND_MFSEQ || ts_j < ts_i));
}

// Tile-level classification of a (query tile, key tile) pair from segment
// sizes alone.  Rows [qa, qb] and columns [ka, kb] are clipped to [0, L).
// Returns 0 when no pair can be visible, 1 when some may be (evaluate the
// mask per element), 2 when every pair with j < L is visible.
// MTGR candidate rows against history are "partial": their timestamp filter is
// applied per element; full-sequence M-FALCON candidates see all history.
__device__ __forceinline__ int tile_class(int kind, int qa, int qb, int ka, int kb, int S, int R) {
    if (kind == HSTU_KIND_CAUSAL) {
        if (ka > qb) return 0;
        return (kb <= qa) ? 2 : 1;
    }
    if (kind == HSTU_KIND_MFALCON) return 2;
    const int H = S + R;
    bool any = false;
    // static rows see static columns
    if (qa < S && ka < S) any = true;
    // real-time rows: static columns, or real-time columns up to the row
    int rlo = max(qa, S), rhi = min(qb, H - 1);
    if (rlo <= rhi) {
        if (ka < S) any = true;
        if (kb >= S && ka <= rhi && ka < H) any = true;
    }
    // candidate rows: themselves, and (timestamp-filtered) history
    int clo = max(qa, H), chi = qb;
    if (clo <= chi) {
        if (ka < H) any = true;
        if (max(clo, ka) <= min(chi, kb)) any = true;
    }
    if (!any) return 0;
    // full tiles: every column static and every row a non-candidate (static rows see
    // all static tokens, real-time rows too), or every row real-time and every column
    // at or before the first row (static or earlier real-time)
    if (kb < S && qb < H) return 2;
    if (qa >= S && qb < H && kb <= qa) return 2;
    if (kind == HSTU_KIND_MFSEQ && qa >= H && kb < H) return 2;   // candidates x history: no filter
    return 1;
}

}  // namespace hstu
