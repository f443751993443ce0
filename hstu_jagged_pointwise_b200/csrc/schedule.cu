// schedule.cu -- device-side work list for the persistent attention kernels.
//
// One CTA validates the jagged offsets (and MTGR segment sizes), sorts the
// sequences by their number of key tiles (longest first, counting sort) and
// writes one work item per (sequence, head, query tile).  The items of one
// (sequence, head) are adjacent, so the CTAs that run them at the same time
// share that sequence's K/V tiles through L2; inside a group the heaviest
// query tile comes first.  Jagged, padding-free batches are the layout the
// MTGR pages describe (JaggedTensor + variable-length HSTU operator; the
// token-balanced batching of MTGR's training system motivates the sort).
#include "internal.h"

namespace hstu {

namespace {

constexpr int kThreads = 1024;

__device__ int n_q_tiles(const SchedParams& p, int Lq) {
    if (Lq <= 0) return 0;
    if (p.kind != HSTU_KIND_MFALCON) return (Lq + kTileM - 1) / kTileM;
    const int tpm = (p.b_m + kTileM - 1) / kTileM;     // tiles per full microbatch
    const int n_mb = (Lq + p.b_m - 1) / p.b_m;
    const int last = Lq - (n_mb - 1) * p.b_m;
    return (n_mb - 1) * tpm + (last + kTileM - 1) / kTileM;
}

// rows [row0, row_end) of query tile k (tile order inside a (sequence, head) group)
__device__ void tile_rows(const SchedParams& p, int Lq, int nt, int k, int* row0, int* row_end) {
    if (p.kind != HSTU_KIND_MFALCON) {
        const int t = p.ascending ? k : nt - 1 - k;      // heaviest tile first
        *row0 = t * kTileM;
        *row_end = min(*row0 + kTileM, Lq);
        return;
    }
    const int tpm = (p.b_m + kTileM - 1) / kTileM;
    const int mb = k / tpm, w = k % tpm;
    *row0 = mb * p.b_m + w * kTileM;
    *row_end = min(*row0 + kTileM, min((mb + 1) * p.b_m, Lq));
}

__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = warp_sums[lane];
        int t = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        warp_sums[lane] = t - s;
        if (lane == 31) *total = t;
    }
    __syncthreads();
    int r = warp_sums[warp] + x - v;
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kThreads) schedule_kernel(SchedParams p) {
    __shared__ int hist[kSchedBins];
    __shared__ int warp_sums[32];
    __shared__ int s_total;
    __shared__ int s_carry;

    const int tid = threadIdx.x;
    for (int i = tid; i < kSchedBins; i += kThreads) hist[i] = 0;
    if (tid == 0) {
        p.ctrl->counter = 0;
        s_carry = 0;
    }

    // ---- 1. validate
    int bad = 0;
    if (tid == 0) {
        if (p.q_off[0] != 0 || p.q_off[p.B] != p.Tq) bad = 1;
        if (p.kv_off != p.q_off && (p.kv_off[0] != 0 || p.kv_off[p.B] != p.Tkv)) bad = 1;
    }
    for (int b = tid; b < p.B; b += kThreads) {
        const int Lq = p.q_off[b + 1] - p.q_off[b];
        if (Lq < 0 || Lq > p.max_q_len) bad = 1;
        if (p.kv_off != p.q_off) {
            const int Lk = p.kv_off[b + 1] - p.kv_off[b];
            if (Lk < 0 || Lk > p.max_kv_len) bad = 1;
        }
        if (p.kind == HSTU_KIND_MTGR || p.kind == HSTU_KIND_MFSEQ) {
            int S = 0, R = 0;
            segment_sizes(p.kind, p.n_static, p.n_rt, b, Lq, &S, &R);
            if (S < 0 || R < 0 || (long long)S + R > Lq) bad = 1;
        }
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0) {
            atomicOr(&p.ctrl->status, kStatusBounds);
            p.ctrl->n_items = 0;
            p.ctrl->valid = 0;
        }
        return;
    }

    // ---- 2. counting sort of sequences by key-tile count, longest first
    for (int b = tid; b < p.B; b += kThreads) {
        const int Lk = p.kv_off[b + 1] - p.kv_off[b];
        const int key = min((Lk + kTileN - 1) / kTileN, kSchedBins - 1);
        atomicAdd(&hist[kSchedBins - 1 - key], 1);
    }
    __syncthreads();
    // exclusive scan over bins (4 bins per thread)
    {
        int v[4], s = 0;
#pragma unroll
        for (int e = 0; e < 4; e++) {
            v[e] = hist[tid * 4 + e];
            s += v[e];
        }
        int base = block_exclusive_scan(s, warp_sums, &s_total);
#pragma unroll
        for (int e = 0; e < 4; e++) {
            hist[tid * 4 + e] = base;
            base += v[e];
        }
    }
    __syncthreads();
    for (int b = tid; b < p.B; b += kThreads) {
        const int Lk = p.kv_off[b + 1] - p.kv_off[b];
        const int key = min((Lk + kTileN - 1) / kTileN, kSchedBins - 1);
        const int pos = atomicAdd(&hist[kSchedBins - 1 - key], 1);
        p.perm[pos] = b;
    }
    __syncthreads();

    // ---- 3. item base of every ranked sequence
    for (int r0 = 0; r0 < p.B; r0 += kThreads) {
        const int r = r0 + tid;
        int nt = 0;
        if (r < p.B) {
            const int b = p.perm[r];
            nt = n_q_tiles(p, p.q_off[b + 1] - p.q_off[b]);
        }
        const int ex = block_exclusive_scan(nt, warp_sums, &s_total);
        if (r < p.B) p.seq_base[r] = s_carry + ex;
        __syncthreads();
        if (tid == 0) s_carry += s_total;
        __syncthreads();
    }
    const long long total_tiles = s_carry;
    if (total_tiles * p.H > p.max_items) {
        if (tid == 0) {
            atomicOr(&p.ctrl->status, kStatusBounds);
            p.ctrl->n_items = 0;
            p.ctrl->valid = 0;
        }
        return;
    }

    // ---- 4. items: (ranked sequence, head, tile)
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = warp; r < p.B; r += kThreads / 32) {
        const int b = p.perm[r];
        const int Lq = p.q_off[b + 1] - p.q_off[b];
        const int nt = n_q_tiles(p, Lq);
        const long long base = (long long)p.seq_base[r] * p.H;
        for (int e = lane; e < nt * p.H; e += 32) {
            const int h = e / nt, k = e % nt;
            int row0, row_end;
            tile_rows(p, Lq, nt, k, &row0, &row_end);
            p.items[base + e] = make_int4(b, row0, h, row_end);
        }
    }
    if (tid == 0) {
        p.ctrl->n_items = (int)(total_tiles * p.H);
        p.ctrl->valid = 1;
    }
}

}  // namespace

cudaError_t launch_schedule(const SchedParams& p, cudaStream_t s) {
    prof_begin(kProfSchedule, s);
    schedule_kernel<<<1, kThreads, 0, s>>>(p);
    prof_end(kProfSchedule, s);
    return cudaGetLastError();
}

}  // namespace hstu
