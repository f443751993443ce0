// sl_pack.cu -- the data step in front of the attention: Stochastic Length sampling and
// token-balanced batch packing, on the device.
//
// Stochastic Length (HSTU blog, section 3.4): user histories are long-tailed, and
// training samples variable-length subsequences; with alpha = 1.6 a 4096-event history
// keeps about 776 = 4096^0.8 events.  Reading: a sequence longer than `cap` keeps a
// uniform random subset of cap events, in their original order.  Event i of sequence b
// gets the key SplitMix64(seed, b * 2^32 + i + 1) (Steele, Lea and Flood, OOPSLA 2014:
// output n of the generator started at `seed`); the cap smallest keys (ties by index)
// are kept, which is a uniform random subset.  One CTA per sequence finds the cap-th
// smallest key with an 8-pass radix select (keys are recomputed, never stored) and
// compacts the kept indices in order.
//
// Token-balanced batches (MTGR deep-dive, section 3, contribution 3): batch sizes adapt
// so that every GPU gets the same number of tokens, and gradients are weighted by the
// samples each holds.  Sequence b (tokens [s_b, s_b + L_b) of T) goes to bin
// floor((2 s_b + L_b) R / (2 T)): contiguous ranges of sequences, each within one
// sequence of T / R tokens; bin r's weight is its sequence count / B.
#include <algorithm>

#include "../../include/hstu.h"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kScanThreads = 1024;
constexpr int kSelThreads = 256;

__device__ __forceinline__ uint64_t splitmix64(uint64_t state, uint64_t n) {
    uint64_t z = state + n * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t sl_key(uint64_t seed, int b, int i) {
    return splitmix64(seed, ((uint64_t)(uint32_t)b << 32) + (uint64_t)i + 1ull);
}

// Exclusive prefix over the block (blockDim.x == kScanThreads) of one int64 per thread.
__device__ long long scan_block(long long x, long long* s_warp, long long* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const long long w = s_warp[lane];
        long long wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        s_warp[lane] = wi - w;
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    return s_warp[warp] + inc - x;
}

// Validates the batch, writes out_off (exclusive scan of min(L_b, cap)); *status = 0, or 1
// for bad offsets or an output larger than the capacity (then nothing else is written).
__global__ void __launch_bounds__(kScanThreads)
sl_scan_kernel(int B, int T, const int32_t* off, int cap, long long capacity, int32_t* out_off, int32_t* status) {
    __shared__ long long s_warp[32];
    __shared__ long long s_total;
    const int tid = threadIdx.x;
    const int chunk = (B + kScanThreads - 1) / kScanThreads;
    const int b0 = min(B, tid * chunk), b1 = min(B, b0 + chunk);
    int bad = 0;
    if (tid == 0 && (off[0] != 0 || off[B] != T)) bad = 1;
    long long local = 0;
    for (int b = b0; b < b1; b++) {
        const int L = off[b + 1] - off[b];
        if (L < 0) bad = 1;
        local += min(max(L, 0), cap);
    }
    bad = __syncthreads_or(bad);
    const long long base = scan_block(local, s_warp, &s_total);
    if (bad || s_total > capacity) {
        if (tid == 0) *status = 1;
        return;
    }
    long long run = base;
    for (int b = b0; b < b1; b++) {
        out_off[b] = (int32_t)run;
        run += min(off[b + 1] - off[b], cap);
    }
    if (tid == 0) {
        out_off[B] = (int32_t)s_total;
        *status = 0;
    }
}

// Exclusive rank of `flag` among the block's threads, and the block's count.
__device__ __forceinline__ int rank_in_block(bool flag, int* s_cnt, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned bal = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) s_cnt[warp] = __popc(bal);
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; w++) {
        const int c = s_cnt[w];
        before += w < warp ? c : 0;
        all += c;
    }
    __syncthreads();
    *total = all;
    return before + __popc(bal & ((1u << lane) - 1u));
}

__global__ void __launch_bounds__(kSelThreads)
sl_select_kernel(int B, const int32_t* off, int cap, uint64_t seed, const int32_t* out_off, int32_t* gather,
                 const int32_t* status) {
    __shared__ int hist[256];
    __shared__ int s_cnt[kSelThreads / 32];
    __shared__ unsigned long long s_prefix;
    __shared__ int s_want;
    if (*status != 0) return;
    const int tid = threadIdx.x;
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        const int s0 = off[b], L = off[b + 1] - s0;
        const int o = out_off[b];
        if (L <= cap) {
            for (int i = tid; i < L; i += kSelThreads) gather[o + i] = s0 + i;
            continue;
        }
        // radix select of the cap-th smallest key, 8 bits per pass from the top
        unsigned long long prefix = 0;
        int want = cap;                                 // keys still to take at or below the prefix
        for (int pass = 0; pass < 8; pass++) {
            const int shift = 56 - 8 * pass;
            const unsigned long long hi_mask = pass == 0 ? 0ull : ~0ull << (shift + 8);
            hist[tid] = 0;                              // kSelThreads == 256 bins
            __syncthreads();
            for (int i = tid; i < L; i += kSelThreads) {
                const uint64_t k = sl_key(seed, b, i);
                if ((k & hi_mask) == prefix) atomicAdd(&hist[(k >> shift) & 255], 1);
            }
            __syncthreads();
            if (tid < 32) {                             // warp 0 finds the bin holding the want-th key
                int c[8], sum = 0;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    c[e] = hist[8 * tid + e];
                    sum += c[e];
                }
                int inc = sum;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, inc, d);
                    if (tid >= d) inc += y;
                }
                const int before = inc - sum;
                const bool mine = before < want && want <= inc;
                if (mine) {
                    int cum = before;
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        if (cum + c[e] >= want) {
                            s_prefix = prefix | ((unsigned long long)(8 * tid + e) << shift);
                            s_want = want - cum;
                            break;
                        }
                        cum += c[e];
                    }
                }
            }
            __syncthreads();
            prefix = s_prefix;
            want = s_want;
            __syncthreads();
        }
        // keep keys below the threshold, and the first `want` keys equal to it, in index order
        int taken = 0, eq_seen = 0;
        for (int i0 = 0; i0 < L; i0 += kSelThreads) {
            const int i = i0 + tid;
            uint64_t k = 0;
            if (i < L) k = sl_key(seed, b, i);
            const bool eq = i < L && k == prefix;
            int eq_total = 0;
            const int eq_rank = rank_in_block(eq, s_cnt, &eq_total);
            const bool sel = i < L && (k < prefix || (eq && eq_seen + eq_rank < want));
            int sel_total = 0;
            const int pos = rank_in_block(sel, s_cnt, &sel_total);
            if (sel) gather[o + taken + pos] = s0 + i;
            taken += sel_total;
            eq_seen += eq_total;
        }
    }
}

// dst row r = src row idx[r] (zeros for an index outside [0, n_src)); rows of row_vecs
// 16-byte vectors, one warp per row.
__global__ void __launch_bounds__(256) gather_rows_kernel(long long n, int row_vecs, const uint4* src, long long n_src,
                                                          const int32_t* idx, uint4* dst) {
    const int lane = threadIdx.x & 31;
    const long long w0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long r = w0; r < n; r += nw) {
        const long long s = __ldg(idx + r);
        const bool in = s >= 0 && s < n_src;
        for (int v = lane; v < row_vecs; v += 32)
            dst[r * row_vecs + v] = in ? __ldg(src + s * row_vecs + v) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// Same for rows that are not a whole number of 16-byte vectors (e.g. 8-byte timestamps).
__global__ void __launch_bounds__(256) gather_bytes_kernel(long long n, int row_bytes, const uint8_t* src,
                                                           long long n_src, const int32_t* idx, uint8_t* dst) {
    const long long total = n * row_bytes;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long r = e / row_bytes;
        const int c = (int)(e - r * row_bytes);
        const long long s = __ldg(idx + r);
        dst[e] = (s >= 0 && s < n_src) ? src[s * row_bytes + c] : (uint8_t)0;
    }
}

__global__ void __launch_bounds__(kScanThreads)
pack_kernel(int B, const int32_t* off, int R, int32_t* bin_start, int32_t* bin_tokens, float* bin_weight) {
    const long long T = off[B];
    auto bin_of = [&](int b) -> int {
        if (T <= 0) return 0;
        const long long mid2 = 2LL * off[b] + (off[b + 1] - off[b]);
        return (int)max(0LL, min((long long)R - 1, mid2 * R / (2 * T)));
    };
    // bin_start[r] = first sequence whose bin is >= r (binary search; always within [0, B])
    for (int r = threadIdx.x; r <= R; r += kScanThreads) {
        int lo = 0, hi = B;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (bin_of(mid) < r) lo = mid + 1;
            else hi = mid;
        }
        bin_start[r] = r == R ? B : lo;
    }
    __syncthreads();
    for (int r = threadIdx.x; r < R; r += kScanThreads) {
        const int a = bin_start[r], z = max(a, bin_start[r + 1]);
        bin_tokens[r] = off[z] - off[a];
        bin_weight[r] = B > 0 ? (float)(z - a) / (float)B : 0.f;
    }
}

bool aligned(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace hstu

using namespace hstu;

int hstu_sl_sample(int32_t B, int32_t T, const int32_t* seq_offsets, int32_t cap, uint64_t seed,
                   int64_t out_capacity, int32_t* out_offsets, int32_t* gather_idx, int32_t* device_status,
                   void* stream) {
    if (B < 0 || T < 0 || cap < 1 || out_capacity < 0) return HSTU_ERR_INVALID_ARG;
    if (!aligned(seq_offsets, 4) || !aligned(out_offsets, 4) || !aligned(device_status, 4))
        return HSTU_ERR_INVALID_ARG;
    if (out_capacity > 0 && !aligned(gather_idx, 4)) return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    prof_begin(kProfSlSample, s);
    sl_scan_kernel<<<1, kScanThreads, 0, s>>>(B, T, seq_offsets, cap, out_capacity, out_offsets, device_status);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess && B > 0) {
        const int grid = std::min(B, 148 * 8);
        sl_select_kernel<<<grid, kSelThreads, 0, s>>>(B, seq_offsets, cap, seed, out_offsets, gather_idx,
                                                      device_status);
        e = cudaGetLastError();
    }
    prof_end(kProfSlSample, s);
    return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

int hstu_gather_rows(int64_t n_rows, int32_t row_bytes, const void* src, int64_t n_src, const int32_t* idx,
                     void* dst, void* stream) {
    if (n_rows < 0 || row_bytes < 1 || n_src < 0) return HSTU_ERR_INVALID_ARG;
    if (n_rows == 0) return HSTU_OK;
    if (!aligned(idx, 4) || !src || !dst) return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    prof_begin(kProfGather, s);
    if (row_bytes % 16 == 0 && aligned(src, 16) && aligned(dst, 16)) {
        const long long blocks = std::min<long long>((n_rows * 32 + 255) / 256, 148 * 16);
        gather_rows_kernel<<<(unsigned)blocks, 256, 0, s>>>(n_rows, row_bytes / 16, static_cast<const uint4*>(src),
                                                             n_src, idx, static_cast<uint4*>(dst));
    } else {
        const long long blocks = std::min<long long>((n_rows * row_bytes + 255) / 256, 148 * 16);
        gather_bytes_kernel<<<(unsigned)blocks, 256, 0, s>>>(n_rows, row_bytes, static_cast<const uint8_t*>(src),
                                                              n_src, idx, static_cast<uint8_t*>(dst));
    }
    prof_end(kProfGather, s);
    return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

int hstu_pack_balanced(int32_t B, const int32_t* seq_offsets, int32_t n_bins, int32_t* bin_seq_start,
                       int32_t* bin_tokens, float* bin_weight, void* stream) {
    if (B < 0 || n_bins < 1) return HSTU_ERR_INVALID_ARG;
    if (!aligned(seq_offsets, 4) || !aligned(bin_seq_start, 4) || !aligned(bin_tokens, 4) ||
        !aligned(bin_weight, 4))
        return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    pack_kernel<<<1, kScanThreads, 0, s>>>(B, seq_offsets, n_bins, bin_seq_start, bin_tokens, bin_weight);
    return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}
