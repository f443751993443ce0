// kv_cache.cu -- the M-FALCON KV-cache producer.
//
// HSTU blog, section 4.3 (KV caching): the keys and values of a user's history are
// computed once and reused by every later candidate microbatch of that user.  A
// full-sequence M-FALCON batch (one jagged row [R_b history ; K_b candidates] per
// user, section 4.2) already holds them in its k / v; this copies the history rows
// into the compact cache layout that hstu_mfalcon_score reads:
//
//   hist_offsets[b] = R_0 + ... + R_{b-1}        (exclusive scan, hist_offsets[B] = sum)
//   row hist_offsets[b] + i of hist_k / hist_v / hist_ts = row seq_offsets[b] + i of
//   k / v / timestamps, for i < R_b.
//
// Two launches: one CTA validates the offsets and history lengths and scans them,
// then a grid of warps copies whole rows with 16-byte vectors.  HBM-bound: it reads
// and writes 2 * row_bytes + 8 bytes per cached row.
#include <algorithm>

#include "../../include/hstu.h"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kScanThreads = 1024;
constexpr int kCopyThreads = 256;
constexpr int kRowsPerWarp = 4;     // rows whose loads a warp keeps in flight together

__device__ __forceinline__ long long block_exclusive_scan(long long x, long long* s_warp, long long* total) {
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
        long long w = lane < kScanThreads / 32 ? s_warp[lane] : 0;
        long long wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < kScanThreads / 32) s_warp[lane] = wi - w;     // exclusive prefix of the warp sums
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    return s_warp[warp] + inc - x;
}

// Validates the batch and writes hist_offsets; *status = 0 when the copy may run, else 1.
__global__ void __launch_bounds__(kScanThreads)
cache_scan_kernel(int B, int T, const int32_t* seq_off, const int32_t* n_hist, long long capacity,
                  int32_t* hist_off, int32_t* status) {
    __shared__ long long s_warp[kScanThreads / 32];
    __shared__ long long s_total;
    const int tid = threadIdx.x;
    const int chunk = (B + kScanThreads - 1) / kScanThreads;
    const int b0 = min(B, tid * chunk), b1 = min(B, b0 + chunk);
    int bad = 0;
    if (tid == 0 && (seq_off[0] != 0 || seq_off[B] != T)) bad = 1;
    long long local = 0;
    for (int b = b0; b < b1; b++) {
        const int L = seq_off[b + 1] - seq_off[b];
        const int R = n_hist[b];
        if (L < 0 || R < 0 || R > L) bad = 1;
        local += max(R, 0);
    }
    bad = __syncthreads_or(bad);
    const long long base = block_exclusive_scan(local, s_warp, &s_total);
    if (bad || s_total > capacity || s_total > 0x7fffffffLL) {
        if (tid == 0) *status = 1;
        return;
    }
    long long run = base;
    for (int b = b0; b < b1; b++) {
        hist_off[b] = (int32_t)run;
        run += n_hist[b];
    }
    if (tid == 0) {
        hist_off[B] = (int32_t)s_total;
        *status = 0;
    }
}

// Row r of the cache belongs to the user b with hist_off[b] <= r < hist_off[b + 1].
__device__ __forceinline__ int owner(const int32_t* hist_off, int B, int r) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(hist_off + mid) <= r) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kCopyThreads)
cache_copy_kernel(int B, int nvec, const int32_t* seq_off, const int32_t* hist_off, const int64_t* ts,
                  const uint4* k, const uint4* v, int64_t* hist_ts, uint4* hk, uint4* hv,
                  const int32_t* status) {
    if (*status != 0) return;
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * kCopyThreads + threadIdx.x) >> 5;
    const long long n_warps = ((long long)gridDim.x * kCopyThreads) >> 5;
    const int total = hist_off[B];
    for (long long r0 = warp0 * kRowsPerWarp; r0 < total; r0 += n_warps * kRowsPerWarp) {
        // lane j < kRowsPerWarp resolves row r0 + j: its source row, or -1 past the end
        int src_mine = -1;
        if (lane < kRowsPerWarp && r0 + lane < total) {
            const int r = (int)(r0 + lane);
            const int b = owner(hist_off, B, r);
            src_mine = __ldg(seq_off + b) + (r - __ldg(hist_off + b));
            hist_ts[r] = __ldg(ts + src_mine);
        }
        int src[kRowsPerWarp];
#pragma unroll
        for (int j = 0; j < kRowsPerWarp; j++) src[j] = __shfl_sync(0xffffffffu, src_mine, j);
        for (int vb = 0; vb < nvec; vb += 64) {
            uint4 a[kRowsPerWarp][2], c[kRowsPerWarp][2];
#pragma unroll
            for (int j = 0; j < kRowsPerWarp; j++)
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int vi = vb + lane + 32 * e;
                    if (src[j] >= 0 && vi < nvec) {
                        const size_t o = (size_t)src[j] * nvec + vi;
                        a[j][e] = __ldcs(k + o);
                        c[j][e] = __ldcs(v + o);
                    }
                }
#pragma unroll
            for (int j = 0; j < kRowsPerWarp; j++)
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int vi = vb + lane + 32 * e;
                    if (src[j] >= 0 && vi < nvec) {
                        const size_t o = (size_t)(r0 + j) * nvec + vi;
                        __stcs(hk + o, a[j][e]);
                        __stcs(hv + o, c[j][e]);
                    }
                }
        }
    }
}

}  // namespace
}  // namespace hstu

using namespace hstu;

int hstu_mfalcon_cache_history(int32_t B, int32_t T, int32_t row_elems, int32_t dtype,
                               const int32_t* seq_offsets, const int64_t* timestamps, const int32_t* n_history,
                               const void* k, const void* v, int64_t hist_capacity, int32_t* hist_offsets,
                               int64_t* hist_ts, void* hist_k, void* hist_v, int32_t* device_status,
                               void* stream) {
    if (B < 0 || T < 0 || row_elems <= 0 || hist_capacity < 0) return HSTU_ERR_INVALID_ARG;
    if (dtype != HSTU_BF16 && dtype != HSTU_F32) return HSTU_ERR_INVALID_ARG;
    const long long row_bytes = (long long)row_elems * (dtype == HSTU_F32 ? 4 : 2);
    if (row_bytes % 16 != 0 || row_bytes / 16 > (1 << 20)) return HSTU_ERR_UNSUPPORTED;
    auto al = [](const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; };
    if (!al(seq_offsets, 4) || !al(hist_offsets, 4) || !al(device_status, 4) || (B > 0 && !al(n_history, 4)))
        return HSTU_ERR_INVALID_ARG;
    const bool rows = T > 0 && hist_capacity > 0;
    if (rows && (!al(timestamps, 8) || !al(k, 16) || !al(v, 16) || !al(hist_ts, 8) || !al(hist_k, 16) ||
                 !al(hist_v, 16)))
        return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    prof_begin(kProfCacheScan, s);
    cache_scan_kernel<<<1, kScanThreads, 0, s>>>(B, T, seq_offsets, n_history, hist_capacity, hist_offsets,
                                                 device_status);
    prof_end(kProfCacheScan, s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return HSTU_ERR_CUDA;
    if (!rows || B == 0) return HSTU_OK;
    const int nvec = (int)(row_bytes / 16);
    const long long warps_needed = (hist_capacity + kRowsPerWarp - 1) / kRowsPerWarp;
    const long long blocks = std::min<long long>((warps_needed * 32 + kCopyThreads - 1) / kCopyThreads, 148LL * 2);   // one resident wave
    prof_begin(kProfCacheCopy, s);
    cache_copy_kernel<<<(int)std::max<long long>(blocks, 1), kCopyThreads, 0, s>>>(
        B, nvec, seq_offsets, hist_offsets, timestamps, static_cast<const uint4*>(k),
        static_cast<const uint4*>(v), hist_ts, static_cast<uint4*>(hist_k), static_cast<uint4*>(hist_v),
        device_status);
    prof_end(kProfCacheCopy, s);
    e = cudaGetLastError();
    return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}
