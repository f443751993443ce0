// proj_gemm.cu -- the dense projections on either side of the attention, as one
// persistent tcgen05 GEMM with per-use epilogues.
//
// Meta HSTU blog, section 3 formula: U(X), V(X), Q(X), K(X) = Split(phi1(f1(X))) with
// phi1 = SiLU, and O(X) = f2(Norm(A(X) V(X)) (.) U(X)).  f1 and f2 are linear maps
// (weights stored [out, in], row-major, bf16; fp32 biases).  The forward uses
//   f1:  Z = X W1^T + b1 -> U, V, Q, K = SiLU(Z) split in four column blocks of D
//   f2:  O = O_pre W2^T + b2 (+ a residual when given)
// and the backward the same kernel with transposed operands (dX = dZ W1, dW1 = dZ^T X, ...).
//
// C[M, N] = sum_k A[m, k] B[n, k].  A is K-major (row-major [M, K]) or MN-major (row-major
// [K, M], i.e. the transpose is read); B likewise ([N, K] or [K, N]).  Tiles are 128 x 256
// with K steps of 64: TMA brings 128-byte swizzled panels into a 4-stage shared-memory
// ring, one thread issues tcgen05.mma (M = 128, N = 256, K = 16) into a double-buffered
// TMEM accumulator (2 x 256 fp32 columns), and eight epilogue warps drain one accumulator
// while the next tile is being multiplied.  Each epilogue warp owns 32 rows x 128 columns
// of a tile; it stages 32 x 64 output chunks in 128-byte-swizzled shared memory (one
// buffer per warp, reused once the previous store has read it) and writes them with TMA
// tensor stores, so every global write is a full line.  Split-K (for the weight gradients, whose K is the token count) adds fp32
// partial tiles with TMA reduce-adds.
//
// Every wait is bounded; on timeout the CTA records kStatusTimeout in *status, drains
// its own copies and MMAs, frees TMEM and returns.
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace hstu {
namespace {

using namespace ptx;

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kStgBufs = 1;                          // staging buffers per epilogue warp
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = 0, kMmaWarp = 1, kFirstEpiWarp = 2;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kATile = kBM * kBK * 2;           // 16 KB
constexpr uint32_t kBTile = kBN * kBK * 2;           // 32 KB
constexpr uint32_t kStage = kATile + kBTile;
constexpr uint32_t kPanel = 64 * 128;                // MN-major panel: 64 K-rows x 128 B
constexpr uint32_t kTmemCols = 2 * kBN;
constexpr uint32_t kStgBytes = kGemmStoreRows * 128;   // one staged chunk: 32 rows x 128 bytes
constexpr unsigned kFull = 0xffffffffu;

enum { kFullBar = 0, kEmptyBar = kStages, kAccFull = 2 * kStages, kAccEmpty = kAccFull + 2,
       kDrainBar = kAccEmpty + 2, kNumBars };

struct Smem {
    static constexpr uint32_t ring = 0;
    static constexpr uint32_t stage = kStages * kStage;                 // staging buffers of the epilogue
    static constexpr uint32_t bars = stage + kEpiWarps * kStgBufs * kStgBytes;
    static constexpr uint32_t tmem = bars + kNumBars * 8;
    static constexpr uint32_t abort_flag = tmem + 4;
    static constexpr uint32_t size = abort_flag + 4;
    static constexpr uint32_t alloc = size + 1024;   // slack for the 1024-byte alignment
};

__device__ __forceinline__ void flag_timeout(const GemmParams& p, volatile int* abort_flag) {
    *abort_flag = 1;
    if (p.status) atomicOr(p.status, kStatusTimeout);
}

struct TileCoord {
    int m0, n0, kb0, kb1;
};

__device__ __forceinline__ TileCoord tile_coord(const GemmParams& p, int t) {
    const int n_m = (p.M + kBM - 1) / kBM, n_n = (p.N + kBN - 1) / kBN;
    const int nkb = (p.K + kBK - 1) / kBK;
    const int per = (nkb + p.k_splits - 1) / p.k_splits;
    const int s = t / (n_m * n_n), r = t % (n_m * n_n);
    TileCoord c;
    c.m0 = (r / n_n) * kBM;                               // N fastest: neighbours share A rows in L2
    c.n0 = (r % n_n) * kBN;
    c.kb0 = s * per;
    c.kb1 = min(nkb, c.kb0 + per);
    return c;
}

// SiLU(z) = z * sigmoid(z) = h + h * tanh(h) with h = z / 2: one hardware tanh per element
__device__ __forceinline__ float silu(float z) {
    float t;
    const float h = 0.5f * z;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Staging: lane r owns row r of a 32-row chunk; its 16-byte piece j sits at
// r * 128 + ((j ^ (r & 7)) * 16), the layout a 128-byte-swizzled TMA box expects.
__device__ __forceinline__ uint32_t stg_addr(uint32_t buf, int r, int j) {
    return buf + r * 128 + ((j ^ (r & 7)) << 4);
}

__device__ __forceinline__ void stage_bf16x64(uint32_t buf, int lane, const float (&x)[64]) {
#pragma unroll
    for (int j = 0; j < 8; j++)
        st_shared_v4(stg_addr(buf, lane, j), pack_bf16x2(x[8 * j], x[8 * j + 1]), pack_bf16x2(x[8 * j + 2], x[8 * j + 3]),
                     pack_bf16x2(x[8 * j + 4], x[8 * j + 5]), pack_bf16x2(x[8 * j + 6], x[8 * j + 7]));
}

__device__ __forceinline__ void stage_f32x32(uint32_t buf, int lane, const uint32_t (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 8; j++) st_shared_v4(stg_addr(buf, lane, j), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

// Waits until this warp's staging buffer is no longer read by an earlier store (with two
// buffers, the other buffer's store may still be reading), so the warp can overwrite it.
__device__ __forceinline__ void stg_acquire(int lane) {
    if (lane == 0) {
        if (kStgBufs == 2) bulk_wait_read_le1();
        else bulk_wait_read_all();
    }
    __syncwarp();
}

// Makes the staged chunk visible to the TMA engine and stores it at (x, y).
__device__ __forceinline__ void stg_store(const CUtensorMap* m, uint8_t* buf, int lane, int x, int y, bool reduce) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        if (reduce) tma_reduce_add_2d(m, buf, x, y);
        else tma_store_2d(m, buf, x, y);
        bulk_commit_group();
    }
}

// Adds rows [row0, row0 + 32) x columns [n, n + 64) of the bf16 residual to x: the warp
// reads them with full-line loads into the staging buffer, then every lane takes its row.
__device__ __forceinline__ void add_residual(const GemmParams& p, uint8_t* buf, int lane, int row0, int n,
                                             float (&x)[64]) {
    const uint32_t b = smem_u32(buf);
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const int r = 4 * i + (lane >> 3), j = lane & 7;
        const int gr = row0 + r, gc = n + 8 * j;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (gr < p.M && gc < p.N) v = __ldg(reinterpret_cast<const uint4*>(p.residual + (size_t)gr * p.N + gc));
        st_shared_v4(stg_addr(b, r, j), v.x, v.y, v.z, v.w);
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const uint4 v = *reinterpret_cast<const uint4*>(buf + (stg_addr(b, lane, j) - b));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int f = 0; f < 4; f++) {
            const float2 t = __bfloat1622float2(h[f]);
            x[8 * j + 2 * f] += t.x;
            x[8 * j + 2 * f + 1] += t.y;
        }
    }
    __syncwarp();
}

template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const __grid_constant__ GemmOutMaps tm_o, const GemmParams p) {
    constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, A_MN ? 1 : 0, B_MN ? 1 : 0);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Smem::bars);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + Smem::tmem);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + Smem::abort_flag);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long wl = p.dbg.limit;   // main-loop wait limit (SM cycles)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&bars[kFullBar + s], 1);
            mbar_init(&bars[kEmptyBar + s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&bars[kAccFull + b], 1);
            mbar_init(&bars[kAccEmpty + b], 32 * kEpiWarps);
        }
        mbar_init(&bars[kDrainBar], 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        prefetch_tmap(&tm_a);
        prefetch_tmap(&tm_b);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    const int n_tiles = ((p.M + kBM - 1) / kBM) * ((p.N + kBN - 1) / kBN) * p.k_splits;

    if (warp == kProducerWarp) {
        // ============================================================ TMA producer
        bool ok = true;
        int use = 0;                                      // k-steps issued so far
        if (lane == 0) {
            for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
                const TileCoord c = tile_coord(p, t);
                for (int kb = c.kb0; kb < c.kb1; kb++) {
                    const int st = use % kStages;
                    ok = mbar_wait(&bars[kEmptyBar + st], ((use / kStages) & 1) ^ 1, s_abort, wl);
                    if (ok && p.dbg.withhold_first_load && use == 0) {
                        // test hook: withhold this CTA's first k-step, so the waits for it run out
                        wait_for_abort(s_abort, 2 * wl);
                        ok = false;
                    }
                    if (!ok) break;
                    uint8_t* sa = sm + st * kStage;
                    uint8_t* sb = sa + kATile;
                    uint64_t* fb = &bars[kFullBar + st];
                    mbar_arrive_expect_tx(fb, kStage);
                    const int k0 = kb * kBK;
                    if (A_MN) {
                        tma_load_2d(sa, &tm_a, fb, c.m0, k0);
                        tma_load_2d(sa + kPanel, &tm_a, fb, c.m0 + 64, k0);
                    } else {
                        tma_load_2d(sa, &tm_a, fb, k0, c.m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int q = 0; q < kBN / 64; q++) tma_load_2d(sb + q * kPanel, &tm_b, fb, c.n0 + 64 * q, k0);
                    } else {
                        tma_load_2d(sb, &tm_b, fb, k0, c.n0);
                    }
                    use++;
                }
            }
            if (!ok && !*s_abort) flag_timeout(p, s_abort);
            if (*s_abort) {
                // drain the copies this thread issued: the last one of each stage
                volatile int dummy = 0;
                for (int s = 0; s < kStages && s < use; s++) {
                    const int last = use - 1 - ((use - 1 - s) % kStages);   // latest use of stage s
                    mbar_wait(&bars[kFullBar + (last % kStages)], (last / kStages) & 1, &dummy);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        bool ok = true;
        if (lane == 0) {
            int use = 0, tile_i = 0;
            const uint32_t a_base = smem_u32(sm), b_base = a_base + kATile;
            for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, tile_i++) {
                const TileCoord c = tile_coord(p, t);
                if (c.kb1 <= c.kb0) { tile_i--; continue; }
                const int buf = tile_i & 1;
                ok = mbar_wait(&bars[kAccEmpty + buf], ((tile_i >> 1) & 1) ^ 1, s_abort, wl);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * kBN;
                for (int kb = c.kb0; kb < c.kb1; kb++) {
                    const int st = use % kStages;
                    ok = mbar_wait(&bars[kFullBar + st], (use / kStages) & 1, s_abort, wl);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sa = a_base + st * kStage, sb = b_base + st * kStage;
                    const uint64_t da = A_MN ? sdesc_sw128(sa, kPanel, 1024) : sdesc_sw128(sa, 16, 1024);
                    const uint64_t db = B_MN ? sdesc_sw128(sb, kPanel, 1024) : sdesc_sw128(sb, 16, 1024);
#pragma unroll
                    for (int j = 0; j < kBK / 16; j++) {
                        // K step of 16: 32 bytes along a K-major row, 16 rows of an MN-major panel
                        const uint32_t oa = A_MN ? j * 2048 : j * 32, ob = B_MN ? j * 2048 : j * 32;
                        mma_ss(d_tmem, da + (oa >> 4), db + (ob >> 4), kIdesc, (kb > c.kb0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&bars[kEmptyBar + st]);
                    use++;
                }
                if (!ok) break;
                tc_commit(&bars[kAccFull + buf]);
            }
            if (!ok && !*s_abort) flag_timeout(p, s_abort);
            volatile int dummy = 0;
            tc_commit(&bars[kDrainBar]);                 // every MMA issued here completes first
            mbar_wait(&bars[kDrainBar], 0, &dummy);
        }
    } else {
        // ============================================================ epilogue (warps 2..9)
        const int ew = warp - kFirstEpiWarp;
        const int wq = warp & 3;                          // TMEM lane quarter this warp may read
        const int half = ew >> 2;                         // columns [128 * half, +128) of the tile
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        uint8_t* stg = sm + Smem::stage + ew * kStgBufs * kStgBytes;
        int sb = 0;                                       // staging buffer the next chunk uses
        bool ok = true;
        int tile_i = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, tile_i++) {
            const TileCoord c = tile_coord(p, t);
            if (c.kb1 <= c.kb0) { tile_i--; continue; }
            const int buf = tile_i & 1;
            ok = mbar_wait(&bars[kAccFull + buf], (tile_i >> 1) & 1, s_abort, wl);
            if (!__all_sync(kFull, ok)) { ok = false; break; }
            tc_fence_after();
            const int row0 = c.m0 + wq * 32;              // this warp's 32 rows
            const uint32_t tacc = tmem + lane_base + buf * kBN;
            if (EPI == kEpiAddF32) {
#pragma unroll 1
                for (int ch = 0; ch < 4; ch++) {
                    const int col = 128 * half + 32 * ch;
                    uint32_t v[32];
                    tmem_ld32(tacc + col, v);
                    tmem_ld_wait(v);
                    if (ch == 3) {                        // the accumulator may be reused now
                        tc_fence_before();
                        mbar_arrive(&bars[kAccEmpty + buf]);
                    }
                    const int n = c.n0 + col;
                    if (n < p.N && row0 < p.M) {
                        uint8_t* sbuf = stg + sb * kStgBytes;
                        stg_acquire(lane);
                        stage_f32x32(smem_u32(sbuf), lane, v);
                        stg_store(&tm_o.out[0], sbuf, lane, n, row0, true);
                        sb = (sb + 1) % kStgBufs;
                    }
                }
            } else {
#pragma unroll 1
                for (int ch = 0; ch < 2; ch++) {
                    const int col = 128 * half + 64 * ch;
                    uint32_t v0[32], v1[32];
                    tmem_ld32(tacc + col, v0);
                    tmem_ld32(tacc + col + 32, v1);
                    tmem_ld_wait(v0);
                    tmem_ld_wait(v1);
                    if (ch == 1) {
                        tc_fence_before();
                        mbar_arrive(&bars[kAccEmpty + buf]);
                    }
                    const int n = c.n0 + col;
                    if (n >= p.N || row0 >= p.M) continue;
                    float x[64];
#pragma unroll
                    for (int e = 0; e < 32; e++) {
                        x[e] = __uint_as_float(v0[e]);
                        x[32 + e] = __uint_as_float(v1[e]);
                    }
                    if (p.bias) {
#pragma unroll
                        for (int e = 0; e < 16; e++)
                            if (n + 4 * e < p.N) {
                                const float4 bb = __ldg(reinterpret_cast<const float4*>(p.bias + n) + e);
                                x[4 * e] += bb.x; x[4 * e + 1] += bb.y; x[4 * e + 2] += bb.z; x[4 * e + 3] += bb.w;
                            }
                    }
                    uint8_t* sbuf = stg + sb * kStgBytes;
                    if (EPI == kEpiF1) {
                        if (p.z) {
                            stg_acquire(lane);
                            stage_bf16x64(smem_u32(sbuf), lane, x);
                            stg_store(&tm_o.z, sbuf, lane, n, row0, false);
                            sb = (sb + 1) % kStgBufs;
                            sbuf = stg + sb * kStgBytes;
                        }
#pragma unroll
                        for (int e = 0; e < 64; e++) x[e] = silu(x[e]);
                        const int which = n / p.D;            // U, V, Q, K column blocks
                        stg_acquire(lane);
                        stage_bf16x64(smem_u32(sbuf), lane, x);
                        stg_store(&tm_o.out[which], sbuf, lane, n - which * p.D, row0, false);
                    } else {
                        stg_acquire(lane);
                        if (EPI == kEpiF2 && p.residual) add_residual(p, sbuf, lane, row0, n, x);
                        stage_bf16x64(smem_u32(sbuf), lane, x);
                        stg_store(&tm_o.out[0], sbuf, lane, n, row0, false);
                    }
                    sb = (sb + 1) % kStgBufs;
                }
            }
        }
        if (!ok && lane == 0 && !*s_abort) flag_timeout(p, s_abort);
        if (lane == 0) bulk_wait_all();                   // this warp's stores have completed
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <bool A_MN, bool B_MN, int EPI>
cudaError_t launch_t(const CUtensorMap& ta, const CUtensorMap& tb, const GemmOutMaps& to, const GemmParams& p,
                     int grid, cudaStream_t s) {
    cudaError_t e = ensure_smem_limit((const void*)gemm_tc_kernel<A_MN, B_MN, EPI>, Smem::alloc);
    if (e != cudaSuccess) return e;
    gemm_tc_kernel<A_MN, B_MN, EPI><<<grid, kThreads, Smem::alloc, s>>>(ta, tb, to, p);
    return cudaGetLastError();
}

}  // namespace

int gemm_tiles(const GemmParams& p) {
    return ((p.M + kBM - 1) / kBM) * ((p.N + kBN - 1) / kBN) * p.k_splits;
}

int gemm_k_steps(int K) { return (K + kBK - 1) / kBK; }

// Box rows of the operand tensor maps: A K-major loads 128 rows, B K-major 256 rows,
// MN-major operands 64 K-rows per 64-column panel.
int gemm_box_rows(bool mn_major, bool is_b) { return mn_major ? 64 : (is_b ? kBN : kBM); }

cudaError_t launch_gemm_tc(bool a_mn, bool b_mn, int epi, const CUtensorMap& ta, const CUtensorMap& tb,
                           const GemmOutMaps& to, const GemmParams& p, int grid, cudaStream_t s) {
    cudaError_t e = cudaErrorInvalidValue;
    prof_begin(kProfGemm, s);
#define HSTU_GEMM_CASE(AM, BM_, EP)                                            \
    if (a_mn == AM && b_mn == BM_ && epi == EP) e = launch_t<AM, BM_, EP>(ta, tb, to, p, grid, s);
    HSTU_GEMM_CASE(false, false, kEpiF1)
    else HSTU_GEMM_CASE(false, false, kEpiF2)
    else HSTU_GEMM_CASE(false, true, kEpiBf16)
    else HSTU_GEMM_CASE(false, true, kEpiF2)
    else HSTU_GEMM_CASE(true, true, kEpiAddF32)
    else HSTU_GEMM_CASE(false, false, kEpiBf16)
#undef HSTU_GEMM_CASE
    prof_end(kProfGemm, s);
    return e;
}

}  // namespace hstu
