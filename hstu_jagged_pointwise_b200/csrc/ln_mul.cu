// ln_mul.cu -- the HSTU layer epilogue O_pre = (LayerNorm(Y) * gamma + beta) (.) U and its backward.
//
// Meta HSTU blog, section 3 formula: O = f2(Norm(A V) (.) U); the Norm is a
// LayerNorm over the D = H*d_v concatenated head outputs (biased variance,
// affine gamma / beta).  f2 is outside this path.
//
// HBM-bound: forward reads Y and U and writes O_pre (6D + 8 bytes per bf16
// token incl. mean/rstd); backward reads dO_pre, U, Y, mean, rstd and writes
// dY, dU (10D + 8 bytes per token).  Up to four warps share one token row; every
// lane moves 16-byte vectors, rows are held in registers between the passes.
#include "internal.h"

namespace hstu {
namespace {

constexpr long long kLnMaxBlocks = 148 * 16;   // resident blocks of up to 4 warps

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const void* base, size_t idx, float* out) {
        const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + idx);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const float2 f = __bfloat1622float2(h[e]);
            out[2 * e] = f.x;
            out[2 * e + 1] = f.y;
        }
    }
    __device__ static void store(void* base, size_t idx, const float* in) {
        uint4 v;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; e++) h[e] = __floats2bfloat162_rn(in[2 * e], in[2 * e + 1]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + idx) = v;
    }
};
template <>
struct Vec<float> {
    static constexpr int N = 4;
    __device__ static void load(const void* base, size_t idx, float* out) {
        const float4 v = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    __device__ static void store(void* base, size_t idx, const float* in) {
        *reinterpret_cast<float4*>(static_cast<float*>(base) + idx) = make_float4(in[0], in[1], in[2], in[3]);
    }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Rows are spread over WPR warps (one block per row at a time, grid-stride over rows):
// thread t of the block owns the 16-byte vectors vi = k * 32 * WPR + t (k < NCW), so a
// warp's lanes touch consecutive vectors.  gamma and beta stay in registers across rows;
// row sums go through shared memory (one slot per reduction of a row).
template <int WPR>
__device__ __forceinline__ float block_sum(float x, float (*red)[4], int slot) {
    x = warp_sum(x);
    if (WPR == 1) return x;
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[slot][warp] = x;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < WPR; w++) t += red[slot][w];
    return t;
}

__device__ __forceinline__ void load_f32v(const float* base, int c, int n, float* out) {
    if (n == 8) {
        const float4 a = *reinterpret_cast<const float4*>(base + c);
        const float4 b = *reinterpret_cast<const float4*>(base + c + 4);
        out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
        out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
    } else {
        const float4 a = *reinterpret_cast<const float4*>(base + c);
        out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    }
}

template <typename T, int WPR, int NCW>
__global__ void __launch_bounds__(32 * WPR) ln_fwd_kernel(LnParams p) {
    constexpr int V = Vec<T>::N;
    __shared__ float red[2][4];
    const int nvec = p.D / V;
    float gm[NCW][V], bt[NCW][V];
#pragma unroll
    for (int k = 0; k < NCW; k++) {
        const int vi = k * 32 * WPR + threadIdx.x;
        if (vi < nvec) {
            load_f32v(p.gamma, vi * V, V, gm[k]);
            load_f32v(p.beta, vi * V, V, bt[k]);
        }
    }
    for (long long row = blockIdx.x; row < p.T; row += gridDim.x) {
        const size_t base = (size_t)row * p.D;
        float x[NCW][V], u[NCW][V];
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < NCW; k++) {
            const int vi = k * 32 * WPR + threadIdx.x;
            if (vi < nvec) {
                Vec<T>::load(p.y, base + (size_t)vi * V, x[k]);
                Vec<T>::load(p.u, base + (size_t)vi * V, u[k]);
#pragma unroll
                for (int e = 0; e < V; e++) s += x[k][e];
            }
        }
        const float mean = block_sum<WPR>(s, red, 0) / p.D;
        float q = 0.f;
#pragma unroll
        for (int k = 0; k < NCW; k++) {
            const int vi = k * 32 * WPR + threadIdx.x;
            if (vi < nvec) {
#pragma unroll
                for (int e = 0; e < V; e++) {
                    const float d = x[k][e] - mean;
                    q += d * d;
                }
            }
        }
        const float rstd = rsqrtf(block_sum<WPR>(q, red, 1) / p.D + p.eps);
#pragma unroll
        for (int k = 0; k < NCW; k++) {
            const int vi = k * 32 * WPR + threadIdx.x;
            if (vi < nvec) {
                float o[V];
#pragma unroll
                for (int e = 0; e < V; e++) o[e] = ((x[k][e] - mean) * rstd * gm[k][e] + bt[k][e]) * u[k][e];
                Vec<T>::store(p.o, base + (size_t)vi * V, o);
            }
        }
        if (threadIdx.x == 0) {
            if (p.mean) p.mean[row] = mean;
            if (p.rstd) p.rstd[row] = rstd;
        }
    }
}

// Each block leaves its partial dgamma / dbeta in p.part[block]: every column is owned by
// one thread of the block, so the partials are deterministic for a given grid.
template <typename T, int WPR, int NCW>
__global__ void __launch_bounds__(32 * WPR) ln_bwd_kernel(LnParams p) {
    constexpr int V = Vec<T>::N;
    __shared__ float red[2][4];
    const int nvec = p.D / V;
    float gm[NCW][V], bt[NCW][V], ag[NCW][V], ab[NCW][V];
#pragma unroll
    for (int k = 0; k < NCW; k++) {
        const int vi = k * 32 * WPR + threadIdx.x;
#pragma unroll
        for (int e = 0; e < V; e++) ag[k][e] = ab[k][e] = 0.f;
        if (vi < nvec) {
            load_f32v(p.gamma, vi * V, V, gm[k]);
            load_f32v(p.beta, vi * V, V, bt[k]);
        }
    }
    for (long long row = blockIdx.x; row < p.T; row += gridDim.x) {
        const size_t base = (size_t)row * p.D;
        const float mean = p.mean[row], rstd = p.rstd[row];
        float xh[NCW][V], gx[NCW][V];
        float m1 = 0.f, m2 = 0.f;
#pragma unroll
        for (int k = 0; k < NCW; k++) {
            const int vi = k * 32 * WPR + threadIdx.x;
            if (vi < nvec) {
                float y[V], u[V], g[V], du[V];
                Vec<T>::load(p.y, base + (size_t)vi * V, y);
                Vec<T>::load(p.u, base + (size_t)vi * V, u);
                Vec<T>::load(p.g, base + (size_t)vi * V, g);
#pragma unroll
                for (int e = 0; e < V; e++) {
                    xh[k][e] = (y[e] - mean) * rstd;
                    du[e] = g[e] * (xh[k][e] * gm[k][e] + bt[k][e]);
                    const float gl = g[e] * u[e];
                    ag[k][e] += gl * xh[k][e];
                    ab[k][e] += gl;
                    gx[k][e] = gl * gm[k][e];
                    m1 += gx[k][e];
                    m2 += gx[k][e] * xh[k][e];
                }
                Vec<T>::store(p.du, base + (size_t)vi * V, du);
            }
        }
        m1 = block_sum<WPR>(m1, red, 0) / p.D;
        m2 = block_sum<WPR>(m2, red, 1) / p.D;
        const float rs = rstd * p.dy_scale;
#pragma unroll
        for (int k = 0; k < NCW; k++) {
            const int vi = k * 32 * WPR + threadIdx.x;
            if (vi < nvec) {
                float dy[V];
#pragma unroll
                for (int e = 0; e < V; e++) dy[e] = rs * (gx[k][e] - m1 - xh[k][e] * m2);
                Vec<T>::store(p.dy, base + (size_t)vi * V, dy);
            }
        }
    }
    float* part = p.part + (size_t)blockIdx.x * 2 * p.D;
#pragma unroll
    for (int k = 0; k < NCW; k++) {
        const int vi = k * 32 * WPR + threadIdx.x;
        if (vi < nvec) {
#pragma unroll
            for (int e = 0; e < V; e++) {
                part[vi * V + e] = ag[k][e];
                part[p.D + vi * V + e] = ab[k][e];
            }
        }
    }
}

// ---------------------------------------------------------------- Group LayerNorm
// MTGR deep-dive, section 2, and the MTGR arXiv report (GLN): tokens from different
// sources (profile, behaviour, real-time, candidate) are normalised by group so that
// each keeps its own distribution.  Reading: the statistics stay per token over D;
// every group has its own affine gamma_g / beta_g.  Row t uses g = group[t].
//
// Every block owns a contiguous chunk of rows.  It reads the chunk's group ids once,
// lists the rows group by group in shared memory (a stable warp-ballot compaction), and
// then runs the plain row loop once per group present: gamma_g / beta_g and the
// backward's dgamma_g / dbeta_g sums stay in registers as in the plain kernels.  The
// backward leaves one partial row per (block, group present) and a bit mask of the groups
// present; the reduction adds a group's rows in block order (deterministic).
constexpr int kGlnSeg = 1024;              // rows listed at a time (a chunk may take several)

struct GlnList {
    uint8_t g[kGlnSeg];
    int16_t row[kGlnSeg];
    int start[kLnMaxGroups];
    int count[kLnMaxGroups];
};

__device__ __forceinline__ long long gln_chunk(const LnParams& p) {
    return (p.T + gridDim.x - 1) / gridDim.x;
}

// Lists rows [r0, r0 + n) group by group: rows of group k are row[start[k] .. + count[k]).
// A group id >= G sets kStatusBounds and counts as G - 1.
__device__ void gln_list(const LnParams& p, long long r0, int n, GlnList& L) {
    int bad = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        int g = p.group[r0 + i];
        if (g >= p.G) {
            bad = 1;
            g = p.G - 1;
        }
        L.g[i] = (uint8_t)g;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(p.status, kStatusBounds);
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int base = 0;
        for (int k = 0; k < p.G; k++) {
            const int first = base;
            for (int i0 = 0; i0 < n; i0 += 32) {
                const int i = i0 + lane;
                const bool mine = i < n && L.g[i] == k;
                const unsigned bal = __ballot_sync(0xffffffffu, mine);
                if (mine) L.row[base + __popc(bal & ((1u << lane) - 1u))] = (int16_t)i;
                base += __popc(bal);
            }
            if (lane == 0) {
                L.start[k] = first;
                L.count[k] = base - first;
            }
        }
    }
    __syncthreads();
}

template <typename T, int WPR, int NCW>
__global__ void __launch_bounds__(32 * WPR) gln_fwd_kernel(LnParams p) {
    constexpr int V = Vec<T>::N;
    __shared__ float red[2][4];
    __shared__ GlnList L;
    const int nvec = p.D / V;
    const long long chunk = gln_chunk(p);
    const long long c0 = (long long)blockIdx.x * chunk, c1 = min(p.T, c0 + chunk);
    for (long long seg = c0; seg < c1; seg += kGlnSeg) {
        const int n = (int)min((long long)kGlnSeg, c1 - seg);
        gln_list(p, seg, n, L);
        for (int grp = 0; grp < p.G; grp++) {
            const int cnt = L.count[grp], st = L.start[grp];
            if (cnt == 0) continue;
            float gm[NCW][V], bt[NCW][V];
#pragma unroll
            for (int k = 0; k < NCW; k++) {
                const int vi = k * 32 * WPR + threadIdx.x;
                if (vi < nvec) {
                    load_f32v(p.gamma + (size_t)grp * p.D, vi * V, V, gm[k]);
                    load_f32v(p.beta + (size_t)grp * p.D, vi * V, V, bt[k]);
                }
            }
            for (int j = 0; j < cnt; j++) {
                const long long row = seg + L.row[st + j];
                const size_t base = (size_t)row * p.D;
                float x[NCW][V], u[NCW][V];
                float s = 0.f;
#pragma unroll
                for (int k = 0; k < NCW; k++) {
                    const int vi = k * 32 * WPR + threadIdx.x;
                    if (vi < nvec) {
                        Vec<T>::load(p.y, base + (size_t)vi * V, x[k]);
                        Vec<T>::load(p.u, base + (size_t)vi * V, u[k]);
#pragma unroll
                        for (int e = 0; e < V; e++) s += x[k][e];
                    }
                }
                const float mean = block_sum<WPR>(s, red, 0) / p.D;
                float q = 0.f;
#pragma unroll
                for (int k = 0; k < NCW; k++) {
                    const int vi = k * 32 * WPR + threadIdx.x;
                    if (vi < nvec) {
#pragma unroll
                        for (int e = 0; e < V; e++) {
                            const float d = x[k][e] - mean;
                            q += d * d;
                        }
                    }
                }
                const float rstd = rsqrtf(block_sum<WPR>(q, red, 1) / p.D + p.eps);
#pragma unroll
                for (int k = 0; k < NCW; k++) {
                    const int vi = k * 32 * WPR + threadIdx.x;
                    if (vi < nvec) {
                        float o[V];
#pragma unroll
                        for (int e = 0; e < V; e++) o[e] = ((x[k][e] - mean) * rstd * gm[k][e] + bt[k][e]) * u[k][e];
                        Vec<T>::store(p.o, base + (size_t)vi * V, o);
                    }
                }
                if (threadIdx.x == 0) {
                    if (p.mean) p.mean[row] = mean;
                    if (p.rstd) p.rstd[row] = rstd;
                }
            }
        }
        __syncthreads();                                   // L is rebuilt for the next segment
    }
}

template <typename T, int WPR, int NCW>
__global__ void __launch_bounds__(32 * WPR) gln_bwd_kernel(LnParams p) {
    constexpr int V = Vec<T>::N;
    __shared__ float red[2][4];
    __shared__ GlnList L;
    const int nvec = p.D / V;
    const long long chunk = gln_chunk(p);
    const long long c0 = (long long)blockIdx.x * chunk, c1 = min(p.T, c0 + chunk);
    unsigned present = 0;                                  // groups with a partial row written
    for (long long seg = c0; seg < c1; seg += kGlnSeg) {
        const int n = (int)min((long long)kGlnSeg, c1 - seg);
        gln_list(p, seg, n, L);
        for (int grp = 0; grp < p.G; grp++) {
            const int cnt = L.count[grp], st = L.start[grp];
            if (cnt == 0) continue;
            float gm[NCW][V], bt[NCW][V], ag[NCW][V], ab[NCW][V];
#pragma unroll
            for (int k = 0; k < NCW; k++) {
                const int vi = k * 32 * WPR + threadIdx.x;
#pragma unroll
                for (int e = 0; e < V; e++) ag[k][e] = ab[k][e] = 0.f;
                if (vi < nvec) {
                    load_f32v(p.gamma + (size_t)grp * p.D, vi * V, V, gm[k]);
                    load_f32v(p.beta + (size_t)grp * p.D, vi * V, V, bt[k]);
                }
            }
            for (int j = 0; j < cnt; j++) {
                const long long row = seg + L.row[st + j];
                const size_t base = (size_t)row * p.D;
                const float mean = p.mean[row], rstd = p.rstd[row];
                float xh[NCW][V], gx[NCW][V];
                float m1 = 0.f, m2 = 0.f;
#pragma unroll
                for (int k = 0; k < NCW; k++) {
                    const int vi = k * 32 * WPR + threadIdx.x;
                    if (vi < nvec) {
                        float y[V], u[V], g[V], du[V];
                        Vec<T>::load(p.y, base + (size_t)vi * V, y);
                        Vec<T>::load(p.u, base + (size_t)vi * V, u);
                        Vec<T>::load(p.g, base + (size_t)vi * V, g);
#pragma unroll
                        for (int e = 0; e < V; e++) {
                            xh[k][e] = (y[e] - mean) * rstd;
                            du[e] = g[e] * (xh[k][e] * gm[k][e] + bt[k][e]);
                            const float gl = g[e] * u[e];
                            ag[k][e] += gl * xh[k][e];
                            ab[k][e] += gl;
                            gx[k][e] = gl * gm[k][e];
                            m1 += gx[k][e];
                            m2 += gx[k][e] * xh[k][e];
                        }
                        Vec<T>::store(p.du, base + (size_t)vi * V, du);
                    }
                }
                m1 = block_sum<WPR>(m1, red, 0) / p.D;
                m2 = block_sum<WPR>(m2, red, 1) / p.D;
                const float rs = rstd * p.dy_scale;
#pragma unroll
                for (int k = 0; k < NCW; k++) {
                    const int vi = k * 32 * WPR + threadIdx.x;
                    if (vi < nvec) {
                        float dy[V];
#pragma unroll
                        for (int e = 0; e < V; e++) dy[e] = rs * (gx[k][e] - m1 - xh[k][e] * m2);
                        Vec<T>::store(p.dy, base + (size_t)vi * V, dy);
                    }
                }
            }
            // this block's partial row of group grp: written the first time, then added to
            // (only this thread ever touches these columns of the row)
            float* part = p.part + ((size_t)blockIdx.x * p.G + grp) * 2 * p.D;
            const bool first = !(present & (1u << grp));
#pragma unroll
            for (int k = 0; k < NCW; k++) {
                const int vi = k * 32 * WPR + threadIdx.x;
                if (vi < nvec) {
#pragma unroll
                    for (int e = 0; e < V; e++) {
                        float* a = part + vi * V + e;
                        float* c = part + p.D + vi * V + e;
                        *a = first ? ag[k][e] : *a + ag[k][e];
                        *c = first ? ab[k][e] : *c + ab[k][e];
                    }
                }
            }
            present |= 1u << grp;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) p.gmask[blockIdx.x] = (int)present;
}

// Sums the per-block partials in a fixed order (deterministic): a block owns 32 of the
// 2D columns of one group (blockIdx.y; the plain LayerNorm is group 0); warp w sums the
// partial rows of blocks w, w+8, w+16, ... that hold the group (coalesced 128-byte rows),
// and warp 0 adds the eight warp sums in order.
__global__ void __launch_bounds__(256) ln_bwd_reduce_kernel(LnParams p) {
    __shared__ float acc[8][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.y;
    const int c = blockIdx.x * 32 + lane;
    float s = 0.f;
    if (c < 2 * p.D) {
        if (p.G > 1) {
            for (int k = warp; k < p.n_part; k += 8)
                if (p.gmask[k] & (1 << g)) s += p.part[((size_t)k * p.G + g) * 2 * p.D + c];
        } else {
            for (int k = warp; k < p.n_part; k += 8) s += p.part[(size_t)k * 2 * p.D + c];
        }
    }
    acc[warp][lane] = s;
    __syncthreads();
    if (warp == 0 && c < 2 * p.D) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; w++) t += acc[w][lane];
        if (c < p.D) p.d_gamma[(size_t)g * p.D + c] = t;
        else p.d_beta[(size_t)g * p.D + c - p.D] = t;
    }
}

// Warps per row and 16-byte vectors per thread for a row of D elements.
template <typename T>
bool pick_shape(int D, int* wpr, int* ncw) {
    constexpr int V = Vec<T>::N;
    const int nvec = D / V;
    *wpr = nvec > 64 ? 4 : (nvec > 32 ? 2 : 1);   // below four warps one vector per thread
    const int per = 32 * *wpr;
    const int n = (nvec + per - 1) / per;
    *ncw = n <= 1 ? 1 : (n <= 2 ? 2 : (n <= 4 ? 4 : (n <= 8 ? 8 : 0)));
    return *ncw != 0;
}

#define HSTU_LN_DISPATCH(KERNEL, GRID, WPR_, NCW_)                                          \
    do {                                                                                     \
        if (WPR_ == 1) KERNEL<T, 1, 1><<<GRID, 32, 0, s>>>(p);                              \
        else if (WPR_ == 2) KERNEL<T, 2, 1><<<GRID, 64, 0, s>>>(p);                          \
        else if (NCW_ == 1) KERNEL<T, 4, 1><<<GRID, 128, 0, s>>>(p);                         \
        else if (NCW_ == 2) KERNEL<T, 4, 2><<<GRID, 128, 0, s>>>(p);                         \
        else if (NCW_ == 4) KERNEL<T, 4, 4><<<GRID, 128, 0, s>>>(p);                         \
        else KERNEL<T, 4, 8><<<GRID, 128, 0, s>>>(p);                                        \
    } while (0)

#define HSTU_GLN_DISPATCH(KERNEL, GRID, WPR_, NCW_) HSTU_LN_DISPATCH(KERNEL, GRID, WPR_, NCW_)

bool grouped(const LnParams& p) { return p.G > 1; }

template <typename T>
cudaError_t fwd_t(const LnParams& p, cudaStream_t s) {
    int wpr = 0, ncw = 0;
    if (!pick_shape<T>(p.D, &wpr, &ncw)) return cudaErrorInvalidValue;
    prof_begin(kProfLnFwd, s);
    if (grouped(p)) {
        HSTU_GLN_DISPATCH(gln_fwd_kernel, (unsigned)p.n_part, wpr, ncw);
    } else {
        const unsigned grid = (unsigned)(p.T < kLnMaxBlocks ? p.T : kLnMaxBlocks);
        HSTU_LN_DISPATCH(ln_fwd_kernel, grid, wpr, ncw);
    }
    prof_end(kProfLnFwd, s);
    return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_t(const LnParams& p, cudaStream_t s) {
    int wpr = 0, ncw = 0;
    if (!pick_shape<T>(p.D, &wpr, &ncw)) return cudaErrorInvalidValue;
    prof_begin(kProfLnBwd, s);
    if (grouped(p)) {
        HSTU_GLN_DISPATCH(gln_bwd_kernel, (unsigned)p.n_part, wpr, ncw);
    } else {
        HSTU_LN_DISPATCH(ln_bwd_kernel, (unsigned)p.n_part, wpr, ncw);
    }
    prof_end(kProfLnBwd, s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prof_begin(kProfLnBwdReduce, s);
    ln_bwd_reduce_kernel<<<dim3((2 * p.D + 31) / 32, grouped(p) ? p.G : 1), 256, 0, s>>>(p);
    prof_end(kProfLnBwdReduce, s);
    return cudaGetLastError();
}

#undef HSTU_LN_DISPATCH
#undef HSTU_GLN_DISPATCH

}  // namespace

int ln_bwd_partials(long long T) {
    long long n = T < kLnMaxBlocks ? T : kLnMaxBlocks;   // one block per row, grid-stride beyond
    return n < 1 ? 1 : (int)n;
}

// Blocks of the grouped kernels (each takes a contiguous chunk of rows) and the partial
// rows of [2][D] the grouped backward leaves: one per (block, group).
int gln_blocks(long long T) {
    const long long n = T < kGlnMaxBlocks ? T : kGlnMaxBlocks;
    return n < 1 ? 1 : (int)n;
}

cudaError_t launch_ln_fwd(int dtype_f32, const LnParams& p, cudaStream_t s) {
    return dtype_f32 ? fwd_t<float>(p, s) : fwd_t<__nv_bfloat16>(p, s);
}

cudaError_t launch_ln_bwd(int dtype_f32, const LnParams& p, cudaStream_t s) {
    return dtype_f32 ? bwd_t<float>(p, s) : bwd_t<__nv_bfloat16>(p, s);
}

}  // namespace hstu
