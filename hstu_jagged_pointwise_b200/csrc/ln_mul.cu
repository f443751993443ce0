// ln_mul.cu -- the HSTU layer epilogue O_pre = (LayerNorm(Y) * gamma + beta) (.) U and its backward.
//
// Meta HSTU blog, section 3 formula: O = f2(Norm(A V) (.) U); the Norm is a
// LayerNorm over the D = H*d_v concatenated head outputs (biased variance,
// affine gamma / beta).  f2 is outside this path.
//
// HBM-bound: forward reads Y and U and writes O_pre (6D + 8 bytes per bf16
// token incl. mean/rstd); backward reads dO_pre, U, Y, mean, rstd and writes
// dY, dU (10D + 8 bytes per token).  One warp owns one token row; every lane
// moves 16-byte vectors, rows are held in registers between the passes.
#include "internal.h"

namespace hstu {
namespace {

constexpr int kWarps = 8;

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

__device__ __forceinline__ void load_f32x(const float* base, int c, int n, float* out) {
#pragma unroll
    for (int e = 0; e < 8; e++)
        if (e < n) out[e] = base[c + e];
}

// NC = vectors per lane (upper bound); D must be a multiple of Vec<T>::N.
template <typename T, int NC>
__global__ void __launch_bounds__(kWarps * 32) ln_fwd_kernel(LnParams p) {
    constexpr int V = Vec<T>::N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarps + warp;
    if (row >= p.T) return;
    const int nvec = p.D / V;
    const size_t base = (size_t)row * p.D;
    float x[NC][V];
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < NC; k++) {
        const int vi = lane + 32 * k;
        if (vi < nvec) {
            Vec<T>::load(p.y, base + (size_t)vi * V, x[k]);
#pragma unroll
            for (int e = 0; e < V; e++) s += x[k][e];
        }
    }
    const float mean = warp_sum(s) / p.D;
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < NC; k++) {
        const int vi = lane + 32 * k;
        if (vi < nvec) {
#pragma unroll
            for (int e = 0; e < V; e++) {
                const float d = x[k][e] - mean;
                q += d * d;
            }
        }
    }
    const float rstd = rsqrtf(warp_sum(q) / p.D + p.eps);
#pragma unroll
    for (int k = 0; k < NC; k++) {
        const int vi = lane + 32 * k;
        if (vi < nvec) {
            float u[V], g[8], bb[8], o[V];
            Vec<T>::load(p.u, base + (size_t)vi * V, u);
            load_f32x(p.gamma, vi * V, V, g);
            load_f32x(p.beta, vi * V, V, bb);
#pragma unroll
            for (int e = 0; e < V; e++) o[e] = ((x[k][e] - mean) * rstd * g[e] + bb[e]) * u[e];
            Vec<T>::store(p.o, base + (size_t)vi * V, o);
        }
    }
    if (lane == 0) {
        if (p.mean) p.mean[row] = mean;
        if (p.rstd) p.rstd[row] = rstd;
    }
}

// Grid-stride over rows; each block leaves its partial dgamma / dbeta in p.part[block].
template <typename T, int NC>
__global__ void __launch_bounds__(kWarps * 32) ln_bwd_kernel(LnParams p) {
    constexpr int V = Vec<T>::N;
    extern __shared__ float s_acc[];                 // [2][D]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nvec = p.D / V;
    for (int c = threadIdx.x; c < 2 * p.D; c += blockDim.x) s_acc[c] = 0.f;
    float ag[NC][V], ab[NC][V];
#pragma unroll
    for (int k = 0; k < NC; k++)
#pragma unroll
        for (int e = 0; e < V; e++) ag[k][e] = ab[k][e] = 0.f;
    __syncthreads();
    for (long long row = (long long)blockIdx.x * kWarps + warp; row < p.T;
         row += (long long)gridDim.x * kWarps) {
        const size_t base = (size_t)row * p.D;
        const float mean = p.mean[row], rstd = p.rstd[row];
        float xh[NC][V], gx[NC][V];
        float m1 = 0.f, m2 = 0.f;
#pragma unroll
        for (int k = 0; k < NC; k++) {
            const int vi = lane + 32 * k;
            if (vi < nvec) {
                float y[V], u[V], g[V], gm[8], bt[8], du[V];
                Vec<T>::load(p.y, base + (size_t)vi * V, y);
                Vec<T>::load(p.u, base + (size_t)vi * V, u);
                Vec<T>::load(p.g, base + (size_t)vi * V, g);
                load_f32x(p.gamma, vi * V, V, gm);
                load_f32x(p.beta, vi * V, V, bt);
#pragma unroll
                for (int e = 0; e < V; e++) {
                    xh[k][e] = (y[e] - mean) * rstd;
                    du[e] = g[e] * (xh[k][e] * gm[e] + bt[e]);
                    const float gl = g[e] * u[e];
                    ag[k][e] += gl * xh[k][e];
                    ab[k][e] += gl;
                    gx[k][e] = gl * gm[e];
                    m1 += gx[k][e];
                    m2 += gx[k][e] * xh[k][e];
                }
                Vec<T>::store(p.du, base + (size_t)vi * V, du);
            }
        }
        m1 = warp_sum(m1) / p.D;
        m2 = warp_sum(m2) / p.D;
        const float rs = rstd * p.dy_scale;
#pragma unroll
        for (int k = 0; k < NC; k++) {
            const int vi = lane + 32 * k;
            if (vi < nvec) {
                float dy[V];
#pragma unroll
                for (int e = 0; e < V; e++) dy[e] = rs * (gx[k][e] - m1 - xh[k][e] * m2);
                Vec<T>::store(p.dy, base + (size_t)vi * V, dy);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < NC; k++) {
        const int vi = lane + 32 * k;
        if (vi < nvec) {
#pragma unroll
            for (int e = 0; e < V; e++) {
                atomicAdd(&s_acc[vi * V + e], ag[k][e]);
                atomicAdd(&s_acc[p.D + vi * V + e], ab[k][e]);
            }
        }
    }
    __syncthreads();
    float* part = p.part + (size_t)blockIdx.x * 2 * p.D;
    for (int c = threadIdx.x; c < 2 * p.D; c += blockDim.x) part[c] = s_acc[c];
}

// Sums the per-block partials (fixed order: deterministic).
__global__ void ln_bwd_reduce_kernel(LnParams p) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= 2 * p.D) return;
    float s = 0.f;
    for (int k = 0; k < p.n_part; k++) s += p.part[(size_t)k * 2 * p.D + c];
    if (c < p.D) p.d_gamma[c] = s;
    else p.d_beta[c - p.D] = s;
}

template <typename T>
cudaError_t fwd_t(const LnParams& p, cudaStream_t s) {
    constexpr int V = Vec<T>::N;
    const int nc = (p.D / V + 31) / 32;
    const unsigned grid = (unsigned)((p.T + kWarps - 1) / kWarps);
    if (nc > 8) return cudaErrorInvalidValue;
    prof_begin(kProfLnFwd, s);
    if (nc <= 1) ln_fwd_kernel<T, 1><<<grid, kWarps * 32, 0, s>>>(p);
    else if (nc <= 2) ln_fwd_kernel<T, 2><<<grid, kWarps * 32, 0, s>>>(p);
    else if (nc <= 4) ln_fwd_kernel<T, 4><<<grid, kWarps * 32, 0, s>>>(p);
    else ln_fwd_kernel<T, 8><<<grid, kWarps * 32, 0, s>>>(p);
    prof_end(kProfLnFwd, s);
    return cudaGetLastError();
}

template <typename T>
cudaError_t bwd_t(const LnParams& p, cudaStream_t s) {
    constexpr int V = Vec<T>::N;
    const int nc = (p.D / V + 31) / 32;
    const size_t smem = 2 * (size_t)p.D * 4;
    const unsigned grid = (unsigned)p.n_part;
    if (nc > 8) return cudaErrorInvalidValue;
    prof_begin(kProfLnBwd, s);
    if (nc <= 1) ln_bwd_kernel<T, 1><<<grid, kWarps * 32, smem, s>>>(p);
    else if (nc <= 2) ln_bwd_kernel<T, 2><<<grid, kWarps * 32, smem, s>>>(p);
    else if (nc <= 4) ln_bwd_kernel<T, 4><<<grid, kWarps * 32, smem, s>>>(p);
    else ln_bwd_kernel<T, 8><<<grid, kWarps * 32, smem, s>>>(p);
    prof_end(kProfLnBwd, s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prof_begin(kProfLnBwdReduce, s);
    ln_bwd_reduce_kernel<<<(2 * p.D + 255) / 256, 256, 0, s>>>(p);
    prof_end(kProfLnBwdReduce, s);
    return cudaGetLastError();
}

}  // namespace

int ln_bwd_partials(long long T) {
    long long rows_per_block = kWarps * 8;   // at least 8 rows per warp
    long long n = (T + rows_per_block - 1) / rows_per_block;
    if (n < 1) n = 1;
    if (n > 1184) n = 1184;                  // 8 blocks per SM on 148 SMs
    return (int)n;
}

cudaError_t launch_ln_fwd(int dtype_f32, const LnParams& p, cudaStream_t s) {
    return dtype_f32 ? fwd_t<float>(p, s) : fwd_t<__nv_bfloat16>(p, s);
}

cudaError_t launch_ln_bwd(int dtype_f32, const LnParams& p, cudaStream_t s) {
    return dtype_f32 ? bwd_t<float>(p, s) : bwd_t<__nv_bfloat16>(p, s);
}

}  // namespace hstu
