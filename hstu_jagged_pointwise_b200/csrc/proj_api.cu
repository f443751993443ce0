// proj_api.cu -- C ABI of the projections around the attention (declared in include/hstu.h).
//
// Meta HSTU blog, section 3 formula: U, V, Q, K = Split(phi1(f1(X))), phi1 = SiLU, and
// O = f2(Norm(A V) (.) U).  f1 and f2 run on the tcgen05 GEMM of proj_gemm.cu; the
// backward adds two small HBM-bound kernels: dZ = dAct (.) SiLU'(Z) and column sums for
// the bias gradients (fixed-order, deterministic).
#include <math.h>
#include <string.h>

#include <algorithm>

#include "../../include/hstu.h"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kColSumChunks = 512;     // row chunks of the bias-gradient column sums

bool al(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool al_or_null(const void* p, size_t a) { return !p || al(p, a); }

// dZ = dAct * SiLU'(Z); dAct is the U, V, Q
// or K gradient of column block c / D.  A block walks rows (grid-stride); thread i owns
// columns 8i + 2048k, so it also sums its columns of dZ (as stored, in bf16) over the
// block's rows: part[block] is that block's row of db1 partial sums.
constexpr int kSiluGradThreads = 256;
constexpr int kSiluGradBlocks = 148 * 8;
constexpr int kSiluGradCols = 4;       // 8-column groups per thread: 4D <= 8192

// SiLU'(z) = s (1 + z (1 - s)) with s = sigmoid(z) = (1 + tanh(z / 2)) / 2 (one hardware tanh)
__device__ __forceinline__ float silu_grad(float z) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    const float s = fmaf(0.5f, t, 0.5f);
    return s * fmaf(z, 1.0f - s, 1.0f);
}

template <int COLS>
__global__ void __launch_bounds__(kSiluGradThreads, COLS == 4 ? 2 : 4) silu_grad_kernel(long long T, int D, const __nv_bfloat16* z,
                                                                         const __nv_bfloat16* du,
                                                                         const __nv_bfloat16* dv,
                                                                         const __nv_bfloat16* dq,
                                                                         const __nv_bfloat16* dk,
                                                                         __nv_bfloat16* dz, float* part) {
    const int N = 4 * D;
    float acc[COLS][8];
#pragma unroll
    for (int k = 0; k < COLS; k++)
#pragma unroll
        for (int e = 0; e < 8; e++) acc[k][e] = 0.f;
    for (long long t = blockIdx.x; t < T; t += gridDim.x) {
        uint4 a[COLS], b[COLS];
#pragma unroll
        for (int k = 0; k < COLS; k++) {
            const int c = 8 * (threadIdx.x + k * kSiluGradThreads);
            if (c < N) {
                const int which = c / D, col = c - which * D;
                const __nv_bfloat16* src = which == 0 ? du : (which == 1 ? dv : (which == 2 ? dq : dk));
                a[k] = __ldcs(reinterpret_cast<const uint4*>(src + t * D + col));
                b[k] = __ldcs(reinterpret_cast<const uint4*>(z + t * N + c));
            }
        }
#pragma unroll
        for (int k = 0; k < COLS; k++) {
            const int c = 8 * (threadIdx.x + k * kSiluGradThreads);
            if (c < N) {
                const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a[k]);
                const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b[k]);
                uint4 o;
                __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const float2 g = __bfloat1622float2(a2[e]);
                    const float2 x = __bfloat1622float2(b2[e]);
                    o2[e] = __floats2bfloat162_rn(g.x * silu_grad(x.x), g.y * silu_grad(x.y));
                    const float2 q = __bfloat1622float2(o2[e]);
                    acc[k][2 * e] += q.x;
                    acc[k][2 * e + 1] += q.y;
                }
                __stcs(reinterpret_cast<uint4*>(dz + t * N + c), o);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < COLS; k++) {
        const int c = 8 * (threadIdx.x + k * kSiluGradThreads);
        if (c < N) {
            float4* out = reinterpret_cast<float4*>(part + (size_t)blockIdx.x * N + c);
            out[0] = make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
            out[1] = make_float4(acc[k][4], acc[k][5], acc[k][6], acc[k][7]);
        }
    }
}

// part[r][c] = sum of x[t][c] over the rows t of chunk r; 8 columns per thread.
__global__ void __launch_bounds__(128) col_sum_partial_kernel(const __nv_bfloat16* x, long long T, int N,
                                                              float* part) {
    const int c = (blockIdx.x * 128 + threadIdx.x) * 8;
    const long long chunk = (T + gridDim.y - 1) / gridDim.y;
    const long long r0 = (long long)blockIdx.y * chunk, r1 = min(T, r0 + chunk);
    if (c >= N) return;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    long long t = r0;
    for (; t + 4 <= r1; t += 4) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; u++) v[u] = __ldg(reinterpret_cast<const uint4*>(x + (t + u) * N + c));
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const float2 f = __bfloat1622float2(h[e]);
                acc[2 * e] += f.x;
                acc[2 * e + 1] += f.y;
            }
        }
    }
    for (; t < r1; t++) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + t * N + c));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const float2 f = __bfloat1622float2(h[e]);
            acc[2 * e] += f.x;
            acc[2 * e + 1] += f.y;
        }
    }
    float4* out = reinterpret_cast<float4*>(part + (size_t)blockIdx.y * N + c);
    out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

__global__ void __launch_bounds__(256) col_sum_reduce_kernel(const float* part, int N, int R, float* out) {
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c >= N) return;
    float s = 0.f;
    for (int r = 0; r < R; r++) s += part[(size_t)r * N + c];
    out[c] = s;
}

cudaError_t col_sum(const __nv_bfloat16* x, long long T, int N, float* part, float* out, cudaStream_t s) {
    prof_begin(kProfColSum, s);
    col_sum_partial_kernel<<<dim3((N / 8 + 127) / 128, kColSumChunks), 128, 0, s>>>(x, T, N, part);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) {
        col_sum_reduce_kernel<<<(N + 255) / 256, 256, 0, s>>>(part, N, kColSumChunks, out);
        e = cudaGetLastError();
    }
    prof_end(kProfColSum, s);
    return e;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA; }

// One GEMM: tensor maps for A ([M, K] or, MN-major, [K, M]), B ([N, K] or [K, N]) and the
// outputs the epilogue stores (bf16 [M, N], the four [M, D] blocks and Z of f1, or fp32 [M, N]).
int run_gemm(bool a_mn, bool b_mn, int epi, const void* a, const void* b, GemmParams p, cudaStream_t s) {
    CUtensorMap ta, tb;
    GemmOutMaps to;
    memset(&to, 0, sizeof(to));
    const long long a_rows = a_mn ? p.K : p.M, a_cols = a_mn ? p.M : p.K;
    const long long b_rows = b_mn ? p.K : p.N, b_cols = b_mn ? p.N : p.K;
    if (!make_tmap_bf16(&ta, a, a_rows, a_cols, gemm_box_rows(a_mn, false)) ||
        !make_tmap_bf16(&tb, b, b_rows, b_cols, gemm_box_rows(b_mn, true)))
        return HSTU_ERR_CUDA;
    bool ok = true;
    if (epi == kEpiF1) {
        for (int i = 0; i < 4; i++) ok = ok && make_tmap_bf16(&to.out[i], p.out4[i], p.M, p.D, kGemmStoreRows);
        if (p.z) ok = ok && make_tmap_bf16(&to.z, p.z, p.M, p.N, kGemmStoreRows);
    } else if (epi == kEpiAddF32) {
        ok = make_tmap_f32_sw128(&to.out[0], p.out, p.M, p.N, kGemmStoreRows);
    } else {
        ok = make_tmap_bf16(&to.out[0], p.out, p.M, p.N, kGemmStoreRows);
    }
    if (!ok) return HSTU_ERR_CUDA;
    const int sms = device_sms();
    if (sms <= 0) return HSTU_ERR_CUDA;
    if (p.k_splits < 1) p.k_splits = 1;
    const int tiles = gemm_tiles(p);
    if (tiles == 0) return HSTU_OK;
    return status_of(launch_gemm_tc(a_mn, b_mn, epi, ta, tb, to, p, std::min(tiles, sms), s));
}

// Split of K for the weight gradients (K = tokens): about two tiles per SM.
int k_splits_for(int M, int N, int K) {
    const int sms = std::max(device_sms(), 1);
    const int mn = ((M + 127) / 128) * ((N + 255) / 256);
    const int want = (2 * sms + mn - 1) / mn;
    return std::max(1, std::min(want, gemm_k_steps(K)));
}

GemmParams gemm_params(int M, int N, int K, int32_t* status) {
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = K;
    p.k_splits = 1;
    p.status = status;
    p.dbg = debug_wait();
    return p;
}

size_t f1_dz_bytes(long long T, int D) { return align_up((size_t)T * 4 * D * 2, 256); }

}  // namespace
}  // namespace hstu

using namespace hstu;

int hstu_f1_fwd(int32_t T, int32_t d_in, int32_t D, const void* x, const void* w1, const float* b1, void* u,
                void* v, void* q, void* k, void* z, int32_t* device_status, void* stream) {
    if (T < 0 || d_in < 8 || D < 64 || (long long)4 * D > (1 << 20) || d_in > (1 << 20))
        return HSTU_ERR_INVALID_ARG;
    if (d_in % 8 || D % 64) return HSTU_ERR_UNSUPPORTED;
    if (!al_or_null(b1, 16) || !al_or_null(z, 16) || !al_or_null(device_status, 4)) return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (device_status && cudaMemsetAsync(device_status, 0, 4, s) != cudaSuccess) return HSTU_ERR_CUDA;
    if (T == 0) return HSTU_OK;
    if (!al(x, 16) || !al(w1, 16) || !al(u, 16) || !al(v, 16) || !al(q, 16) || !al(k, 16))
        return HSTU_ERR_INVALID_ARG;
    GemmParams p = gemm_params(T, 4 * D, d_in, device_status);
    p.bias = b1;
    p.out4[0] = static_cast<__nv_bfloat16*>(u);
    p.out4[1] = static_cast<__nv_bfloat16*>(v);
    p.out4[2] = static_cast<__nv_bfloat16*>(q);
    p.out4[3] = static_cast<__nv_bfloat16*>(k);
    p.z = static_cast<__nv_bfloat16*>(z);
    p.D = D;
    return run_gemm(false, false, kEpiF1, x, w1, p, s);
}

int hstu_f2_fwd(int32_t T, int32_t D, int32_t d_out, const void* o_pre, const void* w2, const float* b2,
                const void* residual, void* out, int32_t* device_status, void* stream) {
    if (T < 0 || D < 8 || d_out < 32 || D > (1 << 20) || d_out > (1 << 20)) return HSTU_ERR_INVALID_ARG;
    if (D % 8 || d_out % 32) return HSTU_ERR_UNSUPPORTED;
    if (!al_or_null(b2, 16) || !al_or_null(residual, 16) || !al_or_null(device_status, 4))
        return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (device_status && cudaMemsetAsync(device_status, 0, 4, s) != cudaSuccess) return HSTU_ERR_CUDA;
    if (T == 0) return HSTU_OK;
    if (!al(o_pre, 16) || !al(w2, 16) || !al(out, 16)) return HSTU_ERR_INVALID_ARG;
    GemmParams p = gemm_params(T, d_out, D, device_status);
    p.bias = b2;
    p.residual = static_cast<const __nv_bfloat16*>(residual);
    p.out = out;
    return run_gemm(false, false, kEpiF2, o_pre, w2, p, s);
}

size_t hstu_f1_bwd_workspace_bytes(int32_t T, int32_t D) {
    if (T < 0 || D < 32 || D % 32 || 4 * D > 8 * kSiluGradThreads * kSiluGradCols) return 0;
    return f1_dz_bytes(T, D) + (size_t)kSiluGradBlocks * 4 * D * 4;
}

size_t hstu_f2_bwd_workspace_bytes(int32_t T, int32_t d_out) {
    if (T < 0 || d_out < 32 || d_out % 32) return 0;
    return (size_t)kColSumChunks * d_out * 4;
}

int hstu_f1_bwd(int32_t T, int32_t d_in, int32_t D, const void* x, const void* w1, const void* z, const void* du,
                const void* dv, const void* dq, const void* dk, const void* dx_add, void* dx, float* dw1, float* db1,
                void* workspace, size_t workspace_bytes, int32_t* device_status, void* stream) {
    if (T < 0 || d_in < 32 || D < 32 || (long long)4 * D > (1 << 20) || d_in > (1 << 20))
        return HSTU_ERR_INVALID_ARG;
    if (d_in % 32 || D % 32 || 4 * D > 8 * kSiluGradThreads * kSiluGradCols) return HSTU_ERR_UNSUPPORTED;
    if (!al(dw1, 16) || !al(db1, 16) || !al_or_null(device_status, 4) || !al_or_null(dx_add, 16))
        return HSTU_ERR_INVALID_ARG;
    if (!al(workspace, 256) || workspace_bytes < hstu_f1_bwd_workspace_bytes(T, D)) return HSTU_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (device_status && cudaMemsetAsync(device_status, 0, 4, s) != cudaSuccess) return HSTU_ERR_CUDA;
    if (cudaMemsetAsync(dw1, 0, sizeof(float) * 4 * D * (size_t)d_in, s) != cudaSuccess) return HSTU_ERR_CUDA;
    if (T == 0) return status_of(cudaMemsetAsync(db1, 0, sizeof(float) * 4 * D, s));
    if (!al(x, 16) || !al(w1, 16) || !al(z, 16) || !al(du, 16) || !al(dv, 16) || !al(dq, 16) || !al(dk, 16) ||
        !al(dx, 16))
        return HSTU_ERR_INVALID_ARG;
    __nv_bfloat16* dz = static_cast<__nv_bfloat16*>(workspace);
    float* part = reinterpret_cast<float*>(static_cast<char*>(workspace) + f1_dz_bytes(T, D));
    // 1. dZ = dAct * SiLU'(Z), with per-block partial column sums of dZ for db1
    const int gblocks = (int)std::min<long long>(T, kSiluGradBlocks);
    prof_begin(kProfSiluGrad, s);
    {
        const int cols = (4 * D + 8 * kSiluGradThreads - 1) / (8 * kSiluGradThreads);
        auto zb = static_cast<const __nv_bfloat16*>(z);
        auto a0 = static_cast<const __nv_bfloat16*>(du), a1 = static_cast<const __nv_bfloat16*>(dv);
        auto a2 = static_cast<const __nv_bfloat16*>(dq), a3 = static_cast<const __nv_bfloat16*>(dk);
        if (cols <= 1) silu_grad_kernel<1><<<gblocks, kSiluGradThreads, 0, s>>>(T, D, zb, a0, a1, a2, a3, dz, part);
        else if (cols == 2) silu_grad_kernel<2><<<gblocks, kSiluGradThreads, 0, s>>>(T, D, zb, a0, a1, a2, a3, dz, part);
        else silu_grad_kernel<4><<<gblocks, kSiluGradThreads, 0, s>>>(T, D, zb, a0, a1, a2, a3, dz, part);
    }
    if (cudaGetLastError() == cudaSuccess)
        col_sum_reduce_kernel<<<(4 * D + 255) / 256, 256, 0, s>>>(part, 4 * D, gblocks, db1);
    prof_end(kProfSiluGrad, s);
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
    // 2. dX = dZ W1 (+ dx_add) (W1 [4D, d_in] read as the MN-major B operand)
    GemmParams p = gemm_params(T, d_in, 4 * D, device_status);
    p.out = dx;
    p.residual = static_cast<const __nv_bfloat16*>(dx_add);
    int st = run_gemm(false, true, dx_add ? kEpiF2 : kEpiBf16, dz, w1, p, s);
    if (st != HSTU_OK) return st;
    // 3. dW1 = dZ^T X (both operands MN-major), split over the tokens
    GemmParams pw = gemm_params(4 * D, d_in, T, device_status);
    pw.out = dw1;
    pw.k_splits = k_splits_for(4 * D, d_in, T);
    return run_gemm(true, true, kEpiAddF32, dz, x, pw, s);
}

int hstu_f2_bwd(int32_t T, int32_t D, int32_t d_out, const void* o_pre, const void* w2, const void* d_out_grad,
                void* d_o_pre, float* dw2, float* db2, void* workspace, size_t workspace_bytes,
                int32_t* device_status, void* stream) {
    if (T < 0 || D < 32 || d_out < 32 || D > (1 << 20) || d_out > (1 << 20)) return HSTU_ERR_INVALID_ARG;
    if (D % 32 || d_out % 32) return HSTU_ERR_UNSUPPORTED;
    if (!al(dw2, 16) || !al(db2, 16) || !al_or_null(device_status, 4)) return HSTU_ERR_INVALID_ARG;
    if (!al(workspace, 256) || workspace_bytes < hstu_f2_bwd_workspace_bytes(T, d_out)) return HSTU_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (device_status && cudaMemsetAsync(device_status, 0, 4, s) != cudaSuccess) return HSTU_ERR_CUDA;
    if (cudaMemsetAsync(dw2, 0, sizeof(float) * (size_t)d_out * D, s) != cudaSuccess) return HSTU_ERR_CUDA;
    if (T == 0) return status_of(cudaMemsetAsync(db2, 0, sizeof(float) * d_out, s));
    if (!al(o_pre, 16) || !al(w2, 16) || !al(d_out_grad, 16) || !al(d_o_pre, 16)) return HSTU_ERR_INVALID_ARG;
    // 1. dO_pre = dOut W2 (W2 [d_out, D] read as the MN-major B operand)
    GemmParams p = gemm_params(T, D, d_out, device_status);
    p.out = d_o_pre;
    int st = run_gemm(false, true, kEpiBf16, d_out_grad, w2, p, s);
    if (st != HSTU_OK) return st;
    // 2. dW2 = dOut^T O_pre, split over the tokens
    GemmParams pw = gemm_params(d_out, D, T, device_status);
    pw.out = dw2;
    pw.k_splits = k_splits_for(d_out, D, T);
    st = run_gemm(true, true, kEpiAddF32, d_out_grad, o_pre, pw, s);
    if (st != HSTU_OK) return st;
    // 3. db2 = column sums of dOut
    return status_of(col_sum(static_cast<const __nv_bfloat16*>(d_out_grad), T, d_out, static_cast<float*>(workspace),
                             db2, s));
}
