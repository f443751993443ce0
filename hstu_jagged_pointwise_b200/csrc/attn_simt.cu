// attn_simt.cu -- CUDA-core jagged HSTU attention, fp32 arithmetic.
//
// Forward (Meta HSTU blog, section 3 formula, 3.1 pointwise attention, 3.2
// relative bias):  Y_i = (1/alpha) sum_j mask(i,j) SiLU(z_ij) v_j,
//                  z_ij = q_i.k_j + rab_pos[pidx] + rab_time[tb].
// Backward (the derivative of that formula; the pages give none): with
// dA_ij = dy_i.v_j / alpha and dz_ij = mask * dA_ij * SiLU'(z_ij),
//   dq_i = sum_j dz_ij k_j,  dk_j = sum_i dz_ij q_i,
//   dv_j = sum_i mask * SiLU(z_ij) / alpha * dy_i,
//   d_rab_pos[p] = sum over pairs with pidx = p of dz (same for rab_time).
// A = SiLU(z) is recomputed from q, k, never stored.
//
// These kernels serve dtype fp32 (where 1e-5 relative accuracy rules out
// bf16 tensor-core operands) and any element type for the backward.  Tiles
// are 64 x 64 with the whole head width staged in shared memory as fp32.
#include "internal.h"

namespace hstu {
namespace {

constexpr int kBM = 64;
constexpr int kBN = 64;
constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float sigmoid_acc(float z) { return 1.0f / (1.0f + expf(-z)); }

struct SeqCtx {
    int off0, L, S, R;
};

__device__ __forceinline__ SeqCtx seq_ctx(const SimtParams& p, int b) {
    SeqCtx c;
    c.off0 = p.off[b];
    c.L = p.off[b + 1] - c.off0;
    segment_sizes(p.kind, p.n_static, p.n_rt, b, c.L, &c.S, &c.R);
    return c;
}

// Loads rows [r0, r0 + 64) of head h (zero past L) into an fp32 tile with row stride D + 1.
template <typename T, int D>
__device__ __forceinline__ void load_tile(float* dst, const T* src, int ld, const SeqCtx& c, int r0,
                                          int h) {
    for (int e = threadIdx.x; e < kBM * D; e += kThreads) {
        const int r = e / D, col = e % D;
        const int i = r0 + r;
        dst[r * (D + 1) + col] =
            i < c.L ? to_f<T>(src[(size_t)(c.off0 + i) * ld + (size_t)h * D + col]) : 0.f;
    }
}

__device__ __forceinline__ void load_tables(float* s_rp, float* s_rt, const SimtParams& p) {
    for (int e = threadIdx.x; e < 2 * p.P - 1; e += kThreads) s_rp[e] = p.rab_pos[e];
    for (int e = threadIdx.x; e < p.nb; e += kThreads) s_rt[e] = p.rab_time[e];
}

template <int D>
struct SimtSmem {
    static constexpr int LD = D + 1;
    static constexpr int tile = kBM * LD;                  // floats
    static constexpr int ptile = kBM * (kBN + 1);
    static constexpr int fwd_floats = 3 * tile + ptile + 2 * kMaxPos + kMaxTBuckets;
    static constexpr int bwd_floats = 4 * tile + 2 * ptile + 4 * kMaxPos + 2 * kMaxTBuckets;
    static constexpr size_t fwd_bytes = (size_t)fwd_floats * 4 + 2 * kBN * 8;
    static constexpr size_t bwd_bytes = (size_t)bwd_floats * 4 + 2 * kBN * 8;
};

// ------------------------------------------------------------------ forward
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) attn_fwd_simt_kernel(SimtParams p) {
    using Sm = SimtSmem<D>;
    constexpr int LD = Sm::LD, NCOL = D / 4;
    extern __shared__ float smf[];
    int64_t* sTsK = reinterpret_cast<int64_t*>(smf);
    float* sQ = smf + 2 * kBN * 2;
    float* sK = sQ + Sm::tile;
    float* sV = sK + Sm::tile;
    float* sP = sV + Sm::tile;
    float* s_rp = sP + Sm::ptile;
    float* s_rt = s_rp + 2 * kMaxPos;

    const int b = blockIdx.z, h = blockIdx.y, row0 = blockIdx.x * kBM;
    if (!p.ctrl->valid) return;
    const SeqCtx c = seq_ctx(p, b);
    if (row0 >= c.L) return;
    const int ld = p.H * D;
    load_tables(s_rp, s_rt, p);
    load_tile<T, D>(sQ, static_cast<const T*>(p.q), ld, c, row0, h);

    const int r = threadIdx.x >> 2, cg = threadIdx.x & 3;
    const int i = row0 + r;
    const bool row_ok = i < c.L;
    const int ic = min(i, c.L - 1);
    const int64_t ts_i = p.ts[c.off0 + ic];
    const int pos_i = token_pos(p.kind, ic, c.S, c.R);
    float acc[NCOL];
#pragma unroll
    for (int e = 0; e < NCOL; e++) acc[e] = 0.f;

    const int n_kt = (c.L + kBN - 1) / kBN;
    const int qb = min(row0 + kBM - 1, c.L - 1);
    for (int t = 0; t < n_kt; t++) {
        const int n0 = t * kBN;
        if (tile_class(p.kind, row0, qb, n0, min(n0 + kBN - 1, c.L - 1), c.S, c.R) == 0) continue;
        __syncthreads();
        load_tile<T, D>(sK, static_cast<const T*>(p.k), ld, c, n0, h);
        load_tile<T, D>(sV, static_cast<const T*>(p.v), ld, c, n0, h);
        for (int e = threadIdx.x; e < kBN; e += kThreads)
            sTsK[e] = n0 + e < c.L ? p.ts[c.off0 + n0 + e] : 0;
        __syncthreads();
        for (int jj = 0; jj < 16; jj++) {
            const int jl = cg * 16 + jj, j = n0 + jl;
            float s = 0.f;
#pragma unroll 8
            for (int e = 0; e < D; e++) s = fmaf(sQ[r * LD + e], sK[jl * LD + e], s);
            const bool vis = row_ok && j < c.L && visible(p.kind, i, j, c.S, c.R, ts_i, sTsK[jl]);
            const float z = s + s_rp[pos_index(pos_i, token_pos(p.kind, j, c.S, c.R), p.P)] +
                            s_rt[time_bucket(ts_i, sTsK[jl], p.nb)];
            sP[r * (kBN + 1) + jl] = vis ? z * sigmoid_acc(z) : 0.f;
        }
        __syncthreads();
        for (int jl = 0; jl < kBN; jl++) {
            const float a = sP[r * (kBN + 1) + jl];
#pragma unroll
            for (int e = 0; e < NCOL; e++) acc[e] = fmaf(a, sV[jl * LD + cg * NCOL + e], acc[e]);
        }
    }
    if (row_ok) {
        T* y = static_cast<T*>(p.y) + (size_t)(c.off0 + i) * ld + (size_t)h * D + cg * NCOL;
#pragma unroll
        for (int e = 0; e < NCOL; e++) y[e] = from_f<T>(acc[e] * p.inv_alpha);
    }
}

// One (query tile, key tile) block of the backward: fills sA = mask*SiLU(z)/alpha and
// sDZ = dz for rows [qa, qa+64) x cols [ka, ka+64).  Thread (x, cg) handles pair
// rows/cols given by the caller's mapping.
struct PairOut {
    float a, dz;
    int pidx, tb;
    bool vis;
};

__device__ __forceinline__ PairOut pair_grad(const SimtParams& p, const SeqCtx& c, float s, float da,
                                             int i, int j, int64_t ts_i, int64_t ts_j,
                                             const float* s_rp, const float* s_rt) {
    PairOut o;
    o.vis = i < c.L && j < c.L && visible(p.kind, i, j, c.S, c.R, ts_i, ts_j);
    const int ic = min(i, c.L - 1), jc = min(j, c.L - 1);
    o.pidx = pos_index(token_pos(p.kind, ic, c.S, c.R), token_pos(p.kind, jc, c.S, c.R), p.P);
    o.tb = time_bucket(ts_i, ts_j, p.nb);
    const float z = s + s_rp[o.pidx] + s_rt[o.tb];
    const float sg = sigmoid_acc(z);
    o.a = o.vis ? z * sg * p.inv_alpha : 0.f;
    o.dz = o.vis ? da * p.inv_alpha * sg * (1.f + z * (1.f - sg)) : 0.f;
    return o;
}

// ------------------------------------------------------------------ backward: dK, dV, d_rab
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) attn_bwd_dkv_simt_kernel(SimtParams p) {
    using Sm = SimtSmem<D>;
    constexpr int LD = Sm::LD, NCOL = D / 4;
    extern __shared__ float smf[];
    int64_t* sTsQ = reinterpret_cast<int64_t*>(smf);
    int64_t* sTsK = sTsQ + kBN;
    float* sQ = smf + 4 * kBN;
    float* sK = sQ + Sm::tile;
    float* sV = sK + Sm::tile;
    float* sDY = sV + Sm::tile;
    float* sA = sDY + Sm::tile;
    float* sDZ = sA + Sm::ptile;
    float* s_rp = sDZ + Sm::ptile;
    float* s_rt = s_rp + 2 * kMaxPos;
    float* g_rp = s_rt + kMaxTBuckets;
    float* g_rt = g_rp + 2 * kMaxPos;

    const int b = blockIdx.z, h = blockIdx.y, n0 = blockIdx.x * kBN;
    if (!p.ctrl->valid) return;
    const SeqCtx c = seq_ctx(p, b);
    if (n0 >= c.L) return;
    const int ld = p.H * D;
    load_tables(s_rp, s_rt, p);
    for (int e = threadIdx.x; e < 2 * p.P - 1; e += kThreads) g_rp[e] = 0.f;
    for (int e = threadIdx.x; e < p.nb; e += kThreads) g_rt[e] = 0.f;
    load_tile<T, D>(sK, static_cast<const T*>(p.k), ld, c, n0, h);
    load_tile<T, D>(sV, static_cast<const T*>(p.v), ld, c, n0, h);
    for (int e = threadIdx.x; e < kBN; e += kThreads)
        sTsK[e] = n0 + e < c.L ? p.ts[c.off0 + n0 + e] : 0;

    const int jl = threadIdx.x >> 2, cg = threadIdx.x & 3;   // key row of this thread
    const int j = n0 + jl;
    float adk[NCOL], adv[NCOL];
#pragma unroll
    for (int e = 0; e < NCOL; e++) adk[e] = adv[e] = 0.f;

    const int n_qt = (c.L + kBM - 1) / kBM;
    const int kb = min(n0 + kBN - 1, c.L - 1);
    for (int t = 0; t < n_qt; t++) {
        const int qa = t * kBM;
        if (tile_class(p.kind, qa, min(qa + kBM - 1, c.L - 1), n0, kb, c.S, c.R) == 0) continue;
        __syncthreads();
        load_tile<T, D>(sQ, static_cast<const T*>(p.q), ld, c, qa, h);
        load_tile<T, D>(sDY, static_cast<const T*>(p.dy), ld, c, qa, h);
        for (int e = threadIdx.x; e < kBM; e += kThreads)
            sTsQ[e] = qa + e < c.L ? p.ts[c.off0 + qa + e] : 0;
        __syncthreads();
        for (int ii = 0; ii < 16; ii++) {
            const int il = cg * 16 + ii, i = qa + il;
            float s = 0.f, da = 0.f;
#pragma unroll 8
            for (int e = 0; e < D; e++) {
                s = fmaf(sQ[il * LD + e], sK[jl * LD + e], s);
                da = fmaf(sDY[il * LD + e], sV[jl * LD + e], da);
            }
            const PairOut o = pair_grad(p, c, s, da, i, j, sTsQ[il], sTsK[jl], s_rp, s_rt);
            sA[il * (kBN + 1) + jl] = o.a;
            sDZ[il * (kBN + 1) + jl] = o.dz;
            if (o.vis) {
                atomicAdd(&g_rp[o.pidx], o.dz);
                atomicAdd(&g_rt[o.tb], o.dz);
            }
        }
        __syncthreads();
        for (int il = 0; il < kBM; il++) {
            const float a = sA[il * (kBN + 1) + jl], dz = sDZ[il * (kBN + 1) + jl];
#pragma unroll
            for (int e = 0; e < NCOL; e++) {
                adv[e] = fmaf(a, sDY[il * LD + cg * NCOL + e], adv[e]);
                adk[e] = fmaf(dz, sQ[il * LD + cg * NCOL + e], adk[e]);
            }
        }
    }
    if (j < c.L) {
        const size_t o = (size_t)(c.off0 + j) * ld + (size_t)h * D + cg * NCOL;
        T* dk = static_cast<T*>(p.dk) + o;
        T* dv = static_cast<T*>(p.dv) + o;
#pragma unroll
        for (int e = 0; e < NCOL; e++) {
            dk[e] = from_f<T>(adk[e]);
            dv[e] = from_f<T>(adv[e]);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 2 * p.P - 1; e += kThreads)
        if (g_rp[e] != 0.f) atomicAdd(&p.d_rab_pos[e], g_rp[e]);
    for (int e = threadIdx.x; e < p.nb; e += kThreads)
        if (g_rt[e] != 0.f) atomicAdd(&p.d_rab_time[e], g_rt[e]);
}

// ------------------------------------------------------------------ backward: dQ
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) attn_bwd_dq_simt_kernel(SimtParams p) {
    using Sm = SimtSmem<D>;
    constexpr int LD = Sm::LD, NCOL = D / 4;
    extern __shared__ float smf[];
    int64_t* sTsQ = reinterpret_cast<int64_t*>(smf);
    int64_t* sTsK = sTsQ + kBN;
    float* sQ = smf + 4 * kBN;
    float* sK = sQ + Sm::tile;
    float* sV = sK + Sm::tile;
    float* sDY = sV + Sm::tile;
    float* sDZ = sDY + Sm::tile;
    float* s_rp = sDZ + 2 * Sm::ptile;
    float* s_rt = s_rp + 2 * kMaxPos;

    const int b = blockIdx.z, h = blockIdx.y, row0 = blockIdx.x * kBM;
    if (!p.ctrl->valid) return;
    const SeqCtx c = seq_ctx(p, b);
    if (row0 >= c.L) return;
    const int ld = p.H * D;
    load_tables(s_rp, s_rt, p);
    load_tile<T, D>(sQ, static_cast<const T*>(p.q), ld, c, row0, h);
    load_tile<T, D>(sDY, static_cast<const T*>(p.dy), ld, c, row0, h);
    for (int e = threadIdx.x; e < kBM; e += kThreads)
        sTsQ[e] = row0 + e < c.L ? p.ts[c.off0 + row0 + e] : 0;

    const int il = threadIdx.x >> 2, cg = threadIdx.x & 3;
    const int i = row0 + il;
    float adq[NCOL];
#pragma unroll
    for (int e = 0; e < NCOL; e++) adq[e] = 0.f;
    const int n_kt = (c.L + kBN - 1) / kBN;
    const int qb = min(row0 + kBM - 1, c.L - 1);
    for (int t = 0; t < n_kt; t++) {
        const int n0 = t * kBN;
        if (tile_class(p.kind, row0, qb, n0, min(n0 + kBN - 1, c.L - 1), c.S, c.R) == 0) continue;
        __syncthreads();
        load_tile<T, D>(sK, static_cast<const T*>(p.k), ld, c, n0, h);
        load_tile<T, D>(sV, static_cast<const T*>(p.v), ld, c, n0, h);
        for (int e = threadIdx.x; e < kBN; e += kThreads)
            sTsK[e] = n0 + e < c.L ? p.ts[c.off0 + n0 + e] : 0;
        __syncthreads();
        for (int jj = 0; jj < 16; jj++) {
            const int jl = cg * 16 + jj, j = n0 + jl;
            float s = 0.f, da = 0.f;
#pragma unroll 8
            for (int e = 0; e < D; e++) {
                s = fmaf(sQ[il * LD + e], sK[jl * LD + e], s);
                da = fmaf(sDY[il * LD + e], sV[jl * LD + e], da);
            }
            const PairOut o = pair_grad(p, c, s, da, i, j, sTsQ[il], sTsK[jl], s_rp, s_rt);
            sDZ[il * (kBN + 1) + jl] = o.dz;
        }
        __syncthreads();
        for (int jl = 0; jl < kBN; jl++) {
            const float dz = sDZ[il * (kBN + 1) + jl];
#pragma unroll
            for (int e = 0; e < NCOL; e++) adq[e] = fmaf(dz, sK[jl * LD + cg * NCOL + e], adq[e]);
        }
    }
    if (i < c.L) {
        T* dq = static_cast<T*>(p.dq) + (size_t)(c.off0 + i) * ld + (size_t)h * D + cg * NCOL;
#pragma unroll
        for (int e = 0; e < NCOL; e++) dq[e] = from_f<T>(adq[e]);
    }
}

template <typename T, int D>
cudaError_t fwd_one(const SimtParams& p, cudaStream_t s) {
    const size_t smem = SimtSmem<D>::fwd_bytes;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_simt_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.max_len + kBM - 1) / kBM, p.H, p.B);
    prof_begin(kProfAttnFwdSimt, s);
    attn_fwd_simt_kernel<T, D><<<grid, kThreads, smem, s>>>(p);
    prof_end(kProfAttnFwdSimt, s);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t bwd_one(const SimtParams& p, cudaStream_t s) {
    const size_t smem = SimtSmem<D>::bwd_bytes;
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkv_simt_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dq_simt_kernel<T, D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.max_len + kBM - 1) / kBM, p.H, p.B);
    prof_begin(kProfAttnBwdDkvSimt, s);
    attn_bwd_dkv_simt_kernel<T, D><<<grid, kThreads, smem, s>>>(p);
    prof_end(kProfAttnBwdDkvSimt, s);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prof_begin(kProfAttnBwdDqSimt, s);
    attn_bwd_dq_simt_kernel<T, D><<<grid, kThreads, smem, s>>>(p);
    prof_end(kProfAttnBwdDqSimt, s);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_simt(int dtype_f32, int d, const SimtParams& p, cudaStream_t s) {
    if (dtype_f32) {
        if (d == 32) return fwd_one<float, 32>(p, s);
        if (d == 64) return fwd_one<float, 64>(p, s);
        if (d == 128) return fwd_one<float, 128>(p, s);
    } else {
        if (d == 64) return fwd_one<__nv_bfloat16, 64>(p, s);
        if (d == 128) return fwd_one<__nv_bfloat16, 128>(p, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd_simt(int dtype_f32, int d, const SimtParams& p, cudaStream_t s) {
    if (dtype_f32) {
        if (d == 32) return bwd_one<float, 32>(p, s);
        if (d == 64) return bwd_one<float, 64>(p, s);
        if (d == 128) return bwd_one<float, 128>(p, s);
    } else {
        if (d == 64) return bwd_one<__nv_bfloat16, 64>(p, s);
        if (d == 128) return bwd_one<__nv_bfloat16, 128>(p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace hstu
