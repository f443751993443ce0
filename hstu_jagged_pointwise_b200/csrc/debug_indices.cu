// debug_indices.cu -- writes the mask bit, rab_pos index and rab_time bucket of
// every pair through the same device functions the attention kernels use, so
// tests can compare the kernels' integer decisions exactly.
#include "internal.h"

namespace hstu {
namespace {

__global__ void debug_indices_kernel(int kind, const int32_t* off, const int64_t* ts,
                                     const int32_t* ns, const int32_t* nr, int P, int nb,
                                     const int64_t* pair_off, uint8_t* m, int16_t* pi, int8_t* tb) {
    const int b = blockIdx.y;
    const int s0 = off[b];
    const int L = off[b + 1] - s0;
    int S = L, R = 0;
    segment_sizes(kind, ns, nr, b, L, &S, &R);
    const long long n = (long long)L * L;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int i = (int)(e / L), j = (int)(e % L);
        const int64_t ti = ts[s0 + i], tj = ts[s0 + j];
        const long long o = pair_off[b] + e;
        m[o] = visible(kind, i, j, S, R, ti, tj) ? 1 : 0;
        pi[o] = (int16_t)pos_index(token_pos(kind, i, S, R), token_pos(kind, j, S, R), P);
        tb[o] = (int8_t)time_bucket(ti, tj, nb);
    }
}

}  // namespace

cudaError_t launch_debug_indices(int B, int kind, const int32_t* off, const int64_t* ts,
                                 const int32_t* ns, const int32_t* nr, int P, int nb,
                                 const int64_t* pair_off, int /*max_len*/, uint8_t* m, int16_t* pi,
                                 int8_t* tb, cudaStream_t s) {
    if (B <= 0) return cudaSuccess;
    dim3 grid(64, B);
    prof_begin(kProfDebugIndices, s);
    debug_indices_kernel<<<grid, 256, 0, s>>>(kind, off, ts, ns, nr, P, nb, pair_off, m, pi, tb);
    prof_end(kProfDebugIndices, s);
    return cudaGetLastError();
}

}  // namespace hstu
