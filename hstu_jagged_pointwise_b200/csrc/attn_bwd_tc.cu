// attn_bwd_tc.cu -- fused jagged HSTU pointwise attention backward on tcgen05 (sm_100a).
//
// The derivative of Y = (1/alpha) sum_j mask * SiLU(z_ij) v_j with
// z_ij = q_i.k_j + rab_pos[pidx] + rab_time[tb] (Meta HSTU blog, sections 3,
// 3.1 and 3.2; the pages give no backward formulas):
//   dA_ij = dy_i . v_j / alpha,  dz_ij = mask * dA_ij * SiLU'(z_ij),
//   SiLU'(z) = sig + SiLU(z) (1 - sig),  sig = sigmoid(z) = (1 + tanh(z/2)) / 2,
//   dV_j = sum_i (mask * SiLU(z_ij) / alpha) dy_i,  dK_j = sum_i dz_ij q_i,
//   dQ_i = sum_j dz_ij k_j,  d_rab_pos[p] / d_rab_time[t] = sum of dz over the pairs using p / t.
// A = SiLU(z) is recomputed from Q and K, never read from memory.
//
// One work item = (sequence, head, 128-key tile); the CTA loops over the
// 128-query tiles that see the key tile, each handled as two 64-query halves so
// that the elementwise warps work on one half while the tensor core runs the
// other half's products.  Per half h (TMEM columns; keys are TMEM lanes):
//   S^T_h  = K Q_h^T    -> [64h, 64h+64)       (SS, both K-major, N = 64)
//   dP^T_h = V dY_h^T   -> [128+64h, +64)      (SS, both K-major, N = 64)
//   elementwise warps: bias, mask, sigmoid; A^T_h (bf16) back into the S^T_h
//                      columns, dZ^T_h (bf16) into shared memory (128-byte swizzle)
//   dV += A^T_h dY_h    -> [256, 256+D)        (TS: A^T from TMEM, dY MN-major)
//   dK += dZ^T_h Q_h    -> [256+D, 256+2D)     (SS: dZ^T K-major, Q MN-major)
//   dQ^T_h = K^T dZ^T_h -> [128+64h, +64)      (SS: K read MN-major, dZ^T MN-major;
//          lanes = head dims), drained by the elementwise warps.
// dY arrives pre-scaled by 1/(2 alpha) (the LayerNorm backward writes it so), which
// turns the elementwise step into, with h = z/2 and t = tanh(h):
//   SiLU(z) = h (1 + t),   2 SiLU'(z) = 1 + t + h (1 - t^2),
//   dz = dP' * 2 SiLU'(z) with dP' = V dY'^T,   dV = 2 A_raw^T dY' (the 2 in the epilogue).
// dQ^T leaves TMEM through registers and a per-warp shared-memory slab; a TMA
// tensor reduce-add sends each slab to the fp32 accumulation buffer.
// Warps 0-15 elementwise (warp w owns TMEM lanes 32*(w%4)..+31 and 16 of the
// half's 64 columns, [16*(w/4), +16)), warp 16 producer (TMA), warp 17 MMA issuer.
// Per visible query tile the elementwise warps run half 0, drain dQ^T_1 of the
// previous tile, run half 1, then drain dQ^T_0 of this tile, so that each drain
// overlaps the tensor core's work on the other half.
// rab gradients: register sums per warp block (uniform bias), per-diagonal sums
// gathered with warp shuffles (position), run-length sums per thread (time),
// sent with fire-and-forget global reductions into this CTA's own partial row;
// a small kernel sums the rows in a fixed order.
// Every wait is bounded; a timeout sets the status word and the CTA exits cleanly.
#include "ew_bias.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace hstu {
namespace {

using namespace ptx;

template <int D>
struct BwdSmem {
    static constexpr uint32_t kTile = 128u * D * 2u;            // one 128-row bf16 tile
    static constexpr uint32_t kHalf = 64u * D * 2u;             // one 64-row bf16 tile
    static constexpr uint32_t k = 0;
    static constexpr uint32_t v = k + kTile;
    static constexpr uint32_t q0 = v + kTile;                    // Q halves (rows 0-63, 64-127)
    static constexpr uint32_t q1 = q0 + kHalf;
    static constexpr uint32_t dy0 = q1 + kHalf;                  // dY halves (rows 0-63, 64-127)
    static constexpr uint32_t dy1 = dy0 + kHalf;
    static constexpr uint32_t dz0 = dy1 + kHalf;                 // dZ^T halves: 128 keys x 64 queries
    static constexpr uint32_t dz1 = dz0 + 128u * 64u * 2u;
    static constexpr uint32_t stg = dz1 + 128u * 64u * 2u;       // float[warps][32 x cols]: dQ slabs
    static constexpr uint32_t rt = stg + 32u * 1024u;            // float[64]
    static constexpr uint32_t rth = rt + kMaxTBuckets * 4u;      // float[64]: rab_time / 2
    static constexpr uint32_t qts = rth + kMaxTBuckets * 4u;     // int64[warps][cols]
    static constexpr uint32_t qrel = qts + 64u * 8u * 4u;        // int32[warps][cols]
    static constexpr uint32_t diag = qrel + 64u * 4u * 4u;       // float[warps][cols + 32]
    static constexpr uint32_t item = diag + 64u * 4u * 4u + 32u * 4u * 16u;   // int4[2]
    static constexpr uint32_t bars = item + 2u * 16u;            // uint64[32]
    static constexpr uint32_t tmem = bars + 32u * 8u;
    static constexpr uint32_t abort_flag = tmem + 4u;
    static constexpr uint32_t rp = abort_flag + 12u;             // float[2P-1], sized at launch
    static constexpr uint32_t alloc(int P) { return rp + 8u * (uint32_t)P + 1024u; }
};

enum {
    kKVFull = 0, kKVEmpty, kQFull0, kQFull1, kQEmpty0, kQEmpty1, kDYFull0, kDYFull1, kDYEmpty0,
    kDYEmpty1, kSFull0, kSFull1, kPFull0, kPFull1, kDQFull0, kDQFull1, kDQDrained0, kDQDrained1,
    kDZEmpty0, kDZEmpty1, kAccFull, kAccEmpty, kItFull0, kItFull1, kItEmpty0, kItEmpty1, kDrain,
    kNumBars
};

// Warp roles: elementwise warps 0 .. kEwWarps-1 (lane quarter w % 4, query group w / 4 of
// kEwCols queries in each 64-query half), then the TMA producer and the MMA issuer.
constexpr int kEwCols = kBwdEwCols;
constexpr int kEwGroups = 64 / kEwCols;
constexpr int kEwWarps = 4 * kEwGroups;
constexpr int kEwThreads = 32 * kEwWarps;
constexpr int kProducerWarp = kEwWarps;
constexpr int kMmaWarp = kEwWarps + 1;
constexpr int kThreads = 32 * (kEwWarps + 2);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 0;
constexpr uint32_t kPCol = 128;
constexpr uint32_t kVCol = 256;
constexpr unsigned kFull = 0xffffffffu;
constexpr uint32_t kPanel = 128u * 128u;                         // 128 rows x 128 B
constexpr uint32_t kHalfPanel = 64u * 128u;                      // 64 rows x 128 B

struct KvItem {
    int b, n0, h, n_end;   // keys [n0, n_end) of sequence b, head h
    int off0, L, S, R;
};

template <int KIND>
__device__ __forceinline__ KvItem load_kv_item(const BwdParams& p, int4 it) {
    KvItem s;
    s.b = it.x; s.n0 = it.y; s.h = it.z; s.n_end = it.w;
    s.off0 = p.off[s.b];
    s.L = p.off[s.b + 1] - s.off0;
    segment_sizes(KIND, p.n_static, p.n_rt, s.b, s.L, &s.S, &s.R);
    return s;
}

// does query tile t see any key of this item?
template <int KIND>
__device__ __forceinline__ int q_class(const KvItem& s, int t) {
    const int qa = t * kTileM;
    const int qb = min(qa + kTileM - 1, s.L - 1);
    return tile_class(KIND, qa, qb, s.n0, s.n_end - 1, s.S, s.R);
}

// first query tile after t that sees the item's keys, n_qt when none
template <int KIND>
__device__ __forceinline__ int next_visible(const KvItem& s, int t, int n_qt) {
    // causal: once a query tile sees the key tile, every later one does
    if (KIND == HSTU_KIND_CAUSAL && t >= 0) return t + 1 < n_qt ? t + 1 : n_qt;
    for (t++; t < n_qt; t++)
        if (q_class<KIND>(s, t) != 0) break;
    return t;
}

__device__ __forceinline__ void flag_timeout(const BwdParams& p, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicOr(&p.ctrl->status, kStatusTimeout);
}

// Per-diagonal sums of a 32-key x C-query block (keys in lanes): at step k lane L takes
// element k of lane (L + k) mod 32, whose key - query offset is L + ka - i0 (dlo) or,
// after the wrap, L - 32 + ka - i0 (dhi).
template <int C>
__device__ __forceinline__ void diag_sums(const float (&zf)[C], float& dlo, float& dhi) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 0; k < C; k++) {
        const float vd = __shfl_sync(0xffffffffu, zf[k], (lane + k) & 31);
        const bool lo = lane + k < 32;
        dlo += lo ? vd : 0.f;
        dhi += lo ? 0.f : vd;
    }
}

// One dense block of 32 keys (lanes) x C queries (along the chunk).  dg points at
// this lane's diagonal-row entry for the block's first query (later queries sit at
// decreasing addresses); the row holds half the position bias, the causal mask and,
// when the block's time bucket is uniform, half the time bias.  TV: the bucket varies
// inside the block and is computed per element from qr, the block's 32-bit query
// times relative to the warp's smallest key time.  Two variants only, so that the
// elementwise code stays small enough for the instruction cache.  CONST: one bias c0
// for the whole block (position and time bias uniform), no diagonal row.
//
// Queries go in pairs through packed fp32 arithmetic.  With h = z / 2, t = tanh(h) and
// p = 1 + t:  SiLU(z) = h + h t = h p  and  2 SiLU'(z) = p + SiLU(z) (1 - t).  SiLU is
// rounded as in the forward (one fused multiply-add), so A matches the forward's P.
template <bool TV, int C, bool CONST = false>
__device__ __forceinline__ void bwd_block(const uint32_t (&sv)[C], const uint32_t (&dp)[C], const float* dg, float c0,
                                          bool pos_diag, float& dlo, float& dhi, const int32_t* qr, int32_t a_j,
                                          const float* rth, int nbm1, float& acc, float* g_rt,
                                          uint32_t (&pa)[C / 2], uint32_t (&pz)[C / 2]) {
    int32_t q[C];
    if (TV) {
        const int4* q4 = reinterpret_cast<const int4*>(qr);
#pragma unroll
        for (int e = 0; e < C / 4; e++) {
            const int4 v = q4[e];
            q[4 * e] = v.x; q[4 * e + 1] = v.y; q[4 * e + 2] = v.z; q[4 * e + 3] = v.w;
        }
    }
    const float2 one2 = make_float2(1.f, 1.f);
    float zf[C];
    float2 acc2 = make_float2(0.f, 0.f);
    // TV: run-length sums of the time-bias gradient along the row (the bucket changes
    // rarely), each run sent to its bucket by a predicated reduction when it ends
    int cur_t = 0;
    float acc_t = 0.f;
#pragma unroll
    for (int e = 0; e < C; e += 2) {
        float2 hb = CONST ? make_float2(c0, c0) : make_float2(dg[-e], dg[-e - 1]);
        int tb0 = 0, tb1 = 0;
        if (TV) {
            tb0 = time_bucket_u32((uint32_t)abs(q[e] - a_j), nbm1);
            tb1 = time_bucket_u32((uint32_t)abs(q[e + 1] - a_j), nbm1);
            hb.x += rth[tb0];
            hb.y += rth[tb1];
        }
        const float2 h = fma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), make_float2(0.5f, 0.5f), hb);
        const float2 t = make_float2(tanh_approx(h.x), tanh_approx(h.y));
        const float2 p1 = add2(t, one2);
        const float2 av = fma2(h, t, h);                                // SiLU(z)
        const float2 g2 = fma2(av, sub2(one2, t), p1);                 // 2 SiLU'(z)
        const float2 z2 = mul2(make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])), g2);
        zf[e] = z2.x;
        zf[e + 1] = z2.y;
        acc2 = add2(acc2, z2);
        pa[e >> 1] = pack_bf16x2(av.x, av.y);
        pz[e >> 1] = pack_bf16x2(z2.x, z2.y);
        if (TV) {
            if (e == 0) {
                cur_t = tb0;
                acc_t = z2.x;
            } else {
                const bool f0 = tb0 != cur_t;
                red_add_f32_if(f0, &g_rt[cur_t], acc_t);
                acc_t = f0 ? z2.x : acc_t + z2.x;
                cur_t = tb0;
            }
            const bool f1 = tb1 != cur_t;
            red_add_f32_if(f1, &g_rt[cur_t], acc_t);
            acc_t = f1 ? z2.y : acc_t + z2.y;
            cur_t = tb1;
        }
    }
    if (TV) red_add_f32(&g_rt[cur_t], acc_t);
    acc += acc2.x + acc2.y;
    if (pos_diag) diag_sums<C>(zf, dlo, dhi);
}

template <int KIND, int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_dy,
                   const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    using L = BwdSmem<D>;
    constexpr int kPanels = D / 64;
    constexpr uint32_t kKCol = kVCol + D;
    constexpr uint32_t kIdSP = idesc_bf16_f32(128, 64, 0, 0);     // S^T_h, dP^T_h
    constexpr uint32_t kIdV = idesc_bf16_f32(128, D, 0, 1);       // dV: A tmem, B MN-major
    constexpr uint32_t kIdK = idesc_bf16_f32(128, D, 0, 1);       // dK: A K-major, B MN-major
    constexpr uint32_t kIdQ = idesc_bf16_f32(D, 64, 1, 1);        // dQ^T_h: A, B MN-major

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    float* s_rp = reinterpret_cast<float*>(sm + L::rp);
    float* s_rt = reinterpret_cast<float*>(sm + L::rt);
    float* s_rth = reinterpret_cast<float*>(sm + L::rth);
    int64_t* s_qts = reinterpret_cast<int64_t*>(sm + L::qts);
    int4* s_item = reinterpret_cast<int4*>(sm + L::item);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::bars);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::tmem);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L::abort_flag);
    // this CTA's rab-gradient partial sums (global, zeroed by the host, summed by rab_reduce)
    float* g_rp = p.rab_part + (size_t)blockIdx.x * (2 * p.P - 1 + p.nb);
    float* g_rt = g_rp + (2 * p.P - 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int np = 2 * p.P - 1;
    for (int i = tid; i < np; i += kThreads) s_rp[i] = p.rab_pos[i];
    for (int i = tid; i < p.nb; i += kThreads) {
        s_rt[i] = p.rab_time[i];
        s_rth[i] = 0.5f * p.rab_time[i];
    }
    if (tid == 0) {
        for (int i = 0; i < kNumBars; i++) {
            uint32_t c = 1;
            if (i == kPFull0 || i == kPFull1 || i == kDQDrained0 || i == kDQDrained1 || i == kAccEmpty)
                c = kEwThreads;
            if (i == kItEmpty0 || i == kItEmpty1) c = kEwThreads + 1;
            mbar_init(&bars[i], c);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_dy);
        prefetch_tmap(&tm_dq);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == kProducerWarp) {
        // ============================================================ producer
        int it_use = 0, kv_use = 0, q_use[2] = {0, 0}, dy_use[2] = {0, 0};
        bool ok = true;
        while (ok) {
            const int slot = it_use & 1;
            if (lane == 0) {
                ok = mbar_wait(&bars[kItEmpty0 + slot], ((it_use >> 1) & 1) ^ 1, s_abort, p.dbg.limit);
                if (ok) {
                    const int idx = atomicAdd(&p.ctrl->counter, 1);
                    s_item[slot] = idx < p.ctrl->n_items ? p.items[idx] : make_int4(-1, 0, 0, 0);
                    mbar_arrive(&bars[kItFull0 + slot]);
                }
            }
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) break;
            int4 it = s_item[slot];
            it.x = __shfl_sync(kFull, it.x, 0);
            it.y = __shfl_sync(kFull, it.y, 0);
            it.z = __shfl_sync(kFull, it.z, 0);
            it.w = __shfl_sync(kFull, it.w, 0);
            it_use++;
            if (it.x < 0) break;
            if (lane == 0) {
                const KvItem s = load_kv_item<KIND>(p, it);
                ok = mbar_wait(&bars[kKVEmpty], (kv_use & 1) ^ 1, s_abort, p.dbg.limit);
                if (ok && p.dbg.withhold_first_load && kv_use == 0) {
                    // test hook: withhold this CTA's first K/V tile, so the waits for it run out
                    wait_for_abort(s_abort, 2 * p.dbg.limit);
                    ok = false;
                }
                if (ok) {
                    mbar_arrive_expect_tx(&bars[kKVFull], 2 * L::kTile);
                    for (int pn = 0; pn < kPanels; pn++) {
                        tma_load_2d(sm + L::k + pn * kPanel, &tm_k, &bars[kKVFull], s.h * D + pn * 64,
                                    s.off0 + s.n0);
                        tma_load_2d(sm + L::v + pn * kPanel, &tm_v, &bars[kKVFull], s.h * D + pn * 64,
                                    s.off0 + s.n0);
                    }
                    kv_use++;
                }
                const int n_qt = (s.L + kTileM - 1) / kTileM;
                int t_pf = 0;                              // next query tile to prefetch into L2
                for (int t = 0; ok && t < n_qt; t++) {
                    if (q_class<KIND>(s, t) == 0) continue;
                    if (t_pf <= t) t_pf = t + 1;
                    while (t_pf < n_qt && q_class<KIND>(s, t_pf) == 0) t_pf++;
                    if (t_pf < n_qt) {
                        for (int pn = 0; pn < kPanels; pn++) {
                            tma_prefetch_2d(&tm_q, s.h * D + pn * 64, s.off0 + t_pf * kTileM);
                            tma_prefetch_2d(&tm_q, s.h * D + pn * 64, s.off0 + t_pf * kTileM + 64);
                            tma_prefetch_2d(&tm_dy, s.h * D + pn * 64, s.off0 + t_pf * kTileM);
                            tma_prefetch_2d(&tm_dy, s.h * D + pn * 64, s.off0 + t_pf * kTileM + 64);
                        }
                        t_pf++;
                    }
                    for (int hh = 0; ok && hh < 2; hh++) {
                        ok = mbar_wait(&bars[kQEmpty0 + hh], (q_use[hh] & 1) ^ 1, s_abort, p.dbg.limit);
                        if (!ok) break;
                        mbar_arrive_expect_tx(&bars[kQFull0 + hh], L::kHalf);
                        for (int pn = 0; pn < kPanels; pn++)
                            tma_load_2d(sm + (hh ? L::q1 : L::q0) + pn * kHalfPanel, &tm_q, &bars[kQFull0 + hh],
                                        s.h * D + pn * 64, s.off0 + t * kTileM + 64 * hh);
                        q_use[hh]++;
                        ok = mbar_wait(&bars[kDYEmpty0 + hh], (dy_use[hh] & 1) ^ 1, s_abort, p.dbg.limit);
                        if (!ok) break;
                        mbar_arrive_expect_tx(&bars[kDYFull0 + hh], L::kHalf);
                        for (int pn = 0; pn < kPanels; pn++)
                            tma_load_2d(sm + (hh ? L::dy1 : L::dy0) + pn * kHalfPanel, &tm_dy,
                                        &bars[kDYFull0 + hh], s.h * D + pn * 64, s.off0 + t * kTileM + 64 * hh);
                        dy_use[hh]++;
                    }
                }
            }
            ok = __shfl_sync(kFull, ok, 0);
        }
        if (lane == 0) {
            if (!ok && !*s_abort) flag_timeout(p, s_abort);
            if (*s_abort) {
                // drain the copies this warp issued (at most the latest one per buffer)
                volatile int dummy = 0;
                if (kv_use) mbar_wait(&bars[kKVFull], (kv_use - 1) & 1, &dummy);
                for (int hh = 0; hh < 2; hh++)
                    if (q_use[hh]) mbar_wait(&bars[kQFull0 + hh], (q_use[hh] - 1) & 1, &dummy);
                for (int hh = 0; hh < 2; hh++)
                    if (dy_use[hh]) mbar_wait(&bars[kDYFull0 + hh], (dy_use[hh] - 1) & 1, &dummy);
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        // Issue order (below, above the item loop) keeps the next half's scores in flight
        // while the elementwise warps work on the current one.  Q_h is released after the
        // dK product of half h, dY'_h after the dV product.
        int it_use = 0, kv_use = 0, acc_use = 0;
        int q_use[2] = {0, 0}, dy_use[2] = {0, 0}, p_use[2] = {0, 0}, dq_use[2] = {0, 0};
        bool ok = true;
        const uint32_t aK = smem_u32(sm + L::k), aV = smem_u32(sm + L::v);
        const uint32_t aQ[2] = {smem_u32(sm + L::q0), smem_u32(sm + L::q1)};
        const uint32_t aDY[2] = {smem_u32(sm + L::dy0), smem_u32(sm + L::dy1)};
        const uint32_t aDZ[2] = {smem_u32(sm + L::dz0), smem_u32(sm + L::dz1)};
        // S^T_h once Q_h of the tile is loaded
        auto issue_s = [&](int hh) -> bool {
            const bool w = mbar_wait(&bars[kQFull0 + hh], q_use[hh] & 1, s_abort, p.dbg.limit);
            q_use[hh]++;
            if (!w) return false;
            tc_fence_after();
            const uint64_t dK = sdesc_sw128(aK, 16, 1024), dQ = sdesc_sw128(aQ[hh], 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; kk++) {
                const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
                const uint32_t offh = (kk >> 2) * kHalfPanel + (kk & 3) * 32;
                mma_ss(tmem + kSCol + 64 * hh, dK + (off >> 4), dQ + (offh >> 4), kIdSP, kk > 0 ? 1u : 0u);
            }
            return true;
        };
        // dP^T_h once dY'_h is loaded and the previous dQ^T_h has left the columns
        auto issue_dp = [&](int hh) -> bool {
            bool w = mbar_wait(&bars[kDYFull0 + hh], dy_use[hh] & 1, s_abort, p.dbg.limit);
            if (w) w = mbar_wait(&bars[kDQDrained0 + hh], (dq_use[hh] & 1) ^ 1, s_abort, p.dbg.limit);
            if (!w) return false;
            dy_use[hh]++;
            tc_fence_after();
            const uint64_t dV = sdesc_sw128(aV, 16, 1024), dY = sdesc_sw128(aDY[hh], 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; kk++) {
                const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
                const uint32_t offh = (kk >> 2) * kHalfPanel + (kk & 3) * 32;
                mma_ss(tmem + kPCol + 64 * hh, dV + (off >> 4), dY + (offh >> 4), kIdSP, kk > 0 ? 1u : 0u);
            }
            tc_commit(&bars[kSFull0 + hh]);
            return true;
        };
        // dK, dV and dQ^T products of half hh once its elementwise step is done.  dK goes
        // first so that Q_h is released (and the next Q_h can load) as early as possible,
        // then dV (releases dY'_h); dQ^T_h is drained only after the other half's step.
        auto issue_prods = [&](int hh, bool init) -> bool {
            if (!mbar_wait(&bars[kPFull0 + hh], p_use[hh] & 1, s_abort, p.dbg.limit)) return false;
            p_use[hh]++;
            if (init && !mbar_wait(&bars[kAccEmpty], (acc_use & 1) ^ 1, s_abort, p.dbg.limit)) return false;
            tc_fence_after();
            const uint64_t dZk = sdesc_sw128(aDZ[hh], 16, 1024), dQm = sdesc_sw128(aQ[hh], kHalfPanel, 1024);
            // dK += dZ^T_h Q_h
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                mma_ss(tmem + kKCol, dZk + (kk * 32 >> 4), dQm + (kk * 2048 >> 4), kIdK,
                       (!init || kk > 0) ? 1u : 0u);
            }
            tc_commit(&bars[kQEmpty0 + hh]);
            const uint64_t dYm = sdesc_sw128(aDY[hh], kHalfPanel, 1024);
            // dV += A^T_h dY'_h   (A^T_h: the kEwCols queries of group c packed into columns
            // 64h + kEwCols*c .. +kEwCols/2)
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                const uint32_t acol = kSCol + 64 * hh + kEwCols * ((16 * kk) / kEwCols) + 8 * ((16 * kk) % kEwCols / 16);
                mma_ts(tmem + kVCol, tmem + acol, dYm + (kk * 2048 >> 4),
                       kIdV, (!init || kk > 0) ? 1u : 0u);
            }
            tc_commit(&bars[kDYEmpty0 + hh]);
            // dQ^T_h = K^T dZ^T_h   (M = head dims, N = 64 queries, K = 128 keys)
            const uint64_t dKm = sdesc_sw128(aK, kPanel, 1024), dZm = sdesc_sw128(aDZ[hh], 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; kk++)
                mma_ss(tmem + kPCol + 64 * hh, dKm + (kk * 2048 >> 4), dZm + (kk * 2048 >> 4), kIdQ, kk > 0 ? 1u : 0u);
            dq_use[hh]++;
            tc_commit(&bars[kDQFull0 + hh]);
            tc_commit(&bars[kDZEmpty0 + hh]);
            return true;
        };
        // Order per visible query tile t (t' = previous tile, tn = next):
        //   dP^T_0(t) [after dQ^T_0(t') is drained];  products of half 1 of t';  S^T_1(t);
        //   dP^T_1(t) [after dQ^T_1(t') is drained];  products of half 0 of t;  S^T_0(tn).
        // The elementwise warps run half 0 of t, drain dQ^T_1(t'), run half 1 of t, drain
        // dQ^T_0(t): each drain sits between two elementwise steps, and each dP^T waits only
        // for the drain just before it.
        while (ok) {
            const int slot = it_use & 1;
            int4 it = make_int4(-1, 0, 0, 0);
            if (lane == 0) {
                ok = mbar_wait(&bars[kItFull0 + slot], (it_use >> 1) & 1, s_abort, p.dbg.limit);
                if (ok) it = s_item[slot];
            }
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) break;
            it.x = __shfl_sync(kFull, it.x, 0);
            it_use++;
            if (it.x < 0) break;
            if (lane == 0) {
                const KvItem s = load_kv_item<KIND>(p, it);
                const int n_qt = (s.L + kTileM - 1) / kTileM;
                ok = mbar_wait(&bars[kKVFull], kv_use & 1, s_abort, p.dbg.limit);
                kv_use++;
                int t = next_visible<KIND>(s, -1, n_qt);
                bool first = true, pend1 = false;
                if (ok && t < n_qt) ok = issue_s(0);
                while (ok && t < n_qt) {
                    const int tn = next_visible<KIND>(s, t, n_qt);
                    ok = issue_dp(0);
                    if (ok && pend1) ok = issue_prods(1, false);
                    if (ok) ok = issue_s(1);
                    if (ok) ok = issue_dp(1);
                    if (ok) ok = issue_prods(0, first);
                    if (ok && tn < n_qt) ok = issue_s(0);
                    first = false;
                    pend1 = true;
                    t = tn;
                }
                if (ok && pend1) ok = issue_prods(1, false);
                if (ok) {
                    tc_commit(&bars[kKVEmpty]);
                    if (first) ok = mbar_wait(&bars[kAccEmpty], (acc_use & 1) ^ 1, s_abort, p.dbg.limit);
                }
                if (ok) {
                    acc_use++;
                    tc_commit(&bars[kAccFull]);
                    mbar_arrive(&bars[kItEmpty0 + slot]);
                }
            }
            ok = __shfl_sync(kFull, ok, 0);
        }
        if (lane == 0) {
            if (!ok && !*s_abort) flag_timeout(p, s_abort);
            volatile int dummy = 0;
            tc_commit(&bars[kDrain]);
            mbar_wait(&bars[kDrain], 0, &dummy);
        }
    } else {
        // ============================================================ elementwise warps
        constexpr int C = kEwCols;
        constexpr int kDqDims = D == 128 ? 32 : 16;   // dQ slab: head dims per warp
        const int wq = warp & 3;                 // lane quarter: key rows 32*wq .. +31
        const int g = warp >> 2;                 // query group: queries C*g .. +C-1 of each half
        const int r = wq * 32 + lane;            // key row within the tile (TMEM lane)
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const uint32_t aDZ[2] = {smem_u32(sm + L::dz0), smem_u32(sm + L::dz1)};
        int64_t* w_qts = s_qts + warp * C;
        float* w_stg = reinterpret_cast<float*>(sm + L::stg) + warp * (32 * C);
        int32_t* w_qrel = reinterpret_cast<int32_t*>(sm + L::qrel) + warp * C;
        float* w_diag = reinterpret_cast<float*>(sm + L::diag) + warp * (C + 32);
        const int nbm1 = p.nb - 1;
        int it_use = 0, acc_use = 0;
        int s_use[2] = {0, 0}, dz_use[2] = {0, 0}, dq_use[2] = {0, 0};
        bool ok = true;
        while (ok) {
            const int slot = it_use & 1;
            ok = mbar_wait(&bars[kItFull0 + slot], (it_use >> 1) & 1, s_abort, p.dbg.limit);
            if (!__all_sync(kFull, ok)) { ok = false; break; }
            const int4 it = s_item[slot];
            it_use++;
            if (it.x < 0) break;
            const KvItem s = load_kv_item<KIND>(p, it);
            const int j = s.n0 + r;
            const bool key_ok = j < s.n_end;
            const int jc = min(j, s.n_end - 1);
            const int64_t ts_j = p.ts[s.off0 + jc];
            const int pos_j = token_pos(KIND, jc, s.S, s.R);
            const int ka = s.n0 + 32 * wq;           // first key of this warp
            int64_t kmin = key_ok ? ts_j : INT64_MAX, kmax = key_ok ? ts_j : INT64_MIN;
            int warp_keys = key_ok ? 1 : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                kmin = min(kmin, (int64_t)__shfl_xor_sync(kFull, (long long)kmin, o));
                kmax = max(kmax, (int64_t)__shfl_xor_sync(kFull, (long long)kmax, o));
                warp_keys += __shfl_xor_sync(kFull, warp_keys, o);
            }
            const int32_t a_j = (int32_t)(uint32_t)((uint64_t)ts_j - (uint64_t)kmin);
            // |kmin| < 2^62: then tq - kmin cannot wrap to a small value unless it is small
            const bool kmin_ok = (uint64_t)kmin + (1ull << 62) < (1ull << 63);
            const int n_qt = (s.L + kTileM - 1) / kTileM;
            int n_done = 0;
            int t = next_visible<KIND>(s, -1, n_qt), t_prev = -1;
            // ---- drain dQ^T_hh of query tile tq (lanes = head dims, columns = queries): one slab
            // of C queries x kDqDims head dims (row-major) per warp, one TMA reduce-add.  M = 128
            // puts head dim 32*wq + lane in this lane; M = 64 puts head dims 16*wq .. +15 in the
            // first 16 lanes of the lane quarter.  Queries past the sequence end carry exact
            // zeros (their dZ is zero).
            auto drain = [&](int hh, int tq) -> bool {
                const bool w = mbar_wait(&bars[kDQFull0 + hh], dq_use[hh] & 1, s_abort, p.dbg.limit);
                if (!__all_sync(kFull, w)) return false;
                dq_use[hh]++;
                tc_fence_after();
                uint32_t v[C];
                tmem_ld(tmem + lane_base + kPCol + 64 * hh + C * g, v);
                tmem_ld_wait(v);
                tc_fence_before();
                mbar_arrive(&bars[kDQDrained0 + hh]);      // the columns are free again
                const int qi = tq * kTileM + 64 * hh + C * g;   // first query of the columns
                if (qi < s.L) {
                    if (lane == 0) bulk_wait_read_all();       // the previous slab has been read
                    __syncwarp();
                    if (D == 128 || lane < 16) {
#pragma unroll
                        for (int e = 0; e < C; e++) w_stg[e * kDqDims + lane] = __uint_as_float(v[e]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_reduce_add_2d(&tm_dq, w_stg, s.h * D + wq * kDqDims, s.off0 + qi);
                        bulk_commit_group();
                    }
                }
                return true;
            };
            // Per visible query tile t: half 0 of t, drain dQ^T_1 of the previous tile, half 1
            // of t, drain dQ^T_0 of t.
            while (ok && t < n_qt) {
                const int t_nx = next_visible<KIND>(s, t, n_qt);
                for (int hh = 0; hh < 2; hh++) {
                    const int i0 = t * kTileM + 64 * hh + C * g;    // first query of this warp's block
                    __syncwarp();
                    const int iq = i0 + lane % C;                  // lanes past C repeat the block
                    const bool q_ok = iq < s.L;
                    const int64_t tq = q_ok ? p.ts[s.off0 + iq] : 0;
                    if (lane < C) w_qts[lane] = tq;
                    // time range of the block's queries: 32-bit offsets from the warp's smallest
                    // key time and two warp reductions; the 64-bit shuffle tree only when the
                    // span needs it
                    const int64_t dq = (int64_t)((uint64_t)tq - (uint64_t)kmin);
                    int64_t qmin, qmax;
                    if (__all_sync(kFull, kmin_ok && (!q_ok || (dq > INT32_MIN && dq < INT32_MAX)))) {
                        const int32_t rmn = __reduce_min_sync(kFull, q_ok ? (int32_t)dq : INT32_MAX);
                        const int32_t rmx = __reduce_max_sync(kFull, q_ok ? (int32_t)dq : INT32_MIN);
                        qmin = rmn == INT32_MAX ? INT64_MAX : kmin + rmn;
                        qmax = rmx == INT32_MIN ? INT64_MIN : kmin + rmx;
                    } else {
                        qmin = q_ok ? tq : INT64_MAX;
                        qmax = q_ok ? tq : INT64_MIN;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            qmin = min(qmin, (int64_t)__shfl_xor_sync(kFull, (long long)qmin, o));
                            qmax = max(qmax, (int64_t)__shfl_xor_sync(kFull, (long long)qmax, o));
                        }
                    }
                    // ---- classify this warp's block: 32 keys x C queries
                    int wcls = 0;
                    if (warp_keys > 0 && i0 < s.L)
                        wcls = tile_class(KIND, i0, min(i0 + C - 1, s.L - 1), ka, min(ka + 31, s.n_end - 1), s.S, s.R);
                    int pm = -1, tm = -1;                // -1 = element-by-element rules
                    int pidx_u = 0;
                    float c0 = 0.f;
                    TimeClass tc;
                    tc.tb_lo = tc.tb_hi = 0;
                    tc.thr = 0;
                    const bool dense = wcls != 0 && warp_keys == 32 && i0 + C <= s.L &&
                                       (KIND == HSTU_KIND_CAUSAL || wcls == 2);
                    const int dmin = ka - (i0 + C - 1);  // smallest key - query of the block
                    if (dense) {
                        tc = classify_time(kmin, kmax, qmin, qmax, p.nb);
                        if (tc.mode >= 0) {
                            tm = tc.mode;
                            const int dmax = ka + 31 - i0;
                            if (wcls == 2 && dmax <= -(p.P - 1)) { pm = kPosUniform; pidx_u = 0; }
                            else if (wcls == 2 && dmin >= p.P - 1) { pm = kPosUniform; pidx_u = 2 * p.P - 2; }
                            else pm = kPosDiag;
                            // diagonal row: key - query = dmin + k, k in [0, C + 31); a single
                            // constant when both biases are uniform over the block
                            const float tadd = tm == kTimeUniform ? s_rth[tc.tb_lo] : 0.f;
                            if (pm == kPosUniform && tm == kTimeUniform) c0 = 0.5f * s_rp[pidx_u] + tadd;
                            else for (int k = lane; k < C + 31; k += 32) {
                                const int dl = dmin + k;
                                const bool masked = KIND == HSTU_KIND_CAUSAL && dl > 0;
                                w_diag[k] = masked ? kMaskedHalfBias
                                                   : 0.5f * s_rp[min(max(dl, -(p.P - 1)), p.P - 1) + p.P - 1] + tadd;
                            }
                            if (tm != kTimeUniform && lane < C) w_qrel[lane] = (int32_t)dq;
                        }
                    }
                    __syncwarp();
                    ok = mbar_wait(&bars[kSFull0 + hh], s_use[hh] & 1, s_abort, p.dbg.limit);
                    if (ok) ok = mbar_wait(&bars[kDZEmpty0 + hh], (dz_use[hh] & 1) ^ 1, s_abort, p.dbg.limit);
                    if (!__all_sync(kFull, ok)) { ok = false; break; }
                    s_use[hh]++;
                    dz_use[hh]++;
                    tc_fence_after();
                    float acc = 0.f, dlo = 0.f, dhi = 0.f;
                    uint32_t pa[C / 2], pz[C / 2];
                    if (wcls == 0) {
#pragma unroll
                        for (int e = 0; e < C / 2; e++) pa[e] = pz[e] = 0u;
                    } else {
                        uint32_t sv[C], dp[C];
                        tmem_ld(tmem + lane_base + kSCol + 64 * hh + C * g, sv);
                        tmem_ld(tmem + lane_base + kPCol + 64 * hh + C * g, dp);
                        tmem_ld_wait(sv);
                        tmem_ld_wait(dp);
                        const float* dg = w_diag + lane + C - 1;
                        if (pm == kPosUniform && tm == kTimeUniform)
                            bwd_block<false, C, true>(sv, dp, dg, c0, false, dlo, dhi, w_qrel, a_j, s_rth, nbm1, acc, g_rt, pa, pz);
                        else if (tm == kTimeUniform)
                            bwd_block<false, C>(sv, dp, dg, c0, pm == kPosDiag, dlo, dhi, w_qrel, a_j, s_rth, nbm1, acc, g_rt, pa, pz);
                        else if (tm >= 0)
                            bwd_block<true, C>(sv, dp, dg, c0, pm == kPosDiag, dlo, dhi, w_qrel, a_j, s_rth, nbm1, acc, g_rt, pa, pz);
                        else {
                            // element by element (MTGR candidates, ragged edges, int64-wide times)
                            int cur_p = -1, cur_t = -1;
                            float acc_p = 0.f, acc_t = 0.f;
                            float zf[C];
#pragma unroll
                            for (int e = 0; e < C; e += 2) {
                                float av[2];
#pragma unroll
                                for (int f = 0; f < 2; f++) {
                                    const int k = e + f;
                                    const int i = i0 + k;
                                    const int64_t ts_i = w_qts[k];
                                    const bool vis = key_ok && i < s.L && visible(KIND, i, j, s.S, s.R, ts_i, ts_j);
                                    const int pidx = pos_index(token_pos(KIND, min(i, s.L - 1), s.S, s.R), pos_j, p.P);
                                    const int tb = time_bucket(ts_i, ts_j, p.nb);
                                    const float h = fmaf(__uint_as_float(sv[k]), 0.5f, 0.5f * s_rp[pidx] + s_rth[tb]);
                                    const float th = tanh_approx(h);
                                    av[f] = vis ? fmaf(h, th, h) : 0.f;
                                    const float g2 = fmaf(h, fmaf(-th, th, 1.f), th + 1.f);
                                    const float dz = vis ? __uint_as_float(dp[k]) * g2 : 0.f;
                                    zf[k] = dz;
                                    if (KIND != HSTU_KIND_CAUSAL) {
                                        if (pidx != cur_p) {
                                            if (cur_p >= 0 && acc_p != 0.f) red_add_f32(&g_rp[cur_p], acc_p);
                                            cur_p = pidx;
                                            acc_p = 0.f;
                                        }
                                        acc_p += dz;
                                    }
                                    if (tb != cur_t) {
                                        if (cur_t >= 0 && acc_t != 0.f) red_add_f32(&g_rt[cur_t], acc_t);
                                        cur_t = tb;
                                        acc_t = 0.f;
                                    }
                                    acc_t += dz;
                                }
                                pa[e >> 1] = pack_bf16x2(av[0], av[1]);
                                pz[e >> 1] = pack_bf16x2(zf[e], zf[e + 1]);
                            }
                            if (cur_p >= 0 && acc_p != 0.f) red_add_f32(&g_rp[cur_p], acc_p);
                            if (cur_t >= 0 && acc_t != 0.f) red_add_f32(&g_rt[cur_t], acc_t);
                            if (KIND == HSTU_KIND_CAUSAL) diag_sums<C>(zf, dlo, dhi);
                        }
                    }
                    // A^T_h back into TMEM inside the S^T_h columns this warp has read
                    tmem_st(tmem + lane_base + kSCol + 64 * hh + C * g, pa);
                    // dZ^T_h into shared memory: row r, queries C*g .. (128-byte swizzle)
                    const uint32_t row_addr = aDZ[hh] + r * 128;
#pragma unroll
                    for (int e = 0; e < C / 8; e++) {
                        const uint32_t ch = (uint32_t)(((C / 8) * g + e) ^ (r & 7));
                        st_shared_v4(row_addr + ch * 16, pz[4 * e], pz[4 * e + 1], pz[4 * e + 2], pz[4 * e + 3]);
                    }
                    tmem_st_wait();
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(&bars[kPFull0 + hh]);
                    // dQ^T of the other half: half 1 of the previous tile, or half 0 of this one
                    const int dt = hh == 0 ? t_prev : t;
                    if (dt >= 0 && !drain(1 - hh, dt)) { ok = false; break; }
                    // ---- rab gradients of the block, sent once the MMA warp and the other half's
                    // dP^T are unblocked
                    if (pm == kPosUniform || tm == kTimeUniform) {
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
                        if (lane == 0) {
                            if (pm == kPosUniform) red_add_f32(&g_rp[pidx_u], acc);
                            if (tm == kTimeUniform) red_add_f32(&g_rt[tc.tb_lo], acc);
                        }
                    }
                    if (pm == kPosDiag || (pm < 0 && wcls != 0 && KIND == HSTU_KIND_CAUSAL)) {
                        const int np1 = p.P - 1;
                        // dlo: key - query = dmin + lane + C - 1;  dhi: dmin + lane + C - 33
                        if (dlo != 0.f) red_add_f32(&g_rp[min(max(dmin + lane + C - 1, -np1), np1) + np1], dlo);
                        if (lane > 32 - C && dhi != 0.f)
                            red_add_f32(&g_rp[min(max(dmin + lane + C - 33, -np1), np1) + np1], dhi);
                    }
                }
                if (!ok) break;
                n_done++;
                t_prev = t;
                t = t_nx;
            }
            if (ok && t_prev >= 0) ok = drain(1, t_prev);   // the last tile's dQ^T_1
            if (!ok) break;
            // ---------------- epilogue: dV, dK rows of this key tile (D / kEwGroups columns per warp)
            ok = mbar_wait(&bars[kAccFull], acc_use & 1, s_abort, p.dbg.limit);
            if (!__all_sync(kFull, ok)) { ok = false; break; }
            acc_use++;
            tc_fence_after();
            constexpr int kEpCols = D / kEwGroups;
#pragma unroll 1
            for (int c = 0; c < kEpCols / 16; c++) {
                const int col = g * kEpCols + 16 * c;
                uint32_t vv[16], kv[16];
                tmem_ld16(tmem + lane_base + kVCol + col, vv);
                tmem_ld16(tmem + lane_base + kKCol + col, kv);
                tmem_ld_wait(vv);
                tmem_ld_wait(kv);
                if (key_ok) {
                    uint4 wv[2], wk[2];
                    uint32_t* pv = reinterpret_cast<uint32_t*>(wv);
                    uint32_t* pk = reinterpret_cast<uint32_t*>(wk);
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        pv[e] = n_done ? pack_bf16x2(2.f * __uint_as_float(vv[2 * e]), 2.f * __uint_as_float(vv[2 * e + 1])) : 0u;
                        pk[e] = n_done ? pack_bf16x2(__uint_as_float(kv[2 * e]), __uint_as_float(kv[2 * e + 1])) : 0u;
                    }
                    const size_t o = (size_t)(s.off0 + j) * p.ld + (size_t)s.h * D + col;
                    uint4* dv = reinterpret_cast<uint4*>(p.dv + o);
                    uint4* dk = reinterpret_cast<uint4*>(p.dk + o);
                    dv[0] = wv[0];
                    dv[1] = wv[1];
                    dk[0] = wk[0];
                    dk[1] = wk[1];
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[kAccEmpty]);
            mbar_arrive(&bars[kItEmpty0 + slot]);
        }
        if (!ok && lane == 0 && !*s_abort) flag_timeout(p, s_abort);
        if (lane == 0) bulk_wait_all();              // reduce-adds done before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int KIND, int D>
cudaError_t launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdy, const CUtensorMap& tdq, const BwdParams& p, int grid,
                       cudaStream_t s) {
    cudaError_t e = ensure_smem_limit((const void*)attn_bwd_tc_kernel<KIND, D>, BwdSmem<D>::alloc(kMaxPos));
    if (e != cudaSuccess) return e;
    prof_begin(kProfAttnBwdTc, s);
    attn_bwd_tc_kernel<KIND, D><<<grid, kThreads, BwdSmem<D>::alloc(p.P), s>>>(tq, tk, tv, tdy, tdq, p);
    prof_end(kProfAttnBwdTc, s);
    return cudaGetLastError();
}

__global__ void f32_to_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst, long long n4) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        const float4 v = src[i];
        uint2 o;
        o.x = pack_bf16x2(v.x, v.y);
        o.y = pack_bf16x2(v.z, v.w);
        dst[i] = o;
    }
}

__global__ void scale_bf16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, float scale,
                                  long long n8) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
         i += (long long)gridDim.x * blockDim.x) {
        const uint4 v = src[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xffff0000u);
            o[e] = pack_bf16x2(lo * scale, hi * scale);
        }
        dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// d_rab[i] = sum over CTAs of part[cta][i], in CTA order.
__global__ void rab_reduce_kernel(const float* __restrict__ part, int n_part, int P, int nb,
                                  float* __restrict__ d_rab_pos, float* __restrict__ d_rab_time) {
    const int w = 2 * P - 1 + nb;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= w) return;
    float s = 0.f;
    for (int c = 0; c < n_part; c++) s += part[(size_t)c * w + i];
    if (i < 2 * P - 1) d_rab_pos[i] = s;
    else d_rab_time[i - (2 * P - 1)] = s;
}

}  // namespace

cudaError_t launch_rab_reduce(const float* part, int n_part, int P, int nb, float* d_rab_pos,
                              float* d_rab_time, cudaStream_t s) {
    const int w = 2 * P - 1 + nb;
    prof_begin(kProfRabReduce, s);
    rab_reduce_kernel<<<(w + 127) / 128, 128, 0, s>>>(part, n_part, P, nb, d_rab_pos, d_rab_time);
    prof_end(kProfRabReduce, s);
    return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc(int kind, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& tdy, const CUtensorMap& tdq,
                               const BwdParams& p, int grid, cudaStream_t s) {
#define HSTU_BWD_CASE(K, DD) \
    if (kind == K && d == DD) return launch_one<K, DD>(tq, tk, tv, tdy, tdq, p, grid, s);
    HSTU_BWD_CASE(HSTU_KIND_CAUSAL, 128)
    HSTU_BWD_CASE(HSTU_KIND_CAUSAL, 64)
    HSTU_BWD_CASE(HSTU_KIND_MTGR, 128)
    HSTU_BWD_CASE(HSTU_KIND_MTGR, 64)
#undef HSTU_BWD_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_scale_bf16(const __nv_bfloat16* src, __nv_bfloat16* dst, float scale, long long n,
                              cudaStream_t s) {
    const long long n8 = n / 8;   // n is a multiple of 8 (H*d with d in {64, 128})
    long long blocks = (n8 + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    prof_begin(kProfScaleDy, s);
    scale_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(src),
                                                        reinterpret_cast<uint4*>(dst), scale, n8);
    prof_end(kProfScaleDy, s);
    return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* src, __nv_bfloat16* dst, long long n, cudaStream_t s) {
    const long long n4 = n / 4;   // n is a multiple of 8 (H*d with d in {64, 128})
    const int threads = 256;
    long long blocks = (n4 + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    prof_begin(kProfDqConvert, s);
    f32_to_bf16_kernel<<<(unsigned)blocks, threads, 0, s>>>(reinterpret_cast<const float4*>(src),
                                                             reinterpret_cast<uint2*>(dst), n4);
    prof_end(kProfDqConvert, s);
    return cudaGetLastError();
}

}  // namespace hstu
