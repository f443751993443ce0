// attn_fwd_tc.cu -- fused jagged HSTU pointwise attention forward on tcgen05 (sm_100a).
//
// Computes, per (sequence, head, 128-row query tile),
//     Y = (1/alpha) * sum_over_key_tiles  [mask (.) SiLU(Q K^T + rab_pos + rab_time)] V
// (Meta HSTU blog, section 3 formula and 3.1 pointwise attention; section 3.2
// relative attention bias; MTGR pages for the dynamic mixed mask; HSTU blog
// sections 4.2-4.3 for the M-FALCON candidate mask, whose self term is added
// in the epilogue).  There is no softmax, so no running maximum and no
// rescaling: P = SiLU(Z) is written once per tile and accumulated.
//
// One CTA = 10 warps, two CTAs per SM (each owns 256 TMEM columns and ~110 KB
// of shared memory, so one CTA's elementwise phase overlaps the other's MMAs):
//   warps 0-7  elementwise (warp w: TMEM lane quarter w % 4, key half w / 4):
//              TMEM S -> bias, mask, SiLU -> bf16 P back into TMEM;
//              epilogue O/alpha -> global (and the M-FALCON self term)
//   warp 8     producer: dynamic work fetch + TMA loads of Q, K, V tiles
//   warp 9     MMA issuer: S = Q K^T (SS), O += P V (TS, P from TMEM)
// TMEM columns: S/P at [0, 128), O at [128, 128 + D).
// Every wait is bounded; on timeout the CTA records a status bit, drains its
// copies and MMAs, frees TMEM and exits.
#include "ew_bias.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace hstu {
namespace {

using namespace ptx;

template <int D>
struct FwdSmem {
    static constexpr uint32_t kTileBytes = 128u * D * 2u;
    static constexpr uint32_t q = 0;
    static constexpr uint32_t k = q + kTileBytes;
    static constexpr uint32_t v = k + kTileBytes;
    static constexpr uint32_t rt = v + kTileBytes;                 // float[64]
    static constexpr uint32_t rth = rt + kMaxTBuckets * 4u;        // float[64]: rab_time / 2
    static constexpr uint32_t cts = rth + kMaxTBuckets * 4u;       // int64[8 warps][64]
    static constexpr uint32_t diag = cts + 8u * 64u * 8u;          // float[8 warps][96]
    static constexpr uint32_t item = diag + 8u * 96u * 4u;         // int4[2]
    static constexpr uint32_t bars = item + 2u * 16u;              // uint64[16]
    static constexpr uint32_t tmem = bars + 16u * 8u;              // uint32
    static constexpr uint32_t abort_flag = tmem + 4u;              // int
    static constexpr uint32_t rp = abort_flag + 12u;               // float[2P-1], sized at launch
    // bytes to request for a given P (1024 B of slack for the alignment of the base)
    static constexpr uint32_t alloc(int P) { return rp + 8u * (uint32_t)P + 1024u; }
};

enum {
    kQFull = 0, kQEmpty, kKFull, kKEmpty, kVFull, kVEmpty, kSFull, kPFull, kOFull, kOEmpty,
    kItFull0, kItFull1, kItEmpty0, kItEmpty1, kDrain, kNumBars
};

// Warp roles: 8 elementwise warps (lane quarter w % 4 of the tile rows, key half w / 4),
// then the TMA producer and the MMA issuer.
constexpr int kEwWarps = 8;
constexpr int kEwThreads = 32 * kEwWarps;
constexpr int kProducerWarp = kEwWarps;
constexpr int kMmaWarp = kEwWarps + 1;
constexpr int kThreads = 32 * (kEwWarps + 2);
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSCol = 0;
constexpr uint32_t kOCol = 128;
constexpr unsigned kFull = 0xffffffffu;

struct Item {
    int b, row0, h, row_end;   // query rows [row0, row_end) of sequence b, head h
    int q0, Lq, kv0, Lk, S, R;
};

template <int KIND>
__device__ __forceinline__ Item load_item(const FwdParams& p, int4 it) {
    Item s;
    s.b = it.x; s.row0 = it.y; s.h = it.z; s.row_end = it.w;
    s.q0 = p.q_off[s.b];
    s.Lq = p.q_off[s.b + 1] - s.q0;
    s.kv0 = p.kv_off[s.b];
    s.Lk = p.kv_off[s.b + 1] - s.kv0;
    segment_sizes(KIND, p.n_static, p.n_rt, s.b, s.Lq, &s.S, &s.R);
    return s;
}

template <int KIND>
__device__ __forceinline__ int kv_class(const Item& s, int t) {
    const int ka = t * kTileN;
    const int kb = min(ka + kTileN - 1, s.Lk - 1);
    return tile_class(KIND, s.row0, s.row_end - 1, ka, kb, s.S, s.R);
}

template <int KIND>
__device__ __forceinline__ int row_pos(const Item& s, int i) {
    if (KIND == HSTU_KIND_MFALCON) return s.Lk;   // every candidate sits right after its history
    return token_pos(KIND, i, s.S, s.R);
}

template <int KIND>
__device__ __forceinline__ int col_pos(const Item& s, int j) {
    if (KIND == HSTU_KIND_MFALCON) return j;
    return token_pos(KIND, j, s.S, s.R);
}

__device__ __forceinline__ void flag_timeout(const FwdParams& p, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicOr(&p.ctrl->status, kStatusTimeout);
}

// One 32-column chunk of a dense block: rows in lanes, keys along the chunk.
// BM = kBiasConst: one bias c0 for the whole block; kBiasRow: bias from the
// diagonal row (dg points at this lane's entry for the chunk's first key);
// kBiasRowTime: diagonal row plus a per-element time bucket from cr, the chunk's
// 32-bit key times relative to the tile's smallest one.  kBiasRowTwo: the block spans
// two time buckets, told apart by one compare against thr (t_lo / t_hi are their half
// biases).  Four small variants, so that the elementwise code stays small enough for
// the instruction cache.
enum { kBiasConst = 0, kBiasRow = 1, kBiasRowTime = 2, kBiasRowTwo = 3 };

// Half of a block: keys E0 .. E0+15 of the chunk, S values in v.
template <int BM, int E0>
__device__ __forceinline__ void fwd_half(const uint32_t (&v)[16], const float* dg, const int32_t (&b)[16], int32_t a_i,
                                         float c0, const float* rth, int nbm1, uint32_t (&pk)[16],
                                         uint32_t thr, float t_lo, float t_hi) {
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
        float hb[2];
#pragma unroll
        for (int f = 0; f < 2; f++) {
            const int k = E0 + e + f;
            hb[f] = BM == kBiasConst ? c0 : dg[k];
            if (BM == kBiasRowTime) hb[f] += rth[time_bucket_u32((uint32_t)abs(b[k - E0] - a_i), nbm1)];
            if (BM == kBiasRowTwo) hb[f] += (uint32_t)abs(b[k - E0] - a_i) >= thr ? t_hi : t_lo;
        }
        const float2 h = fma2(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), make_float2(0.5f, 0.5f),
                              make_float2(hb[0], hb[1]));
        const float2 a = fma2(h, make_float2(tanh_approx(h.x), tanh_approx(h.y)), h);
        pk[(E0 + e) >> 1] = pack_bf16x2(a.x, a.y);
    }
}

// The chunk's S is read from TMEM in two 16-column halves: the second half's load is in
// flight while the first half is computed.
template <int BM>
__device__ __forceinline__ void fwd_block2(uint32_t taddr, const float* dg, const int32_t* cr, int32_t a_i, float c0,
                                           const float* rth, int nbm1, uint32_t (&pk)[16], uint32_t thr = 0,
                                           float t_lo = 0.f, float t_hi = 0.f) {
    int32_t b[16];
    auto load_b = [&](int h) {
        if (BM == kBiasRowTime || BM == kBiasRowTwo) {
            const int4* b4 = reinterpret_cast<const int4*>(cr + 16 * h);
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int4 x = b4[e];
                b[4 * e] = x.x; b[4 * e + 1] = x.y; b[4 * e + 2] = x.z; b[4 * e + 3] = x.w;
            }
        }
    };
    uint32_t va[16], vb[16];
    tmem_ld16(taddr, va);
    load_b(0);
    tmem_ld_wait(va);
    tmem_ld16(taddr + 16, vb);
    fwd_half<BM, 0>(va, dg, b, a_i, c0, rth, nbm1, pk, thr, t_lo, t_hi);
    load_b(1);
    tmem_ld_wait(vb);
    fwd_half<BM, 16>(vb, dg, b, a_i, c0, rth, nbm1, pk, thr, t_lo, t_hi);
}

// ------------------------------------------------------------------ kernel
template <int KIND, int D>
__global__ void __launch_bounds__(kThreads, 2)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using L = FwdSmem<D>;
    constexpr int kPanels = D / 64;
    constexpr uint32_t kPanelBytes = 128u * 128u;               // 128 rows x 128 B
    constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t kIdescO = idesc_bf16_f32(128, D, 0, 1);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    uint8_t* sQ = sm + L::q;
    uint8_t* sK = sm + L::k;
    uint8_t* sV = sm + L::v;
    float* s_rp = reinterpret_cast<float*>(sm + L::rp);
    float* s_rt = reinterpret_cast<float*>(sm + L::rt);
    float* s_rth = reinterpret_cast<float*>(sm + L::rth);
    int64_t* s_cts = reinterpret_cast<int64_t*>(sm + L::cts);
    float* s_diag = reinterpret_cast<float*>(sm + L::diag);
    int4* s_item = reinterpret_cast<int4*>(sm + L::item);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::bars);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::tmem);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L::abort_flag);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int i = tid; i < 2 * p.P - 1; i += kThreads) s_rp[i] = p.rab_pos[i];
    for (int i = tid; i < p.nb; i += kThreads) {
        s_rt[i] = p.rab_time[i];
        s_rth[i] = 0.5f * p.rab_time[i];
    }
    if (tid == 0) {
        mbar_init(&bars[kQFull], 1);
        mbar_init(&bars[kQEmpty], 1);
        mbar_init(&bars[kKFull], 1);
        mbar_init(&bars[kKEmpty], 1);
        mbar_init(&bars[kVFull], 1);
        mbar_init(&bars[kVEmpty], 1);
        mbar_init(&bars[kSFull], 1);
        mbar_init(&bars[kPFull], kEwThreads);
        mbar_init(&bars[kOFull], 1);
        mbar_init(&bars[kOEmpty], kEwThreads);
        mbar_init(&bars[kItFull0], 1);
        mbar_init(&bars[kItFull1], 1);
        mbar_init(&bars[kItEmpty0], kEwThreads + 1);
        mbar_init(&bars[kItEmpty1], kEwThreads + 1);
        mbar_init(&bars[kDrain], 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
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
        int it_use = 0, q_use = 0, k_use = 0, v_use = 0;
        bool ok = true;
        while (ok) {
            const int slot = it_use & 1;
            if (lane == 0) {
                ok = mbar_wait(&bars[kItEmpty0 + slot], ((it_use >> 1) & 1) ^ 1, s_abort, p.dbg.limit);
                if (ok) {
                    const int idx = atomicAdd(&p.ctrl->counter, 1);
                    const int4 it = idx < p.ctrl->n_items ? p.items[idx] : make_int4(-1, 0, 0, 0);
                    s_item[slot] = it;
                    mbar_arrive(&bars[kItFull0 + slot]);
                }
            }
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) break;
            int4 it = s_item[slot];                 // lane 0 wrote it; broadcast below
            it.x = __shfl_sync(kFull, it.x, 0);
            it.y = __shfl_sync(kFull, it.y, 0);
            it.z = __shfl_sync(kFull, it.z, 0);
            it.w = __shfl_sync(kFull, it.w, 0);
            it_use++;
            if (it.x < 0) break;
            const Item s = load_item<KIND>(p, it);
            if (lane == 0) {
                ok = mbar_wait(&bars[kQEmpty], (q_use & 1) ^ 1, s_abort, p.dbg.limit);
                if (ok && p.dbg.withhold_first_load && q_use == 0) {
                    // test hook: withhold this CTA's first Q tile, so the waits for it run out
                    wait_for_abort(s_abort, 2 * p.dbg.limit);
                    ok = false;
                }
                if (ok) {
                    mbar_arrive_expect_tx(&bars[kQFull], L::kTileBytes);
                    for (int pn = 0; pn < kPanels; pn++)
                        tma_load_2d(sQ + pn * kPanelBytes, &tm_q, &bars[kQFull], s.h * D + pn * 64,
                                    s.q0 + s.row0);
                    q_use++;
                }
                const int n_kt = (s.Lk + kTileN - 1) / kTileN;
                int t_pf = 0;                              // next key tile to prefetch into L2
                for (int t = 0; ok && t < n_kt; t++) {
                    if (kv_class<KIND>(s, t) == 0) continue;
                    if (t_pf <= t) t_pf = t + 1;
                    while (t_pf < n_kt && kv_class<KIND>(s, t_pf) == 0) t_pf++;
                    if (t_pf < n_kt) {
                        for (int pn = 0; pn < kPanels; pn++) {
                            tma_prefetch_2d(&tm_k, s.h * D + pn * 64, s.kv0 + t_pf * kTileN);
                            tma_prefetch_2d(&tm_v, s.h * D + pn * 64, s.kv0 + t_pf * kTileN);
                        }
                        t_pf++;
                    }
                    const int y = s.kv0 + t * kTileN;
                    ok = mbar_wait(&bars[kKEmpty], (k_use & 1) ^ 1, s_abort, p.dbg.limit);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bars[kKFull], L::kTileBytes);
                    for (int pn = 0; pn < kPanels; pn++)
                        tma_load_2d(sK + pn * kPanelBytes, &tm_k, &bars[kKFull], s.h * D + pn * 64, y);
                    k_use++;
                    ok = mbar_wait(&bars[kVEmpty], (v_use & 1) ^ 1, s_abort, p.dbg.limit);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bars[kVFull], L::kTileBytes);
                    for (int pn = 0; pn < kPanels; pn++)
                        tma_load_2d(sV + pn * kPanelBytes, &tm_v, &bars[kVFull], s.h * D + pn * 64, y);
                    v_use++;
                }
            }
            ok = __shfl_sync(kFull, ok, 0);
        }
        if (lane == 0) {
            if (!ok && !*s_abort) flag_timeout(p, s_abort);
            if (*s_abort) {
                // drain the copies this warp issued (at most the last one per buffer)
                volatile int dummy = 0;
                if (q_use) mbar_wait(&bars[kQFull], (q_use - 1) & 1, &dummy);
                if (k_use) mbar_wait(&bars[kKFull], (k_use - 1) & 1, &dummy);
                if (v_use) mbar_wait(&bars[kVFull], (v_use - 1) & 1, &dummy);
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        int it_use = 0, q_use = 0, k_use = 0, v_use = 0, p_use = 0, o_use = 0;
        bool ok = true;
        const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
        // operand descriptors: per-buffer bases plus constant offsets
        const uint64_t dQ = sdesc_sw128(aQ, 16, 1024), dK = sdesc_sw128(aK, 16, 1024);
        const uint64_t dV = sdesc_sw128(aV, kPanelBytes, 1024);
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
                const Item s = load_item<KIND>(p, it);
                const int n_kt = (s.Lk + kTileN - 1) / kTileN;
                int last = -1;
                for (int t = 0; t < n_kt; t++)
                    if (kv_class<KIND>(s, t) != 0) last = t;
                ok = mbar_wait(&bars[kQFull], q_use & 1, s_abort, p.dbg.limit);
                q_use++;
                tc_fence_after();
                int n_done = 0;
                for (int t = 0; ok && t <= last; t++) {
                    if (kv_class<KIND>(s, t) == 0) continue;
                    ok = mbar_wait(&bars[kKFull], k_use & 1, s_abort, p.dbg.limit);
                    if (!ok) break;
                    k_use++;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; kk++) {
                        const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
                        mma_ss(tmem + kSCol, dQ + (off >> 4), dK + (off >> 4), kIdescS, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&bars[kSFull]);
                    tc_commit(&bars[kKEmpty]);
                    if (t == last) tc_commit(&bars[kQEmpty]);
                    ok = mbar_wait(&bars[kPFull], p_use & 1, s_abort, p.dbg.limit);
                    if (!ok) break;
                    p_use++;
                    ok = mbar_wait(&bars[kVFull], v_use & 1, s_abort, p.dbg.limit);
                    if (!ok) break;
                    v_use++;
                    if (n_done == 0) {
                        ok = mbar_wait(&bars[kOEmpty], (o_use & 1) ^ 1, s_abort, p.dbg.limit);
                        if (!ok) break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kTileN / 16; kk++) {
                        // P of keys 32c .. 32c+31 sits in the first 16 columns of S chunk c
                        mma_ts(tmem + kOCol, tmem + kSCol + 32 * (kk >> 1) + 8 * (kk & 1),
                               dV + (kk * 2048 >> 4), kIdescO,
                               (n_done > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(&bars[kVEmpty]);
                    n_done++;
                }
                if (ok && n_done == 0) {
                    tc_commit(&bars[kQEmpty]);
                    ok = mbar_wait(&bars[kOEmpty], (o_use & 1) ^ 1, s_abort, p.dbg.limit);
                }
                if (ok) {
                    o_use++;
                    tc_commit(&bars[kOFull]);
                    mbar_arrive(&bars[kItEmpty0 + slot]);
                }
            }
            ok = __shfl_sync(kFull, ok, 0);
        }
        if (lane == 0) {
            if (!ok && !*s_abort) flag_timeout(p, s_abort);
            // every MMA this thread issued completes before TMEM is released
            volatile int dummy = 0;
            tc_commit(&bars[kDrain]);
            mbar_wait(&bars[kDrain], 0, &dummy);
        }
    } else {
        // ============================================================ elementwise (warps 0-7)
        int it_use = 0, s_use = 0, o_use = 0;
        const int wq = warp & 3;                            // lane quarter: tile rows 32*wq .. +31
        const int g = warp >> 2;                            // key half: tile keys 64*g .. +63
        const int r = wq * 32 + lane;                       // TMEM lane = tile row
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        int64_t* w_cts = s_cts + warp * 64;                 // this warp's column times (int64)
        int32_t* w_crel = reinterpret_cast<int32_t*>(w_cts); // or 32-bit relative times
        float* w_diag = s_diag + warp * 96;
        const int nbm1 = p.nb - 1;
        const float rp_self = s_rp[p.P - 1];
        const float rt_zero = s_rt[0];
        bool ok = true;
        while (ok) {
            const int slot = it_use & 1;
            ok = mbar_wait(&bars[kItFull0 + slot], (it_use >> 1) & 1, s_abort, p.dbg.limit);
            if (!__all_sync(kFull, ok)) { ok = false; break; }
            const int4 it = s_item[slot];
            it_use++;
            if (it.x < 0) break;
            const Item s = load_item<KIND>(p, it);
            const int i = s.row0 + r;
            const bool row_ok = i < s.row_end;
            const int ic = min(i, s.row_end - 1);           // clamped row for lookups
            const int64_t ts_i = p.q_ts[s.q0 + ic];
            const int pos_i = row_pos<KIND>(s, ic);
            const int r0 = s.row0 + 32 * wq;                // first row of this warp
            // this warp's row range (positions and timestamps)
            int64_t rmin = row_ok ? ts_i : INT64_MAX, rmax = row_ok ? ts_i : INT64_MIN;
            int pr_lo = row_ok ? pos_i : INT32_MAX, pr_hi = row_ok ? pos_i : INT32_MIN;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                rmin = min(rmin, (int64_t)__shfl_xor_sync(kFull, (long long)rmin, o));
                rmax = max(rmax, (int64_t)__shfl_xor_sync(kFull, (long long)rmax, o));
                pr_lo = min(pr_lo, __shfl_xor_sync(kFull, pr_lo, o));
                pr_hi = max(pr_hi, __shfl_xor_sync(kFull, pr_hi, o));
            }
            const bool warp_rows = pr_lo <= pr_hi;          // any valid row in this warp
            const int n_kt = (s.Lk + kTileN - 1) / kTileN;
            // column timestamps of this warp's keys, loaded one key tile ahead
            auto next_tile = [&](int tt) {
                for (tt++; tt < n_kt; tt++)
                    if (kv_class<KIND>(s, tt) != 0) break;
                return tt;
            };
            int64_t tj_next[2];
            auto load_tj = [&](int tt) {
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int j = tt * kTileN + 64 * g + lane + 32 * e;
                    tj_next[e] = (tt < n_kt && j < s.Lk) ? __ldg(p.kv_ts + s.kv0 + j) : 0;
                }
            };
            int n_done = 0;
            int t = next_tile(-1);
            load_tj(t);
            for (int t_next; t < n_kt; t = t_next) {
                const int n0 = t * kTileN + 64 * g;         // first key of this warp's half
                __syncwarp();
                int64_t tj[2] = {tj_next[0], tj_next[1]};
                t_next = next_tile(t);
                load_tj(t_next);
                // time range of the warp's keys: 32-bit offsets from the first key's time and
                // two warp reductions; the 64-bit shuffle tree only when the span needs it
                const int64_t ref = __shfl_sync(kFull, (long long)tj[0], 0);
                int32_t dmn = INT32_MAX, dmx = INT32_MIN;
                // |ref| < 2^62: then tj - ref cannot wrap to a small value unless it is small
                bool fits = (uint64_t)ref + (1ull << 62) < (1ull << 63);
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int j = n0 + lane + 32 * e;
                    if (j < s.Lk) {
                        const int64_t dt = (int64_t)((uint64_t)tj[e] - (uint64_t)ref);
                        fits = fits && dt > INT32_MIN && dt < INT32_MAX;
                        dmn = min(dmn, (int32_t)dt);
                        dmx = max(dmx, (int32_t)dt);
                    }
                }
                int64_t cmin, cmax;
                if (__all_sync(kFull, fits)) {
                    dmn = __reduce_min_sync(kFull, dmn);
                    dmx = __reduce_max_sync(kFull, dmx);
                    cmin = dmn == INT32_MAX ? INT64_MAX : ref + dmn;
                    cmax = dmx == INT32_MIN ? INT64_MIN : ref + dmx;
                } else {
                    cmin = INT64_MAX;
                    cmax = INT64_MIN;
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const int j = n0 + lane + 32 * e;
                        if (j < s.Lk) {
                            cmin = min(cmin, tj[e]);
                            cmax = max(cmax, tj[e]);
                        }
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        cmin = min(cmin, (int64_t)__shfl_xor_sync(kFull, (long long)cmin, o));
                        cmax = max(cmax, (int64_t)__shfl_xor_sync(kFull, (long long)cmax, o));
                    }
                }
                // ---- classify this warp's block: 32 rows x 64 columns
                int pm = -1, tm = -1;
                float c0 = 0.f;
                TimeClass tc;
                tc.tb_lo = tc.tb_hi = 0;
                tc.thr = 0;
                int wcls = 0;
                if (warp_rows && n0 < s.Lk)
                    wcls = KIND == HSTU_KIND_MFALCON
                               ? 2
                               : tile_class(KIND, r0, min(r0 + 31, s.row_end - 1), n0,
                                            min(n0 + 63, s.Lk - 1), s.S, s.R);
                const int r_hi = min(r0 + 31, s.row_end - 1);
                // every row of the block is a candidate sharing one position
                const bool rows_shared = KIND == HSTU_KIND_MFALCON || (KIND != HSTU_KIND_CAUSAL && r0 >= s.S + s.R);
                // real-time / history rows against non-candidate keys: the mask is j <= i (a
                // static key precedes every real-time row)
                const bool causal_rows = KIND == HSTU_KIND_CAUSAL ||
                                         (KIND != HSTU_KIND_MFALCON && r0 >= s.S && r_hi < s.S + s.R &&
                                          n0 < s.S + s.R);
                // keys n0 + k with k >= jlim are masked for every row of the block: static rows
                // against a key block that crosses the end of the static segment, real-time rows
                // against one that crosses the end of the history
                int jlim = 64;
                if (KIND == HSTU_KIND_MTGR || KIND == HSTU_KIND_MFSEQ) {
                    if (r_hi < s.S && n0 < s.S && n0 + 63 >= s.S && wcls != 0) {
                        jlim = s.S - n0;
                        wcls = 2;
                    } else if (causal_rows && n0 + 63 >= s.S + s.R) {
                        jlim = s.S + s.R - n0;
                    }
                }
                // MTGR candidate rows against history keys: the timestamp filter passes every
                // pair when the rows' earliest time is after the keys' latest, and no pair when
                // the rows' latest time is at or before the keys' earliest
                if (KIND == HSTU_KIND_MTGR && wcls == 1 && r0 >= s.S + s.R && n0 + 63 < s.S + s.R) {
                    if (rmin > cmax) wcls = 2;
                    else if (rmax <= cmin) wcls = 0;
                }
                const bool dense = wcls != 0 && n0 + 64 <= s.Lk && (wcls == 2 || causal_rows);
                if (dense) {
                    tc = classify_time(rmin, rmax, cmin, cmax, p.nb);
                    const int dmax = col_pos<KIND>(s, n0 + 63) - pr_lo;
                    const int dmin = col_pos<KIND>(s, n0) - pr_hi;
                    int pidx_u = -1;
                    if (wcls == 2 && dmax <= -(p.P - 1)) pidx_u = 0;
                    else if (wcls == 2 && dmin >= p.P - 1) pidx_u = 2 * p.P - 2;
                    // a dense block's rows are all candidates or all indexed by position
                    // (pos_j - pos_i == j - i): one tile class never mixes the two
                    if (pidx_u >= 0) pm = kPosUniform;
                    else pm = rows_shared ? kPosCol : kPosDiag;
                    if (pm >= 0 && tc.mode >= 0) {
                        tm = tc.mode;
                        const float tadd = tm == kTimeUniform ? s_rth[tc.tb_lo] : 0.f;
                        if (pm == kPosUniform && tm == kTimeUniform) {
                            c0 = 0.5f * s_rp[pidx_u] + tadd;
                        } else if (KIND != HSTU_KIND_CAUSAL && pm == kPosCol) {
                            // one row position pr_lo: the bias of key n0 + k sits at w_diag[31 + k]
                            for (int k = lane; k < 64; k += 32)
                                w_diag[31 + k] = 0.5f * s_rp[pos_index(pr_lo, col_pos<KIND>(s, n0 + k), p.P)] + tadd;
                        } else {
                            // diagonal row: delta = j - i = (n0 - r0 - 31) + k, k in [0, 95);
                            // constant when the position index is clamped across the block
                            const int d0 = n0 - r0 - 31;
                            for (int k = lane; k < 95; k += 32) {
                                const int dl = d0 + k;
                                const bool masked = causal_rows && dl > 0;
                                const int pi = pm == kPosUniform ? pidx_u : min(max(dl, -(p.P - 1)), p.P - 1) + p.P - 1;
                                w_diag[k] = masked ? kMaskedHalfBias : 0.5f * s_rp[pi] + tadd;
                            }
                        }
                    } else {
                        pm = -1;
                    }
                }
                if (pm >= 0) {
                    if (tm != kTimeUniform) {
#pragma unroll
                        for (int e = 0; e < 2; e++) w_crel[lane + 32 * e] = (int32_t)(uint32_t)((uint64_t)tj[e] - (uint64_t)cmin);
                    }
                } else if (wcls != 0) {
#pragma unroll
                    for (int e = 0; e < 2; e++) w_cts[lane + 32 * e] = tj[e];
                }
                __syncwarp();
                const int32_t a_i = (int32_t)(uint32_t)((uint64_t)ts_i - (uint64_t)cmin);
                ok = mbar_wait(&bars[kSFull], s_use & 1, s_abort, p.dbg.limit);
                if (!__all_sync(kFull, ok)) { ok = false; break; }
                s_use++;
                tc_fence_after();
#pragma unroll 1
                for (int cc = 0; cc < 2; cc++) {
                    const int c = 2 * g + cc;                // 32-column chunk of the tile
                    uint32_t pk[16];
                    if (wcls == 0) {
                        // nothing visible (masked or past the sequence): P = 0, S is never read
#pragma unroll
                        for (int e = 0; e < 16; e++) pk[e] = 0u;
                        tmem_st16(tmem + lane_base + kSCol + 32 * c, pk);
                        continue;
                    }
                    if (pm < 0) {
                        // element by element (MTGR candidates, ragged key tiles, int64-wide time
                        // spans): a compact loop over key pairs that reads S and writes P in TMEM
                        // pair by pair, so that this rare path adds little code
                        const uint32_t col = tmem + lane_base + kSCol + 32 * c;
#pragma unroll 1
                        for (int e = 0; e < 32; e += 2) {
                            uint32_t s0, s1;
                            tmem_ld2(col + e, s0, s1);
                            float pv[2];
#pragma unroll
                            for (int f = 0; f < 2; f++) {
                                const int jj = 32 * cc + e + f;
                                const int j = n0 + jj;
                                const int64_t ts_j = w_cts[jj];
                                bool vis = row_ok && j < s.Lk;
                                if (KIND != HSTU_KIND_MFALCON)
                                    vis = vis && visible(KIND, i, j, s.S, s.R, ts_i, ts_j);
                                const int pidx = pos_index(pos_i, col_pos<KIND>(s, j), p.P);
                                const int tb = time_bucket(ts_i, ts_j, p.nb);
                                const float h = fmaf(__uint_as_float(f ? s1 : s0), 0.5f, 0.5f * s_rp[pidx] + s_rth[tb]);
                                pv[f] = vis ? fmaf(h, tanh_approx(h), h) : 0.f;
                            }
                            // P pair e/2 into column e/2 of the chunk: its S values were read already
                            tmem_st1(col + (e >> 1), pack_bf16x2(pv[0], pv[1]));
                        }
                        continue;
                    }
                    const uint32_t sa = tmem + lane_base + kSCol + 32 * c;
                    const float* dg = w_diag + 31 - (KIND != HSTU_KIND_CAUSAL && pm == kPosCol ? 0 : lane) + 32 * cc;
                    const int32_t* cr = w_crel + 32 * cc;
                    if (pm == kPosUniform && tm == kTimeUniform) fwd_block2<kBiasConst>(sa, dg, cr, a_i, c0, s_rth, nbm1, pk);
                    else if (pm >= 0 && tm == kTimeUniform) fwd_block2<kBiasRow>(sa, dg, cr, a_i, c0, s_rth, nbm1, pk);
                    else if (pm >= 0 && tm == kTimeTwo)
                        fwd_block2<kBiasRowTwo>(sa, dg, cr, a_i, c0, s_rth, nbm1, pk, tc.thr, s_rth[tc.tb_lo], s_rth[tc.tb_hi]);
                    else fwd_block2<kBiasRowTime>(sa, dg, cr, a_i, c0, s_rth, nbm1, pk);
                    if ((KIND == HSTU_KIND_MTGR || KIND == HSTU_KIND_MFSEQ) && pm >= 0 && jlim - 32 * cc < 32) {
                        // keys past the block's column limit: P = 0 (bf16 pairs, key 2e in the low half)
                        const int lim = jlim - 32 * cc;
#pragma unroll
                        for (int e = 0; e < 16; e++)
                            pk[e] &= 2 * e + 1 < lim ? 0xffffffffu : (2 * e < lim ? 0x0000ffffu : 0u);
                    }
                    // P (bf16 pairs) into the chunk's own, already read, S columns: two warps
                    // share these TMEM lanes and each may only overwrite what it has read
                    tmem_st16(tmem + lane_base + kSCol + 32 * c, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars[kPFull]);
                n_done++;
            }
            if (!ok) break;
            // ---------------- epilogue
            float a_self = 0.f;
            const __nv_bfloat16* vself = nullptr;
            if (KIND == HSTU_KIND_MFALCON && row_ok) {
                const size_t ro = (size_t)(s.q0 + i) * p.ld + (size_t)s.h * D;
                const uint4* qs = reinterpret_cast<const uint4*>(p.self_q + ro);
                const uint4* ks = reinterpret_cast<const uint4*>(p.self_k + ro);
                float dot = 0.f;
#pragma unroll 4
                for (int e = 0; e < D / 8; e++) {
                    const uint4 a = qs[e], b = ks[e];
                    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
                    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
                    for (int f = 0; f < 4; f++) {
                        const float2 x = __bfloat1622float2(a2[f]), y2 = __bfloat1622float2(b2[f]);
                        dot = fmaf(x.x, y2.x, dot);
                        dot = fmaf(x.y, y2.y, dot);
                    }
                }
                a_self = silu_fast(dot + rp_self + rt_zero);
                vself = p.self_v + ro;
            }
            ok = mbar_wait(&bars[kOFull], o_use & 1, s_abort, p.dbg.limit);
            if (!__all_sync(kFull, ok)) { ok = false; break; }
            o_use++;
            tc_fence_after();
#pragma unroll 1
            for (int c = g * (D / 64); c < (g + 1) * (D / 64); c++) {   // this warp's half of the columns
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + kOCol + 32 * c, v);
                tmem_ld_wait(v);
                if (row_ok) {
                    float o[32];
#pragma unroll
                    for (int e = 0; e < 32; e++) o[e] = n_done ? __uint_as_float(v[e]) : 0.f;
                    if (KIND == HSTU_KIND_MFALCON) {
                        const uint4* vs = reinterpret_cast<const uint4*>(vself + 32 * c);
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const uint4 a = vs[e];
                            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
#pragma unroll
                            for (int f = 0; f < 4; f++) {
                                const float2 x = __bfloat1622float2(a2[f]);
                                o[8 * e + 2 * f] = fmaf(a_self, x.x, o[8 * e + 2 * f]);
                                o[8 * e + 2 * f + 1] = fmaf(a_self, x.y, o[8 * e + 2 * f + 1]);
                            }
                        }
                    }
                    uint4 w[4];
                    uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
                    for (int e = 0; e < 16; e++)
                        wp[e] = pack_bf16x2(o[2 * e] * p.inv_alpha, o[2 * e + 1] * p.inv_alpha);
                    uint4* dst = reinterpret_cast<uint4*>(p.y + (size_t)(s.q0 + i) * p.ld +
                                                          (size_t)s.h * D + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; e++) dst[e] = w[e];
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[kOEmpty]);
            mbar_arrive(&bars[kItEmpty0 + slot]);
        }
        if (!ok && lane == 0 && !*s_abort) flag_timeout(p, s_abort);
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
                       const FwdParams& p, int grid, cudaStream_t s) {
    const uint32_t smem = FwdSmem<D>::alloc(p.P);
    cudaError_t e = ensure_smem_limit((const void*)attn_fwd_tc_kernel<KIND, D>, FwdSmem<D>::alloc(kMaxPos));
    if (e != cudaSuccess) return e;
    prof_begin(kProfAttnFwdTc, s);
    attn_fwd_tc_kernel<KIND, D><<<grid, kThreads, smem, s>>>(tq, tk, tv, p);
    prof_end(kProfAttnFwdTc, s);
    return cudaGetLastError();
}

template <int KIND, int D>
int ctas_per_sm_one() {
    // Shared memory decides: each CTA holds ~110 KB (plus the 1 KB the driver
    // reserves per CTA) and 256 TMEM columns, so at most two fit on an SM.
    constexpr uint32_t smem = FwdSmem<D>::alloc(kMaxPos);
    ensure_smem_limit((const void*)attn_fwd_tc_kernel<KIND, D>, smem);
    cudaFuncSetAttribute(attn_fwd_tc_kernel<KIND, D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                         100);
    int dev = 0, per_sm = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
        return 1;
    const int n = per_sm / (int)(smem + 1024);
    return n < 1 ? 1 : (n > 2 ? 2 : n);
}

}  // namespace

cudaError_t launch_attn_fwd_tc(int kind, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const FwdParams& p, int grid, cudaStream_t s) {
#define HSTU_FWD_CASE(K, DD) \
    if (kind == K && d == DD) return launch_one<K, DD>(tq, tk, tv, p, grid, s);
    HSTU_FWD_CASE(HSTU_KIND_CAUSAL, 128)
    HSTU_FWD_CASE(HSTU_KIND_CAUSAL, 64)
    HSTU_FWD_CASE(HSTU_KIND_MTGR, 128)
    HSTU_FWD_CASE(HSTU_KIND_MTGR, 64)
    HSTU_FWD_CASE(HSTU_KIND_MFALCON, 128)
    HSTU_FWD_CASE(HSTU_KIND_MFALCON, 64)
    HSTU_FWD_CASE(HSTU_KIND_MFSEQ, 128)
    HSTU_FWD_CASE(HSTU_KIND_MFSEQ, 64)
#undef HSTU_FWD_CASE
    return cudaErrorInvalidValue;
}

int attn_fwd_tc_ctas_per_sm(int kind, int d) {
#define HSTU_OCC_CASE(K, DD) \
    if (kind == K && d == DD) return ctas_per_sm_one<K, DD>();
    HSTU_OCC_CASE(HSTU_KIND_CAUSAL, 128)
    HSTU_OCC_CASE(HSTU_KIND_CAUSAL, 64)
    HSTU_OCC_CASE(HSTU_KIND_MTGR, 128)
    HSTU_OCC_CASE(HSTU_KIND_MTGR, 64)
    HSTU_OCC_CASE(HSTU_KIND_MFALCON, 128)
    HSTU_OCC_CASE(HSTU_KIND_MFALCON, 64)
    HSTU_OCC_CASE(HSTU_KIND_MFSEQ, 128)
    HSTU_OCC_CASE(HSTU_KIND_MFSEQ, 64)
#undef HSTU_OCC_CASE
    return 1;
}

}  // namespace hstu
