// hstu_api.cu -- the C ABI of libhstu_b200 (declared in include/hstu.h).
//
// Host side only: argument checks, workspace layout, TMA descriptors and the
// launch sequence of each entry point.  Every step of the computation runs in
// the library's own kernels.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/hstu.h"
#include "internal.h"
#include "ptx.cuh"

namespace hstu {
namespace {

// ------------------------------------------------------------------ device info
struct DevInfo {
    bool ready = false;
    int sms = 0;
    int occ[4][2] = {{0, 0}, {0, 0}, {0, 0}, {0, 0}};   // [kind][d == 128]
};
std::mutex g_mu;
DevInfo g_dev[64];

const DevInfo* dev_info() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo& d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return nullptr;
        for (int k = 0; k < 4; k++) {
            d.occ[k][0] = attn_fwd_tc_ctas_per_sm(k, 64);
            d.occ[k][1] = attn_fwd_tc_ctas_per_sm(k, 128);
        }
        d.ready = true;
    }
    return &d;
}

}  // namespace

// Test hook settings of the pipelined kernels' bounded waits (hstu_debug_set_wait_fault).
std::atomic<long long> g_wait_limit{0};
std::atomic<int> g_withhold{0};

DebugWait debug_wait() {
    DebugWait w;
    const long long l = g_wait_limit.load();
    w.limit = l > 0 ? l : ptx::kWaitLimitCycles;
    w.withhold_first_load = g_withhold.load();
    return w;
}

// The dynamic shared-memory limit is a per-device attribute of a kernel: set it once
// per (device, kernel), under a lock, the first time that kernel is launched on the
// current device.
cudaError_t ensure_smem_limit(const void* fn, int bytes) {
    struct Entry { int dev; const void* fn; int bytes; };
    static std::mutex mu;
    static Entry done[256];
    static int n_done = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < n_done; i++)
        if (done[i].dev == dev && done[i].fn == fn && done[i].bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (n_done < 256) done[n_done++] = Entry{dev, fn, bytes};
    return cudaSuccess;
}

namespace {

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [rows, cols] bf16 row-major; box = 64 columns (128 B, one swizzle row) x box_rows rows.
bool make_tmap(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows = 128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// [rows, cols] fp32 row-major, no swizzle; box = box_cols x box_rows (box_cols * 4 B a multiple of 16).
bool make_tmap_f32(CUtensorMap* m, void* base, long long rows, long long cols, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ checks
bool aligned(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elem_size(int dtype) { return dtype == HSTU_F32 ? 4 : 2; }

bool d_supported(int dtype, int d) {
    if (dtype == HSTU_BF16) return d == 64 || d == 128;
    if (dtype == HSTU_F32) return d == 32 || d == 64 || d == 128;
    return false;
}

int check_dims(const hstu_dims* d) {
    if (!d) return HSTU_ERR_INVALID_ARG;
    if (d->B < 0 || d->T < 0 || d->H < 1 || d->d_qk < 1 || d->d_v < 1) return HSTU_ERR_INVALID_ARG;
    if (d->dtype != HSTU_BF16 && d->dtype != HSTU_F32) return HSTU_ERR_INVALID_ARG;
    if (d->d_qk != d->d_v || !d_supported(d->dtype, d->d_qk)) return HSTU_ERR_UNSUPPORTED;
    if (d->n_pos < 1 || d->n_pos > kMaxPos) return HSTU_ERR_UNSUPPORTED;
    if (d->n_tbuckets < 1 || d->n_tbuckets > kMaxTBuckets) return HSTU_ERR_UNSUPPORTED;
    if (d->max_seq_len < 0 || d->max_seq_len > kMaxSeqLen) return HSTU_ERR_UNSUPPORTED;
    if (d->T > 0 && (d->max_seq_len < 1 || d->B < 1)) return HSTU_ERR_INVALID_ARG;
    if (!(d->alpha > 0.f) || !isfinite(d->alpha)) return HSTU_ERR_INVALID_ARG;
    if (!(d->ln_eps >= 0.f) || !isfinite(d->ln_eps)) return HSTU_ERR_INVALID_ARG;
    if ((long long)d->H * d->d_v > 8192) return HSTU_ERR_UNSUPPORTED;
    // LayerNorm rows are held in registers: at most 8 x 4 x 32 vectors of 8 bf16 or 4 fp32
    if (d->dtype == HSTU_F32 && (long long)d->H * d->d_v > 4096) return HSTU_ERR_UNSUPPORTED;
    return HSTU_OK;
}

int check_mask(const hstu_mask_spec* m, int* kind) {
    if (!m) return HSTU_ERR_INVALID_ARG;
    if (m->kind == HSTU_MASK_CAUSAL) {
        *kind = HSTU_KIND_CAUSAL;
        return HSTU_OK;
    }
    if (m->kind == HSTU_MASK_MTGR) {
        if (!aligned(m->n_static, 4) || !aligned(m->n_realtime, 4)) return HSTU_ERR_INVALID_ARG;
        *kind = HSTU_KIND_MTGR;
        return HSTU_OK;
    }
    if (m->kind == HSTU_MASK_MFALCON_SEQ) {
        if (!aligned(m->n_realtime, 4)) return HSTU_ERR_INVALID_ARG;
        *kind = HSTU_KIND_MFSEQ;
        return HSTU_OK;
    }
    return HSTU_ERR_INVALID_ARG;
}

// ------------------------------------------------------------------ workspace layout
struct Layout {
    size_t items = 0, perm = 0, seq_base = 0, dy = 0, part = 0, dq_acc = 0, rab_part = 0, gmask = 0, total = 0;
    long long max_items = 0;
    int n_part = 0;
};

Layout attn_layout(const hstu_dims& d, int is_bwd, int n_groups = 1) {
    Layout L;
    size_t off = sizeof(Control);
    L.max_items = (long long)d.H * (((long long)d.T + kTileM - 1) / kTileM + d.B);
    L.items = off;
    off = align_up(off + (size_t)L.max_items * sizeof(int4), 256);
    L.perm = off;
    off = align_up(off + (size_t)d.B * 4, 256);
    L.seq_base = off;
    off = align_up(off + (size_t)d.B * 4, 256);
    if (is_bwd) {
        const size_t D = (size_t)d.H * d.d_v;
        L.dy = off;
        off = align_up(off + (size_t)d.T * D * elem_size(d.dtype), 256);
        // LayerNorm partial rows: one per block, or one per (block, group) for Group LayerNorm
        L.n_part = n_groups > 1 ? gln_blocks(d.T) : ln_bwd_partials(d.T);
        L.part = off;
        off = align_up(off + (size_t)L.n_part * (n_groups > 1 ? n_groups : 1) * 2 * D * 4, 256);
        if (n_groups > 1) {
            L.gmask = off;                       // groups each grouped block holds
            off = align_up(off + (size_t)L.n_part * 4, 256);
        }
        if (d.dtype == HSTU_BF16) {
            L.dq_acc = off;                      // fp32 dQ accumulated across key tiles
            off = align_up(off + (size_t)d.T * D * 4, 256);
            L.rab_part = off;                    // per-CTA rab gradient partial sums
            off = align_up(off + (size_t)kMaxBwdCtas * (2 * d.n_pos - 1 + d.n_tbuckets) * 4, 256);
        }
    }
    L.total = off;
    return L;
}

Layout mfalcon_layout(const hstu_mfalcon_dims& d, int b_m) {
    Layout L;
    size_t off = sizeof(Control);
    const long long tc = d.T_cand;
    L.max_items = (long long)d.H * ((tc + kTileM - 1) / kTileM + (tc + b_m - 1) / b_m + d.B);
    L.items = off;
    off = align_up(off + (size_t)L.max_items * sizeof(int4), 256);
    L.perm = off;
    off = align_up(off + (size_t)d.B * 4, 256);
    L.seq_base = off;
    off = align_up(off + (size_t)d.B * 4, 256);
    L.total = off;
    return L;
}

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return HSTU_OK;
    fprintf(stderr, "libhstu_b200: CUDA error %s\n", cudaGetErrorString(e));
    return HSTU_ERR_CUDA;
}

SimtParams simt_params(const hstu_dims& d, int kind, const hstu_mask_spec& m, const int32_t* off,
                       const int64_t* ts, const float* rp, const float* rt, const void* q,
                       const void* k, const void* v, const Control* ctrl) {
    SimtParams p;
    memset(&p, 0, sizeof(p));
    p.kind = kind;
    p.B = d.B;
    p.H = d.H;
    p.P = d.n_pos;
    p.nb = d.n_tbuckets;
    p.max_len = d.max_seq_len;
    p.off = off;
    p.ts = ts;
    p.n_static = m.n_static;
    p.n_rt = m.n_realtime;
    p.rab_pos = rp;
    p.rab_time = rt;
    p.q = q;
    p.k = k;
    p.v = v;
    p.inv_alpha = 1.0f / d.alpha;
    p.ctrl = ctrl;
    return p;
}

}  // namespace
}  // namespace hstu

namespace hstu {

bool make_tmap_bf16(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows) {
    return make_tmap(m, base, rows, cols, box_rows);
}

bool make_tmap_f32_sw128(CUtensorMap* m, void* base, long long rows, long long cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int device_sms() {
    const DevInfo* di = dev_info();
    return di ? di->sms : 0;
}

}  // namespace hstu

using namespace hstu;

extern "C" {

const char* hstu_version(void) { return "0.1.0"; }

int hstu_debug_set_wait_fault(int64_t wait_limit_cycles, int32_t withhold_first_load) {
    if (wait_limit_cycles < 0 || (withhold_first_load != 0 && withhold_first_load != 1))
        return HSTU_ERR_INVALID_ARG;
    g_wait_limit.store(wait_limit_cycles);
    g_withhold.store(withhold_first_load);
    return HSTU_OK;
}

const char* hstu_status_string(int s) {
    switch (s) {
        case HSTU_OK: return "ok";
        case HSTU_ERR_INVALID_ARG: return "invalid argument";
        case HSTU_ERR_UNSUPPORTED: return "unsupported shape or type";
        case HSTU_ERR_CUDA: return "CUDA runtime error";
        case HSTU_ERR_DEVICE_TIMEOUT: return "a bounded device wait timed out";
        case HSTU_ERR_DEVICE_BOUNDS: return "offsets, lengths or segment sizes are invalid";
        case HSTU_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

size_t hstu_attn_workspace_bytes(const hstu_dims* dims, int32_t mask_kind, int32_t is_bwd) {
    if (check_dims(dims) != HSTU_OK) return 0;
    if (mask_kind != HSTU_MASK_CAUSAL && mask_kind != HSTU_MASK_MTGR && mask_kind != HSTU_MASK_MFALCON_SEQ)
        return 0;
    if (is_bwd && mask_kind == HSTU_MASK_MFALCON_SEQ) return 0;
    return attn_layout(*dims, is_bwd ? 1 : 0).total;
}

size_t hstu_attn_workspace_bytes_gln(const hstu_dims* dims, int32_t mask_kind, int32_t n_groups, int32_t is_bwd) {
    if (n_groups < 1 || n_groups > kLnMaxGroups) return 0;
    if (hstu_attn_workspace_bytes(dims, mask_kind, is_bwd) == 0) return 0;
    if ((long long)n_groups * dims->H * dims->d_v > kLnMaxGroupCols) return 0;
    return attn_layout(*dims, is_bwd ? 1 : 0, n_groups).total;
}

namespace {

// Group LayerNorm arguments: n_groups in [1, kLnMaxGroups], G * D within the backward's
// shared-memory sums, and a token_group array whenever G > 1.
int check_norm(const hstu_norm_spec* n, const hstu_dims& d, int* G, const uint8_t** group) {
    if (!n) {
        *G = 1;
        *group = nullptr;
        return HSTU_OK;
    }
    if (n->n_groups < 1 || n->n_groups > kLnMaxGroups) return HSTU_ERR_INVALID_ARG;
    if ((long long)n->n_groups * d.H * d.d_v > kLnMaxGroupCols) return HSTU_ERR_UNSUPPORTED;
    if (n->n_groups > 1 && d.T > 0 && !n->token_group) return HSTU_ERR_INVALID_ARG;
    *G = n->n_groups;
    *group = n->n_groups > 1 ? n->token_group : nullptr;
    return HSTU_OK;
}

int attn_fwd_impl(const hstu_dims* dims, const hstu_mask_spec* mask, const hstu_norm_spec* norm,
                  const void* q, const void* k, const void* v, const void* u, const int32_t* seq_offsets,
                  const int64_t* timestamps, const float* rab_pos, const float* rab_time,
                  const float* ln_gamma, const float* ln_beta, void* y, void* o_pre, float* ln_mean,
                  float* ln_rstd, void* workspace, size_t workspace_bytes, void* stream) {
    int st = check_dims(dims);
    if (st != HSTU_OK) return st;
    int G = 1;
    const uint8_t* group = nullptr;
    st = check_norm(norm, *dims, &G, &group);
    if (st != HSTU_OK) return st;
    int kind = 0;
    st = check_mask(mask, &kind);
    if (st != HSTU_OK) return st;
    const hstu_dims& d = *dims;
    const Layout L = attn_layout(d, 0, G);
    if (!aligned(workspace, 256)) return HSTU_ERR_WORKSPACE;
    if (workspace_bytes < L.total) return HSTU_ERR_WORKSPACE;
    if (d.T == 0) return HSTU_OK;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(u, 16) || !aligned(y, 16) ||
        !aligned(o_pre, 16) || !aligned(seq_offsets, 4) || !aligned(timestamps, 8) ||
        !aligned(rab_pos, 4) || !aligned(rab_time, 4) || !aligned(ln_gamma, 16) ||
        !aligned(ln_beta, 16) || !aligned(ln_mean, 4) || !aligned(ln_rstd, 4))
        return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Control* ctrl = at<Control>(workspace, 0);
    const int D = d.H * d.d_v;

    // 1. validation + work list
    SchedParams sp;
    memset(&sp, 0, sizeof(sp));
    sp.kind = kind;
    sp.B = d.B;
    sp.Tq = sp.Tkv = d.T;
    sp.H = d.H;
    sp.q_off = sp.kv_off = seq_offsets;
    sp.n_static = mask->n_static;
    sp.n_rt = mask->n_realtime;
    sp.max_q_len = sp.max_kv_len = d.max_seq_len;
    sp.b_m = 1;
    sp.ctrl = ctrl;
    sp.items = at<int4>(workspace, L.items);
    sp.perm = at<int>(workspace, L.perm);
    sp.seq_base = at<int>(workspace, L.seq_base);
    sp.max_items = L.max_items;
    st = cuda_status(launch_schedule(sp, s));
    if (st != HSTU_OK) return st;

    // 2. attention
    if (d.dtype == HSTU_BF16) {
        const DevInfo* di = dev_info();
        if (!di) return HSTU_ERR_CUDA;
        CUtensorMap tq, tk, tv;
        if (!make_tmap(&tq, q, d.T, D) || !make_tmap(&tk, k, d.T, D) || !make_tmap(&tv, v, d.T, D))
            return HSTU_ERR_CUDA;
        FwdParams fp;
        memset(&fp, 0, sizeof(fp));
        fp.dbg = debug_wait();
        fp.q_off = fp.kv_off = seq_offsets;
        fp.q_ts = fp.kv_ts = timestamps;
        fp.n_static = mask->n_static;
        fp.n_rt = mask->n_realtime;
        fp.rab_pos = rab_pos;
        fp.rab_time = rab_time;
        fp.items = sp.items;
        fp.ctrl = ctrl;
        fp.y = static_cast<__nv_bfloat16*>(y);
        fp.H = d.H;
        fp.P = d.n_pos;
        fp.nb = d.n_tbuckets;
        fp.ld = D;
        fp.inv_alpha = 1.0f / d.alpha;
        const int grid = di->sms * di->occ[kind][d.d_qk == 128 ? 1 : 0];
        st = cuda_status(launch_attn_fwd_tc(kind, d.d_qk, tq, tk, tv, fp, grid, s));
    } else {
        SimtParams p = simt_params(d, kind, *mask, seq_offsets, timestamps, rab_pos, rab_time, q, k, v,
                                   ctrl);
        p.y = y;
        st = cuda_status(launch_attn_fwd_simt(1, d.d_qk, p, s));
    }
    if (st != HSTU_OK) return st;

    // 3. LayerNorm(Y) * U
    LnParams lp;
    memset(&lp, 0, sizeof(lp));
    lp.T = d.T;
    lp.D = D;
    lp.y = y;
    lp.u = u;
    lp.gamma = ln_gamma;
    lp.beta = ln_beta;
    lp.eps = d.ln_eps;
    lp.o = o_pre;
    lp.mean = ln_mean;
    lp.rstd = ln_rstd;
    lp.G = G;
    lp.group = group;
    lp.status = &ctrl->status;
    if (G > 1) lp.n_part = gln_blocks(d.T);           // grid of the grouped forward
    return cuda_status(launch_ln_fwd(d.dtype == HSTU_F32, lp, s));
}

int attn_bwd_impl(const hstu_dims* dims, const hstu_mask_spec* mask, const hstu_norm_spec* norm,
                  const void* q, const void* k, const void* v, const void* u, const int32_t* seq_offsets,
                  const int64_t* timestamps, const float* rab_pos, const float* rab_time,
                  const float* ln_gamma, const float* ln_beta, const void* y, const float* ln_mean,
                  const float* ln_rstd, const void* d_o_pre, void* dq, void* dk, void* dv, void* du,
                  float* d_rab_pos, float* d_rab_time, float* d_gamma, float* d_beta, void* workspace,
                  size_t workspace_bytes, void* stream, const void* dy_in = nullptr) {
    // dy_in != nullptr: attention-only backward from dL/dY (no LayerNorm backward; u, ln_*,
    // y, d_o_pre, du, d_gamma and d_beta are not used)
    const bool from_dy = dy_in != nullptr;
    int st = check_dims(dims);
    if (st != HSTU_OK) return st;
    int G = 1;
    const uint8_t* group = nullptr;
    st = check_norm(norm, *dims, &G, &group);
    if (st != HSTU_OK) return st;
    int kind = 0;
    st = check_mask(mask, &kind);
    if (st != HSTU_OK) return st;
    if (kind == HSTU_KIND_MFSEQ) return HSTU_ERR_UNSUPPORTED;   // scoring pass: forward only
    const hstu_dims& d = *dims;
    const Layout L = attn_layout(d, 1, G);
    if (!aligned(workspace, 256)) return HSTU_ERR_WORKSPACE;
    if (workspace_bytes < L.total) return HSTU_ERR_WORKSPACE;
    if (!aligned(d_rab_pos, 4) || !aligned(d_rab_time, 4) ||
        (!from_dy && (!aligned(d_gamma, 4) || !aligned(d_beta, 4))))
        return HSTU_ERR_INVALID_ARG;
    // every argument is checked before the first CUDA call
    if (d.T > 0) {
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dq, 16) || !aligned(dk, 16) ||
            !aligned(dv, 16) || !aligned(seq_offsets, 4) || !aligned(timestamps, 8) || !aligned(rab_pos, 4) ||
            !aligned(rab_time, 4))
            return HSTU_ERR_INVALID_ARG;
        if (from_dy ? !aligned(dy_in, 16)
                    : (!aligned(u, 16) || !aligned(y, 16) || !aligned(d_o_pre, 16) || !aligned(du, 16) ||
                       !aligned(ln_gamma, 16) || !aligned(ln_beta, 16) || !aligned(ln_mean, 4) ||
                       !aligned(ln_rstd, 4)))
            return HSTU_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int D = d.H * d.d_v;
    cudaError_t e = cudaMemsetAsync(d_rab_pos, 0, sizeof(float) * (2 * d.n_pos - 1), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_rab_time, 0, sizeof(float) * d.n_tbuckets, s);
    if (e == cudaSuccess && d.T == 0 && !from_dy) {
        e = cudaMemsetAsync(d_gamma, 0, sizeof(float) * D * G, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(d_beta, 0, sizeof(float) * D * G, s);
    }
    if (e != cudaSuccess) return cuda_status(e);
    if (d.T == 0) return HSTU_OK;
    Control* ctrl = at<Control>(workspace, 0);

    // 1. validation + work list of (sequence, head, key tile)
    SchedParams sp;
    memset(&sp, 0, sizeof(sp));
    sp.kind = kind;
    sp.B = d.B;
    sp.Tq = sp.Tkv = d.T;
    sp.H = d.H;
    sp.q_off = sp.kv_off = seq_offsets;
    sp.n_static = mask->n_static;
    sp.n_rt = mask->n_realtime;
    sp.max_q_len = sp.max_kv_len = d.max_seq_len;
    sp.b_m = 1;
    sp.ascending = 1;        // backward items are key tiles: the first one is seen by most queries
    sp.ctrl = ctrl;
    sp.items = at<int4>(workspace, L.items);
    sp.perm = at<int>(workspace, L.perm);
    sp.seq_base = at<int>(workspace, L.seq_base);
    sp.max_items = L.max_items;
    st = cuda_status(launch_schedule(sp, s));
    if (st != HSTU_OK) return st;

    // 2. LayerNorm backward: dY (into the workspace), dU, dgamma, dbeta; or, from dL/dY,
    //    only the scaled copy of dY the tensor-core backward reads
    // the tensor-core backward takes dY / (2 alpha): its elementwise step then needs no scaling
    const float dy_scale = d.dtype == HSTU_F32 ? 1.0f : 0.5f / d.alpha;
    const void* dy_ws = at<void>(workspace, L.dy);
    if (from_dy) {
        if (d.dtype == HSTU_F32) {
            dy_ws = dy_in;                        // the CUDA-core backward reads dY as it is
        } else {
            st = cuda_status(launch_scale_bf16(static_cast<const __nv_bfloat16*>(dy_in),
                                               at<__nv_bfloat16>(workspace, L.dy), dy_scale,
                                               (long long)d.T * D, s));
            if (st != HSTU_OK) return st;
        }
    }
    LnParams lp;
    memset(&lp, 0, sizeof(lp));
    lp.T = d.T;
    lp.D = D;
    lp.y = y;
    lp.u = u;
    lp.gamma = ln_gamma;
    lp.beta = ln_beta;
    lp.eps = d.ln_eps;
    lp.mean = const_cast<float*>(ln_mean);
    lp.rstd = const_cast<float*>(ln_rstd);
    lp.g = d_o_pre;
    lp.dy = const_cast<void*>(dy_ws);
    lp.dy_scale = dy_scale;
    lp.du = du;
    lp.part = at<float>(workspace, L.part);
    lp.n_part = L.n_part;
    lp.d_gamma = d_gamma;
    lp.d_beta = d_beta;
    lp.G = G;
    lp.group = group;
    lp.status = &ctrl->status;
    if (G > 1) lp.gmask = at<int>(workspace, L.gmask);
    if (!from_dy) {
        st = cuda_status(launch_ln_bwd(d.dtype == HSTU_F32, lp, s));
        if (st != HSTU_OK) return st;
    }

    // 3. attention backward
    if (d.dtype == HSTU_F32) {
        SimtParams p = simt_params(d, kind, *mask, seq_offsets, timestamps, rab_pos, rab_time, q, k, v,
                                   ctrl);
        p.dy = lp.dy;
        p.dq = dq;
        p.dk = dk;
        p.dv = dv;
        p.d_rab_pos = d_rab_pos;
        p.d_rab_time = d_rab_time;
        return cuda_status(launch_attn_bwd_simt(1, d.d_qk, p, s));
    }
    const DevInfo* di = dev_info();
    if (!di) return HSTU_ERR_CUDA;
    CUtensorMap tq, tk, tv, tdy, tdq;
    float* dq_acc = at<float>(workspace, L.dq_acc);
    const int dq_box_cols = d.d_qk == 128 ? 32 : 16;
    if (!make_tmap(&tq, q, d.T, D, 64) || !make_tmap(&tk, k, d.T, D) || !make_tmap(&tv, v, d.T, D) ||
        !make_tmap(&tdy, lp.dy, d.T, D, 64) || !make_tmap_f32(&tdq, dq_acc, d.T, D, dq_box_cols, kBwdEwCols))
        return HSTU_ERR_CUDA;
    st = cuda_status(cudaMemsetAsync(dq_acc, 0, (size_t)d.T * D * sizeof(float), s));
    if (st != HSTU_OK) return st;
    const int grid = di->sms < kMaxBwdCtas ? di->sms : kMaxBwdCtas;
    const int rab_w = 2 * d.n_pos - 1 + d.n_tbuckets;
    float* rab_part = at<float>(workspace, L.rab_part);
    st = cuda_status(cudaMemsetAsync(rab_part, 0, (size_t)grid * rab_w * sizeof(float), s));
    if (st != HSTU_OK) return st;
    BwdParams bp;
    memset(&bp, 0, sizeof(bp));
    bp.dbg = debug_wait();
    bp.off = seq_offsets;
    bp.ts = timestamps;
    bp.n_static = mask->n_static;
    bp.n_rt = mask->n_realtime;
    bp.rab_pos = rab_pos;
    bp.rab_time = rab_time;
    bp.items = sp.items;
    bp.ctrl = ctrl;
    bp.dq_acc = dq_acc;
    bp.dk = static_cast<__nv_bfloat16*>(dk);
    bp.dv = static_cast<__nv_bfloat16*>(dv);
    bp.rab_part = rab_part;
    bp.H = d.H;
    bp.P = d.n_pos;
    bp.nb = d.n_tbuckets;
    bp.ld = D;
    st = cuda_status(launch_attn_bwd_tc(kind, d.d_qk, tq, tk, tv, tdy, tdq, bp, grid, s));
    if (st != HSTU_OK) return st;
    st = cuda_status(launch_rab_reduce(rab_part, grid, d.n_pos, d.n_tbuckets, d_rab_pos, d_rab_time, s));
    if (st != HSTU_OK) return st;
    return cuda_status(launch_f32_to_bf16(dq_acc, static_cast<__nv_bfloat16*>(dq), (long long)d.T * D, s));
}

}  // namespace

int hstu_attn_fwd(const hstu_dims* dims, const hstu_mask_spec* mask, const void* q, const void* k,
                  const void* v, const void* u, const int32_t* seq_offsets, const int64_t* timestamps,
                  const float* rab_pos, const float* rab_time, const float* ln_gamma,
                  const float* ln_beta, void* y, void* o_pre, float* ln_mean, float* ln_rstd,
                  void* workspace, size_t workspace_bytes, void* stream) {
    return attn_fwd_impl(dims, mask, nullptr, q, k, v, u, seq_offsets, timestamps, rab_pos, rab_time, ln_gamma,
                         ln_beta, y, o_pre, ln_mean, ln_rstd, workspace, workspace_bytes, stream);
}

int hstu_attn_fwd_gln(const hstu_dims* dims, const hstu_mask_spec* mask, const hstu_norm_spec* norm,
                      const void* q, const void* k, const void* v, const void* u, const int32_t* seq_offsets,
                      const int64_t* timestamps, const float* rab_pos, const float* rab_time,
                      const float* ln_gamma, const float* ln_beta, void* y, void* o_pre, float* ln_mean,
                      float* ln_rstd, void* workspace, size_t workspace_bytes, void* stream) {
    if (!norm) return HSTU_ERR_INVALID_ARG;
    return attn_fwd_impl(dims, mask, norm, q, k, v, u, seq_offsets, timestamps, rab_pos, rab_time, ln_gamma,
                         ln_beta, y, o_pre, ln_mean, ln_rstd, workspace, workspace_bytes, stream);
}

int hstu_attn_bwd(const hstu_dims* dims, const hstu_mask_spec* mask, const void* q, const void* k,
                  const void* v, const void* u, const int32_t* seq_offsets, const int64_t* timestamps,
                  const float* rab_pos, const float* rab_time, const float* ln_gamma,
                  const float* ln_beta, const void* y, const float* ln_mean, const float* ln_rstd,
                  const void* d_o_pre, void* dq, void* dk, void* dv, void* du, float* d_rab_pos,
                  float* d_rab_time, float* d_gamma, float* d_beta, void* workspace,
                  size_t workspace_bytes, void* stream) {
    return attn_bwd_impl(dims, mask, nullptr, q, k, v, u, seq_offsets, timestamps, rab_pos, rab_time, ln_gamma,
                         ln_beta, y, ln_mean, ln_rstd, d_o_pre, dq, dk, dv, du, d_rab_pos, d_rab_time, d_gamma,
                         d_beta, workspace, workspace_bytes, stream);
}

int hstu_attn_bwd_dy(const hstu_dims* dims, const hstu_mask_spec* mask, const void* q, const void* k,
                     const void* v, const int32_t* seq_offsets, const int64_t* timestamps, const float* rab_pos,
                     const float* rab_time, const void* dy, void* dq, void* dk, void* dv, float* d_rab_pos,
                     float* d_rab_time, void* workspace, size_t workspace_bytes, void* stream) {
    if (!dy && dims && dims->T > 0) return HSTU_ERR_INVALID_ARG;
    static const char kNoDy = 0;   // stands for dY when T == 0 (nothing is read)
    return attn_bwd_impl(dims, mask, nullptr, q, k, v, nullptr, seq_offsets, timestamps, rab_pos, rab_time,
                         nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dq, dk, dv, nullptr, d_rab_pos,
                         d_rab_time, nullptr, nullptr, workspace, workspace_bytes, stream, dy ? dy : &kNoDy);
}

int hstu_attn_bwd_gln(const hstu_dims* dims, const hstu_mask_spec* mask, const hstu_norm_spec* norm,
                      const void* q, const void* k, const void* v, const void* u, const int32_t* seq_offsets,
                      const int64_t* timestamps, const float* rab_pos, const float* rab_time,
                      const float* ln_gamma, const float* ln_beta, const void* y, const float* ln_mean,
                      const float* ln_rstd, const void* d_o_pre, void* dq, void* dk, void* dv, void* du,
                      float* d_rab_pos, float* d_rab_time, float* d_gamma, float* d_beta, void* workspace,
                      size_t workspace_bytes, void* stream) {
    if (!norm) return HSTU_ERR_INVALID_ARG;
    return attn_bwd_impl(dims, mask, norm, q, k, v, u, seq_offsets, timestamps, rab_pos, rab_time, ln_gamma,
                         ln_beta, y, ln_mean, ln_rstd, d_o_pre, dq, dk, dv, du, d_rab_pos, d_rab_time, d_gamma,
                         d_beta, workspace, workspace_bytes, stream);
}

size_t hstu_mfalcon_workspace_bytes(const hstu_mfalcon_dims* dims, int32_t b_m) {
    if (!dims || b_m < 1 || dims->B < 0 || dims->T_cand < 0 || dims->H < 1) return 0;
    return mfalcon_layout(*dims, b_m).total;
}

int hstu_mfalcon_score(const hstu_mfalcon_dims* dims, const void* hist_k, const void* hist_v,
                       const int32_t* hist_offsets, const int64_t* hist_ts, const void* cand_q,
                       const void* cand_k, const void* cand_v, const void* cand_u,
                       const int32_t* cand_offsets, const int64_t* cand_ts, const float* rab_pos,
                       const float* rab_time, const float* ln_gamma, const float* ln_beta,
                       int32_t b_m, void* y, void* o_pre, void* workspace, size_t workspace_bytes,
                       void* stream) {
    if (!dims) return HSTU_ERR_INVALID_ARG;
    const hstu_mfalcon_dims& d = *dims;
    if (d.B < 0 || d.T_hist < 0 || d.T_cand < 0 || d.H < 1 || b_m < 1) return HSTU_ERR_INVALID_ARG;
    if (d.dtype != HSTU_BF16) return HSTU_ERR_UNSUPPORTED;
    if (d.d_qk != d.d_v || (d.d_qk != 64 && d.d_qk != 128)) return HSTU_ERR_UNSUPPORTED;
    if (d.n_pos < 1 || d.n_pos > kMaxPos || d.n_tbuckets < 1 || d.n_tbuckets > kMaxTBuckets)
        return HSTU_ERR_UNSUPPORTED;
    if (d.max_hist_len < 0 || d.max_hist_len > kMaxSeqLen || d.max_cand_len < 0 ||
        d.max_cand_len > kMaxSeqLen)
        return HSTU_ERR_UNSUPPORTED;
    if (!(d.alpha > 0.f) || !isfinite(d.alpha) || !(d.ln_eps >= 0.f)) return HSTU_ERR_INVALID_ARG;
    if ((long long)d.H * d.d_v > 8192) return HSTU_ERR_UNSUPPORTED;
    const Layout L = mfalcon_layout(d, b_m);
    if (!aligned(workspace, 256)) return HSTU_ERR_WORKSPACE;
    if (workspace_bytes < L.total) return HSTU_ERR_WORKSPACE;
    if (d.T_cand == 0) return HSTU_OK;
    if (d.B < 1) return HSTU_ERR_INVALID_ARG;
    if (!aligned(cand_q, 16) || !aligned(cand_k, 16) || !aligned(cand_v, 16) || !aligned(cand_u, 16) ||
        !aligned(y, 16) || !aligned(o_pre, 16) || !aligned(cand_offsets, 4) ||
        !aligned(hist_offsets, 4) || !aligned(cand_ts, 8) || !aligned(rab_pos, 4) ||
        !aligned(rab_time, 4) || !aligned(ln_gamma, 16) || !aligned(ln_beta, 16))
        return HSTU_ERR_INVALID_ARG;
    if (d.T_hist > 0 && (!aligned(hist_k, 16) || !aligned(hist_v, 16) || !aligned(hist_ts, 8)))
        return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    Control* ctrl = at<Control>(workspace, 0);
    const int D = d.H * d.d_v;

    SchedParams sp;
    memset(&sp, 0, sizeof(sp));
    sp.kind = HSTU_KIND_MFALCON;
    sp.B = d.B;
    sp.Tq = d.T_cand;
    sp.Tkv = d.T_hist;
    sp.H = d.H;
    sp.q_off = cand_offsets;
    sp.kv_off = hist_offsets;
    sp.max_q_len = d.max_cand_len;
    sp.max_kv_len = d.max_hist_len;
    sp.b_m = b_m;
    sp.ctrl = ctrl;
    sp.items = at<int4>(workspace, L.items);
    sp.perm = at<int>(workspace, L.perm);
    sp.seq_base = at<int>(workspace, L.seq_base);
    sp.max_items = L.max_items;
    int st = cuda_status(launch_schedule(sp, s));
    if (st != HSTU_OK) return st;

    const DevInfo* di = dev_info();
    if (!di) return HSTU_ERR_CUDA;
    // With no history at all no key tile is ever loaded; the candidate tensors
    // then stand in as the (unused) key/value descriptors.
    const bool has_hist = d.T_hist > 0;
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, cand_q, d.T_cand, D) ||
        !make_tmap(&tk, has_hist ? hist_k : cand_k, has_hist ? d.T_hist : d.T_cand, D) ||
        !make_tmap(&tv, has_hist ? hist_v : cand_v, has_hist ? d.T_hist : d.T_cand, D))
        return HSTU_ERR_CUDA;
    FwdParams fp;
    memset(&fp, 0, sizeof(fp));
    fp.dbg = debug_wait();
    fp.q_off = cand_offsets;
    fp.kv_off = hist_offsets;
    fp.q_ts = cand_ts;
    fp.kv_ts = has_hist ? hist_ts : cand_ts;
    fp.rab_pos = rab_pos;
    fp.rab_time = rab_time;
    fp.items = sp.items;
    fp.ctrl = ctrl;
    fp.y = static_cast<__nv_bfloat16*>(y);
    fp.self_q = static_cast<const __nv_bfloat16*>(cand_q);
    fp.self_k = static_cast<const __nv_bfloat16*>(cand_k);
    fp.self_v = static_cast<const __nv_bfloat16*>(cand_v);
    fp.H = d.H;
    fp.P = d.n_pos;
    fp.nb = d.n_tbuckets;
    fp.ld = D;
    fp.inv_alpha = 1.0f / d.alpha;
    const int grid = di->sms * di->occ[HSTU_KIND_MFALCON][d.d_qk == 128 ? 1 : 0];
    st = cuda_status(launch_attn_fwd_tc(HSTU_KIND_MFALCON, d.d_qk, tq, tk, tv, fp, grid, s));
    if (st != HSTU_OK) return st;

    LnParams lp;
    memset(&lp, 0, sizeof(lp));
    lp.T = d.T_cand;
    lp.D = D;
    lp.y = y;
    lp.u = cand_u;
    lp.gamma = ln_gamma;
    lp.beta = ln_beta;
    lp.eps = d.ln_eps;
    lp.o = o_pre;
    return cuda_status(launch_ln_fwd(0, lp, s));
}

int hstu_debug_indices(int32_t B, int32_t mask_kind, const int32_t* seq_offsets,
                       const int64_t* timestamps, const int32_t* n_static, const int32_t* n_realtime,
                       int32_t n_pos, int32_t n_tbuckets, const int64_t* pair_offsets,
                       uint8_t* mask_bits, int16_t* pos_idx, int8_t* time_bucket, void* stream) {
    if (B < 0 || n_pos < 1 || n_pos > 16384 || n_tbuckets < 1 || n_tbuckets > 64)
        return HSTU_ERR_INVALID_ARG;
    if (mask_kind != HSTU_MASK_CAUSAL && mask_kind != HSTU_MASK_MTGR && mask_kind != HSTU_MASK_MFALCON_SEQ)
        return HSTU_ERR_INVALID_ARG;
    if (B == 0) return HSTU_OK;
    if (!seq_offsets || !timestamps || !pair_offsets || !mask_bits || !pos_idx || !time_bucket)
        return HSTU_ERR_INVALID_ARG;
    if (mask_kind == HSTU_MASK_MTGR && (!n_static || !n_realtime)) return HSTU_ERR_INVALID_ARG;
    if (mask_kind == HSTU_MASK_MFALCON_SEQ && !n_realtime) return HSTU_ERR_INVALID_ARG;
    const int kind = mask_kind == HSTU_MASK_MTGR ? HSTU_KIND_MTGR
                   : (mask_kind == HSTU_MASK_MFALCON_SEQ ? HSTU_KIND_MFSEQ : HSTU_KIND_CAUSAL);
    return cuda_status(launch_debug_indices(B, kind, seq_offsets, timestamps, n_static, n_realtime,
                                            n_pos, n_tbuckets, pair_offsets, 0, mask_bits, pos_idx,
                                            time_bucket, static_cast<cudaStream_t>(stream)));
}

int hstu_check_device_error(void* workspace, void* stream) {
    if (!aligned(workspace, 256)) return HSTU_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    int status = 0;
    e = cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    if (status != 0) {
        e = cudaMemset(workspace, 0, sizeof(int));
        if (e != cudaSuccess) return cuda_status(e);
    }
    if (status & kStatusTimeout) return HSTU_ERR_DEVICE_TIMEOUT;
    if (status & kStatusBounds) return HSTU_ERR_DEVICE_BOUNDS;
    return HSTU_OK;
}

}  // extern "C"
