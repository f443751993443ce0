// profile.cu -- opt-in per-kernel timing of the library's own launches.
//
// When enabled, every kernel launch is bracketed by two CUDA events recorded
// on the launching stream; hstu_profile_read() sums the elapsed times per
// kernel kind.  Off by default: then prof_begin / prof_end cost one relaxed
// atomic load.
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/hstu.h"
#include "internal.h"

namespace hstu {
namespace {

struct Rec {
    int kind;
    cudaEvent_t a, b;
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;
cudaEvent_t g_open[kProfKinds];
bool g_has_open[kProfKinds];

const char* const kNames[kProfKinds] = {
    "schedule_kernel", "attn_fwd_tc_kernel", "attn_fwd_simt_kernel", "ln_fwd_kernel",
    "ln_bwd_kernel", "ln_bwd_reduce_kernel", "attn_bwd_dkv_simt_kernel", "attn_bwd_dq_simt_kernel",
    "debug_indices_kernel", "attn_bwd_tc_kernel", "dq_convert_kernel", "rab_reduce_kernel",
    "cache_scan_kernel", "cache_copy_kernel", "gemm_tc_kernel", "silu_grad_kernel", "col_sum_kernel",
    "sl_sample_kernels", "gather_rows_kernel", "scale_dy_kernel"};

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

}  // namespace

void prof_begin(int kind, cudaStream_t s) {
    if (!g_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEvent_t a = take_event();
    cudaEventRecord(a, s);
    g_open[kind] = a;
    g_has_open[kind] = true;
}

void prof_end(int kind, cudaStream_t s) {
    if (!g_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_has_open[kind]) return;
    cudaEvent_t b = take_event();
    cudaEventRecord(b, s);
    g_recs.push_back(Rec{kind, g_open[kind], b});
    g_has_open[kind] = false;
}

}  // namespace hstu

using namespace hstu;

extern "C" {

int hstu_profile_enable(int32_t on) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto& r : g_recs) {
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_recs.clear();
    for (int k = 0; k < kProfKinds; k++) g_has_open[k] = false;
    g_on.store(on != 0);
    return HSTU_OK;
}

int hstu_profile_read(int32_t n_kinds, int32_t* launches, double* total_ms) {
    if (n_kinds < 0 || (n_kinds > 0 && (!launches || !total_ms))) return HSTU_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    for (int k = 0; k < n_kinds; k++) {
        launches[k] = 0;
        total_ms[k] = 0.0;
    }
    for (auto& r : g_recs) {
        if (cudaEventSynchronize(r.b) != cudaSuccess) return HSTU_ERR_CUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return HSTU_ERR_CUDA;
        if (r.kind < n_kinds) {
            launches[r.kind] += 1;
            total_ms[r.kind] += ms;
        }
    }
    return kProfKinds;
}

const char* hstu_profile_kind_name(int32_t kind) {
    if (kind < 0 || kind >= kProfKinds) return "";
    return kNames[kind];
}

}  // extern "C"
