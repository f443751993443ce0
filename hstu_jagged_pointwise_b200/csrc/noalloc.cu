// noalloc.cu -- hstu_attn_fwd_noalloc: the forward with its scratch in a static device array.
//
// Some callers cannot hand the library a workspace: a serving loop that reserves all
// device memory at start-up and treats any later allocation as a failure, or a host
// thread that has no access to the framework's caching allocator.  For them this
// entry point runs exactly the hstu_attn_fwd path with the work list and status word
// placed in a file-scope device array of HSTU_NOALLOC_SCRATCH_BYTES, part of the
// library's own module image.  Nothing here calls cudaMalloc, cudaFree or any
// allocating routine.
#include <mutex>

#include "../../include/hstu.h"
#include "internal.h"

namespace {

// One scratch area per device context; zero-initialised when the module loads.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HSTU_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's scratch, looked up on the first call per device
// (which may load the module on that device); nullptr when the lookup fails.
void* scratch_for_current_device(int* status) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        *status = HSTU_ERR_CUDA;
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        *status = HSTU_ERR_UNSUPPORTED;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            *status = HSTU_ERR_CUDA;
            return nullptr;
        }
        g_scratch_ptr[dev] = p;
    }
    *status = HSTU_OK;
    return g_scratch_ptr[dev];
}

}  // namespace

int hstu_attn_fwd_noalloc(const hstu_dims* dims, const hstu_mask_spec* mask, const void* q, const void* k,
                          const void* v, const void* u, const int32_t* seq_offsets, const int64_t* timestamps,
                          const float* rab_pos, const float* rab_time, const float* ln_gamma,
                          const float* ln_beta, void* y, void* o_pre, float* ln_mean, float* ln_rstd,
                          int32_t* device_status, void* stream) {
    if (!dims || !mask) return HSTU_ERR_INVALID_ARG;
    // hstu_attn_workspace_bytes is 0 for invalid dims or mask kind; hstu_attn_fwd then
    // returns the precise argument error without launching anything.
    const size_t need = hstu_attn_workspace_bytes(dims, mask->kind, 0);
    if (need > (size_t)HSTU_NOALLOC_SCRATCH_BYTES) return HSTU_ERR_WORKSPACE;
    int st = HSTU_OK;
    void* scratch = scratch_for_current_device(&st);
    if (!scratch) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The control block (status word, work counter) is the part that must start at
    // zero; the scratch outlives every call, so clear it each time.
    cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(hstu::Control), s);
    if (e != cudaSuccess) return HSTU_ERR_CUDA;
    st = hstu_attn_fwd(dims, mask, q, k, v, u, seq_offsets, timestamps, rab_pos, rab_time, ln_gamma,
                       ln_beta, y, o_pre, ln_mean, ln_rstd, scratch, HSTU_NOALLOC_SCRATCH_BYTES, stream);
    if (st != HSTU_OK || !device_status) return st;
    e = cudaMemcpyAsync(device_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}
