// internal.h -- shared declarations of libhstu_b200 (not part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "hstu_rules.cuh"

namespace hstu {

constexpr int kTileM = 128;         // query rows per tcgen05 tile
constexpr int kTileN = 128;         // key rows per tcgen05 tile
constexpr int kMaxPos = 1024;       // largest P the kernels keep in shared memory
constexpr int kMaxTBuckets = 64;
constexpr int kSchedBins = 4096;    // distinct sort keys in the scheduler
constexpr int kMaxSeqLen = kSchedBins * kTileM - 1;

// device status word bits (inside the workspace control block)
constexpr int kStatusBounds = 1;
constexpr int kStatusTimeout = 2;

// Control block at the start of every workspace.
struct Control {
    int status;      // kStatus* bits, cleared by hstu_check_device_error
    int n_items;     // work items written by the scheduler
    int counter;     // dynamic item counter of the persistent kernels
    int valid;       // 1 when the latest scheduler run accepted the inputs
    int pad[60];
};
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bounded waits of the pipelined (TMA + tcgen05) kernels.  limit: SM cycles a
// main-loop wait may last before the kernel records kStatusTimeout and leaves
// (about a second by default; the drain waits at exit always keep the default).
// withhold_first_load (test hook, 0 in normal use): each CTA's producer withholds
// its first tile load and waits for the abort, so that the consumers' bounded
// waits run out.  Both come from hstu_debug_set_wait_fault.
struct DebugWait {
    long long limit;
    int withhold_first_load;
};
DebugWait debug_wait();

// Work item: sequence b, query rows [row0, row_end) local to the sequence, head h.
// Stored as int4 {b, row0, h, row_end}.

struct SchedParams {
    int kind, B, Tq, Tkv, H;
    const int32_t* q_off;
    const int32_t* kv_off;
    const int32_t* n_static;
    const int32_t* n_rt;
    int max_q_len, max_kv_len, b_m;
    int ascending;   // causal/MTGR tile order inside a group: 1 = first tile first (backward key tiles)
    Control* ctrl;
    int4* items;
    int* perm;       // [B]
    int* seq_base;   // [B]
    long long max_items;
};

struct FwdParams {
    const int32_t* q_off;
    const int32_t* kv_off;
    const int64_t* q_ts;
    const int64_t* kv_ts;
    const int32_t* n_static;
    const int32_t* n_rt;
    const float* rab_pos;
    const float* rab_time;
    const int4* items;
    Control* ctrl;
    __nv_bfloat16* y;
    const __nv_bfloat16* self_q;   // M-FALCON candidate q/k/v for the self term
    const __nv_bfloat16* self_k;
    const __nv_bfloat16* self_v;
    int H, P, nb, ld;
    float inv_alpha;
    DebugWait dbg;
};

// tcgen05 backward: one work item = (sequence, head, 128-key tile).
struct BwdParams {
    const int32_t* off;
    const int64_t* ts;
    const int32_t* n_static;
    const int32_t* n_rt;
    const float* rab_pos;
    const float* rab_time;
    const int4* items;
    Control* ctrl;
    float* dq_acc;            // [T, H*d] fp32, zeroed before the launch (written via tm_dq)
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* rab_part;          // [grid][2P-1 + nb] per-CTA rab gradient partial sums, zeroed
    int H, P, nb, ld;
    DebugWait dbg;
};

constexpr int kMaxBwdCtas = 1024;   // bound on the backward's persistent grid (workspace sizing)

// Generic (CUDA-core, fp32 arithmetic) attention kernels' parameters.
struct SimtParams {
    int kind, B, H, P, nb, max_len;
    const int32_t* off;
    const int64_t* ts;
    const int32_t* n_static;
    const int32_t* n_rt;
    const float* rab_pos;
    const float* rab_time;
    const void* q;
    const void* k;
    const void* v;
    const void* dy;      // backward: dL/dY
    void* y;             // forward output
    void* dq;
    void* dk;
    void* dv;
    float* d_rab_pos;
    float* d_rab_time;
    float inv_alpha;
    const Control* ctrl;   // kernels do nothing unless ctrl->valid
};

struct LnParams {
    long long T;
    int D;
    const void* y;
    const void* u;
    const float* gamma;
    const float* beta;
    float eps;
    void* o;
    float* mean;
    float* rstd;
    // backward
    const void* g;
    void* dy;
    float dy_scale;  // dY is written times this (1/(2 alpha) for the tensor-core backward)
    void* du;
    float* part;     // [n_blocks][G][2][D]
    int n_part;
    float* d_gamma;  // [G][D]
    float* d_beta;   // [G][D]
    // Group LayerNorm: gamma / beta (and their gradients) are [G][D], row t uses
    // group[t]; G <= 1 and group == nullptr is the plain LayerNorm
    const uint8_t* group;
    int G;
    int* status;     // kStatusBounds is set here for a group id >= G (the row then uses G - 1)
    int* gmask;      // [blocks] groups each grouped backward block left a partial row for
};

constexpr int kLnMaxGroups = 16;
constexpr int kGlnMaxBlocks = 148 * 16;   // grouped LayerNorm blocks (each a contiguous chunk of rows)
constexpr int kLnMaxGroupCols = 16384;   // G * D: bound on the [G][D] affine tables

// ---- dense projections (proj_gemm.cu, proj_api.cu)
enum GemmEpi { kEpiF1 = 0, kEpiF2 = 1, kEpiBf16 = 2, kEpiAddF32 = 3 };

struct GemmParams {
    int M, N, K;
    int k_splits;                       // K split over this many tiles (kEpiAddF32 only)
    const float* bias;                  // [N] or nullptr
    const __nv_bfloat16* residual;      // [M, N] or nullptr (kEpiF2)
    void* out;                          // [M, N]: bf16, or fp32 for kEpiAddF32
    __nv_bfloat16* out4[4];             // kEpiF1: U, V, Q, K, each [M, D]
    __nv_bfloat16* z;                   // kEpiF1: pre-activation [M, N] or nullptr
    int D;                              // kEpiF1: width of each output block
    int* status;                        // kStatusTimeout is OR-ed here, or nullptr
    DebugWait dbg;
};

// Output tensor maps of the epilogue: out[0..3] (kEpiF1: U, V, Q, K; otherwise out[0] only)
// and z (kEpiF1 pre-activation), each stored from 32-row boxes.
struct GemmOutMaps {
    CUtensorMap out[4];
    CUtensorMap z;
};
constexpr int kGemmStoreRows = 32;

cudaError_t launch_gemm_tc(bool a_mn, bool b_mn, int epi, const CUtensorMap& ta, const CUtensorMap& tb,
                           const GemmOutMaps& to, const GemmParams& p, int grid, cudaStream_t s);
int gemm_tiles(const GemmParams& p);
int gemm_k_steps(int K);
int gemm_box_rows(bool mn_major, bool is_b);

// [rows, cols] bf16 row-major, 128-byte swizzle, box = 64 columns x box_rows rows
bool make_tmap_bf16(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows);
// [rows, cols] fp32 row-major, 128-byte swizzle, box = 32 columns x box_rows rows
bool make_tmap_f32_sw128(CUtensorMap* m, void* base, long long rows, long long cols, int box_rows);
int device_sms();
// cudaFuncAttributeMaxDynamicSharedMemorySize of kernel fn on the current device, set
// once per (device, kernel) and thread-safe.
cudaError_t ensure_smem_limit(const void* fn, int bytes);

// ---- opt-in per-kernel timing (profile.cu)
enum ProfKind {
    kProfSchedule = 0, kProfAttnFwdTc, kProfAttnFwdSimt, kProfLnFwd, kProfLnBwd, kProfLnBwdReduce,
    kProfAttnBwdDkvSimt, kProfAttnBwdDqSimt, kProfDebugIndices, kProfAttnBwdTc, kProfDqConvert,
    kProfRabReduce, kProfCacheScan, kProfCacheCopy, kProfGemm, kProfSiluGrad, kProfColSum, kProfSlSample, kProfGather,
    kProfScaleDy, kProfKinds
};
void prof_begin(int kind, cudaStream_t s);
void prof_end(int kind, cudaStream_t s);

// ---- launchers (return cudaError_t of the launch)
cudaError_t launch_schedule(const SchedParams& p, cudaStream_t s);
cudaError_t launch_attn_fwd_tc(int kind, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const FwdParams& p, int grid, cudaStream_t s);
int attn_fwd_tc_ctas_per_sm(int kind, int d);
cudaError_t launch_attn_fwd_simt(int dtype_f32, int d, const SimtParams& p, cudaStream_t s);
cudaError_t launch_attn_bwd_simt(int dtype_f32, int d, const SimtParams& p, cudaStream_t s);
// Queries per elementwise warp and 64-query half in the tensor-core backward (16 or 32);
// it also sets the row count of the dQ reduce-add boxes.
constexpr int kBwdEwCols = 16;

// tq and tdy map Q and dY / (2 alpha) (bf16, 64-row boxes); tdq maps the fp32 dQ
// accumulator with boxes of (32 dims x kBwdEwCols rows) for d = 128 and (16 dims x kBwdEwCols
// rows) for d = 64.
cudaError_t launch_attn_bwd_tc(int kind, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& tdy, const CUtensorMap& tdq,
                               const BwdParams& p, int grid, cudaStream_t s);
cudaError_t launch_f32_to_bf16(const float* src, __nv_bfloat16* dst, long long n, cudaStream_t s);
// dst = bf16(src * scale), n a multiple of 8 (16-byte vectors)
cudaError_t launch_scale_bf16(const __nv_bfloat16* src, __nv_bfloat16* dst, float scale, long long n,
                              cudaStream_t s);
cudaError_t launch_rab_reduce(const float* part, int n_part, int P, int nb, float* d_rab_pos,
                              float* d_rab_time, cudaStream_t s);
cudaError_t launch_ln_fwd(int dtype_f32, const LnParams& p, cudaStream_t s);
cudaError_t launch_ln_bwd(int dtype_f32, const LnParams& p, cudaStream_t s);
int ln_bwd_partials(long long T);
int gln_blocks(long long T);
cudaError_t launch_debug_indices(int B, int kind, const int32_t* off, const int64_t* ts,
                                 const int32_t* ns, const int32_t* nr, int P, int nb,
                                 const int64_t* pair_off, int max_len, uint8_t* m, int16_t* pi,
                                 int8_t* tb, cudaStream_t s);

}  // namespace hstu
