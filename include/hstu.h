/*
 * hstu.h -- C ABI of libhstu_b200: jagged HSTU pointwise attention on B200 (sm_100a).
 *
 * The operation (Meta HSTU blog, section 3 "HSTU formula" and 3.1 "Pointwise
 * Attention"): for every sequence b, head h and query i of a jagged batch,
 *
 *     z_ij = q_i . k_j + rab_pos[pidx(i, j)] + rab_time[tb(i, j)]          (section 3.2)
 *     Y_i  = (1/alpha) * sum_j mask(i, j) * SiLU(z_ij) * v_j               (no row normalisation)
 *     O_pre_i = (LayerNorm(Y_i) * gamma + beta) (.) u_i                    (LayerNorm over D = H*d_v)
 *
 *   pidx(i, j) = clamp(pos(j) - pos(i), -(P-1), P-1) + (P-1)    (rab_pos has 2P-1 entries)
 *   tb(i, j)   = min(nb - 1, bit_length(|ts(i) - ts(j)|))       (rab_time has nb entries)
 *   pos(i)     = i, except candidates (MTGR, full-sequence M-FALCON), which all
 *                sit at pos = S + R
 *
 * Masks: HSTU_MASK_CAUSAL (j <= i; MTGR deep-dive section 2, "classic GR causal
 * mask") and HSTU_MASK_MTGR, the dynamic mixed mask (MTGR deep-dive section 2;
 * MTGR arXiv report section 3.1): in a row laid out as [S static | R real-time |
 * K candidates], static tokens see static tokens, a real-time token sees static
 * tokens and real-time tokens j <= i, a candidate sees itself and every
 * non-candidate whose timestamp is strictly smaller than its own.
 * hstu_mfalcon_score is the M-FALCON candidate mask over cached history K/V
 * (HSTU blog, sections 4.2-4.3): candidates see all history and themselves.
 * HSTU_MASK_MFALCON_SEQ is the same candidate mask with history and
 * candidates in one row [R history | K candidates] (HSTU blog, section 4.2:
 * one pass scores the candidates against a causal history): history tokens are
 * causal, a candidate sees every history token and itself, and all candidates
 * sit at pos = R.  It is forward only (a scoring pass).
 *
 * Conventions shared by every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller.  Host structs
 *    (hstu_dims, hstu_mask_spec, hstu_mfalcon_dims) are read before return and
 *    may be freed afterwards; the device arrays they point to must stay valid
 *    until the stream work finishes.  The library keeps no pointer after return
 *    and allocates no device memory: all scratch comes from `workspace`.
 *  - Layout: values are row-major [T, H*d] (token-major, heads concatenated),
 *    element type given by dims.dtype; seq_offsets is int32 [B+1] with
 *    seq_offsets[0] = 0, non-decreasing, seq_offsets[B] = T; timestamps are
 *    int64 [T] (seconds); rab_pos fp32 [2P-1]; rab_time fp32 [nb];
 *    ln_gamma / ln_beta fp32 [H*d_v]; ln_mean / ln_rstd fp32 [T].
 *  - All work is asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *  - Synchronous argument checks return a negative hstu_status and launch
 *    nothing.  Errors that only the device can see (offsets that are not
 *    monotone, a sequence longer than dims.max_seq_len, MTGR segment sizes that
 *    do not fit, a bounded wait that ran out) are recorded in a status word
 *    inside `workspace`; the affected launch then does no work.  Read and
 *    clear it with hstu_check_device_error().
 *  - Alignment: every tensor pointer 16-byte aligned; H*d*elem_size a multiple of 16.
 *  - Supported: dtype HSTU_BF16 with d_qk = d_v in {64, 128}; dtype HSTU_F32 with
 *    d_qk = d_v in {32, 64, 128}; P in [1, 1024]; nb in [1, 64]; H >= 1; H*d_v <= 8192
 *    (<= 4096 for HSTU_F32);
 *    max_seq_len <= 524287.
 */
#ifndef HSTU_B200_H
#define HSTU_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HSTU_API __attribute__((visibility("default")))
#else
#define HSTU_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HSTU_OK = 0,
    HSTU_ERR_INVALID_ARG = -1,   /* a pointer, size or flag failed the host check */
    HSTU_ERR_UNSUPPORTED = -2,   /* a valid request this build does not implement */
    HSTU_ERR_CUDA = -3,          /* a CUDA runtime call or launch failed */
    HSTU_ERR_DEVICE_TIMEOUT = -4,/* a bounded device wait ran out (device status word) */
    HSTU_ERR_DEVICE_BOUNDS = -5, /* offsets / lengths / segments invalid (device status word) */
    HSTU_ERR_WORKSPACE = -6      /* workspace missing or smaller than the query returned */
} hstu_status;

typedef enum { HSTU_BF16 = 0, HSTU_F32 = 1 } hstu_dtype;

typedef enum { HSTU_MASK_CAUSAL = 0, HSTU_MASK_MTGR = 1, HSTU_MASK_MFALCON_SEQ = 2 } hstu_mask_kind;

/* Mask description.  For HSTU_MASK_MTGR, n_static[b] (profile + long-term
 * tokens, seen bidirectionally) and n_realtime[b] are DEVICE int32 [B]; the
 * remaining L_b - n_static[b] - n_realtime[b] tokens of row b are candidates.
 * For HSTU_MASK_MFALCON_SEQ, n_realtime[b] is the history length of row b (the
 * rest are candidates) and n_static is ignored (may be NULL).  Both pointers
 * are ignored for HSTU_MASK_CAUSAL.  Segment sizes outside [0, L_b] set the
 * device status word (HSTU_ERR_DEVICE_BOUNDS) and the launch writes nothing. */
typedef struct {
    int32_t kind;                /* hstu_mask_kind */
    const int32_t* n_static;     /* device [B] */
    const int32_t* n_realtime;   /* device [B] */
} hstu_mask_spec;

typedef struct {
    int32_t B;            /* sequences in the jagged batch */
    int32_t T;            /* total tokens = seq_offsets[B] */
    int32_t H;            /* heads */
    int32_t d_qk;         /* per-head query/key width */
    int32_t d_v;          /* per-head value width (must equal d_qk) */
    int32_t dtype;        /* hstu_dtype of q, k, v, u, y, o_pre and the gradients */
    int32_t n_pos;        /* P: rab_pos has 2P-1 entries (256 in the workloads) */
    int32_t n_tbuckets;   /* nb: rab_time entries (64 in the workloads) */
    int32_t max_seq_len;  /* upper bound on every L_b (checked on the device) */
    float alpha;          /* Y = sum(...) / alpha; > 0 */
    float ln_eps;         /* LayerNorm epsilon (1e-5 in the workloads) */
} hstu_dims;

/* Group LayerNorm (MTGR deep-dive, section 2; MTGR arXiv report, GLN): tokens
 * from different sources (profile, behaviour, real-time, candidate) are
 * normalised per group so that each keeps its own distribution.  Reading used
 * here: mean and variance stay per token over D; group g has its own affine
 * gamma_g, beta_g, so token t gets LN(Y_t) * gamma_{group[t]} + beta_{group[t]}.
 * n_groups = 1 is the plain LayerNorm (token_group is then ignored). */
typedef struct {
    int32_t n_groups;              /* G in [1, 16]; G * H * d_v <= 16384 */
    const uint8_t* token_group;    /* DEVICE uint8 [T], values in [0, G); required when G > 1 */
} hstu_norm_spec;

/* Bytes of workspace hstu_attn_fwd (is_bwd = 0) or hstu_attn_bwd (is_bwd = 1)
 * needs for these dims and mask kind; 0 when the arguments are invalid, and 0
 * for is_bwd = 1 with HSTU_MASK_MFALCON_SEQ (no backward for that mask). */
HSTU_API size_t hstu_attn_workspace_bytes(const hstu_dims* dims, int32_t mask_kind, int32_t is_bwd);

/* Forward of one HSTU attention layer (formula above).
 * In:  q, k [T, H*d_qk]; v, u [T, H*d_v]; seq_offsets, timestamps, rab tables,
 *      mask, ln_gamma, ln_beta.
 * Out: y [T, H*d_v] (the attention output Y, saved for the backward),
 *      o_pre [T, H*d_v], ln_mean [T], ln_rstd [T].
 * Rows of y / o_pre that belong to no sequence are not written. */
HSTU_API int hstu_attn_fwd(const hstu_dims* dims, const hstu_mask_spec* mask,
                  const void* q, const void* k, const void* v, const void* u,
                  const int32_t* seq_offsets, const int64_t* timestamps,
                  const float* rab_pos, const float* rab_time,
                  const float* ln_gamma, const float* ln_beta,
                  void* y, void* o_pre, float* ln_mean, float* ln_rstd,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of hstu_attn_fwd_gln (is_bwd = 0) / hstu_attn_bwd_gln
 * (is_bwd = 1) with n_groups groups (the backward keeps LayerNorm partial sums
 * per group); 0 when the arguments are invalid.  n_groups = 1 gives the plain
 * size. */
HSTU_API size_t hstu_attn_workspace_bytes_gln(const hstu_dims* dims, int32_t mask_kind, int32_t n_groups,
                  int32_t is_bwd);

/* hstu_attn_fwd with Group LayerNorm: ln_gamma and ln_beta are fp32 [G, H*d_v]
 * (row g is group g's affine); the workspace is sized by
 * hstu_attn_workspace_bytes_gln; everything else as hstu_attn_fwd.  A token whose group id is >= G sets the device status word
 * (HSTU_ERR_DEVICE_BOUNDS through hstu_check_device_error) and is normalised
 * with group G - 1.  NULL norm: HSTU_ERR_INVALID_ARG; n_groups outside
 * [1, 16] or G > 1 without token_group: HSTU_ERR_INVALID_ARG; G * H * d_v >
 * 16384: HSTU_ERR_UNSUPPORTED. */
HSTU_API int hstu_attn_fwd_gln(const hstu_dims* dims, const hstu_mask_spec* mask,
                  const hstu_norm_spec* norm,
                  const void* q, const void* k, const void* v, const void* u,
                  const int32_t* seq_offsets, const int64_t* timestamps,
                  const float* rab_pos, const float* rab_time,
                  const float* ln_gamma, const float* ln_beta,
                  void* y, void* o_pre, float* ln_mean, float* ln_rstd,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Scratch built into the library for hstu_attn_fwd_noalloc (bytes, per device). */
#define HSTU_NOALLOC_SCRATCH_BYTES (4u << 20)

/* hstu_attn_fwd without a caller workspace.  Library plumbing only: the pages
 * describe no such call; it computes exactly what hstu_attn_fwd computes.
 *
 * For callers that must not allocate device memory on the call path, e.g. a
 * serving loop that reserves all memory at start-up and treats any later
 * allocation as an error, or a host thread without access to the framework's
 * allocator.  The work list and status word live in a static device array of
 * HSTU_NOALLOC_SCRATCH_BYTES inside the library's module; nothing is allocated.
 *  - Size limit: returns HSTU_ERR_WORKSPACE, launching nothing, when
 *    hstu_attn_workspace_bytes(dims, mask->kind, 0) exceeds
 *    HSTU_NOALLOC_SCRATCH_BYTES (4 MiB: H * (ceil(T/128) + B) below about 262000);
 *    use hstu_attn_fwd with a workspace for larger problems.
 *  - First call per device: looks up the scratch address (cudaGetSymbolAddress),
 *    which may load the library's module on that device.  Make the first call on
 *    each device before any stream capture begins.  The address is kept for the
 *    life of the process: after cudaDeviceReset (or anything else that destroys
 *    the device's primary context) this entry point must not be called again on
 *    that device in the same process.
 *  - Each call clears the scratch's control block (status word and work counter)
 *    on `stream` before the forward's launches.
 *  - One scratch per device: calls whose work can overlap on the device (other
 *    streams, other host threads without ordering between them) race on it and
 *    give undefined results.  Calls on one stream are ordered and safe.
 *  - device_status: optional DEVICE int32 (NULL to skip) that receives, on
 *    `stream`, the device status bits after the forward: 0 clean, 1 inputs out of
 *    bounds (offsets, lengths, MTGR segments), 2 a bounded wait ran out; when
 *    nonzero the outputs were not written.
 * Other arguments, layouts and return codes as hstu_attn_fwd. */
HSTU_API int hstu_attn_fwd_noalloc(const hstu_dims* dims, const hstu_mask_spec* mask,
                  const void* q, const void* k, const void* v, const void* u,
                  const int32_t* seq_offsets, const int64_t* timestamps,
                  const float* rab_pos, const float* rab_time,
                  const float* ln_gamma, const float* ln_beta,
                  void* y, void* o_pre, float* ln_mean, float* ln_rstd,
                  int32_t* device_status, void* stream);

/* Backward of hstu_attn_fwd for the upstream gradient d_o_pre [T, H*d_v].
 * The A = SiLU(z) matrix is recomputed, never stored.
 * Out: dq, dk [T, H*d_qk]; dv, du [T, H*d_v] (element type dims.dtype);
 *      d_rab_pos fp32 [2P-1], d_rab_time fp32 [nb], d_gamma, d_beta fp32 [H*d_v].
 * Every output is overwritten, not accumulated.  y, ln_mean and ln_rstd are the
 * forward's outputs for the same inputs.  HSTU_MASK_MFALCON_SEQ returns
 * HSTU_ERR_UNSUPPORTED (a scoring pass: forward only). */
HSTU_API int hstu_attn_bwd(const hstu_dims* dims, const hstu_mask_spec* mask,
                  const void* q, const void* k, const void* v, const void* u,
                  const int32_t* seq_offsets, const int64_t* timestamps,
                  const float* rab_pos, const float* rab_time,
                  const float* ln_gamma, const float* ln_beta,
                  const void* y, const float* ln_mean, const float* ln_rstd,
                  const void* d_o_pre,
                  void* dq, void* dk, void* dv, void* du,
                  float* d_rab_pos, float* d_rab_time, float* d_gamma, float* d_beta,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Attention-only backward: the gradient of the attention output Y itself in,
 * the gradients of q, k, v and the two bias tables out.  Y = (1/alpha) sum_j
 * mask(i, j) SiLU(z_ij) v_j (Meta HSTU blog, section 3 formula and 3.1; rab
 * from section 3.2) is the A(X)V(X) part of the HSTU layer; this entry point is
 * hstu_attn_bwd without its LayerNorm-times-U step, for callers that apply their
 * own normalisation after the attention (or none).  Derivatives as in
 * hstu_attn_bwd; A is recomputed, never stored.
 * In:  dy [T, H*d_v] = dL/dY (element type dims.dtype); q, k, v, offsets,
 *      timestamps, bias tables and mask as hstu_attn_fwd.
 * Out: dq, dk [T, H*d_qk], dv [T, H*d_v]; d_rab_pos fp32 [2P-1], d_rab_time fp32
 *      [nb]; all overwritten.
 * Workspace: hstu_attn_workspace_bytes(dims, mask->kind, 1).  Errors as
 * hstu_attn_bwd (dy NULL with T > 0: HSTU_ERR_INVALID_ARG). */
HSTU_API int hstu_attn_bwd_dy(const hstu_dims* dims, const hstu_mask_spec* mask,
                  const void* q, const void* k, const void* v,
                  const int32_t* seq_offsets, const int64_t* timestamps,
                  const float* rab_pos, const float* rab_time, const void* dy,
                  void* dq, void* dk, void* dv, float* d_rab_pos, float* d_rab_time,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Backward of hstu_attn_fwd_gln: ln_gamma, ln_beta, d_gamma and d_beta are fp32
 * [G, H*d_v] (d_gamma[g] and d_beta[g] sum over the tokens of group g only;
 * they are deterministic); the workspace is sized by
 * hstu_attn_workspace_bytes_gln; everything else as hstu_attn_bwd.  Argument
 * errors and bad group ids as hstu_attn_fwd_gln. */
HSTU_API int hstu_attn_bwd_gln(const hstu_dims* dims, const hstu_mask_spec* mask,
                  const hstu_norm_spec* norm,
                  const void* q, const void* k, const void* v, const void* u,
                  const int32_t* seq_offsets, const int64_t* timestamps,
                  const float* rab_pos, const float* rab_time,
                  const float* ln_gamma, const float* ln_beta,
                  const void* y, const float* ln_mean, const float* ln_rstd,
                  const void* d_o_pre,
                  void* dq, void* dk, void* dv, void* du,
                  float* d_rab_pos, float* d_rab_time, float* d_gamma, float* d_beta,
                  void* workspace, size_t workspace_bytes, void* stream);

/* M-FALCON (HSTU blog, sections 4.2-4.3): candidates scored against cached history K/V. */
typedef struct {
    int32_t B;            /* users */
    int32_t T_hist;       /* hist_offsets[B] */
    int32_t T_cand;       /* cand_offsets[B] */
    int32_t H, d_qk, d_v; /* heads and per-head widths (d_qk = d_v) */
    int32_t dtype;        /* HSTU_BF16 only */
    int32_t n_pos, n_tbuckets;
    int32_t max_hist_len; /* upper bound on every history length (device-checked) */
    int32_t max_cand_len; /* upper bound on every user's candidate count (device-checked) */
    float alpha, ln_eps;
} hstu_mfalcon_dims;

/* Workspace bytes hstu_mfalcon_score needs; 0 when the arguments are invalid. */
HSTU_API size_t hstu_mfalcon_workspace_bytes(const hstu_mfalcon_dims* dims, int32_t b_m);

/* For candidate c of user b with n = history length of b, history positions
 * 0..n-1 and every candidate at position n:
 *   Y_c = (1/alpha) [ sum_{j<n} SiLU(q_c.k_j + rab_pos[pidx(n, j)] + rab_time[tb(ts_c, ts_j)]) v_j
 *                     + SiLU(q_c.k_c + rab_pos[P-1] + rab_time[0]) v_c ]
 *   O_pre_c = (LayerNorm(Y_c) * gamma + beta) (.) u_c
 * In:  hist_k, hist_v [T_hist, H*d] with hist_offsets int32 [B+1], hist_ts int64 [T_hist];
 *      cand_q, cand_k, cand_v, cand_u [T_cand, H*d] with cand_offsets [B+1], cand_ts [T_cand].
 * b_m (> 0) is the candidate microbatch: candidates are processed in groups of b_m
 * per user; it changes the schedule only, never the results.
 * Out: y [T_cand, H*d] and o_pre [T_cand, H*d]. */
HSTU_API int hstu_mfalcon_score(const hstu_mfalcon_dims* dims,
                       const void* hist_k, const void* hist_v,
                       const int32_t* hist_offsets, const int64_t* hist_ts,
                       const void* cand_q, const void* cand_k, const void* cand_v, const void* cand_u,
                       const int32_t* cand_offsets, const int64_t* cand_ts,
                       const float* rab_pos, const float* rab_time,
                       const float* ln_gamma, const float* ln_beta, int32_t b_m,
                       void* y, void* o_pre, void* workspace, size_t workspace_bytes, void* stream);

/* KV-cache producer for hstu_mfalcon_score (HSTU blog, section 4.3 "KV caching":
 * a user's history keys and values are computed once and reused by every later
 * candidate microbatch).  Input is a full-sequence M-FALCON batch, one row
 * [R_b history ; candidates] per user (section 4.2); output is the compact
 * history layout hstu_mfalcon_score reads.
 * In:  B users; T rows; row_elems elements per row of k and v (H*d), element
 *      type dtype (HSTU_BF16 or HSTU_F32; row_elems * elem_size a multiple of
 *      16); seq_offsets int32 [B+1], timestamps int64 [T], n_history int32 [B]
 *      (R_b, the mask's n_realtime), k, v [T, row_elems]; hist_capacity = rows
 *      allocated in hist_ts / hist_k / hist_v.
 * Out: hist_offsets int32 [B+1] = exclusive prefix sums of R_b; for i < R_b,
 *      row hist_offsets[b] + i of hist_ts / hist_k / hist_v is row
 *      seq_offsets[b] + i of timestamps / k / v (exact copies).  Rows past
 *      hist_offsets[B] are not written.
 * device_status: DEVICE int32, required.  Set on `stream` to 0 on success, or
 *      to 1 when seq_offsets is not a valid jagged layout of T rows, some R_b
 *      lies outside [0, L_b], or sum(R_b) exceeds hist_capacity; then nothing
 *      else is written.
 * Returns HSTU_ERR_INVALID_ARG for negative sizes, a bad dtype, or a missing or
 * misaligned pointer (16 bytes for k, v, hist_k, hist_v; 8 for the timestamps;
 * 4 for the int32 arrays), HSTU_ERR_UNSUPPORTED for rows that are not whole
 * 16-byte vectors, each time before any launch. */
HSTU_API int hstu_mfalcon_cache_history(int32_t B, int32_t T, int32_t row_elems, int32_t dtype,
                       const int32_t* seq_offsets, const int64_t* timestamps, const int32_t* n_history,
                       const void* k, const void* v, int64_t hist_capacity,
                       int32_t* hist_offsets, int64_t* hist_ts, void* hist_k, void* hist_v,
                       int32_t* device_status, void* stream);

/* ---- The projections on either side of the attention (Meta HSTU blog, section 3
 * formula: U(X), V(X), Q(X), K(X) = Split(phi1(f1(X))), phi1 = SiLU, and
 * O(X) = f2(Norm(A(X)V(X)) (.) U(X))).  f1 and f2 are linear maps with weights
 * stored [out, in] row-major (bf16) and optional fp32 biases; activations are
 * bf16 row-major, accumulation fp32 on the tensor cores.
 * device_status (optional DEVICE int32, NULL to skip) is set to 0 on `stream`,
 * then gets bit 2 if a bounded wait in the GEMM ran out (outputs then
 * incomplete).  Argument errors return before any launch:
 * HSTU_ERR_INVALID_ARG for sizes out of range or missing / misaligned pointers
 * (16 bytes for tensors and biases, 4 for device_status), HSTU_ERR_UNSUPPORTED
 * for widths off the multiples stated below. */

/* Z = X W1^T + b1 (X [T, d_in], W1 [4D, d_in], b1 [4D] or NULL);
 * U, V, Q, K = SiLU(Z) column blocks [0, D), [D, 2D), [2D, 3D), [3D, 4D), each
 * written to its own [T, D] tensor (the attention's input layout).  z (NULL to
 * skip) receives Z [T, 4D] for the backward.  d_in a multiple of 8, D of 64. */
HSTU_API int hstu_f1_fwd(int32_t T, int32_t d_in, int32_t D, const void* x, const void* w1, const float* b1,
                  void* u, void* v, void* q, void* k, void* z, int32_t* device_status, void* stream);

/* out = O_pre W2^T + b2 (+ residual): O_pre [T, D], W2 [d_out, D], b2 [d_out] or
 * NULL, residual [T, d_out] or NULL (added when given, e.g. the layer input
 * of a residual stack), out [T, d_out].  D a multiple of 8, d_out of 32. */
HSTU_API int hstu_f2_fwd(int32_t T, int32_t D, int32_t d_out, const void* o_pre, const void* w2,
                  const float* b2, const void* residual, void* out, int32_t* device_status, void* stream);

/* Workspace bytes of hstu_f1_bwd / hstu_f2_bwd; 0 for invalid sizes. */
HSTU_API size_t hstu_f1_bwd_workspace_bytes(int32_t T, int32_t D);
HSTU_API size_t hstu_f2_bwd_workspace_bytes(int32_t T, int32_t d_out);

/* Backward of hstu_f1_fwd for the U, V, Q, K gradients du, dv, dq, dk [T, D]
 * (z = the forward's Z).  dZ = dAct * SiLU'(Z) is kept in bf16 in the
 * workspace; dx = dZ W1 (+ dx_add [T, d_in] when not NULL, e.g. the gradient
 * arriving through a residual connection) [T, d_in] (bf16); dw1 = dZ^T X [4D, d_in] and
 * db1 = column sums of the stored dZ [4D] in fp32, overwritten.  dw1 sums split-K tiles
 * with atomics (last-bit order effects); db1 is deterministic.  d_in and D
 * multiples of 32, 4D <= 8192. */
HSTU_API int hstu_f1_bwd(int32_t T, int32_t d_in, int32_t D, const void* x, const void* w1, const void* z,
                  const void* du, const void* dv, const void* dq, const void* dk, const void* dx_add,
                  void* dx, float* dw1, float* db1, void* workspace, size_t workspace_bytes,
                  int32_t* device_status, void* stream);

/* Backward of hstu_f2_fwd for d_out_grad = dL/d out [T, d_out]: d_o_pre =
 * d_out_grad W2 [T, D] (bf16); dw2 = d_out_grad^T O_pre [d_out, D] and db2
 * [d_out] in fp32, overwritten (dw2 with split-K atomics, db2 deterministic).
 * The residual's gradient is d_out_grad itself.  D and d_out multiples of 32. */
HSTU_API int hstu_f2_bwd(int32_t T, int32_t D, int32_t d_out, const void* o_pre, const void* w2,
                  const void* d_out_grad, void* d_o_pre, float* dw2, float* db2,
                  void* workspace, size_t workspace_bytes, int32_t* device_status, void* stream);

/* ---- The data step in front of the attention. */

/* Stochastic Length (HSTU blog, section 3.4: training samples variable-length
 * subsequences of long-tailed histories; alpha = 1.6 keeps about 776 = 4096^0.8
 * of 4096 events).  Reading: a sequence longer than `cap` keeps a uniform
 * random subset of cap events in their original order; shorter ones are kept
 * whole.  Event i of sequence b draws the key SplitMix64(seed, b * 2^32 + i + 1)
 * (output number b * 2^32 + i + 1 of the SplitMix64 generator started at
 * `seed`); the cap smallest keys, ties by index, are kept.
 * In:  seq_offsets DEVICE int32 [B+1] of a jagged batch of T tokens.
 * Out: out_offsets DEVICE int32 [B+1] of the sampled batch; gather_idx DEVICE
 *      int32 [out_capacity]: input token index of each output token (apply it
 *      with hstu_gather_rows to features, timestamps, ...).  Positions are
 *      re-indexed implicitly: an output token's position is its index in its
 *      output sequence.
 * device_status: DEVICE int32, required; set to 0, or 1 when seq_offsets is not
 *      a valid layout of T tokens or the output exceeds out_capacity (then
 *      nothing else is written).
 * Returns HSTU_ERR_INVALID_ARG for negative sizes, cap < 1 or a missing /
 * misaligned pointer, before any launch. */
HSTU_API int hstu_sl_sample(int32_t B, int32_t T, const int32_t* seq_offsets, int32_t cap, uint64_t seed,
                  int64_t out_capacity, int32_t* out_offsets, int32_t* gather_idx,
                  int32_t* device_status, void* stream);

/* dst row r = src row idx[r] for r < n_rows (rows of row_bytes bytes; src has
 * n_src rows; an index outside [0, n_src) gives a zero row).  16-byte rows use
 * one warp per row with 16-byte vectors. */
HSTU_API int hstu_gather_rows(int64_t n_rows, int32_t row_bytes, const void* src, int64_t n_src,
                  const int32_t* idx, void* dst, void* stream);

/* Token-balanced batches (MTGR deep-dive, section 3, contribution 3: batch sizes
 * adapt so that every GPU gets the same token count, and gradient aggregation
 * is weighted).  Sequence b, tokens [s_b, s_b + L_b) of T, goes to bin
 * floor((2 s_b + L_b) n_bins / (2 T)): bins are contiguous sequence ranges
 * [bin_seq_start[r], bin_seq_start[r+1]) (DEVICE int32 [n_bins+1]) holding
 * bin_tokens[r] tokens (int32 [n_bins]), each within one sequence length of
 * T / n_bins; bin_weight[r] (fp32 [n_bins]) = sequences in bin r / B, the
 * factor that turns per-bin mean gradients into the batch mean.  seq_offsets
 * must be a valid jagged layout (results are unspecified otherwise, reads stay
 * in bounds). */
HSTU_API int hstu_pack_balanced(int32_t B, const int32_t* seq_offsets, int32_t n_bins, int32_t* bin_seq_start,
                  int32_t* bin_tokens, float* bin_weight, void* stream);

/* Integer decisions of the fused kernels, written through the same device
 * functions they use, for exact comparison in tests.  For every sequence b and
 * pair (i, j) of it, entry pair_offsets[b] + i*L_b + j (pair_offsets: device
 * int64 [B+1], prefix sums of L_b^2) receives the mask bit, the rab_pos index
 * and the rab_time bucket.  Meant for small batches. */
HSTU_API int hstu_debug_indices(int32_t B, int32_t mask_kind, const int32_t* seq_offsets,
                       const int64_t* timestamps, const int32_t* n_static, const int32_t* n_realtime,
                       int32_t n_pos, int32_t n_tbuckets, const int64_t* pair_offsets,
                       uint8_t* mask_bits, int16_t* pos_idx, int8_t* time_bucket, void* stream);

/* Synchronizes `stream`, reads the device status word inside `workspace`,
 * clears it and returns it as an hstu_status (HSTU_OK when clean). */
HSTU_API int hstu_check_device_error(void* workspace, void* stream);

/* Static English text for a status code. */
HSTU_API const char* hstu_status_string(int status);

/* Opt-in timing of the library's own kernel launches (off by default).
 * hstu_profile_enable(1) clears the record and starts bracketing every kernel
 * launch with two CUDA events on its stream; hstu_profile_enable(0) clears and
 * stops.  hstu_profile_read() synchronizes on the recorded events and fills
 * launches[k] and total_ms[k] for kernel kinds k < n_kinds (host arrays);
 * it returns the number of kinds the library knows, or a negative status.
 * hstu_profile_kind_name(k) names kind k ("" when out of range).  Meant for
 * benchmarks: recording costs two event records per launch. */
HSTU_API int hstu_profile_enable(int32_t on);
HSTU_API int hstu_profile_read(int32_t n_kinds, int32_t* launches, double* total_ms);
HSTU_API const char* hstu_profile_kind_name(int32_t kind);

/* Test hook for the bounded waits of the pipelined kernels (the tcgen05
 * attention forward and backward, the M-FALCON scorer and the projection GEMM).
 * Not part of the pages' method: it exists so that tests can make a device wait
 * run out without a fault.  Applies to the launches that follow, in every host
 * thread, until it is called again.
 *  - wait_limit_cycles > 0: a main-loop wait gives up after that many SM cycles
 *    (the default, used when it is 0, is about one second); waits that drain a
 *    kernel's own copies and MMAs at exit keep the default.
 *  - withhold_first_load = 1: each CTA's TMA producer withholds its first tile
 *    load and waits for the abort, so the consumers' waits for that tile run
 *    out.  The kernel then records the timeout bit in the status word, drains
 *    what it issued, frees its tensor memory and returns without writing its
 *    outputs; hstu_check_device_error reports HSTU_ERR_DEVICE_TIMEOUT (the GEMM
 *    entry points set bit 2 of device_status).  The context stays usable.
 * Call hstu_debug_set_wait_fault(0, 0) to restore normal operation.  Returns
 * HSTU_ERR_INVALID_ARG for a negative limit or a flag other than 0 or 1. */
HSTU_API int hstu_debug_set_wait_fault(int64_t wait_limit_cycles, int32_t withhold_first_load);

/* Library version, e.g. "0.1.0". */
HSTU_API const char* hstu_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_B200_H */
