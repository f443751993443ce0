/*
 * hstu_oracle.c -- fp64 CPU oracle for jagged HSTU pointwise attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may call this code; the product path never does.  It
 * shares no source with the CUDA library.
 *
 * What it computes (plain definition, no blocking, no fusion):
 *
 *   HSTU layer (Meta HSTU blog, section 3, "HSTU formula"):
 *     A(X)V(X) = phi2(Q K^T + rab^{p,t}) V,   phi2 = SiLU (section 3.1: pointwise,
 *     not softmax, rows are not normalised)
 *     O = Norm(A V) (.) U        (the f2 projection is outside this path)
 *   rab^{p,t} = rab_pos[position offset] + rab_time[time bucket]  (section 3.2)
 *   Masks:
 *     causal  (MTGR deep-dive section 2: classic GR uses a causal mask)
 *     MTGR dynamic mixed mask (MTGR deep-dive section 2; MTGR report section 3.1):
 *       static tokens (profile + long-term) are seen bidirectionally,
 *       real-time tokens causally, candidates only by themselves, and a
 *       candidate sees history only with a strictly earlier timestamp.
 *     M-FALCON (HSTU blog, sections 4.2-4.3): candidates see the whole cached
 *       history and themselves, never each other.
 *     Full-sequence M-FALCON (HSTU blog, section 4.2, the single pass over
 *       [history ; candidates] before caching): history tokens causal among
 *       themselves, each candidate sees every history token and itself; no
 *       timestamp filter.
 *
 * Readings where the pages are silent (each also listed with the design notes):
 *   - alpha divides A after SiLU (Y = sum_j mask*SiLU(z)*v / alpha); no 1/sqrt(d).
 *   - position index pidx = clamp(pos(j) - pos(i), -(P-1), P-1) + (P-1), table 2P-1.
 *   - time bucket = min(nb-1, bitlen(|ts(i) - ts(j)|)), bitlen(0) = 0.
 *   - one rab table shared by all heads; the mask multiplies after SiLU.
 *   - MTGR / M-FALCON candidates all sit at position n_hist (right after the
 *     last non-candidate token).
 *   - Norm = LayerNorm over D = H*d_v, biased variance, affine gamma/beta.
 *
 * Floating point: every input value is read as float (bf16 and fp32 values
 * are exact in float) and all arithmetic is in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_CAUSAL 0
#define ORACLE_MTGR 1
#define ORACLE_MFSEQ 2      /* full-sequence M-FALCON: n_rt[b] = history length, no static part */

/* ------------------------------------------------------------------ */
/* index rules                                                         */
/* ------------------------------------------------------------------ */

/* token class inside an MTGR row: 0 static, 1 real-time, 2 candidate */
static int token_class(int64_t i, int64_t S, int64_t R) {
    if (i < S) return 0;
    if (i < S + R) return 1;
    return 2;
}

/* position used by the relative position bias */
static int64_t token_pos(int kind, int64_t i, int64_t S, int64_t R) {
    if ((kind == ORACLE_MTGR || kind == ORACLE_MFSEQ) && i >= S + R) return S + R;
    return i;
}

static int pos_index(int64_t pos_i, int64_t pos_j, int P) {
    int64_t dp = pos_j - pos_i;
    if (dp < -(int64_t)(P - 1)) dp = -(int64_t)(P - 1);
    if (dp > (int64_t)(P - 1)) dp = (int64_t)(P - 1);
    return (int)(dp + (P - 1));
}

/* number of binary digits of x (0 for x == 0) */
static int bit_length_u64(uint64_t x) {
    int n = 0;
    while (x) {
        n++;
        x >>= 1;
    }
    return n;
}

static int time_bucket(int64_t ti, int64_t tj, int nb) {
    uint64_t d = (ti >= tj) ? (uint64_t)ti - (uint64_t)tj : (uint64_t)tj - (uint64_t)ti;
    int b = bit_length_u64(d);
    return b < nb - 1 ? b : nb - 1;
}

/* ts points at the first token of the sequence */
static int visible(int kind, int64_t i, int64_t j, int64_t S, int64_t R, const int64_t* ts) {
    if (kind == ORACLE_CAUSAL) return j <= i;
    int ci = token_class(i, S, R), cj = token_class(j, S, R);
    if (ci == 0) return cj == 0;
    if (ci == 1) return cj == 0 || (cj == 1 && j <= i);
    if (j == i) return 1;
    if (kind == ORACLE_MFSEQ) return cj != 2;
    return cj != 2 && ts[j] < ts[i];
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Error model of a bf16 tensor-core implementation (off by default; used only to
 * derive tolerances).  When on, the operands that such an implementation must hold
 * in bf16 to multiply them on the tensor cores are rounded to bf16 (round to
 * nearest even): A = SiLU(z) before it multiplies V (forward) and dY (dV), and dz
 * before it multiplies K (dQ) and Q (dK).  The rab gradients keep the unrounded dz. */
static int g_bf16_operands = 0;

void hstu_oracle_set_bf16_operands(int on) { g_bf16_operands = on ? 1 : 0; }

static double round_bf16(double x) {
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) != 0x7f800000u) u += 0x7fffu + ((u >> 16) & 1u);
    u &= 0xffff0000u;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double operand(double x) { return g_bf16_operands ? round_bf16(x) : x; }

/* derivative of z * sigmoid(z) */
static double silu_grad(double z) {
    double s = 1.0 / (1.0 + exp(-z));
    return s * (1.0 + z * (1.0 - s));
}

static int64_t find_seq(const int32_t* off, int32_t B, int64_t t) {
    int64_t lo = 0, hi = B; /* off[lo] <= t < off[hi] */
    while (hi - lo > 1) {
        int64_t mid = (lo + hi) / 2;
        if (off[mid] <= t) lo = mid; else hi = mid;
    }
    /* skip empty sequences that share the same start */
    while (lo + 1 <= B && off[lo + 1] <= t) lo++;
    return lo;
}

static void seg_sizes(int kind, const int32_t* n_static, const int32_t* n_rt, int64_t b, int64_t L,
                      int64_t* S, int64_t* R) {
    if (kind == ORACLE_MTGR) {
        *S = n_static[b];
        *R = n_rt[b];
    } else if (kind == ORACLE_MFSEQ) {
        *S = 0;
        *R = n_rt[b];
    } else {
        *S = L;
        *R = 0;
    }
}

/* ------------------------------------------------------------------ */
/* debug: per-pair integer decisions                                   */
/* ------------------------------------------------------------------ */

/* For every sequence b and every (i, j) in it, write mask, pos index and time
 * bucket at pair_off[b] + i*L + j (pair_off[b] = sum of L^2 over earlier b). */
void hstu_oracle_indices(int32_t B, const int32_t* offsets, const int64_t* ts, int32_t kind,
                         const int32_t* n_static, const int32_t* n_rt, int32_t P, int32_t nb,
                         const int64_t* pair_off, uint8_t* mask, int16_t* pidx, int8_t* tb) {
    for (int64_t b = 0; b < B; b++) {
        int64_t s0 = offsets[b], L = offsets[b + 1] - offsets[b], S, R;
        seg_sizes(kind, n_static, n_rt, b, L, &S, &R);
        const int64_t* tsb = ts + s0;
        for (int64_t i = 0; i < L; i++)
            for (int64_t j = 0; j < L; j++) {
                int64_t o = pair_off[b] + i * L + j;
                mask[o] = (uint8_t)visible(kind, i, j, S, R, tsb);
                pidx[o] = (int16_t)pos_index(token_pos(kind, i, S, R), token_pos(kind, j, S, R), P);
                tb[o] = (int8_t)time_bucket(tsb[i], tsb[j], nb);
            }
    }
}

/* ------------------------------------------------------------------ */
/* attention forward                                                    */
/* ------------------------------------------------------------------ */

/* y[r, h*dv + c] = (1/alpha) * sum_j mask(i,j) SiLU(z_ij) v[j, h*dv + c]
 * for the token rows listed in rows[0..n_rows) (all T rows when rows == NULL). */
void hstu_oracle_attn_fwd(int32_t B, const int32_t* offsets, int32_t H, int32_t dqk, int32_t dv,
                          const float* q, const float* k, const float* v, const int64_t* ts,
                          const float* rab_pos, int32_t P, const float* rab_time, int32_t nb,
                          int32_t kind, const int32_t* n_static, const int32_t* n_rt, double alpha,
                          int64_t n_rows, const int64_t* rows, double* y) {
    const int64_t ldq = (int64_t)H * dqk, ldv = (int64_t)H * dv;
    const int64_t n = rows ? n_rows : (int64_t)offsets[B];
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t rh = 0; rh < n * H; rh++) {
        int64_t r = rh / H, h = rh % H;
        int64_t t = rows ? rows[r] : r;
        int64_t b = find_seq(offsets, B, t);
        int64_t s0 = offsets[b], L = offsets[b + 1] - s0, i = t - s0, S, R;
        seg_sizes(kind, n_static, n_rt, b, L, &S, &R);
        const int64_t* tsb = ts + s0;
        double* out = y + r * ldv + h * dv;
        for (int c = 0; c < dv; c++) out[c] = 0.0;
        const float* qi = q + t * ldq + h * dqk;
        for (int64_t j = 0; j < L; j++) {
            if (!visible(kind, i, j, S, R, tsb)) continue;
            const float* kj = k + (s0 + j) * ldq + h * dqk;
            double z = 0.0;
            for (int c = 0; c < dqk; c++) z += (double)qi[c] * (double)kj[c];
            z += (double)rab_pos[pos_index(token_pos(kind, i, S, R), token_pos(kind, j, S, R), P)];
            z += (double)rab_time[time_bucket(tsb[i], tsb[j], nb)];
            double a = operand(silu(z));
            const float* vj = v + (s0 + j) * ldv + h * dv;
            for (int c = 0; c < dv; c++) out[c] += a * (double)vj[c];
        }
        for (int c = 0; c < dv; c++) out[c] /= alpha;
    }
}

/* ------------------------------------------------------------------ */
/* LayerNorm(Y) (.) U                                                   */
/* ------------------------------------------------------------------ */

void hstu_oracle_ln_mul_fwd(int64_t n, int32_t D, const double* y, const float* u, const float* gamma,
                            const float* beta, double eps, double* o, double* mean, double* rstd) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        const double* yr = y + r * D;
        double mu = 0.0;
        for (int c = 0; c < D; c++) mu += yr[c];
        mu /= D;
        double var = 0.0;
        for (int c = 0; c < D; c++) var += (yr[c] - mu) * (yr[c] - mu);
        var /= D;
        double rs = 1.0 / sqrt(var + eps);
        for (int c = 0; c < D; c++) {
            double ln = (yr[c] - mu) * rs * (double)gamma[c] + (double)beta[c];
            o[r * D + c] = ln * (double)u[r * D + c];
        }
        if (mean) mean[r] = mu;
        if (rstd) rstd[r] = rs;
    }
}

/* Given g = dL/d o_pre: dy, du (per row) and dgamma, dbeta (summed over rows). */
void hstu_oracle_ln_mul_bwd(int64_t n, int32_t D, const double* y, const float* u, const float* gamma,
                            const float* beta, double eps, const float* g, double* dy, double* du,
                            double* dgamma, double* dbeta) {
    for (int c = 0; c < D; c++) {
        dgamma[c] = 0.0;
        dbeta[c] = 0.0;
    }
    double* xh = (double*)malloc(sizeof(double) * (size_t)D);
    double* gx = (double*)malloc(sizeof(double) * (size_t)D);
    for (int64_t r = 0; r < n; r++) {
        const double* yr = y + r * D;
        double mu = 0.0;
        for (int c = 0; c < D; c++) mu += yr[c];
        mu /= D;
        double var = 0.0;
        for (int c = 0; c < D; c++) var += (yr[c] - mu) * (yr[c] - mu);
        var /= D;
        double rs = 1.0 / sqrt(var + eps);
        double m1 = 0.0, m2 = 0.0;
        for (int c = 0; c < D; c++) {
            double gr = (double)g[r * D + c];
            double ur = (double)u[r * D + c];
            xh[c] = (yr[c] - mu) * rs;
            double ln = xh[c] * (double)gamma[c] + (double)beta[c];
            du[r * D + c] = gr * ln;
            double gl = gr * ur; /* gradient w.r.t. the LayerNorm output */
            dgamma[c] += gl * xh[c];
            dbeta[c] += gl;
            gx[c] = gl * (double)gamma[c];
            m1 += gx[c];
            m2 += gx[c] * xh[c];
        }
        m1 /= D;
        m2 /= D;
        for (int c = 0; c < D; c++) dy[r * D + c] = rs * (gx[c] - m1 - xh[c] * m2);
    }
    free(xh);
    free(gx);
}

/* ------------------------------------------------------------------ */
/* attention backward                                                   */
/* ------------------------------------------------------------------ */

/* Given dy = dL/dY for all T rows, write dq, dk, dv ([T, H*d]) and the rab
 * gradients d_rab_pos[2P-1], d_rab_time[nb] (summed over b, h, i, j). */
void hstu_oracle_attn_bwd(int32_t B, const int32_t* offsets, int32_t H, int32_t dqk, int32_t dv,
                          const float* q, const float* k, const float* v, const int64_t* ts,
                          const float* rab_pos, int32_t P, const float* rab_time, int32_t nb,
                          int32_t kind, const int32_t* n_static, const int32_t* n_rt, double alpha,
                          const double* dy, double* dq, double* dk, double* dvv, double* d_rab_pos,
                          double* d_rab_time) {
    const int64_t ldq = (int64_t)H * dqk, ldv = (int64_t)H * dv;
    const int64_t T = offsets[B];
    memset(dq, 0, sizeof(double) * (size_t)(T * ldq));
    memset(dk, 0, sizeof(double) * (size_t)(T * ldq));
    memset(dvv, 0, sizeof(double) * (size_t)(T * ldv));
    const int np = 2 * P - 1;
    for (int p = 0; p < np; p++) d_rab_pos[p] = 0.0;
    for (int p = 0; p < nb; p++) d_rab_time[p] = 0.0;
#pragma omp parallel
    {
        double* lp = (double*)calloc((size_t)np, sizeof(double));
        double* lt = (double*)calloc((size_t)nb, sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < (int64_t)B * H; bh++) {
            int64_t b = bh / H, h = bh % H;
            int64_t s0 = offsets[b], L = offsets[b + 1] - s0, S, R;
            seg_sizes(kind, n_static, n_rt, b, L, &S, &R);
            const int64_t* tsb = ts + s0;
            for (int64_t i = 0; i < L; i++) {
                const float* qi = q + (s0 + i) * ldq + h * dqk;
                const double* dyi = dy + (s0 + i) * ldv + h * dv;
                for (int64_t j = 0; j < L; j++) {
                    if (!visible(kind, i, j, S, R, tsb)) continue;
                    const float* kj = k + (s0 + j) * ldq + h * dqk;
                    const float* vj = v + (s0 + j) * ldv + h * dv;
                    int pi = pos_index(token_pos(kind, i, S, R), token_pos(kind, j, S, R), P);
                    int ti = time_bucket(tsb[i], tsb[j], nb);
                    double z = 0.0;
                    for (int c = 0; c < dqk; c++) z += (double)qi[c] * (double)kj[c];
                    z += (double)rab_pos[pi] + (double)rab_time[ti];
                    double dA = 0.0;
                    for (int c = 0; c < dv; c++) dA += dyi[c] * (double)vj[c];
                    dA /= alpha;
                    double dz = dA * silu_grad(z);
                    double a = operand(silu(z)) / alpha;
                    double dzo = operand(dz);
                    double* dqi = dq + (s0 + i) * ldq + h * dqk;
                    double* dkj = dk + (s0 + j) * ldq + h * dqk;
                    double* dvj = dvv + (s0 + j) * ldv + h * dv;
                    for (int c = 0; c < dqk; c++) {
                        dqi[c] += dzo * (double)kj[c];
                        dkj[c] += dzo * (double)qi[c];
                    }
                    for (int c = 0; c < dv; c++) dvj[c] += a * dyi[c];
                    lp[pi] += dz;
                    lt[ti] += dz;
                }
            }
        }
#pragma omp critical
        {
            for (int p = 0; p < np; p++) d_rab_pos[p] += lp[p];
            for (int p = 0; p < nb; p++) d_rab_time[p] += lt[p];
        }
        free(lp);
        free(lt);
    }
}

/* ------------------------------------------------------------------ */
/* M-FALCON candidate scoring over cached history K/V                   */
/* ------------------------------------------------------------------ */

/* For candidate row c of user b (n = history length of b):
 *   y_c = (1/alpha) [ sum_{j<n} SiLU(q_c.k_j + rab_pos[pidx(n, j)] + rab_time[tb(ts_c, ts_j)]) v_j
 *                     + SiLU(q_c.k_c + rab_pos[pidx(n, n)] + rab_time[tb(ts_c, ts_c)]) v_c ]
 * Candidates never see one another.  Rows listed in rows[] (all when NULL). */
void hstu_oracle_mfalcon(int32_t B, const int32_t* hist_off, const int32_t* cand_off, int32_t H,
                         int32_t dqk, int32_t dv, const float* hist_k, const float* hist_v,
                         const int64_t* hist_ts, const float* cand_q, const float* cand_k,
                         const float* cand_v, const int64_t* cand_ts, const float* rab_pos, int32_t P,
                         const float* rab_time, int32_t nb, double alpha, int64_t n_rows,
                         const int64_t* rows, double* y) {
    const int64_t ldq = (int64_t)H * dqk, ldv = (int64_t)H * dv;
    const int64_t n_all = rows ? n_rows : (int64_t)cand_off[B];
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t rh = 0; rh < n_all * H; rh++) {
        int64_t r = rh / H, h = rh % H;
        int64_t c = rows ? rows[r] : r;
        int64_t b = find_seq(cand_off, B, c);
        int64_t h0 = hist_off[b], n = hist_off[b + 1] - h0;
        const float* qc = cand_q + c * ldq + h * dqk;
        double* out = y + r * ldv + h * dv;
        for (int e = 0; e < dv; e++) out[e] = 0.0;
        for (int64_t j = 0; j <= n; j++) {
            const float* kj = (j < n) ? hist_k + (h0 + j) * ldq + h * dqk : cand_k + c * ldq + h * dqk;
            const float* vj = (j < n) ? hist_v + (h0 + j) * ldv + h * dv : cand_v + c * ldv + h * dv;
            int64_t tj = (j < n) ? hist_ts[h0 + j] : cand_ts[c];
            double z = 0.0;
            for (int e = 0; e < dqk; e++) z += (double)qc[e] * (double)kj[e];
            z += (double)rab_pos[pos_index(n, j, P)];
            z += (double)rab_time[time_bucket(cand_ts[c], tj, nb)];
            double a = operand(silu(z));
            for (int e = 0; e < dv; e++) out[e] += a * (double)vj[e];
        }
        for (int e = 0; e < dv; e++) out[e] /= alpha;
    }
}

int hstu_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void hstu_oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
