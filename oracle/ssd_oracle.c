/*
 * ssd_oracle.c -- plain fp64 CPU oracle for the Mamba2 SSD chunk-scan layer
 * ("combined" forward: the selective state-space scan with skip and gate).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only tests/ and bench.py's CPU-baseline leg load it.  It
 * shares no code, header or table with the CUDA path.
 *
 * The tensors and their roles are those of page
 * "flashinfer.mamba.ssd_combined_fwd" (parameter list): x [T, H, P] inputs,
 * dt [T, H] step sizes, A [H] fp32 state-transition coefficients, B and C
 * [T, G, N] input and output projections, optional D (skip, [H] or [H, P]),
 * optional z (gate, like x), optional dt_bias [H], dt_softplus, dt_limit,
 * initial states [num_seqs, H, P, N], packed varlen sequences, checkpoint
 * boundaries and final states.  The page gives no formulas; this file takes
 * the Mamba2 selective SSM that those names belong to (Dao and Gu,
 * "Transformers are SSMs", ICML 2024, the SSD layer), per sequence n and head h
 * (group g = h / (H / G)), with the state h_t in R^{P x N}:
 *
 *     dt'_t = clamp(softplus?(dt_t + dt_bias_h), lo, hi)
 *     h_t   = exp(dt'_t A_h) h_{t-1} + dt'_t x_t B_t^T        (x_t in R^P, B_t in R^N)
 *     y_t   = h_t C_t + D_h x_t
 *     y_t  *= silu(z_t)           (when z is given)
 *
 * Readings taken where the page is silent (each listed in the design notes):
 *   - dt_bias is added before softplus, and dt_limit clamps the processed step
 *     (inclusive); softplus(x) = log(1 + e^x), returning x for x > 20;
 *   - y_t reads the state after token t (inclusive scan);
 *   - the gate multiplies by z * sigmoid(z) after the skip term;
 *   - packed sequences are given by cu_seqlens (the page's seq_idx,
 *     chunk_indices and chunk_offsets are metadata derived from it);
 *   - a checkpoint boundary b is absolute and exclusive: the state after the
 *     sequence's rows before b (its initial state when b is the first row);
 *     negative boundaries or rows disable it.
 *
 * Besides the token-by-token definition this file holds the chunked form the
 * GPU kernel follows (intra-chunk quadratic part plus the carried state), so
 * that the chunk algebra is pinned against the definition on the CPU.
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t H, P, N, G;   /* heads, head dim, state dim, groups */
    int32_t dt_softplus;  /* apply softplus to dt + dt_bias */
    double dt_lo, dt_hi;  /* inclusive limits on the processed step */
    int32_t d_per_dim;    /* D is [H, P] (1) or [H] (0) */
} ssd_cfg;

static double ssd_softplus(double x) { return x > 20.0 ? x : log1p(exp(x)); }
static double ssd_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* the processed step size of one (token, head) */
double ssd_dt(const ssd_cfg* c, double dt, double bias) {
    double v = dt + bias;
    if (c->dt_softplus) v = ssd_softplus(v);
    if (v < c->dt_lo) v = c->dt_lo;
    if (v > c->dt_hi) v = c->dt_hi;
    return v;
}

int ssd_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* skip and gate of one output row y[0..P) of head h at token t */
static void ssd_finish_row(const ssd_cfg* c, int h, const double* xt, const double* D, const double* zt, double* y) {
    for (int p = 0; p < c->P; ++p) {
        double v = y[p];
        if (D) v += (c->d_per_dim ? D[(int64_t)h * c->P + p] : D[h]) * xt[p];
        if (zt) v *= zt[p] * ssd_sigmoid(zt[p]);
        y[p] = v;
    }
}

/* the checkpoint boundary of sequence n: its offset inside the sequence (row set), -1 when none
 * is asked for, -2 when the boundary is outside the sequence or the row is out of range */
static int ssd_ckpt(const int32_t* ck_idx, const int32_t* ck_row, int num_ck, const int32_t* cu, int n, int* row) {
    if (!ck_idx) return -1;
    const int b = ck_idx[n], r = ck_row[n];
    if (b < 0 || r < 0) return -1;
    if (b < cu[n] || b > cu[n + 1] || r >= num_ck) return -2;
    *row = r;
    return b - cu[n];
}

/*
 * Token-by-token scan over packed sequences (the definition above).
 *   x [T,H,P], dt [T,H], A [H], B, C [T,G,N], D (nullable), z (nullable, [T,H,P]),
 *   dt_bias (nullable, [H]), cu [Nseq+1], init (nullable, [Nseq,H,P,N]).
 * Writes y [T,H,P], final (nullable, [Nseq,H,P,N]) and, for each sequence with
 * a checkpoint, ck_states[row] ([num_ck,H,P,N]).
 * Returns 0, or 4 when a checkpoint boundary lies outside its sequence or its
 * row is out of range (that checkpoint is then skipped).
 */
int ssd_scan(const ssd_cfg* c, int T, int Nseq, const double* x, const double* dt, const double* A,
             const double* B, const double* C, const double* D, const double* z, const double* dt_bias,
             const int32_t* cu, const double* init, double* y, double* final_states, const int32_t* ck_idx,
             const int32_t* ck_row, int num_ck, double* ck_states) {
    const int H = c->H, P = c->P, N = c->N, G = c->G, hpg = H / G;
    const int64_t ss = (int64_t)P * N;
    int rc = 0;
    (void)T;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : rc)
    for (int n = 0; n < Nseq; ++n)
        for (int h = 0; h < H; ++h) {
            const int g = h / hpg;
            double* S = (double*)malloc(sizeof(double) * ss);
            if (init) memcpy(S, init + ((int64_t)n * H + h) * ss, sizeof(double) * ss);
            else memset(S, 0, sizeof(double) * ss);
            int row = 0;
            const int ck = ssd_ckpt(ck_idx, ck_row, num_ck, cu, n, &row);
            if (ck == -2) rc |= 4;
            double* ckd = ck >= 0 ? ck_states + ((int64_t)row * H + h) * ss : NULL;
            if (ck == 0) memcpy(ckd, S, sizeof(double) * ss);
            for (int t = cu[n]; t < cu[n + 1]; ++t) {
                const double d = ssd_dt(c, dt[(int64_t)t * H + h], dt_bias ? dt_bias[h] : 0.0);
                const double decay = exp(d * A[h]);
                const double* xt = x + ((int64_t)t * H + h) * P;
                const double* Bt = B + ((int64_t)t * G + g) * N;
                const double* Ct = C + ((int64_t)t * G + g) * N;
                double* yt = y + ((int64_t)t * H + h) * P;
                for (int p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int i = 0; i < N; ++i) {
                        double v = decay * S[(int64_t)p * N + i] + d * xt[p] * Bt[i];
                        S[(int64_t)p * N + i] = v;
                        acc += v * Ct[i];
                    }
                    yt[p] = acc;
                }
                ssd_finish_row(c, h, xt, D, z ? z + ((int64_t)t * H + h) * P : NULL, yt);
                if (ckd && t + 1 - cu[n] == ck) memcpy(ckd, S, sizeof(double) * ss);
            }
            if (final_states) memcpy(final_states + ((int64_t)n * H + h) * ss, S, sizeof(double) * ss);
            free(S);
        }
    return rc;
}

/*
 * The same layer in chunks of L rows (the form the GPU kernel evaluates).  In
 * a chunk starting at row t0 with processed steps d_r, gamma_r = sum_{q<=r} d_q A_h
 * (0-based rows r inside the chunk) and carried state h_in:
 *
 *     y_r   = sum_{s<=r} exp(gamma_r - gamma_s) d_s (C_r . B_s) x_s + exp(gamma_r) h_in C_r
 *     h_out = exp(gamma_last) h_in + sum_s exp(gamma_last - gamma_s) d_s x_s B_s^T
 *
 * followed by the skip and gate of each row.  No checkpoints here.
 */
int ssd_scan_chunked(const ssd_cfg* c, int T, int Nseq, int L, const double* x, const double* dt, const double* A,
                     const double* B, const double* C, const double* D, const double* z, const double* dt_bias,
                     const int32_t* cu, const double* init, double* y, double* final_states) {
    const int H = c->H, P = c->P, N = c->N, G = c->G, hpg = H / G;
    const int64_t ss = (int64_t)P * N;
    (void)T;
    if (L <= 0) return 1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int n = 0; n < Nseq; ++n)
        for (int h = 0; h < H; ++h) {
            const int g = h / hpg;
            double* S = (double*)malloc(sizeof(double) * ss);
            double* Sn = (double*)malloc(sizeof(double) * ss);
            double* gam = (double*)malloc(sizeof(double) * L);
            double* dd = (double*)malloc(sizeof(double) * L);
            if (init) memcpy(S, init + ((int64_t)n * H + h) * ss, sizeof(double) * ss);
            else memset(S, 0, sizeof(double) * ss);
            for (int t0 = cu[n]; t0 < cu[n + 1]; t0 += L) {
                const int len = cu[n + 1] - t0 < L ? cu[n + 1] - t0 : L;
                double run = 0.0;
                for (int r = 0; r < len; ++r) {
                    dd[r] = ssd_dt(c, dt[(int64_t)(t0 + r) * H + h], dt_bias ? dt_bias[h] : 0.0);
                    run += dd[r] * A[h];
                    gam[r] = run;
                }
                for (int r = 0; r < len; ++r) {
                    const double* Cr = C + ((int64_t)(t0 + r) * G + g) * N;
                    double* yr = y + ((int64_t)(t0 + r) * H + h) * P;
                    for (int p = 0; p < P; ++p) {
                        double inter = 0.0;
                        for (int i = 0; i < N; ++i) inter += S[(int64_t)p * N + i] * Cr[i];
                        yr[p] = exp(gam[r]) * inter;
                    }
                    for (int s = 0; s <= r; ++s) {
                        const double* Bs = B + ((int64_t)(t0 + s) * G + g) * N;
                        const double* xs = x + ((int64_t)(t0 + s) * H + h) * P;
                        double cb = 0.0;
                        for (int i = 0; i < N; ++i) cb += Cr[i] * Bs[i];
                        const double w = exp(gam[r] - gam[s]) * dd[s] * cb;
                        for (int p = 0; p < P; ++p) yr[p] += w * xs[p];
                    }
                }
                const double gl = gam[len - 1];
                for (int64_t e = 0; e < ss; ++e) Sn[e] = exp(gl) * S[e];
                for (int s = 0; s < len; ++s) {
                    const double* Bs = B + ((int64_t)(t0 + s) * G + g) * N;
                    const double* xs = x + ((int64_t)(t0 + s) * H + h) * P;
                    const double w = exp(gl - gam[s]) * dd[s];
                    for (int p = 0; p < P; ++p)
                        for (int i = 0; i < N; ++i) Sn[(int64_t)p * N + i] += w * xs[p] * Bs[i];
                }
                memcpy(S, Sn, sizeof(double) * ss);
                for (int r = 0; r < len; ++r)
                    ssd_finish_row(c, h, x + ((int64_t)(t0 + r) * H + h) * P, D,
                                   z ? z + ((int64_t)(t0 + r) * H + h) * P : NULL, y + ((int64_t)(t0 + r) * H + h) * P);
            }
            if (final_states) memcpy(final_states + ((int64_t)n * H + h) * ss, S, sizeof(double) * ss);
            free(S);
            free(Sn);
            free(gam);
            free(dd);
        }
    return 0;
}
