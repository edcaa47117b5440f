/*
 * gdn_oracle.c -- plain fp64 CPU oracle for the Gated DeltaNet (GDN) layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only tests/, the smoke check and bench.py's CPU-baseline
 * leg load it.  It shares no code, header or table with the CUDA path.
 *
 * What it computes (the layer a hybrid full-attention + GDN model reaches
 * through HybridAttnBackend.forward_gdn(layer, forward_batch, mixed_qkv, a, b),
 * page "pymllm.layers.attention.hybrid_backend", class HybridAttnBackend):
 *
 *   1. causal depthwise conv1d of width K over the packed rows of mixed_qkv,
 *      the window reaching back into the request's conv-state slot, then SiLU;
 *   2. split of the channels into q [HK,dk] | k [HK,dk] | v [HV,dv];
 *   3. L2 normalisation of q and k per head: x / sqrt(sum x^2 + eps);
 *   4. gates g = -exp(A_log[h]) * softplus(a + dt_bias[h]),
 *      beta = sigmoid(b), one pair per value head;
 *   5. the gated delta rule of Gated DeltaNet (Yang, Kautz, Hatamizadeh,
 *      "Gated Delta Networks: Improving Mamba2 with Delta Rule", ICLR 2025):
 *         S_t = exp(g_t) (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *         o_t = scale * S_t^T q_t
 *      with S in R^{dk x dv}; value head h reads qk head h / (HV/HK) (GQA
 *      grouping as in page "pymllm.layers.attention.radix_attention",
 *      RadixAttention parameter num_kv_heads).  scale defaults to 1/sqrt(dk)
 *      (same page, parameter `scaling`, "typically 1 / sqrt(head_dim)").
 *
 * Readings taken where the pages are silent (each listed in the design notes):
 *   - channel order [q | k | v], head-major, dim-minor inside each block;
 *   - conv is a cross-correlation: w[c, K-1] multiplies the current row;
 *     SiLU on every channel; optional bias;
 *   - conv state = the K-1 most recent raw (pre-conv) rows, index 0 oldest;
 *   - softplus(x) = log(1 + e^x), returning x for x > 20;
 *   - state_indices < 0 marks a padded request: its output rows are zero and
 *     no slot is touched; has_initial_state == 0 reads the slot as zeros;
 *   - verify runs D tokens from the slot, records the state after every token
 *     and leaves both pools untouched (the speculative Mamba-state buffer of
 *     the target-verify path on page "SGLang GDN hybrid linear attention test
 *     matrix", section on verification conventions).
 *
 * Step 5 is evaluated in the order
 *      S <- exp(g) S ;  u = beta (v - S^T k) ;  S <- S + k u^T ;  o = scale S^T q
 * which is the defining update expanded (exp(g)(I - b k k^T) S + b k v^T =
 * exp(g) S + k * b (v - exp(g) S^T k)^T).
 *
 * Besides the token-by-token definition this file holds two independent
 * evaluations used to pin it: the chunked WY/UT form (the algebra the GPU
 * prefill follows) and the explicit product form with dk x dk matrices.
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t HK, HV, dk, dv, K; /* qk heads, value heads, head dims, conv width */
    double scale;              /* <= 0: 1/sqrt(dk) */
    double eps;                /* L2-norm epsilon */
} ora_cfg;

static double ora_softplus(double x) { return x > 20.0 ? x : log1p(exp(x)); }
static double ora_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
static double ora_silu(double x) { return x / (1.0 + exp(-x)); }
static double ora_scale(const ora_cfg* c) { return c->scale > 0 ? c->scale : 1.0 / sqrt((double)c->dk); }
static int64_t ora_conv_dim(const ora_cfg* c) { return 2LL * c->HK * c->dk + (int64_t)c->HV * c->dv; }

/* ---------------------------------------------------------------------- */
/* Single steps, exported so that each can be pinned on its own.            */
/* ---------------------------------------------------------------------- */

double ora_gate_g(double A_log, double a, double dt_bias) { return -exp(A_log) * ora_softplus(a + dt_bias); }
double ora_gate_beta(double b) { return ora_sigmoid(b); }
double ora_softplus_exported(double x) { return ora_softplus(x); }

/* number of OpenMP threads the layer functions use (1 without OpenMP) */
int ora_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* x <- x / sqrt(sum x^2 + eps) over n entries */
void ora_l2norm(double* x, int n, double eps) {
    double ss = 0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < n; ++i) x[i] *= inv;
}

/*
 * Causal depthwise conv + SiLU over one sequence for `nch` channels.
 * x:      [L, ldx] raw rows (channel ch at column ch)
 * hist:   [nch, K-1] the K-1 rows before the sequence, oldest first (nullable = zeros)
 * w:      [nch, K]; bias nullable
 * y:      [L, nch]
 */
void ora_conv_silu(int L, int nch, int K, const double* x, int64_t ldx, const double* hist,
                   const double* w, const double* bias, double* y) {
    for (int t = 0; t < L; ++t)
        for (int c = 0; c < nch; ++c) {
            double acc = bias ? bias[c] : 0.0;
            for (int j = 0; j < K; ++j) {
                int src = t - (K - 1) + j; /* row index relative to sequence start */
                double xv;
                if (src >= 0) xv = x[(int64_t)src * ldx + c];
                else xv = hist ? hist[(int64_t)c * (K - 1) + (K - 1 + src)] : 0.0;
                acc += w[(int64_t)c * K + j] * xv;
            }
            y[(int64_t)t * nch + c] = ora_silu(acc);
        }
}

/*
 * The gated delta rule for one (sequence, value head), token by token.
 * q,k: [L, dk] (already normalised), v: [L, dv], g, beta: [L]
 * S: [dk, dv] in/out.  o: [L, dv].  states (nullable): [L, dk, dv], S after each token.
 */
void ora_core_recurrent(int L, int dk, int dv, const double* q, const double* k, const double* v,
                        const double* g, const double* beta, double scale, double* S, double* o,
                        double* states) {
    double* u = (double*)malloc(sizeof(double) * dv);
    for (int t = 0; t < L; ++t) {
        const double* qt = q + (int64_t)t * dk;
        const double* kt = k + (int64_t)t * dk;
        const double* vt = v + (int64_t)t * dv;
        double decay = exp(g[t]);
        for (int i = 0; i < dk * dv; ++i) S[i] *= decay;
        for (int j = 0; j < dv; ++j) {
            double kS = 0;
            for (int i = 0; i < dk; ++i) kS += kt[i] * S[(int64_t)i * dv + j];
            u[j] = beta[t] * (vt[j] - kS);
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(int64_t)i * dv + j] += kt[i] * u[j];
        for (int j = 0; j < dv; ++j) {
            double acc = 0;
            for (int i = 0; i < dk; ++i) acc += qt[i] * S[(int64_t)i * dv + j];
            o[(int64_t)t * dv + j] = scale * acc;
        }
        if (states) memcpy(states + (int64_t)t * dk * dv, S, sizeof(double) * dk * dv);
    }
    free(u);
}

/*
 * Explicit product form for small L: builds the dk x dk transition matrices
 *   A_t = exp(g_t) (I - beta_t k_t k_t^T)
 * and evaluates S_t = A_t S_{t-1} + beta_t k_t v_t^T directly (no u-form), so
 * that it shares no algebraic rearrangement with ora_core_recurrent.
 * The final state is also returned as the closed sum
 *   S_L = (A_L...A_1) S_0 + sum_t (A_L...A_{t+1}) beta_t k_t v_t^T
 * in S_sum (both are written; a pin compares them with each other and with the
 * recurrent evaluation).
 */
void ora_core_bruteforce(int L, int dk, int dv, const double* q, const double* k, const double* v,
                         const double* g, const double* beta, double scale, const double* S0,
                         double* S_step, double* S_sum, double* o) {
    int64_t mm = (int64_t)dk * dk, ms = (int64_t)dk * dv;
    double* A = (double*)malloc(sizeof(double) * mm * (L > 0 ? L : 1));
    double* tmp = (double*)malloc(sizeof(double) * ms);
    for (int t = 0; t < L; ++t) {
        double e = exp(g[t]);
        for (int r = 0; r < dk; ++r)
            for (int c = 0; c < dk; ++c)
                A[t * mm + (int64_t)r * dk + c] =
                    e * ((r == c ? 1.0 : 0.0) - beta[t] * k[(int64_t)t * dk + r] * k[(int64_t)t * dk + c]);
    }
    /* stepwise */
    memcpy(S_step, S0, sizeof(double) * ms);
    for (int t = 0; t < L; ++t) {
        for (int r = 0; r < dk; ++r)
            for (int j = 0; j < dv; ++j) {
                double acc = 0;
                for (int c = 0; c < dk; ++c) acc += A[t * mm + (int64_t)r * dk + c] * S_step[(int64_t)c * dv + j];
                tmp[(int64_t)r * dv + j] = acc + beta[t] * k[(int64_t)t * dk + r] * v[(int64_t)t * dv + j];
            }
        memcpy(S_step, tmp, sizeof(double) * ms);
        for (int j = 0; j < dv; ++j) {
            double acc = 0;
            for (int r = 0; r < dk; ++r) acc += q[(int64_t)t * dk + r] * S_step[(int64_t)r * dv + j];
            o[(int64_t)t * dv + j] = scale * acc;
        }
    }
    /* closed sum: P runs over suffix products, built from the last token backwards */
    double* P = (double*)malloc(sizeof(double) * mm);
    double* P2 = (double*)malloc(sizeof(double) * mm);
    for (int r = 0; r < dk; ++r)
        for (int c = 0; c < dk; ++c) P[(int64_t)r * dk + c] = (r == c);
    memset(S_sum, 0, sizeof(double) * ms);
    for (int t = L - 1; t >= 0; --t) {
        /* term t: P * beta_t k_t v_t^T, P = A_L ... A_{t+1} */
        for (int r = 0; r < dk; ++r) {
            double pk = 0;
            for (int c = 0; c < dk; ++c) pk += P[(int64_t)r * dk + c] * k[(int64_t)t * dk + c];
            for (int j = 0; j < dv; ++j) S_sum[(int64_t)r * dv + j] += beta[t] * pk * v[(int64_t)t * dv + j];
        }
        /* P <- P * A_t */
        for (int r = 0; r < dk; ++r)
            for (int c = 0; c < dk; ++c) {
                double acc = 0;
                for (int m = 0; m < dk; ++m) acc += P[(int64_t)r * dk + m] * A[t * mm + (int64_t)m * dk + c];
                P2[(int64_t)r * dk + c] = acc;
            }
        memcpy(P, P2, sizeof(double) * mm);
    }
    for (int r = 0; r < dk; ++r)
        for (int j = 0; j < dv; ++j) {
            double acc = 0;
            for (int c = 0; c < dk; ++c) acc += P[(int64_t)r * dk + c] * S0[(int64_t)c * dv + j];
            S_sum[(int64_t)r * dv + j] += acc;
        }
    free(A); free(tmp); free(P); free(P2);
}

/*
 * Chunked WY / UT-transform evaluation for one (sequence, value head), chunk
 * size C.  Inside a chunk of length n with state S0 at its start and
 * gamma_r = sum_{s<=r} g_s:
 *   A[r,s] = beta_r exp(gamma_r - gamma_s) k_r.k_s   (s < r), zero otherwise
 *   T      = (I + A)^{-1}
 *   W      = T diag(beta exp(gamma)) K,   U~ = T diag(beta) V
 *   V'     = U~ - W S0                      (the per-token pseudo-values u_r)
 *   o_r    = scale (exp(gamma_r) q_r^T S0 + sum_{s<=r} exp(gamma_r-gamma_s) (q_r.k_s) V'_s)
 *   S_end  = exp(gamma_n) S0 + sum_s exp(gamma_n - gamma_s) k_s V'_s^T
 * T is formed by forward substitution on the unit lower-triangular I + A.
 */
void ora_core_chunked(int L, int dk, int dv, const double* q, const double* k, const double* v,
                      const double* g, const double* beta, double scale, int C, double* S, double* o) {
    double* gam = (double*)malloc(sizeof(double) * C);
    double* A = (double*)malloc(sizeof(double) * C * C);
    double* Tm = (double*)malloc(sizeof(double) * C * C);
    double* W = (double*)malloc(sizeof(double) * C * dk);
    double* U = (double*)malloc(sizeof(double) * C * dv);
    double* Vn = (double*)malloc(sizeof(double) * C * dv);
    double* Sn = (double*)malloc(sizeof(double) * dk * dv);
    for (int c0 = 0; c0 < L; c0 += C) {
        int n = L - c0 < C ? L - c0 : C;
        const double* Q = q + (int64_t)c0 * dk;
        const double* Kc = k + (int64_t)c0 * dk;
        const double* V = v + (int64_t)c0 * dv;
        const double* bb = beta + c0;
        double run = 0;
        for (int r = 0; r < n; ++r) { run += g[c0 + r]; gam[r] = run; }
        for (int r = 0; r < n; ++r)
            for (int s = 0; s < n; ++s) {
                double val = 0;
                if (s < r) {
                    double kk = 0;
                    for (int i = 0; i < dk; ++i) kk += Kc[(int64_t)r * dk + i] * Kc[(int64_t)s * dk + i];
                    val = bb[r] * exp(gam[r] - gam[s]) * kk;
                }
                A[r * C + s] = val;
            }
        /* T = (I + A)^{-1}: row r of T solves T[r,:] + sum_{s<r} A[r,s] T[s,:] = e_r */
        for (int r = 0; r < n; ++r)
            for (int c = 0; c < n; ++c) {
                double val = (r == c) ? 1.0 : 0.0;
                for (int s = 0; s < r; ++s) val -= A[r * C + s] * Tm[s * C + c];
                Tm[r * C + c] = val;
            }
        for (int r = 0; r < n; ++r) {
            for (int i = 0; i < dk; ++i) {
                double acc = 0;
                for (int s = 0; s < n; ++s) acc += Tm[r * C + s] * bb[s] * exp(gam[s]) * Kc[(int64_t)s * dk + i];
                W[(int64_t)r * dk + i] = acc;
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0;
                for (int s = 0; s < n; ++s) acc += Tm[r * C + s] * bb[s] * V[(int64_t)s * dv + j];
                U[(int64_t)r * dv + j] = acc;
            }
        }
        for (int r = 0; r < n; ++r)
            for (int j = 0; j < dv; ++j) {
                double acc = 0;
                for (int i = 0; i < dk; ++i) acc += W[(int64_t)r * dk + i] * S[(int64_t)i * dv + j];
                Vn[(int64_t)r * dv + j] = U[(int64_t)r * dv + j] - acc;
            }
        for (int r = 0; r < n; ++r)
            for (int j = 0; j < dv; ++j) {
                double inter = 0;
                for (int i = 0; i < dk; ++i) inter += Q[(int64_t)r * dk + i] * S[(int64_t)i * dv + j];
                double intra = 0;
                for (int s = 0; s <= r; ++s) {
                    double qk = 0;
                    for (int i = 0; i < dk; ++i) qk += Q[(int64_t)r * dk + i] * Kc[(int64_t)s * dk + i];
                    intra += exp(gam[r] - gam[s]) * qk * Vn[(int64_t)s * dv + j];
                }
                o[(int64_t)(c0 + r) * dv + j] = scale * (exp(gam[r]) * inter + intra);
            }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double acc = exp(gam[n - 1]) * S[(int64_t)i * dv + j];
                for (int s = 0; s < n; ++s)
                    acc += exp(gam[n - 1] - gam[s]) * Kc[(int64_t)s * dk + i] * Vn[(int64_t)s * dv + j];
                Sn[(int64_t)i * dv + j] = acc;
            }
        memcpy(S, Sn, sizeof(double) * dk * dv);
    }
    free(gam); free(A); free(Tm); free(W); free(U); free(Vn); free(Sn);
}

/* ---------------------------------------------------------------------- */
/* The layer over a packed batch.                                          */
/* ---------------------------------------------------------------------- */

/*
 * Per (sequence, value head): run conv+SiLU on the head's q, k and v channels,
 * normalise, form gates and apply the core.  `chunk` <= 0 selects the
 * token-by-token core, > 0 the chunked form with that chunk size.
 * `head_mask` (nullable, [HV]) restricts the work to heads with a nonzero
 * entry; outputs of masked-off heads are left as they were, and so is their
 * state.  Conv state is updated for all channels after every head ran.
 */
static int ora_layer(const ora_cfg* cfg, const double* A_log, const double* dt_bias, const double* conv_w,
                     const double* conv_b, const double* x, const double* a, const double* b,
                     const int32_t* cu, int N, const int32_t* slots, const int32_t* has_init,
                     double* conv_state, double* ssm_state, int P, double* out, int chunk,
                     const int32_t* head_mask, double* states_per_token /* [T,HV,dk,dv] nullable */) {
    const int HK = cfg->HK, HV = cfg->HV, dk = cfg->dk, dv = cfg->dv, K = cfg->K;
    if (HK <= 0 || HV <= 0 || HV % HK != 0 || dk <= 0 || dv <= 0 || K < 1) return 1;
    const int G = HV / HK;
    const int64_t CD = ora_conv_dim(cfg);
    const double scale = ora_scale(cfg);
    const int64_t T = cu[N];
    for (int n = 0; n < N; ++n)
        if (cu[n + 1] < cu[n] || slots[n] >= P) return 2;

    int64_t work = (int64_t)N * HV;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t wi = 0; wi < work; ++wi) {
        int n = (int)(wi / HV), h = (int)(wi % HV);
        if (head_mask && !head_mask[h]) continue;
        int L = cu[n + 1] - cu[n];
        int slot = slots[n];
        const int64_t t0 = cu[n];
        if (slot < 0) { /* padded request: zero output rows, nothing else */
            for (int t = 0; t < L; ++t)
                for (int j = 0; j < dv; ++j) out[((t0 + t) * HV + h) * dv + j] = 0.0;
            continue;
        }
        if (L == 0) continue;
        int hk = h / G;
        int use_init = has_init ? has_init[n] != 0 : 1;
        /* channel offsets of this head's q, k, v inside a mixed_qkv row */
        int64_t cq = (int64_t)hk * dk, ck = (int64_t)HK * dk + (int64_t)hk * dk,
                cv = 2LL * HK * dk + (int64_t)h * dv;
        double* q = (double*)malloc(sizeof(double) * L * dk);
        double* kk = (double*)malloc(sizeof(double) * L * dk);
        double* v = (double*)malloc(sizeof(double) * L * dv);
        double* gg = (double*)malloc(sizeof(double) * L);
        double* bb = (double*)malloc(sizeof(double) * L);
        double* o = (double*)malloc(sizeof(double) * L * dv);
        const double* hist_base = conv_state + (int64_t)slot * CD * (K - 1);
        ora_conv_silu(L, dk, K, x + t0 * CD + cq, CD, use_init ? hist_base + cq * (K - 1) : NULL,
                      conv_w + cq * K, conv_b ? conv_b + cq : NULL, q);
        ora_conv_silu(L, dk, K, x + t0 * CD + ck, CD, use_init ? hist_base + ck * (K - 1) : NULL,
                      conv_w + ck * K, conv_b ? conv_b + ck : NULL, kk);
        ora_conv_silu(L, dv, K, x + t0 * CD + cv, CD, use_init ? hist_base + cv * (K - 1) : NULL,
                      conv_w + cv * K, conv_b ? conv_b + cv : NULL, v);
        for (int t = 0; t < L; ++t) {
            ora_l2norm(q + (int64_t)t * dk, dk, cfg->eps);
            ora_l2norm(kk + (int64_t)t * dk, dk, cfg->eps);
            gg[t] = ora_gate_g(A_log[h], a[(t0 + t) * HV + h], dt_bias[h]);
            bb[t] = ora_gate_beta(b[(t0 + t) * HV + h]);
        }
        double* S = ssm_state + ((int64_t)slot * HV + h) * dk * dv;
        if (!use_init) memset(S, 0, sizeof(double) * dk * dv);
        if (chunk > 0) {
            ora_core_chunked(L, dk, dv, q, kk, v, gg, bb, scale, chunk, S, o);
        } else if (states_per_token) {
            double* st = (double*)malloc(sizeof(double) * L * dk * dv);
            ora_core_recurrent(L, dk, dv, q, kk, v, gg, bb, scale, S, o, st);
            for (int t = 0; t < L; ++t)
                memcpy(states_per_token + ((t0 + t) * HV + h) * dk * dv, st + (int64_t)t * dk * dv,
                       sizeof(double) * dk * dv);
            free(st);
        } else {
            ora_core_recurrent(L, dk, dv, q, kk, v, gg, bb, scale, S, o, NULL);
        }
        for (int t = 0; t < L; ++t)
            for (int j = 0; j < dv; ++j) out[((t0 + t) * HV + h) * dv + j] = o[(int64_t)t * dv + j];
        free(q); free(kk); free(v); free(gg); free(bb); free(o);
    }
    /* conv state: the K-1 most recent raw rows of (old state | sequence) */
    for (int n = 0; n < N; ++n) {
        int L = cu[n + 1] - cu[n], slot = slots[n];
        if (slot < 0 || L == 0) continue;
        int use_init = has_init ? has_init[n] != 0 : 1;
        double* st = conv_state + (int64_t)slot * CD * (K - 1);
        /* concatenation positions L .. L+K-2; position p < K-1 is old[p], else row p-(K-1) */
        double* tail = (double*)malloc(sizeof(double) * (K > 1 ? K - 1 : 1));
        for (int64_t c = 0; c < CD; ++c) {
            for (int i = 0; i < K - 1; ++i) {
                int64_t pos = (int64_t)L + i;
                tail[i] = pos < K - 1 ? (use_init ? st[c * (K - 1) + pos] : 0.0)
                                      : x[(cu[n] + pos - (K - 1)) * CD + c];
            }
            for (int i = 0; i < K - 1; ++i) st[c * (K - 1) + i] = tail[i];
        }
        free(tail);
    }
    (void)T;
    return 0;
}

int ora_extend(const ora_cfg* cfg, const double* A_log, const double* dt_bias, const double* conv_w,
               const double* conv_b, const double* x, const double* a, const double* b, const int32_t* cu,
               int N, const int32_t* slots, const int32_t* has_init, double* conv_state, double* ssm_state,
               int P, double* out, const int32_t* head_mask) {
    return ora_layer(cfg, A_log, dt_bias, conv_w, conv_b, x, a, b, cu, N, slots, has_init, conv_state,
                     ssm_state, P, out, 0, head_mask, NULL);
}

int ora_extend_chunked(const ora_cfg* cfg, const double* A_log, const double* dt_bias, const double* conv_w,
                       const double* conv_b, const double* x, const double* a, const double* b,
                       const int32_t* cu, int N, const int32_t* slots, const int32_t* has_init,
                       double* conv_state, double* ssm_state, int P, double* out, int chunk) {
    if (chunk <= 0) return 1;
    return ora_layer(cfg, A_log, dt_bias, conv_w, conv_b, x, a, b, cu, N, slots, has_init, conv_state,
                     ssm_state, P, out, chunk, NULL, NULL);
}

/*
 * Single-token decode for B requests: each request is a sequence of length 1
 * continuing from its slot.  x: [B, conv_dim], a, b: [B, HV], out [B, HV, dv].
 */
int ora_decode(const ora_cfg* cfg, const double* A_log, const double* dt_bias, const double* conv_w,
               const double* conv_b, const double* x, const double* a, const double* b, int B,
               const int32_t* slots, double* conv_state, double* ssm_state, int P, double* out) {
    int32_t* cu = (int32_t*)malloc(sizeof(int32_t) * (B + 1));
    for (int i = 0; i <= B; ++i) cu[i] = i;
    int rc = ora_layer(cfg, A_log, dt_bias, conv_w, conv_b, x, a, b, cu, B, slots, NULL, conv_state, ssm_state,
                       P, out, 0, NULL, NULL);
    free(cu);
    return rc;
}

/*
 * Speculative verify: request i runs D tokens (rows i*D .. i*D+D-1 of x, a, b)
 * from its slot.  The pools are read only; ckpt [B, D, HV, dk, dv] receives the
 * state after every token and conv_ckpt [B, D, conv_dim, K-1] (nullable) the
 * conv window (K-1 most recent raw rows) after every token.
 * Padded requests (slot < 0) get zero output rows and untouched checkpoints.
 */
int ora_verify(const ora_cfg* cfg, const double* A_log, const double* dt_bias, const double* conv_w,
               const double* conv_b, const double* x, const double* a, const double* b, int B, int D,
               const int32_t* slots, const double* conv_state, const double* ssm_state, int P, double* ckpt,
               double* conv_ckpt, double* out) {
    const int HV = cfg->HV, dk = cfg->dk, dv = cfg->dv, K = cfg->K;
    const int64_t CD = ora_conv_dim(cfg);
    const int64_t sslot = (int64_t)HV * dk * dv, cslot = CD * (K - 1);
    if (B < 0 || D < 1) return 1;
    /* private copies of each request's slot, so the pools stay untouched */
    double* cs = (double*)malloc(sizeof(double) * (B > 0 ? B : 1) * cslot);
    double* ss = (double*)malloc(sizeof(double) * (B > 0 ? B : 1) * sslot);
    double* st = (double*)malloc(sizeof(double) * (int64_t)(B > 0 ? B : 1) * D * HV * dk * dv);
    int32_t* cu = (int32_t*)malloc(sizeof(int32_t) * (B + 1));
    int32_t* loc = (int32_t*)malloc(sizeof(int32_t) * (B > 0 ? B : 1));
    for (int i = 0; i < B; ++i) {
        if (slots[i] >= P) { free(cs); free(ss); free(st); free(cu); free(loc); return 2; }
        loc[i] = slots[i] < 0 ? -1 : i;
        if (slots[i] >= 0) {
            memcpy(cs + i * cslot, conv_state + slots[i] * cslot, sizeof(double) * cslot);
            memcpy(ss + i * sslot, ssm_state + slots[i] * sslot, sizeof(double) * sslot);
        }
    }
    for (int i = 0; i <= B; ++i) cu[i] = i * D;
    int rc = ora_layer(cfg, A_log, dt_bias, conv_w, conv_b, x, a, b, cu, B, loc, NULL, cs, ss, B, out, 0,
                       NULL, st);
    if (rc == 0) {
        for (int i = 0; i < B; ++i) {
            if (slots[i] < 0) continue;
            for (int t = 0; t < D; ++t)
                for (int h = 0; h < HV; ++h)
                    memcpy(ckpt + (((int64_t)i * D + t) * HV + h) * dk * dv,
                           st + (((int64_t)i * D + t) * HV + h) * dk * dv, sizeof(double) * dk * dv);
            if (conv_ckpt) {
                const double* old = conv_state + slots[i] * cslot;
                for (int t = 0; t < D; ++t)
                    for (int64_t c = 0; c < CD; ++c)
                        for (int j = 0; j < K - 1; ++j) {
                            /* window after token t: rows (t+1)-(K-1)+j of the request, negative = old state */
                            int src = t + 1 - (K - 1) + j;
                            double val = src >= 0 ? x[((int64_t)i * D + src) * CD + c]
                                                  : old[c * (K - 1) + (K - 1 + src)];
                            conv_ckpt[(((int64_t)i * D + t) * CD + c) * (K - 1) + j] = val;
                        }
            }
        }
    }
    free(cs); free(ss); free(st); free(cu); free(loc);
    return rc;
}

/*
 * Speculative commit, the step after verify: request i accepted acc[i] of its D
 * draft tokens; for acc[i] >= 1 its slot takes the checkpoints recorded after
 * token acc[i]-1 (state and, when conv_ckpt is non-NULL, conv window), so the
 * pools hold what running the accepted tokens from the slot would have left;
 * acc[i] == 0 and padded requests (slot < 0) leave everything untouched.  The
 * commit of the speculative state buffer for the accepted draft prefix, page
 * "SGLang GDN hybrid linear attention test matrix", verification conventions.
 * Returns 2 for a slot >= P and 3 for an accepted count outside 0..D (nothing
 * written for that request).
 */
int ora_commit(const ora_cfg* cfg, int B, int D, const int32_t* slots, const int32_t* acc, const double* ckpt,
               const double* conv_ckpt, double* conv_state, double* ssm_state, int P) {
    const int HV = cfg->HV, dk = cfg->dk, dv = cfg->dv, K = cfg->K;
    const int64_t CD = ora_conv_dim(cfg);
    const int64_t sslot = (int64_t)HV * dk * dv, cslot = CD * (K - 1);
    int rc = 0;
    for (int i = 0; i < B; ++i) {
        if (slots[i] < 0) continue;
        if (slots[i] >= P) { rc = 2; continue; }
        if (acc[i] < 0 || acc[i] > D) { rc = 3; continue; }
        if (acc[i] == 0) continue;
        const int64_t t = (int64_t)i * D + (acc[i] - 1);
        memcpy(ssm_state + slots[i] * sslot, ckpt + t * sslot, sizeof(double) * sslot);
        if (conv_ckpt) memcpy(conv_state + slots[i] * cslot, conv_ckpt + t * cslot, sizeof(double) * cslot);
    }
    return rc;
}

/*
 * Extend with one state checkpoint per sequence (prefix caching): sequence n
 * names an exclusive absolute packed-row boundary ck_idx[n] with
 * cu[n] <= ck_idx[n] <= cu[n+1] and a row ck_slot[n] of ck_states
 * [num_ck, HV, dk, dv]; that row receives the state after rows
 * cu[n] .. ck_idx[n]-1 (the state the sequence started from when the boundary
 * is its first row), and ck_conv [num_ck, conv_dim, K-1] (nullable) the conv
 * window there: the K-1 raw rows before the boundary, reaching into the
 * sequence's starting conv window.  Page "flashinfer ... ssd_combined"
 * (checkpoint_token_indices: one exclusive boundary per sequence, absolute for
 * packed varlen, negative disables; checkpoint_state_slots: the row, negative
 * disables; checkpoint_states: [num_checkpoints, nheads, headdim, dstate]).
 * Padded sequences (slot < 0) capture nothing.  Everything else is ora_extend.
 * Returns 4 when a boundary lies outside its sequence or a row >= num_ck
 * (that sequence is skipped), else ora_extend's code.
 */
int ora_extend_ckpt(const ora_cfg* cfg, const double* A_log, const double* dt_bias, const double* conv_w,
                    const double* conv_b, const double* x, const double* a, const double* b, const int32_t* cu,
                    int N, const int32_t* slots, const int32_t* has_init, double* conv_state, double* ssm_state,
                    int P, double* out, const int32_t* ck_idx, const int32_t* ck_slot, double* ck_states,
                    double* ck_conv, int num_ck) {
    const int HV = cfg->HV, dk = cfg->dk, dv = cfg->dv, K = cfg->K;
    const int64_t CD = ora_conv_dim(cfg);
    const int64_t sslot = (int64_t)HV * dk * dv, cslot = CD * (K - 1);
    const int64_t T = cu[N];
    double* st = (double*)malloc(sizeof(double) * (T > 0 ? T : 1) * sslot);
    double* ss0 = (double*)malloc(sizeof(double) * (P > 0 ? P : 1) * sslot);
    double* cs0 = (double*)malloc(sizeof(double) * (P > 0 ? P : 1) * cslot);
    memcpy(ss0, ssm_state, sizeof(double) * P * sslot);
    memcpy(cs0, conv_state, sizeof(double) * P * cslot);
    int rc = ora_layer(cfg, A_log, dt_bias, conv_w, conv_b, x, a, b, cu, N, slots, has_init, conv_state, ssm_state,
                       P, out, 0, NULL, st);
    if (rc == 0) {
        for (int n = 0; n < N; ++n) {
            if (ck_idx[n] < 0 || ck_slot[n] < 0 || slots[n] < 0) continue;
            if (ck_idx[n] < cu[n] || ck_idx[n] > cu[n + 1] || ck_slot[n] >= num_ck) { rc = 4; continue; }
            const int64_t bnd = ck_idx[n];
            const int init = has_init ? has_init[n] != 0 : 1;
            double* dst = ck_states + (int64_t)ck_slot[n] * sslot;
            if (bnd > cu[n]) memcpy(dst, st + (bnd - 1) * sslot, sizeof(double) * sslot);
            else if (init) memcpy(dst, ss0 + (int64_t)slots[n] * sslot, sizeof(double) * sslot);
            else memset(dst, 0, sizeof(double) * sslot);
            if (ck_conv) {
                double* cdst = ck_conv + (int64_t)ck_slot[n] * cslot;
                for (int64_t c = 0; c < CD; ++c)
                    for (int j = 0; j < K - 1; ++j) {
                        const int64_t r = bnd - (K - 1) + j; /* raw row j of the window, index 0 oldest */
                        double v;
                        if (r >= cu[n]) v = x[r * CD + c];
                        else v = init ? cs0[(int64_t)slots[n] * cslot + c * (K - 1) + (K - 1) + (r - cu[n])] : 0.0;
                        cdst[c * (K - 1) + j] = v;
                    }
            }
        }
    }
    free(st); free(ss0); free(cs0);
    return rc;
}
