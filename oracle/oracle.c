/*
 * CPU ORACLE of the batch-1 transformer decode step.  TEST INFRASTRUCTURE:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this library.  It shares no code with the CUDA path.
 *
 * What it computes.  One autoregressive decode step of a Llama-style decoder
 * (RMSNorm, rotary position embedding, grouped-query attention over a KV
 * cache, SiLU-gated feed-forward or a routed mixture of experts, LM head).
 * The pages name the operators of that step: QKV projection, attention,
 * O-projection, MoE router and expert up/down projections (page "Cohere
 * megakerneles kiszolgálót mutatott be a North Mini Code modellhez",
 * sections "Egyetlen tartós kernelre épül a kiszolgálás" and "Honnan jön a
 * gyorsulás?"), matmul and attention tasks (MPK digest page "LLM को
 * MegaKernel में compile करके low-latency inference हासिल करना", section
 * "Part 2. Runtime", Worker); bf16 weights streamed once per step (Cohere
 * page, section "A szűk keresztmetszet a memória-sávszélesség").  The
 * megakernel computes exactly this result; nothing here is an approximation,
 * so the oracle is the plain definition written out.
 *
 * Precision: weights and the KV cache are bf16 (exactly widened); every
 * activation and every accumulation is double.  The only rounding the
 * definition itself performs is the KV-cache append, bf16 round-to-nearest-
 * even.  Readings taken where the pages are silent (each one listed in the
 * design notes): rotate-half RoPE with inv_freq_i = theta^(-2i/d); q head h
 * reads kv head floor(h * n_kv / n_q); the new token attends to positions
 * 0..p inclusive after its own append, scores scaled by 1/sqrt(d); router
 * softmax over all experts, top-k ties to the lower index, selected weights
 * renormalised when moe_renorm != 0; argmax ties to the lower index.
 *
 * Parity pins: every function here is checked by tests against closed forms,
 * invariants and library routines (tests/test_oracle_pins.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
    double rms_eps, rope_theta;
    int n_experts, top_k, expert_ffn, moe_renorm;
} oc_config;

/* Optional supplier of one expert's matrix when the caller does not hold all
 * experts in memory.  which: 0 gate [Fe][H], 1 up [Fe][H], 2 down [H][Fe].
 * Returns 0 once dst holds the whole matrix, nonzero on failure; a failure
 * ends the step with an error code, never with a partly filled matrix. */
typedef int (*oc_expert_provider)(int layer, int expert, int which, uint16_t* dst, void* user);

/* ------------------------------------------------------------------ scalars */

double oc_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even, in one step (no
 * intermediate fp32 rounding).  bf16 keeps 8 significant bits; subnormals
 * are multiples of 2^-133.  Returns the bf16 bit pattern. */
uint16_t oc_bf16_round(double x) {
    if (x == 0.0) return signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return 0x7FC0u;
    double ax = fabs(x);
    double q;
    if (ax < ldexp(1.0, -126)) {
        q = ldexp(1.0, -133);
    } else {
        int e;
        frexp(ax, &e);               /* ax in [2^(e-1), 2^e) */
        q = ldexp(1.0, e - 8);
    }
    double r = nearbyint(x / q) * q; /* default rounding mode: ties to even */
    float f = (float)r;              /* exact, or +-inf when r reaches 2^128 */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

double oc_silu(double z) { return z / (1.0 + exp(-z)); }

/* ------------------------------------------------------------------ vectors */

/* out_i = x_i * (sum_j x_j^2 / n + eps)^(-1/2) * g_i */
void oc_rmsnorm(const double* x, const uint16_t* g, int n, double eps, double* out) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss / n + eps);
    for (int i = 0; i < n; ++i) out[i] = x[i] * r * oc_bf16_to_double(g[i]);
}

/* Rotate-half rotary embedding of one head vector v[0..d) at position pos:
 * pairs (i, i + d/2) rotate by angle pos * theta^(-2i/d). */
void oc_rope(double* v, int d, int pos, double theta) {
    int h = d / 2;
    for (int i = 0; i < h; ++i) {
        double inv_freq = pow(theta, -2.0 * (double)i / (double)d);
        double a = (double)pos * inv_freq;
        double c = cos(a), s = sin(a);
        double x0 = v[i], x1 = v[i + h];
        v[i] = x0 * c - x1 * s;
        v[i + h] = x1 * c + x0 * s;
    }
}

/* y_r = sum_c W[r][c] * x[c]; W is bf16 row-major [rows][cols]. */
void oc_gemv(const uint16_t* W, int rows, int cols, const double* x, double* y) {
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const uint16_t* w = W + (size_t)r * cols;
        double acc = 0.0;
        for (int c = 0; c < cols; ++c) acc += oc_bf16_to_double(w[c]) * x[c];
        y[r] = acc;
    }
}

/* Decode attention for all q heads over n_tok cached positions.
 * q [n_q][d]; K, V bf16 [n_tok][n_kv][d] (position-major); o [n_q][d].
 * q head h uses kv head floor(h * n_kv / n_q); scores scaled by 1/sqrt(d). */
void oc_attention(const double* q, const uint16_t* K, const uint16_t* V, int n_tok, int n_q,
                  int n_kv, int d, double* o) {
#pragma omp parallel for schedule(static)
    for (int h = 0; h < n_q; ++h) {
        int g = (int)((long)h * n_kv / n_q);
        double* s = (double*)malloc(sizeof(double) * (n_tok > 0 ? n_tok : 1));
        double m = -INFINITY;
        for (int j = 0; j < n_tok; ++j) {
            const uint16_t* kj = K + ((size_t)j * n_kv + g) * d;
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += q[h * d + i] * oc_bf16_to_double(kj[i]);
            s[j] = acc / sqrt((double)d);
            if (s[j] > m) m = s[j];
        }
        double den = 0.0;
        for (int j = 0; j < n_tok; ++j) {
            s[j] = exp(s[j] - m);
            den += s[j];
        }
        for (int i = 0; i < d; ++i) o[h * d + i] = 0.0;
        for (int j = 0; j < n_tok; ++j) {
            const uint16_t* vj = V + ((size_t)j * n_kv + g) * d;
            double a = s[j] / den;
            for (int i = 0; i < d; ++i) o[h * d + i] += a * oc_bf16_to_double(vj[i]);
        }
        free(s);
    }
}

/* Index of the largest value, ties to the lowest index. */
int oc_argmax(const double* v, int n) {
    int best = 0;
    for (int i = 1; i < n; ++i)
        if (v[i] > v[best]) best = i;
    return best;
}

/* ------------------------------------------------------------------ feed-forward */

/* SiLU-gated FFN: y = W_down (silu(W_gate h) * (W_up h)).  W_gate, W_up
 * [F][H]; W_down [H][F]. */
void oc_swiglu_ffn(const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down, int H,
                   int F, const double* h, double* y) {
    double* gt = (double*)malloc(sizeof(double) * F);
    double* up = (double*)malloc(sizeof(double) * F);
    oc_gemv(w_gate, F, H, h, gt);
    oc_gemv(w_up, F, H, h, up);
    for (int i = 0; i < F; ++i) gt[i] = oc_silu(gt[i]) * up[i];
    oc_gemv(w_down, H, F, gt, y);
    free(gt);
    free(up);
}

/* Router: r = W_r h (E logits), pi = softmax(r).  Selects the top_k largest
 * pi (ties to the lower expert index) into sel[], their weights into wts[]
 * (renormalised to sum 1 when renorm != 0), and writes pi into probs[] when
 * given.  If override_sel is non-NULL it is used as the selected set instead
 * (harness use: a near-tie where either set is a correct result). */
void oc_moe_route(const uint16_t* w_router, int E, int H, const double* h, int top_k, int renorm,
                  const int* override_sel, int* sel, double* wts, double* probs) {
    double* r = (double*)malloc(sizeof(double) * E);
    oc_gemv(w_router, E, H, h, r);
    double m = r[0];
    for (int e = 1; e < E; ++e)
        if (r[e] > m) m = r[e];
    double den = 0.0;
    for (int e = 0; e < E; ++e) {
        r[e] = exp(r[e] - m);
        den += r[e];
    }
    for (int e = 0; e < E; ++e) r[e] /= den;
    if (probs)
        for (int e = 0; e < E; ++e) probs[e] = r[e];
    char* taken = (char*)calloc(E, 1);
    for (int k = 0; k < top_k; ++k) {
        int best = -1;
        if (override_sel) {
            best = override_sel[k];
        } else {
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || r[e] > r[best])) best = e;
        }
        taken[best] = 1;
        sel[k] = best;
        wts[k] = r[best];
    }
    if (renorm) {
        double s = 0.0;
        for (int k = 0; k < top_k; ++k) s += wts[k];
        for (int k = 0; k < top_k; ++k) wts[k] /= s;
    }
    free(taken);
    free(r);
}

/* ------------------------------------------------------------------ model plumbing */

static int layer_slots(const oc_config* c) { return c->n_experts > 0 ? 10 : 9; }

/* Weight pointer order (host bf16): tok_emb, then per layer attn_norm, wq,
 * wk, wv, wo, ffn_norm, [w_router,] w_gate, w_up, w_down, then final_norm,
 * lm_head. */
static const uint16_t* wptr(const oc_config* c, const uint16_t* const* w, int layer, int slot) {
    return w[1 + layer * layer_slots(c) + slot];
}
enum { S_ATTN_NORM = 0, S_WQ, S_WK, S_WV, S_WO, S_FFN_NORM };

/* Returns 0, or -2 when the expert weights are neither held nor supplied. */
static int moe_ffn_layer(const oc_config* c, const uint16_t* const* w, int l,
                         oc_expert_provider prov, void* user, const int* override_sel,
                         const double* h, double* y, int* sel_out, double* wts_out) {
    int H = c->hidden, E = c->n_experts, Fe = c->expert_ffn, K = c->top_k;
    const uint16_t* w_router = wptr(c, w, l, 6);
    const uint16_t* wg_all = wptr(c, w, l, 7);
    const uint16_t* wu_all = wptr(c, w, l, 8);
    const uint16_t* wd_all = wptr(c, w, l, 9);
    int* sel = (int*)malloc(sizeof(int) * K);
    double* wts = (double*)malloc(sizeof(double) * K);
    oc_moe_route(w_router, E, H, h, K, c->moe_renorm, override_sel, sel, wts, NULL);
    double* ye = (double*)malloc(sizeof(double) * H);
    uint16_t* tmp = NULL;
    int rc = 0;
    if (!wg_all) tmp = (uint16_t*)malloc(sizeof(uint16_t) * 3 * (size_t)Fe * H);
    for (int i = 0; i < H; ++i) y[i] = 0.0;
    for (int k = 0; k < K && rc == 0; ++k) {
        int e = sel[k];
        const uint16_t *wg, *wu, *wd;
        if (wg_all) {
            wg = wg_all + (size_t)e * Fe * H;
            wu = wu_all + (size_t)e * Fe * H;
            wd = wd_all + (size_t)e * H * Fe;
        } else {
            if (!prov || prov(l, e, 0, tmp, user) != 0 || prov(l, e, 1, tmp + (size_t)Fe * H, user) != 0 ||
                prov(l, e, 2, tmp + 2 * (size_t)Fe * H, user) != 0) {
                rc = -2;
                break;
            }
            wg = tmp;
            wu = tmp + (size_t)Fe * H;
            wd = tmp + 2 * (size_t)Fe * H;
        }
        oc_swiglu_ffn(wg, wu, wd, H, Fe, h, ye);
        for (int i = 0; i < H; ++i) y[i] += wts[k] * ye[i];
    }
    if (sel_out)
        for (int k = 0; k < K; ++k) sel_out[k] = sel[k];
    if (wts_out)
        for (int k = 0; k < K; ++k) wts_out[k] = wts[k];
    free(tmp);
    free(ye);
    free(wts);
    free(sel);
    return rc;
}

/*
 * One decode step for one sequence: token `token` at position `pos` (= number
 * of tokens already cached).  kcache[l] / vcache[l] are bf16 [ctx_cap][n_kv][d]
 * position-major; the step writes position pos of every layer.  Outputs:
 * logits [vocab] (double).  Optional: hidden [2L+1][H] gets the residual
 * stream after the embedding and after each attention / FFN residual add;
 * moe_sel [L][top_k] and moe_wts [L][top_k] the router's choice per layer;
 * moe_override [L][top_k] (entries < 0 mean "no override for this layer")
 * forces a selected set.  Returns 0, -1 on a bad argument, or -2 when the
 * expert provider failed (the outputs are then not valid).
 */
int oc_decode_step(const oc_config* c, const uint16_t* const* w, uint16_t* const* kcache,
                   uint16_t* const* vcache, int ctx_cap, int token, int pos, double* logits,
                   double* hidden, oc_expert_provider prov, void* user, const int* moe_override,
                   int* moe_sel, double* moe_wts) {
    if (pos < 0 || pos >= ctx_cap || token < 0 || token >= c->vocab) return -1;
    int H = c->hidden, d = c->head_dim, nq = c->n_q_heads, nkv = c->n_kv_heads;
    int L = c->n_layers;
    double* x = (double*)malloc(sizeof(double) * H);
    double* h = (double*)malloc(sizeof(double) * H);
    double* q = (double*)malloc(sizeof(double) * nq * d);
    double* k = (double*)malloc(sizeof(double) * nkv * d);
    double* v = (double*)malloc(sizeof(double) * nkv * d);
    double* o = (double*)malloc(sizeof(double) * nq * d);
    double* y = (double*)malloc(sizeof(double) * H);
    int rc = 0;

    const uint16_t* emb = w[0] + (size_t)token * H;
    for (int i = 0; i < H; ++i) x[i] = oc_bf16_to_double(emb[i]);
    if (hidden) memcpy(hidden, x, sizeof(double) * H);

    for (int l = 0; l < L && rc == 0; ++l) {
        /* attention block */
        oc_rmsnorm(x, wptr(c, w, l, S_ATTN_NORM), H, c->rms_eps, h);
        oc_gemv(wptr(c, w, l, S_WQ), nq * d, H, h, q);
        oc_gemv(wptr(c, w, l, S_WK), nkv * d, H, h, k);
        oc_gemv(wptr(c, w, l, S_WV), nkv * d, H, h, v);
        for (int hh = 0; hh < nq; ++hh) oc_rope(q + hh * d, d, pos, c->rope_theta);
        for (int g = 0; g < nkv; ++g) oc_rope(k + g * d, d, pos, c->rope_theta);
        uint16_t* kl = kcache[l] + (size_t)pos * nkv * d;
        uint16_t* vl = vcache[l] + (size_t)pos * nkv * d;
        for (int i = 0; i < nkv * d; ++i) {
            kl[i] = oc_bf16_round(k[i]);
            vl[i] = oc_bf16_round(v[i]);
        }
        oc_attention(q, kcache[l], vcache[l], pos + 1, nq, nkv, d, o);
        oc_gemv(wptr(c, w, l, S_WO), H, nq * d, o, y);
        for (int i = 0; i < H; ++i) x[i] += y[i];
        if (hidden) memcpy(hidden + (size_t)(2 * l + 1) * H, x, sizeof(double) * H);

        /* feed-forward block */
        oc_rmsnorm(x, wptr(c, w, l, S_FFN_NORM), H, c->rms_eps, h);
        if (c->n_experts > 0) {
            const int* ov = NULL;
            if (moe_override && moe_override[l * c->top_k] >= 0) ov = moe_override + l * c->top_k;
            rc = moe_ffn_layer(c, w, l, prov, user, ov, h, y, moe_sel ? moe_sel + l * c->top_k : NULL,
                               moe_wts ? moe_wts + l * c->top_k : NULL);
            if (rc != 0) break;
        } else {
            oc_swiglu_ffn(wptr(c, w, l, 6), wptr(c, w, l, 7), wptr(c, w, l, 8), H, c->ffn, h, y);
        }
        for (int i = 0; i < H; ++i) x[i] += y[i];
        if (hidden) memcpy(hidden + (size_t)(2 * l + 2) * H, x, sizeof(double) * H);
    }
    if (rc == 0) {
        const uint16_t* final_norm = w[1 + L * layer_slots(c)];
        const uint16_t* lm_head = w[2 + L * layer_slots(c)];
        oc_rmsnorm(x, final_norm, H, c->rms_eps, h);
        oc_gemv(lm_head, c->vocab, H, h, logits);
    }

    free(x); free(h); free(q); free(k); free(v); free(o); free(y);
    return rc;
}

/*
 * Full recomputation without a cache: runs all T tokens of one sequence
 * (positions 0..T-1) layer by layer, computing every position's K and V
 * afresh (rounded to bf16 as the cache would hold them) and causal attention
 * for every position.  logits [T][vocab].  Used to check that the cached
 * incremental decode reproduces it.  Dense and MoE models.  Returns 0, -1 on
 * a bad argument, -2 when the expert provider failed.
 */
int oc_forward_nocache(const oc_config* c, const uint16_t* const* w, const int* tokens, int T,
                       double* logits, oc_expert_provider prov, void* user) {
    int H = c->hidden, d = c->head_dim, nq = c->n_q_heads, nkv = c->n_kv_heads;
    int L = c->n_layers;
    for (int t = 0; t < T; ++t)
        if (tokens[t] < 0 || tokens[t] >= c->vocab) return -1;
    double* X = (double*)malloc(sizeof(double) * (size_t)T * H);
    double* h = (double*)malloc(sizeof(double) * H);
    double* q = (double*)malloc(sizeof(double) * (size_t)T * nq * d);
    double* kv = (double*)malloc(sizeof(double) * nkv * d);
    uint16_t* K = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)T * nkv * d);
    uint16_t* V = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)T * nkv * d);
    double* o = (double*)malloc(sizeof(double) * nq * d);
    double* y = (double*)malloc(sizeof(double) * H);
    int rc = 0;

    for (int t = 0; t < T; ++t)
        for (int i = 0; i < H; ++i) X[(size_t)t * H + i] = oc_bf16_to_double(w[0][(size_t)tokens[t] * H + i]);

    for (int l = 0; l < L && rc == 0; ++l) {
        for (int t = 0; t < T; ++t) {
            oc_rmsnorm(X + (size_t)t * H, wptr(c, w, l, S_ATTN_NORM), H, c->rms_eps, h);
            double* qt = q + (size_t)t * nq * d;
            oc_gemv(wptr(c, w, l, S_WQ), nq * d, H, h, qt);
            for (int hh = 0; hh < nq; ++hh) oc_rope(qt + hh * d, d, t, c->rope_theta);
            oc_gemv(wptr(c, w, l, S_WK), nkv * d, H, h, kv);
            for (int g = 0; g < nkv; ++g) oc_rope(kv + g * d, d, t, c->rope_theta);
            for (int i = 0; i < nkv * d; ++i) K[(size_t)t * nkv * d + i] = oc_bf16_round(kv[i]);
            oc_gemv(wptr(c, w, l, S_WV), nkv * d, H, h, kv);
            for (int i = 0; i < nkv * d; ++i) V[(size_t)t * nkv * d + i] = oc_bf16_round(kv[i]);
        }
        for (int t = 0; t < T && rc == 0; ++t) {
            /* causal: position t sees positions 0..t */
            oc_attention(q + (size_t)t * nq * d, K, V, t + 1, nq, nkv, d, o);
            oc_gemv(wptr(c, w, l, S_WO), H, nq * d, o, y);
            double* xt = X + (size_t)t * H;
            for (int i = 0; i < H; ++i) xt[i] += y[i];
            oc_rmsnorm(xt, wptr(c, w, l, S_FFN_NORM), H, c->rms_eps, h);
            if (c->n_experts > 0) {
                rc = moe_ffn_layer(c, w, l, prov, user, NULL, h, y, NULL, NULL);
                if (rc != 0) break;
            } else
                oc_swiglu_ffn(wptr(c, w, l, 6), wptr(c, w, l, 7), wptr(c, w, l, 8), H, c->ffn, h, y);
            for (int i = 0; i < H; ++i) xt[i] += y[i];
        }
    }
    const uint16_t* final_norm = w[1 + L * layer_slots(c)];
    const uint16_t* lm_head = w[2 + L * layer_slots(c)];
    for (int t = 0; t < T && rc == 0; ++t) {
        oc_rmsnorm(X + (size_t)t * H, final_norm, H, c->rms_eps, h);
        oc_gemv(lm_head, c->vocab, H, h, logits + (size_t)t * c->vocab);
    }
    free(X); free(h); free(q); free(kv); free(K); free(V); free(o); free(y);
    return rc;
}

int oc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
