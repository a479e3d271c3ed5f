/*
 * Oracle for the DuoLM ranker forward -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU code that states what the ranker computes, one step
 * at a time.  Only the tests, the smoke check and the benchmark's CPU
 * baseline may load it; the CUDA library never does, and shares no code,
 * header or table with it.
 *
 * What it computes (DuoLM summary page, paper.rainbus.top, section 核心方法:
 * a Qwen3 ranker reads instruction, history entries and the candidate vector
 * and a shared linear head reads s = w^T h at the candidate's last hidden
 * state, no decoding).  The decoder layer is the Qwen3 pre-norm layer:
 *
 *   n = RMSNorm(x) * g_attn
 *   q = Wq n, k = Wk n, v = Wv n               (matrices stored [out][in])
 *   q_h = RMSNorm(q_h) * g_q, k_h = RMSNorm(k_h) * g_k   per head
 *   q, k rotated by RoPE at the row's position (rotate-half pairing)
 *   o_h = softmax(q_h . K_kv(h) / sqrt(head_dim)) V_kv(h)  over the row's keys
 *   x += Wo o
 *   n = RMSNorm(x) * g_mlp
 *   x += Wd (silu(Wg n) * (Wu n))
 *
 * and the score is s = head . (RMSNorm(x_last) * g_final).
 *
 * Which rows a row attends to is an input (a list of key rows per row, in
 * summation order).  The Python side builds those lists for the two modes:
 * independent sequences (plain causal) and the packed multi-item layout with
 * the tree mask.  Every per-row step sums in a fixed order that does not
 * depend on which other rows are present, so the two modes give the same bits
 * whenever a row sees the same keys in the same order.
 *
 * Weights arrive as float32 arrays (bfloat16 and fp32 weights are exact in
 * float32); every arithmetic step is fp64, multiply and add rounded
 * separately (built with -ffp-contract=off), sums taken in ascending index
 * order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int n_layers, d, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
    double rope_theta, rms_eps;
} oshape;

enum { W_ATTN_NORM, W_Q, W_K, W_V, W_QNORM, W_KNORM, W_O, W_MLP_NORM, W_GATE, W_UP, W_DOWN, W_PER_LAYER };

/* RMSNorm of n values: y_i = (x_i * (1 / sqrt(mean(x^2) + eps))) * g_i */
void oracle_rmsnorm(const double *x, const float *g, int n, double eps, double *y) {
    double ss = 0.0;
    for (int i = 0; i < n; i++) ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss / (double)n + eps);
    for (int i = 0; i < n; i++) y[i] = (x[i] * r) * (double)g[i];
}

/* Y[r][j] = sum_{k=0..in-1} W[j][k] * X[r][k], for n rows.
 * Loop order only groups independent sums (eight rows share one pass over a
 * weight row); each output is still the plain ascending-k sum. */
static void linear(const float *W, int out, int in, const double *X, int n, double *Y) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int jb = 0; jb < out; jb += 32) {
        int je = jb + 32 < out ? jb + 32 : out;
        for (int r0 = 0; r0 < n; r0 += 8) {
            int nr = n - r0 < 8 ? n - r0 : 8;
            for (int j = jb; j < je; j++) {
                const float *w = W + (size_t)j * in;
                double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                for (int k = 0; k < in; k++) {
                    double wk = (double)w[k];
                    for (int r = 0; r < nr; r++) acc[r] += wk * X[(size_t)(r0 + r) * in + k];
                }
                for (int r = 0; r < nr; r++) Y[(size_t)(r0 + r) * out + j] = acc[r];
            }
        }
    }
}

/* Rotate-half RoPE of one head vector at integer position pos:
 * for i < hd/2, angle = pos * theta^(-2i/hd), the pair (v_i, v_{i+hd/2})
 * is rotated by that angle. */
void oracle_rope(double *v, int hd, int pos, double theta) {
    int half = hd / 2;
    for (int i = 0; i < half; i++) {
        double inv_freq = pow(theta, -2.0 * (double)i / (double)hd);
        double ang = (double)pos * inv_freq;
        double c = cos(ang), s = sin(ang);
        double a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

/* Softmax attention of one query over n keys (rows of K and V with stride
 * `stride` doubles, head vectors of length hd):
 *   p_j = exp(s_j - max s) / sum_j exp(s_j - max s),  s_j = (q . k_j) * scale
 *   out = sum_j p_j v_j.
 * probs (length n) may be NULL. */
void oracle_attend(const double *q, const double *K, const double *V, int n, int hd, long stride,
                   double scale, double *probs, double *out, double *work) {
    double m = -INFINITY;
    for (int j = 0; j < n; j++) {
        const double *k = K + (size_t)j * stride;
        double dot = 0.0;
        for (int c = 0; c < hd; c++) dot += q[c] * k[c];
        work[j] = dot * scale;
        if (work[j] > m) m = work[j];
    }
    double l = 0.0;
    for (int j = 0; j < n; j++) {
        work[j] = exp(work[j] - m);
        l += work[j];
    }
    for (int c = 0; c < hd; c++) out[c] = 0.0;
    for (int j = 0; j < n; j++) {
        double p = work[j] / l;
        if (probs) probs[j] = p;
        const double *v = V + (size_t)j * stride;
        for (int c = 0; c < hd; c++) out[c] += p * v[c];
    }
}

static double silu(double g) { return g / (1.0 + exp(-g)); }

/*
 * Forward over n_rows rows.
 *   shape_i: n_layers, d, n_q_heads, n_kv_heads, head_dim, ffn, vocab
 *   shape_f: rope_theta, rms_eps
 *   w: 1 + 11 * n_layers + 2 float32 tensors in load order (embed; per layer
 *      attn_norm, wq, wk, wv, q_norm, k_norm, wo, mlp_norm, w_gate, w_up,
 *      w_down; final_norm, head)
 *   vid: [n_vid][d] float32 (the FP16 table rows, widened exactly)
 *   ids[r]: ranker id (< vocab: embedding row; vocab + i: table row i)
 *   pos[r]: position id used by RoPE
 *   keys of row r: key_idx[key_ptr[r] .. key_ptr[r+1]) in summation order
 *   out_rows: rows whose score is wanted -> scores[n_out]
 *   final_hidden: optional [n_out][d], the normed last hidden state
 *   layer_x: optional [n_layers + 1][n_rows][d], residual stream after the
 *            embedding and after each layer
 * Returns 0, or -1 on an id out of range, -2 on a key index out of range,
 * -3 on allocation failure.
 */
int oracle_forward(const int *shape_i, const double *shape_f, const float *const *w,
                   const float *vid, int64_t n_vid, int n_rows, const int32_t *ids,
                   const int32_t *pos, const int64_t *key_ptr, const int32_t *key_idx, int n_out,
                   const int32_t *out_rows, double *scores, double *final_hidden, double *layer_x) {
    oshape s = {shape_i[0], shape_i[1], shape_i[2], shape_i[3], shape_i[4], shape_i[5], shape_i[6],
                shape_f[0], shape_f[1]};
    const int d = s.d, hd = s.head_dim, qd = s.n_q_heads * hd, kd = s.n_kv_heads * hd, F = s.ffn;
    const int group = s.n_q_heads / s.n_kv_heads;
    const double scale = 1.0 / sqrt((double)hd);

    for (int r = 0; r < n_rows; r++) {
        if (ids[r] < 0 || (int64_t)ids[r] >= (int64_t)s.vocab + n_vid) return -1;
        for (int64_t e = key_ptr[r]; e < key_ptr[r + 1]; e++)
            if (key_idx[e] < 0 || key_idx[e] >= n_rows) return -2;
    }
    for (int o = 0; o < n_out; o++)
        if (out_rows[o] < 0 || out_rows[o] >= n_rows) return -2;
    int max_keys = 1;
    for (int r = 0; r < n_rows; r++) {
        int64_t nk = key_ptr[r + 1] - key_ptr[r];
        if (nk > max_keys) max_keys = (int)nk;
    }

    size_t R = (size_t)n_rows;
    double *x = malloc(R * d * sizeof(double));
    double *nrm = malloc(R * d * sizeof(double));
    double *q = malloc(R * qd * sizeof(double));
    double *k = malloc(R * kd * sizeof(double));
    double *v = malloc(R * kd * sizeof(double));
    double *o = malloc(R * qd * sizeof(double));
    double *g = malloc(R * F * sizeof(double));
    double *u = malloc(R * F * sizeof(double));
    double *y = malloc(R * d * sizeof(double));
    if (!x || !nrm || !q || !k || !v || !o || !g || !u || !y) {
        free(x); free(nrm); free(q); free(k); free(v); free(o); free(g); free(u); free(y);
        return -3;
    }

    /* Embedding: vocabulary ids read the embedding, virtual ids read the
     * item table (DuoLM summary page, 方法步骤详情 step 3). */
    for (int r = 0; r < n_rows; r++) {
        const float *src = ids[r] < s.vocab ? w[0] + (size_t)ids[r] * d
                                            : vid + (size_t)(ids[r] - s.vocab) * d;
        for (int c = 0; c < d; c++) x[(size_t)r * d + c] = (double)src[c];
    }
    if (layer_x) memcpy(layer_x, x, R * d * sizeof(double));

    for (int l = 0; l < s.n_layers; l++) {
        const float *const *lw = w + 1 + (size_t)l * W_PER_LAYER;
        for (int r = 0; r < n_rows; r++)
            oracle_rmsnorm(x + (size_t)r * d, lw[W_ATTN_NORM], d, s.rms_eps, nrm + (size_t)r * d);
        linear(lw[W_Q], qd, d, nrm, n_rows, q);
        linear(lw[W_K], kd, d, nrm, n_rows, k);
        linear(lw[W_V], kd, d, nrm, n_rows, v);
        #pragma omp parallel
        {
            double *tmp = malloc((size_t)hd * sizeof(double));
            #pragma omp for
            for (int r = 0; r < n_rows; r++) {
                for (int h = 0; h < s.n_q_heads; h++) {
                    double *qh = q + (size_t)r * qd + (size_t)h * hd;
                    oracle_rmsnorm(qh, lw[W_QNORM], hd, s.rms_eps, tmp);
                    memcpy(qh, tmp, hd * sizeof(double));
                    oracle_rope(qh, hd, pos[r], s.rope_theta);
                }
                for (int h = 0; h < s.n_kv_heads; h++) {
                    double *kh = k + (size_t)r * kd + (size_t)h * hd;
                    oracle_rmsnorm(kh, lw[W_KNORM], hd, s.rms_eps, tmp);
                    memcpy(kh, tmp, hd * sizeof(double));
                    oracle_rope(kh, hd, pos[r], s.rope_theta);
                }
            }
            free(tmp);
        }
        #pragma omp parallel
        {
            int nk_max = max_keys;
            double *Kg = malloc((size_t)nk_max * hd * sizeof(double));
            double *Vg = malloc((size_t)nk_max * hd * sizeof(double));
            double *work = malloc((size_t)nk_max * sizeof(double));
            #pragma omp for schedule(dynamic, 4)
            for (int r = 0; r < n_rows; r++) {
                int nk = (int)(key_ptr[r + 1] - key_ptr[r]);
                const int32_t *kl = key_idx + key_ptr[r];
                for (int h = 0; h < s.n_q_heads; h++) {
                    int kvh = h / group; /* grouped-query attention: query head h reads kv head h / group */
                    for (int j = 0; j < nk; j++) {
                        memcpy(Kg + (size_t)j * hd, k + (size_t)kl[j] * kd + (size_t)kvh * hd, hd * sizeof(double));
                        memcpy(Vg + (size_t)j * hd, v + (size_t)kl[j] * kd + (size_t)kvh * hd, hd * sizeof(double));
                    }
                    oracle_attend(q + (size_t)r * qd + (size_t)h * hd, Kg, Vg, nk, hd, hd, scale, NULL,
                                  o + (size_t)r * qd + (size_t)h * hd, work);
                }
            }
            free(Kg); free(Vg); free(work);
        }
        linear(lw[W_O], d, qd, o, n_rows, y);
        for (size_t i = 0; i < R * d; i++) x[i] += y[i];

        for (int r = 0; r < n_rows; r++)
            oracle_rmsnorm(x + (size_t)r * d, lw[W_MLP_NORM], d, s.rms_eps, nrm + (size_t)r * d);
        linear(lw[W_GATE], F, d, nrm, n_rows, g);
        linear(lw[W_UP], F, d, nrm, n_rows, u);
        for (size_t i = 0; i < R * F; i++) g[i] = silu(g[i]) * u[i];
        linear(lw[W_DOWN], d, F, g, n_rows, y);
        for (size_t i = 0; i < R * d; i++) x[i] += y[i];
        if (layer_x) memcpy(layer_x + (size_t)(l + 1) * R * d, x, R * d * sizeof(double));
    }

    /* Score head: s = w . (RMSNorm(x_last) * g_final), no decoding
     * (DuoLM summary page, 核心方法). */
    const float *gf = w[1 + (size_t)s.n_layers * W_PER_LAYER];
    const float *head = w[2 + (size_t)s.n_layers * W_PER_LAYER];
    double *h = malloc((size_t)d * sizeof(double));
    for (int oi = 0; oi < n_out; oi++) {
        oracle_rmsnorm(x + (size_t)out_rows[oi] * d, gf, d, s.rms_eps, h);
        double acc = 0.0;
        for (int c = 0; c < d; c++) acc += (double)head[c] * h[c];
        scores[oi] = acc;
        if (final_hidden) memcpy(final_hidden + (size_t)oi * d, h, d * sizeof(double));
    }
    free(h);
    free(x); free(nrm); free(q); free(k); free(v); free(o); free(g); free(u); free(y);
    return 0;
}
