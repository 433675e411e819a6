/*
 * CPU oracle for one decode step of a Llama-style decoder.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline arm may load this library. The product path (the
 * CUDA library and its Python binding) never calls it, and the two share no
 * code: no headers, helpers, tables or constants.
 *
 * What it computes. The megakernel write-ups ("Look Ma, No Bubbles" and its
 * summaries, sections "Megakernel: The Core Solution" and "Fusing Operations
 * with an On-GPU Interpreter") run the whole Llama-3.2-1B forward for one new
 * token as a sequence of fused instructions: RMSNorm + QKV + RoPE, attention,
 * O-projection, RMSNorm + gate/up + SiLU, down-projection, final norm + LM
 * head. Fusion reorders work but does not approximate, so the oracle is the
 * plain definition of that forward, written out step by step:
 *
 *   x   = E[token]                                   (bf16 row, as fp32)
 *   per layer:
 *     xn  = (x_i * r) * w_i,  r = 1/sqrt(mean(x^2) + eps)
 *     q,k,v = W_q xn, W_k xn, W_v xn                 (fp32 dot products)
 *     RoPE on q and k (rotate-half pairs (i, i+d/2))
 *     k, v rounded to bf16 and stored in cache slot `pos`            [KV]
 *     attn_h = softmax(q_h . K_g / sqrt(d)) V_g,  g = h / group
 *     x   = x + W_o attn
 *     xn  = rmsnorm(x) with the MLP norm
 *     h   = silu(W_g xn) * (W_u xn)
 *     x   = x + W_d h
 *   logits = E . (rmsnorm(x) with the final norm)
 *
 * Precision: fp32 arithmetic over the bf16 weights and the bf16 KV cache.
 * Activations stay fp32 between steps; the one rounding to bf16 (round to
 * nearest, ties to even) is where the data format forces it: the key and value
 * written to the bf16 cache [KV]. Every sum runs in plain index order. Where
 * the write-ups are silent this follows the plainest reading: fp32 activations,
 * rotate-half RoPE pairs (i, i + d/2) with inverse frequencies theta^(-2i/d)
 * and no frequency scaling, and the new token at position p attending to keys
 * 0..p, its own included.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math, so
 * no reassociation and no fused multiply-add).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- bf16 <-> fp32, from the bit layout (bf16 = top 16 bits of fp32) ---- */

static float bf2f(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint16_t f2bf(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u)          /* NaN: keep it a quiet NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    /* round to nearest, ties to even: add 0x7fff plus the lowest kept bit */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

void orc_round_bf16(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = f2bf(in[i]);
}

void orc_bf16_to_f32(const uint16_t* in, float* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf2f(in[i]);
}

/* ---- RMSNorm: eps inside the root, weight applied after scaling ---- */

void orc_rmsnorm(const float* x, const uint16_t* w, int n, float eps, float* out) {
    float ss = 0.0f;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    float r = 1.0f / sqrtf(ss / (float)n + eps);
    for (int i = 0; i < n; ++i) out[i] = (x[i] * r) * bf2f(w[i]);
}

/* ---- RoPE, rotate-half pairing (i, i + d/2), plain theta^(-2i/d) ----
 * The angle pos * theta^(-2i/d) is formed in double and its cosine and sine
 * are then cast to float; the rotation itself is fp32. */

void orc_rope(float* v, int d, int pos, double theta) {
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double inv_freq = pow(theta, -(2.0 * (double)i) / (double)d);
        double ang = (double)pos * inv_freq;
        float c = (float)cos(ang), s = (float)sin(ang);
        float a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

/* ---- y = W x, W bf16 [rows][cols] row-major, x and y fp32 ---- */

void orc_matvec(const uint16_t* W, const float* x, int rows, int cols, float* y, int threads) {
#pragma omp parallel for schedule(static) num_threads(threads > 0 ? threads : 1)
    for (int r = 0; r < rows; ++r) {
        const uint16_t* wr = W + (size_t)r * (size_t)cols;
        float acc = 0.0f;
        for (int k = 0; k < cols; ++k) acc += bf2f(wr[k]) * x[k];
        y[r] = acc;
    }
}

/* ---- decode attention for one sequence and one layer ----
 * q: fp32 [nq][d]; K, V: bf16 [nkv][seq_stride][d], keys 0..n_keys-1 valid.
 * Query head h reads KV head h / (nq / nkv). Scale 1/sqrt(d) in fp32.
 * out: fp32 [nq][d]. */

void orc_attention(const float* q, const uint16_t* K, const uint16_t* V, int nq, int nkv,
                   int d, int n_keys, int seq_stride, float* out) {
    int group = nq / nkv;
    float scale = 1.0f / sqrtf((float)d);
    float* s = (float*)malloc(sizeof(float) * (size_t)(n_keys > 0 ? n_keys : 1));
    for (int h = 0; h < nq; ++h) {
        int g = h / group;
        const float* qh = q + (size_t)h * d;
        const uint16_t* Kg = K + (size_t)g * seq_stride * d;
        const uint16_t* Vg = V + (size_t)g * seq_stride * d;
        float* o = out + (size_t)h * d;
        float m = -INFINITY;
        for (int j = 0; j < n_keys; ++j) {
            float dot = 0.0f;
            for (int i = 0; i < d; ++i) dot += qh[i] * bf2f(Kg[(size_t)j * d + i]);
            s[j] = dot * scale;
            if (s[j] > m) m = s[j];
        }
        float l = 0.0f;
        for (int j = 0; j < n_keys; ++j) {
            s[j] = expf(s[j] - m);
            l += s[j];
        }
        for (int i = 0; i < d; ++i) o[i] = 0.0f;
        for (int j = 0; j < n_keys; ++j)
            for (int i = 0; i < d; ++i) o[i] += s[j] * bf2f(Vg[(size_t)j * d + i]);
        for (int i = 0; i < d; ++i) o[i] = o[i] / l;
    }
    free(s);
}

/* ---- SiLU-gated product: h = (g / (1 + exp(-g))) * u ---- */

void orc_silu_mul(const float* g, const float* u, int n, float* out) {
    for (int i = 0; i < n; ++i) out[i] = (g[i] / (1.0f + expf(-g[i]))) * u[i];
}

/* ---- greedy choice: largest logit, lowest index on ties ---- */

int orc_argmax(const float* x, int n) {
    int best = 0;
    for (int i = 1; i < n; ++i)
        if (x[i] > x[best]) best = i;
    return best;
}

/* ---- the whole decode step ---- */

typedef struct {
    int n_layers, hidden, n_heads, n_kv_heads, head_dim, ffn, vocab;
    float rms_eps;
    double rope_theta;
    /* bf16 host arrays, row-major [out][in]; per-layer arrays hold n_layers pointers */
    const uint16_t* embed;
    const uint16_t* const* attn_norm;
    const uint16_t* const* wq;
    const uint16_t* const* wk;
    const uint16_t* const* wv;
    const uint16_t* const* wo;
    const uint16_t* const* mlp_norm;
    const uint16_t* const* wgate;
    const uint16_t* const* wup;
    const uint16_t* const* wdown;
    const uint16_t* final_norm;
    const uint16_t* lm_head; /* NULL: tied to embed */
} orc_model;

/* tokens, positions: [batch]. k_cache, v_cache: bf16
 * [n_layers][batch][n_kv_heads][max_seq][head_dim]; slot positions[b] of
 * sequence b is written, slots 0..positions[b] are read. logits: fp32
 * [batch][vocab]. Returns 0, or -1 on a token or position out of range (then
 * nothing is written). */
int orc_decode_step(const orc_model* m, int batch, const int32_t* tokens,
                    const int32_t* positions, uint16_t* k_cache, uint16_t* v_cache,
                    int max_seq, float* logits, int threads) {
    const int H = m->hidden, d = m->head_dim, nq = m->n_heads, nkv = m->n_kv_heads;
    const int Q = nq * d, KV = nkv * d, F = m->ffn, V = m->vocab;
    for (int b = 0; b < batch; ++b)
        if (tokens[b] < 0 || tokens[b] >= V || positions[b] < 0 || positions[b] >= max_seq)
            return -1;

    float* x = (float*)malloc(4 * (size_t)H);
    float* xn = (float*)malloc(4 * (size_t)H);
    float* q = (float*)malloc(4 * (size_t)Q);
    float* kf = (float*)malloc(4 * (size_t)KV);
    float* vf = (float*)malloc(4 * (size_t)KV);
    float* attn = (float*)malloc(4 * (size_t)Q);
    float* y = (float*)malloc(4 * (size_t)(H > F ? H : F));
    float* g = (float*)malloc(4 * (size_t)F);
    float* u = (float*)malloc(4 * (size_t)F);
    float* hb = (float*)malloc(4 * (size_t)F);
    const size_t slot_stride = (size_t)max_seq * d;             /* one kv head */
    const size_t seq_stride = (size_t)nkv * slot_stride;        /* one sequence */
    const size_t layer_stride = (size_t)batch * seq_stride;     /* one layer */

    for (int b = 0; b < batch; ++b) {
        const int pos = positions[b];
        orc_bf16_to_f32(m->embed + (size_t)tokens[b] * H, x, H);
        for (int l = 0; l < m->n_layers; ++l) {
            uint16_t* Kl = k_cache + (size_t)l * layer_stride + (size_t)b * seq_stride;
            uint16_t* Vl = v_cache + (size_t)l * layer_stride + (size_t)b * seq_stride;
            /* attention block */
            orc_rmsnorm(x, m->attn_norm[l], H, m->rms_eps, xn);
            orc_matvec(m->wq[l], xn, Q, H, q, threads);
            orc_matvec(m->wk[l], xn, KV, H, kf, threads);
            orc_matvec(m->wv[l], xn, KV, H, vf, threads);
            for (int h = 0; h < nq; ++h) orc_rope(q + (size_t)h * d, d, pos, m->rope_theta);
            for (int h = 0; h < nkv; ++h) orc_rope(kf + (size_t)h * d, d, pos, m->rope_theta);
            for (int h = 0; h < nkv; ++h) {   /* [KV]: the only rounding to bf16 */
                orc_round_bf16(kf + (size_t)h * d, Kl + (size_t)h * slot_stride + (size_t)pos * d, d);
                orc_round_bf16(vf + (size_t)h * d, Vl + (size_t)h * slot_stride + (size_t)pos * d, d);
            }
            orc_attention(q, Kl, Vl, nq, nkv, d, pos + 1, max_seq, attn);
            orc_matvec(m->wo[l], attn, H, Q, y, threads);
            for (int i = 0; i < H; ++i) x[i] += y[i];
            /* MLP block */
            orc_rmsnorm(x, m->mlp_norm[l], H, m->rms_eps, xn);
            orc_matvec(m->wgate[l], xn, F, H, g, threads);
            orc_matvec(m->wup[l], xn, F, H, u, threads);
            orc_silu_mul(g, u, F, hb);
            orc_matvec(m->wdown[l], hb, H, F, y, threads);
            for (int i = 0; i < H; ++i) x[i] += y[i];
        }
        orc_rmsnorm(x, m->final_norm, H, m->rms_eps, xn);
        orc_matvec(m->lm_head ? m->lm_head : m->embed, xn, V, H, logits + (size_t)b * V, threads);
    }
    free(x); free(xn); free(q); free(kf); free(vf); free(attn);
    free(y); free(g); free(u); free(hb);
    return 0;
}

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
