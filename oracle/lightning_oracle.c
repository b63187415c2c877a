/*
 * Lightning Attention oracle: plain, slow, float64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or
 * calls this file; only the test suite, the smoke check and the bench's
 * CPU-baseline leg do. It shares no code, header or constant with the CUDA
 * library, and it reads its inputs exactly as the GPU does: bf16 bit
 * patterns or float32 values are widened to double without rounding, and
 * the per-head slopes are the same float32 numbers, widened.
 *
 * What is computed (per batch b, head h with decay slope s, length L):
 *
 *   o_i   = sum_{j<=i} e^{-s(i-j)} (q_i . k_j) v_j  +  e^{-s(i+1)} q_i S_in
 *   S_out = e^{-sL} S_in + sum_{j<L} e^{-s(L-1-j)} k_j^T v_j
 *
 * S_in is the carried-in state, read as the state "one position before the
 * first token". Source: "MINIMAX SIGNAL LAB · M1" (ailearn.mscapital.top),
 * §03 Lightning Attention: the intra-block term O_intra = [(Q K^T) ⊙ D] V
 * with D_ij = e^{-s_h(i-j)} 1[i>=j], the inter-block term
 * O_inter = (Q ⊙ d_q) S_{t-1}, the state update
 * S_t = e^{-s_h B} S_{t-1} + (K ⊙ d_k)^T V, the recursive fixed-size KV
 * state of the same section, and the last-short-block rule (a final block
 * of m < B tokens uses m). The pages print no values for d_q and d_k; the
 * readings used here are d_q[i] = e^{-s(i+1)}, d_k[j] = e^{-s(m-1-j)} and a
 * block decay of e^{-s m}: the only exponents for which the blockwise form
 * equals the token-level definition above (the tests check that equality
 * for every block size).
 *
 * Three forms, each written straight from its definition:
 *   F1 la_oracle_definition : the quadratic sum above, O(L^2 d) per head.
 *   F2 la_oracle_recurrence : token recurrence S_i = e^{-s} S_{i-1} + k_i^T v_i,
 *                             o_i = q_i S_i  (the "cumsum" form of naive
 *                             linear attention, fishai.com.cn article on
 *                             M1), O(L d^2) per head; the full-size oracle.
 *   F3 la_oracle_blockwise  : the block formulas of §03 for a given B.
 * plus la_oracle_decode, one recurrent step for a single new token,
 * la_oracle_snapshots, the state after every `interval` tokens (F2's state),
 * la_oracle_backward, the gradients of one prefill, la_oracle_norm_gate, the
 * normalisation and gating of the attention output, la_oracle_gqa_decode,
 * one decode step of the softmax attention layer of the hybrid model, and
 * la_oracle_gqa_prefill, the same layer over a run of new tokens.
 *
 * Layouts: q, k, v, o are [batch][heads][seq][dim] contiguous (o for decode
 * is [batch][heads][dim]); states are [batch][heads][dim(k)][dim(v)].
 * Parallelism: OpenMP over (batch, head) only (over output rows for the
 * softmax layer's prefill); the arithmetic inside one head or row is a plain
 * sequential loop.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* Widen one stored element to double. bf16 is the top half of a float32. */
static double widen(const void *base, int dtype, size_t idx) {
    if (dtype == ORACLE_BF16) {
        uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float *)base)[idx];
}

/* Copy one head's [seq][dim] slice into a double buffer. */
static void widen_head(const void *src, int dtype, size_t offset, size_t count, double *dst) {
    for (size_t n = 0; n < count; ++n) dst[n] = widen(src, dtype, offset + n);
}

static int check_args(const void *q, const void *k, const void *v, int dtype, const float *slopes,
                      int batch, int heads, int seq, int dim) {
    if (!q || !k || !v || !slopes) return 1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return 1;
    if (batch < 0 || heads <= 0 || seq < 0 || dim <= 0) return 1;
    return 0;
}

int la_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void la_oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* F1: the definition, term by term. */
int la_oracle_definition(const void *q, const void *k, const void *v, int dtype,
                         const float *slopes, int batch, int heads, int seq, int dim,
                         const float *state_in, double *o, double *state_out) {
    if (check_args(q, k, v, dtype, slopes, batch, heads, seq, dim) || !o) return 1;
    const long BH = (long)batch * heads;
    const size_t L = (size_t)seq, d = (size_t)dim;
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        const int h = (int)(bh % heads);
        const double s = (double)slopes[h];
        double *Q = malloc(sizeof(double) * L * d + 1);
        double *K = malloc(sizeof(double) * L * d + 1);
        double *V = malloc(sizeof(double) * L * d + 1);
        double *S0 = malloc(sizeof(double) * d * d);
        if (!Q || !K || !V || !S0) {
            fail = 1;
            free(Q); free(K); free(V); free(S0);
            continue;
        }
        widen_head(q, dtype, (size_t)bh * L * d, L * d, Q);
        widen_head(k, dtype, (size_t)bh * L * d, L * d, K);
        widen_head(v, dtype, (size_t)bh * L * d, L * d, V);
        for (size_t n = 0; n < d * d; ++n)
            S0[n] = state_in ? (double)state_in[(size_t)bh * d * d + n] : 0.0;
        double *O = o + (size_t)bh * L * d;
        for (size_t i = 0; i < L; ++i) {
            for (size_t c = 0; c < d; ++c) O[i * d + c] = 0.0;
            for (size_t j = 0; j <= i; ++j) {
                double qk = 0.0;
                for (size_t c = 0; c < d; ++c) qk += Q[i * d + c] * K[j * d + c];
                const double w = exp(-s * (double)(i - j)) * qk;
                for (size_t c = 0; c < d; ++c) O[i * d + c] += w * V[j * d + c];
            }
            /* carried-in state, seen from position i: i+1 steps of decay */
            const double dq = exp(-s * (double)(i + 1));
            for (size_t c = 0; c < d; ++c) {
                double acc = 0.0;
                for (size_t r = 0; r < d; ++r) acc += Q[i * d + r] * S0[r * d + c];
                O[i * d + c] += dq * acc;
            }
        }
        if (state_out) {
            double *S = state_out + (size_t)bh * d * d;
            const double dL = exp(-s * (double)L);
            for (size_t n = 0; n < d * d; ++n) S[n] = dL * S0[n];
            for (size_t j = 0; j < L; ++j) {
                const double w = exp(-s * (double)(L - 1 - j));
                for (size_t r = 0; r < d; ++r)
                    for (size_t c = 0; c < d; ++c) S[r * d + c] += w * K[j * d + r] * V[j * d + c];
            }
        }
        free(Q); free(K); free(V); free(S0);
    }
    return fail;
}

/* F2: token recurrence. S_i = e^{-s} S_{i-1} + k_i^T v_i ; o_i = q_i S_i. */
int la_oracle_recurrence(const void *q, const void *k, const void *v, int dtype,
                         const float *slopes, int batch, int heads, int seq, int dim,
                         const float *state_in, double *o, double *state_out) {
    if (check_args(q, k, v, dtype, slopes, batch, heads, seq, dim) || !o) return 1;
    const long BH = (long)batch * heads;
    const size_t L = (size_t)seq, d = (size_t)dim;
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        const int h = (int)(bh % heads);
        const double decay = exp(-(double)slopes[h]);
        double *S = malloc(sizeof(double) * d * d);
        double *qi = malloc(sizeof(double) * d), *ki = malloc(sizeof(double) * d),
               *vi = malloc(sizeof(double) * d);
        if (!S || !qi || !ki || !vi) {
            fail = 1;
            free(S); free(qi); free(ki); free(vi);
            continue;
        }
        for (size_t n = 0; n < d * d; ++n)
            S[n] = state_in ? (double)state_in[(size_t)bh * d * d + n] : 0.0;
        const size_t base = (size_t)bh * L * d;
        for (size_t i = 0; i < L; ++i) {
            widen_head(q, dtype, base + i * d, d, qi);
            widen_head(k, dtype, base + i * d, d, ki);
            widen_head(v, dtype, base + i * d, d, vi);
            for (size_t r = 0; r < d; ++r)
                for (size_t c = 0; c < d; ++c) S[r * d + c] = decay * S[r * d + c] + ki[r] * vi[c];
            double *oi = o + base + i * d;
            for (size_t c = 0; c < d; ++c) oi[c] = 0.0;
            for (size_t r = 0; r < d; ++r)
                for (size_t c = 0; c < d; ++c) oi[c] += qi[r] * S[r * d + c];
        }
        if (state_out) memcpy(state_out + (size_t)bh * d * d, S, sizeof(double) * d * d);
        free(S); free(qi); free(ki); free(vi);
    }
    return fail;
}

/* State snapshots: the state after the first (n+1)*interval tokens, for
 * n = 0 .. seq/interval - 1, by the same token recurrence as F2
 * (S_i = e^{-s} S_{i-1} + k_i^T v_i, starting from S_in). These are the
 * states a prefix cache stores ("MINIMAX SIGNAL LAB · M1", §03 Lightning
 * Attention: the recursive fixed-size state, and the page's note on prefix
 * caching and speculative decoding with such states).
 * snapshots: [batch][heads][seq/interval][dim][dim] float64. */
int la_oracle_snapshots(const void *k, const void *v, int dtype, const float *slopes, int batch,
                        int heads, int seq, int dim, const float *state_in, int interval,
                        double *snapshots) {
    if (!k || !v || !slopes || !snapshots) return 1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return 1;
    if (batch < 0 || heads <= 0 || seq < 0 || dim <= 0 || interval <= 0) return 1;
    const long BH = (long)batch * heads;
    const size_t L = (size_t)seq, d = (size_t)dim, count = (size_t)(seq / interval);
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        const int h = (int)(bh % heads);
        const double decay = exp(-(double)slopes[h]);
        double *S = malloc(sizeof(double) * d * d);
        double *ki = malloc(sizeof(double) * d), *vi = malloc(sizeof(double) * d);
        if (!S || !ki || !vi) {
            fail = 1;
            free(S); free(ki); free(vi);
            continue;
        }
        for (size_t n = 0; n < d * d; ++n)
            S[n] = state_in ? (double)state_in[(size_t)bh * d * d + n] : 0.0;
        const size_t base = (size_t)bh * L * d;
        for (size_t i = 0; i < L; ++i) {
            widen_head(k, dtype, base + i * d, d, ki);
            widen_head(v, dtype, base + i * d, d, vi);
            for (size_t r = 0; r < d; ++r)
                for (size_t c = 0; c < d; ++c) S[r * d + c] = decay * S[r * d + c] + ki[r] * vi[c];
            if ((i + 1) % (size_t)interval == 0) {
                const size_t n = (i + 1) / (size_t)interval - 1;
                memcpy(snapshots + ((size_t)bh * count + n) * d * d, S, sizeof(double) * d * d);
            }
        }
        free(S); free(ki); free(vi);
    }
    return fail;
}

/* Gradients of one prefill, for training through the layer. With the loss
 * l = sum_i dO_i . o_i + sum dS_out * S_out, and S_i the state after token i
 * (S_i = e^{-s} S_{i-1} + k_i^T v_i from S_{-1} = S_in, so o_i = q_i S_i and
 * S_out = S_{L-1}):
 *   dq_i = dO_i S_i^T
 *   R_j  = q_j^T dO_j + e^{-s} R_{j+1},  R_{L-1} = q_{L-1}^T dO_{L-1} + dS_out
 *          (R_j = d l / d S_j: everything token j's outer product k_j^T v_j
 *          feeds, each later token i seen with e^{-s(i-j)})
 *   dk_j = R_j v_j,  dv_j = R_j^T k_j
 *   dS_in = e^{-s} R_0  (= dS_out when L = 0)
 * Derived from the token-level definition of the forward result
 * ("MINIMAX SIGNAL LAB · M1", §03 Lightning Attention); the pages print no
 * backward pass. d_o has the dtype of q, k, v; d_state_out (may be NULL:
 * zero) and state_in (NULL: zero) are float32; outputs are float64, and
 * d_state_in may be NULL. */
int la_oracle_backward(const void *q, const void *k, const void *v, const void *d_o, int dtype,
                       const float *slopes, int batch, int heads, int seq, int dim,
                       const float *state_in, const float *d_state_out, double *dq, double *dk,
                       double *dv, double *d_state_in) {
    if (check_args(q, k, v, dtype, slopes, batch, heads, seq, dim)) return 1;
    if (!d_o || !dq || !dk || !dv) return 1;
    const long BH = (long)batch * heads;
    const size_t L = (size_t)seq, d = (size_t)dim;
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        const int h = (int)(bh % heads);
        const double decay = exp(-(double)slopes[h]);
        double *S = malloc(sizeof(double) * d * d);
        double *R = malloc(sizeof(double) * d * d);
        double *Q = malloc(sizeof(double) * L * d + 1), *K = malloc(sizeof(double) * L * d + 1);
        double *V = malloc(sizeof(double) * L * d + 1), *G = malloc(sizeof(double) * L * d + 1);
        if (!S || !R || !Q || !K || !V || !G) {
            fail = 1;
            free(S); free(R); free(Q); free(K); free(V); free(G);
            continue;
        }
        const size_t base = (size_t)bh * L * d;
        widen_head(q, dtype, base, L * d, Q);
        widen_head(k, dtype, base, L * d, K);
        widen_head(v, dtype, base, L * d, V);
        widen_head(d_o, dtype, base, L * d, G);
        /* forward sweep: S_i, then dq_i = dO_i S_i^T */
        for (size_t n = 0; n < d * d; ++n)
            S[n] = state_in ? (double)state_in[(size_t)bh * d * d + n] : 0.0;
        for (size_t i = 0; i < L; ++i) {
            for (size_t r = 0; r < d; ++r)
                for (size_t c = 0; c < d; ++c) S[r * d + c] = decay * S[r * d + c] + K[i * d + r] * V[i * d + c];
            for (size_t r = 0; r < d; ++r) {
                double acc = 0.0;
                for (size_t c = 0; c < d; ++c) acc += G[i * d + c] * S[r * d + c];
                dq[base + i * d + r] = acc;
            }
        }
        /* backward sweep: R_j, then dk_j = R_j v_j and dv_j = R_j^T k_j */
        for (size_t n = 0; n < d * d; ++n)
            R[n] = d_state_out ? (double)d_state_out[(size_t)bh * d * d + n] : 0.0;
        for (size_t jj = L; jj-- > 0;) {
            const double carry = (jj + 1 == L) ? 1.0 : decay;  /* dS_out joins at the last token */
            for (size_t r = 0; r < d; ++r)
                for (size_t c = 0; c < d; ++c) R[r * d + c] = carry * R[r * d + c] + Q[jj * d + r] * G[jj * d + c];
            for (size_t r = 0; r < d; ++r) {
                double acc = 0.0;
                for (size_t c = 0; c < d; ++c) acc += R[r * d + c] * V[jj * d + c];
                dk[base + jj * d + r] = acc;
            }
            for (size_t c = 0; c < d; ++c) {
                double acc = 0.0;
                for (size_t r = 0; r < d; ++r) acc += K[jj * d + r] * R[r * d + c];
                dv[base + jj * d + c] = acc;
            }
        }
        if (d_state_in) {
            const double f = L > 0 ? decay : 1.0;
            for (size_t n = 0; n < d * d; ++n) d_state_in[(size_t)bh * d * d + n] = f * R[n];
        }
        free(S); free(R); free(Q); free(K); free(V); free(G);
    }
    return fail;
}

/* Normalisation and gating of the attention output. "MINIMAX SIGNAL LAB ·
 * M1", §03 Lightning Attention: the figure adds the intra- and inter-block
 * outputs, then normalises and gates them; the pages print no formula. The
 * reading taken: an RMS normalisation with a learned per-channel weight, then
 * an elementwise sigmoid gate,
 *   y[b][l][n] = gamma[n] * x[n] / sqrt(mean_{n' in group(n)} x[n']^2 + eps)
 *                * 1 / (1 + e^{-g[b][l][n]})
 * over the token's channels n = h*dim + c, x[n] = o[b][h][l][c]; the RMS is
 * taken per head (group = the head's dim channels, per_head = 1) or over all
 * heads*dim channels of the token (per_head = 0).
 * o: [batch][heads][seq][dim]; g and y: [batch][seq][heads*dim]; gamma:
 * [heads*dim] float32; o and g have one dtype; y is float64. */
int la_oracle_norm_gate(const void *o, const void *g, int dtype, const float *gamma, double eps, int batch,
                        int heads, int seq, int dim, int per_head, double *y) {
    if (!o || !g || !gamma || !y) return 1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return 1;
    if (batch < 0 || heads <= 0 || seq < 0 || dim <= 0 || eps < 0.0) return 1;
    const size_t N = (size_t)heads * dim, L = (size_t)seq, d = (size_t)dim;
    const long T = (long)batch * seq;
#pragma omp parallel for schedule(static)
    for (long tk = 0; tk < T; ++tk) {
        const size_t b = (size_t)tk / L, l = (size_t)tk % L;
        const size_t group = per_head ? d : N;
        for (size_t g0 = 0; g0 < N; g0 += group) {
            double ss = 0.0;
            for (size_t n = g0; n < g0 + group; ++n) {
                const double x = widen(o, dtype, ((b * heads + n / d) * L + l) * d + n % d);
                ss += x * x;
            }
            const double inv = 1.0 / sqrt(ss / (double)group + eps);
            for (size_t n = g0; n < g0 + group; ++n) {
                const double x = widen(o, dtype, ((b * heads + n / d) * L + l) * d + n % d);
                const double gv = widen(g, dtype, (size_t)tk * N + n);
                y[(size_t)tk * N + n] = (double)gamma[n] * x * inv / (1.0 + exp(-gv));
            }
        }
    }
    return 0;
}

/* Rotary position embedding on the first `rot` dims of a head, rotate-half
 * pairing: for i < rot/2 the pair (x[i], x[i + rot/2]) turns by pos * theta_i,
 * theta_i = base^{-2i/rot}; dims from rot on are unchanged. */
static void rope_head(const double *x, double *out, int dim, int rot, double base, long pos) {
    const int half = rot / 2;
    for (int c = 0; c < dim; ++c) out[c] = x[c];
    for (int i = 0; i < half; ++i) {
        const double ang = (double)pos * pow(base, -2.0 * i / (double)rot);
        const double cs = cos(ang), sn = sin(ang);
        out[i] = x[i] * cs - x[i + half] * sn;
        out[i + half] = x[i + half] * cs + x[i] * sn;
    }
}

/* One decode step of the softmax attention layer that M1 places after every
 * seven Lightning layers ("MINIMAX SIGNAL LAB · M1", §02: 64 query heads x 128,
 * softmax K/V 8 x 128, RoPE on 64 of the 128 dims in the softmax layers only;
 * §04: the softmax layers keep a bf16 KV cache that grows with the context).
 * Readings (the pages print no formula): grouped-query attention, query head
 * h reads KV head h / (heads / kv_heads); scores scaled by `scale`; RoPE as in
 * rope_head with the token's position; the cache holds rotated keys.
 * Per sequence b the new token sits at position pos[b]: its key (rotated) and
 * value join the cache there, and each query head attends to positions
 * 0 .. pos[b]:  o = sum_p softmax_p(scale * rope(q) . k_p) v_p.
 * q: [batch][heads][dim]; k_new, v_new: [batch][kv_heads][dim]; caches:
 * [batch][kv_heads][cap][dim] with positions < pos[b] filled; o: float64
 * [batch][heads][dim]. All inputs share `dtype`. */
int la_oracle_gqa_decode(const void *q, const void *k_new, const void *v_new, const void *k_cache,
                         const void *v_cache, int dtype, const int *pos, int batch, int heads, int kv_heads,
                         int dim, int cap, int rot, double base, double scale, double *o) {
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !o) return 1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return 1;
    if (batch < 0 || kv_heads <= 0 || heads % kv_heads != 0 || dim <= 0 || rot < 0 || rot > dim || rot % 2)
        return 1;
    for (int b = 0; b < batch; ++b)
        if (pos[b] < 0 || pos[b] >= cap) return 1;
    const int group = heads / kv_heads;
    const size_t d = (size_t)dim;
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)batch * heads; ++bh) {
        const int b = (int)(bh / heads), h = (int)(bh % heads), hk = h / group;
        const long P = pos[b];
        double *x = malloc(sizeof(double) * d * 4), *sc = malloc(sizeof(double) * (size_t)(P + 1));
        if (!x || !sc) {
            fail = 1;
            free(x); free(sc);
            continue;
        }
        double *qr = x, *kr = x + d, *tmp = x + 2 * d, *acc = x + 3 * d;
        for (size_t c = 0; c < d; ++c) tmp[c] = widen(q, dtype, (size_t)bh * d + c);
        rope_head(tmp, qr, dim, rot, base, P);
        const size_t kv = (size_t)b * kv_heads + hk;
        double mx = -INFINITY;
        for (long p = 0; p <= P; ++p) {
            if (p < P) {
                for (size_t c = 0; c < d; ++c) kr[c] = widen(k_cache, dtype, (kv * cap + p) * d + c);
            } else {
                for (size_t c = 0; c < d; ++c) tmp[c] = widen(k_new, dtype, kv * d + c);
                rope_head(tmp, kr, dim, rot, base, P);
            }
            double dot = 0.0;
            for (size_t c = 0; c < d; ++c) dot += qr[c] * kr[c];
            sc[p] = scale * dot;
            if (sc[p] > mx) mx = sc[p];
        }
        double den = 0.0;
        for (size_t c = 0; c < d; ++c) acc[c] = 0.0;
        for (long p = 0; p <= P; ++p) {
            const double w = exp(sc[p] - mx);
            den += w;
            for (size_t c = 0; c < d; ++c)
                acc[c] += w * (p < P ? widen(v_cache, dtype, (kv * cap + p) * d + c) : widen(v_new, dtype, kv * d + c));
        }
        for (size_t c = 0; c < d; ++c) o[(size_t)bh * d + c] = acc[c] / den;
        free(x); free(sc);
    }
    return fail;
}

/* F3: the blockwise method, block by block, as the block formulas state it. */
int la_oracle_blockwise(const void *q, const void *k, const void *v, int dtype,
                        const float *slopes, int batch, int heads, int seq, int dim, int block,
                        const float *state_in, double *o, double *state_out) {
    if (check_args(q, k, v, dtype, slopes, batch, heads, seq, dim) || !o || block <= 0) return 1;
    const long BH = (long)batch * heads;
    const size_t L = (size_t)seq, d = (size_t)dim, B = (size_t)block;
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        const int h = (int)(bh % heads);
        const double s = (double)slopes[h];
        double *S = malloc(sizeof(double) * d * d);     /* S_{t-1} */
        double *Sn = malloc(sizeof(double) * d * d);    /* S_t     */
        double *Qt = malloc(sizeof(double) * B * d), *Kt = malloc(sizeof(double) * B * d),
               *Vt = malloc(sizeof(double) * B * d), *P = malloc(sizeof(double) * B * B);
        if (!S || !Sn || !Qt || !Kt || !Vt || !P) {
            fail = 1;
            free(S); free(Sn); free(Qt); free(Kt); free(Vt); free(P);
            continue;
        }
        for (size_t n = 0; n < d * d; ++n)
            S[n] = state_in ? (double)state_in[(size_t)bh * d * d + n] : 0.0;
        const size_t base = (size_t)bh * L * d;
        for (size_t t0 = 0; t0 < L; t0 += B) {
            const size_t m = (L - t0 < B) ? (L - t0) : B; /* last block: actual length m */
            widen_head(q, dtype, base + t0 * d, m * d, Qt);
            widen_head(k, dtype, base + t0 * d, m * d, Kt);
            widen_head(v, dtype, base + t0 * d, m * d, Vt);
            /* P = (Q_t K_t^T) ⊙ D,  D_ij = e^{-s(i-j)} 1[i>=j] */
            for (size_t i = 0; i < m; ++i)
                for (size_t j = 0; j < m; ++j) {
                    double qk = 0.0;
                    for (size_t c = 0; c < d; ++c) qk += Qt[i * d + c] * Kt[j * d + c];
                    const double D = (i >= j) ? exp(-s * (double)(i - j)) : 0.0;
                    P[i * B + j] = qk * D;
                }
            double *Ot = o + base + t0 * d;
            for (size_t i = 0; i < m; ++i) {
                const double dq = exp(-s * (double)(i + 1)); /* query decay d_q[i] */
                for (size_t c = 0; c < d; ++c) {
                    double intra = 0.0, inter = 0.0;
                    for (size_t j = 0; j < m; ++j) intra += P[i * B + j] * Vt[j * d + c];
                    for (size_t r = 0; r < d; ++r) inter += (Qt[i * d + r] * dq) * S[r * d + c];
                    Ot[i * d + c] = intra + inter;
                }
            }
            /* S_t = e^{-s m} S_{t-1} + (K_t ⊙ d_k)^T V_t,  d_k[j] = e^{-s(m-1-j)} */
            const double dblock = exp(-s * (double)m);
            for (size_t r = 0; r < d; ++r)
                for (size_t c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (size_t j = 0; j < m; ++j)
                        acc += (Kt[j * d + r] * exp(-s * (double)(m - 1 - j))) * Vt[j * d + c];
                    Sn[r * d + c] = dblock * S[r * d + c] + acc;
                }
            double *tmp = S; S = Sn; Sn = tmp;
        }
        if (state_out) memcpy(state_out + (size_t)bh * d * d, S, sizeof(double) * d * d);
        free(S); free(Sn); free(Qt); free(Kt); free(Vt); free(P);
    }
    return fail;
}

/* One recurrent step for a single new token per (batch, head):
 * S <- e^{-s} S + k^T v, then o = q S (the new token is seen with e^0 = 1).
 * q, k, v: [batch][heads][dim]; state: [batch][heads][dim][dim] float64, in/out. */
int la_oracle_decode(const void *q, const void *k, const void *v, int dtype, const float *slopes,
                     int batch, int heads, int dim, double *state, double *o) {
    if (check_args(q, k, v, dtype, slopes, batch, heads, 1, dim) || !state || !o) return 1;
    const long BH = (long)batch * heads;
    const size_t d = (size_t)dim;
#pragma omp parallel for schedule(static)
    for (long bh = 0; bh < BH; ++bh) {
        const int h = (int)(bh % heads);
        const double decay = exp(-(double)slopes[h]);
        double *S = state + (size_t)bh * d * d;
        const size_t base = (size_t)bh * d;
        for (size_t r = 0; r < d; ++r) {
            const double kr = widen(k, dtype, base + r);
            for (size_t c = 0; c < d; ++c)
                S[r * d + c] = decay * S[r * d + c] + kr * widen(v, dtype, base + c);
        }
        double *oi = o + base;
        for (size_t c = 0; c < d; ++c) oi[c] = 0.0;
        for (size_t r = 0; r < d; ++r) {
            const double qr = widen(q, dtype, base + r);
            for (size_t c = 0; c < d; ++c) oi[c] += qr * S[r * d + c];
        }
    }
    return 0;
}

/* The softmax GQA layer over a run of `seq` new tokens per sequence, at
 * positions start .. start+seq-1 (§02 and §04 of "MINIMAX SIGNAL LAB · M1" as
 * for la_oracle_gqa_decode, whose readings this follows: query head h reads
 * KV head h / (heads / kv_heads), rotate-half RoPE on the first `rot` dims at
 * the token's position, scores scaled by `scale`, causal order). Token i of
 * sequence b, query head h, sits at position P = start + i and attends to
 * every position p <= P:
 *   o = sum_{p <= P} softmax_p(scale * rope(q_i, P) . key_p) val_p,
 *   key_p = k_cache[p] (already rotated), val_p = v_cache[p]          for p < start,
 *   key_p = rope(k_new[p - start], p), val_p = v_new[p - start]        for p >= start.
 * q: [batch][heads][seq][dim]; k_new, v_new: [batch][kv_heads][seq][dim];
 * caches: [batch][kv_heads][cap][dim] with positions < start filled. All
 * inputs share `dtype`. rows: the outputs to compute, as indices
 * (b * heads + h) * seq + i, or NULL for all batch*heads*seq of them in that
 * order; o: float64 [nrows][dim]. The angles are those of rope_head. */
int la_oracle_gqa_prefill(const void *q, const void *k_new, const void *v_new, const void *k_cache,
                          const void *v_cache, int dtype, int start, int batch, int heads, int kv_heads, int seq,
                          int dim, int cap, int rot, double base, double scale, const long long *rows,
                          long long nrows, double *o) {
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !o) return 1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return 1;
    if (batch < 0 || seq < 0 || start < 0 || kv_heads <= 0 || heads % kv_heads != 0 || dim <= 0 || rot < 0 ||
        rot > dim || rot % 2 || (long long)start + seq > cap)
        return 1;
    const long long total = (long long)batch * heads * seq;
    if (!rows) nrows = total;
    if (nrows < 0) return 1;
    for (long long n = 0; rows && n < nrows; ++n)
        if (rows[n] < 0 || rows[n] >= total) return 1;
    const int group = heads / kv_heads, half = rot / 2;
    const size_t d = (size_t)dim;
    /* cos and sin of every new position's angles, as rope_head takes them */
    double *cs = malloc(sizeof(double) * ((size_t)seq * half + 1)), *sn = malloc(sizeof(double) * ((size_t)seq * half + 1));
    if (!cs || !sn) {
        free(cs); free(sn);
        return 1;
    }
    for (int i = 0; i < seq; ++i)
        for (int c = 0; c < half; ++c) {
            const double ang = (double)(start + i) * pow(base, -2.0 * c / (double)rot);
            cs[(size_t)i * half + c] = cos(ang);
            sn[(size_t)i * half + c] = sin(ang);
        }
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long n = 0; n < nrows; ++n) {
        const long long r = rows ? rows[n] : n;
        const int i = (int)(r % seq), h = (int)((r / seq) % heads), b = (int)(r / ((long long)seq * heads));
        const size_t kv = (size_t)b * kv_heads + h / group;
        const long P = (long)start + i;
        double *x = malloc(sizeof(double) * d * 4), *sc = malloc(sizeof(double) * (size_t)(P + 1));
        if (!x || !sc) {
            fail = 1;
            free(x); free(sc);
            continue;
        }
        double *qr = x, *kr = x + d, *tmp = x + 2 * d, *acc = x + 3 * d;
        /* rotate a head row given at tmp by the angles of new token t into out */
#define ROPE_NEW(out, t)                                                                  \
        do {                                                                              \
            for (size_t c_ = 0; c_ < d; ++c_) (out)[c_] = tmp[c_];                        \
            for (int c_ = 0; c_ < half; ++c_) {                                           \
                const double cv = cs[(size_t)(t) * half + c_], sv = sn[(size_t)(t) * half + c_]; \
                (out)[c_] = tmp[c_] * cv - tmp[c_ + half] * sv;                           \
                (out)[c_ + half] = tmp[c_ + half] * cv + tmp[c_] * sv;                    \
            }                                                                             \
        } while (0)
        for (size_t c = 0; c < d; ++c) tmp[c] = widen(q, dtype, (size_t)r * d + c);
        ROPE_NEW(qr, i);
        double mx = -INFINITY;
        for (long p = 0; p <= P; ++p) {
            if (p < start) {
                for (size_t c = 0; c < d; ++c) kr[c] = widen(k_cache, dtype, (kv * cap + p) * d + c);
            } else {
                for (size_t c = 0; c < d; ++c) tmp[c] = widen(k_new, dtype, (kv * seq + (p - start)) * d + c);
                ROPE_NEW(kr, p - start);
            }
            double dot = 0.0;
            for (size_t c = 0; c < d; ++c) dot += qr[c] * kr[c];
            sc[p] = scale * dot;
            if (sc[p] > mx) mx = sc[p];
        }
#undef ROPE_NEW
        double den = 0.0;
        for (size_t c = 0; c < d; ++c) acc[c] = 0.0;
        for (long p = 0; p <= P; ++p) {
            const double w = exp(sc[p] - mx);
            den += w;
            for (size_t c = 0; c < d; ++c)
                acc[c] += w * (p < start ? widen(v_cache, dtype, (kv * cap + p) * d + c)
                                         : widen(v_new, dtype, (kv * seq + (p - start)) * d + c));
        }
        for (size_t c = 0; c < d; ++c) o[(size_t)n * d + c] = acc[c] / den;
        free(x); free(sc);
    }
    free(cs); free(sn);
    return fail;
}
