/*
 * CPU oracle for causal linear attention (Lightning Attention), fp64.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library calls, links or
 * includes this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline / reference arm load it. It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What is computed (the plain definition, no decay, no feature map, no
 * normaliser; the decay variant and the feature map are at the end):
 *
 *     O_t = q_t . S0  +  sum_{s in seq(t), s <= t} (q_t . k_s) v_s
 *
 * where S0 is an optional carried-in d x d state (zero by default). This is the
 * causal linear attention of the page "MiniMax-01 Lightning Attention", section
 * "Lightning Attention 设计" (linear attention whose causal cumsum is the
 * obstacle the tiling removes). Every function below reaches this result;
 * they differ only in how the sums are associated:
 *
 *   oracle_quadratic  - the masked left product over the whole sequence,
 *                       (tril(Q K^T)) V, O(n^2 d);
 *   oracle_recurrent  - the token-by-token state form S += k^T v, o = q S
 *                       ("inference only updates the KV state recurrently,
 *                       O(d^2) per token", same section);
 *   oracle_blocked    - the pages' block decomposition: inside a block of B
 *                       tokens the left product with a causal mask, across
 *                       blocks the right product Q_b . KV with KV += K_b^T V_b
 *                       (same section, and page "首个线性注意力架构的大模型来了…",
 *                       section "4.1 创新的线性注意力", 序列划分 / 双阶段计算);
 *   oracle_state      - the final state sum_s k_s^T v_s (+ S0) per sequence;
 *   oracle_decode_step- one recurrent step on a batch of states;
 *   oracle_backward   - the gradients of L = sum_t dO_t . O_t with respect to
 *                       q, k, v and S0 (the training pass; the pages give the
 *                       forward only, so this is the calculus of the forward
 *                       definition above, written out);
 *   oracle_decay_*    - the same forms with a per-head decay on the state (an
 *                       extension the pages do not give; defined further down),
 *                       and their gradients;
 *   oracle_feature_map- the feature map phi one page gives, elementwise.
 *
 * Layout (all row-major, innermost index fastest):
 *   q, k, v, o   : [T][H][d]      tokens of all sequences packed back to back
 *   cu_seqlens   : int32 [nseq+1], cu_seqlens[0] = 0, non-decreasing, last = T
 *   init, state  : [nseq][H][d][d], element [i][j] = sum over tokens k_i * v_j
 *
 * Sequences never exchange state: the causal sum runs only over tokens of the
 * same sequence ("data packing" of the page "MiniMax-01 Lightning Attention",
 * section "计算优化").
 *
 * Parallelism: OpenMP over independent (sequence, head) pairs only; the order
 * of every floating-point sum inside a pair is the plain left-to-right order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline int64_t at3(int64_t t, int h, int x, int H, int d) {
    return (t * H + h) * (int64_t)d + x;
}

static inline const double* state_ptr(const double* S, int s, int h, int H, int d) {
    return S + ((int64_t)s * H + h) * (int64_t)d * d;
}

/* O = tril(Q K^T) V over each sequence, plus Q S0. */
void oracle_quadratic(const double* q, const double* k, const double* v, double* o,
                      const int32_t* cu_seqlens, int nseq, int H, int d,
                      const double* init)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        const double* S0 = init ? state_ptr(init, s, h, H, d) : NULL;
        for (int64_t t = start; t < end; ++t) {
            double* ot = o + at3(t, h, 0, H, d);
            for (int j = 0; j < d; ++j) ot[j] = 0.0;
            if (S0) {
                for (int i = 0; i < d; ++i) {
                    double qi = q[at3(t, h, i, H, d)];
                    for (int j = 0; j < d; ++j) ot[j] += qi * S0[(int64_t)i * d + j];
                }
            }
            for (int64_t u = start; u <= t; ++u) {          /* causal, diagonal kept */
                double score = 0.0;
                for (int i = 0; i < d; ++i)
                    score += q[at3(t, h, i, H, d)] * k[at3(u, h, i, H, d)];
                const double* vu = v + at3(u, h, 0, H, d);
                for (int j = 0; j < d; ++j) ot[j] += score * vu[j];
            }
        }
    }
}

/* S = S0; for each token: S += k^T v, then o = q S (the updated state). */
void oracle_recurrent(const double* q, const double* k, const double* v, double* o,
                      const int32_t* cu_seqlens, int nseq, int H, int d,
                      const double* init, double* state_out)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        double* S = (double*)calloc((size_t)d * d, sizeof(double));
        if (init) memcpy(S, state_ptr(init, s, h, H, d), sizeof(double) * d * d);
        for (int64_t t = start; t < end; ++t) {
            const double* kt = k + at3(t, h, 0, H, d);
            const double* vt = v + at3(t, h, 0, H, d);
            const double* qt = q + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) S[(int64_t)i * d + j] += kt[i] * vt[j];
            double* ot = o + at3(t, h, 0, H, d);
            for (int j = 0; j < d; ++j) ot[j] = 0.0;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) ot[j] += qt[i] * S[(int64_t)i * d + j];
        }
        if (state_out)
            memcpy((double*)state_ptr(state_out, s, h, H, d), S, sizeof(double) * d * d);
        free(S);
    }
}

/*
 * The block decomposition. Blocks restart at every sequence start; the last
 * block of a sequence may be shorter than B.
 *   intra: O_b  = (tril(Q_b K_b^T)) V_b          (left product, causal mask)
 *   inter: O_b += Q_b KV                          (right product, prefix state)
 *   then   KV  += K_b^T V_b
 */
void oracle_blocked(const double* q, const double* k, const double* v, double* o,
                    const int32_t* cu_seqlens, int nseq, int H, int d, int B,
                    const double* init, double* state_out)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        double* KV = (double*)calloc((size_t)d * d, sizeof(double));
        if (init) memcpy(KV, state_ptr(init, s, h, H, d), sizeof(double) * d * d);
        for (int64_t b0 = start; b0 < end; b0 += B) {
            int64_t b1 = b0 + B < end ? b0 + B : end;
            /* intra-block left product with causal mask */
            for (int64_t t = b0; t < b1; ++t) {
                double* ot = o + at3(t, h, 0, H, d);
                for (int j = 0; j < d; ++j) ot[j] = 0.0;
                for (int64_t u = b0; u <= t; ++u) {
                    double score = 0.0;
                    for (int i = 0; i < d; ++i)
                        score += q[at3(t, h, i, H, d)] * k[at3(u, h, i, H, d)];
                    for (int j = 0; j < d; ++j) ot[j] += score * v[at3(u, h, j, H, d)];
                }
                /* inter-block right product with the prefix state of earlier blocks */
                for (int i = 0; i < d; ++i) {
                    double qi = q[at3(t, h, i, H, d)];
                    for (int j = 0; j < d; ++j) ot[j] += qi * KV[(int64_t)i * d + j];
                }
            }
            /* fold this block into the prefix state */
            for (int64_t u = b0; u < b1; ++u)
                for (int i = 0; i < d; ++i)
                    for (int j = 0; j < d; ++j)
                        KV[(int64_t)i * d + j] += k[at3(u, h, i, H, d)] * v[at3(u, h, j, H, d)];
        }
        if (state_out)
            memcpy((double*)state_ptr(state_out, s, h, H, d), KV, sizeof(double) * d * d);
        free(KV);
    }
}

/* Final state per (sequence, head): S0 + sum_s k_s^T v_s. */
void oracle_state(const double* k, const double* v, const int32_t* cu_seqlens,
                  int nseq, int H, int d, const double* init, double* state_out)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        double* S = (double*)state_ptr(state_out, s, h, H, d);
        if (init) memcpy(S, state_ptr(init, s, h, H, d), sizeof(double) * d * d);
        else memset(S, 0, sizeof(double) * d * d);
        for (int64_t t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t)
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j)
                    S[(int64_t)i * d + j] += k[at3(t, h, i, H, d)] * v[at3(t, h, j, H, d)];
    }
}

/*
 * One decode step for `batch` independent sequences:
 *   S <- S + k^T v ;  o = q S   (the output sees the updated state, so the
 *   current token attends to itself, matching s <= t in the prefill).
 * q, k, v, o: [batch][H][d]; state: [batch][H][d][d], updated in place.
 */
void oracle_decode_step(const double* q, const double* k, const double* v,
                        double* state, double* o, int batch, int H, int d)
{
    int64_t npairs = (int64_t)batch * H;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < npairs; ++p) {
        double* S = state + p * (int64_t)d * d;
        const double* qp = q + p * d;
        const double* kp = k + p * d;
        const double* vp = v + p * d;
        double* op = o + p * d;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) S[(int64_t)i * d + j] += kp[i] * vp[j];
        for (int j = 0; j < d; ++j) op[j] = 0.0;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) op[j] += qp[i] * S[(int64_t)i * d + j];
    }
}

/*
 * Gradients of L = sum_t dO_t . O_t, per (sequence, head), from the forward
 * definition O_t = q_t S_t with S_t = S0 + sum_{s <= t} k_s^T v_s:
 *   dq_t = dO_t S_t^T                                   (forward pass over t)
 *   R_s  = sum_{t >= s} q_t^T dO_t                       (reverse pass over s)
 *   dk_s = v_s R_s^T,   dv_s = k_s R_s,   dS0 = R_start  (R of the whole sequence)
 * dinit may be NULL; init may be NULL (zero S0).
 */
void oracle_backward(const double* q, const double* k, const double* v, const double* dout,
                     const int32_t* cu_seqlens, int nseq, int H, int d, const double* init,
                     double* dq, double* dk, double* dv, double* dinit)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        double* S = (double*)calloc((size_t)d * d, sizeof(double));
        if (init) memcpy(S, state_ptr(init, s, h, H, d), sizeof(double) * d * d);
        for (int64_t t = start; t < end; ++t) {
            const double* kt = k + at3(t, h, 0, H, d);
            const double* vt = v + at3(t, h, 0, H, d);
            const double* gt = dout + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) S[(int64_t)i * d + j] += kt[i] * vt[j];
            double* dqt = dq + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += gt[j] * S[(int64_t)i * d + j];
                dqt[i] = acc;
            }
        }
        double* R = S;                                   /* reused: reverse state */
        memset(R, 0, sizeof(double) * d * d);
        for (int64_t t = end - 1; t >= start; --t) {
            const double* qt = q + at3(t, h, 0, H, d);
            const double* kt = k + at3(t, h, 0, H, d);
            const double* vt = v + at3(t, h, 0, H, d);
            const double* gt = dout + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) R[(int64_t)i * d + j] += qt[i] * gt[j];
            double* dkt = dk + at3(t, h, 0, H, d);
            double* dvt = dv + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += R[(int64_t)i * d + j] * vt[j];
                dkt[i] = acc;
            }
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i) acc += kt[i] * R[(int64_t)i * d + j];
                dvt[j] = acc;
            }
        }
        if (dinit) memcpy((double*)state_ptr(dinit, s, h, H, d), R, sizeof(double) * d * d);
        free(S);
    }
}

/*
 * ---------------------------------------------------------------- decay variant
 * Not on the pages: a per-head decay rate lambda_h in [0, 1] on the state, the
 * Lightning Attention-2 form of the same method, taken in its plainest reading
 * (lambda = 1 is the method above):
 *
 *     S_t = lambda_h S_{t-1} + k_t^T v_t,   S_{start-1} = S0,   o_t = q_t S_t
 *
 * so that, written out over a sequence starting at `start`,
 *
 *     O_t = lambda^(t-start+1) q_t . S0 + sum_{s in seq(t), s <= t} lambda^(t-s) (q_t . k_s) v_s.
 *
 * lam: [H]. Powers are pow(lambda, n) with n >= 0 an integer, pow(0, 0) = 1.
 */

/* The written-out sum above, term by term. */
void oracle_decay_quadratic(const double* q, const double* k, const double* v, double* o,
                            const int32_t* cu_seqlens, int nseq, int H, int d,
                            const double* init, const double* lam)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        const double* S0 = init ? state_ptr(init, s, h, H, d) : NULL;
        for (int64_t t = start; t < end; ++t) {
            double* ot = o + at3(t, h, 0, H, d);
            for (int j = 0; j < d; ++j) ot[j] = 0.0;
            if (S0) {
                double w = pow(lam[h], (double)(t - start + 1));
                for (int i = 0; i < d; ++i) {
                    double qi = q[at3(t, h, i, H, d)];
                    for (int j = 0; j < d; ++j) ot[j] += w * qi * S0[(int64_t)i * d + j];
                }
            }
            for (int64_t u = start; u <= t; ++u) {
                double score = 0.0;
                for (int i = 0; i < d; ++i)
                    score += q[at3(t, h, i, H, d)] * k[at3(u, h, i, H, d)];
                double w = pow(lam[h], (double)(t - u)) * score;
                const double* vu = v + at3(u, h, 0, H, d);
                for (int j = 0; j < d; ++j) ot[j] += w * vu[j];
            }
        }
    }
}

/* The recurrence itself: S = lambda S + k^T v, then o = q S. */
void oracle_decay_recurrent(const double* q, const double* k, const double* v, double* o,
                            const int32_t* cu_seqlens, int nseq, int H, int d,
                            const double* init, const double* lam, double* state_out)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        double* S = (double*)calloc((size_t)d * d, sizeof(double));
        if (init) memcpy(S, state_ptr(init, s, h, H, d), sizeof(double) * d * d);
        for (int64_t t = start; t < end; ++t) {
            const double* kt = k + at3(t, h, 0, H, d);
            const double* vt = v + at3(t, h, 0, H, d);
            const double* qt = q + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j)
                    S[(int64_t)i * d + j] = lam[h] * S[(int64_t)i * d + j] + kt[i] * vt[j];
            double* ot = o + at3(t, h, 0, H, d);
            for (int j = 0; j < d; ++j) ot[j] = 0.0;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) ot[j] += qt[i] * S[(int64_t)i * d + j];
        }
        if (state_out)
            memcpy((double*)state_ptr(state_out, s, h, H, d), S, sizeof(double) * d * d);
        free(S);
    }
}

/*
 * The block decomposition with decay (Lightning Attention-2). For a block of
 * n tokens starting at b0, with KV the state just before b0 and r = t - b0:
 *   intra: O_t  = sum_{u=b0..t} lambda^(t-u) (q_t . k_u) v_u       (decay mask)
 *   inter: O_t += lambda^(r+1) q_t KV
 *   then   KV   = lambda^n KV + sum_u lambda^(b0+n-1-u) k_u^T v_u
 */
void oracle_decay_blocked(const double* q, const double* k, const double* v, double* o,
                          const int32_t* cu_seqlens, int nseq, int H, int d, int B,
                          const double* init, const double* lam, double* state_out)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        double* KV = (double*)calloc((size_t)d * d, sizeof(double));
        if (init) memcpy(KV, state_ptr(init, s, h, H, d), sizeof(double) * d * d);
        for (int64_t b0 = start; b0 < end; b0 += B) {
            int64_t b1 = b0 + B < end ? b0 + B : end;
            for (int64_t t = b0; t < b1; ++t) {
                double* ot = o + at3(t, h, 0, H, d);
                for (int j = 0; j < d; ++j) ot[j] = 0.0;
                for (int64_t u = b0; u <= t; ++u) {
                    double score = 0.0;
                    for (int i = 0; i < d; ++i)
                        score += q[at3(t, h, i, H, d)] * k[at3(u, h, i, H, d)];
                    double w = pow(lam[h], (double)(t - u)) * score;
                    for (int j = 0; j < d; ++j) ot[j] += w * v[at3(u, h, j, H, d)];
                }
                double w = pow(lam[h], (double)(t - b0 + 1));
                for (int i = 0; i < d; ++i) {
                    double qi = w * q[at3(t, h, i, H, d)];
                    for (int j = 0; j < d; ++j) ot[j] += qi * KV[(int64_t)i * d + j];
                }
            }
            double wn = pow(lam[h], (double)(b1 - b0));
            for (int64_t x = 0; x < (int64_t)d * d; ++x) KV[x] *= wn;
            for (int64_t u = b0; u < b1; ++u) {
                double w = pow(lam[h], (double)(b1 - 1 - u));
                for (int i = 0; i < d; ++i)
                    for (int j = 0; j < d; ++j)
                        KV[(int64_t)i * d + j] += w * k[at3(u, h, i, H, d)] * v[at3(u, h, j, H, d)];
            }
        }
        if (state_out)
            memcpy((double*)state_ptr(state_out, s, h, H, d), KV, sizeof(double) * d * d);
        free(KV);
    }
}

/* Final state per (sequence, head): lambda^n S0 + sum_t lambda^(end-1-t) k_t^T v_t. */
void oracle_decay_state(const double* k, const double* v, const int32_t* cu_seqlens,
                        int nseq, int H, int d, const double* init, const double* lam,
                        double* state_out)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        double* S = (double*)state_ptr(state_out, s, h, H, d);
        double w0 = pow(lam[h], (double)(end - start));
        for (int64_t x = 0; x < (int64_t)d * d; ++x)
            S[x] = init ? w0 * state_ptr(init, s, h, H, d)[x] : 0.0;
        for (int64_t t = start; t < end; ++t) {
            double w = pow(lam[h], (double)(end - 1 - t));
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j)
                    S[(int64_t)i * d + j] += w * k[at3(t, h, i, H, d)] * v[at3(t, h, j, H, d)];
        }
    }
}

/* One decode step with decay: S <- lambda_h S + k^T v ; o = q S. */
void oracle_decay_decode_step(const double* q, const double* k, const double* v,
                              double* state, double* o, int batch, int H, int d,
                              const double* lam)
{
    int64_t npairs = (int64_t)batch * H;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < npairs; ++p) {
        int h = (int)(p % H);
        double* S = state + p * (int64_t)d * d;
        const double* qp = q + p * d;
        const double* kp = k + p * d;
        const double* vp = v + p * d;
        double* op = o + p * d;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j)
                S[(int64_t)i * d + j] = lam[h] * S[(int64_t)i * d + j] + kp[i] * vp[j];
        for (int j = 0; j < d; ++j) op[j] = 0.0;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) op[j] += qp[i] * S[(int64_t)i * d + j];
    }
}

/*
 * Gradients of L = sum_t dO_t . O_t for the decay variant, per (sequence, head):
 *   dq_t = dO_t S_t^T                         with S_t = lambda S_{t-1} + k_t^T v_t (forward)
 *   R_s  = lambda R_{s+1} + q_s^T dO_s        (reverse, R past the end = 0)
 *   dk_s = v_s R_s^T,   dv_s = k_s R_s,   dS0 = lambda R_start
 * (R_s = sum_{t >= s} lambda^(t-s) q_t^T dO_t; S0 enters O_t with lambda^(t-start+1)).
 */
void oracle_decay_backward(const double* q, const double* k, const double* v, const double* dout,
                           const int32_t* cu_seqlens, int nseq, int H, int d, const double* init,
                           const double* lam, double* dq, double* dk, double* dv, double* dinit)
{
    int64_t npairs = (int64_t)nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t p = 0; p < npairs; ++p) {
        int s = (int)(p / H), h = (int)(p % H);
        int64_t start = cu_seqlens[s], end = cu_seqlens[s + 1];
        double* S = (double*)calloc((size_t)d * d, sizeof(double));
        if (init) memcpy(S, state_ptr(init, s, h, H, d), sizeof(double) * d * d);
        for (int64_t t = start; t < end; ++t) {
            const double* kt = k + at3(t, h, 0, H, d);
            const double* vt = v + at3(t, h, 0, H, d);
            const double* gt = dout + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j)
                    S[(int64_t)i * d + j] = lam[h] * S[(int64_t)i * d + j] + kt[i] * vt[j];
            double* dqt = dq + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += gt[j] * S[(int64_t)i * d + j];
                dqt[i] = acc;
            }
        }
        double* R = S;                                   /* reused: reverse state */
        memset(R, 0, sizeof(double) * d * d);
        for (int64_t t = end - 1; t >= start; --t) {
            const double* qt = q + at3(t, h, 0, H, d);
            const double* kt = k + at3(t, h, 0, H, d);
            const double* vt = v + at3(t, h, 0, H, d);
            const double* gt = dout + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j)
                    R[(int64_t)i * d + j] = lam[h] * R[(int64_t)i * d + j] + qt[i] * gt[j];
            double* dkt = dk + at3(t, h, 0, H, d);
            double* dvt = dv + at3(t, h, 0, H, d);
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += R[(int64_t)i * d + j] * vt[j];
                dkt[i] = acc;
            }
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i) acc += kt[i] * R[(int64_t)i * d + j];
                dvt[j] = acc;
            }
        }
        if (dinit) {
            double* g0 = (double*)state_ptr(dinit, s, h, H, d);
            for (int64_t x = 0; x < (int64_t)d * d; ++x) g0[x] = lam[h] * R[x];
        }
        free(S);
    }
}

/*
 * Feature map of the page "MiniMax-M2.5语言模型：Linear Attention架构解析与实践",
 * section "2.2 Linear Attention的数学原理" (alpha = 0.3 there):
 * phi(x) = ELU(x) + alpha x, ELU(x) = x for x > 0 and e^x - 1 otherwise,
 * applied elementwise to n values.
 */
void oracle_feature_map(const double* x, double* y, int64_t n, double alpha)
{
    for (int64_t i = 0; i < n; ++i) {
        double e = x[i] > 0.0 ? x[i] : expm1(x[i]);
        y[i] = e + alpha * x[i];
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
