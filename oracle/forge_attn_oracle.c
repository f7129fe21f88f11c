/*
 * forge_attn_oracle.c -- plain fp64 CPU oracle for causal multi-head attention,
 * forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent definition that the
 * CUDA library is checked against.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load it; the library itself never links,
 * loads or calls it, and the two share no code.
 *
 * What it computes (one attention head at a time; all arrays row-major, fp64):
 *
 *   S[i][j]  = scale * sum_k q[i][k] * kk[j][k]          for all i, j in [0, T)
 *   S[i][j]  = -inf  when causal and j > i                (causal mask)
 *   LSE[i]   = m_i + ln sum_j exp(S[i][j] - m_i),  m_i = max_j S[i][j]
 *   P[i][j]  = exp(S[i][j] - LSE[i])
 *   O[i]     = sum_j P[i][j] * v[j]
 *   D[i]     = sum_k dO[i][k] * O[i][k]
 *   dP[i][j] = sum_k dO[i][k] * v[j][k]
 *   dS[i][j] = P[i][j] * (dP[i][j] - D[i])
 *   dV[j]    = sum_i P[i][j] * dO[i]
 *   dQ[i]    = scale * sum_j dS[i][j] * kk[j]
 *   dK[j]    = scale * sum_i dS[i][j] * q[i]
 *
 * Sources (Forge: "Building an LLM Training Framework from Scratch in C++ and
 * Metal on Apple Silicon"):
 *   - section "Attention kernel design": the forward is a softmax attention whose
 *     normaliser is saved per row as a log-sum-exp, and the backward uses that
 *     saved log-sum-exp instead of re-deriving the normalisation;
 *   - section "Ecosystem survey" (the fused-backward paragraph): the backward is a
 *     pre-pass D = rowsum(dO o O) in float, a dQ stage over queries and a dK/dV
 *     stage over key/value rows;
 *   - section "Methodology" ("Correctness gates optimization"): every GPU kernel is
 *     checked against a plain CPU reference, gradients also against central finite
 *     differences.
 * The tiled online softmax of the GPU kernels reaches this same result up to
 * rounding, so the oracle is the plain definition above: the full T x T score
 * matrix is materialised, with no tiling, fusion or reordering.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - dQ and dK carry the factor `scale`: dS is the gradient with respect to the
 *     scaled logits S, and S = scale * Q K^T;
 *   - LSE is the natural logarithm over the scaled, masked scores;
 *   - D uses the oracle's own fp64 O.
 *
 * Error behaviour: every entry point returns 0 on success, -1 on bad arguments
 * and -2 when a temporary buffer cannot be allocated.  Outputs are written only
 * on success.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EBADARG (-1)
#define ORACLE_ENOMEM (-2)

/* True when key j is masked out for query i. */
static int masked(int causal, int i, int j) { return causal && j > i; }

/* Materialise S = scale * Q K^T (T x T) with the causal mask applied.
 * The product is written as S[i][:] += q[i][c] * K^T[c][:], so each S[i][j] is
 * still the plain sum over c = 0..d-1 taken in order. */
static int scores(int T, int d, double scale, int causal, const double* q,
                  const double* kk, double* S)
{
    double* kt = (double*)malloc(sizeof(double) * (size_t)d * (size_t)T);
    if (!kt) return ORACLE_ENOMEM;
    for (int j = 0; j < T; ++j)
        for (int c = 0; c < d; ++c) kt[(size_t)c * T + j] = kk[(size_t)j * d + c];
    for (int i = 0; i < T; ++i) {
        double* srow = S + (size_t)i * T;
        for (int j = 0; j < T; ++j) srow[j] = 0.0;
        for (int c = 0; c < d; ++c) {
            const double qc = q[(size_t)i * d + c];
            const double* kr = kt + (size_t)c * T;
            for (int j = 0; j < T; ++j) srow[j] += qc * kr[j];
        }
        for (int j = 0; j < T; ++j)
            srow[j] = masked(causal, i, j) ? -INFINITY : scale * srow[j];
    }
    free(kt);
    return ORACLE_OK;
}

/* Row softmax of S in place into P, with the row log-sum-exp. */
static void softmax_rows(int T, const double* S, double* P, double* lse)
{
    for (int i = 0; i < T; ++i) {
        const double* srow = S + (size_t)i * T;
        double* prow = P + (size_t)i * T;
        double m = -INFINITY;
        for (int j = 0; j < T; ++j) m = srow[j] > m ? srow[j] : m;
        double sum = 0.0;
        for (int j = 0; j < T; ++j) sum += exp(srow[j] - m);
        const double l = m + log(sum);
        lse[i] = l;
        for (int j = 0; j < T; ++j) prow[j] = exp(srow[j] - l);
    }
}

/* C (T x d) = A (T x T) B (T x d):  C[i][:] = sum_j A[i][j] * B[j][:]. */
static void matmul_tt_td(int T, int d, const double* A, const double* B, double* C)
{
    for (int i = 0; i < T; ++i) {
        double* crow = C + (size_t)i * d;
        for (int c = 0; c < d; ++c) crow[c] = 0.0;
        for (int j = 0; j < T; ++j) {
            const double a = A[(size_t)i * T + j];
            if (a == 0.0) continue; /* exact: adding 0 * finite changes nothing */
            const double* brow = B + (size_t)j * d;
            for (int c = 0; c < d; ++c) crow[c] += a * brow[c];
        }
    }
}

/* C (T x d) = A^T (T x T) B (T x d):  C[j][:] = sum_i A[i][j] * B[i][:]. */
static void matmul_ttT_td(int T, int d, const double* A, const double* B, double* C)
{
    for (size_t x = 0; x < (size_t)T * d; ++x) C[x] = 0.0;
    for (int i = 0; i < T; ++i) {
        const double* brow = B + (size_t)i * d;
        for (int j = 0; j < T; ++j) {
            const double a = A[(size_t)i * T + j];
            if (a == 0.0) continue;
            double* crow = C + (size_t)j * d;
            for (int c = 0; c < d; ++c) crow[c] += a * brow[c];
        }
    }
}

/*
 * Forward of one head.  q, kk, v: [T][d]; o: [T][d]; lse: [T].
 * p_out, when not NULL, receives P ([T][T]).
 */
int oracle_attn_fwd(int T, int d, double scale, int causal, const double* q,
                    const double* kk, const double* v, double* o, double* lse,
                    double* p_out)
{
    if (T < 1 || d < 1 || !q || !kk || !v || !o || !lse) return ORACLE_EBADARG;
    const size_t tt = (size_t)T * T;
    double* S = (double*)malloc(sizeof(double) * tt);
    double* P = p_out ? p_out : (double*)malloc(sizeof(double) * tt);
    if (!S || !P) {
        free(S);
        if (!p_out) free(P);
        return ORACLE_ENOMEM;
    }
    int rc = scores(T, d, scale, causal, q, kk, S);
    if (rc == ORACLE_OK) {
        softmax_rows(T, S, P, lse);
        matmul_tt_td(T, d, P, v, o);
    }
    free(S);
    if (!p_out) free(P);
    return rc;
}

/*
 * Backward of one head, from the definition (forward recomputed in fp64).
 * q, kk, v, dO: [T][d]; dq, dk, dv: [T][d].
 * ds_out ([T][T]) and d_out ([T]) are optional (NULL to skip).
 */
int oracle_attn_bwd(int T, int d, double scale, int causal, const double* q,
                    const double* kk, const double* v, const double* dO, double* dq,
                    double* dk, double* dv, double* ds_out, double* d_out)
{
    if (T < 1 || d < 1 || !q || !kk || !v || !dO || !dq || !dk || !dv)
        return ORACLE_EBADARG;
    const size_t tt = (size_t)T * T;
    const size_t td = (size_t)T * d;
    double* S = (double*)malloc(sizeof(double) * tt);   /* S, then dP */
    double* P = (double*)malloc(sizeof(double) * tt);
    double* dS = ds_out ? ds_out : (double*)malloc(sizeof(double) * tt);
    double* O = (double*)malloc(sizeof(double) * td);
    double* lse = (double*)malloc(sizeof(double) * (size_t)T);
    double* Dv = (double*)malloc(sizeof(double) * (size_t)T);
    int rc = ORACLE_ENOMEM;
    if (!S || !P || !dS || !O || !lse || !Dv) goto done;

    rc = scores(T, d, scale, causal, q, kk, S);
    if (rc != ORACLE_OK) goto done;
    softmax_rows(T, S, P, lse);
    matmul_tt_td(T, d, P, v, O);

    /* D[i] = rowsum(dO o O) */
    for (int i = 0; i < T; ++i) {
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += dO[(size_t)i * d + c] * O[(size_t)i * d + c];
        Dv[i] = s;
    }
    /* dP = dO V^T (reuse the S buffer), dS = P o (dP - D) */
    for (int i = 0; i < T; ++i) {
        for (int j = 0; j < T; ++j) {
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += dO[(size_t)i * d + c] * v[(size_t)j * d + c];
            S[(size_t)i * T + j] = s;
        }
    }
    for (int i = 0; i < T; ++i)
        for (int j = 0; j < T; ++j) {
            const size_t x = (size_t)i * T + j;
            dS[x] = P[x] * (S[x] - Dv[i]);
        }
    /* dV = P^T dO */
    matmul_ttT_td(T, d, P, dO, dv);
    /* dQ = scale * dS K */
    matmul_tt_td(T, d, dS, kk, dq);
    for (size_t x = 0; x < td; ++x) dq[x] *= scale;
    /* dK = scale * dS^T Q */
    matmul_ttT_td(T, d, dS, q, dk);
    for (size_t x = 0; x < td; ++x) dk[x] *= scale;
    if (d_out)
        for (int i = 0; i < T; ++i) d_out[i] = Dv[i];
    rc = ORACLE_OK;
done:
    free(S);
    free(P);
    if (!ds_out) free(dS);
    free(O);
    free(lse);
    free(Dv);
    return rc;
}

/* One query row i from the definition: scores s[0..T), its log-sum-exp, the
 * probabilities p[0..T) and the output row o[0..d).  Masked entries of p are 0. */
static void row_forward(int T, int d, double scale, int causal, const double* q,
                        const double* kk, const double* v, int i, double* s, double* p,
                        double* lse_i, double* o)
{
    double m = -INFINITY;
    for (int j = 0; j < T; ++j) {
        if (masked(causal, i, j)) {
            s[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += q[(size_t)i * d + c] * kk[(size_t)j * d + c];
        s[j] = scale * acc;
        m = s[j] > m ? s[j] : m;
    }
    double sum = 0.0;
    for (int j = 0; j < T; ++j) sum += exp(s[j] - m);
    const double l = m + log(sum);
    *lse_i = l;
    for (int j = 0; j < T; ++j) p[j] = exp(s[j] - l);
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int j = 0; j < T; ++j) {
        if (p[j] == 0.0) continue;
        for (int c = 0; c < d; ++c) o[c] += p[j] * v[(size_t)j * d + c];
    }
}

/*
 * Sampled outputs of one head, from the same definition, for sizes where the
 * T x T matrices are too large to keep: O, LSE and dQ for the query rows qidx[],
 * dK and dV for the key rows kidx[].  Row by row, so memory is O(T d).
 * o_out, dq_out: [nq][d]; lse_out: [nq]; dk_out, dv_out: [nk][d].
 * Any output pointer may be NULL when its part is not wanted.
 */
int oracle_attn_rows(int T, int d, double scale, int causal, const double* q,
                     const double* kk, const double* v, const double* dO, int nq,
                     const int* qidx, double* o_out, double* lse_out, double* dq_out,
                     int nk, const int* kidx, double* dk_out, double* dv_out)
{
    if (T < 1 || d < 1 || !q || !kk || !v || nq < 0 || nk < 0) return ORACLE_EBADARG;
    if ((nq > 0 && !qidx) || (nk > 0 && !kidx)) return ORACLE_EBADARG;
    if ((dq_out || nk > 0) && !dO) return ORACLE_EBADARG;
    for (int a = 0; a < nq; ++a)
        if (qidx[a] < 0 || qidx[a] >= T) return ORACLE_EBADARG;
    for (int a = 0; a < nk; ++a)
        if (kidx[a] < 0 || kidx[a] >= T) return ORACLE_EBADARG;

    double* s = (double*)malloc(sizeof(double) * (size_t)T);
    double* p = (double*)malloc(sizeof(double) * (size_t)T);
    double* orow = (double*)malloc(sizeof(double) * (size_t)d);
    double* lse_all = nk > 0 ? (double*)malloc(sizeof(double) * (size_t)T) : NULL;
    double* D_all = nk > 0 ? (double*)malloc(sizeof(double) * (size_t)T) : NULL;
    int rc = ORACLE_ENOMEM;
    if (!s || !p || !orow || (nk > 0 && (!lse_all || !D_all))) goto done;

    /* Query rows: O, LSE, and dQ[i] = scale * sum_j P_ij (dP_ij - D_i) k_j. */
    for (int a = 0; a < nq; ++a) {
        const int i = qidx[a];
        double l;
        row_forward(T, d, scale, causal, q, kk, v, i, s, p, &l, orow);
        if (o_out)
            for (int c = 0; c < d; ++c) o_out[(size_t)a * d + c] = orow[c];
        if (lse_out) lse_out[a] = l;
        if (dq_out) {
            double Di = 0.0;
            for (int c = 0; c < d; ++c) Di += dO[(size_t)i * d + c] * orow[c];
            double* dqr = dq_out + (size_t)a * d;
            for (int c = 0; c < d; ++c) dqr[c] = 0.0;
            for (int j = 0; j < T; ++j) {
                if (p[j] == 0.0) continue;
                double dp = 0.0;
                for (int c = 0; c < d; ++c) dp += dO[(size_t)i * d + c] * v[(size_t)j * d + c];
                const double ds = p[j] * (dp - Di);
                for (int c = 0; c < d; ++c) dqr[c] += ds * kk[(size_t)j * d + c];
            }
            for (int c = 0; c < d; ++c) dqr[c] *= scale;
        }
    }

    if (nk > 0) {
        /* LSE and D of every query row (each key row's gradient sums over them). */
        for (int i = 0; i < T; ++i) {
            row_forward(T, d, scale, causal, q, kk, v, i, s, p, &lse_all[i], orow);
            double Di = 0.0;
            for (int c = 0; c < d; ++c) Di += dO[(size_t)i * d + c] * orow[c];
            D_all[i] = Di;
        }
        /* dV[j] = sum_i P_ij dO_i ;  dK[j] = scale * sum_i dS_ij q_i */
        for (int a = 0; a < nk; ++a) {
            const int j = kidx[a];
            double* dvr = dv_out ? dv_out + (size_t)a * d : NULL;
            double* dkr = dk_out ? dk_out + (size_t)a * d : NULL;
            if (dvr)
                for (int c = 0; c < d; ++c) dvr[c] = 0.0;
            if (dkr)
                for (int c = 0; c < d; ++c) dkr[c] = 0.0;
            for (int i = 0; i < T; ++i) {
                if (masked(causal, i, j)) continue;
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += q[(size_t)i * d + c] * kk[(size_t)j * d + c];
                const double pij = exp(scale * acc - lse_all[i]);
                if (pij == 0.0) continue;
                if (dvr)
                    for (int c = 0; c < d; ++c) dvr[c] += pij * dO[(size_t)i * d + c];
                if (dkr) {
                    double dp = 0.0;
                    for (int c = 0; c < d; ++c) dp += dO[(size_t)i * d + c] * v[(size_t)j * d + c];
                    const double ds = pij * (dp - D_all[i]);
                    for (int c = 0; c < d; ++c) dkr[c] += ds * q[(size_t)i * d + c];
                }
            }
            if (dkr)
                for (int c = 0; c < d; ++c) dkr[c] *= scale;
        }
    }
    rc = ORACLE_OK;
done:
    free(s);
    free(p);
    free(orow);
    free(lse_all);
    free(D_all);
    return rc;
}
