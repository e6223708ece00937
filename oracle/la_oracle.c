/*
 * Plain fp64 CPU oracle for causal linear attention (Lightning Attention with
 * phi = identity, no decay, no normaliser, no 1/sqrt(d) scale).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is compiled into a separate shared
 * object that only the test suite, the smoke check and the benchmark's CPU
 * baseline load.  It shares no code, header, table or helper with the CUDA
 * library and must never be called from the product path.
 *
 * Source of every formula: page "MiniMax-M1で理解する：大規模言語モデルの
 * コンテキスト長限界を突破する革新的アーキテクチャ" (zenn.dev), section
 * "線形アテンションの数学的基礎" (mathematical basis of linear attention):
 *   LinearAttn(Q,K,V) = phi(Q) (phi(K)^T V)
 *   S_t = S_{t-1} + phi(k_t) v_t^T ,  o_t = phi(q_t) S_t ,  S_t in R^{D x d}
 * and the tiled reading from page "MiniMax: «Почему M2 в итоге стала моделью
 * с полным вниманием?» (конспект)" (ai.flicky.cc), section 1, glossary entry
 * "Lightning Attention": linear attention with tiling, a masked matrix inside
 * each block and a K^T V state carried between blocks.
 *
 * Conventions (readings where the pages are silent):
 *   - q_t, k_t are row vectors of length dk, v_t, o_t of length dv;
 *     S is dk x dv, indexed S[i][j] (key dim i, value dim j), row-major.
 *   - o_t uses S_t, i.e. the state AFTER adding token t (inclusive).
 *   - heads are independent; S0 (optional) is the state before token 1.
 * Layouts: dense tensors are [U][N][d] with U = B*H units, row-major;
 * packed varlen tensors are [T][H][d]; states are [U][dk][dv].
 * All arithmetic is double precision; summation order is the plain
 * left-to-right order of the formulas.
 */
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* One unit of the token-by-token recurrence.
 * q,k: rows of length dk at stride q_stride/k_stride doubles; v,o: length dv
 * at stride v_stride/o_stride.  S (dk*dv) holds S0 on entry and S_N on exit. */
static void recurrent_unit(int N, int dk, int dv,
                           const double* q, long q_stride,
                           const double* k, long k_stride,
                           const double* v, long v_stride,
                           double* o, long o_stride, double* S) {
    for (int t = 0; t < N; ++t) {
        const double* qt = q + (long)t * q_stride;
        const double* kt = k + (long)t * k_stride;
        const double* vt = v + (long)t * v_stride;
        double* ot = o + (long)t * o_stride;
        /* S_t = S_{t-1} + k_t v_t^T */
        for (int i = 0; i < dk; ++i) {
            double ki = kt[i];
            double* Si = S + (long)i * dv;
            for (int j = 0; j < dv; ++j) Si[j] += ki * vt[j];
        }
        /* o_t = q_t S_t */
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            double qi = qt[i];
            const double* Si = S + (long)i * dv;
            for (int j = 0; j < dv; ++j) ot[j] += qi * Si[j];
        }
    }
}

/* Dense recurrent form.  q,k [U][N][dk], v [U][N][dv], o [U][N][dv],
 * s0 [U][dk][dv] or NULL (zero), s_out [U][dk][dv] or NULL. */
void oracle_recurrent(int U, int N, int dk, int dv,
                      const double* q, const double* k, const double* v,
                      const double* s0, double* o, double* s_out) {
    long sd = (long)dk * dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < U; ++u) {
        double* S = (double*)malloc(sizeof(double) * (size_t)(sd > 0 ? sd : 1));
        if (s0) memcpy(S, s0 + (long)u * sd, sizeof(double) * (size_t)sd);
        else memset(S, 0, sizeof(double) * (size_t)sd);
        recurrent_unit(N, dk, dv,
                       q + (long)u * N * dk, dk, k + (long)u * N * dk, dk,
                       v + (long)u * N * dv, dv, o + (long)u * N * dv, dv, S);
        if (s_out) memcpy(s_out + (long)u * sd, S, sizeof(double) * (size_t)sd);
        free(S);
    }
}

/* Dense quadratic masked form:
 *   A = Q K^T, A[t][s] = 0 for s > t (diagonal kept),
 *   O = A V + Q S0,  S_N = S0 + K^T V.
 * Memory O(N^2) per unit: intended for small N only. */
void oracle_quadratic(int U, int N, int dk, int dv,
                      const double* q, const double* k, const double* v,
                      const double* s0, double* o, double* s_out) {
    long sd = (long)dk * dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < U; ++u) {
        const double* Q = q + (long)u * N * dk;
        const double* K = k + (long)u * N * dk;
        const double* V = v + (long)u * N * dv;
        double* O = o + (long)u * N * dv;
        const double* S0 = s0 ? s0 + (long)u * sd : NULL;
        double* A = (double*)malloc(sizeof(double) * (size_t)N * (size_t)N + 8);
        for (int t = 0; t < N; ++t)
            for (int s = 0; s < N; ++s) {
                double a = 0.0;
                if (s <= t)
                    for (int i = 0; i < dk; ++i) a += Q[(long)t * dk + i] * K[(long)s * dk + i];
                A[(long)t * N + s] = a;
            }
        for (int t = 0; t < N; ++t)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int s = 0; s < N; ++s) acc += A[(long)t * N + s] * V[(long)s * dv + j];
                if (S0)
                    for (int i = 0; i < dk; ++i) acc += Q[(long)t * dk + i] * S0[(long)i * dv + j];
                O[(long)t * dv + j] = acc;
            }
        if (s_out) {
            double* So = s_out + (long)u * sd;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) {
                    double acc = S0 ? S0[(long)i * dv + j] : 0.0;
                    for (int s = 0; s < N; ++s) acc += K[(long)s * dk + i] * V[(long)s * dv + j];
                    So[(long)i * dv + j] = acc;
                }
        }
        free(A);
    }
}

/* One decode step per unit: S <- S + k v^T (in place), o = q S (post-update).
 * q,k [U][dk], v,o [U][dv], S [U][dk][dv]. */
void oracle_decode(int U, int dk, int dv, const double* q, const double* k,
                   const double* v, double* S, double* o) {
    long sd = (long)dk * dv;
#pragma omp parallel for schedule(static)
    for (int u = 0; u < U; ++u)
        recurrent_unit(1, dk, dv, q + (long)u * dk, dk, k + (long)u * dk, dk,
                       v + (long)u * dv, dv, o + (long)u * dv, dv, S + (long)u * sd);
}

/* Packed ragged batch.  q,k [T][H][dk], v,o [T][H][dv]; sequence n covers
 * tokens [cu[n], cu[n+1]).  Initial state of (n, h): pool[init_idx[n]][h]
 * when init_idx != NULL and init_idx[n] >= 0, else zero.  s_out [n_seq][H][dk][dv]
 * or NULL.  Each (sequence, head) is the recurrent form on its own tokens. */
void oracle_varlen(int n_seq, const int* cu, int H, int dk, int dv,
                   const double* q, const double* k, const double* v,
                   const double* pool, const int* init_idx,
                   double* o, double* s_out) {
    long sd = (long)dk * dv;
    int units = n_seq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int w = 0; w < units; ++w) {
        int n = w / H, h = w % H;
        long t0 = cu[n];
        int len = cu[n + 1] - cu[n];
        double* S = (double*)malloc(sizeof(double) * (size_t)(sd > 0 ? sd : 1));
        int idx = init_idx ? init_idx[n] : -1;
        if (pool && idx >= 0) memcpy(S, pool + ((long)idx * H + h) * sd, sizeof(double) * (size_t)sd);
        else memset(S, 0, sizeof(double) * (size_t)sd);
        recurrent_unit(len, dk, dv,
                       q + (t0 * H + h) * dk, (long)H * dk,
                       k + (t0 * H + h) * dk, (long)H * dk,
                       v + (t0 * H + h) * dv, (long)H * dv,
                       o + (t0 * H + h) * dv, (long)H * dv, S);
        if (s_out) memcpy(s_out + ((long)n * H + h) * sd, S, sizeof(double) * (size_t)sd);
        free(S);
    }
}

/* Gradients of the dense recurrent form, by the chain rule through
 *   S_t = S_{t-1} + k_t v_t^T (S_0 = s0),   o_t = q_t S_t,
 * for a loss L with dL/do_t = do_t and dL/dS_N = ds_n (NULL = zero):
 *   dq_t = do_t S_t^T                                   (forward sweep)
 *   G_t  = sum_{t' >= t} q_t'^T do_t' + ds_n            (reverse sweep: the
 *          gradient reaching k_t v_t^T through every later state)
 *   dk_t = G_t v_t,   dv_t = G_t^T k_t,   ds0 = G_1.
 * q,k,dq,dk [U][N][d_k]; v,do,dv [U][N][d_v]; s0, ds_n, ds0 [U][d_k][d_v]
 * (s0, ds_n may be NULL = zero; ds0 may be NULL). */
void oracle_backward(int U, int N, int d_k, int d_v,
                     const double* q, const double* k, const double* v, const double* s0,
                     const double* dout, const double* ds_n,
                     double* dq, double* dk, double* dv, double* ds0) {
    long sd = (long)d_k * d_v;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < U; ++u) {
        const double* Q = q + (long)u * N * d_k;
        const double* K = k + (long)u * N * d_k;
        const double* V = v + (long)u * N * d_v;
        const double* DO = dout + (long)u * N * d_v;
        double* DQ = dq + (long)u * N * d_k;
        double* DK = dk + (long)u * N * d_k;
        double* DV = dv + (long)u * N * d_v;
        double* S = (double*)malloc(sizeof(double) * (size_t)(sd > 0 ? sd : 1));
        /* forward sweep: S_t, then dq_t = do_t S_t^T */
        if (s0) memcpy(S, s0 + (long)u * sd, sizeof(double) * (size_t)sd);
        else memset(S, 0, sizeof(double) * (size_t)sd);
        for (int t = 0; t < N; ++t) {
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_v; ++j) S[(long)i * d_v + j] += K[(long)t * d_k + i] * V[(long)t * d_v + j];
            for (int i = 0; i < d_k; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d_v; ++j) acc += DO[(long)t * d_v + j] * S[(long)i * d_v + j];
                DQ[(long)t * d_k + i] = acc;
            }
        }
        /* reverse sweep: G_t, then dk_t = G_t v_t, dv_t = G_t^T k_t */
        double* G = S;
        if (ds_n) memcpy(G, ds_n + (long)u * sd, sizeof(double) * (size_t)sd);
        else memset(G, 0, sizeof(double) * (size_t)sd);
        for (int t = N - 1; t >= 0; --t) {
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_v; ++j) G[(long)i * d_v + j] += Q[(long)t * d_k + i] * DO[(long)t * d_v + j];
            for (int i = 0; i < d_k; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d_v; ++j) acc += G[(long)i * d_v + j] * V[(long)t * d_v + j];
                DK[(long)t * d_k + i] = acc;
            }
            for (int j = 0; j < d_v; ++j) {
                double acc = 0.0;
                for (int i = 0; i < d_k; ++i) acc += G[(long)i * d_v + j] * K[(long)t * d_k + i];
                DV[(long)t * d_v + j] = acc;
            }
        }
        if (ds0) memcpy(ds0 + (long)u * sd, G, sizeof(double) * (size_t)sd);
        free(S);
    }
}
