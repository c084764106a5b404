/*
 * la_oracle.c -- fp64 recurrent-form oracle for causal linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load, link or call
 * this file: only the test-suite, the package smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only through seeded inputs.
 *
 * Source of every formula: the lesson page "Линейное внимание и гибриды"
 * ("Linear attention and hybrids", ai.flicky.cc, stage 5.5).  Section names below
 * are that page's, translated:
 *   [kernel trick]  "Ядерный трюк: убираем softmax"        -- phi(x)=elu(x)+1, S_i, z_i
 *   [three forms]   "Три формы одного вычисления"          -- recurrent form
 *   [decay/gates]   "Память должна забывать: затухание и гейты"
 *   [delta rule]    "Дельта-правило и Gated DeltaNet"      -- delta rule, Gated DeltaNet
 *
 * What is computed, per (batch b, head h), for t = 1..T, updating first and then
 * reading (the recurrent form of [three forms]):
 *
 *   mode 0 (elu+1, normalised; [kernel trick], [three forms]):
 *       S_t = S_{t-1} + v_t phi(k_t)^T,   z_t = z_{t-1} + phi(k_t),
 *       o_t = S_t phi(q_t) / (z_t^T phi(q_t)).
 *   mode 1 (scalar gate, no feature map, no denominator; [decay/gates]):
 *       S_t = a_t S_{t-1} + v_t k_t^T,    o_t = S_t q_t.
 *   mode 2 (gated delta rule, Gated DeltaNet equation of [delta rule]):
 *       S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t.
 *     The product S_{t-1}(I - b k k^T) is evaluated as S_{t-1} - b (S_{t-1} k) k^T,
 *     which is the same matrix (distributivity), at O(d_k d_v) per token.
 *   mode 3 (Kimi Delta Attention of [delta rule]: the scalar a_t of mode 2 becomes the
 *     diagonal matrix Diag(a_t), each memory channel forgetting at its own rate; the
 *     channels are the d_k columns of S):
 *       S_t = S_{t-1} Diag(a_t) (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t,
 *     evaluated as M = S_{t-1} Diag(a_t), S_t = M - b (M k) k^T + b v k^T.
 *
 * S is d_v x d_k (the page's orientation), stored row-major [d_v][d_k]; z has
 * d_k entries.  A NULL gate means a_t = 1.  Mode 0 ignores gate and beta, mode 1
 * ignores beta.  In mode 3 the gate holds d_k values per token.  Readings where the page is silent (no 1/sqrt(d) inside the
 * attention, no epsilon in the mode-0 denominator, the gate multiplies the old
 * state before token t is written) are listed in the design notes; this file
 * implements exactly the equations above.
 *
 * Layouts (all dense, row-major, fp64):
 *   q, k [B,H,T,d_k]; v, o [B,H,T,d_v]; gate, beta [B,H,T] (mode 3: gate [B,H,T,d_k]);
 *   S [B,H,d_v,d_k]; z [B,H,d_k].
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* phi(x) = elu(x) + 1: x + 1 for x > 0, e^x otherwise ([kernel trick]). */
static double oracle_phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

/* One token of the recurrence on one head.  fq/fk are d_k scratch vectors,
 * sk is d_v scratch. */
static void oracle_token(int mode, int dk, int dv, const double *q, const double *k,
                         const double *v, double a, const double *av, double beta, double *S,
                         double *z, double *o, double *fq, double *fk, double *sk)
{
    if (mode == 0) {
        for (int j = 0; j < dk; ++j) {
            fk[j] = oracle_phi(k[j]);
            fq[j] = oracle_phi(q[j]);
        }
        for (int i = 0; i < dv; ++i) {
            double *row = S + (size_t)i * dk;
            for (int j = 0; j < dk; ++j) row[j] += v[i] * fk[j];
        }
        double den = 0.0;
        for (int j = 0; j < dk; ++j) {
            z[j] += fk[j];
            den += z[j] * fq[j];
        }
        for (int i = 0; i < dv; ++i) {
            const double *row = S + (size_t)i * dk;
            double num = 0.0;
            for (int j = 0; j < dk; ++j) num += row[j] * fq[j];
            o[i] = num / den;
        }
    } else if (mode == 1) {
        for (int i = 0; i < dv; ++i) {
            double *row = S + (size_t)i * dk;
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) {
                row[j] = a * row[j] + v[i] * k[j];
                acc += row[j] * q[j];
            }
            o[i] = acc;
        }
    } else if (mode == 3) {
        /* M = S_{t-1} Diag(a_t); (M k)_i */
        for (int i = 0; i < dv; ++i) {
            const double *row = S + (size_t)i * dk;
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += row[j] * (av ? av[j] : 1.0) * k[j];
            sk[i] = acc;
        }
        for (int i = 0; i < dv; ++i) {
            double *row = S + (size_t)i * dk;
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) {
                /* [M (I - b k k^T)]_{ij} + b v_i k_j */
                row[j] = row[j] * (av ? av[j] : 1.0) - beta * sk[i] * k[j] + beta * v[i] * k[j];
                acc += row[j] * q[j];
            }
            o[i] = acc;
        }
    } else {
        /* (S k)_i with the old state */
        for (int i = 0; i < dv; ++i) {
            const double *row = S + (size_t)i * dk;
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += row[j] * k[j];
            sk[i] = acc;
        }
        for (int i = 0; i < dv; ++i) {
            double *row = S + (size_t)i * dk;
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) {
                /* a * [S(I - b k k^T)]_{ij} + b v_i k_j */
                row[j] = a * (row[j] - beta * sk[i] * k[j]) + beta * v[i] * k[j];
                acc += row[j] * q[j];
            }
            o[i] = acc;
        }
    }
}

/*
 * Run the recurrence over T tokens for every (b,h).  If init_state is zero the
 * state starts at S_0 = 0, z_0 = 0; otherwise S and z are read as S_0, z_0.
 * On return S, z hold the state after the last token and o holds o_1..o_T.
 * z may be NULL for modes 1 and 2.  nthreads <= 0 lets OpenMP decide.
 * Returns 0, or -1 on an argument error.
 */
int oracle_prefill(int mode, long B, long H, long T, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *gate, const double *beta,
                   double *S, double *z, double *o, int init_state, int nthreads)
{
    if (mode < 0 || mode > 3 || B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    if ((T > 0 && (!q || !k || !v || !o)) || !S) return -1;
    if (mode == 0 && !z) return -1;
    if (mode >= 2 && T > 0 && !beta) return -1;
    const long BH = B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double *scratch = (double *)malloc(sizeof(double) * (size_t)(2 * dk + dv));
        if (!scratch) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < BH; ++bh) {
            if (!scratch) continue;
            double *Sh = S + (size_t)bh * dv * dk;
            double *zh = z ? z + (size_t)bh * dk : NULL;
            if (!init_state) {
                memset(Sh, 0, sizeof(double) * (size_t)dv * dk);
                if (zh) memset(zh, 0, sizeof(double) * (size_t)dk);
            }
            for (long t = 0; t < T; ++t) {
                const size_t tok = (size_t)bh * T + t;
                const double a = (gate && mode != 3) ? gate[tok] : 1.0;
                const double *av = (gate && mode == 3) ? gate + tok * dk : NULL;
                const double b = beta ? beta[tok] : 0.0;
                oracle_token(mode, dk, dv, q + tok * dk, k + tok * dk, v + tok * dv, a, av, b,
                             Sh, zh, o + tok * dv, scratch, scratch + dk, scratch + 2 * dk);
            }
        }
        free(scratch);
    }
    return failed ? -1 : 0;
}

/*
 * One decode token for N sequences x H heads: the same single step of the
 * recurrence applied in place to a given state.  Layouts: q,k [N,H,d_k];
 * v, o [N,H,d_v]; gate, beta [N,H] (mode 3: gate [N,H,d_k]); S [N,H,d_v,d_k];
 * z [N,H,d_k].
 */
int oracle_decode_step(int mode, long N, long H, int dk, int dv,
                       const double *q, const double *k, const double *v,
                       const double *gate, const double *beta,
                       double *S, double *z, double *o, int nthreads)
{
    return oracle_prefill(mode, N, H, 1, dk, dv, q, k, v, gate, beta, S, z, o, 1, nthreads);
}

/* The number of OpenMP threads a parallel region would use (1 without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
