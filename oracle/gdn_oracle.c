/*
 * gdn_oracle.c -- fp64 CPU oracle for Tail-Replay state reconstruction of
 * Gated DeltaNet layers.  TEST INFRASTRUCTURE ONLY: the product path (the
 * CUDA library and its Python binding) never links, loads or calls this
 * file.  Only tests/, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header or constant with the CUDA path.
 *
 * What it computes, and from where:
 *
 *  - The gated delta rule of Gated DeltaNet (Yang, Kautz & Hatamizadeh,
 *    "Gated Delta Networks: Improving Mamba2 with Delta Rule", 2024), the
 *    recurrence that the Tail-Replay pages replay ("Tail-Replay: Escaping the
 *    Curse of Linear Attention in Prefix Caching for Hybrid LLMs", gist.science
 *    summary, section "Mecanismos Principais", item "Reconstrucao de Estado
 *    Independente", third bullet).  Per head, with a d_k x d_v state S whose
 *    rows are indexed by the key dimension:
 *        S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *        o_t = S_t^T q_t                       (post-update state)
 *    The decay alpha_t multiplies the old state including the erase term;
 *    the write term beta_t k_t v_t^T is not decayed.  No query scaling.
 *
 *  - Tail replay (same section, first and second bullets): the state at the
 *    end of a matched prefix of length L is rebuilt from a zero state by
 *    running the recurrence over only the last R tokens of that prefix,
 *    rows [L - R, L) of the request's cached sequence.  R > L is clamped to
 *    L; R = 0 (or L = 0) gives the zero state -- the "Zero-Only" baseline of
 *    the "Resultados" section.
 *
 *  - Suffix prefill: the same recurrence continued over the request's new
 *    tokens from a given state, emitting o_t for every token (the
 *    time-to-first-token path of the "Resultados" section).
 *
 * Everything is a plain token-by-token loop in double precision.  Inputs are
 * taken as the exact bytes a GPU kernel would consume: fp32 values, or bf16
 * bit patterns that are widened exactly.  The loop over (sequence, head)
 * units may run on several OpenMP threads; each unit's arithmetic is the
 * same sequential loop either way.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

static double widen(const void* base, int dtype, int64_t idx) {
    if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t*)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One head, n tokens, dense fp64 arrays.
 *   k[n*dk], v[n*dv], alpha[n], beta[n], q[n*dk] (may be NULL)
 *   S[dk*dv] row-major (row = key index): read as the initial state and
 *   overwritten with the final state.  o[n*dv] (may be NULL) receives o_t.
 * work[dv] is scratch.
 */
void oracle_recurrence_f64(int64_t n, int dk, int dv,
                           const double* k, const double* v,
                           const double* alpha, const double* beta,
                           const double* q, double* S, double* o,
                           double* work) {
    for (int64_t t = 0; t < n; ++t) {
        const double* kt = k + t * dk;
        const double* vt = v + t * dv;
        const double a = alpha[t], b = beta[t];
        /* work = k_t^T S_{t-1}  (a d_v row vector) */
        for (int j = 0; j < dv; ++j) work[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) work[j] += kt[i] * S[(int64_t)i * dv + j];
        /* S_t = a (S_{t-1} - b k_t (k_t^T S_{t-1})) + b k_t v_t^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double* s = &S[(int64_t)i * dv + j];
                *s = a * (*s - b * kt[i] * work[j]) + b * kt[i] * vt[j];
            }
        if (q) {
            const double* qt = q + t * dk;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(int64_t)i * dv + j] * qt[i];
                o[t * dv + j] = acc;
            }
        }
    }
}

/* Gather rows [row0, row0+n) of head h from a packed [rows, H, d] buffer. */
static void gather_rows(const void* src, int dtype, int64_t row0, int64_t n,
                        int H, int h, int d, double* dst) {
    for (int64_t t = 0; t < n; ++t)
        for (int i = 0; i < d; ++i)
            dst[t * d + i] = widen(src, dtype, ((row0 + t) * H + h) * (int64_t)d + i);
}

static void gather_gate(const float* src, int64_t row0, int64_t n, int H, int h, double* dst) {
    for (int64_t t = 0; t < n; ++t) dst[t] = (double)src[(row0 + t) * H + h];
}

/*
 * Replay window of sequence b: rows [seq_offsets[b] + match_len[b] - Reff,
 * seq_offsets[b] + match_len[b]) with Reff = min(R[b], match_len[b]).
 * Returns 0, or -1 for arguments that describe no valid window.
 */
int oracle_replay_window(int batch, const int32_t* seq_offsets, const int32_t* match_len,
                         const int32_t* R, int b, int64_t* row0, int64_t* len) {
    if (b < 0 || b >= batch) return -1;
    int64_t cached = (int64_t)seq_offsets[b + 1] - seq_offsets[b];
    if (cached < 0 || match_len[b] < 0 || match_len[b] > cached || R[b] < 0) return -1;
    int64_t reff = R[b] < match_len[b] ? R[b] : match_len[b];
    *row0 = (int64_t)seq_offsets[b] + match_len[b] - reff;
    *len = reff;
    return 0;
}

/*
 * Tail replay over a packed varlen batch.
 *   k: [rows, H, dk], v: [rows, H, dv] in dtype; alpha, beta: [rows, H] fp32.
 *   state_out: [batch, H, dk, dv] fp64.
 */
int oracle_replay_state(int batch, int H, int dk, int dv, int dtype,
                        const void* k, const void* v, const float* alpha, const float* beta,
                        const int32_t* seq_offsets, const int32_t* match_len, const int32_t* R,
                        double* state_out) {
    for (int b = 0; b < batch; ++b) {
        int64_t r0, n;
        if (oracle_replay_window(batch, seq_offsets, match_len, R, b, &r0, &n)) return -1;
    }
    int units = batch * H;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < units; ++u) {
        int b = u / H, h = u % H;
        int64_t r0 = 0, n = 0;
        oracle_replay_window(batch, seq_offsets, match_len, R, b, &r0, &n);
        double* S = state_out + (int64_t)u * dk * dv;
        memset(S, 0, sizeof(double) * (size_t)dk * dv);   /* zero replay state */
        int64_t nn = n > 0 ? n : 1;
        double* kk = malloc(sizeof(double) * nn * dk);
        double* vv = malloc(sizeof(double) * nn * dv);
        double* aa = malloc(sizeof(double) * nn);
        double* bb = malloc(sizeof(double) * nn);
        double* work = malloc(sizeof(double) * dv);
        if (!kk || !vv || !aa || !bb || !work) {
#pragma omp atomic write
            bad = 1;
        } else {
            gather_rows(k, dtype, r0, n, H, h, dk, kk);
            gather_rows(v, dtype, r0, n, H, h, dv, vv);
            gather_gate(alpha, r0, n, H, h, aa);
            gather_gate(beta, r0, n, H, h, bb);
            oracle_recurrence_f64(n, dk, dv, kk, vv, aa, bb, NULL, S, NULL, work);
        }
        free(kk); free(vv); free(aa); free(bb); free(work);
    }
    return bad ? -2 : 0;
}

/*
 * Prefill over a packed varlen batch: sequence b is rows [cu[b], cu[b+1]).
 *   q, k: [rows, H, dk], v: [rows, H, dv]; alpha, beta: [rows, H] fp32.
 *   state_in: [batch, H, dk, dv] fp64 or NULL (zero state).
 *   o_out: [rows, H, dv] fp64; state_out: [batch, H, dk, dv] fp64 or NULL.
 */
int oracle_prefill(int batch, int H, int dk, int dv, int dtype,
                   const void* q, const void* k, const void* v,
                   const float* alpha, const float* beta, const int32_t* cu,
                   const double* state_in, double* o_out, double* state_out) {
    for (int b = 0; b < batch; ++b)
        if (cu[b + 1] < cu[b] || cu[b] < 0) return -1;
    int units = batch * H;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < units; ++u) {
        int b = u / H, h = u % H;
        int64_t r0 = cu[b], n = (int64_t)cu[b + 1] - cu[b];
        int64_t nn = n > 0 ? n : 1;
        double* S = malloc(sizeof(double) * (size_t)dk * dv);
        double* qq = malloc(sizeof(double) * nn * dk);
        double* kk = malloc(sizeof(double) * nn * dk);
        double* vv = malloc(sizeof(double) * nn * dv);
        double* aa = malloc(sizeof(double) * nn);
        double* bb = malloc(sizeof(double) * nn);
        double* oo = malloc(sizeof(double) * nn * dv);
        double* work = malloc(sizeof(double) * dv);
        if (!S || !qq || !kk || !vv || !aa || !bb || !oo || !work) {
#pragma omp atomic write
            bad = 1;
        } else {
            if (state_in) memcpy(S, state_in + (int64_t)u * dk * dv, sizeof(double) * (size_t)dk * dv);
            else memset(S, 0, sizeof(double) * (size_t)dk * dv);
            gather_rows(q, dtype, r0, n, H, h, dk, qq);
            gather_rows(k, dtype, r0, n, H, h, dk, kk);
            gather_rows(v, dtype, r0, n, H, h, dv, vv);
            gather_gate(alpha, r0, n, H, h, aa);
            gather_gate(beta, r0, n, H, h, bb);
            oracle_recurrence_f64(n, dk, dv, kk, vv, aa, bb, qq, S, oo, work);
            for (int64_t t = 0; t < n; ++t)
                memcpy(o_out + ((r0 + t) * H + h) * (int64_t)dv, oo + t * dv, sizeof(double) * dv);
            if (state_out) memcpy(state_out + (int64_t)u * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        }
        free(S); free(qq); free(kk); free(vv); free(aa); free(bb); free(oo); free(work);
    }
    return bad ? -2 : 0;
}
