/*
 * FP64 reference for the Mamba-2 SSD selective scan and its per-token decode step.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call this
 * file: only the test suite, the smoke check and the benchmark's CPU-baseline leg use
 * it. It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (the recurrence the SSD pages define):
 *   per sequence s and head h, with group g = h / (H / G)      (B/C shared by groups
 *   of heads, as keys/values are in grouped-query attention: JAX Nemotron 3 Nano page,
 *   NemotronConfig `mamba_ngroups`):
 *     dt_t   = softplus(dt_raw[t,h] + dt_bias[h])              (RL-Kernel issue page,
 *                                                               Figure 2: softplus of dt plus its bias)
 *     h_t    = exp(dt_t * A[h]) * h_{t-1} + dt_t * x_t B_t^T   (the SSD recurrence, FP32
 *                                                               state: RL-Kernel issue §1)
 *     y_t[p] = sum_n C_t[n] h_t[p][n] + D[h] x_t[p]            (D skip: JAX page,
 *                                                               "Key Components")
 *   with h_0 = the caller's initial state (or zero). The state is stored [P][N]
 *   (the transpose of B x^T), N contiguous; the arithmetic is unchanged.
 *
 * Inputs are read exactly as the GPU receives them (float32, or bf16 bit patterns
 * widened to double) and every operation is done in double precision, token by
 * token, in the order the recurrence is written. No chunking, blocking or
 * reordering: the chunked algorithm is the thing under test.
 *
 * Also here: the quadratic closed form of the same map (brute force, for tiny
 * inputs), which pins the recurrence without sharing its loop structure.
 *
 * Threads: independent (sequence, head) pairs run on separate pthreads; each
 * recurrence stays sequential.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Deliberate-mistake switch for the oracle's own pin tests: a test sets it to a
 * nonzero code, checks that some pin now fails, and sets it back to 0. Code 0 is
 * the only value the oracle is ever used with for parity. */
static int g_mutation = 0;
void oracle_set_mutation(int m) { g_mutation = m; }
int oracle_get_mutation(void) { return g_mutation; }

enum {
    MUT_NONE = 0,
    MUT_DROP_D = 1,         /* y without the D skip */
    MUT_GROUP_MOD = 2,      /* head -> group as h % G instead of contiguous blocks */
    MUT_NO_SOFTPLUS = 3,    /* dt = dt_raw + dt_bias */
    MUT_DECAY_NO_DT = 4,    /* decay exp(A) instead of exp(dt*A) */
    MUT_INPUT_NO_DT = 5,    /* input term x B^T without dt */
    MUT_Y_OLD_STATE = 6,    /* y from h_{t-1} instead of h_t */
    MUT_SWAP_BC = 7,        /* C used where B belongs */
    MUT_INIT_IGNORED = 8,   /* initial state dropped */
};

static double widen(const void* p, int dtype, int64_t i)
{
    if (dtype == 0) return (double)((const float*)p)[i];
    uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* softplus(z) = log(1 + e^z), evaluated without overflow for large z. */
double oracle_softplus(double z)
{
    if (g_mutation == MUT_NO_SOFTPLUS) return z;
    return z > 0 ? z + log1p(exp(-z)) : log1p(exp(z));
}

static int group_of(int h, int H, int G)
{
    if (g_mutation == MUT_GROUP_MOD) return h % G;
    return h / (H / G);
}

typedef struct {
    /* problem */
    int64_t nseq;
    const int64_t* seq_off;  /* [nseq+1] packed token offsets */
    int H, P, G, N, dtype;
    const void* x;           /* [T,H,P] */
    const float* dt_raw;     /* [T,H] */
    const float* dt_bias;    /* [H] */
    const float* A;          /* [H] */
    const void* B;           /* [T,G,N] */
    const void* C;           /* [T,G,N] */
    const float* D;          /* [H] */
    const double* init;      /* [nseq,H,P,N] or NULL */
    /* work list */
    int64_t npairs;
    const int64_t* pairs;    /* [npairs][2] = (seq, head) */
    const int64_t* y_off;    /* [npairs] offset (in doubles) of each pair's y block */
    double* y;               /* per pair: [len][P] */
    double* final_state;     /* per pair: [P][N], or NULL */
    int64_t snap;            /* snapshot interval in tokens (0: none) */
    const int64_t* snap_off; /* per pair: where its [len/snap][P][N] snapshots start in snaps */
    double* snaps;
    /* threading */
    int64_t next;
    pthread_mutex_t lock;
} scan_job;

/* One (sequence, head) recurrence over its tokens. */
static void scan_pair(const scan_job* j, int64_t k)
{
    const int64_t s = j->pairs[2 * k], h = j->pairs[2 * k + 1];
    const int H = j->H, P = j->P, G = j->G, N = j->N;
    const int g = group_of((int)h, H, G);
    const int64_t t0 = j->seq_off[s], t1 = j->seq_off[s + 1];
    double* st = (double*)calloc((size_t)P * N, sizeof(double));
    double* prev = (double*)malloc((size_t)P * N * sizeof(double));
    if (j->init && g_mutation != MUT_INIT_IGNORED)
        memcpy(st, j->init + ((s * H + h) * (int64_t)P * N), (size_t)P * N * sizeof(double));
    double* yo = j->y ? j->y + j->y_off[k] : NULL;
    const double A = j->A[h], Dh = j->D[h], bias = j->dt_bias[h];

    for (int64_t t = t0; t < t1; t++) {
        const double dt = oracle_softplus((double)j->dt_raw[t * H + h] + bias);
        const double decay = exp((g_mutation == MUT_DECAY_NO_DT ? 1.0 : dt) * A);
        const double win = (g_mutation == MUT_INPUT_NO_DT) ? 1.0 : dt;
        const void* Bsrc = (g_mutation == MUT_SWAP_BC) ? j->C : j->B;
        if (g_mutation == MUT_Y_OLD_STATE) memcpy(prev, st, (size_t)P * N * sizeof(double));
        for (int p = 0; p < P; p++) {
            const double xp = widen(j->x, j->dtype, (t * H + h) * P + p);
            for (int n = 0; n < N; n++) {
                const double bn = widen(Bsrc, j->dtype, (t * G + g) * N + n);
                st[p * N + n] = decay * st[p * N + n] + win * xp * bn;
            }
        }
        if (yo) {
            const double* hs = (g_mutation == MUT_Y_OLD_STATE) ? prev : st;
            for (int p = 0; p < P; p++) {
                double acc = 0.0;
                for (int n = 0; n < N; n++)
                    acc += widen(j->C, j->dtype, (t * G + g) * N + n) * hs[p * N + n];
                if (g_mutation != MUT_DROP_D)
                    acc += Dh * widen(j->x, j->dtype, (t * H + h) * P + p);
                yo[(t - t0) * P + p] = acc;
            }
        }
        /* snapshot: the state after the first m * snap tokens of the sequence */
        if (j->snap > 0 && (t - t0 + 1) % j->snap == 0)
            memcpy(j->snaps + j->snap_off[k] + ((t - t0 + 1) / j->snap - 1) * (int64_t)P * N, st,
                   (size_t)P * N * sizeof(double));
    }
    if (j->final_state) memcpy(j->final_state + k * (int64_t)P * N, st, (size_t)P * N * sizeof(double));
    free(st);
    free(prev);
}

static void* scan_worker(void* arg)
{
    scan_job* j = (scan_job*)arg;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        int64_t k = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (k >= j->npairs) break;
        scan_pair(j, k);
    }
    return NULL;
}

/*
 * Run the recurrence for the listed (sequence, head) pairs.
 *   seq_off[nseq+1]: packed token offsets of each sequence (dense batch: s*L).
 *   dtype: 0 = float32 x/B/C, 1 = bf16 bit patterns.
 *   init: [nseq,H,P,N] doubles or NULL (zero initial state).
 *   y_off[k]: where pair k's [len][P] output block starts in y (NULL y: skip y).
 *   final_state: [npairs][P][N] or NULL.
 *   snap, snap_off, snaps: if snap > 0, pair k's state after the first m * snap tokens
 *     of its sequence (m = 1 .. len / snap) goes to snaps + snap_off[k] + (m-1)*P*N.
 * Returns 0, or -1 on a bad argument. oracle_ssd_scan is the same without snapshots.
 */
int oracle_ssd_scan_snapshots(int64_t nseq, const int64_t* seq_off, int H, int P, int G, int N, int dtype,
                              const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                              const void* B, const void* C, const float* D, const double* init,
                              int64_t npairs, const int64_t* pairs, const int64_t* y_off, double* y,
                              double* final_state, int64_t snap, const int64_t* snap_off, double* snaps,
                              int nthreads)
{
    if (H <= 0 || G <= 0 || H % G != 0 || P <= 0 || N <= 0 || nseq < 0 || snap < 0) return -1;
    if (snap > 0 && (!snap_off || !snaps)) return -1;
    for (int64_t k = 0; k < npairs; k++)
        if (pairs[2 * k] < 0 || pairs[2 * k] >= nseq || pairs[2 * k + 1] < 0 || pairs[2 * k + 1] >= H)
            return -1;
    scan_job j = {nseq, seq_off, H, P, G, N, dtype, x, dt_raw, dt_bias, A, B, C, D, init,
                  npairs, pairs, y_off, y, final_state, snap, snap_off, snaps, 0};
    pthread_mutex_init(&j.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    for (int i = 0; i < nthreads; i++) pthread_create(&th[i], NULL, scan_worker, &j);
    for (int i = 0; i < nthreads; i++) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&j.lock);
    return 0;
}

int oracle_ssd_scan(int64_t nseq, const int64_t* seq_off, int H, int P, int G, int N, int dtype,
                    const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                    const void* B, const void* C, const float* D, const double* init,
                    int64_t npairs, const int64_t* pairs, const int64_t* y_off, double* y,
                    double* final_state, int nthreads)
{
    return oracle_ssd_scan_snapshots(nseq, seq_off, H, P, G, N, dtype, x, dt_raw, dt_bias, A, B, C, D, init,
                                     npairs, pairs, y_off, y, final_state, 0, NULL, NULL, nthreads);
}

/*
 * One decode step for every (sequence, head): the same recurrence applied to a
 * single token per sequence. state: [nseq,H,P,N] doubles, updated in place.
 * x [nseq,H,P], dt_raw [nseq,H], B/C [nseq,G,N]; y [nseq,H,P] doubles.
 */
int oracle_state_update(int64_t nseq, int H, int P, int G, int N, int dtype, double* state,
                        const void* x, const float* dt_raw, const float* dt_bias, const float* A,
                        const void* B, const void* C, const float* D, double* y)
{
    if (H <= 0 || G <= 0 || H % G != 0 || P <= 0 || N <= 0 || nseq < 0) return -1;
    for (int64_t s = 0; s < nseq; s++)
        for (int h = 0; h < H; h++) {
            const int g = group_of(h, H, G);
            const double dt = oracle_softplus((double)dt_raw[s * H + h] + dt_bias[h]);
            const double decay = exp((g_mutation == MUT_DECAY_NO_DT ? 1.0 : dt) * A[h]);
            const double win = (g_mutation == MUT_INPUT_NO_DT) ? 1.0 : dt;
            double* st = state + (s * H + h) * (int64_t)P * N;
            for (int p = 0; p < P; p++) {
                const double xp = widen(x, dtype, (s * H + h) * P + p);
                double acc = 0.0;
                for (int n = 0; n < N; n++) {
                    st[p * N + n] = decay * st[p * N + n] + win * xp * widen(B, dtype, (s * G + g) * N + n);
                    acc += widen(C, dtype, (s * G + g) * N + n) * st[p * N + n];
                }
                if (g_mutation != MUT_DROP_D) acc += D[h] * xp;
                y[(s * H + h) * P + p] = acc;
            }
        }
    return 0;
}

/*
 * Quadratic closed form of the same map (brute force; tiny inputs only):
 *   y_t = sum_{s<=t} (C_t . B_s) exp(sum_{s<r<=t} dt_r A) dt_s x_s
 *         + exp(sum_{r<=t} dt_r A) (C_t . h0) + D x_t
 *   h_L = exp(sum_{r<=L} dt_r A) h0 + sum_s exp(sum_{s<r<=L} dt_r A) dt_s x_s B_s^T
 * Every decay sum is taken afresh from its definition (no running products).
 * Dense layout only: x [L,H,P], dt_raw [L,H], B/C [L,G,N] of ONE sequence,
 * h0 [H,P,N] or NULL; outputs y [L,H,P] and hL [H,P,N] (doubles).
 */
int oracle_closed_form(int L, int H, int P, int G, int N, int dtype, const void* x,
                       const float* dt_raw, const float* dt_bias, const float* A, const void* B,
                       const void* C, const float* D, const double* h0, double* y, double* hL)
{
    if (H <= 0 || G <= 0 || H % G != 0 || P <= 0 || N <= 0 || L < 0) return -1;
    double* dt = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * H);
    for (int t = 0; t < L; t++)
        for (int h = 0; h < H; h++) dt[t * H + h] = oracle_softplus((double)dt_raw[t * H + h] + dt_bias[h]);
    for (int h = 0; h < H; h++) {
        const int g = group_of(h, H, G);
        for (int t = 0; t < L; t++)
            for (int p = 0; p < P; p++) {
                double acc = 0.0;
                for (int s = 0; s <= t; s++) {
                    double seg = 0.0;
                    for (int r = s + 1; r <= t; r++) seg += dt[r * H + h] * A[h];
                    double cb = 0.0;
                    for (int n = 0; n < N; n++)
                        cb += widen(C, dtype, (t * G + g) * N + n) * widen(B, dtype, (s * G + g) * N + n);
                    acc += cb * exp(seg) * dt[s * H + h] * widen(x, dtype, (s * H + h) * P + p);
                }
                if (h0) {
                    double seg = 0.0;
                    for (int r = 0; r <= t; r++) seg += dt[r * H + h] * A[h];
                    double ch = 0.0;
                    for (int n = 0; n < N; n++)
                        ch += widen(C, dtype, (t * G + g) * N + n) * h0[(h * P + p) * N + n];
                    acc += exp(seg) * ch;
                }
                acc += D[h] * widen(x, dtype, (t * H + h) * P + p);
                y[(t * H + h) * P + p] = acc;
            }
        for (int p = 0; p < P; p++)
            for (int n = 0; n < N; n++) {
                double acc = 0.0;
                if (h0) {
                    double seg = 0.0;
                    for (int r = 0; r < L; r++) seg += dt[r * H + h] * A[h];
                    acc += exp(seg) * h0[(h * P + p) * N + n];
                }
                for (int s = 0; s < L; s++) {
                    double seg = 0.0;
                    for (int r = s + 1; r < L; r++) seg += dt[r * H + h] * A[h];
                    acc += exp(seg) * dt[s * H + h] * widen(x, dtype, (s * H + h) * P + p) *
                           widen(B, dtype, (s * G + g) * N + n);
                }
                hL[(h * P + p) * N + n] = acc;
            }
    }
    free(dt);
    return 0;
}
