/*
 * gdn_oracle.c -- CPU oracle for gated-delta-rule tree verification.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA library, and the CUDA library
 * never calls it.
 *
 * What it computes (plain, slow, double precision, no blocking or reordering):
 *
 * The gated delta rule of Gated DeltaNet (the recurrence behind
 * ggml_gated_delta_net, named in the GreenGames post, "TL;DR" and "Why the
 * experiment exists"; formula as published in Yang, Kautz & Hatamizadeh,
 * "Gated Delta Networks: Improving Mamba2 with Delta Rule", eq. for S_t),
 * run over a draft tree: every node n takes the state of its parent p
 * (tree spec-decode on a GDN hybrid, dflash-caddtree-integrations README,
 * "What's in here", DDTree row):
 *
 *     a_n = exp(g_n),   b_n = beta_n
 *     S_n = a_n * S_p + b_n * (v_n - a_n * S_p k_n) k_n^T        (d_v x d_k)
 *     o_n = scale * S_n q_n                                        (d_v)
 *
 * The root (node 0, parent -1) takes S_p = state_in.  The v-head h reads
 * k-head h / G with G = H_v / H_k (contiguous groups).  Each node's state is
 * persisted, rounded to the persisted dtype (fp32, or f16 round-to-nearest-
 * even: the f16 intermediate cache of the GreenGames post, "Key wins"); the
 * recurrence itself always continues from the unrounded state.  Commit copies
 * the persisted state of the last node of the accepted root-to-leaf path
 * (the persist-write kernel of the same section) into state_out.
 *
 * Pins: every function here is checked by tests against closed forms and
 * invariants (identity, reset, delta-rule write, linearity, GQA grouping,
 * path composition, a hand-worked example; for the gate maps, their values
 * at ln 3 and 0, the softplus and sigmoid symmetries and the limits), never
 * against itself.
 *
 * Layouts, row-major with the last index contiguous:
 *   q, k        [B][N][H_k][d_k]
 *   v           [B][N][H_v][d_v]
 *   g, beta     [B][N][H_v]
 *   parent      [B][N]                int32, parent[b][0] = -1, parent[b][n] < n
 *   state_in    [B][H_v][d_v][d_k]
 *   out         [B][N][H_v][d_v]
 *   states      [B][N][H_v][d_v][d_k]
 *   accept_path [B][max_path_len]     int32
 *   accept_len  [B]                   int32
 *   state_out   [B][H_v][d_v][d_k]
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_OK = 0, ORACLE_ERR_INVALID_ARG = 1, ORACLE_ERR_BAD_TREE = 3,
       ORACLE_ERR_BAD_PATH = 4 };
enum { ORACLE_STATE_F32 = 0, ORACLE_STATE_F16 = 1 };

/* Round a double to the persisted dtype and widen it back to double.
 * fp32: C conversion (round to nearest even).  f16: _Float16 conversion
 * (IEEE binary16, round to nearest even, straight from double). */
double gdn_oracle_round(int state_dtype, double x)
{
    if (state_dtype == ORACLE_STATE_F16)
        return (double)(_Float16)x;
    return (double)(float)x;
}

void gdn_oracle_round_array(int state_dtype, const double* x, double* y, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        y[i] = gdn_oracle_round(state_dtype, x[i]);
}

/* parent[0] = -1 and 0 <= parent[n] < n for n >= 1. */
/* L2 normalisation of n rows of length d, in place: x / sqrt(sum_j x_j^2),
 * with no epsilon (a zero row becomes NaN).  This is the workloads' input
 * preparation of q and k ("then L2-normalised per head", per node and
 * head over d_k), which the library can fuse into its verify kernels. */
void gdn_oracle_l2norm_rows(double* x, int64_t n, int d)
{
    for (int64_t r = 0; r < n; ++r) {
        double* row = x + r * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j)
            ss += row[j] * row[j];
        const double nrm = sqrt(ss);
        for (int j = 0; j < d; ++j)
            row[j] = row[j] / nrm;
    }
}

/* The gate maps of the workloads' input recipe, in double: from raw
 * pre-activations x and y, the decay's log g = -softplus(x) = -log(1 + e^x)
 * and the write strength beta = sigmoid(y) = 1 / (1 + e^-y) (the library's
 * GDN_FLAG_GATES applies them inside its verify kernels).  softplus is taken
 * as max(x, 0) + log1p(e^-|x|) and sigmoid through e^-|y|, forms that
 * neither overflow nor cancel: x = +inf gives g = -inf (a = 0, a reset),
 * x = -inf gives g = 0 (a = 1); y = +-inf gives beta = 1 or 0; NaN stays NaN. */
void gdn_oracle_gates(const double* x, const double* y, double* g, double* beta, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        const double xi = x[i], yi = y[i];
        g[i] = isnan(xi) ? xi : -(fmax(xi, 0.0) + log1p(exp(-fabs(xi))));
        if (isnan(yi))
            beta[i] = yi;
        else if (yi >= 0.0)
            beta[i] = 1.0 / (1.0 + exp(-yi));
        else
            beta[i] = exp(yi) / (1.0 + exp(yi));
    }
}

int gdn_oracle_check_tree(int n_nodes, const int32_t* parent)
{
    if (n_nodes < 1 || parent[0] != -1)
        return ORACLE_ERR_BAD_TREE;
    for (int n = 1; n < n_nodes; ++n)
        if (parent[n] < 0 || parent[n] >= n)
            return ORACLE_ERR_BAD_TREE;
    return ORACLE_OK;
}

typedef struct {
    int B, N, Hk, Hv, dk, dv, state_dtype;
    double scale;
    const double *q, *k, *v, *g, *beta, *state_in;
    const int32_t* parent;
    double *out, *states, *exact;
    int next_pair;          /* work counter over (b, h) pairs */
    pthread_mutex_t lock;
} verify_job;

/* One (sequence b, v-head h): walk the nodes in index order (a topological
 * order, since parent[n] < n) and apply the recurrence literally. */
static void verify_pair(verify_job* J, int b, int h, double* S)
{
    const int N = J->N, Hk = J->Hk, Hv = J->Hv, dk = J->dk, dv = J->dv;
    const int G = Hv / Hk;
    const int hk = h / G;
    const size_t SS = (size_t)dv * dk;
    double* Sp_scaled = (double*)malloc(SS * sizeof(double));
    double* w = (double*)malloc((size_t)dv * sizeof(double));
    double* u = (double*)malloc((size_t)dv * sizeof(double));
    for (int n = 0; n < N; ++n) {
        const int p = J->parent[(size_t)b * N + n];
        const double* Sp = (p < 0) ? J->state_in + ((size_t)b * Hv + h) * SS
                                   : S + (size_t)p * SS;
        const double* kn = J->k + (((size_t)b * N + n) * Hk + hk) * dk;
        const double* qn = J->q + (((size_t)b * N + n) * Hk + hk) * dk;
        const double* vn = J->v + (((size_t)b * N + n) * Hv + h) * dv;
        const double a = exp(J->g[((size_t)b * N + n) * Hv + h]);
        const double be = J->beta[((size_t)b * N + n) * Hv + h];
        double* Sn = S + (size_t)n * SS;
        /* S' = a * S_p */
        for (size_t e = 0; e < SS; ++e)
            Sp_scaled[e] = a * Sp[e];
        /* w = S' k ; u = beta * (v - w) */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j)
                acc += Sp_scaled[(size_t)i * dk + j] * kn[j];
            w[i] = acc;
            u[i] = be * (vn[i] - w[i]);
        }
        /* S_n = S' + u k^T */
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j)
                Sn[(size_t)i * dk + j] = Sp_scaled[(size_t)i * dk + j] + u[i] * kn[j];
        /* o_n = scale * S_n q */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j)
                acc += Sn[(size_t)i * dk + j] * qn[j];
            J->out[(((size_t)b * N + n) * Hv + h) * dv + i] = J->scale * acc;
        }
        /* persist: rounded copy; the recurrence keeps the exact S_n */
        double* dst = J->states + (((size_t)b * N + n) * Hv + h) * SS;
        for (size_t e = 0; e < SS; ++e)
            dst[e] = gdn_oracle_round(J->state_dtype, Sn[e]);
        if (J->exact) {
            double* ex = J->exact + (((size_t)b * N + n) * Hv + h) * SS;
            memcpy(ex, Sn, SS * sizeof(double));
        }
    }
    free(Sp_scaled);
    free(w);
    free(u);
}

static void* verify_worker(void* arg)
{
    verify_job* J = (verify_job*)arg;
    double* S = (double*)malloc((size_t)J->N * J->dv * J->dk * sizeof(double));
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int pair = J->next_pair++;
        pthread_mutex_unlock(&J->lock);
        if (pair >= J->B * J->Hv)
            break;
        verify_pair(J, pair / J->Hv, pair % J->Hv, S);
    }
    free(S);
    return NULL;
}

/* Tree verify.  Returns ORACLE_OK, ORACLE_ERR_INVALID_ARG or
 * ORACLE_ERR_BAD_TREE (then nothing is written).  ``exact`` may be NULL.
 * ``nthreads`` <= 1 runs on the calling thread. */
int gdn_oracle_verify(int B, int N, int Hk, int Hv, int dk, int dv, double scale,
                      int state_dtype, const double* q, const double* k, const double* v,
                      const double* g, const double* beta, const int32_t* parent,
                      const double* state_in, double* out, double* states, double* exact,
                      int nthreads)
{
    if (B < 0 || N < 1 || Hk < 1 || Hv < 1 || dk < 1 || dv < 1 || Hv % Hk != 0)
        return ORACLE_ERR_INVALID_ARG;
    if (state_dtype != ORACLE_STATE_F32 && state_dtype != ORACLE_STATE_F16)
        return ORACLE_ERR_INVALID_ARG;
    for (int b = 0; b < B; ++b)
        if (gdn_oracle_check_tree(N, parent + (size_t)b * N) != ORACLE_OK)
            return ORACLE_ERR_BAD_TREE;
    verify_job J;
    J.B = B; J.N = N; J.Hk = Hk; J.Hv = Hv; J.dk = dk; J.dv = dv;
    J.state_dtype = state_dtype; J.scale = scale;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.state_in = state_in;
    J.parent = parent; J.out = out; J.states = states; J.exact = exact;
    J.next_pair = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads <= 1) {
        verify_worker(&J);
    } else {
        pthread_t* th = (pthread_t*)malloc((size_t)nthreads * sizeof(pthread_t));
        for (int t = 0; t < nthreads; ++t)
            pthread_create(&th[t], NULL, verify_worker, &J);
        for (int t = 0; t < nthreads; ++t)
            pthread_join(th[t], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return ORACLE_OK;
}

/* accept_len in [1, N] and <= max_path_len; path[0] = 0;
 * parent[path[i]] = path[i-1] (which also bounds every entry in [1, N)). */
int gdn_oracle_check_path(int N, const int32_t* parent, const int32_t* path, int len,
                          int max_path_len)
{
    if (len < 1 || len > N || len > max_path_len)
        return ORACLE_ERR_BAD_PATH;
    if (path[0] != 0)
        return ORACLE_ERR_BAD_PATH;
    for (int i = 1; i < len; ++i) {
        if (path[i] < 1 || path[i] >= N)
            return ORACLE_ERR_BAD_PATH;
        if (parent[path[i]] != path[i - 1])
            return ORACLE_ERR_BAD_PATH;
    }
    return ORACLE_OK;
}

/* Commit: state_out[b] = persisted state of node path_b[len_b - 1].
 * ``states`` holds the persisted (already rounded) node states.  Every
 * sequence's path is checked first; on any bad path nothing is written and
 * ORACLE_ERR_BAD_PATH is returned. */
int gdn_oracle_commit(int B, int N, int Hv, int dk, int dv, const double* states,
                      const int32_t* parent, const int32_t* accept_path,
                      const int32_t* accept_len, int max_path_len, double* state_out)
{
    if (B < 0 || N < 1 || Hv < 1 || dk < 1 || dv < 1 || max_path_len < 1)
        return ORACLE_ERR_INVALID_ARG;
    for (int b = 0; b < B; ++b) {
        if (gdn_oracle_check_tree(N, parent + (size_t)b * N) != ORACLE_OK)
            return ORACLE_ERR_BAD_TREE;
        if (gdn_oracle_check_path(N, parent + (size_t)b * N,
                                  accept_path + (size_t)b * max_path_len, accept_len[b],
                                  max_path_len) != ORACLE_OK)
            return ORACLE_ERR_BAD_PATH;
    }
    const size_t per_seq = (size_t)Hv * dv * dk;
    for (int b = 0; b < B; ++b) {
        const int last = accept_path[(size_t)b * max_path_len + accept_len[b] - 1];
        memcpy(state_out + (size_t)b * per_seq, states + ((size_t)b * N + last) * per_seq,
               per_seq * sizeof(double));
    }
    return ORACLE_OK;
}
