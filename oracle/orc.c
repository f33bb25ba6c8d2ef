/*
 * Attention oracle: plain, slow, obviously-correct CPU reference in fp64.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may load or call this
 * file: only the tests, the smoke check and the benchmark's CPU-baseline leg
 * use it. It shares no code, header or constant with the CUDA library.
 *
 * Everything is written from the defining formulas, in the pages' notation:
 *   - scores s_ij = scale * <q_i, k_j>, scale = 1/sqrt(D), log-sum-exp over the
 *     keys, output = softmax(scores) * V  ("DeDLOC Guide: Decentralized
 *     Long-Context Attention", Step 3, the local attention step that returns the
 *     output together with its log-sum-exp);
 *   - causal masking: key j is visible to query i iff j <= i in GLOBAL token
 *     positions ("DeDLOC Guide", Best Practices table, Causal Mask Handling);
 *     with a sliding window of W keys (axolotl-ringmaster README, Status:
 *     sliding-window attention via flash's `window`), also j > i - W;
 *   - packed variable-length documents (axolotl-ringmaster README, Status:
 *     packing / varlen): with boundaries cu[0] = 0 <= cu[1] <= ... <= cu[n] = S,
 *     key j is visible to query i only if both lie in the same document
 *     [cu[d], cu[d+1]) (and the causal and window rules hold);
 *   - the merge of two partial (O, LSE) pairs by max-shifted exponential weights
 *     ("DeDLOC Guide", section 3 "Online Softmax Rescaling Across Decentralized
 *     Ranks", the alpha/beta equations, in the normalised-output form of Step 3);
 *   - the ring: each rank keeps its query block and sees the key/value block of
 *     owner r = (i - t) mod P at step t ("Sequence Parallelism III: Ring
 *     Attention for Context That Does Not Fit", duoan.github.io LLM tag index);
 *   - the load-balanced (zigzag) chunk order: 2P chunks, rank i holding chunks i
 *     and 2P-1-i ("context parallelism", Last Dictionary: causal imbalance is
 *     handled by reordering chunks; axolotl-ringmaster README, Layout,
 *     balancers.py head_tail index generation).
 *
 * Inputs are fp64 arrays in NATURAL token order, one head at a time
 * (q, k, v, dout are [S, D] row-major). bf16 inputs are widened exactly before
 * the call. Rows are evaluated independently (OpenMP over rows); every sum is a
 * plain left-to-right loop.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#define ORC_ORDER_CONTIGUOUS 0
#define ORC_ORDER_ZIGZAG 1

/* ------------------------------------------------------------------------- */
/* Token order of the ring: which natural position rank-major slot s holds.   */
/* ------------------------------------------------------------------------- */

/* Rank-major layout: rank 0's L = S/P tokens, then rank 1's, and so on.
 * Contiguous order: rank i holds natural tokens [i*L, (i+1)*L).
 * Zigzag order: the sequence is cut into 2P chunks of c = S/(2P); rank i holds
 * chunk i followed by chunk 2P-1-i. Returns -1 on bad arguments. */
int64_t orc_rank_major_position(int64_t S, int64_t P, int order, int64_t s)
{
    if (P <= 0 || S <= 0 || s < 0 || s >= S) return -1;
    if (order == ORC_ORDER_CONTIGUOUS) {
        if (S % P) return -1;
        return s; /* rank i's local token u sits at slot i*L+u = natural i*L+u */
    }
    if (order != ORC_ORDER_ZIGZAG || S % (2 * P)) return -1;
    int64_t L = S / P, c = S / (2 * P);
    int64_t i = s / L, u = s % L;
    if (u < c) return i * c + u;
    return (2 * P - 1 - i) * c + (u - c);
}

/* Rank (0..P-1) that holds natural position x. */
static int64_t rank_of_position(int64_t S, int64_t P, int order, int64_t x)
{
    if (order == ORC_ORDER_CONTIGUOUS) return x / (S / P);
    int64_t c = S / (2 * P), chunk = x / c;
    return chunk < P ? chunk : 2 * P - 1 - chunk;
}

/* Owner of the key/value block that rank i holds at ring step t: blocks move
 * one rank forward per step (r -> r+1), so it is (i - t) mod P. */
int64_t orc_ring_owner(int64_t P, int64_t i, int64_t t)
{
    return ((i - t) % P + P) % P;
}

/* Whether natural key position j belongs to rank r's block. */
static int rank_holds(int64_t S, int64_t P, int order, int64_t r, int64_t j)
{
    return rank_of_position(S, P, order, j) == r;
}

/* ------------------------------------------------------------------------- */
/* Dense attention of one head, the plain definition.                         */
/* ------------------------------------------------------------------------- */

/* Which keys a query sees: S tokens, causal flag, window W (0 = none) and the
 * document boundaries cu[0..ndoc] (cu = NULL: one document of all S tokens). */
typedef struct {
    int64_t S;
    int causal;
    int64_t window;
    const int64_t* cu;
    int64_t ndoc;
} orc_mask;

/* Visible keys of the query at position i: [lo, hi). The query's document
 * [cu[d], cu[d+1]) bounds it; causal: j <= i; window of W > 0 keys: j > i - W. */
static void visible_range(int64_t i, const orc_mask* mk, int64_t* lo, int64_t* hi)
{
    *lo = 0;
    *hi = mk->S;
    if (mk->cu) {
        for (int64_t d = 0; d < mk->ndoc; ++d)
            if (mk->cu[d] <= i && i < mk->cu[d + 1]) {
                *lo = mk->cu[d];
                *hi = mk->cu[d + 1];
                break;
            }
    }
    if (!mk->causal) return;
    if (i + 1 < *hi) *hi = i + 1;
    if (mk->window > 0 && i - mk->window + 1 > *lo) *lo = i - mk->window + 1;
}

static double dot(const double* a, const double* b, int64_t D)
{
    double acc = 0.0;
    for (int64_t d = 0; d < D; ++d) acc += a[d] * b[d];
    return acc;
}

/* For query at natural position i over the visible key set
 * V(i) = the query's document (non-causal), its part j <= i (causal), and with
 * a window of W > 0 keys only j > i - W; S keys in k, v:
 *   LSE_i = m + ln sum_j exp(s_ij - m),  m = max_j s_ij
 *   O_i   = sum_j exp(s_ij - LSE_i) v_j
 * scratch must hold S doubles. */
static void attend_row(const double* qi, const double* k, const double* v, int64_t D,
                       const orc_mask* mk, double scale, int64_t i, double* s, double* o,
                       double* lse)
{
    int64_t j0, n;
    visible_range(i, mk, &j0, &n);
    double m = -INFINITY;
    for (int64_t j = j0; j < n; ++j) {
        s[j] = scale * dot(qi, k + j * D, D);
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (int64_t j = j0; j < n; ++j) sum += exp(s[j] - m);
    double L = m + log(sum);
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = j0; j < n; ++j) {
        double p = exp(s[j] - L);
        const double* vj = v + j * D;
        for (int64_t d = 0; d < D; ++d) o[d] += p * vj[d];
    }
    *lse = L;
}

/* q holds nrows query rows (row-major [nrows, D]); rows[r] is the natural
 * position of q row r. k, v hold the Sk keys 0..Sk-1. The mask: causal flag,
 * window (0 = none), document boundaries cu[0..ndoc] (NULL = one document). */
void orc_attn_fwd_head(const double* q, const double* k, const double* v, int64_t Sk,
                       int64_t D, int causal, int64_t window, const int64_t* cu, int64_t ndoc,
                       double scale, const int64_t* rows, int64_t nrows, double* o, double* lse)
{
    const orc_mask mk = {Sk, causal, window, cu, ndoc};
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)Sk);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrows; ++r)
            attend_row(q + r * D, k, v, D, &mk, scale, rows[r], s, o + r * D, lse + r);
        free(s);
    }
}

/* ------------------------------------------------------------------------- */
/* Merge of two partial results.                                              */
/* ------------------------------------------------------------------------- */

/* (O_a, LSE_a) and (O_b, LSE_b) are softmax-normalised partials over disjoint
 * key sets. With M = max(LSE_a, LSE_b), wa = exp(LSE_a - M), wb = exp(LSE_b - M):
 *   O = (wa O_a + wb O_b) / (wa + wb),  LSE = M + ln(wa + wb).
 * A partial over an empty key set is (0, -inf); when both are empty the result
 * is (0, -inf) (the printed formula would take exp(-inf - -inf) = NaN there). */
static void merge_pair(double* o_acc, double* lse_acc, const double* o_part,
                       double lse_part, int64_t D)
{
    double a = *lse_acc, b = lse_part;
    double M = a > b ? a : b;
    if (M == -INFINITY) {
        for (int64_t d = 0; d < D; ++d) o_acc[d] = 0.0;
        *lse_acc = -INFINITY;
        return;
    }
    double wa = exp(a - M), wb = exp(b - M);
    for (int64_t d = 0; d < D; ++d) o_acc[d] = (wa * o_acc[d] + wb * o_part[d]) / (wa + wb);
    *lse_acc = M + log(wa + wb);
}

void orc_lse_merge(double* o_acc, double* lse_acc, const double* o_part,
                   const double* lse_part, int64_t rows, int64_t D)
{
    for (int64_t r = 0; r < rows; ++r)
        merge_pair(o_acc + r * D, lse_acc + r, o_part + r * D, lse_part[r], D);
}

/* ------------------------------------------------------------------------- */
/* Ring-structured forward: per-step partials over one owner's keys, merged.  */
/* ------------------------------------------------------------------------- */

/* q holds nrows query rows; rows[r] is the natural position of q row r.
 * Query row at natural position x lives on rank i. At step t = 0..P-1 rank i
 * holds the key/value block of owner r = (i - t) mod P (blocks move one rank
 * forward per step). The step's partial is attention over the keys of owner r
 * that x may see; an empty set gives (0, -inf). Partials are merged in step
 * order with merge_pair. The result equals the dense definition exactly up to
 * rounding, which the tests check. */
void orc_ring_fwd_head(const double* q, const double* k, const double* v, int64_t S,
                       int64_t D, int causal, int64_t window, const int64_t* cu, int64_t ndoc,
                       double scale, int64_t P, int order, const int64_t* rows, int64_t nrows,
                       double* o, double* lse)
{
    const orc_mask mk = {S, causal, window, cu, ndoc};
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        double* op = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 4)
        for (int64_t rr = 0; rr < nrows; ++rr) {
            int64_t x = rows[rr];
            int64_t i = rank_of_position(S, P, order, x);
            int64_t jlo, jhi;
            visible_range(x, &mk, &jlo, &jhi);
            double* oacc = o + rr * D;
            double lacc = -INFINITY;
            for (int64_t d = 0; d < D; ++d) oacc[d] = 0.0;
            for (int64_t t = 0; t < P; ++t) {
                int64_t r = orc_ring_owner(P, i, t);
                /* partial over visible keys of owner r */
                double m = -INFINITY;
                for (int64_t j = 0; j < S; ++j) {
                    if (!rank_holds(S, P, order, r, j) || j < jlo || j >= jhi) continue;
                    s[j] = scale * dot(q + rr * D, k + j * D, D);
                    if (s[j] > m) m = s[j];
                }
                double lpart = -INFINITY;
                for (int64_t d = 0; d < D; ++d) op[d] = 0.0;
                if (m != -INFINITY) {
                    double sum = 0.0;
                    for (int64_t j = 0; j < S; ++j) {
                        if (!rank_holds(S, P, order, r, j) || j < jlo || j >= jhi) continue;
                        sum += exp(s[j] - m);
                    }
                    lpart = m + log(sum);
                    for (int64_t j = 0; j < S; ++j) {
                        if (!rank_holds(S, P, order, r, j) || j < jlo || j >= jhi) continue;
                        double p = exp(s[j] - lpart);
                        for (int64_t d = 0; d < D; ++d) op[d] += p * v[j * D + d];
                    }
                }
                merge_pair(oacc, &lacc, op, lpart, D);
            }
            lse[rr] = lacc;
        }
        free(op);
        free(s);
    }
}

/* ------------------------------------------------------------------------- */
/* Backward of one head: analytic gradients of L = sum(dO * O).               */
/* ------------------------------------------------------------------------- */

/* With P_ij = exp(s_ij - LSE_i) over visible keys and Delta_i = <dO_i, O_i>:
 *   dV_j = sum_i P_ij dO_i
 *   dS_ij = P_ij (<dO_i, v_j> - Delta_i)
 *   dQ_i = scale * sum_j dS_ij k_j
 *   dK_j = scale * sum_i dS_ij q_i
 * dQ is produced for the query rows `qrows`, dK/dV for the key rows `krows`
 * (natural positions). For one head; a KV head shared by G query heads gets the
 * sum of its query heads' dK/dV, which the caller forms. */
void orc_attn_bwd_head(const double* q, const double* k, const double* v,
                       const double* dout, int64_t S, int64_t D, int causal, int64_t window,
                       const int64_t* cu, int64_t ndoc, double scale, const int64_t* qrows,
                       int64_t nq, double* dq, const int64_t* krows, int64_t nk, double* dk,
                       double* dv)
{
    const orc_mask mk = {S, causal, window, cu, ndoc};
    /* dQ rows: one forward row each, then the sum over its keys. */
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        double* oi = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nq; ++r) {
            int64_t i = qrows[r];
            double L;
            attend_row(q + i * D, k, v, D, &mk, scale, i, s, oi, &L);
            double delta = dot(dout + i * D, oi, D);
            int64_t j0, n;
            visible_range(i, &mk, &j0, &n);
            double* g = dq + r * D;
            for (int64_t d = 0; d < D; ++d) g[d] = 0.0;
            for (int64_t j = j0; j < n; ++j) {
                double p = exp(s[j] - L);
                double ds = p * (dot(dout + i * D, v + j * D, D) - delta);
                for (int64_t d = 0; d < D; ++d) g[d] += ds * k[j * D + d];
            }
            for (int64_t d = 0; d < D; ++d) g[d] *= scale;
        }
        free(oi);
        free(s);
    }
    if (nk == 0) return;

    /* dK/dV rows need LSE_i and Delta_i of every query row that sees them. */
    double* lse_all = (double*)malloc(sizeof(double) * (size_t)S);
    double* delta_all = (double*)malloc(sizeof(double) * (size_t)S);
    int64_t jmin = S;
    for (int64_t r = 0; r < nk; ++r) if (krows[r] < jmin) jmin = krows[r];
    int64_t i0 = causal ? jmin : 0; /* rows i < jmin never see a requested key */
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)S);
        double* oi = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = i0; i < S; ++i) {
            attend_row(q + i * D, k, v, D, &mk, scale, i, s, oi, &lse_all[i]);
            delta_all[i] = dot(dout + i * D, oi, D);
        }
        free(oi);
        free(s);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nk; ++r) {
        int64_t j = krows[r];
        double* gk = dk + r * D;
        double* gv = dv + r * D;
        for (int64_t d = 0; d < D; ++d) { gk[d] = 0.0; gv[d] = 0.0; }
        /* every query row whose visible range holds key j */
        for (int64_t i = i0; i < S; ++i) {
            int64_t lo, hi;
            visible_range(i, &mk, &lo, &hi);
            if (j < lo || j >= hi) continue;
            double sij = scale * dot(q + i * D, k + j * D, D);
            double p = exp(sij - lse_all[i]);
            double ds = p * (dot(dout + i * D, v + j * D, D) - delta_all[i]);
            for (int64_t d = 0; d < D; ++d) {
                gv[d] += p * dout[i * D + d];
                gk[d] += ds * q[i * D + d];
            }
        }
        for (int64_t d = 0; d < D; ++d) gk[d] *= scale;
    }
    free(delta_all);
    free(lse_all);
}

/* Threads OpenMP will use (reported next to timings). */
int orc_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
}
