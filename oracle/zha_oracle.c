/*
 * zha_oracle.c - plain float64 CPU oracle for Zyphra Hierarchical Attention (ZHA):
 * chunk/node summaries, tangent-plane estimates, top-down top-p routing, and exact
 * softmax attention over the attended token set.
 *
 * TEST INFRASTRUCTURE ONLY.  This library is loaded by the test-suite, by the
 * smoke check and by the CPU-baseline leg of the benchmark, nothing else.  It
 * shares no code, header or constant with the CUDA path.  It is deliberately slow:
 * every summary is computed from the raw tokens by its definition (no merging,
 * no blocking, no reordering), every cut sorts its candidates.
 *
 * Sources, cited by page and section:
 *  [fluxbbs] "Zyphra ZHA 稀疏注意力：8.2 万参数与 373 倍加速推算" (fluxbbs.com),
 *            section "树形索引是怎么搭的".
 *  [icwork]  ic.work article on ZHA, section "给 KV Cache 建一棵 B-Tree，在 256K 检索上打赢 MiniMax".
 *  [wqu]     "Zyphra发布层级注意力ZHA：稀疏搜索实现亚二次复杂度" (wqu.guru), sections
 *            "What is Zyphra Hierarchical Attention (ZHA)?", "Building the tree",
 *            "How does top-p routing pick tokens?".
 *  [abstract] "Subquadratic Attention with a Hierarchical Tree-Structured Indexer"
 *            (aitop.news, abstract).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - score scale s = 1/sqrt(d), no softcap;
 *  - the tangent plane of f(q) = log sum_t exp(s q.k_t) at q_r is
 *    lse_r + s (q - q_r).m_r with m_r the softmax-weighted mean of the keys
 *    (grad f(q_r) = s m_r), written as s q.m_r + b_r, b_r = lse_r - s q_r.m_r;
 *  - the same R reference queries serve every level; a level-l node covers the
 *    C^l consecutive tokens [i C^l, (i+1) C^l), only complete nodes exist;
 *  - top-p normalises over the current frontier only, orders candidates by
 *    (score descending, node index ascending) and keeps the shortest prefix whose
 *    cumulative mass is >= p (at least one node; p >= 1 keeps all);
 *  - attended set = {token 0} U tokens of kept level-1 chunks U tail [T C^L, N),
 *    a set (token 0 counted once); with no complete top node it is [0, N).
 *
 * Build: gcc -O3 -fopenmp -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

/* Attention score scale: the standard 1/sqrt(d) (pages silent; reading). */
static double score_scale(int d) { return 1.0 / sqrt((double)d); }

int zo_num_threads(void) { return omp_get_max_threads(); }

/*
 * Summary of the node made of tokens [t0, t1) of one KV head, for each reference
 * query q_r (fluxbbs.com, section 树形索引是怎么搭的, and wqu.guru, section Building the
 * tree: every reference query yields a tangent plane of the chunk's log attention mass):
 *   a_t   = s (q_r . k_t)
 *   lse_r = log sum_t exp(a_t)                       (computed max-shifted)
 *   m_r   = sum_t exp(a_t - lse_r) k_t               (softmax-weighted mean of keys)
 *   b_r   = lse_r - s (q_r . m_r)
 * K rows are K + t*d.  a is scratch of t1 - t0 doubles.
 */
static void node_summary(const double* K, int64_t t0, int64_t t1, int d,
                         const double* qref, int R, double* m, double* lse, double* b,
                         double* a)
{
    const double s = score_scale(d);
    for (int r = 0; r < R; ++r) {
        const double* q = qref + (int64_t)r * d;
        double mx = -INFINITY;
        for (int64_t t = t0; t < t1; ++t) {
            const double* k = K + t * d;
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += q[i] * k[i];
            a[t - t0] = s * dot;
            if (a[t - t0] > mx) mx = a[t - t0];
        }
        double z = 0.0;
        for (int64_t t = t0; t < t1; ++t) z += exp(a[t - t0] - mx);
        const double l = mx + log(z);
        double* mr = m + (int64_t)r * d;
        for (int i = 0; i < d; ++i) mr[i] = 0.0;
        for (int64_t t = t0; t < t1; ++t) {
            const double w = exp(a[t - t0] - l);
            const double* k = K + t * d;
            for (int i = 0; i < d; ++i) mr[i] += w * k[i];
        }
        double qm = 0.0;
        for (int i = 0; i < d; ++i) qm += q[i] * mr[i];
        lse[r] = l;
        b[r] = l - s * qm;
    }
}

/*
 * Summaries of the listed nodes of one KV head.  Node i covers tokens
 * [i*span, (i+1)*span) ([fluxbbs]/[wqu]: contiguous chunks, compressed level by level;
 * a level-l node covers span = C^l tokens).
 * K: [*][d] rows of one head; qref: [R][d]; outputs m [n][R][d], lse [n][R], b [n][R].
 */
void zo_summaries(const double* K, int d, const double* qref, int R, int64_t span,
                  const int64_t* nodes, int64_t n_nodes, double* m, double* lse, double* b)
{
#pragma omp parallel
    {
        double* a = (double*)malloc(sizeof(double) * (size_t)span);
#pragma omp for schedule(dynamic, 1)
        for (int64_t k = 0; k < n_nodes; ++k) {
            const int64_t i = nodes[k];
            node_summary(K, i * span, (i + 1) * span, d, qref, R,
                         m + k * (int64_t)R * d, lse + k * R, b + k * R, a);
        }
        free(a);
    }
}

/*
 * Plane estimate of a node's log attention mass for query q: the maximum over the
 * R tangent planes, est = max_r [ s (q . m_r) + b_r ]
 * (fluxbbs.com, section 树形索引是怎么搭的, and wqu.guru, section Building the tree: the
 * estimate is the largest of the R planes).
 */
double zo_plane_estimate(const double* m, const double* b, int R, int d, const double* q)
{
    const double s = score_scale(d);
    double best = -INFINITY;
    for (int r = 0; r < R; ++r) {
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += q[i] * m[(int64_t)r * d + i];
        const double v = s * dot + b[r];
        if (v > best) best = v;
    }
    return best;
}

/* log-sum-exp of s q.k_t over tokens [t0, t1): the node's true log attention mass. */
double zo_true_log_mass(const double* K, int64_t t0, int64_t t1, int d, const double* q)
{
    const double s = score_scale(d);
    double mx = -INFINITY;
    for (int64_t t = t0; t < t1; ++t) {
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += q[i] * K[t * d + i];
        if (s * dot > mx) mx = s * dot;
    }
    double z = 0.0;
    for (int64_t t = t0; t < t1; ++t) {
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += q[i] * K[t * d + i];
        z += exp(s * dot - mx);
    }
    return mx + log(z);
}

typedef struct { double e; int64_t idx; int64_t pos; } cand_t;

/* (score descending, node index ascending) */
static int cand_cmp(const void* pa, const void* pb)
{
    const cand_t* x = (const cand_t*)pa;
    const cand_t* y = (const cand_t*)pb;
    if (x->e > y->e) return -1;
    if (x->e < y->e) return 1;
    return (x->idx < y->idx) ? -1 : (x->idx > y->idx ? 1 : 0);
}

/*
 * Top-p cut over n candidates (fluxbbs.com, section 树形索引是怎么搭的, and wqu.guru,
 * section How does top-p routing pick tokens?: the kept nodes are the fewest whose
 * estimated mass together reaches the fraction p).
 * P_i = exp(e_i - max e) / sum_j exp(e_j - max e) over the candidates; order by
 * (e desc, idx asc); k* = min{k >= 1 : sum_{t<k} P_(t) >= p}; p >= 1 keeps all.
 * keep[i] is set for kept candidates (positions as given).  Returns k*.
 * info (nullable) gets four margins of the decision, +inf where undefined:
 *   info[0] = cum_{k*} - p, info[1] = p - cum_{k*-1} (cum_0 = 0),
 *   info[2] = P_(k*-1) - P_(k*), info[3] = e_(k*-1) - e_(k*).
 */
int64_t zo_topp(const double* e, const int64_t* idx, int64_t n, double p, uint8_t* keep, double* info)
{
    if (info) info[0] = info[1] = info[2] = info[3] = INFINITY;
    for (int64_t i = 0; i < n; ++i) keep[i] = 0;
    if (n == 0) return 0;
    if (p >= 1.0) {
        for (int64_t i = 0; i < n; ++i) keep[i] = 1;
        return n;
    }
    cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)n);
    double mx = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        c[i].e = e[i]; c[i].idx = idx[i]; c[i].pos = i;
        if (e[i] > mx) mx = e[i];
    }
    qsort(c, (size_t)n, sizeof(cand_t), cand_cmp);
    double z = 0.0;
    for (int64_t i = 0; i < n; ++i) z += exp(c[i].e - mx);
    double cum = 0.0, prev = 0.0;
    int64_t kstar = n;
    for (int64_t k = 0; k < n; ++k) {
        prev = cum;
        cum += exp(c[k].e - mx) / z;
        if (cum >= p) { kstar = k + 1; break; }
    }
    for (int64_t k = 0; k < kstar; ++k) keep[c[k].pos] = 1;
    if (info) {
        info[0] = cum - p;
        info[1] = p - prev;
        if (kstar < n) {
            info[2] = exp(c[kstar - 1].e - mx) / z - exp(c[kstar].e - mx) / z;
            info[3] = c[kstar - 1].e - c[kstar].e;
        }
    }
    free(c);
    return kstar;
}

/*
 * Top-down routing of n_lanes (query, head) lanes through the tree of one sequence
 * (fluxbbs.com, section 树形索引是怎么搭的, and wqu.guru, section How does top-p routing
 * pick tokens?: routing starts at the top level, cuts each level at mass p and descends
 * only into the kept nodes' children, down to level 1).
 *
 * K: [Hkv][ld][d] keys (rows t < N used); qref: [Hkv][R][d]; q: [n_lanes][d];
 * lane_g[x]: KV head of lane x.  Level l (1..L) has n_l = N / C^l nodes; the frontier
 * of level L is all of them, the frontier of level l-1 is the children
 * {i*C + c : i kept at level l, 0 <= c < C}.
 * Outputs, with n1 = N / C and level index v = l - 1:
 *   kept[v][x][0..n_l)  1 = kept by the oracle's own cut of lane x's level-l frontier;
 *   info[v][x][4], kstar[v][x], nfront[v][x] (frontier size).
 * forced (nullable, same layout as kept): replay mode - the level-(l-1) frontier is built
 * from forced[v] instead of kept[v], so each level is judged on the frontier another
 * implementation actually used.
 * scores (nullable): [L][n_lanes][n1] plane estimates of every frontier node (others
 * untouched), so a caller can see how close two nodes at the cut were.
 * Node summaries are recomputed from the raw keys for every frontier node at every level.
 */
void zo_route(const double* K, int64_t ld, int64_t N, int Hkv, int d,
              const double* qref, int R, int C, int L,
              const double* q, const int32_t* lane_g, int n_lanes, double p,
              uint8_t* kept, const uint8_t* forced, double* info, int64_t* kstar, int64_t* nfront,
              double* scores)
{
    const int64_t n1 = N / C;
    const size_t lane_stride = (size_t)(n1 > 0 ? n1 : 1);
    memset(kept, 0, (size_t)L * n_lanes * lane_stride);
    for (int64_t i = 0; i < (int64_t)L * n_lanes * 4; ++i) info[i] = INFINITY;
    for (int64_t i = 0; i < (int64_t)L * n_lanes; ++i) { kstar[i] = 0; nfront[i] = 0; }
    if (n1 == 0) return;

    uint8_t* front = (uint8_t*)calloc((size_t)n_lanes * lane_stride, 1);
    double* e = (double*)malloc(sizeof(double) * (size_t)n_lanes * lane_stride);

    for (int l = L; l >= 1; --l) {
        int64_t span = 1;
        for (int i = 0; i < l; ++i) span *= C;
        const int64_t nl = N / span;
        const int v = l - 1;
        if (nl == 0) continue;
        /* frontier of this level */
        for (int x = 0; x < n_lanes; ++x) {
            uint8_t* fx = front + (size_t)x * lane_stride;
            if (l == L) {
                for (int64_t j = 0; j < nl; ++j) fx[j] = 1;
            } else {
                const uint8_t* src = (forced ? forced : kept) + ((size_t)(v + 1) * n_lanes + x) * lane_stride;
                for (int64_t j = 0; j < nl; ++j) fx[j] = src[j / C];
            }
        }
        /* scores of every (lane, frontier node); summaries by definition */
#pragma omp parallel
        {
            double* a = (double*)malloc(sizeof(double) * (size_t)span);
            double* m = (double*)malloc(sizeof(double) * (size_t)R * d);
            double* lse = (double*)malloc(sizeof(double) * (size_t)R);
            double* b = (double*)malloc(sizeof(double) * (size_t)R);
#pragma omp for schedule(dynamic, 4) collapse(2)
            for (int g = 0; g < Hkv; ++g) {
                for (int64_t j = 0; j < nl; ++j) {
                    int needed = 0;
                    for (int x = 0; x < n_lanes; ++x)
                        if (lane_g[x] == g && front[(size_t)x * lane_stride + j]) { needed = 1; break; }
                    if (!needed) continue;
                    const double* Kg = K + (int64_t)g * ld * d;
                    node_summary(Kg, j * span, (j + 1) * span, d, qref + (int64_t)g * R * d, R, m, lse, b, a);
                    for (int x = 0; x < n_lanes; ++x)
                        if (lane_g[x] == g && front[(size_t)x * lane_stride + j])
                            e[(size_t)x * lane_stride + j] = zo_plane_estimate(m, b, R, d, q + (int64_t)x * d);
                }
            }
            free(a); free(m); free(lse); free(b);
        }
        /* top-p cut per lane */
#pragma omp parallel for schedule(dynamic, 1)
        for (int x = 0; x < n_lanes; ++x) {
            const uint8_t* fx = front + (size_t)x * lane_stride;
            int64_t n = 0;
            for (int64_t j = 0; j < nl; ++j) n += fx[j];
            double* ec = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
            int64_t* ic = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
            uint8_t* kc = (uint8_t*)malloc((size_t)(n > 0 ? n : 1));
            int64_t k = 0;
            for (int64_t j = 0; j < nl; ++j)
                if (fx[j]) { ec[k] = e[(size_t)x * lane_stride + j]; ic[k] = j; ++k; }
            const size_t o = (size_t)v * n_lanes + x;
            kstar[o] = zo_topp(ec, ic, n, p, kc, info + o * 4);
            nfront[o] = n;
            if (scores)
                for (int64_t t = 0; t < n; ++t) scores[o * lane_stride + ic[t]] = ec[t];
            uint8_t* kx = kept + o * lane_stride;
            for (int64_t t = 0; t < n; ++t) if (kc[t]) kx[ic[t]] = 1;
            free(ec); free(ic); free(kc);
        }
    }
    free(front);
    free(e);
}

/*
 * Attended token set of one lane (fluxbbs.com, section 树形索引是怎么搭的: exact attention
 * runs only over the raw rows the routing kept; wqu.guru, section How does top-p routing
 * pick tokens?: token 0 is attended as a sink in every case):
 *   A = {0} U {jC .. jC+C-1 : j kept at level 1} U [T C^L, N),  T = N / C^L;
 * with T = 0 (no complete top node) A = [0, N).  kept1: [N / C].
 * Writes the sorted token list (capacity N) and returns |A|.
 */
int64_t zo_attended_set(const uint8_t* kept1, int64_t N, int C, int L, int64_t* tokens)
{
    int64_t top = 1;
    for (int i = 0; i < L; ++i) top *= C;
    const int64_t T = N / top;
    uint8_t* mark = (uint8_t*)calloc((size_t)(N > 0 ? N : 1), 1);
    if (T == 0) {
        for (int64_t t = 0; t < N; ++t) mark[t] = 1;
    } else {
        mark[0] = 1;
        const int64_t n1 = N / C;
        for (int64_t j = 0; j < n1; ++j)
            if (kept1[j])
                for (int64_t t = j * C; t < (j + 1) * C; ++t) mark[t] = 1;
        for (int64_t t = T * top; t < N; ++t) mark[t] = 1;
    }
    int64_t n = 0;
    for (int64_t t = 0; t < N; ++t) if (mark[t]) tokens[n++] = t;
    free(mark);
    return n;
}

/*
 * Exact softmax attention over a token set (fluxbbs.com, section 树形索引是怎么搭的;
 * wqu.guru, section What is Zyphra Hierarchical Attention (ZHA)?: the tree only chooses
 * the keys, the attention over them is ordinary softmax attention):
 *   o = sum_{t in A} exp(s q.k_t - M) v_t / sum_{t in A} exp(s q.k_t - M),  M = max.
 * K, V: [*][d] rows of one head.
 */
void zo_attend(const double* K, const double* V, int d, const double* q,
               const int64_t* tokens, int64_t n_tok, double* out)
{
    const double s = score_scale(d);
    double* a = (double*)malloc(sizeof(double) * (size_t)(n_tok > 0 ? n_tok : 1));
    double mx = -INFINITY;
    for (int64_t k = 0; k < n_tok; ++k) {
        const double* kt = K + tokens[k] * d;
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += q[i] * kt[i];
        a[k] = s * dot;
        if (a[k] > mx) mx = a[k];
    }
    double z = 0.0;
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    for (int64_t k = 0; k < n_tok; ++k) {
        const double w = exp(a[k] - mx);
        z += w;
        const double* vt = V + tokens[k] * d;
        for (int i = 0; i < d; ++i) out[i] += w * vt[i];
    }
    for (int i = 0; i < d; ++i) out[i] /= z;
    free(a);
}

/* zo_attend for many lanes; lane x reads head lane_g[x] of K, V ([Hkv][ld][d]) and the
 * token list tokens[offsets[x] .. offsets[x+1]).  out: [n_lanes][d]. */
void zo_attend_batch(const double* K, const double* V, int64_t ld, int d,
                     const double* q, const int32_t* lane_g, int n_lanes,
                     const int64_t* tokens, const int64_t* offsets, double* out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int x = 0; x < n_lanes; ++x) {
        const int64_t off = (int64_t)lane_g[x] * ld * d;
        zo_attend(K + off, V + off, d, q + (int64_t)x * d, tokens + offsets[x],
                  offsets[x + 1] - offsets[x], out + (int64_t)x * d);
    }
}
