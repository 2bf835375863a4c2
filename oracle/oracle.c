/*
 * oracle.c -- TEST INFRASTRUCTURE ONLY (never part of the product path).
 *
 * A plain, slow, single-threaded CPU restatement in fp64 of what the target model's verify
 * step computes in tree speculative decoding.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg load it.  It shares no code, header, table or helper with
 * the CUDA library, and it reads inputs as the exact stored values (fp32, or bf16 bits
 * widened to fp64 here).  Every routine follows a definition stated on the source pages:
 *
 *   [EP]  "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
 *         technical summary, section 2 (methodology): branchable KV cache with commit by
 *         length or by path index; shifted indexing with a dummy row 0 for the root;
 *         ancestor index tables; range / acyclicity / depth invariants; the 4D tree mask
 *         that lets a token see only its ancestors on its own branch.
 *   [SO]  "Acelerando Sonar a traves de la especulacion" (Perplexity), sections
 *         "Decodificacion especulativa" (longest accepted prefix plus one free target token:
 *         n drafts give up to n+1 tokens), "Objetivo-Borrador" (acceptance compares the full
 *         draft and target distributions; the target's logits after the accepted run are
 *         sampled for one more token) and "EAGLE" (tree verify needs a custom mask).
 *         Its reference list cites Leviathan et al., "Fast Inference from Transformers via
 *         Speculative Decoding", whose min(1, p/q) test and max(p - q, 0) residual are used.
 *   [SSD] "Speculative Speculative Decoding", technical summary, section 2: the speculation
 *         cache keyed by the verify outcome (bonus token), hit or miss.
 *
 * Readings where the pages are silent are listed beside each routine.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Oracle-local result codes (tests map them to the library's codes by name). */
enum { ORC_OK = 0, ORC_BAD_PARENT = 1, ORC_TOO_DEEP = 2, ORC_EXTRA_ROOT = 3, ORC_BAD_ARG = 4 };

/* dt: 0 = fp32 storage, 1 = bf16 bits. */
static double widen(const void *base, int dt, long idx)
{
    if (dt == 0)
        return (double)((const float *)base)[idx];
    uint32_t u = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------------------
 * Tree structure [EP, sec. 2, "accelerator-safe tree tensor semantics"].
 *
 * parent[i] is node i's parent (topological order, -1 for a root).  Checks, node by node in
 * index order, reporting the first offending node:
 *   range / acyclicity: -1 <= parent[i] < i (parent < i makes every walk end at a root);
 *   roots: exactly one root unless `forest` (node 0 is always a root once range holds);
 *   depth: depth(i) = depth(parent) + 1 <= Dmax, root depth 0.
 * Outputs (slot s = i + 1; slot 0 is the dummy row that replaces the -1 placeholder):
 *   parent_s[N+1]: parent_s[0] = 0, parent_s[i+1] = parent[i] + 1;
 *   depth_s[N+1]:  depth_s[0] = 0, depth_s[i+1] = depth(i);
 *   M[N*N]:        explicit ancestor matrix, M[i][j] = 1 iff j lies on the root->i path
 *                  (i included), built by walking parent[] upward;
 *   anc[(N+1)*(Dmax+1)]: ancestor table, row s lists the slots of the root->node path
 *                  indexed by depth (anc[s][k] = slot of the depth-k ancestor, the node itself
 *                  at k = depth), 0 beyond; derived from M, not from a second walk.
 * ------------------------------------------------------------------------------------ */
int orc_tree_structure(const int32_t *parent, int N, int Dmax, int forest, int32_t *parent_s,
                       int32_t *depth_s, int32_t *anc, uint8_t *M, int32_t *bad_node)
{
    *bad_node = 0;
    if (N < 0 || Dmax < 0)
        return ORC_BAD_ARG;
    int32_t *depth = (int32_t *)calloc((size_t)(N > 0 ? N : 1), sizeof(int32_t));
    int roots = 0, code = ORC_OK;
    for (int i = 0; i < N && code == ORC_OK; ++i) {
        int p = parent[i];
        if (p < -1 || p >= i) {
            code = ORC_BAD_PARENT;
        } else if (p == -1) {
            roots += 1;
            depth[i] = 0;
            if (!forest && roots > 1)
                code = ORC_EXTRA_ROOT;
        } else {
            depth[i] = depth[p] + 1;
            if (depth[i] > Dmax)
                code = ORC_TOO_DEEP;
        }
        if (code != ORC_OK)
            *bad_node = i;
    }
    if (code != ORC_OK) {
        free(depth);
        return code;
    }
    memset(M, 0, (size_t)N * (size_t)N);
    for (int i = 0; i < N; ++i)
        for (int j = i; j >= 0; j = parent[j])
            M[(size_t)i * N + j] = 1;
    parent_s[0] = 0;
    depth_s[0] = 0;
    for (int i = 0; i < N; ++i) {
        parent_s[i + 1] = parent[i] + 1;
        depth_s[i + 1] = depth[i];
    }
    memset(anc, 0, sizeof(int32_t) * (size_t)(N + 1) * (size_t)(Dmax + 1));
    for (int i = 0; i < N; ++i)
        for (int j = 0; j < N; ++j)
            if (M[(size_t)i * N + j])
                anc[(size_t)(i + 1) * (Dmax + 1) + depth[j]] = j + 1;
    free(depth);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------
 * One attention output row [EP, sec. 2, "fused tree-mask teacher execution"; SO, "EAGLE"].
 *
 * o = softmax(scale * q . K^T) V over the key list: every committed prefix row 0..L-1
 * (unmasked) followed by each tree node j with mask[j] = 1 (the row of the explicit ancestor
 * matrix for this query's node).  Plain two-pass softmax in fp64: scores, maximum,
 * exponentials, sum, weighted sum of V.  Prefix row k sits at Kp + k*ldp elements, tree row j
 * at Kt + j*ldt (same for V).  lse = m + log(sum) in natural-log units of the scaled scores.
 * ------------------------------------------------------------------------------------ */
void orc_attn_row(const void *q, int dt, const void *Kp, const void *Vp, int L, long ldp,
                  const void *Kt, const void *Vt, long ldt, const uint8_t *mask, int N, int d,
                  double scale, double *out, double *lse)
{
    int nk = L;
    for (int j = 0; j < N; ++j)
        nk += mask[j] ? 1 : 0;
    for (int c = 0; c < d; ++c)
        out[c] = 0.0;
    if (nk == 0) {
        *lse = -INFINITY;
        return;
    }
    double *qv = (double *)malloc(sizeof(double) * (size_t)d);
    double *s = (double *)malloc(sizeof(double) * (size_t)nk);
    for (int c = 0; c < d; ++c)
        qv[c] = widen(q, dt, c);
    /* pass 1: scores */
    int n = 0;
    for (int k = 0; k < L; ++k, ++n) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
            acc += qv[c] * widen(Kp, dt, (long)k * ldp + c);
        s[n] = scale * acc;
    }
    for (int j = 0; j < N; ++j) {
        if (!mask[j])
            continue;
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
            acc += qv[c] * widen(Kt, dt, (long)j * ldt + c);
        s[n++] = scale * acc;
    }
    double m = s[0];
    for (int t = 1; t < nk; ++t)
        if (s[t] > m)
            m = s[t];
    double z = 0.0;
    for (int t = 0; t < nk; ++t) {
        s[t] = exp(s[t] - m);
        z += s[t];
    }
    /* pass 2: weighted sum of values */
    n = 0;
    for (int k = 0; k < L; ++k, ++n)
        for (int c = 0; c < d; ++c)
            out[c] += s[n] * widen(Vp, dt, (long)k * ldp + c);
    for (int j = 0; j < N; ++j) {
        if (!mask[j])
            continue;
        for (int c = 0; c < d; ++c)
            out[c] += s[n] * widen(Vt, dt, (long)j * ldt + c);
        ++n;
    }
    for (int c = 0; c < d; ++c)
        out[c] /= z;
    *lse = m + log(z);
    free(s);
    free(qv);
}

/* Argmax of one logits row by a sequential scan keeping the first maximum.  NaN counts as
 * -inf (never chosen); a row with no value above -inf gives 0. */
long orc_argmax_row(const void *row, int dt, long V)
{
    double best = -INFINITY;
    long arg = 0;
    for (long v = 0; v < V; ++v) {
        double x = widen(row, dt, v);
        if (isnan(x))
            x = -INFINITY;
        if (x > best) {
            best = x;
            arg = v;
        }
    }
    return arg;
}

/* ------------------------------------------------------------------------------------
 * Greedy tree acceptance [SO, "Decodificacion especulativa" and "EAGLE"; SSD, sec. 2].
 *
 * t*(i) = argmax of node i's target logits row (the target's own next token after i).
 * A root is accepted unconditionally when root_key is NULL; otherwise only the lowest-index
 * root whose token equals *root_key is accepted (the speculation-cache hit) and no root is
 * accepted when none matches (a miss).  A non-root i is accepted iff its parent p is accepted
 * and tokens[i] == t*(p): the accepted nodes are exactly the nodes whose whole root->node
 * path reproduces greedy target decoding.  a* = the accepted node of greatest depth (ties:
 * lowest index).  Outputs: accept_len = depth(a*) (drafted tokens accepted beyond the root);
 * path[0..A] = slots (node + 1) of the root->a* path, 0 beyond; out_tok[0..A-1] = tokens of
 * path nodes 1..A, out_tok[A] = t*(a*) (the free target token), -1 beyond.  A miss gives
 * accept_len = -1, path all 0, out_tok all -1.  N == 0 is treated like a miss.
 * Returns the tree-structure code (the inputs are validated the same way first).
 * ------------------------------------------------------------------------------------ */
int orc_accept_greedy(const void *logits, int dt, long V, const int32_t *tokens,
                      const int32_t *parent, int N, int Dmax, int forest, const int32_t *root_key,
                      int32_t *accept_len, int32_t *path, int32_t *out_tok)
{
    for (int k = 0; k <= Dmax; ++k) {
        path[k] = 0;
        out_tok[k] = -1;
    }
    *accept_len = -1;
    if (N == 0)
        return ORC_OK;
    int32_t *ps = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N + 1));
    int32_t *ds = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N + 1));
    int32_t *anc = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N + 1) * (size_t)(Dmax + 1));
    uint8_t *M = (uint8_t *)malloc((size_t)N * (size_t)N);
    int32_t bad = 0;
    int code = orc_tree_structure(parent, N, Dmax, forest, ps, ds, anc, M, &bad);
    if (code != ORC_OK) {
        free(ps), free(ds), free(anc), free(M);
        return code;
    }
    long *tstar = (long *)malloc(sizeof(long) * (size_t)N);
    uint8_t *acc = (uint8_t *)calloc((size_t)N, 1);
    for (int i = 0; i < N; ++i)
        tstar[i] = orc_argmax_row((const char *)logits + (size_t)i * (size_t)V * (dt ? 2 : 4), dt, V);
    int hit = -1;
    if (root_key)
        for (int i = 0; i < N && hit < 0; ++i)
            if (parent[i] == -1 && tokens[i] == *root_key)
                hit = i;
    for (int i = 0; i < N; ++i) {   /* topological: parents come first */
        int p = parent[i];
        if (p < 0)
            acc[i] = root_key ? (uint8_t)(i == hit) : 1;
        else
            acc[i] = (uint8_t)(acc[p] && (long)tokens[i] == tstar[p]);
    }
    int best = -1;
    for (int i = 0; i < N; ++i)
        if (acc[i] && (best < 0 || ds[i + 1] > ds[best + 1]))
            best = i;
    if (best >= 0) {
        int A = ds[best + 1];
        *accept_len = A;
        int k = A;
        for (int j = best; j >= 0; j = parent[j])
            path[k--] = j + 1;
        for (k = 0; k < A; ++k)
            out_tok[k] = tokens[path[k + 1] - 1];
        out_tok[A] = (int32_t)tstar[best];
    }
    free(tstar), free(acc), free(ps), free(ds), free(anc), free(M);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------
 * Chain rejection sampling [SO, "Objetivo-Borrador"; the Leviathan et al. rule it cites].
 *
 * zp: K+1 target rows (row k = target logits after the k-th chain node, the root first);
 * zq: K draft rows (row k = the draft distribution token x[k] was drawn from); u: K+1
 * uniforms in [0,1).  Temperature T > 0: p_k = softmax(zp[k]/T), q_k = softmax(zq[k]/T),
 * each as exp(z/T - max) normalised by its sum.  For k = 0..K-1 in order: accept x[k] iff
 * u[k] * q_k(x[k]) < p_k(x[k]) (probability min(1, p/q)); stop at the first rejection j.
 * After a rejection the last token is drawn from the residual r = max(p_j - q_j, 0) by
 * inverse CDF with u[K]: the smallest t with sum_{v<=t} r_v > u[K] * sum_v r_v (if the
 * residual sums to 0, p_j is used).  With all K accepted, the bonus token is drawn the same
 * way from p_K.  T == 0 is greedy: accept iff x[k] == argmax zp[k], last token = argmax zp[j].
 * Outputs: accept_len = number accepted, out_tok[0..A-1] = x, out_tok[A] = the drawn token,
 * -1 beyond.  margin[k] (k < decisions made) = |u q - p| / max(p, u q) of each test, and
 * margin[K] = distance of the inverse-CDF threshold to the nearest cumulative boundary of the
 * drawn token, relative to the total mass; unused entries = 1e300.  The margins say how far a
 * decision is from flipping under a different (e.g. fp32) rounding.
 * ------------------------------------------------------------------------------------ */
static void softmax_row(const void *z, int dt, long V, double T, double *p)
{
    double m = -INFINITY;
    for (long v = 0; v < V; ++v) {
        double x = widen(z, dt, v) / T;
        if (x > m)
            m = x;
    }
    double s = 0.0;
    for (long v = 0; v < V; ++v) {
        p[v] = exp(widen(z, dt, v) / T - m);
        s += p[v];
    }
    for (long v = 0; v < V; ++v)
        p[v] /= s;
}

static int32_t inverse_cdf(const double *r, long V, double u, double *margin)
{
    double R = 0.0;
    for (long v = 0; v < V; ++v)
        R += r[v];
    double thr = u * R, c = 0.0;
    long last_pos = 0;
    for (long v = 0; v < V; ++v) {
        if (r[v] > 0.0)
            last_pos = v;
        double prev = c;
        c += r[v];
        if (c > thr) {
            double a = thr - prev, b = c - thr;
            *margin = (a < b ? a : b) / R;
            return (int32_t)v;
        }
    }
    *margin = 0.0;   /* threshold at or past the rounded total: no safe decision */
    return (int32_t)last_pos;
}

int orc_chain_sample(const void *zp, const void *zq, int dt, long V, int K, const int32_t *x,
                     const float *u, double T, int32_t *accept_len, int32_t *out_tok,
                     double *margin)
{
    size_t rb = (size_t)V * (dt ? 2 : 4);
    for (int k = 0; k <= K; ++k) {
        out_tok[k] = -1;
        margin[k] = 1e300;
    }
    if (T == 0.0) {
        int j = K;
        for (int k = 0; k < K; ++k)
            if ((long)x[k] != orc_argmax_row((const char *)zp + k * rb, dt, V)) {
                j = k;
                break;
            }
        *accept_len = j;
        for (int k = 0; k < j; ++k)
            out_tok[k] = x[k];
        out_tok[j] = (int32_t)orc_argmax_row((const char *)zp + j * rb, dt, V);
        return ORC_OK;
    }
    double *p = (double *)malloc(sizeof(double) * (size_t)V);
    double *q = (double *)malloc(sizeof(double) * (size_t)V);
    int j = K;
    for (int k = 0; k < K; ++k) {
        softmax_row((const char *)zp + k * rb, dt, V, T, p);
        softmax_row((const char *)zq + k * rb, dt, V, T, q);
        double px = p[x[k]], uq = (double)u[k] * q[x[k]];
        double den = px > uq ? px : uq;
        margin[k] = den > 0.0 ? fabs(uq - px) / den : 0.0;
        if (!(uq < px)) {
            j = k;
            break;
        }
    }
    *accept_len = j;
    for (int k = 0; k < j; ++k)
        out_tok[k] = x[k];
    if (j < K) {   /* p and q still hold row j */
        double R = 0.0;
        for (long v = 0; v < V; ++v) {
            double r = p[v] - q[v];
            q[v] = r > 0.0 ? r : 0.0;
            R += q[v];
        }
        out_tok[j] = inverse_cdf(R > 0.0 ? q : p, V, (double)u[K], &margin[K]);
    } else {
        softmax_row((const char *)zp + (size_t)K * rb, dt, V, T, p);
        out_tok[K] = inverse_cdf(p, V, (double)u[K], &margin[K]);
    }
    free(p);
    free(q);
    return ORC_OK;
}

/* Many independent chains in one call (used by the distribution tests). */
int orc_chain_sample_many(int trials, const void *zp, const void *zq, int dt, long V, int K,
                          const int32_t *x, const float *u, double T, int32_t *accept_len,
                          int32_t *out_tok, double *margin)
{
    size_t rb = (size_t)V * (dt ? 2 : 4);
    for (int t = 0; t < trials; ++t) {
        int c = orc_chain_sample((const char *)zp + (size_t)t * (K + 1) * rb,
                                 (const char *)zq + (size_t)t * K * rb, dt, V, K, x + (size_t)t * K,
                                 u + (size_t)t * (K + 1), T, accept_len + t,
                                 out_tok + (size_t)t * (K + 1), margin + (size_t)t * (K + 1));
        if (c != ORC_OK)
            return c;
    }
    return ORC_OK;
}
