/*
 * stree_oracle.c -- plain, slow, fp64 CPU oracle for the packed-tree SSM scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes is the plain definition the packed scan must reproduce:
 *
 *   "STree: Speculative Tree Decoding for Hybrid State Space Models"
 *   (scime.ai summary, section "Approach"): a packed token tree with a tree mask
 *   must give the exact per-path SSM outputs.  The per-path SSM is the diagonal
 *   (scalar decay per head) Mamba2 / SSD recurrence that the page lists under
 *   "Builds on" (Mamba2, Fused Selective Scan):
 *
 *       s_i = exp(dt_i * A_h) * s_parent(i) + dt_i * outer(x_i, B_i)      (P x N)
 *       y_i = s_i . C_i + D_h * x_i                                        (P)
 *
 *   with s_parent(root) = h0, the cached state.  "Exact per-path outputs" means
 *   node i's output is what an ordinary sequential scan over the root->i path
 *   produces, so the oracle literally walks that path, node by node.
 *
 *   Section "Approach", "activation replay for state backtracking": after
 *   acceptance the state of the accepted root->leaf path is rebuilt from the
 *   stored inputs.  The oracle replays the same recurrence along that path.
 *
 * Readings of points the pages leave open (the tree packing order, the path
 * format, the group mapping) are stated next to the code that takes them.
 *
 * Layouts (all contiguous, row-major, fp64 on this side):
 *   x [b,T,H,P]  dt [b,T,H]  A [H]  B,C [b,T,G,N]  D [H]  h0 [b,H,P,N]
 *   y [b,T,H,P]  h_new [b,H,P,N]  parent int32 [b,T]
 *   anc uint32 [b,T,W] with W = ceil(T/32)  depth int32 [b,T]
 *   path int32 [b,maxlen]  path_len int32 [b]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/*
 * A packed tree is valid when node 0 is its only root (parent -1) and every
 * other node's parent is an earlier node.  Reading: the tree is packed "into
 * one sequence" (STree summary, "Approach") in topological order, the root
 * first; any such order works, breadth-first is what the inputs use.
 */
static int tree_is_valid(const int32_t *par, int T)
{
    if (T <= 0) return 1;
    if (par[0] != -1) return 0;
    for (int i = 1; i < T; ++i)
        if (par[i] < 0 || par[i] >= i) return 0;
    return 1;
}

/* Root->node path of `node`, written root first into path[]; returns its length. */
static int root_path(const int32_t *par, int node, int32_t *path)
{
    int len = 0;
    for (int k = node; k != -1; k = par[k]) path[len++] = k;
    for (int a = 0, z = len - 1; a < z; ++a, --z) {
        int32_t t = path[a]; path[a] = path[z]; path[z] = t;
    }
    return len;
}

/*
 * Tree mask: anc[b,i] has bit j set iff j lies on the root->i path (i itself
 * included); depth[b,i] is the number of edges from the root.  ok[b] is 1 for a
 * valid tree, 0 otherwise (then that sequence's anc/depth are left zero).
 * Returns the number of invalid sequences.
 */
int oracle_build_tree(const int32_t *parent, int T, int batch,
                      uint32_t *anc, int32_t *depth, int32_t *ok)
{
    int W = (T + 31) / 32, bad = 0;
    int32_t *path = (int32_t *)malloc(sizeof(int32_t) * (T > 0 ? T : 1));
    for (int b = 0; b < batch; ++b) {
        const int32_t *par = parent + (size_t)b * T;
        memset(anc + (size_t)b * T * W, 0, sizeof(uint32_t) * (size_t)T * W);
        memset(depth + (size_t)b * T, 0, sizeof(int32_t) * (size_t)T);
        ok[b] = tree_is_valid(par, T);
        if (!ok[b]) { ++bad; continue; }
        for (int i = 0; i < T; ++i) {
            int len = root_path(par, i, path);
            for (int k = 0; k < len; ++k)
                anc[((size_t)b * T + i) * W + path[k] / 32] |= 1u << (path[k] % 32);
            depth[(size_t)b * T + i] = len - 1;
        }
    }
    free(path);
    return bad;
}

/* s <- exp(dt*A) * s + dt * outer(x, B): one step of the recurrence (P x N). */
static void recur_step(double *s, int P, int N, double dt, double A,
                       const double *x, const double *B)
{
    double decay = exp(dt * A);
    for (int p = 0; p < P; ++p)
        for (int n = 0; n < N; ++n)
            s[(size_t)p * N + n] = decay * s[(size_t)p * N + n] + dt * x[p] * B[n];
}

/*
 * y for every node of every (sequence, head): walk the node's root path from h0.
 * The head -> group map is Mamba2's: g(h) = h / (H/G) (reading: the pages do not
 * say; H must be a multiple of G).  Returns the number of invalid trees; their
 * outputs are left untouched.
 */
int oracle_tree_scan(const double *x, const double *dt, const double *A,
                     const double *Bm, const double *Cm, const double *D,
                     const double *h0, const int32_t *parent,
                     int T, int batch, int H, int P, int N, int G,
                     double *y, int nthreads)
{
    int bad = 0;
    for (int b = 0; b < batch; ++b) bad += !tree_is_valid(parent + (size_t)b * T, T);
    if (nthreads < 1) nthreads = 1;
    int hpg = H / G;

#pragma omp parallel for collapse(2) schedule(dynamic) num_threads(nthreads)
    for (int b = 0; b < batch; ++b) {
        for (int h = 0; h < H; ++h) {
            const int32_t *par = parent + (size_t)b * T;
            if (!tree_is_valid(par, T)) continue;
            int g = h / hpg;
            double *s = (double *)malloc(sizeof(double) * (size_t)P * N);
            int32_t *path = (int32_t *)malloc(sizeof(int32_t) * (size_t)T);
            for (int i = 0; i < T; ++i) {
                memcpy(s, h0 + ((size_t)b * H + h) * P * N, sizeof(double) * (size_t)P * N);
                int len = root_path(par, i, path);
                for (int k = 0; k < len; ++k) {
                    int j = path[k];
                    recur_step(s, P, N, dt[((size_t)b * T + j) * H + h], A[h],
                               x + (((size_t)b * T + j) * H + h) * P,
                               Bm + (((size_t)b * T + j) * G + g) * N);
                }
                const double *Ci = Cm + (((size_t)b * T + i) * G + g) * N;
                const double *xi = x + (((size_t)b * T + i) * H + h) * P;
                double *yi = y + (((size_t)b * T + i) * H + h) * P;
                for (int p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) acc += s[(size_t)p * N + n] * Ci[n];
                    yi[p] = acc + D[h] * xi[p];
                }
            }
            free(path);
            free(s);
        }
    }
    return bad;
}

/*
 * Accepted path: reading -- a root-prefixed chain of node indices, path[0] = 0
 * and parent[path[k]] = path[k-1], of length 0..min(maxlen, T); length 0 keeps
 * the cached state (h_new = h0).  Returns 1 when valid.
 */
static int path_is_valid(const int32_t *par, int T, const int32_t *path, int len, int maxlen)
{
    if (len < 0 || len > maxlen || len > T) return 0;
    if (len == 0) return 1;
    if (path[0] != 0) return 0;
    for (int k = 1; k < len; ++k) {
        int j = path[k];
        if (j < 0 || j >= T || par[j] != path[k - 1]) return 0;
    }
    return 1;
}

/*
 * Activation replay: h_new[b,h] = state after running the recurrence from h0
 * over the accepted path's nodes, in path order.  ok[b] = 1 when the tree and
 * the path are valid (else h_new[b] is left untouched).  leaf[b] is the last
 * path node (-1 for an empty path).  Returns the number of rejected sequences.
 */
int oracle_commit(const double *x, const double *dt, const double *A,
                  const double *Bm, const double *h0, const int32_t *parent,
                  const int32_t *path, const int32_t *path_len, int maxlen,
                  int T, int batch, int H, int P, int N, int G,
                  double *h_new, int32_t *ok, int32_t *leaf, int nthreads)
{
    int bad = 0;
    for (int b = 0; b < batch; ++b) {
        const int32_t *par = parent + (size_t)b * T;
        ok[b] = tree_is_valid(par, T) &&
                path_is_valid(par, T, path + (size_t)b * maxlen, path_len[b], maxlen);
        leaf[b] = (ok[b] && path_len[b] > 0) ? path[(size_t)b * maxlen + path_len[b] - 1] : -1;
        bad += !ok[b];
    }
    if (nthreads < 1) nthreads = 1;
    int hpg = H / G;

#pragma omp parallel for collapse(2) schedule(dynamic) num_threads(nthreads)
    for (int b = 0; b < batch; ++b) {
        for (int h = 0; h < H; ++h) {
            if (!ok[b]) continue;
            int g = h / hpg;
            double *s = h_new + ((size_t)b * H + h) * P * N;
            memmove(s, h0 + ((size_t)b * H + h) * P * N, sizeof(double) * (size_t)P * N);
            for (int k = 0; k < path_len[b]; ++k) {
                int j = path[(size_t)b * maxlen + k];
                recur_step(s, P, N, dt[((size_t)b * T + j) * H + h], A[h],
                           x + (((size_t)b * T + j) * H + h) * P,
                           Bm + (((size_t)b * T + j) * G + g) * N);
            }
        }
    }
    return bad;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
