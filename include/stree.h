/*
 * stree.h -- C ABI of libstree.so: the packed-tree selective-SSM scan on B200.
 *
 * The method ("STree: Speculative Tree Decoding for Hybrid State Space Models",
 * scime.ai summary, sections "Problem" and "Approach"): a speculative draft tree
 * is packed into one sequence with a tree mask; accumulating the diagonal log
 * state transitions along each node's ancestors (A_tree = L . log A) gives the
 * exact per-path SSM output of every node in one scan, and after acceptance the
 * state of the accepted path is rebuilt from the stored inputs ("activation
 * replay") instead of keeping per-node states.  The same replay-on-commit design
 * appears in "Bole" (abstract: reconstruct only the selected state) and "TreeWY"
 * (abstract: reconstruct only the accepted state on commit).
 *
 * Per sequence b, head h (group g = h / (H/G)) and node i with parent p(i):
 *     s_i = exp(dt_i A_h) s_p(i) + dt_i x_i (outer) B_i,   s_p(root) = h0[b,h]
 *     y_i = s_i C_i + D_h x_i
 * computed in packed form as
 *     L_i = A_h * sum_{j in anc(i)} dt_j                      (tree cumsum)
 *     y_i = exp(L_i) (h0 C_i) + sum_{j in anc(i)} exp(L_i - L_j) (C_i . B_j) dt_j x_j + D_h x_i
 * and the commit of an accepted root->leaf path as
 *     h_new = exp(L_leaf) h0 + sum_{j on path} exp(L_leaf - L_j) dt_j x_j (outer) B_j.
 * anc(i) is the ancestor-or-self set of i.  dt is taken as given (already passed
 * through softplus); there is no dt bias, gating or normalisation in this op.
 *
 * Layouts (contiguous, row-major, device memory unless stated):
 *   x     [batch, n_nodes, nheads, headdim]   dtype (fp32 or bf16)
 *   dt    [batch, n_nodes, nheads]            dtype
 *   A, D  [nheads]                            fp32
 *   B, C  [batch, n_nodes, ngroups, dstate]   dtype
 *   h0    [batch, nheads, headdim, dstate]    fp32 (the cached state)
 *   y     [batch, n_nodes, nheads, headdim]   dtype
 *   h_new [batch, nheads, headdim, dstate]    fp32
 *   parent [batch, n_nodes] int32: parent[b,0] = -1 and 0 <= parent[b,i] < i
 *          for i > 0 (the tree is packed in a topological order, root first).
 *   accepted_path [batch, maxlen] int32, path_len [batch] int32: path[b,0] = 0
 *          and parent[path[b,k]] = path[b,k-1]; entries past path_len ignored;
 *          path_len = 0 keeps the cached state (h_new = h0).
 *   anc   [batch, n_nodes, ceil(n_nodes/32)] uint32: bit j of word j/32 set iff
 *          j is i or an ancestor of i.  depth [batch, n_nodes] int32 (root 0).
 *
 * Supported shapes: 1 <= n_nodes <= 256, batch >= 0, headdim and dstate multiples
 * of 8 in [8, 256], nheads a multiple of ngroups.  Pointers to tensors must be
 * 16-byte aligned.  batch = 0 is a no-op that returns STREE_OK.
 *
 * Precision: all accumulation is fp32.  The CUDA-core kernels (STREE_KERNEL_SIMT
 * and STREE_KERNEL_SMALL, and every fp32 input) compute in fp32 throughout.  The
 * tensor-core kernel (bf16 inputs, dstate 128, n_nodes <= 128, headdim a multiple
 * of 32) rounds h0 to tf32 in the root term, the masked decay matrix (D_h on its
 * diagonal included) to bf16, and the commit coefficients dt-weighted x to tf32;
 * each rounding is below the bf16 rounding of y itself.
 *
 * Ownership and threading: the caller owns every tensor.  A context (stree_ctx)
 * owns the library's device workspace (tree masks, depths, per-sequence flags,
 * the error word, a C.B scratch for the tree term).  Workspace is allocated by
 * cudaMalloc the first time a call needs more than the context holds; later
 * calls with the same or smaller sizes never allocate, so warm a context up
 * before capturing its calls in a CUDA graph.  A context is not thread-safe;
 * use one per stream.  All calls are asynchronous on `stream` (a cudaStream_t;
 * NULL is the legacy default stream) except stree_sync_check and
 * stree_ctx_destroy.
 *
 * Errors: every call returns a status and never aborts.  Argument and shape
 * checks happen on the host before anything is launched.  Tree and path validity
 * are checked on the device: a bad sequence is skipped (its outputs are left
 * untouched) and the first such error is latched in the context's error word,
 * which stree_sync_check reads and clears.
 */
#ifndef STREE_H
#define STREE_H

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    STREE_OK = 0,
    STREE_ERR_INVALID_ARG = 1,  /* null pointer, negative size, aliasing not allowed */
    STREE_ERR_UNSUPPORTED = 2,  /* shape or dtype outside the supported set */
    STREE_ERR_BAD_TREE = 3,     /* device-detected: parent array is not a packed tree */
    STREE_ERR_BAD_PATH = 4,     /* device-detected: accepted path is not a root->node chain */
    STREE_ERR_MISALIGNED = 5,   /* a tensor pointer is not 16-byte aligned */
    STREE_ERR_CUDA = 6,         /* a CUDA runtime call failed (launch, allocation) */
    STREE_ERR_TIMEOUT = 7,      /* a bounded wait inside the tensor-core kernel gave up (about 1 s) */
    STREE_ERR_NO_TREE = 8       /* scan with parent = NULL before any tree was built, or
                                   commit before any scan, or a size mismatch with them */
} stree_status;

typedef enum { STREE_F32 = 0, STREE_BF16 = 1 } stree_dtype;

/* Which scan kernel a context uses (stree_ctx_set_kernel). */
typedef enum {
    STREE_KERNEL_AUTO = 0,      /* SMALL for up to 16384 state rows (batch x nheads x headdim)
                                   where supported, else TC where supported, else SIMT */
    STREE_KERNEL_SIMT = 1,      /* CUDA-core fp32 kernel, every supported shape */
    STREE_KERNEL_TC = 2,        /* tcgen05 kernel; STREE_ERR_UNSUPPORTED if the shape is not */
    STREE_KERNEL_SMALL = 3      /* small-batch CUDA-core kernel (dstate 128, headdim a multiple
                                   of 32, n_nodes <= 64, a scan with y); else STREE_ERR_UNSUPPORTED */
} stree_kernel;

typedef struct stree_ctx stree_ctx;

/* Create / destroy a context.  destroy synchronises the device and frees the
 * workspace; it accepts NULL. */
stree_status stree_ctx_create(stree_ctx **out);
stree_status stree_ctx_destroy(stree_ctx *ctx);

/* Select the scan kernel for later scan calls on this context (default AUTO). */
stree_status stree_ctx_set_kernel(stree_ctx *ctx, stree_kernel kernel);

/* Number of CUDA kernels this context has launched so far (host counter). */
stree_status stree_ctx_launch_count(stree_ctx *ctx, int64_t *count);

/* The kernel (SIMT, TC or SMALL) that ran the last scan call on this context;
 * STREE_KERNEL_AUTO before the first one. */
stree_status stree_ctx_last_kernel(stree_ctx *ctx, stree_kernel *kernel);

/* Limit, in nanoseconds of device time, of every bounded wait inside the
 * tensor-core kernel for later calls on this context (0, the default, means
 * about 1 s).  A wait that runs out latches STREE_ERR_TIMEOUT; the CTA then does
 * no further work, waits (bounded) for its own copies and MMAs in flight, frees
 * its tensor memory and exits, and the context stays usable. */
stree_status stree_ctx_set_wait_limit(stree_ctx *ctx, uint64_t ns);

/* Test hook of that failure path: with fault = 1, later tensor-core scans on this
 * context withhold one hand-off between two of the kernel's warp roles (the first
 * tile's coefficients, on which no copy or MMA depends), so that a bounded wait
 * runs out and the call reports STREE_ERR_TIMEOUT; 0 (the default) turns it off.
 * Nothing faults or hangs the GPU.  Other values: STREE_ERR_INVALID_ARG. */
stree_status stree_ctx_set_test_fault(stree_ctx *ctx, int fault);

/*
 * Tree builder ("tree mask" of the packed sequence, STree summary "Approach"):
 * validates parent[] and builds the ancestor-or-self bitmask and depth of every
 * node into the context.  anc_out / depth_out, when not NULL, receive copies
 * (device buffers of the layouts above).  An invalid tree latches
 * STREE_ERR_BAD_TREE and marks the sequence so that scans skip it.
 */
stree_status stree_build_tree(stree_ctx *ctx, const int32_t *parent, int n_nodes, int batch,
                              uint32_t *anc_out, int32_t *depth_out, void *stream);

/*
 * Packed tree scan: y for every node of every sequence and head.  When parent is
 * not NULL the tree is (re)built into the context by the same launch (with the
 * checks and error reporting of stree_build_tree); when it is NULL the context's
 * current tree is used and n_nodes / batch must match it.  The input pointers
 * are recorded for a later stree_commit (activation replay), so x, dt, A, B and
 * h0 must stay alive and unchanged until that commit.
 */
stree_status stree_tree_scan(stree_ctx *ctx, const void *x, const void *dt, const float *A,
                             const void *B, const void *C, const float *D, const float *h0,
                             const int32_t *parent, int n_nodes, int batch, int nheads,
                             int headdim, int dstate, int ngroups, stree_dtype dtype,
                             void *y, void *stream);

/*
 * Commit by activation replay (STree summary, "Approach"): h_new for the
 * accepted path of every sequence, from the inputs recorded by the last
 * stree_tree_scan on this context.  h_new may alias the recorded h0 (in-place
 * commit); no other aliasing is allowed.  An invalid path latches
 * STREE_ERR_BAD_PATH and leaves that sequence's h_new untouched.
 */
stree_status stree_commit(stree_ctx *ctx, const int32_t *accepted_path, const int32_t *path_len,
                          int maxlen, float *h_new, void *stream);

/*
 * Fused scan + commit: y and h_new in one pass that reads h0 once.  Arguments as
 * for stree_tree_scan followed by those of stree_commit.  h_new may alias h0.
 */
stree_status stree_tree_scan_commit(stree_ctx *ctx, const void *x, const void *dt, const float *A,
                                    const void *B, const void *C, const float *D, const float *h0,
                                    const int32_t *parent, int n_nodes, int batch, int nheads,
                                    int headdim, int dstate, int ngroups, stree_dtype dtype,
                                    const int32_t *accepted_path, const int32_t *path_len,
                                    int maxlen, void *y, float *h_new, void *stream);

/*
 * Fused scan + commit that allocates nothing (the paper has no counterpart:
 * this is a deployment convenience).  For callers that may not allocate device
 * memory where they run the scan -- a serving runtime that hands out all device
 * memory from its own pool, a process already at its memory cap, or a hot loop
 * where an allocator call would synchronise the device.  Arguments are those of
 * stree_tree_scan_commit without the context, plus err_out: a device int32[4]
 * that receives the error word of this call ({status, sequence, position,
 * detail}; cleared by the call), or NULL to discard device-detected errors.
 *
 * Scratch: the tree masks, depths and flags (and the CUDA-core kernel's C.B
 * pair scratch) live in one file-scope device array of 8 MiB that every GPU
 * loading the library keeps until the process exits.  With lazy module loading
 * (the CUDA default) the array is placed on a device when the library's code is
 * first loaded there, at the latest by the first call of this entry point on that
 * device: a caller that will later run at its memory cap should make one call (a
 * warm-up) before it reaches the cap, and before any stream capture, since that
 * first call also looks the array's device address up (cudaGetSymbolAddress).  A
 * call that finds a new CUDA context on the device (after cudaDeviceReset) looks
 * the address up again.  Sizes whose scratch does not fit return
 * STREE_ERR_UNSUPPORTED before anything is launched.  Every call on a device
 * shares the array, so calls that overlap on the GPU (other streams, other host
 * threads) race; serialise them.  The call never calls cudaMalloc or cudaFree.
 */
stree_status stree_tree_scan_commit_noalloc(const void *x, const void *dt, const float *A, const void *B,
                                            const void *C, const float *D, const float *h0, const int32_t *parent,
                                            int n_nodes, int batch, int nheads, int headdim, int dstate,
                                            int ngroups, stree_dtype dtype, const int32_t *accepted_path,
                                            const int32_t *path_len, int maxlen, void *y, float *h_new,
                                            int32_t *err_out, void *stream);

/*
 * Unrolled-tree baseline (STree summary, "Problem" and "Key results": the
 * alternative the packed tree is compared with).  Every given path -- normally
 * each root-to-leaf path of the draft tree -- is scanned as its own sequence with
 * the plain recurrence, s <- exp(dt_k A_h) s + dt_k x_k (outer) B_k and
 * y_k = s . C_k + D_h x_k from h0, and keeps its own final state.  Nodes shared by
 * several paths are recomputed once per path.  No context is used.
 *
 *   x, dt, A, B, C, D, h0: as for stree_tree_scan (n_nodes nodes per sequence)
 *   paths    [batch, n_paths, max_depth] int32 node ids, first node first
 *   path_len [batch, n_paths] int32, 0 <= len <= max_depth (entries past len ignored)
 *   y_paths  [batch, n_paths, max_depth, nheads, headdim] in x's dtype: y of the
 *            node at each position (positions >= len untouched)
 *   h_paths  [batch, n_paths, nheads, headdim, dstate] fp32: each path's final state
 *            (h0 itself for an empty path)
 *   err_out  device int32[4] error word of this call (cleared by the call), or NULL
 *
 * A path with a length out of range or a node id outside [0, n_nodes) latches
 * STREE_ERR_BAD_PATH and leaves that path's outputs untouched.  Shapes: headdim a
 * multiple of 8 and dstate a multiple of 16, both up to 256; n_nodes and
 * max_depth up to 256 (else STREE_ERR_UNSUPPORTED).  The caller owns every
 * buffer; the call allocates nothing and runs on `stream`.
 */
stree_status stree_unrolled_scan(const void *x, const void *dt, const float *A, const void *B, const void *C,
                                 const float *D, const float *h0, const int32_t *paths, const int32_t *path_len,
                                 int n_nodes, int batch, int n_paths, int max_depth, int nheads, int headdim,
                                 int dstate, int ngroups, stree_dtype dtype, void *y_paths, float *h_paths,
                                 int32_t *err_out, void *stream);

/*
 * Greedy (temperature 0) verification of the draft tree (STree summary, "Key
 * results" at temperature 0; "Builds on": SpecInfer, speculative sampling).  The
 * target's prediction after node i is pred[i] = argmax_v logits[i][v] (ties: the
 * smaller token id).  From the root, a child is accepted when its draft token
 * equals the prediction after its parent (equal sibling tokens: the smaller node
 * index), and the walk continues from it, for at most maxlen nodes.  The result
 * is exactly the accepted_path / path_len that stree_commit takes.
 *
 *   logits        [batch, n_nodes, vocab] fp32 or bf16 (logit_dtype), finite
 *   draft_tokens  [batch, n_nodes] int32: the token of each node (root's unused)
 *   parent        [batch, n_nodes] int32: the packed tree (as for the scan)
 *   pred_out      [batch, n_nodes] int32: receives pred
 *   accepted_path [batch, maxlen] int32: receives the root-first accepted nodes, -1 after
 *   path_len      [batch] int32: receives the number of accepted nodes (>= 1)
 *   bonus_token   [batch] int32: receives pred of the last accepted node
 *   err_out       device int32[4] error word of this call (cleared by the call), or NULL
 *
 * An invalid tree latches STREE_ERR_BAD_TREE for that sequence and gives it
 * path_len 0, bonus -1 and a path of -1.  n_nodes up to 256.  The caller owns every
 * buffer; the call allocates nothing and runs on `stream`.
 */
stree_status stree_accept_greedy(const void *logits, stree_dtype logit_dtype, int vocab,
                                 const int32_t *draft_tokens, const int32_t *parent, int n_nodes, int batch,
                                 int maxlen, int32_t *pred_out, int32_t *accepted_path, int32_t *path_len,
                                 int32_t *bonus_token, int32_t *err_out, void *stream);

/*
 * Stochastic verification of the draft tree by multi-step speculative sampling
 * (STree summary, "Builds on": SpecInfer and speculative sampling, the setting at
 * temperature > 0; TreeSpark summary, "Guaranteeing Lossless Decoding": residual
 * resampling).  At the current node u, with target distribution
 * p = softmax(target_logits[u] / temperature) and draft distribution
 * q = softmax(draft_logits[u] / temperature) (from which the tokens of u's
 * children were drawn), the children are tried in increasing node order: child c
 * with token t is accepted when u_accept[c] * q[t] < p[t], i.e. with probability
 * min(1, p[t] / q[t]), and the walk continues from c; after each rejection p
 * becomes max(p - q, 0) renormalised (unchanged when that is all zero).  When no
 * child is accepted, u is a leaf or the path holds maxlen nodes, the bonus token
 * is drawn from the current p by inverse CDF: the first token whose cumulative
 * probability exceeds u_bonus times the total (the last token if none does).
 *
 *   target_logits, draft_logits [batch, n_nodes, vocab] fp32 or bf16 (logit_dtype), finite
 *   draft_tokens  [batch, n_nodes] int32: the token of each node (root's unused), in [0, vocab)
 *   parent        [batch, n_nodes] int32: the packed tree (as for the scan)
 *   temperature   > 0
 *   u_accept      [batch, n_nodes] fp32 in [0, 1): the uniform of each node, used when it is tried
 *   u_bonus       [batch] fp32 in [0, 1): the uniform of the bonus draw
 *   accepted_path [batch, maxlen] int32: receives the root-first accepted nodes, -1 after
 *   path_len      [batch] int32: receives the number of accepted nodes (>= 1)
 *   bonus_token   [batch] int32: receives the bonus token
 *   err_out       device int32[4] error word of this call (cleared by the call), or NULL
 *
 * All arithmetic is fp32.  vocab up to 53248 (the current distribution is kept
 * on chip); n_nodes up to 256.  An invalid tree latches STREE_ERR_BAD_TREE and a
 * draft token outside [0, vocab) STREE_ERR_INVALID_ARG (position, token) for
 * that sequence, which gets path_len 0, bonus -1 and a path of -1.  The caller
 * owns every buffer; the call allocates nothing and runs on `stream`.
 */
stree_status stree_accept_sampling(const void *target_logits, const void *draft_logits, stree_dtype logit_dtype,
                                   int vocab, const int32_t *draft_tokens, const int32_t *parent, int n_nodes,
                                   int batch, float temperature, const float *u_accept, const float *u_bonus,
                                   int maxlen, int32_t *accepted_path, int32_t *path_len, int32_t *bonus_token,
                                   int32_t *err_out, void *stream);

/*
 * The gated delta rule (the linear-attention layers of hybrid models) over the
 * packed tree, with the commit of the accepted path ("TreeWY" abstract: every
 * draft node's output from one triangular solve and only the accepted state
 * rebuilt on commit; "Bole" abstract: the tree-structured closed form of the
 * linear-attention recurrence).  Per sequence and value head h (query/key head
 * g = h / (heads_v / heads_k)), node i with parent p(i), write strength beta and
 * erase strength a:
 *     S_i = alpha_i S_p(i) (I - a_i k_i k_i^T) + beta_i v_i k_i^T,  S_p(root) = S0[b,h]
 *     o_i = S_i q_i
 * With erase NULL, a = beta: the gated delta rule.  Given apart, the decoupled
 * erase and write of Gated DeltaNet-2 (related entry on the TreeWY page); all
 * zero, gated linear attention (S_i = alpha_i S_p(i) + beta_i v_i k_i^T).
 * Computed through the pseudo-values u (an ancestor-triangular solve) and
 * gamma_i = product of alpha over the root path of i:
 *     u_j   = beta_j v_j - a_j gamma_j S0 k_j - sum_{l strict ancestor of j} a_j (gamma_j/gamma_l) (k_j . k_l) u_l
 *     o_i   = gamma_i S0 q_i + sum_{j in anc(i)} (gamma_i/gamma_j) (q_i . k_j) u_j
 *     S_new = gamma_leaf S0 + sum_{j on path} (gamma_leaf/gamma_j) u_j k_j^T   (S0 for an empty path)
 *
 *   q, k   [batch, n_nodes, heads_k, dk]   dtype (fp32 or bf16)
 *   v, o   [batch, n_nodes, heads_v, dv]   dtype
 *   alpha, beta [batch, n_nodes, heads_v]  fp32 (gate in (0, 1] and write strength, after activation)
 *   erase       [batch, n_nodes, heads_v]  fp32 erase strength, or NULL (erase = beta)
 *   S0, S_new   [batch, heads_v, dv, dk]   fp32 (S_new may alias S0)
 *   parent [batch, n_nodes], accepted_path [batch, maxlen], path_len [batch] int32: as for the scan
 *   err_out device int32[4] error word of this call (cleared by the call), or NULL
 * accepted_path, path_len and S_new all NULL: no commit.
 *
 * Shapes: dk = 128, dv a multiple of 32 up to 256, n_nodes up to 64, heads_v a
 * multiple of heads_k (else STREE_ERR_UNSUPPORTED).  fp32 arithmetic; for bf16
 * inputs with dv = 128 the contractions run on the tensor cores, which round S0,
 * the pseudo-values and the pair weights to tf32 (fp32 accumulation).
 * An invalid tree latches STREE_ERR_BAD_TREE (that sequence's o and S_new are
 * untouched), an invalid path STREE_ERR_BAD_PATH (S_new untouched).  The caller
 * owns every buffer; the call allocates nothing and runs on `stream`.
 */
stree_status stree_gdn_tree_scan_commit(const void *q, const void *k, const void *v, const float *alpha,
                                        const float *beta, const float *erase, const float *S0,
                                        const int32_t *parent, int n_nodes,
                                        int batch, int heads_v, int heads_k, int dk, int dv, stree_dtype dtype,
                                        const int32_t *accepted_path, const int32_t *path_len, int maxlen, void *o,
                                        float *S_new, int32_t *err_out, void *stream);

/*
 * Tree-masked attention of the hybrid model's Transformer layers over the packed
 * tree (STree abstract: hybrid SSM and Transformer layers; STree summary,
 * "Approach": the packed tree sequence with a tree mask).  Node i, query head h
 * (key/value head g = h / (heads_q / heads_kv)) attends to the valid context and
 * to its own root path:
 *     o[b,i,h] = sum_j softmax_j(scale q[b,i,h] . k_j) v_j,
 *     j over k_ctx/v_ctx[b, 0 .. ctx_len[b]-1, g] and k_tree/v_tree[b, anc(i), g].
 *
 *   q, o          [batch, n_nodes, heads_q, 128]  bf16
 *   k_ctx, v_ctx  [batch, ctx_cap, heads_kv, 128] bf16 (the cache; positions past
 *                 ctx_len[b] are never used, whatever they hold)
 *   k_tree, v_tree [batch, n_nodes, heads_kv, 128] bf16 (the tree's own keys and values)
 *   ctx_len       [batch] int32, clamped to [0, ctx_cap]
 *   parent        [batch, n_nodes] int32: the packed tree (as for the scan)
 *   workspace     device scratch of at least stree_tree_attention_workspace_size()
 *                 bytes, 16-byte aligned, or NULL; owned by the caller, overwritten
 *   err_out       device int32[4] error word of this call (cleared by the call); required
 *
 * fp32 accumulation and softmax; P rounded to bf16 for the second product.
 * With few query tiles and a long context the key blocks are split over several
 * CTAs whose partial outputs go to the workspace and are merged by a second
 * launch on the same stream; with workspace NULL or too small the call runs one
 * CTA per query tile (same result up to rounding order, slower on long contexts).
 * Two calls that share a workspace must be ordered (same stream).
 * Shapes: head dim 128, n_nodes up to 128, heads_q / heads_kv dividing 128
 * (else STREE_ERR_UNSUPPORTED); scale > 0.  An invalid tree latches
 * STREE_ERR_BAD_TREE and leaves that sequence's o untouched.  The caller owns
 * every buffer; the call allocates nothing and runs on `stream`.
 */
stree_status stree_tree_attention(const void *q, const void *k_ctx, const void *v_ctx, const void *k_tree,
                                  const void *v_tree, const int32_t *ctx_len, const int32_t *parent, int n_nodes,
                                  int batch, int ctx_cap, int heads_q, int heads_kv, int head_dim, float scale,
                                  stree_dtype dtype, void *o, void *workspace, size_t workspace_bytes,
                                  int32_t *err_out, void *stream);

/*
 * Workspace bytes that stree_tree_attention wants for these shapes on the current
 * device (its split plan depends on the device's SM count); 0 when it does not
 * split.  Same shape rules as stree_tree_attention (STREE_ERR_UNSUPPORTED).
 */
stree_status stree_tree_attention_workspace_size(int n_nodes, int batch, int ctx_cap, int heads_q, int heads_kv,
                                                 int head_dim, size_t *bytes);

/*
 * Resolve accepted paths against the context's current tree: leaf_out[b] (device
 * int32 [batch]) receives the last node of a valid path, -1 for an empty path and
 * -2 for an invalid one (which also latches STREE_ERR_BAD_PATH).
 */
stree_status stree_resolve_path(stree_ctx *ctx, const int32_t *accepted_path, const int32_t *path_len,
                                int maxlen, int32_t *leaf_out, void *stream);

/*
 * Synchronise `stream`, read and clear the context's device error word.  Returns
 * the latched status (STREE_OK when none).  info, when not NULL, receives four
 * host int32: status, sequence index, node or path position, detail.
 */
stree_status stree_sync_check(stree_ctx *ctx, void *stream, int32_t *info);

/* Static text for a status code. */
const char *stree_status_string(stree_status status);

/* ABI version: major * 10000 + minor * 100 + patch. */
int stree_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STREE_H */
