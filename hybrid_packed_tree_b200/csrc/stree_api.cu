// stree_api.cu -- the C ABI of include/stree.h: argument checks, the context's
// workspace and the dispatch to the kernels.  No call here synchronises the
// device except stree_sync_check and stree_ctx_destroy.
#include <new>
#include <string.h>

#include "stree_internal.cuh"

using namespace stree;

struct stree_ctx {
    int device = -1;
    stree_kernel kernel = STREE_KERNEL_AUTO;
    // tree workspace
    uint32_t *anc = nullptr;
    int32_t *depth = nullptr, *ok = nullptr;
    size_t cap_anc = 0, cap_nodes = 0, cap_batch = 0;
    int tree_T = 0, tree_batch = -1;
    // C.B pair scratch
    float *cb = nullptr;
    size_t cap_cb = 0;
    // stand-alone commit workspace
    float *cw = nullptr;
    int32_t *ci = nullptr;
    size_t cap_cw = 0, cap_ci = 0;
    // error word {status, sequence, position, detail}
    int32_t *err = nullptr;
    // inputs recorded by the last scan, for stree_commit
    bool has_scan = false;
    ScanArgs last{};
    int64_t launches = 0;
    stree_kernel last_kernel = STREE_KERNEL_AUTO;   // the kernel of the last scan (AUTO: none yet)
    unsigned long long wait_ns = 0;                 // bounded-wait limit (0: the kernel's default)
    int fault = 0;                                  // failure-path test hook
};

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

stree_status cuda_status(cudaError_t e) { return e == cudaSuccess ? STREE_OK : STREE_ERR_CUDA; }

template <typename T>
stree_status ensure(T **buf, size_t *cap, size_t need)
{
    if (need <= *cap) return STREE_OK;
    if (*buf) cudaFree(*buf);
    *buf = nullptr;
    *cap = 0;
    if (cudaMalloc(reinterpret_cast<void **>(buf), need * sizeof(T)) != cudaSuccess) {
        *buf = nullptr;
        return STREE_ERR_CUDA;
    }
    *cap = need;
    return STREE_OK;
}

TreeView tree_view(const stree_ctx *c)
{
    TreeView tv;
    tv.anc = c->anc;
    tv.depth = c->depth;
    tv.ok = c->ok;
    tv.T = c->tree_T;
    tv.W = (c->tree_T + 31) / 32;
    tv.batch = c->tree_batch;
    return tv;
}

// Sizes the context's tree workspace for (T, batch) and records them; nothing is
// launched (the scan kernels or the tree builder fill it).
stree_status ensure_tree(stree_ctx *c, const int32_t *parent, int T, int batch)
{
    if (T < 1 || T > kMaxNodes || batch < 0) return STREE_ERR_UNSUPPORTED;
    if (!parent && batch > 0) return STREE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(parent) & 3u) != 0) return STREE_ERR_MISALIGNED;
    size_t W = (T + 31) / 32;
    size_t nb = batch > 0 ? (size_t)batch : 1;
    stree_status st;
    if ((st = ensure(&c->anc, &c->cap_anc, nb * T * W)) != STREE_OK) return st;
    if ((st = ensure(&c->depth, &c->cap_nodes, nb * T)) != STREE_OK) return st;
    if ((st = ensure(&c->ok, &c->cap_batch, nb)) != STREE_OK) return st;
    c->tree_T = T;
    c->tree_batch = batch;
    return STREE_OK;
}

stree_status build_into_ctx(stree_ctx *c, const int32_t *parent, int T, int batch, cudaStream_t s)
{
    stree_status st = ensure_tree(c, parent, T, batch);
    if (st != STREE_OK) return st;
    if (batch > 0) ++c->launches;
    return cuda_status(launch_build_tree(parent, T, batch, c->anc, c->depth, c->ok, c->err, s));
}

stree_status check_scan_args(const ScanArgs &a)
{
    if (a.batch < 0 || a.T < 1 || a.H < 1 || a.G < 1 || a.P < 1 || a.N < 1) return STREE_ERR_UNSUPPORTED;
    if (a.batch == 0) return STREE_OK;             // no-op: empty tensors may have NULL data
    if (!a.x || !a.dt || !a.A || !a.B || !a.C || !a.D || !a.h0 || !a.y) return STREE_ERR_INVALID_ARG;
    if (a.T > kMaxNodes || a.P > kMaxDim || a.N > kMaxDim) return STREE_ERR_UNSUPPORTED;
    if (a.P % 8 != 0 || a.N % 8 != 0 || a.H % a.G != 0) return STREE_ERR_UNSUPPORTED;
    if (a.H > 65535) return STREE_ERR_UNSUPPORTED;
    if (a.dtype != STREE_F32 && a.dtype != STREE_BF16) return STREE_ERR_UNSUPPORTED;
    const void *ptrs[] = {a.x, a.dt, a.A, a.B, a.C, a.D, a.h0, a.y};
    for (const void *p : ptrs)
        if (!aligned16(p)) return STREE_ERR_MISALIGNED;
    return STREE_OK;
}

stree_status check_commit_args(const int32_t *path, const int32_t *path_len, int maxlen, const float *h_new,
                               int batch)
{
    if (batch == 0) return maxlen >= 0 ? STREE_OK : STREE_ERR_INVALID_ARG;
    if (!path || !path_len || !h_new) return STREE_ERR_INVALID_ARG;
    if (maxlen < 1) return STREE_ERR_INVALID_ARG;
    if (!aligned16(h_new)) return STREE_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(path) & 3u) || (reinterpret_cast<uintptr_t>(path_len) & 3u))
        return STREE_ERR_MISALIGNED;
    return STREE_OK;
}

// Runs the scan (and the fused commit when a.path is set).  With a.parent set the
// tree is rebuilt into the context by the launch; otherwise the context's tree is used.
stree_status run_scan(stree_ctx *c, ScanArgs &a, cudaStream_t s)
{
    if (c->tree_batch != a.batch || c->tree_T != a.T) return STREE_ERR_NO_TREE;
    a.tree = tree_view(c);
    a.err = c->err;
    a.wait_ns = c->wait_ns;
    a.fault = c->fault;
    if (a.parent) {
        a.tree_anc = c->anc;
        a.tree_depth = c->depth;
        a.tree_ok = c->ok;
    }
    if (a.batch == 0) return STREE_OK;
    ScanPath path;
    if (!select_path(c->kernel, a, &path)) return STREE_ERR_UNSUPPORTED;
    c->last_kernel = path == ScanPath::Small ? STREE_KERNEL_SMALL
                     : path == ScanPath::Tc  ? STREE_KERNEL_TC
                                             : STREE_KERNEL_SIMT;
    if (path == ScanPath::Simt) {
        stree_status st = ensure(&c->cb, &c->cap_cb, (size_t)a.batch * a.G * a.T * a.T);
        if (st != STREE_OK) return st;
        a.cb = c->cb;
    } else if (path == ScanPath::Tc) {
        const size_t nf = tc_pair_scratch_floats(a);
        if (nf) {
            stree_status st = ensure(&c->cb, &c->cap_cb, nf);
            if (st != STREE_OK) return st;
            a.pair_scratch = c->cb;
        }
    }
    return cuda_status(launch_scan(path, a, s, &c->launches));
}

ScanArgs make_args(const void *x, const void *dt, const float *A, const void *B, const void *C,
                   const float *D, const float *h0, int T, int batch, int H, int P, int N, int G,
                   stree_dtype dtype, void *y)
{
    ScanArgs a{};
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D; a.h0 = h0;
    a.T = T; a.batch = batch; a.H = H; a.P = P; a.N = N; a.G = G;
    a.dtype = dtype;
    a.y = y;
    return a;
}

}  // namespace

namespace stree {

// Batches up to this many state rows (batch x nheads x headdim) take the
// small-batch kernel when both it and the tensor-core kernel support the shape:
// below it a launch is bound by latency, which the small kernel's short chain
// serves better than the tensor-core pipeline.
constexpr long long kSmallRows = 16384;

bool select_path(stree_kernel sel, const ScanArgs &a, ScanPath *out)
{
    switch (sel) {
    case STREE_KERNEL_SIMT:
        *out = ScanPath::Simt;
        return true;
    case STREE_KERNEL_TC:
        if (!tc_supported(a)) return false;
        *out = ScanPath::Tc;
        return true;
    case STREE_KERNEL_SMALL:
        if (!small_supported(a)) return false;
        *out = ScanPath::Small;
        return true;
    case STREE_KERNEL_AUTO: {
        const bool small = small_supported(a), tc = tc_supported(a);
        const long long rows = (long long)a.batch * a.H * a.P;
        if (small && (!tc || rows <= kSmallRows)) *out = ScanPath::Small;
        else if (tc) *out = ScanPath::Tc;
        else *out = ScanPath::Simt;
        return true;
    }
    }
    return false;
}

cudaError_t launch_scan(ScanPath path, const ScanArgs &a, cudaStream_t s, int64_t *launches)
{
    if (a.batch == 0) return cudaSuccess;
    cudaError_t e;
    switch (path) {
    case ScanPath::Small:
        ++*launches;
        return launch_scan_small(a, s);
    case ScanPath::Tc:
        ++*launches;
        return launch_scan_tc(a, s);
    case ScanPath::Simt:
        if (a.parent) {
            ++*launches;
            if ((e = launch_build_tree(a.parent, a.T, a.batch, a.tree_anc, a.tree_depth, a.tree_ok, a.err, s)) !=
                cudaSuccess)
                return e;
        }
        if (a.y) {
            ++*launches;
            if ((e = launch_cb_pairs(a, s)) != cudaSuccess) return e;
        }
        ++*launches;
        return launch_scan_simt(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace stree

extern "C" {

stree_status stree_ctx_create(stree_ctx **out)
{
    if (!out) return STREE_ERR_INVALID_ARG;
    *out = nullptr;
    stree_ctx *c = new (std::nothrow) stree_ctx();
    if (!c) return STREE_ERR_CUDA;
    if (cudaGetDevice(&c->device) != cudaSuccess ||
        cudaMalloc(reinterpret_cast<void **>(&c->err), 4 * sizeof(int32_t)) != cudaSuccess ||
        cudaMemset(c->err, 0, 4 * sizeof(int32_t)) != cudaSuccess) {
        if (c->err) cudaFree(c->err);
        delete c;
        return STREE_ERR_CUDA;
    }
    *out = c;
    return STREE_OK;
}

stree_status stree_ctx_destroy(stree_ctx *c)
{
    if (!c) return STREE_OK;
    cudaDeviceSynchronize();
    cudaFree(c->anc);
    cudaFree(c->depth);
    cudaFree(c->ok);
    cudaFree(c->cb);
    cudaFree(c->cw);
    cudaFree(c->ci);
    cudaFree(c->err);
    delete c;
    return STREE_OK;
}

stree_status stree_ctx_set_kernel(stree_ctx *c, stree_kernel k)
{
    if (!c) return STREE_ERR_INVALID_ARG;
    if (k != STREE_KERNEL_AUTO && k != STREE_KERNEL_SIMT && k != STREE_KERNEL_TC && k != STREE_KERNEL_SMALL)
        return STREE_ERR_INVALID_ARG;
    c->kernel = k;
    return STREE_OK;
}

stree_status stree_ctx_launch_count(stree_ctx *c, int64_t *count)
{
    if (!c || !count) return STREE_ERR_INVALID_ARG;
    *count = c->launches;
    return STREE_OK;
}

stree_status stree_ctx_set_wait_limit(stree_ctx *c, uint64_t ns)
{
    if (!c) return STREE_ERR_INVALID_ARG;
    c->wait_ns = ns;
    return STREE_OK;
}

stree_status stree_ctx_set_test_fault(stree_ctx *c, int fault)
{
    if (!c || fault < 0 || fault > 1) return STREE_ERR_INVALID_ARG;
    c->fault = fault;
    return STREE_OK;
}

stree_status stree_ctx_last_kernel(stree_ctx *c, stree_kernel *kernel)
{
    if (!c || !kernel) return STREE_ERR_INVALID_ARG;
    *kernel = c->last_kernel;
    return STREE_OK;
}

stree_status stree_build_tree(stree_ctx *c, const int32_t *parent, int n_nodes, int batch,
                              uint32_t *anc_out, int32_t *depth_out, void *stream)
{
    if (!c) return STREE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    stree_status st = build_into_ctx(c, parent, n_nodes, batch, s);
    if (st != STREE_OK) return st;
    size_t W = (n_nodes + 31) / 32;
    if (anc_out && batch > 0)
        if (cudaMemcpyAsync(anc_out, c->anc, (size_t)batch * n_nodes * W * sizeof(uint32_t),
                            cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return STREE_ERR_CUDA;
    if (depth_out && batch > 0)
        if (cudaMemcpyAsync(depth_out, c->depth, (size_t)batch * n_nodes * sizeof(int32_t),
                            cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return STREE_ERR_CUDA;
    return STREE_OK;
}

stree_status stree_tree_scan(stree_ctx *c, const void *x, const void *dt, const float *A,
                             const void *B, const void *C, const float *D, const float *h0,
                             const int32_t *parent, int n_nodes, int batch, int nheads,
                             int headdim, int dstate, int ngroups, stree_dtype dtype,
                             void *y, void *stream)
{
    if (!c) return STREE_ERR_INVALID_ARG;
    ScanArgs a = make_args(x, dt, A, B, C, D, h0, n_nodes, batch, nheads, headdim, dstate, ngroups, dtype, y);
    stree_status st = check_scan_args(a);
    if (st != STREE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((parent || batch == 0) && (st = ensure_tree(c, parent, n_nodes, batch)) != STREE_OK) return st;
    ScanArgs rec = a;
    a.parent = parent;                      // the launch rebuilds the context's tree
    if ((st = run_scan(c, a, s)) != STREE_OK) return st;
    c->last = rec;
    c->has_scan = true;
    return STREE_OK;
}

stree_status stree_commit(stree_ctx *c, const int32_t *path, const int32_t *path_len, int maxlen,
                          float *h_new, void *stream)
{
    if (!c) return STREE_ERR_INVALID_ARG;
    if (!c->has_scan) return STREE_ERR_NO_TREE;
    stree_status st = check_commit_args(path, path_len, maxlen, h_new, c->last.batch);
    if (st != STREE_OK) return st;
    ScanArgs a = c->last;
    a.y = nullptr;
    a.path = path;
    a.path_len = path_len;
    a.maxlen = maxlen;
    a.h_new = h_new;
    if (c->tree_batch != a.batch || c->tree_T != a.T) return STREE_ERR_NO_TREE;
    a.tree = tree_view(c);
    a.err = c->err;
    if (a.batch == 0) return STREE_OK;
    if (commit_supported(a)) {
        const size_t nf = commit_work_floats(a), ni = commit_work_ints(a);
        if ((st = ensure(&c->cw, &c->cap_cw, nf)) != STREE_OK) return st;
        if ((st = ensure(&c->ci, &c->cap_ci, ni)) != STREE_OK) return st;
        const size_t Lc = (size_t)(a.maxlen < a.T ? a.maxlen : a.T);
        CommitWork ws;
        ws.w = c->cw;
        ws.alpha = c->cw + (size_t)a.batch * a.H * Lc;
        ws.pn = c->ci;
        ws.len = c->ci + (size_t)a.batch * Lc;
        c->launches += 2;
        return cuda_status(launch_commit(a, ws, static_cast<cudaStream_t>(stream)));
    }
    ++c->launches;
    return cuda_status(launch_scan_simt(a, static_cast<cudaStream_t>(stream)));
}

stree_status stree_tree_scan_commit(stree_ctx *c, const void *x, const void *dt, const float *A,
                                    const void *B, const void *C, const float *D, const float *h0,
                                    const int32_t *parent, int n_nodes, int batch, int nheads,
                                    int headdim, int dstate, int ngroups, stree_dtype dtype,
                                    const int32_t *path, const int32_t *path_len, int maxlen,
                                    void *y, float *h_new, void *stream)
{
    if (!c) return STREE_ERR_INVALID_ARG;
    ScanArgs a = make_args(x, dt, A, B, C, D, h0, n_nodes, batch, nheads, headdim, dstate, ngroups, dtype, y);
    stree_status st = check_scan_args(a);
    if (st != STREE_OK) return st;
    if ((st = check_commit_args(path, path_len, maxlen, h_new, batch)) != STREE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((parent || batch == 0) && (st = ensure_tree(c, parent, n_nodes, batch)) != STREE_OK) return st;
    ScanArgs rec = a;
    a.parent = parent;                      // the launch rebuilds the context's tree
    a.path = path;
    a.path_len = path_len;
    a.maxlen = maxlen;
    a.h_new = h_new;
    if ((st = run_scan(c, a, s)) != STREE_OK) return st;
    c->last = rec;
    c->has_scan = true;
    return STREE_OK;
}

stree_status stree_resolve_path(stree_ctx *c, const int32_t *path, const int32_t *path_len, int maxlen,
                                int32_t *leaf_out, void *stream)
{
    if (!c || !path || !path_len || !leaf_out || maxlen < 1) return STREE_ERR_INVALID_ARG;
    if (c->tree_batch < 0) return STREE_ERR_NO_TREE;
    if (c->tree_batch > 0) ++c->launches;
    return cuda_status(launch_resolve_path(tree_view(c), path, path_len, maxlen, leaf_out, c->err,
                                           static_cast<cudaStream_t>(stream)));
}

stree_status stree_sync_check(stree_ctx *c, void *stream, int32_t *info)
{
    if (!c) return STREE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h[4] = {0, 0, 0, 0};
    if (cudaStreamSynchronize(s) != cudaSuccess) return STREE_ERR_CUDA;
    if (cudaMemcpy(h, c->err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return STREE_ERR_CUDA;
    if (cudaMemset(c->err, 0, sizeof(h)) != cudaSuccess) return STREE_ERR_CUDA;
    if (info) memcpy(info, h, sizeof(h));
    return static_cast<stree_status>(h[0]);
}

const char *stree_status_string(stree_status st)
{
    switch (st) {
    case STREE_OK: return "ok";
    case STREE_ERR_INVALID_ARG: return "invalid argument";
    case STREE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case STREE_ERR_BAD_TREE: return "parent array is not a packed tree";
    case STREE_ERR_BAD_PATH: return "accepted path is not a root->node chain of the tree";
    case STREE_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case STREE_ERR_CUDA: return "CUDA runtime error";
    case STREE_ERR_TIMEOUT: return "device wait timed out";
    case STREE_ERR_NO_TREE: return "no tree or scan recorded for these sizes";
    }
    return "unknown status";
}

int stree_version(void) { return 100; }

}  // extern "C"
