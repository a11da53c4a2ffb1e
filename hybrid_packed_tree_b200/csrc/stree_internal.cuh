// stree_internal.cuh -- types shared by the libstree translation units.
//
// Nothing here is part of the C ABI (include/stree.h is).  The context owns the
// device workspace; kernels receive plain pointers through ScanArgs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "stree.h"

namespace stree {

constexpr int kMaxNodes = 256;                 // n_nodes limit (mask words <= 8)
constexpr int kMaxWords = kMaxNodes / 32;
constexpr int kMaxDim = 256;                   // headdim / dstate limit

// Device error word: {status, sequence, position, detail}.  The first error wins.
__device__ __forceinline__ void latch_error(int32_t *err, int code, int b, int pos, int detail)
{
    if (atomicCAS(err, 0, code) == 0) {
        err[1] = b;
        err[2] = pos;
        err[3] = detail;
    }
}

struct TreeView {
    const uint32_t *anc;     // [batch, T, W]
    const int32_t *depth;    // [batch, T]
    const int32_t *ok;       // [batch]
    int T, W, batch;
};

struct ScanArgs {
    const void *x, *dt, *B, *C;
    const float *A, *D, *h0;
    int T, batch, H, P, N, G;
    stree_dtype dtype;
    void *y;                           // NULL: no outputs y (commit only)
    const int32_t *path, *path_len;    // NULL path: no commit
    int maxlen;
    float *h_new;
    TreeView tree;
    // Set when the call passes the tree: the small-batch and tensor-core kernels
    // then build the masks themselves from parent[] and write them (masks, depths,
    // flags, the same layouts as TreeView) to the tree_* arrays for later calls;
    // the CUDA-core path has the tree builder write them first.
    const int32_t *parent;
    uint32_t *tree_anc;
    int32_t *tree_depth, *tree_ok;
    float *cb;                         // scratch [batch, G, T, T]: C_i . B_j on ancestor pairs
    float *pair_scratch;               // tensor-core kernel, trees with more ancestor pairs than its
                                       // shared memory holds: tc_pair_scratch_floats() floats (or NULL)
    int32_t *err;
    unsigned long long wait_ns;        // tensor-core kernel: bounded-wait limit (0: the default)
    int fault;                         // tensor-core kernel: failure-path test hook (0: off)
};

// The kernels that can run a scan.
enum class ScanPath { Small, Tc, Simt };

// Kernel launchers (each returns cudaSuccess or the launch error).
cudaError_t launch_build_tree(const int32_t *parent, int T, int batch, uint32_t *anc, int32_t *depth,
                              int32_t *ok, int32_t *err, cudaStream_t s);
cudaError_t launch_resolve_path(const TreeView &tv, const int32_t *path, const int32_t *path_len,
                                int maxlen, int32_t *leaf_out, int32_t *err, cudaStream_t s);
cudaError_t launch_cb_pairs(const ScanArgs &a, cudaStream_t s);
cudaError_t launch_scan_simt(const ScanArgs &a, cudaStream_t s);

// Tensor-core path: whether the shape is supported, and the launcher.
bool tc_supported(const ScanArgs &a);
cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t s);
// Floats of ScanArgs::pair_scratch the tensor-core kernel uses for this shape
// (0: every tree's pairs fit in its shared memory).
size_t tc_pair_scratch_floats(const ScanArgs &a);

// Gated delta rule on the tensor cores (bf16, d_k = d_v = 128, up to 64 nodes).
bool gdn_tc_supported(int n_nodes, int dk, int dv, stree_dtype dtype);
cudaError_t launch_gdn_tc(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                          const float *erase, const float *S0, const int32_t *parent, int n_nodes, int batch,
                          int heads_v, int heads_k, const int32_t *path, const int32_t *path_len, int maxlen, void *o,
                          float *S_new, int32_t *err, cudaStream_t s);

// Small-batch path: whether the shape is supported, and the launcher.
bool small_supported(const ScanArgs &a);
cudaError_t launch_scan_small(const ScanArgs &a, cudaStream_t s);

// Commit by replay of the accepted path alone (no tree term, no root term).  Its
// workspace: per sequence the path's nodes and length, per (sequence, head) the
// replay weights and exp(L_leaf).  Sizes in floats / ints from the two helpers.
struct CommitWork {
    float *w;          // [batch, H, Lc]
    float *alpha;      // [batch, H]
    int32_t *pn;       // [batch, Lc]
    int32_t *len;      // [batch]
};
bool commit_supported(const ScanArgs &a);
size_t commit_work_floats(const ScanArgs &a);
size_t commit_work_ints(const ScanArgs &a);
cudaError_t launch_commit(const ScanArgs &a, const CommitWork &ws, cudaStream_t s);

// Resolves a kernel selection against the shape; false when the selection
// cannot run it (STREE_ERR_UNSUPPORTED).
bool select_path(stree_kernel sel, const ScanArgs &a, ScanPath *out);

// Launches the scan (and the fused commit when a.path is set) on `path`.  With
// a.parent set the tree is rebuilt into a.tree_*; the CUDA-core path needs a.cb.
// *launches is increased by the number of kernels launched.
cudaError_t launch_scan(ScanPath path, const ScanArgs &a, cudaStream_t s, int64_t *launches);

__device__ __forceinline__ float load_as_float(const void *p, size_t i, stree_dtype dt)
{
    if (dt == STREE_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ void store_from_float(void *p, size_t i, float v, stree_dtype dt)
{
    if (dt == STREE_BF16) reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
    else reinterpret_cast<float *>(p)[i] = v;
}

}  // namespace stree
