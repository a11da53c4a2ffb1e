// k_tree.cu -- tree builder, accepted-path resolver and the C.B pair kernel.
//
// Tree builder: the "tree mask" of the packed token tree ("STree: Speculative
// Tree Decoding for Hybrid State Space Models", scime.ai summary, "Approach"):
// the ancestor matrix L of A_tree = L . log A, stored as one bitmask row per node.
#include "stree_internal.cuh"

namespace stree {
namespace {

// One CTA per sequence.  Validation: node 0 is the only root and every other
// node's parent is an earlier node.  Masks: each thread walks its node's root
// path (at most i steps, since parents strictly decrease) and sets one bit per
// step in its own shared-memory row.
__global__ void __launch_bounds__(256) build_tree_kernel(const int32_t *__restrict__ parent, int T, int W,
                                                         uint32_t *__restrict__ anc,
                                                         int32_t *__restrict__ depth,
                                                         int32_t *__restrict__ ok, int32_t *err)
{
    __shared__ int32_t par[kMaxNodes];
    __shared__ uint32_t rows[kMaxNodes * kMaxWords];
    __shared__ int bad;
    const int b = blockIdx.x;
    // A scan launched as a programmatic dependent may start its prologue now; it
    // waits for this grid's completion before it reads the masks.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < T; i += blockDim.x) {
        int p = parent[(size_t)b * T + i];
        par[i] = p;
        bool valid = (i == 0) ? (p == -1) : (p >= 0 && p < i);
        if (!valid) {
            atomicOr(&bad, 1);
            latch_error(err, STREE_ERR_BAD_TREE, b, i, p);
        }
    }
    for (int k = threadIdx.x; k < T * W; k += blockDim.x) rows[k] = 0u;
    __syncthreads();
    uint32_t *anc_b = anc + (size_t)b * T * W;
    if (bad) {
        for (int k = threadIdx.x; k < T * W; k += blockDim.x) anc_b[k] = 0u;
        for (int i = threadIdx.x; i < T; i += blockDim.x) depth[(size_t)b * T + i] = 0;
        if (threadIdx.x == 0) ok[b] = 0;
        return;
    }
    for (int i = threadIdx.x; i < T; i += blockDim.x) {
        int d = -1;
        for (int k = i; k >= 0; k = par[k]) {
            rows[i * W + (k >> 5)] |= 1u << (k & 31);
            ++d;
        }
        depth[(size_t)b * T + i] = d;
    }
    __syncthreads();
    for (int k = threadIdx.x; k < T * W; k += blockDim.x) anc_b[k] = rows[k];
    if (threadIdx.x == 0) ok[b] = 1;
}

// One thread per sequence.  A path is valid when 0 <= len <= min(maxlen, T) and
// path[k] is the ancestor of its last node at depth k, for every k (with the
// last node at depth len-1): exactly the root->leaf chain, since a node has one
// ancestor at each depth.
__global__ void resolve_path_kernel(TreeView tv, const int32_t *__restrict__ path,
                                    const int32_t *__restrict__ path_len, int maxlen,
                                    int32_t *__restrict__ leaf_out, int32_t *err)
{
    int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= tv.batch) return;
    int len = path_len[b];
    int result = -1;
    if (!tv.ok[b]) {
        result = -2;
    } else if (len < 0 || len > maxlen || len > tv.T) {
        result = -2;
        latch_error(err, STREE_ERR_BAD_PATH, b, -1, len);
    } else if (len > 0) {
        const int32_t *pb = path + (size_t)b * maxlen;
        int leaf = pb[len - 1];
        if (leaf < 0 || leaf >= tv.T || tv.depth[(size_t)b * tv.T + leaf] != len - 1) {
            result = -2;
            latch_error(err, STREE_ERR_BAD_PATH, b, len - 1, leaf);
        } else {
            const uint32_t *m = tv.anc + ((size_t)b * tv.T + leaf) * tv.W;
            result = leaf;
            for (int k = 0; k < len; ++k) {
                int j = pb[k];
                bool good = j >= 0 && j < tv.T && ((m[j >> 5] >> (j & 31)) & 1u) &&
                            tv.depth[(size_t)b * tv.T + j] == k;
                if (!good) {
                    result = -2;
                    latch_error(err, STREE_ERR_BAD_PATH, b, k, j);
                    break;
                }
            }
        }
    }
    leaf_out[b] = result;
}

// cb[b,g,i,j] = C_i . B_j for j an ancestor-or-self of i, 0 elsewhere (the
// "C.B on tree pairs" factor of the tree term).  One CTA per (sequence, group);
// a warp per pair row chunk, lanes over the state dimension.
__global__ void __launch_bounds__(256) cb_pairs_kernel(ScanArgs a)
{
    const int b = blockIdx.x, g = blockIdx.y;
    const int T = a.T, N = a.N, G = a.G, W = a.tree.W;
    float *out = a.cb + ((size_t)b * G + g) * T * T;
    if (!a.tree.ok[b]) return;
    const uint32_t *anc_b = a.tree.anc + (size_t)b * T * W;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    for (int i = warp; i < T; i += nwarps) {
        const size_t ci = (((size_t)b * T + i) * G + g) * N;
        for (int j = 0; j < T; ++j) {
            bool is_anc = (anc_b[i * W + (j >> 5)] >> (j & 31)) & 1u;
            float acc = 0.f;
            if (is_anc) {
                const size_t bj = (((size_t)b * T + j) * G + g) * N;
                for (int n = lane; n < N; n += 32)
                    acc = fmaf(load_as_float(a.C, ci + n, a.dtype), load_as_float(a.B, bj + n, a.dtype), acc);
                for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            }
            if (lane == 0) out[(size_t)i * T + j] = acc;
        }
    }
}

}  // namespace

cudaError_t launch_build_tree(const int32_t *parent, int T, int batch, uint32_t *anc, int32_t *depth,
                              int32_t *ok, int32_t *err, cudaStream_t s)
{
    if (batch == 0) return cudaSuccess;
    int W = (T + 31) / 32;
    build_tree_kernel<<<batch, 256, 0, s>>>(parent, T, W, anc, depth, ok, err);
    return cudaGetLastError();
}

cudaError_t launch_resolve_path(const TreeView &tv, const int32_t *path, const int32_t *path_len,
                                int maxlen, int32_t *leaf_out, int32_t *err, cudaStream_t s)
{
    if (tv.batch == 0) return cudaSuccess;
    resolve_path_kernel<<<(tv.batch + 127) / 128, 128, 0, s>>>(tv, path, path_len, maxlen, leaf_out, err);
    return cudaGetLastError();
}

cudaError_t launch_cb_pairs(const ScanArgs &a, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    cb_pairs_kernel<<<dim3(a.batch, a.G), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace stree
