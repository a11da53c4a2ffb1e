// k_accept.cu -- greedy (temperature 0) verification of the draft tree.
//
// Tree speculative decoding at temperature 0 ("STree: Speculative Tree Decoding
// for Hybrid State Space Models", scime.ai summary, "Key results" at temperature
// 0; "Builds on": SpecInfer, speculative sampling): the target's prediction after
// node i is the most probable next token, argmax_v logits[i][v]; from the root, a
// child is accepted when its draft token equals the prediction after its parent,
// and the walk continues from it.  The accepted path (root first) is what the
// commit replays; the bonus token is the prediction after the last accepted node.
// Ties resolve to the smaller token id, equal sibling tokens to the smaller node.
//
// Two kernels: the argmax of every (sequence, node) row of logits -- the bytes
// of the step, streamed with 16-byte loads by one CTA per row -- then one warp per
// sequence validates the tree and walks it (a ballot finds the first matching
// child among 32 nodes at a time).
#include "stree_internal.cuh"

namespace stree {
namespace {

constexpr int kArgThreads = 256;

// (value, index) pairs: larger value wins, then the smaller index.
__device__ __forceinline__ void better(float &v, int &i, float v2, int i2)
{
    if (v2 > v || (v2 == v && i2 < i)) {
        v = v2;
        i = i2;
    }
}

template <typename E, int kVec>
__global__ void __launch_bounds__(kArgThreads) argmax_rows_kernel(const E *__restrict__ logits, int V,
                                                                  int32_t *__restrict__ pred)
{
    const size_t row = blockIdx.x;
    const E *lr = logits + row * (size_t)V;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    // Rows start 16-byte aligned when V * sizeof(E) is a multiple of 16 (kVec > 1).
    const int nvec = kVec > 1 ? V / kVec : 0;
    for (int q = threadIdx.x; q < nvec; q += kArgThreads) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(lr) + q);
        const E *e = reinterpret_cast<const E *>(&raw);
#pragma unroll
        for (int u = 0; u < kVec; ++u) better(best, bi, (float)e[u], q * kVec + u);
    }
    for (int v = nvec * kVec + threadIdx.x; v < V; v += kArgThreads) better(best, bi, (float)lr[v], v);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, best, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
        better(best, bi, v2, i2);
    }
    __shared__ float wv[kArgThreads / 32];
    __shared__ int wi[kArgThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        wv[warp] = best;
        wi[warp] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kArgThreads / 32; ++w) better(best, bi, wv[w], wi[w]);
        pred[row] = bi == 0x7fffffff ? 0 : bi;       // a row of NaN only: token 0
    }
}

// One warp per sequence.
__global__ void accept_walk_kernel(const int32_t *__restrict__ parent, const int32_t *__restrict__ tokens,
                                   const int32_t *__restrict__ pred, int T, int batch, int maxlen,
                                   int32_t *__restrict__ path, int32_t *__restrict__ path_len,
                                   int32_t *__restrict__ bonus, int32_t *err)
{
    const int s = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (s >= batch) return;
    const int32_t *par = parent + (size_t)s * T;
    const int32_t *tok = tokens + (size_t)s * T;
    int32_t *out = path + (size_t)s * maxlen;
    bool bad = false;
    for (int i = lane; i < T; i += 32) {
        const int p = par[i];
        bad |= (i == 0) ? (p != -1) : (p < 0 || p >= i);
    }
    if (__any_sync(0xffffffffu, bad)) {
        for (int k = lane; k < maxlen; k += 32) out[k] = -1;
        if (lane == 0) {
            path_len[s] = 0;
            bonus[s] = -1;
            if (err) latch_error(err, STREE_ERR_BAD_TREE, s, -1, 0);
        }
        return;
    }
    int cur = 0, len = 1;
    if (lane == 0) out[0] = 0;
    while (len < maxlen) {
        const int want = pred[(size_t)s * T + cur];
        int next = -1;
        for (int c0 = cur + 1; c0 < T && next < 0; c0 += 32) {      // children follow their parent
            const int c = c0 + lane;
            const bool hit = c < T && par[c] == cur && tok[c] == want;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            if (m) next = c0 + __ffs(m) - 1;
        }
        if (next < 0) break;
        if (lane == 0) out[len] = next;
        cur = next;
        ++len;
    }
    for (int k = len + lane; k < maxlen; k += 32) out[k] = -1;
    if (lane == 0) {
        path_len[s] = len;
        bonus[s] = pred[(size_t)s * T + cur];
    }
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace stree

using namespace stree;

extern "C" stree_status stree_accept_greedy(const void *logits, stree_dtype logit_dtype, int vocab,
                                            const int32_t *draft_tokens, const int32_t *parent, int n_nodes,
                                            int batch, int maxlen, int32_t *pred_out, int32_t *accepted_path,
                                            int32_t *path_len, int32_t *bonus_token, int32_t *err_out,
                                            void *stream)
{
    if (batch < 0 || n_nodes < 1 || n_nodes > kMaxNodes || vocab < 1 || maxlen < 1) return STREE_ERR_UNSUPPORTED;
    if (logit_dtype != STREE_F32 && logit_dtype != STREE_BF16) return STREE_ERR_UNSUPPORTED;
    if ((long long)batch * n_nodes > 0x7fffffffLL) return STREE_ERR_UNSUPPORTED;
    if (batch == 0) return STREE_OK;
    if (!logits || !draft_tokens || !parent || !pred_out || !accepted_path || !path_len || !bonus_token)
        return STREE_ERR_INVALID_ARG;
    const size_t es = logit_dtype == STREE_BF16 ? 2 : 4;
    if (!aligned(logits, es) || !aligned(draft_tokens, 4) || !aligned(parent, 4) || !aligned(pred_out, 4) ||
        !aligned(accepted_path, 4) || !aligned(path_len, 4) || !aligned(bonus_token, 4) || !aligned(err_out, 4))
        return STREE_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (err_out && cudaMemsetAsync(err_out, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return STREE_ERR_CUDA;
    const unsigned rows = (unsigned)(batch * n_nodes);
    // 16-byte loads when every row starts on a 16-byte boundary.
    const bool vec = aligned(logits, 16) && ((size_t)vocab * es) % 16 == 0;
    if (logit_dtype == STREE_BF16) {
        if (vec)
            argmax_rows_kernel<__nv_bfloat16, 8><<<rows, kArgThreads, 0, s>>>(
                static_cast<const __nv_bfloat16 *>(logits), vocab, pred_out);
        else
            argmax_rows_kernel<__nv_bfloat16, 1><<<rows, kArgThreads, 0, s>>>(
                static_cast<const __nv_bfloat16 *>(logits), vocab, pred_out);
    } else {
        if (vec)
            argmax_rows_kernel<float, 4><<<rows, kArgThreads, 0, s>>>(static_cast<const float *>(logits), vocab,
                                                                     pred_out);
        else
            argmax_rows_kernel<float, 1><<<rows, kArgThreads, 0, s>>>(static_cast<const float *>(logits), vocab,
                                                                     pred_out);
    }
    if (cudaGetLastError() != cudaSuccess) return STREE_ERR_CUDA;
    const int warps = 4;
    accept_walk_kernel<<<(batch + warps - 1) / warps, warps * 32, 0, s>>>(parent, draft_tokens, pred_out, n_nodes,
                                                                          batch, maxlen, accepted_path, path_len,
                                                                          bonus_token, err_out);
    return cudaGetLastError() == cudaSuccess ? STREE_OK : STREE_ERR_CUDA;
}
