// k_sample.cu -- stochastic verification of the draft tree by multi-step
// speculative sampling, sm_100a.
//
// The rule (STree summary, "Builds on": SpecInfer and speculative sampling, used at
// temperature > 0; TreeSpark summary, "Guaranteeing Lossless Decoding": residual
// resampling keeps the output distribution the target's): at the current node u
// with target distribution p = softmax(target_logits[u] / temperature) and draft
// distribution q = softmax(draft_logits[u] / temperature) -- from which the tokens
// of u's children were drawn -- the children are tried in increasing node order;
// child c with token t is accepted when u_accept[c] * q[t] < p[t] (probability
// min(1, p[t] / q[t])) and the walk moves on to c; after each rejection p becomes
// the residual max(p - q, 0), renormalised (kept as it is when that residual is
// all zero).  When no child is accepted, u is a leaf, or the path holds maxlen
// nodes, the bonus token is drawn from the current p by inverse CDF: the first
// token whose cumulative probability exceeds u_bonus times the total.
//
// Design.  The walk is sequential, every step a pass over the vocabulary: one CTA
// of 1024 threads per sequence keeps the current p (fp32, the residuals
// included) in shared memory -- up to 53,248 tokens, 208 KB -- and streams the
// logits rows of the visited nodes from HBM (a draft row is read once for its
// softmax statistics, then again from L2 by each residual).  Each pass walks
// the row in 16-byte chunks per thread (when rows are 16-byte aligned), unrolled
// so that several chunk loads are in flight, with block reductions of (max, sum)
// pairs; the bonus draw is a block prefix sum over contiguous per-thread chunks.
// All arithmetic is fp32.
#include <mutex>

#include "stree_internal.cuh"

namespace stree {
namespace {

constexpr int kSThreads = 1024;
constexpr int kSWarps = kSThreads / 32;
constexpr int kMaxVocabSmem = 53248;
constexpr int kMaxDevices = 64;

// kE consecutive logits starting at v (one 16-byte load when kE > 1: the row
// start and v are then multiples of 16 bytes).
template <int kE>
__device__ __forceinline__ void ld_chunk(const float *r, int v, float (&out)[kE])
{
    if constexpr (kE == 4) {
        const float4 x = __ldg(reinterpret_cast<const float4 *>(r + v));
        out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
    } else {
#pragma unroll
        for (int e = 0; e < kE; ++e) out[e] = __ldg(r + v + e);
    }
}
template <int kE>
__device__ __forceinline__ void ld_chunk(const __nv_bfloat16 *r, int v, float (&out)[kE])
{
    if constexpr (kE == 8) {
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(r + v));
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            out[2 * e] = f.x;
            out[2 * e + 1] = f.y;
        }
    } else {
#pragma unroll
        for (int e = 0; e < kE; ++e) out[e] = __bfloat162float(r[v + e]);
    }
}

__device__ __forceinline__ float ld_logit(const float *r, int v) { return __ldg(r + v); }
__device__ __forceinline__ float ld_logit(const __nv_bfloat16 *r, int v) { return __bfloat162float(r[v]); }

struct Red {
    float a[kSWarps], b[kSWarps];
};

// Block-wide sum; every thread gets the result.
__device__ __forceinline__ float block_sum(float v, Red &red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red.a[warp] = v;
    __syncthreads();
    v = red.a[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Merges (m, s) pairs meaning s * exp(-m) (running softmax statistics).
__device__ __forceinline__ void merge_ms(float &m, float &s, float m2, float s2)
{
    const float mm = fmaxf(m, m2);
    s = (m == -INFINITY ? 0.f : s * __expf(m - mm)) + (m2 == -INFINITY ? 0.f : s2 * __expf(m2 - mm));
    m = mm;
}

// Max and sum of exp(z - max) over z_v = row[v] * inv_t; every thread gets both.
// Each thread takes chunks of kE consecutive values, the loop unrolled so that
// several chunk loads are in flight at once.
template <typename E, int kE>
__device__ __forceinline__ void row_stats(const E *row, int V, float inv_t, Red &red, float &m, float &s)
{
    m = -INFINITY;
    s = 0.f;
#pragma unroll 4
    for (int v0 = threadIdx.x * kE; v0 < V; v0 += kSThreads * kE) {
        float z[kE];
        ld_chunk<kE>(row, v0, z);
#pragma unroll
        for (int e = 0; e < kE; ++e) {
            const float ze = z[e] * inv_t;
            if (ze > m) {
                s = (m == -INFINITY ? 0.f : s * __expf(m - ze)) + 1.f;
                m = ze;
            } else {
                s += __expf(ze - m);
            }
        }
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) merge_ms(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
    __syncthreads();
    if (lane == 0) {
        red.a[warp] = m;
        red.b[warp] = s;
    }
    __syncthreads();
    m = red.a[lane];
    s = red.b[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) merge_ms(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
}

// p = softmax(row * inv_t) into shared memory.
template <typename E, int kE>
__device__ __forceinline__ void load_softmax(const E *row, int V, float inv_t, float *p, Red &red)
{
    float m, s;
    row_stats<E, kE>(row, V, inv_t, red, m, s);
    const float inv = 1.f / s;
#pragma unroll 4
    for (int v0 = threadIdx.x * kE; v0 < V; v0 += kSThreads * kE) {
        float z[kE];
        ld_chunk<kE>(row, v0, z);
#pragma unroll
        for (int e = 0; e < kE; ++e) p[v0 + e] = __expf(z[e] * inv_t - m) * inv;
    }
    __syncthreads();
}

template <typename E, int kE>
__global__ void __launch_bounds__(kSThreads, 1)
accept_sampling_kernel(const E *__restrict__ tl, const E *__restrict__ dl, int V, const int32_t *__restrict__ tokens,
                       const int32_t *__restrict__ parent, int T, float inv_t, const float *__restrict__ u_accept,
                       const float *__restrict__ u_bonus, int maxlen, int32_t *__restrict__ path,
                       int32_t *__restrict__ path_len, int32_t *__restrict__ bonus, int32_t *err)
{
    extern __shared__ __align__(16) float p[];          // [V] current target distribution
    __shared__ int32_t par[kMaxNodes], tok[kMaxNodes];
    __shared__ float ua[kMaxNodes];
    __shared__ Red red;
    __shared__ int32_t s_first, s_badtree, s_badtok;
    const int s = blockIdx.x, tid = threadIdx.x;
    int32_t *out = path + (size_t)s * maxlen;
    if (tid == 0) {
        s_badtree = 0;
        s_badtok = T;
    }
    __syncthreads();
    for (int i = tid; i < T; i += kSThreads) {
        par[i] = parent[(size_t)s * T + i];
        tok[i] = tokens[(size_t)s * T + i];
        ua[i] = u_accept[(size_t)s * T + i];
        const int pi = par[i];
        if ((i == 0) ? (pi != -1) : (pi < 0 || pi >= i)) s_badtree = 1;
        if (i > 0 && (tok[i] < 0 || tok[i] >= V)) atomicMin(&s_badtok, i);
    }
    __syncthreads();
    if (s_badtree || s_badtok < T) {
        // Not a packed tree, or a draft token outside the vocabulary.
        for (int k = tid; k < maxlen; k += kSThreads) out[k] = -1;
        if (tid == 0) {
            path_len[s] = 0;
            bonus[s] = -1;
            if (err) {
                if (s_badtree) latch_error(err, STREE_ERR_BAD_TREE, s, -1, 0);
                else latch_error(err, STREE_ERR_INVALID_ARG, s, s_badtok, tok[s_badtok]);
            }
        }
        return;
    }
    const E *trow0 = tl + (size_t)s * T * V, *drow0 = dl + (size_t)s * T * V;
    int cur = 0, len = 1;
    if (tid == 0) out[0] = 0;
    load_softmax<E, kE>(trow0, V, inv_t, p, red);
    while (true) {
        int next = -1;
        if (len < maxlen) {
            const E *drow = drow0 + (size_t)cur * V;
            float mq, sq;
            row_stats<E, kE>(drow, V, inv_t, red, mq, sq);
            const float inv_sq = 1.f / sq;
            for (int c = cur + 1; c < T; ++c) {             // children follow their parent
                if (par[c] != cur) continue;
                const int t = tok[c];
                const float qt = __expf(ld_logit(drow, t) * inv_t - mq) * inv_sq;
                if (ua[c] * qt < p[t]) {
                    next = c;
                    break;
                }
                // Rejected: p <- max(p - q, 0), renormalised (unchanged if all zero).
                float r = 0.f;
#pragma unroll 4
                for (int v0 = tid * kE; v0 < V; v0 += kSThreads * kE) {
                    float z[kE];
                    ld_chunk<kE>(drow, v0, z);
#pragma unroll
                    for (int e = 0; e < kE; ++e) r += fmaxf(p[v0 + e] - __expf(z[e] * inv_t - mq) * inv_sq, 0.f);
                }
                r = block_sum(r, red);
                if (r > 0.f) {
                    const float inv_r = 1.f / r;
#pragma unroll 4
                    for (int v0 = tid * kE; v0 < V; v0 += kSThreads * kE) {
                        float z[kE];
                        ld_chunk<kE>(drow, v0, z);
#pragma unroll
                        for (int e = 0; e < kE; ++e)
                            p[v0 + e] = fmaxf(p[v0 + e] - __expf(z[e] * inv_t - mq) * inv_sq, 0.f) * inv_r;
                    }
                }
                __syncthreads();
            }
        }
        if (next < 0) break;
        if (tid == 0) out[len] = next;
        cur = next;
        ++len;
        load_softmax<E, kE>(trow0 + (size_t)cur * V, V, inv_t, p, red);
    }
    // Bonus token: inverse CDF of p over contiguous per-thread chunks.
    const int chunk = (V + kSThreads - 1) / kSThreads;
    const int v0 = min(V, tid * chunk), v1 = min(V, v0 + chunk);
    float local = 0.f;
    for (int v = v0; v < v1; ++v) local += p[v];
    // Exclusive prefix of the chunk sums: warp scan, then across warps.
    const int lane = tid & 31, warp = tid >> 5;
    float incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    __syncthreads();
    if (lane == 31) red.a[warp] = incl;
    if (tid == 0) s_first = V;
    __syncthreads();
    float wpre = 0.f, total = 0.f;
    for (int w = 0; w < kSWarps; ++w) {
        if (w < warp) wpre += red.a[w];
        total += red.a[w];
    }
    const float x = u_bonus[s] * total;
    float run = wpre + incl - local;
    for (int v = v0; v < v1; ++v) {
        run += p[v];
        if (run > x) {
            atomicMin(&s_first, v);
            break;
        }
    }
    __syncthreads();
    for (int k = len + tid; k < maxlen; k += kSThreads) out[k] = -1;
    if (tid == 0) {
        path_len[s] = len;
        bonus[s] = min(s_first, V - 1);
    }
}

std::mutex g_mutex;
bool g_prepared[kMaxDevices] = {};

cudaError_t prepare()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_prepared[dev]) return cudaSuccess;
    const int bytes = kMaxVocabSmem * (int)sizeof(float);
    if ((e = cudaFuncSetAttribute(accept_sampling_kernel<float, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  bytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(accept_sampling_kernel<float, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  bytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(accept_sampling_kernel<__nv_bfloat16, 1>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(accept_sampling_kernel<__nv_bfloat16, 8>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess)
        return e;
    g_prepared[dev] = true;
    return cudaSuccess;
}

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace
}  // namespace stree

using namespace stree;

extern "C" stree_status stree_accept_sampling(const void *target_logits, const void *draft_logits,
                                              stree_dtype logit_dtype, int vocab, const int32_t *draft_tokens,
                                              const int32_t *parent, int n_nodes, int batch, float temperature,
                                              const float *u_accept, const float *u_bonus, int maxlen,
                                              int32_t *accepted_path, int32_t *path_len, int32_t *bonus_token,
                                              int32_t *err_out, void *stream)
{
    if (batch < 0 || n_nodes < 1 || n_nodes > kMaxNodes || vocab < 1 || vocab > kMaxVocabSmem || maxlen < 1)
        return STREE_ERR_UNSUPPORTED;
    if (logit_dtype != STREE_F32 && logit_dtype != STREE_BF16) return STREE_ERR_UNSUPPORTED;
    if (!(temperature > 0.f) || (long long)batch * n_nodes * vocab > (1ll << 40)) return STREE_ERR_INVALID_ARG;
    if (batch == 0) return STREE_OK;
    if (!target_logits || !draft_logits || !draft_tokens || !parent || !u_accept || !u_bonus || !accepted_path ||
        !path_len || !bonus_token)
        return STREE_ERR_INVALID_ARG;
    const uintptr_t es = logit_dtype == STREE_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(target_logits) & (es - 1)) || (reinterpret_cast<uintptr_t>(draft_logits) & (es - 1)) ||
        !aligned4(draft_tokens) || !aligned4(parent) || !aligned4(u_accept) || !aligned4(u_bonus) ||
        !aligned4(accepted_path) || !aligned4(path_len) || !aligned4(bonus_token) || !aligned4(err_out))
        return STREE_ERR_MISALIGNED;
    if (prepare() != cudaSuccess) return STREE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (err_out && cudaMemsetAsync(err_out, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return STREE_ERR_CUDA;
    const size_t smem = (size_t)vocab * sizeof(float);
    const float inv_t = 1.f / temperature;
    // 16-byte chunk loads when every row starts on a 16-byte boundary.
    const bool vec = (reinterpret_cast<uintptr_t>(target_logits) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(draft_logits) & 15u) == 0 && ((size_t)vocab * es) % 16 == 0;
    if (logit_dtype == STREE_BF16) {
        const __nv_bfloat16 *t = static_cast<const __nv_bfloat16 *>(target_logits);
        const __nv_bfloat16 *d = static_cast<const __nv_bfloat16 *>(draft_logits);
        if (vec)
            accept_sampling_kernel<__nv_bfloat16, 8><<<batch, kSThreads, smem, s>>>(
                t, d, vocab, draft_tokens, parent, n_nodes, inv_t, u_accept, u_bonus, maxlen, accepted_path, path_len,
                bonus_token, err_out);
        else
            accept_sampling_kernel<__nv_bfloat16, 1><<<batch, kSThreads, smem, s>>>(
                t, d, vocab, draft_tokens, parent, n_nodes, inv_t, u_accept, u_bonus, maxlen, accepted_path, path_len,
                bonus_token, err_out);
    } else {
        const float *t = static_cast<const float *>(target_logits);
        const float *d = static_cast<const float *>(draft_logits);
        if (vec)
            accept_sampling_kernel<float, 4><<<batch, kSThreads, smem, s>>>(
                t, d, vocab, draft_tokens, parent, n_nodes, inv_t, u_accept, u_bonus, maxlen, accepted_path, path_len,
                bonus_token, err_out);
        else
            accept_sampling_kernel<float, 1><<<batch, kSThreads, smem, s>>>(
                t, d, vocab, draft_tokens, parent, n_nodes, inv_t, u_accept, u_bonus, maxlen, accepted_path, path_len,
                bonus_token, err_out);
    }
    return cudaGetLastError() == cudaSuccess ? STREE_OK : STREE_ERR_CUDA;
}
