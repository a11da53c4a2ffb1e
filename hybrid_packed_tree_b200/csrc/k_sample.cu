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
// Design.  The walk is sequential, every step a pass over the vocabulary.  A
// sequence is walked by a cluster of up to eight CTAs of 1024 threads (about 1024
// tokens or more each); CTA r keeps its slice of the current p (fp32, the residuals
// included) in shared memory and streams that slice of the visited nodes' logits
// rows from HBM (a draft row is read once for its softmax statistics, then again
// from L2 by each residual).  Statistics, residual sums and the bonus draw's prefix
// are reduced over the CTA, then over the cluster through distributed shared memory
// in the same order in every CTA, so the CTAs take identical decisions; the
// acceptance test reads p[t] from the CTA that owns t.  Each pass walks the slice in
// 16-byte chunks per thread (when rows are 16-byte aligned), unrolled so that
// several chunk loads are in flight.  All arithmetic is fp32.
#include <algorithm>
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

// ---------------------------------------------------------------- the cluster
// A sequence is walked by a cluster of C CTAs (C <= 8); CTA r owns the vocabulary
// slice [lo_r, hi_r) and keeps that slice of p.  Every reduction is first taken over
// the CTA, then over the cluster through distributed shared memory: each CTA puts
// its value in a slot, the cluster synchronises, and warp 0 of every CTA combines
// the C slots in the same order, so all CTAs hold the same bits and take the same
// decisions.  Slots alternate between two buffers, so a slot is not rewritten before
// every CTA has read it (one cluster barrier lies between).

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A float in CTA `rank`'s shared memory at the address of `local` in this CTA.
__device__ __forceinline__ float ld_peer(const float *local, uint32_t rank)
{
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local));
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

struct Cl {
    float slot[2][2];                                  // two buffers of (a, b)
    float res[2];
};


// Cluster-wide combination of each CTA's (a, b): kind 0 merges softmax statistics,
// kind 1 adds a (b unused), kind 2 takes the minimum of a.  Every thread gets it.
// rc counts the cluster exchanges so far (the same in every thread).
__device__ __forceinline__ void cluster_combine(float &a, float &b, int kind, Cl &cl, uint32_t nct, int &rc)
{
    const int k = rc & 1;
    ++rc;
    if (threadIdx.x == 0) {
        cl.slot[k][0] = a;
        cl.slot[k][1] = b;
    }
    cluster_sync();
    if (threadIdx.x < 32) {
        const uint32_t lane = threadIdx.x;
        float x = kind == 0 ? -INFINITY : kind == 1 ? 0.f : INFINITY, y = 0.f;
        if (lane < nct) {
            x = ld_peer(&cl.slot[k][0], lane);
            y = ld_peer(&cl.slot[k][1], lane);
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float x2 = __shfl_xor_sync(0xffffffffu, x, o), y2 = __shfl_xor_sync(0xffffffffu, y, o);
            if (kind == 0) merge_ms(x, y, x2, y2);
            else if (kind == 1) x += x2;
            else x = fminf(x, x2);
        }
        if (lane == 0) {
            cl.res[0] = x;
            cl.res[1] = y;
        }
    }
    __syncthreads();
    a = cl.res[0];
    b = cl.res[1];
    __syncthreads();                                   // res is rewritten by the next combine
}

// Max and sum of exp(z - max) over z_v = row[v] * inv_t, v in [lo, hi) (this
// CTA's slice), then over the cluster; every thread gets both.  Each thread takes
// chunks of kE consecutive values, the loop unrolled so that several chunk loads
// are in flight at once.
template <typename E, int kE>
__device__ __forceinline__ void row_stats(const E *row, int lo, int hi, float inv_t, Red &red, Cl &cl, uint32_t nct,
                                          int &rc, float &m, float &s)
{
    m = -INFINITY;
    s = 0.f;
#pragma unroll 4
    for (int v0 = lo + threadIdx.x * kE; v0 < hi; v0 += kSThreads * kE) {
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
    cluster_combine(m, s, 0, cl, nct, rc);
}

// This CTA's slice of p = softmax(row * inv_t) into shared memory.
template <typename E, int kE>
__device__ __forceinline__ void load_softmax(const E *row, int lo, int hi, float inv_t, float *p, Red &red, Cl &cl,
                                             uint32_t nct, int &rc)
{
    float m, s;
    row_stats<E, kE>(row, lo, hi, inv_t, red, cl, nct, rc, m, s);
    const float inv = 1.f / s;
#pragma unroll 4
    for (int v0 = lo + threadIdx.x * kE; v0 < hi; v0 += kSThreads * kE) {
        float z[kE];
        ld_chunk<kE>(row, v0, z);
#pragma unroll
        for (int e = 0; e < kE; ++e) p[v0 - lo + e] = __expf(z[e] * inv_t - m) * inv;
    }
    __syncthreads();
}

// One cluster of nct CTAs per sequence (grid = batch x nct); `slice` tokens per CTA
// (a multiple of kE), the last slice possibly shorter.
template <typename E, int kE>
__global__ void __launch_bounds__(kSThreads, 1)
accept_sampling_kernel(const E *__restrict__ tl, const E *__restrict__ dl, int V, int slice,
                       const int32_t *__restrict__ tokens, const int32_t *__restrict__ parent, int T, float inv_t,
                       const float *__restrict__ u_accept, const float *__restrict__ u_bonus, int maxlen,
                       int32_t *__restrict__ path, int32_t *__restrict__ path_len, int32_t *__restrict__ bonus,
                       int32_t *err)
{
    extern __shared__ __align__(16) float p[];          // [slice] this CTA's part of the target distribution
    __shared__ int32_t par[kMaxNodes], tok[kMaxNodes];
    __shared__ float ua[kMaxNodes];
    __shared__ Red red;
    __shared__ Cl cl;
    __shared__ int32_t s_first, s_badtree, s_badtok;
    const uint32_t rank = cluster_ctarank();
    uint32_t ncl;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(ncl));
    const int s = blockIdx.x / ncl, tid = threadIdx.x;
    const int lo = min(V, (int)rank * slice), hi = min(V, lo + slice);
    int32_t *out = path + (size_t)s * maxlen;
    int rc = 0;                                          // cluster exchanges so far
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
        // Not a packed tree, or a draft token outside the vocabulary (every CTA of
        // the cluster sees the same, before any cluster barrier).
        if (rank == 0) {
            for (int k = tid; k < maxlen; k += kSThreads) out[k] = -1;
            if (tid == 0) {
                path_len[s] = 0;
                bonus[s] = -1;
                if (err) {
                    if (s_badtree) latch_error(err, STREE_ERR_BAD_TREE, s, -1, 0);
                    else latch_error(err, STREE_ERR_INVALID_ARG, s, s_badtok, tok[s_badtok]);
                }
            }
        }
        return;
    }
    const E *trow0 = tl + (size_t)s * T * V, *drow0 = dl + (size_t)s * T * V;
    int cur = 0, len = 1;
    if (rank == 0 && tid == 0) out[0] = 0;
    load_softmax<E, kE>(trow0, lo, hi, inv_t, p, red, cl, ncl, rc);
    while (true) {
        int next = -1;
        if (len < maxlen) {
            const E *drow = drow0 + (size_t)cur * V;
            float mq, sq;
            row_stats<E, kE>(drow, lo, hi, inv_t, red, cl, ncl, rc, mq, sq);   // its cluster barrier publishes p
            const float inv_sq = 1.f / sq;
            for (int c = cur + 1; c < T; ++c) {             // children follow their parent
                if (par[c] != cur) continue;
                const int t = tok[c];
                const float qt = __expf(ld_logit(drow, t) * inv_t - mq) * inv_sq;
                const uint32_t owner = (uint32_t)(t / slice);
                const float pt = ld_peer(&p[t - (int)owner * slice], owner);
                if (ua[c] * qt < pt) {
                    next = c;
                    break;
                }
                // Rejected: p <- max(p - q, 0), renormalised (unchanged if all zero).
                float r = 0.f;
#pragma unroll 4
                for (int v0 = lo + tid * kE; v0 < hi; v0 += kSThreads * kE) {
                    float z[kE];
                    ld_chunk<kE>(drow, v0, z);
#pragma unroll
                    for (int e = 0; e < kE; ++e)
                        r += fmaxf(p[v0 - lo + e] - __expf(z[e] * inv_t - mq) * inv_sq, 0.f);
                }
                r = block_sum(r, red);
                float unused = 0.f;
                cluster_combine(r, unused, 1, cl, ncl, rc);
                if (r > 0.f) {
                    const float inv_r = 1.f / r;
#pragma unroll 4
                    for (int v0 = lo + tid * kE; v0 < hi; v0 += kSThreads * kE) {
                        float z[kE];
                        ld_chunk<kE>(drow, v0, z);
#pragma unroll
                        for (int e = 0; e < kE; ++e)
                            p[v0 - lo + e] = fmaxf(p[v0 - lo + e] - __expf(z[e] * inv_t - mq) * inv_sq, 0.f) * inv_r;
                    }
                }
                cluster_sync();                               // the updated slices, before any peer reads them
            }
        }
        if (next < 0) break;
        if (rank == 0 && tid == 0) out[len] = next;
        cur = next;
        ++len;
        load_softmax<E, kE>(trow0 + (size_t)cur * V, lo, hi, inv_t, p, red, cl, ncl, rc);
    }
    // Bonus token: inverse CDF of p; contiguous per-thread chunks within the slice,
    // slices in rank order.
    const int n = hi - lo;
    const int chunk = (n + kSThreads - 1) / kSThreads;
    const int v0 = min(n, tid * chunk), v1 = min(n, v0 + chunk);
    float local = 0.f;
    for (int v = v0; v < v1; ++v) local += p[v];
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
    float wpre = 0.f, cta_total = 0.f;
    for (int w = 0; w < kSWarps; ++w) {
        if (w < warp) wpre += red.a[w];
        cta_total += red.a[w];
    }
    // The slices' totals in rank order: this CTA's offset and the grand total.
    const int kt = rc & 1;
    ++rc;
    if (tid == 0) cl.slot[kt][0] = cta_total;
    cluster_sync();
    float before = 0.f, total = 0.f;
    for (uint32_t r = 0; r < ncl; ++r) {
        const float tr = ld_peer(&cl.slot[kt][0], r);
        if (r < rank) before += tr;
        total += tr;
    }
    const float x = u_bonus[s] * total;
    float run = before + wpre + incl - local;
    for (int v = v0; v < v1; ++v) {
        run += p[v];
        if (run > x) {
            atomicMin(&s_first, lo + v);
            break;
        }
    }
    __syncthreads();
    float first = (float)s_first, unused = 0.f;
    cluster_combine(first, unused, 2, cl, ncl, rc);
    if (rank == 0) {
        for (int k = len + tid; k < maxlen; k += kSThreads) out[k] = -1;
        if (tid == 0) {
            path_len[s] = len;
            bonus[s] = min((int)first, V - 1);
        }
    }
    cluster_sync();                                       // no CTA leaves while a peer may read its slots
}

std::mutex g_mutex;
bool g_prepared[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

cudaError_t prepare(int *sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_prepared[dev]) {
        *sms = g_sms[dev];
        return cudaSuccess;
    }
    int n = 0;
    if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    g_sms[dev] = n > 0 ? n : 1;
    *sms = g_sms[dev];
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
    int sms = 0;
    if (prepare(&sms) != cudaSuccess) return STREE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (err_out && cudaMemsetAsync(err_out, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return STREE_ERR_CUDA;
    const float inv_t = 1.f / temperature;
    // 16-byte chunk loads when every row starts on a 16-byte boundary.
    const bool vec = (reinterpret_cast<uintptr_t>(target_logits) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(draft_logits) & 15u) == 0 && ((size_t)vocab * es) % 16 == 0;
    const int kE = vec ? (logit_dtype == STREE_BF16 ? 8 : 4) : 1;
    // A cluster of up to 8 CTAs per sequence, each with at least about 1024 tokens,
    // and no more CTAs in all than one wave over the SMs (one 1024-thread CTA per
    // SM); slices are whole chunks.
    const int ncl = std::min({8, std::max(1, (vocab + 1023) / 1024), std::max(1, sms / batch)});
    int slice = (vocab + ncl - 1) / ncl;
    slice = (slice + kE - 1) / kE * kE;
    if ((long long)batch * ncl > 0x7fffffffLL) return STREE_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(batch * ncl));
    cfg.blockDim = dim3(kSThreads);
    cfg.dynamicSmemBytes = (size_t)slice * sizeof(float);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (logit_dtype == STREE_BF16) {
        const __nv_bfloat16 *t = static_cast<const __nv_bfloat16 *>(target_logits);
        const __nv_bfloat16 *d = static_cast<const __nv_bfloat16 *>(draft_logits);
        e = vec ? cudaLaunchKernelEx(&cfg, accept_sampling_kernel<__nv_bfloat16, 8>, t, d, vocab, slice, draft_tokens,
                                     parent, n_nodes, inv_t, u_accept, u_bonus, maxlen, accepted_path, path_len,
                                     bonus_token, err_out)
                : cudaLaunchKernelEx(&cfg, accept_sampling_kernel<__nv_bfloat16, 1>, t, d, vocab, slice, draft_tokens,
                                     parent, n_nodes, inv_t, u_accept, u_bonus, maxlen, accepted_path, path_len,
                                     bonus_token, err_out);
    } else {
        const float *t = static_cast<const float *>(target_logits);
        const float *d = static_cast<const float *>(draft_logits);
        e = vec ? cudaLaunchKernelEx(&cfg, accept_sampling_kernel<float, 4>, t, d, vocab, slice, draft_tokens, parent,
                                     n_nodes, inv_t, u_accept, u_bonus, maxlen, accepted_path, path_len, bonus_token,
                                     err_out)
                : cudaLaunchKernelEx(&cfg, accept_sampling_kernel<float, 1>, t, d, vocab, slice, draft_tokens, parent,
                                     n_nodes, inv_t, u_accept, u_bonus, maxlen, accepted_path, path_len, bonus_token,
                                     err_out);
    }
    return e == cudaSuccess ? STREE_OK : STREE_ERR_CUDA;
}
