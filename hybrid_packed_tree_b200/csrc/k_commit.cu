// k_commit.cu -- commit by activation replay, sm_100a: the accepted path's state
// rebuilt from the inputs the scan read, streamed at HBM bandwidth.
//
// Method ("STree: Speculative Tree Decoding for Hybrid State Space Models",
// scime.ai summary, "Approach": after acceptance the state of the accepted path is
// recomputed from the stored inputs instead of being kept for every node):
//   h_new = exp(L_leaf) h0 + sum_{q on path} exp(L_leaf - L_q) dt_q x_q (outer) B_q
// with L_q = A_h * sum of dt over the ancestors-or-self of path node q.  The path
// is a root-first chain, so the ancestors of its q-th node are its first q + 1
// nodes and L needs no tree masks: it is a prefix sum along the path (taken in
// path order, which is increasing node order -- the order the scan kernels sum in,
// so both give the same fp32 L).
//
// Design.  The op streams the state (read h0, write h_new: 2 x 4 bytes per
// element) and adds at most a path's worth of rank-1 terms, so it is HBM-bound.
// One CTA per (sequence, head, slab of R = 8192 / dstate rows): the slab is
// R x dstate contiguous fp32 (32 KB).  At entry one bulk request prefetches the
// slab into L2 while the threads read the path; the second round (the checks of
// every path position, dt, and the path's B rows and x values staged in shared
// memory, sixteen positions at a time) is issued before the slab's register
// loads, so the small dependent loads never queue behind the slab.  Several CTAs
// per SM overlap one another's round trips.
#include <climits>

#include "stree_internal.cuh"
#include "tc_ptx.cuh"

namespace stree {
namespace {

constexpr int kCThreads = 256;
constexpr int kCVec = 8;                     // float4 of the slab per thread
constexpr int kSlabFloats = kCThreads * kCVec * 4;
constexpr int kQChunk = 16;                  // path positions staged at a time

struct CommitParams {
    const void *x, *dt, *B;
    const float *A, *h0;
    TreeView tree;
    const int32_t *path, *path_len;
    int maxlen;
    float *h_new;
    int32_t *err;
    int T, H, P, N, G, R, chunks;
    stree_dtype dtype;
};

// Stages B rows and x values (of the slab's rows) of path positions q0 .. q0 + nq - 1;
// node ids are clamped into range (an invalid path's values are never used).
__device__ __forceinline__ void stage_path_rows(const CommitParams &p, float *Bq, float *cfq, const int32_t *pn,
                                                int q0, int nq, int b, int h, int g, int p0, int rows)
{
    const int T = p.T, N = p.N;
    const size_t xrow = (size_t)p.H * p.P;
    for (int e = threadIdx.x; e < nq * N; e += kCThreads) {
        const int qq = e / N, n = e - qq * N;
        const int j = min(max(pn[q0 + qq], 0), T - 1);
        Bq[qq * N + n] = load_as_float(p.B, (((size_t)b * T + j) * p.G + g) * N + n, p.dtype);
    }
    for (int e = threadIdx.x; e < nq * rows; e += kCThreads) {
        const int qq = e / rows, r = e - qq * rows;
        const int j = min(max(pn[q0 + qq], 0), T - 1);
        cfq[qq * rows + r] = load_as_float(p.x, ((size_t)b * T + j) * xrow + (size_t)h * p.P + p0 + r, p.dtype);
    }
}

__global__ void __launch_bounds__(kCThreads, 4) commit_kernel(const CommitParams p)
{
    __shared__ __align__(16) float Bq[kQChunk * kMaxDim];   // staged path rows of B
    __shared__ float cfq[kQChunk * kMaxDim];                // x_q per slab row
    __shared__ int32_t pn[kMaxNodes];
    __shared__ float dq[kMaxNodes], wq[kMaxNodes];
    __shared__ int32_t s_badq, s_ok, s_len;
    __shared__ float s_A;

    const int tid = threadIdx.x;
    const int T = p.T, H = p.H, P = p.P, N = p.N, G = p.G, W = p.tree.W;
    const int chunk = blockIdx.x % p.chunks;
    const int h = (blockIdx.x / p.chunks) % H;
    const int b = blockIdx.x / (p.chunks * H);
    const int g = h / (H / G);
    const int p0 = chunk * p.R, rows = min(p.R, P - p0);
    const bool leader = h == 0 && chunk == 0;
    const int n4 = N / 4, nf = rows * n4;

    // Round one: the slab is prefetched into L2 by one bulk request (it does not
    // depend on the path), and the path, its length and the tree flag are read.
    const int plim = min(p.maxlen, T);
    const float *slab = p.h0 + (((size_t)b * H + h) * P + p0) * N;
    if (tid == 0) ptx::prefetch_l2(slab, (uint32_t)nf * 16u);
    int pv = 0, okv = 0, lenv = 0;
    float Av = 0.f;
    if (tid < plim) pv = p.path[(size_t)b * p.maxlen + tid];
    if (tid == 0) {
        okv = p.tree.ok[b];
        lenv = p.path_len[b];
        Av = p.A[h];
    }
    if (tid < plim) pn[tid] = pv;
    if (tid == 0) {
        s_ok = okv;
        s_len = lenv;
        s_A = Av;
        s_badq = INT_MAX;
    }
    __syncthreads();
    const int len = s_len;
    if (!s_ok) return;                             // invalid tree: h_new untouched
    if (len < 0 || len > p.maxlen || len > T) {
        if (leader && tid == 0) latch_error(p.err, STREE_ERR_BAD_PATH, b, -1, len);
        return;
    }

    // Round two, all at once: the checks of every path position (depth, the
    // leaf's ancestor bit), dt at the path's nodes, and the first chunk's B rows
    // and x values (node ids clamped into range; an invalid path discards them).
    const int leaf = len > 0 ? pn[len - 1] : 0;
    const bool leaf_ok = leaf >= 0 && leaf < T;
    int bad = 0;
    for (int q = tid; q < len; q += kCThreads) {
        const int j = pn[q];
        const bool in = leaf_ok && j >= 0 && j < T;
        const bool good = in && ((p.tree.anc[((size_t)b * T + leaf) * W + (j >> 5)] >> (j & 31)) & 1u) &&
                          p.tree.depth[(size_t)b * T + j] == q;
        if (!good) {
            bad = 1;
            atomicMin(&s_badq, q);
        }
        dq[q] = in ? load_as_float(p.dt, ((size_t)b * T + j) * H + h, p.dtype) : 0.f;
    }
    stage_path_rows(p, Bq, cfq, pn, 0, min(kQChunk, len), b, h, g, p0, rows);
    // The slab into registers (from L2 by now), issued after the small loads so
    // that they are not queued behind it.
    const float4 *src = reinterpret_cast<const float4 *>(slab);
    float4 hv[kCVec];
#pragma unroll
    for (int k = 0; k < kCVec; ++k) {
        const int f = tid + k * kCThreads;
        hv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (f < nf)
            asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(hv[k].x), "=f"(hv[k].y), "=f"(hv[k].z), "=f"(hv[k].w)
                         : "l"(src + f)
                         : "memory");
    }
    if (__syncthreads_or(bad)) {
        if (leader && tid == 0) latch_error(p.err, STREE_ERR_BAD_PATH, b, s_badq, pn[s_badq]);
        return;
    }
    const float Ah = s_A;
    if (tid == 0) {
        // L along the path (a prefix sum), then the replay weights.
        float s = 0.f;
        for (int q = 0; q < len; ++q) {
            s += dq[q];
            wq[q] = Ah * s;
        }
    }
    __syncthreads();
    const float Lleaf = len > 0 ? wq[len - 1] : 0.f;
    __syncthreads();
    for (int q = tid; q < len; q += kCThreads) wq[q] = expf(Lleaf - wq[q]) * dq[q];
    const float al = len > 0 ? expf(Lleaf) : 1.f;

    float4 acc[kCVec];
#pragma unroll
    for (int k = 0; k < kCVec; ++k) acc[k] = make_float4(al * hv[k].x, al * hv[k].y, al * hv[k].z, al * hv[k].w);
    for (int q0 = 0; q0 < len; q0 += kQChunk) {
        const int nq = min(kQChunk, len - q0);
        if (q0 > 0) {
            __syncthreads();
            stage_path_rows(p, Bq, cfq, pn, q0, nq, b, h, g, p0, rows);
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kCVec; ++k) {
            const int f = tid + k * kCThreads;
            if (f < nf) {
                const int r = f / n4, c = f - r * n4;
                for (int qq = 0; qq < nq; ++qq) {
                    const float cf = wq[q0 + qq] * cfq[qq * rows + r];
                    const float4 bv = *reinterpret_cast<const float4 *>(Bq + qq * N + 4 * c);
                    acc[k].x = fmaf(cf, bv.x, acc[k].x);
                    acc[k].y = fmaf(cf, bv.y, acc[k].y);
                    acc[k].z = fmaf(cf, bv.z, acc[k].z);
                    acc[k].w = fmaf(cf, bv.w, acc[k].w);
                }
            }
        }
    }
    float4 *dst = reinterpret_cast<float4 *>(p.h_new + (((size_t)b * H + h) * P + p0) * N);
#pragma unroll
    for (int k = 0; k < kCVec; ++k) {
        const int f = tid + k * kCThreads;
        if (f < nf) __stcs(dst + f, acc[k]);
    }
}

}  // namespace

bool commit_supported(const ScanArgs &a)
{
    if (a.N % 4 != 0 || a.N > kMaxDim || a.P > kMaxDim || a.T > kMaxNodes) return false;
    const int R = kSlabFloats / a.N;
    return R >= 1;
}

cudaError_t launch_commit(const ScanArgs &a, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    if (!commit_supported(a)) return cudaErrorNotSupported;
    CommitParams p{};
    p.x = a.x; p.dt = a.dt; p.B = a.B; p.A = a.A; p.h0 = a.h0;
    p.tree = a.tree;
    p.path = a.path; p.path_len = a.path_len; p.maxlen = a.maxlen;
    p.h_new = a.h_new;
    p.err = a.err;
    p.T = a.T; p.H = a.H; p.P = a.P; p.N = a.N; p.G = a.G;
    p.dtype = a.dtype;
    p.R = kSlabFloats / a.N;
    if (p.R > a.P) p.R = a.P;
    p.chunks = (a.P + p.R - 1) / p.R;
    const long long grid = (long long)a.batch * a.H * p.chunks;
    if (grid > 0x7fffffffLL) return cudaErrorNotSupported;
    commit_kernel<<<(unsigned)grid, kCThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace stree
