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
// R x dstate contiguous fp32 (32 KB), eight 16-byte loads per thread issued at
// entry, before the path is known, so the state is in flight during the two
// dependent rounds of small loads (path; then dt, x and B at the path nodes).
// The path's B rows and the per-row coefficients w_q x_q are staged in shared
// memory sixteen path positions at a time.  Several CTAs per SM overlap one
// another's round trips.
#include <climits>

#include "stree_internal.cuh"

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

__global__ void __launch_bounds__(kCThreads) commit_kernel(const CommitParams p)
{
    __shared__ __align__(16) float Bq[kQChunk * kMaxDim];   // staged path rows of B
    __shared__ float cfq[kQChunk * kMaxDim];                // w_q x_q per slab row
    __shared__ int32_t pn[kMaxNodes];
    __shared__ float dq[kMaxNodes], wq[kMaxNodes];
    __shared__ int32_t s_badq;

    const int tid = threadIdx.x;
    const int T = p.T, H = p.H, P = p.P, N = p.N, G = p.G, W = p.tree.W;
    const int chunk = blockIdx.x % p.chunks;
    const int h = (blockIdx.x / p.chunks) % H;
    const int b = blockIdx.x / (p.chunks * H);
    const int g = h / (H / G);
    const int p0 = chunk * p.R, rows = min(p.R, P - p0);
    const bool leader = h == 0 && chunk == 0;
    const int n4 = N / 4, nf = rows * n4;

    // The state slab first: it does not depend on the path.
    const float4 *src = reinterpret_cast<const float4 *>(p.h0 + (((size_t)b * H + h) * P + p0) * N);
    float4 hv[kCVec];
#pragma unroll
    for (int k = 0; k < kCVec; ++k) {
        const int f = tid + k * kCThreads;
        hv[k] = f < nf ? __ldcs(src + f) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (!p.tree.ok[b]) return;                     // invalid tree: h_new untouched
    const int len = p.path_len[b];
    if (len < 0 || len > p.maxlen || len > T) {
        if (leader && tid == 0) latch_error(p.err, STREE_ERR_BAD_PATH, b, -1, len);
        return;
    }
    if (tid < len) pn[tid] = p.path[(size_t)b * p.maxlen + tid];
    if (tid == 0) s_badq = INT_MAX;
    __syncthreads();

    // Position q must hold the depth-q ancestor of the last node.
    int bad = 0;
    for (int q = tid; q < len; q += kCThreads) {
        const int leaf = pn[len - 1], j = pn[q];
        const bool good = leaf >= 0 && leaf < T && j >= 0 && j < T &&
                          ((p.tree.anc[((size_t)b * T + leaf) * W + (j >> 5)] >> (j & 31)) & 1u) &&
                          p.tree.depth[(size_t)b * T + j] == q;
        if (!good) {
            bad = 1;
            atomicMin(&s_badq, q);
        }
        dq[q] = good ? load_as_float(p.dt, ((size_t)b * T + j) * H + h, p.dtype) : 0.f;
    }
    if (__syncthreads_or(bad)) {
        if (leader && tid == 0) latch_error(p.err, STREE_ERR_BAD_PATH, b, s_badq, pn[s_badq]);
        return;
    }
    const float Ah = __ldg(p.A + h);
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
    const size_t xrow = (size_t)H * P;
    for (int q0 = 0; q0 < len; q0 += kQChunk) {
        const int nq = min(kQChunk, len - q0);
        __syncthreads();
        for (int e = tid; e < nq * N; e += kCThreads) {
            const int qq = e / N, n = e - qq * N;
            Bq[qq * N + n] = load_as_float(p.B, (((size_t)b * T + pn[q0 + qq]) * G + g) * N + n, p.dtype);
        }
        for (int e = tid; e < nq * rows; e += kCThreads) {
            const int qq = e / rows, r = e - qq * rows;
            const size_t xi = ((size_t)b * T + pn[q0 + qq]) * xrow + (size_t)h * P + p0 + r;
            cfq[qq * rows + r] = wq[q0 + qq] * load_as_float(p.x, xi, p.dtype);
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kCVec; ++k) {
            const int f = tid + k * kCThreads;
            if (f < nf) {
                const int r = f / n4, c = f - r * n4;
                for (int qq = 0; qq < nq; ++qq) {
                    const float cf = cfq[qq * rows + r];
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
