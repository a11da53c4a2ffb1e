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
// element) and adds at most a path's worth of rank-1 terms, so it is HBM-bound;
// what must not happen is a chain of small dependent reads in front of every
// slab.  Two launches:
//   * commit_prep_kernel (one CTA per sequence): checks the path against the
//     tree, and writes the path's nodes, its length (-1 when invalid) and for
//     every head the weights w_q = exp(L_leaf - L_q) dt_q and exp(L_leaf) into a
//     small workspace;
//   * commit_stream_kernel (one CTA per (sequence, head, slab of R = 8192 /
//     dstate rows), a programmatic dependent of the first): issues its 32 KB of
//     h0 at entry -- h0 is not written by the prep launch -- then waits for the
//     prep, reads the path and weights (L2), stages the path's B rows and x
//     values in shared memory sixteen positions at a time, and writes h_new.
// The first stream CTAs' state loads run while the prep launch works.
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
    int maxlen, Lc;                          // Lc = min(maxlen, T): path slots in the workspace
    float *h_new;
    int32_t *err;
    CommitWork ws;
    int T, H, P, N, G, R, chunks;
    stree_dtype dtype;
};

// One CTA per sequence: the path's check, nodes and length; per head the weights.
__global__ void __launch_bounds__(kCThreads) commit_prep_kernel(const CommitParams p)
{
    __shared__ int32_t pn[kMaxNodes];
    __shared__ int32_t s_badq, s_len;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int b = blockIdx.x, tid = threadIdx.x;
    const int T = p.T, H = p.H, W = p.tree.W;
    const int plim = min(p.maxlen, T);
    if (tid < plim) pn[tid] = p.path[(size_t)b * p.maxlen + tid];
    if (tid == 0) {
        s_badq = INT_MAX;
        const int len = p.path_len[b];
        const bool ok = p.tree.ok[b] != 0;
        s_len = !ok ? -1 : (len < 0 || len > p.maxlen || len > T) ? -2 : len;
    }
    __syncthreads();
    const int len = s_len;
    if (len == -2) {
        if (tid == 0) {
            latch_error(p.err, STREE_ERR_BAD_PATH, b, -1, p.path_len[b]);
            p.ws.len[b] = -1;
        }
        return;
    }
    if (len < 0) {                                 // invalid tree: h_new untouched
        if (tid == 0) p.ws.len[b] = -1;
        return;
    }
    // Position q must hold the depth-q ancestor of the last node.
    int bad = 0;
    if (tid < len) {
        const int leaf = pn[len - 1], j = pn[tid];
        const bool good = leaf >= 0 && leaf < T && j >= 0 && j < T &&
                          ((p.tree.anc[((size_t)b * T + leaf) * W + (j >> 5)] >> (j & 31)) & 1u) &&
                          p.tree.depth[(size_t)b * T + j] == tid;
        if (!good) {
            bad = 1;
            atomicMin(&s_badq, tid);
        }
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0) {
            latch_error(p.err, STREE_ERR_BAD_PATH, b, s_badq, pn[s_badq]);
            p.ws.len[b] = -1;
        }
        return;
    }
    if (tid < len) p.ws.pn[(size_t)b * p.Lc + tid] = pn[tid];
    if (tid == 0) p.ws.len[b] = len;
    // Per head: L along the path (a prefix sum of dt in path order), then the weights.
    for (int h = tid; h < H; h += kCThreads) {
        const float Ah = p.A[h];
        float s = 0.f;
        for (int q = 0; q < len; ++q) s += load_as_float(p.dt, ((size_t)b * T + pn[q]) * H + h, p.dtype);
        const float Lleaf = Ah * s;
        float pre = 0.f;
        float *wh = p.ws.w + ((size_t)b * H + h) * p.Lc;
        for (int q = 0; q < len; ++q) {
            const float d = load_as_float(p.dt, ((size_t)b * T + pn[q]) * H + h, p.dtype);
            pre += d;
            wh[q] = expf(Lleaf - Ah * pre) * d;
        }
        p.ws.alpha[(size_t)b * H + h] = len > 0 ? expf(Lleaf) : 1.f;
    }
}

// Stages B rows and x values (of the slab's rows) of path positions q0 .. q0 + nq - 1.
__device__ __forceinline__ void stage_path_rows(const CommitParams &p, float *Bq, float *cfq, const int32_t *pn,
                                                int q0, int nq, int b, int h, int g, int p0, int rows)
{
    const int T = p.T, N = p.N;
    const size_t xrow = (size_t)p.H * p.P;
    for (int e = threadIdx.x; e < nq * N; e += kCThreads) {
        const int qq = e / N, n = e - qq * N;
        Bq[qq * N + n] = load_as_float(p.B, (((size_t)b * T + pn[q0 + qq]) * p.G + g) * N + n, p.dtype);
    }
    for (int e = threadIdx.x; e < nq * rows; e += kCThreads) {
        const int qq = e / rows, r = e - qq * rows;
        cfq[qq * rows + r] = load_as_float(p.x, ((size_t)b * T + pn[q0 + qq]) * xrow + (size_t)h * p.P + p0 + r, p.dtype);
    }
}

__global__ void __launch_bounds__(kCThreads, 4) commit_stream_kernel(const CommitParams p)
{
    __shared__ __align__(16) float Bq[kQChunk * kMaxDim];   // staged path rows of B
    __shared__ float cfq[kQChunk * kMaxDim];                // x_q per slab row
    __shared__ int32_t pn[kMaxNodes];
    __shared__ float wq[kMaxNodes];
    __shared__ int32_t s_len;
    __shared__ float s_alpha;

    const int tid = threadIdx.x;
    const int H = p.H, P = p.P, N = p.N, G = p.G;
    const int chunk = blockIdx.x % p.chunks;
    const int h = (blockIdx.x / p.chunks) % H;
    const int b = blockIdx.x / (p.chunks * H);
    const int g = h / (H / G);
    const int p0 = chunk * p.R, rows = min(p.R, P - p0);
    const int n4 = N / 4, nf = rows * n4;

    // The slab first: h0 is an input of the scan, complete before the prep launch.
    const float4 *src = reinterpret_cast<const float4 *>(p.h0 + (((size_t)b * H + h) * P + p0) * N);
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
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) {
        s_len = p.ws.len[b];
        s_alpha = p.ws.alpha[(size_t)b * H + h];
    }
    if (tid < p.Lc) {
        pn[tid] = p.ws.pn[(size_t)b * p.Lc + tid];
        wq[tid] = p.ws.w[((size_t)b * H + h) * p.Lc + tid];
    }
    __syncthreads();
    const int len = s_len;
    if (len < 0) return;                             // invalid tree or path: h_new untouched
    const float al = s_alpha;
    float4 acc[kCVec];
#pragma unroll
    for (int k = 0; k < kCVec; ++k) acc[k] = make_float4(al * hv[k].x, al * hv[k].y, al * hv[k].z, al * hv[k].w);
    for (int q0 = 0; q0 < len; q0 += kQChunk) {
        const int nq = min(kQChunk, len - q0);
        if (q0 > 0) __syncthreads();
        stage_path_rows(p, Bq, cfq, pn, q0, nq, b, h, g, p0, rows);
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

// The same stream for dstate 128 (slabs of 64 rows): thread t owns the four state
// columns 4 (t % 32) .. +3 of rows t / 32 + 8k, k = 0..7, so each path position
// costs one shared-memory read of its B columns for all eight rows; the staged x
// values already carry the position's weight, and the updates go two lanes per
// fp32x2 FMA.
__global__ void __launch_bounds__(kCThreads, 4) commit_stream128_kernel(const CommitParams p)
{
    constexpr int N = 128, R = 64, kRowsPerThread = R * N / 4 / kCThreads;   // 8
    __shared__ __align__(16) float Bq[kQChunk * N];          // staged path rows of B
    __shared__ float cfq[kQChunk * R];                       // w_q x_q[row]
    __shared__ int32_t pn[kMaxNodes];
    __shared__ float wq[kMaxNodes];
    __shared__ int32_t s_len;
    __shared__ float s_alpha;

    const int tid = threadIdx.x;
    const int H = p.H, P = p.P, G = p.G, T = p.T;
    const int chunk = blockIdx.x % p.chunks;
    const int h = (blockIdx.x / p.chunks) % H;
    const int b = blockIdx.x / (p.chunks * H);
    const int g = h / (H / G);
    const int p0 = chunk * R, rows = min(R, P - p0);
    const int c4 = tid & 31, r0 = tid >> 5;

    const float4 *src = reinterpret_cast<const float4 *>(p.h0 + (((size_t)b * H + h) * P + p0) * N);
    float4 hv[kRowsPerThread];
#pragma unroll
    for (int k = 0; k < kRowsPerThread; ++k) {
        hv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r0 + 8 * k < rows)
            asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(hv[k].x), "=f"(hv[k].y), "=f"(hv[k].z), "=f"(hv[k].w)
                         : "l"(src + tid + k * kCThreads)
                         : "memory");
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) {
        s_len = p.ws.len[b];
        s_alpha = p.ws.alpha[(size_t)b * H + h];
    }
    if (tid < p.Lc) {
        pn[tid] = p.ws.pn[(size_t)b * p.Lc + tid];
        wq[tid] = p.ws.w[((size_t)b * H + h) * p.Lc + tid];
    }
    __syncthreads();
    const int len = s_len;
    if (len < 0) return;                             // invalid tree or path: h_new untouched
    const float al = s_alpha;
    float2 acc[kRowsPerThread][2];
#pragma unroll
    for (int k = 0; k < kRowsPerThread; ++k) {
        acc[k][0] = make_float2(al * hv[k].x, al * hv[k].y);
        acc[k][1] = make_float2(al * hv[k].z, al * hv[k].w);
    }
    const size_t xrow = (size_t)H * P;
    for (int q0 = 0; q0 < len; q0 += kQChunk) {
        const int nq = min(kQChunk, len - q0);
        if (q0 > 0) __syncthreads();
        for (int e = tid; e < nq * N; e += kCThreads) {
            const int qq = e >> 7;
            Bq[e] = load_as_float(p.B, (((size_t)b * T + pn[q0 + qq]) * G + g) * N + (e & (N - 1)), p.dtype);
        }
        for (int e = tid; e < nq * R; e += kCThreads) {
            const int qq = e >> 6, r = e & (R - 1);
            cfq[e] = r < rows ? wq[q0 + qq] * load_as_float(p.x, ((size_t)b * T + pn[q0 + qq]) * xrow +
                                                                       (size_t)h * P + p0 + r, p.dtype)
                              : 0.f;
        }
        __syncthreads();
        for (int qq = 0; qq < nq; ++qq) {
            const float4 bv = *reinterpret_cast<const float4 *>(Bq + qq * N + 4 * c4);
            const float2 b01 = make_float2(bv.x, bv.y), b23 = make_float2(bv.z, bv.w);
#pragma unroll
            for (int k = 0; k < kRowsPerThread; ++k) {
                const float cf = cfq[qq * R + r0 + 8 * k];
                const float2 cc = make_float2(cf, cf);
                acc[k][0] = ptx::ffma2(cc, b01, acc[k][0]);
                acc[k][1] = ptx::ffma2(cc, b23, acc[k][1]);
            }
        }
    }
    float4 *dst = reinterpret_cast<float4 *>(p.h_new + (((size_t)b * H + h) * P + p0) * N);
#pragma unroll
    for (int k = 0; k < kRowsPerThread; ++k)
        if (r0 + 8 * k < rows)
            __stcs(dst + tid + k * kCThreads, make_float4(acc[k][0].x, acc[k][0].y, acc[k][1].x, acc[k][1].y));
}

}  // namespace

bool commit_supported(const ScanArgs &a)
{
    if (a.N % 4 != 0 || a.N > kMaxDim || a.P > kMaxDim || a.T > kMaxNodes) return false;
    return kSlabFloats / a.N >= 1;
}

size_t commit_work_floats(const ScanArgs &a)
{
    const size_t Lc = (size_t)(a.maxlen < a.T ? a.maxlen : a.T);
    return (size_t)a.batch * a.H * (Lc + 1);
}

size_t commit_work_ints(const ScanArgs &a)
{
    const size_t Lc = (size_t)(a.maxlen < a.T ? a.maxlen : a.T);
    return (size_t)a.batch * (Lc + 1);
}

cudaError_t launch_commit(const ScanArgs &a, const CommitWork &ws, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    if (!commit_supported(a)) return cudaErrorNotSupported;
    CommitParams p{};
    p.x = a.x; p.dt = a.dt; p.B = a.B; p.A = a.A; p.h0 = a.h0;
    p.tree = a.tree;
    p.path = a.path; p.path_len = a.path_len; p.maxlen = a.maxlen;
    p.Lc = a.maxlen < a.T ? a.maxlen : a.T;
    p.h_new = a.h_new;
    p.err = a.err;
    p.ws = ws;
    p.T = a.T; p.H = a.H; p.P = a.P; p.N = a.N; p.G = a.G;
    p.dtype = a.dtype;
    p.R = kSlabFloats / a.N;
    if (p.R > a.P) p.R = a.P;
    p.chunks = (a.P + p.R - 1) / p.R;
    const long long grid = (long long)a.batch * a.H * p.chunks;
    if (grid > 0x7fffffffLL) return cudaErrorNotSupported;
    commit_prep_kernel<<<a.batch, kCThreads, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kCThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.N == 128 && p.R == 64) return cudaLaunchKernelEx(&cfg, commit_stream128_kernel, p);
    return cudaLaunchKernelEx(&cfg, commit_stream_kernel, p);
}

}  // namespace stree
