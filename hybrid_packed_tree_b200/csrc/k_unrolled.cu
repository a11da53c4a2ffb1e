// k_unrolled.cu -- the unrolled-tree baseline: every root-to-leaf path of the
// draft tree scanned as its own sequence, each with its own copy of the state.
//
// This is the alternative the packed tree is measured against ("STree:
// Speculative Tree Decoding for Hybrid State Space Models", scime.ai summary,
// "Problem": verifying a tree on an SSM by unrolling it into separate sequences
// costs extra states and memory; "Key results": the packed tree against the
// unrolled one on Mamba2-2.7B).  Per path and head the plain recurrence runs node
// by node from h0:
//   s <- exp(dt_k A_h) s + dt_k x_k (outer) B_k,   y_k = s . C_k + D_h x_k
// and the final state of every path is written out (the per-path state copies).
// Nodes shared by several paths are recomputed once per path, which is the
// redundancy the packed scan removes.
//
// One CTA per (sequence x path, head, 64-row slice of headdim); 256 threads, four
// per state row, each owning every fourth 4-column chunk of the row (so the four
// threads of a row move 64 contiguous bytes of the state and read adjacent words
// of B and C).  The state slice lives in registers; B, C, dt and x of up to 16
// path nodes at a time are staged in shared memory.
#include "stree_internal.cuh"

namespace stree {
namespace {

constexpr int kRows = 64;                       // headdim rows per CTA
constexpr int kParts = 4;                       // threads per row
constexpr int kThreads = kRows * kParts;
constexpr int kMaxChunks = kMaxDim / 16;        // 4-column chunks per thread (<= 16)
constexpr int kSeg = 16;                        // path nodes staged at a time

struct UnrolledArgs {
    const void *x, *dt, *B, *C;
    const float *A, *D, *h0;
    const int32_t *paths, *path_len;
    int T, batch, n_paths, max_depth, H, P, N, G;
    stree_dtype dtype;
    void *y;             // [batch, n_paths, max_depth, H, P]
    float *h_paths;      // [batch, n_paths, H, P, N]
    int32_t *err;        // error word, or NULL
};

__global__ void __launch_bounds__(kThreads) unrolled_scan_kernel(UnrolledArgs a)
{
    extern __shared__ float4 sh4[];
    const int bp = blockIdx.x, h = blockIdx.y, p0 = blockIdx.z * kRows;
    const int b = bp / a.n_paths;
    const int g = h / (a.H / a.G);
    const int tid = threadIdx.x, r = tid / kParts, part = tid % kParts;
    const int T = a.T, H = a.H, P = a.P, N = a.N, G = a.G;
    const int nch = N / 16;                      // chunks per thread (N is a multiple of 16 here)
    const bool row_ok = p0 + r < P;
    const int32_t *path = a.paths + (size_t)bp * a.max_depth;
    float4 *Bs = sh4;                            // [kSeg][N/4]
    float4 *Cs = sh4 + kSeg * (N / 4);           // [kSeg][N/4]
    float *dts = reinterpret_cast<float *>(sh4 + 2 * kSeg * (N / 4));   // [kSeg]
    float *xs = dts + kSeg;                                             // [kSeg][kRows]

    // The path must have 0 <= len <= max_depth and node ids in [0, T).
    const int len = a.path_len[bp];
    int bad = len < 0 || len > a.max_depth;
    if (!bad)
        for (int k = tid; k < len; k += kThreads) {
            const int node = path[k];
            bad |= node < 0 || node >= T;
        }
    bad = __syncthreads_or(bad);
    if (bad) {
        if (a.err && tid == 0 && blockIdx.y == 0 && blockIdx.z == 0)
            latch_error(a.err, STREE_ERR_BAD_PATH, b, bp % a.n_paths, len);
        return;
    }

    const float Ah = a.A[h], Dh = a.D[h];
    const float4 *hrow = reinterpret_cast<const float4 *>(a.h0 + (((size_t)b * H + h) * P + p0 + r) * N);
    float4 s[kMaxChunks];
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c)
        s[c] = (c < nch && row_ok) ? hrow[c * kParts + part] : make_float4(0.f, 0.f, 0.f, 0.f);

    for (int k0 = 0; k0 < len; k0 += kSeg) {
        const int nseg = min(kSeg, len - k0);
        __syncthreads();                         // the previous segment is consumed
        for (int idx = tid; idx < nseg * (N / 4); idx += kThreads) {
            const int k = idx / (N / 4), q = idx - k * (N / 4);
            const size_t base = (((size_t)b * T + path[k0 + k]) * G + g) * N + 4 * q;
            Bs[idx] = make_float4(load_as_float(a.B, base, a.dtype), load_as_float(a.B, base + 1, a.dtype),
                                  load_as_float(a.B, base + 2, a.dtype), load_as_float(a.B, base + 3, a.dtype));
            Cs[idx] = make_float4(load_as_float(a.C, base, a.dtype), load_as_float(a.C, base + 1, a.dtype),
                                  load_as_float(a.C, base + 2, a.dtype), load_as_float(a.C, base + 3, a.dtype));
        }
        for (int idx = tid; idx < nseg * kRows; idx += kThreads) {
            const int k = idx / kRows, rr = idx - k * kRows;
            const size_t tn = (size_t)b * T + path[k0 + k];
            xs[idx] = p0 + rr < P ? load_as_float(a.x, (tn * H + h) * P + p0 + rr, a.dtype) : 0.f;
            if (rr == 0) dts[k] = load_as_float(a.dt, tn * H + h, a.dtype);
        }
        __syncthreads();
        for (int k = 0; k < nseg; ++k) {
            const float decay = expf(dts[k] * Ah);
            const float xv = xs[k * kRows + r];
            const float coef = dts[k] * xv;
            const float4 *Bk = Bs + k * (N / 4), *Ck = Cs + k * (N / 4);
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < kMaxChunks; ++c) {
                if (c < nch) {
                    const float4 bv = Bk[c * kParts + part], cv = Ck[c * kParts + part];
                    s[c].x = fmaf(decay, s[c].x, coef * bv.x);
                    s[c].y = fmaf(decay, s[c].y, coef * bv.y);
                    s[c].z = fmaf(decay, s[c].z, coef * bv.z);
                    s[c].w = fmaf(decay, s[c].w, coef * bv.w);
                    acc = fmaf(s[c].x, cv.x, acc);
                    acc = fmaf(s[c].y, cv.y, acc);
                    acc = fmaf(s[c].z, cv.z, acc);
                    acc = fmaf(s[c].w, cv.w, acc);
                }
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (part == 0 && row_ok)
                store_from_float(a.y, ((((size_t)bp * a.max_depth + k0 + k) * H + h) * P) + p0 + r,
                                 fmaf(Dh, xv, acc), a.dtype);
        }
    }
    if (row_ok) {
        float4 *out = reinterpret_cast<float4 *>(a.h_paths + (((size_t)bp * H + h) * P + p0 + r) * N);
#pragma unroll
        for (int c = 0; c < kMaxChunks; ++c)
            if (c < nch) out[c * kParts + part] = s[c];
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace stree

using namespace stree;

extern "C" stree_status stree_unrolled_scan(const void *x, const void *dt, const float *A, const void *B,
                                            const void *C, const float *D, const float *h0, const int32_t *paths,
                                            const int32_t *path_len, int n_nodes, int batch, int n_paths,
                                            int max_depth, int nheads, int headdim, int dstate, int ngroups,
                                            stree_dtype dtype, void *y_paths, float *h_paths, int32_t *err_out,
                                            void *stream)
{
    if (batch < 0 || n_nodes < 1 || n_paths < 1 || max_depth < 1 || nheads < 1 || headdim < 1 || dstate < 1 ||
        ngroups < 1)
        return STREE_ERR_UNSUPPORTED;
    if (n_nodes > kMaxNodes || max_depth > kMaxNodes || headdim > kMaxDim || dstate > kMaxDim) return STREE_ERR_UNSUPPORTED;
    if (headdim % 8 != 0 || dstate % 16 != 0 || nheads % ngroups != 0 || nheads > 65535) return STREE_ERR_UNSUPPORTED;
    if ((long long)batch * n_paths > 0x7fffffffLL) return STREE_ERR_UNSUPPORTED;
    if (dtype != STREE_F32 && dtype != STREE_BF16) return STREE_ERR_UNSUPPORTED;
    if (batch == 0) return STREE_OK;
    if (!x || !dt || !A || !B || !C || !D || !h0 || !paths || !path_len || !y_paths || !h_paths)
        return STREE_ERR_INVALID_ARG;
    const void *ptrs[] = {x, dt, A, B, C, D, h0, y_paths, h_paths};
    for (const void *p : ptrs)
        if (!aligned16(p)) return STREE_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(paths) & 3u) || (reinterpret_cast<uintptr_t>(path_len) & 3u) ||
        (reinterpret_cast<uintptr_t>(err_out) & 3u))
        return STREE_ERR_MISALIGNED;

    UnrolledArgs a{};
    a.x = x; a.dt = dt; a.B = B; a.C = C; a.A = A; a.D = D; a.h0 = h0;
    a.paths = paths; a.path_len = path_len;
    a.T = n_nodes; a.batch = batch; a.n_paths = n_paths; a.max_depth = max_depth;
    a.H = nheads; a.P = headdim; a.N = dstate; a.G = ngroups;
    a.dtype = dtype;
    a.y = y_paths;
    a.h_paths = h_paths;
    // Without an error word, device-detected errors are dropped (nothing is allocated).
    a.err = err_out;
    if (err_out && cudaMemsetAsync(err_out, 0, 4 * sizeof(int32_t), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return STREE_ERR_CUDA;
    const dim3 grid((unsigned)(batch * n_paths), (unsigned)nheads, (unsigned)((headdim + kRows - 1) / kRows));
    const size_t smem = (size_t)2 * kSeg * dstate * sizeof(float) + (size_t)kSeg * (1 + kRows) * sizeof(float);
    unrolled_scan_kernel<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? STREE_OK : STREE_ERR_CUDA;
}
