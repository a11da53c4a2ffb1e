// k_scan_simt.cu -- CUDA-core (fp32 FMA) packed tree scan with optional commit.
//
// The packed form of the per-path recurrence ("STree: Speculative Tree Decoding
// for Hybrid State Space Models", scime.ai summary, "Approach": the accumulated
// transition A_tree = L . log A over the tree mask, and activation replay):
//   L_i   = A_h * sum_{j in anc(i)} dt_j
//   y_i   = exp(L_i) (h0 . C_i) + sum_{j in anc(i)} exp(L_i - L_j) cb_ij dt_j x_j + D_h x_i
//   h_new = exp(L_leaf) h0 + sum_{j on path} exp(L_leaf - L_j) dt_j x_j (outer) B_j
// with cb_ij = C_i . B_j from cb_pairs_kernel.  Only ancestor pairs are
// exponentiated, so exp never sees a positive argument.
//
// This kernel covers every supported shape and both dtypes in exact fp32
// arithmetic; it is the path for fp32 inputs.  One CTA per (sequence, head,
// 32-row slice of headdim); lane = row of the slice.  The h0 slice is read once
// into shared memory and serves both the root term and the commit.
#include "stree_internal.cuh"

namespace stree {
namespace {

constexpr int PT = 32;        // headdim rows per CTA (one per lane)
constexpr int kThreads = 128;

__device__ __forceinline__ bool bit_set(const uint32_t *row, int j)
{
    return (row[j >> 5] >> (j & 31)) & 1u;
}

__global__ void __launch_bounds__(kThreads) scan_simt_kernel(ScanArgs a)
{
    const int b = blockIdx.x, h = blockIdx.y, pt = blockIdx.z;
    if (!a.tree.ok[b]) return;                       // invalid tree: outputs untouched

    const int T = a.T, H = a.H, P = a.P, N = a.N, G = a.G, W = a.tree.W;
    const int g = h / (H / G);
    const int p0 = pt * PT;
    const int np = min(PT, P - p0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const stree_dtype dty = a.dtype;

    extern __shared__ float smem[];
    const int NS = N + 1;                            // padded row: lanes hit distinct banks
    float *h0s = smem;                               // [PT][N+1]
    float *xs = h0s + PT * NS;                       // [T][PT]
    float *Ls = xs + T * PT;                         // [T]
    float *dts = Ls + T;                             // [T]
    uint32_t *ancs = reinterpret_cast<uint32_t *>(dts + T);   // [T][W]
    __shared__ int pnode[kMaxNodes];
    __shared__ float pw[kMaxNodes];
    __shared__ int s_len, s_state;

    const float Ah = a.A[h], Dh = a.D[h];
    for (int k = tid; k < T * W; k += kThreads) ancs[k] = a.tree.anc[(size_t)b * T * W + k];
    for (int i = tid; i < T; i += kThreads) dts[i] = load_as_float(a.dt, ((size_t)b * T + i) * H + h, dty);
    for (int k = tid; k < T * PT; k += kThreads) {
        int i = k / PT, p = k % PT;
        xs[k] = (p < np) ? load_as_float(a.x, (((size_t)b * T + i) * H + h) * P + p0 + p, dty) : 0.f;
    }
    const float *h0_bh = a.h0 + ((size_t)b * H + h) * P * N;
    for (int k = tid; k < PT * N; k += kThreads) {
        int p = k / N, n = k % N;
        h0s[p * NS + n] = (p < np) ? h0_bh[(size_t)(p0 + p) * N + n] : 0.f;
    }
    __syncthreads();

    // Tree cumsum: L_i over the ancestor-or-self set of i.
    for (int i = tid; i < T; i += kThreads) {
        float s = 0.f;
        for (int w = 0; w < W; ++w) {
            uint32_t bits = ancs[i * W + w];
            while (bits) {
                int j = (w << 5) + __ffs(bits) - 1;
                bits &= bits - 1;
                s += dts[j];
            }
        }
        Ls[i] = Ah * s;
    }
    __syncthreads();

    if (a.y != nullptr) {
        const float *cb = a.cb + ((size_t)b * G + g) * T * T;
        for (int i = warp; i < T; i += kThreads / 32) {
            const size_t ci = (((size_t)b * T + i) * G + g) * N;
            float root = 0.f;
            for (int n = 0; n < N; ++n)
                root = fmaf(h0s[lane * NS + n], load_as_float(a.C, ci + n, dty), root);
            const float Li = Ls[i];
            float tree = 0.f;
            for (int w = 0; w < W; ++w) {
                uint32_t bits = ancs[i * W + w];
                while (bits) {
                    int j = (w << 5) + __ffs(bits) - 1;
                    bits &= bits - 1;
                    float m = expf(Li - Ls[j]) * cb[(size_t)i * T + j] * dts[j];
                    tree = fmaf(m, xs[j * PT + lane], tree);
                }
            }
            float yv = expf(Li) * root + tree + Dh * xs[i * PT + lane];
            if (lane < np) store_from_float(a.y, (((size_t)b * T + i) * H + h) * P + p0 + lane, yv, dty);
        }
    }

    if (a.path != nullptr) {
        if (tid == 0) {
            // Same validity rule as the resolver: path[k] is the depth-k ancestor of its last node.
            int len = a.path_len[b];
            int state = 1;
            if (len < 0 || len > a.maxlen || len > T) {
                state = 0;
                if (h == 0 && pt == 0) latch_error(a.err, STREE_ERR_BAD_PATH, b, -1, len);
            } else if (len > 0) {
                const int32_t *pb = a.path + (size_t)b * a.maxlen;
                int leaf = pb[len - 1];
                if (leaf < 0 || leaf >= T || a.tree.depth[(size_t)b * T + leaf] != len - 1) {
                    state = 0;
                    if (h == 0 && pt == 0) latch_error(a.err, STREE_ERR_BAD_PATH, b, len - 1, leaf);
                } else {
                    for (int k = 0; k < len; ++k) {
                        int j = pb[k];
                        bool good = j >= 0 && j < T && bit_set(ancs + leaf * W, j) &&
                                    a.tree.depth[(size_t)b * T + j] == k;
                        if (!good) {
                            state = 0;
                            if (h == 0 && pt == 0) latch_error(a.err, STREE_ERR_BAD_PATH, b, k, j);
                            break;
                        }
                        pnode[k] = j;
                    }
                }
            }
            s_len = len;
            s_state = state;
        }
        __syncthreads();
        const int len = s_len;
        if (s_state) {
            const float Lleaf = len > 0 ? Ls[pnode[len - 1]] : 0.f;
            for (int k = tid; k < len; k += kThreads) {
                int j = pnode[k];
                pw[k] = expf(Lleaf - Ls[j]) * dts[j];
            }
            __syncthreads();
            const float alpha = expf(Lleaf);
            float *hn = a.h_new + ((size_t)b * H + h) * P * N;
            for (int e = tid; e < np * N; e += kThreads) {
                int p = e / N, n = e % N;
                float v = alpha * h0s[p * NS + n];
                for (int k = 0; k < len; ++k) {
                    int j = pnode[k];
                    v = fmaf(pw[k] * xs[j * PT + p], load_as_float(a.B, (((size_t)b * T + j) * G + g) * N + n, dty), v);
                }
                hn[(size_t)(p0 + p) * N + n] = v;
            }
        }
    }
}

size_t simt_smem_bytes(int T, int N, int W)
{
    return sizeof(float) * ((size_t)PT * (N + 1) + (size_t)T * PT + 2 * (size_t)T) + sizeof(uint32_t) * (size_t)T * W;
}

}  // namespace

cudaError_t launch_scan_simt(const ScanArgs &a, cudaStream_t s)
{
    if (a.batch == 0) return cudaSuccess;
    size_t smem = simt_smem_bytes(a.T, a.N, a.tree.W);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(scan_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(a.batch, a.H, (a.P + PT - 1) / PT);
    scan_simt_kernel<<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace stree
