// k_scan_small.cu -- packed tree scan + commit for small batches, sm_100a: one CTA
// per (sequence, head, 32 rows of headdim), every global read issued at entry.
//
// Method ("STree: Speculative Tree Decoding for Hybrid State Space Models",
// scime.ai summary, "Approach"), for node i of the packed tree with
// ancestor-or-self set anc(i):
//   L_i   = A_h * sum_{j in anc(i)} dt_j
//   y_i   = exp(L_i) (h0 . C_i) + sum_{j in anc(i)} exp(L_i - L_j) (C_i . B_j) dt_j x_j + D_h x_i
//   h_new = exp(L_leaf) h0 + sum_{j on path} exp(L_leaf - L_j) dt_j x_j (outer) B_j
//
// Design.  At batch 1 a layer's state is a few MB (Mamba2-2.7B: 80 heads x 64 x
// 128 fp32, 2.6 MB), so a launch is bound by its chain of latencies -- launch,
// one DRAM round trip, the dependent on-chip steps, the stores -- not by
// bandwidth.  This kernel keeps that chain short:
//   * grid = batch x heads x headdim/32 CTAs of 256 threads, several per SM;
//   * at entry every thread issues all of its loads: its 4 x 4 fp32 of h0 into
//     registers (warp w owns rows 4w..4w+3, lane l columns 4l..4l+3, so each
//     row is one warp's 512 contiguous bytes), 16-byte asynchronous copies of
//     the sequence's C and B rows and of the CTA's x columns into shared
//     memory, and the scalars (parent, dt, path, A, D);
//   * the tree is rebuilt in shared memory by walking parent[] (one thread per
//     node: ancestor bits, depth, L), and the accepted path is checked against it;
//   * C_i . B_j on ancestor pairs: one warp per node i, lanes over the state;
//   * root term: each lane multiplies its 4 columns of 4 rows with every C_i,
//     then a butterfly reduce-scatter over the warp (62 shuffles per 16 nodes)
//     leaves each lane two (row, node) sums, to which it adds the tree and skip
//     terms; y is staged in shared memory and written with 16-byte stores;
//   * the commit is applied to the h0 registers and stored straight to h_new.
// No tensor cores: the root term is 2T flops per state element (T <= 64), a few
// hundred FMAs per thread, and tcgen05 set-up and round trips would lengthen the
// chain that bounds the launch.  Large batches take the tensor-core kernel.
//
// When the call passes parent[], CTA (b, head 0, slice 0) writes sequence b's
// masks, depths and flag for later calls and reports an invalid tree or path.
#include <climits>
#include <mutex>

#include "stree_internal.cuh"
#include "tc_ptx.cuh"

namespace stree {
namespace {

constexpr int kN = 128;                     // dstate of this kernel
constexpr int kRows = 32;                   // headdim rows per CTA
constexpr int kWarpsS = 8;                  // 4 rows per warp
constexpr int kThreadsS = kWarpsS * 32;
constexpr int kMaxSmallNodes = 64;          // two mask words per node
constexpr int kMaxDevices = 64;

struct SmallParams {
    const void *x, *dt, *B, *C;
    const float *A, *D, *h0;
    const int32_t *parent;                  // non-NULL: tree from parent[]; NULL: `tree`
    TreeView tree;
    uint32_t *anc_out;                      // with parent: the tree written here (may be NULL)
    int32_t *depth_out, *ok_out;
    const int32_t *path, *path_len;
    int maxlen;
    void *y;                                // NULL: no y
    float *h_new;                           // NULL: no commit
    int32_t *err;
    int T, H, P, G, slices;
};

// Shared-memory layout for T nodes and input element size e (bytes).
struct SmallLayout {
    uint32_t c, b, x, y, m, L, eL, dt, par, dep, anc, praw, pnode, wq, misc, total;
    __host__ __device__ SmallLayout(int T, int e)
    {
        uint32_t o = 0;
        auto take = [&](uint32_t bytes) {
            const uint32_t at = o;
            o = (o + bytes + 15u) & ~15u;
            return at;
        };
        c = take((uint32_t)T * kN * e);
        b = take((uint32_t)T * kN * e);
        x = take((uint32_t)T * kRows * e);
        y = take((uint32_t)T * kRows * e);
        m = take((uint32_t)T * T * 4);
        L = take((uint32_t)T * 4);
        eL = take((uint32_t)T * 4);
        dt = take((uint32_t)T * 4);
        par = take((uint32_t)T * 4);
        dep = take((uint32_t)T * 4);
        anc = take((uint32_t)T * 8);
        praw = take((uint32_t)T * 4);
        pnode = take((uint32_t)T * 4);
        wq = take((uint32_t)T * 4);
        misc = take(4 * 4);
        total = o;
    }
};

enum SmallMisc { S_BADI = 0, S_BADQ = 1 };

__device__ __forceinline__ float in_to_f(float v) { return v; }
__device__ __forceinline__ float in_to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename In> __device__ __forceinline__ In f_to_in(float v);
template <> __device__ __forceinline__ float f_to_in<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 f_to_in<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Four consecutive state columns 4 lane .. 4 lane + 3 of row `row` of a [*][128] array.
__device__ __forceinline__ float4 row4(const float *base, int row, int lane)
{
    return *reinterpret_cast<const float4 *>(base + row * kN + 4 * lane);
}
__device__ __forceinline__ float4 row4(const __nv_bfloat16 *base, int row, int lane)
{
    const uint2 raw = *reinterpret_cast<const uint2 *>(base + row * kN + 4 * lane);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}

__device__ __forceinline__ float dot4(float4 a, float4 b)
{
    return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, a.x * b.x)));
}

// Butterfly reduce-scatter of 64 per-lane values over the warp: afterwards
// v[0] and v[1] hold the warp-wide sums of entries 2*lane and 2*lane + 1.
// At the stage with xor distance m the lanes with bit m set keep the upper half
// of their current block and the others the lower half; lane bit m thereby
// selects index weight 2m, which makes the surviving index 2*lane + k.
__device__ __forceinline__ void reduce_scatter64(float (&v)[64], int lane)
{
#pragma unroll
    for (int st = 0; st < 5; ++st) {
        const int m = 16 >> st, half = 32 >> st;
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = up ? v[k] : v[k + half];
            const float keep = up ? v[k + half] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
}

template <typename In>
__global__ void __launch_bounds__(kThreadsS, 2) scan_small_kernel(const SmallParams p)
{
    extern __shared__ __align__(16) uint8_t sm[];
    const int T = p.T, H = p.H, P = p.P, G = p.G;
    const SmallLayout ly(T, (int)sizeof(In));
    In *Cs = reinterpret_cast<In *>(sm + ly.c);          // [T][128] C rows of (b, g)
    In *Bs = reinterpret_cast<In *>(sm + ly.b);          // [T][128] B rows of (b, g)
    In *xs = reinterpret_cast<In *>(sm + ly.x);          // [T][32]  x columns of the CTA
    In *ys = reinterpret_cast<In *>(sm + ly.y);          // [T][32]  y staging
    float *Ms = reinterpret_cast<float *>(sm + ly.m);    // [T][T]   masked decay (ancestor entries)
    float *Ls = reinterpret_cast<float *>(sm + ly.L);
    float *eLs = reinterpret_cast<float *>(sm + ly.eL);
    float *dts = reinterpret_cast<float *>(sm + ly.dt);
    int32_t *par = reinterpret_cast<int32_t *>(sm + ly.par);
    int32_t *dep = reinterpret_cast<int32_t *>(sm + ly.dep);
    uint32_t *ancs = reinterpret_cast<uint32_t *>(sm + ly.anc);   // [T][2]
    int32_t *praw = reinterpret_cast<int32_t *>(sm + ly.praw);
    int32_t *pnode = reinterpret_cast<int32_t *>(sm + ly.pnode);
    float *wq = reinterpret_cast<float *>(sm + ly.wq);
    int32_t *misc = reinterpret_cast<int32_t *>(sm + ly.misc);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = (T + 31) >> 5;
    const int slice = blockIdx.x % p.slices;
    const int h = (blockIdx.x / p.slices) % H;
    const int b = blockIdx.x / (p.slices * H);
    const int g = h / (H / G);
    const int p0 = slice * kRows;
    const bool leader = h == 0 && slice == 0;
    const bool do_y = p.y != nullptr, do_commit = p.h_new != nullptr;

    // The kernel is launched as a programmatic dependent of the preceding grid on
    // the stream: it may start while that grid drains, and waits for its
    // completion before the first global read.  A later launch may likewise start
    // now; it waits for this grid's completion before it reads anything.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---------------------------------------------------------------- 1. loads
    const size_t row0 = ((size_t)b * H + h) * P + p0 + 4 * warp;
    const float *h0r = p.h0 + row0 * kN + 4 * lane;
    float4 hv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) hv[r] = __ldcs(reinterpret_cast<const float4 *>(h0r + r * kN));

    constexpr int kEl16 = 16 / (int)sizeof(In);          // elements per 16-byte chunk
    constexpr int kRowChunks = kN / kEl16;
    constexpr int kXChunks = kRows / kEl16;
    const size_t brow = (size_t)G * kN;
    const In *Cg = static_cast<const In *>(p.C) + ((size_t)b * T * G + g) * kN;
    const In *Bg = static_cast<const In *>(p.B) + ((size_t)b * T * G + g) * kN;
    const In *Xg = static_cast<const In *>(p.x) + ((size_t)b * T * H + h) * P + p0;
    const size_t xrow = (size_t)H * P;
    {
        const uint32_t cs = ptx::smem_u32(Cs), bs = ptx::smem_u32(Bs), xsu = ptx::smem_u32(xs);
        if (do_y)
            for (int q = tid; q < T * kRowChunks; q += kThreadsS)
                ptx::cp_async16(cs + (uint32_t)q * 16u, Cg + (size_t)(q / kRowChunks) * brow + (q % kRowChunks) * kEl16);
        for (int q = tid; q < T * kRowChunks; q += kThreadsS)
            ptx::cp_async16(bs + (uint32_t)q * 16u, Bg + (size_t)(q / kRowChunks) * brow + (q % kRowChunks) * kEl16);
        for (int q = tid; q < T * kXChunks; q += kThreadsS)
            ptx::cp_async16(xsu + (uint32_t)q * 16u, Xg + (size_t)(q / kXChunks) * xrow + (q % kXChunks) * kEl16);
    }
    const In *dtg = static_cast<const In *>(p.dt);
    float dt_v = 0.f;
    int par_v = 0, dep_v = 0, path_v = 0;
    uint32_t anc_v0 = 0u, anc_v1 = 0u;
    if (tid < T) {
        dt_v = in_to_f(dtg[((size_t)b * T + tid) * H + h]);
        if (p.parent) {
            par_v = p.parent[(size_t)b * T + tid];
        } else {
            const uint32_t *ar = p.tree.anc + ((size_t)b * T + tid) * W;
            anc_v0 = ar[0];
            if (W > 1) anc_v1 = ar[1];
            dep_v = p.tree.depth[(size_t)b * T + tid];
        }
    }
    const int plim = min(p.maxlen, T);
    if (do_commit && tid < plim) path_v = p.path[(size_t)b * p.maxlen + tid];
    const float Ah = __ldg(p.A + h), Dh = __ldg(p.D + h);
    const int len = do_commit ? __ldg(p.path_len + b) : 0;
    const int okc = p.parent ? 1 : __ldg(p.tree.ok + b);

    if (tid < T) {
        dts[tid] = dt_v;
        par[tid] = par_v;
    }
    if (do_commit && tid < plim) praw[tid] = path_v;
    if (tid == 0) {
        misc[S_BADI] = INT_MAX;
        misc[S_BADQ] = INT_MAX;
    }
    __syncthreads();

    // ---------------------------------------------------------------- 2. tree
    bool okb = okc != 0;
    if (p.parent) {
        int bad = 0;
        if (tid < T) {
            bad = tid == 0 ? par_v != -1 : (par_v < 0 || par_v >= tid);
            if (bad) atomicMin(&misc[S_BADI], tid);
        }
        okb = !__syncthreads_or(bad);
    }
    if (!okb) {
        // Invalid tree: this sequence's outputs stay untouched.
        if (leader && p.parent) {
            for (int q = tid; q < T * W; q += kThreadsS)
                if (p.anc_out) p.anc_out[(size_t)b * T * W + q] = 0u;
            if (tid < T && p.depth_out) p.depth_out[(size_t)b * T + tid] = 0;
            if (tid == 0) {
                if (p.ok_out) p.ok_out[b] = 0;
                const int i = misc[S_BADI];
                latch_error(p.err, STREE_ERR_BAD_TREE, b, i, par[i]);
            }
        }
        ptx::cp_async_wait_all();
        return;
    }
    if (tid < T) {
        uint32_t a0 = anc_v0, a1 = anc_v1;
        int d = dep_v;
        if (p.parent) {
            d = -1;
            for (int j = tid; j >= 0; j = par[j]) {
                if (j < 32) a0 |= 1u << j; else a1 |= 1u << (j - 32);
                ++d;
            }
        }
        // Sum over the ancestors in increasing index order.
        float s = 0.f;
        for (uint32_t bits = a0; bits; bits &= bits - 1) s += dts[__ffs(bits) - 1];
        for (uint32_t bits = a1; bits; bits &= bits - 1) s += dts[32 + __ffs(bits) - 1];
        const float L = Ah * s;
        ancs[2 * tid] = a0;
        ancs[2 * tid + 1] = a1;
        dep[tid] = d;
        Ls[tid] = L;
        eLs[tid] = expf(L);
        if (leader && p.parent) {
            if (p.anc_out) {
                p.anc_out[((size_t)b * T + tid) * W] = a0;
                if (W > 1) p.anc_out[((size_t)b * T + tid) * W + 1] = a1;
            }
            if (p.depth_out) p.depth_out[(size_t)b * T + tid] = d;
        }
    }
    if (leader && p.parent && p.ok_out && tid == 0) p.ok_out[b] = 1;
    __syncthreads();

    // ---------------------------------------------------------------- 3. accepted path
    // Position q must hold the depth-q ancestor of the last node.
    bool commit = do_commit;
    if (do_commit) {
        if (len < 0 || len > p.maxlen || len > T) {
            commit = false;
            if (leader && tid == 0) latch_error(p.err, STREE_ERR_BAD_PATH, b, -1, len);
        } else {
            int badq = 0;
            if (tid < len) {
                const int leaf = praw[len - 1];
                const int j = praw[tid];
                const bool good = leaf >= 0 && leaf < T && j >= 0 && j < T &&
                                  ((ancs[2 * leaf + (j >> 5)] >> (j & 31)) & 1u) && dep[j] == tid;
                if (!good) {
                    badq = 1;
                    atomicMin(&misc[S_BADQ], tid);
                }
                pnode[tid] = good ? j : 0;
                wq[tid] = good ? expf(Ls[leaf] - Ls[j]) * dts[j] : 0.f;
            }
            commit = !__syncthreads_or(badq);
            if (!commit && leader && tid == 0) {
                const int q = misc[S_BADQ];
                latch_error(p.err, STREE_ERR_BAD_PATH, b, q, praw[q]);
            }
        }
    }
    ptx::cp_async_wait_all();
    __syncthreads();

    if (do_y) {
        // ------------------------------------------------------------ 4. masked decay
        // M[i][j] = exp(L_i - L_j) (C_i . B_j) dt_j for j in anc(i), plus D_h on the diagonal.
        for (int i = warp; i < T; i += kWarpsS) {
            const float4 ci = row4(Cs, i, lane);
            const float Li = Ls[i];
            for (int wd = 0; wd < W; ++wd) {
                for (uint32_t bits = ancs[2 * i + wd]; bits; bits &= bits - 1) {
                    const int j = (wd << 5) + __ffs(bits) - 1;
                    float d = dot4(ci, row4(Bs, j, lane));
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                    if (lane == 0) Ms[i * T + j] = expf(Li - Ls[j]) * d * dts[j] + (i == j ? Dh : 0.f);
                }
            }
        }
        __syncthreads();

        // ------------------------------------------------------------ 5. root + tree terms
        const int rr = lane >> 3, row = 4 * warp + rr;
        for (int n0 = 0; n0 < T; n0 += 16) {
            float v[64];
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                const float4 ci = row4(Cs, min(n0 + n, T - 1), lane);
#pragma unroll
                for (int r = 0; r < 4; ++r) v[r * 16 + n] = dot4(hv[r], ci);
            }
            reduce_scatter64(v, lane);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = n0 + 2 * (lane & 7) + u;
                if (i < T) {
                    float acc = eLs[i] * v[u];
                    const float *Mi = Ms + i * T;
                    for (int wd = 0; wd < W; ++wd)
                        for (uint32_t bits = ancs[2 * i + wd]; bits; bits &= bits - 1) {
                            const int j = (wd << 5) + __ffs(bits) - 1;
                            acc = fmaf(Mi[j], in_to_f(xs[j * kRows + row]), acc);
                        }
                    ys[i * kRows + row] = f_to_in<In>(acc);
                }
            }
        }
    }

    // ---------------------------------------------------------------- 6. commit
    if (commit) {
        const float al = len > 0 ? eLs[pnode[len - 1]] : 1.f;
        float4 acc[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
            acc[r] = make_float4(al * hv[r].x, al * hv[r].y, al * hv[r].z, al * hv[r].w);
        for (int q = 0; q < len; ++q) {
            const int j = pnode[q];
            const float4 bq = row4(Bs, j, lane);
            const float w = wq[q];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float cf = w * in_to_f(xs[j * kRows + 4 * warp + r]);
                acc[r].x = fmaf(cf, bq.x, acc[r].x);
                acc[r].y = fmaf(cf, bq.y, acc[r].y);
                acc[r].z = fmaf(cf, bq.z, acc[r].z);
                acc[r].w = fmaf(cf, bq.w, acc[r].w);
            }
        }
        float *hn = p.h_new + row0 * kN + 4 * lane;
#pragma unroll
        for (int r = 0; r < 4; ++r) __stcs(reinterpret_cast<float4 *>(hn + r * kN), acc[r]);
    }

    // ---------------------------------------------------------------- 7. y
    if (do_y) {
        __syncthreads();
        In *Yg = static_cast<In *>(p.y) + ((size_t)b * T * H + h) * P + p0;
        for (int q = tid; q < T * kXChunks; q += kThreadsS) {
            const int i = q / kXChunks, c = q % kXChunks;
            *reinterpret_cast<uint4 *>(Yg + (size_t)i * xrow + c * kEl16) =
                *reinterpret_cast<const uint4 *>(ys + i * kRows + c * kEl16);
        }
    }
}

std::mutex g_small_mutex;
bool g_small_prepared[kMaxDevices] = {};

// Raises the dynamic shared-memory limit of both instances to the largest layout
// (T = 64, fp32), once per device.
cudaError_t prepare_small()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_small_mutex);
    if (g_small_prepared[dev]) return cudaSuccess;
    const int most = (int)SmallLayout(kMaxSmallNodes, 4).total;
    if ((e = cudaFuncSetAttribute(scan_small_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, most)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(scan_small_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  most)) != cudaSuccess)
        return e;
    g_small_prepared[dev] = true;
    return cudaSuccess;
}

}  // namespace

bool small_supported(const ScanArgs &a)
{
    if (a.dtype != STREE_BF16 && a.dtype != STREE_F32) return false;
    if (a.N != kN || a.P % kRows != 0 || a.T < 1 || a.T > kMaxSmallNodes || a.batch < 1) return false;
    if (!a.y) return false;
    const long long grid = (long long)a.batch * a.H * (a.P / kRows);
    return grid <= 0x7fffffffLL;
}

cudaError_t launch_scan_small(const ScanArgs &a, cudaStream_t s)
{
    if (!small_supported(a)) return cudaErrorNotSupported;
    cudaError_t e = prepare_small();
    if (e != cudaSuccess) return e;
    SmallParams p{};
    p.x = a.x; p.dt = a.dt; p.B = a.B; p.C = a.C;
    p.A = a.A; p.D = a.D; p.h0 = a.h0;
    p.parent = a.parent;
    p.tree = a.tree;
    p.anc_out = a.tree_anc;
    p.depth_out = a.tree_depth;
    p.ok_out = a.tree_ok;
    const bool commit = a.path != nullptr && a.h_new != nullptr;
    p.path = commit ? a.path : nullptr;
    p.path_len = commit ? a.path_len : nullptr;
    p.maxlen = commit ? a.maxlen : 0;
    p.y = a.y;
    p.h_new = commit ? a.h_new : nullptr;
    p.err = a.err;
    p.T = a.T; p.H = a.H; p.P = a.P; p.G = a.G;
    p.slices = a.P / kRows;
    const int e16 = a.dtype == STREE_BF16 ? 2 : 4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((long long)a.batch * a.H * p.slices));
    cfg.blockDim = dim3(kThreadsS);
    cfg.dynamicSmemBytes = SmallLayout(a.T, e16).total;
    cfg.stream = s;
    // Programmatic dependent launch: the kernel waits for the preceding grid
    // before its first global read, so its launch overlaps that grid's tail.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.dtype == STREE_BF16) return cudaLaunchKernelEx(&cfg, scan_small_kernel<__nv_bfloat16>, p);
    return cudaLaunchKernelEx(&cfg, scan_small_kernel<float>, p);
}

}  // namespace stree
