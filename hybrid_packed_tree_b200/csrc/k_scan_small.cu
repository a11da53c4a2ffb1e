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
//   * at entry every global read is issued: the per-node scalars (parent, dt,
//     path, A, D), and bulk copies into shared memory (one mbarrier) of the CTA's
//     32 rows of h0 (16 KB, contiguous), the sequence's C and B rows and the CTA's
//     x columns; the four root warps then hold 8 rows x 4 columns of h0 per lane
//     in registers (warp w rows 8w..8w+7, lane l columns 4l..4l+3);
//   * two warp groups then work side by side: the tree group (warps 4-7)
//     rebuilds the tree from parent[] (one thread per node: ancestor bits, depth,
//     L), checks the accepted path and forms the masked decay matrix (C_i . B_j on
//     ancestor pairs, four lanes per pair), while the root group multiplies its
//     rows of h0 with every C_i (each lane its 4 columns, then a butterfly
//     reduce-scatter over the warp: 62 shuffles per 4 rows and 16 nodes);
//   * all threads then form y = exp(L) R + M x (D_h on M's diagonal), the root
//     group applies the commit to its h0 registers and stores h_new, and y is
//     written with 16-byte stores.
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
#include "warp_tiles.cuh"

namespace stree {
namespace {

using namespace tiles;

constexpr int kN = 128;                     // dstate of this kernel
constexpr int kRows = 32;                   // headdim rows per CTA
constexpr int kWarpsS = 8;
constexpr int kThreadsS = kWarpsS * 32;
constexpr int kRootWarps = 4;               // warps 0-3: the root term and the commit, 8 rows each
constexpr int kTreeThreads = (kWarpsS - kRootWarps) * 32;
constexpr int kBarTree = 1;                 // named barrier of the tree group (0 is __syncthreads)
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

enum SmallMisc { S_BADI = 0, S_BADQ, S_LEN, S_TREEOK, S_PATHOK, S_COMMIT, S_DATAOK, S_MAXD, S_A, S_D, kSmallMisc };

// Shared-memory layout for T nodes and input element size e (bytes).
struct SmallLayout {
    uint32_t h, c, b, x, y, r, m, L, eL, dt, par, dep, anc, praw, pnode, wq, misc, bar, total;
    __host__ __device__ SmallLayout(int T, int e)
    {
        uint32_t o = 0;
        auto take = [&](uint32_t bytes) {
            const uint32_t at = o;
            o = (o + bytes + 15u) & ~15u;
            return at;
        };
        h = take((uint32_t)kRows * kN * 4);
        c = take((uint32_t)T * kN * e);
        b = take((uint32_t)T * kN * e);
        x = take((uint32_t)T * kRows * e);
        y = take((uint32_t)T * kRows * e);
        r = take((uint32_t)T * kRows * 4);
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
        misc = take(kSmallMisc * 4);
        bar = take(8);
        total = o;
    }
};


template <typename In>
__global__ void __launch_bounds__(kThreadsS, 2) scan_small_kernel(const SmallParams p)
{
    extern __shared__ __align__(16) uint8_t sm[];
    const int T = p.T, H = p.H, P = p.P, G = p.G;
    const SmallLayout ly(T, (int)sizeof(In));
    float *h0s = reinterpret_cast<float *>(sm + ly.h);   // [32][128] the CTA's rows of h0
    In *Cs = reinterpret_cast<In *>(sm + ly.c);          // [T][128] C rows of (b, g)
    In *Bs = reinterpret_cast<In *>(sm + ly.b);          // [T][128] B rows of (b, g)
    In *xs = reinterpret_cast<In *>(sm + ly.x);          // [T][32]  x columns of the CTA
    In *ys = reinterpret_cast<In *>(sm + ly.y);          // [T][32]  y staging
    float *Rs = reinterpret_cast<float *>(sm + ly.r);    // [T][32]  root term h0 . C_i
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
    float *miscf = reinterpret_cast<float *>(misc);
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sm + ly.bar);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool tree_warp = warp >= kRootWarps;            // warps 4-7: tree, path, masked decay
    const int ttid = tid - kRootWarps * 32;               // index within the tree group
    const int W = (T + 31) >> 5;
    const int slice = blockIdx.x % p.slices;
    const int h = (blockIdx.x / p.slices) % H;
    const int b = blockIdx.x / (p.slices * H);
    const int g = h / (H / G);
    const int p0 = slice * kRows;
    const bool leader = h == 0 && slice == 0;
    const bool do_commit = p.h_new != nullptr;
    const uint32_t bar = ptx::smem_u32(mbar);

    // The kernel is launched as a programmatic dependent of the preceding grid on
    // the stream: it may start while that grid drains, and waits for its
    // completion before the first global read.  A later launch may likewise start
    // now; it waits for this grid's completion before it reads anything.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---------------------------------------------------------------- 1. loads
    // Every global read is issued before any is waited for: the tree group loads
    // the per-node scalars (they start the dependent chain), the root group its
    // rows of the state into registers, and one thread the bulk copies of C, B and
    // x into shared memory.  asm volatile with a memory clobber keeps the compiler
    // from moving loads across the copies.
    const In *dtg = static_cast<const In *>(p.dt);
    const int plim = min(p.maxlen, T);
    In dt_raw{};
    int par_v = 0, dep_v = 0, path_v = 0, len_v = 0, ok_v = 1;
    uint32_t anc_v0 = 0u, anc_v1 = 0u;
    float A_v = 0.f, D_v = 0.f;
    if (tree_warp) {
        if (ttid < T) {
            dt_raw = dtg[((size_t)b * T + ttid) * H + h];
            if (p.parent) {
                par_v = p.parent[(size_t)b * T + ttid];
            } else {
                const uint32_t *ar = p.tree.anc + ((size_t)b * T + ttid) * W;
                anc_v0 = ar[0];
                if (W > 1) anc_v1 = ar[1];
                dep_v = p.tree.depth[(size_t)b * T + ttid];
            }
        }
        if (do_commit && ttid < plim) path_v = p.path[(size_t)b * p.maxlen + ttid];
        if (ttid == 0) {
            A_v = p.A[h];
            D_v = p.D[h];
            if (do_commit) len_v = p.path_len[b];
            if (!p.parent) ok_v = p.tree.ok[b];
        }
    }
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
        misc[S_DATAOK] = 1;
    }
    __syncthreads();
    constexpr uint32_t kRowBytes = kN * sizeof(In), kXBytes = kRows * sizeof(In);
    const size_t brow = (size_t)G * kN, xrow = (size_t)H * P;
    const In *Cg = static_cast<const In *>(p.C) + ((size_t)b * T * G + g) * kN;
    const In *Bg = static_cast<const In *>(p.B) + ((size_t)b * T * G + g) * kN;
    const In *Xg = static_cast<const In *>(p.x) + ((size_t)b * T * H + h) * P + p0;
    if (warp == 0) {
        constexpr uint32_t kSliceBytes = kRows * kN * 4;
        if (lane == 0) {
            ptx::mbar_expect_tx(bar, kSliceBytes + (uint32_t)T * (2u * kRowBytes + kXBytes));
            ptx::bulk_g2s(ptx::smem_u32(h0s), p.h0 + (((size_t)b * H + h) * P + p0) * kN, kSliceBytes, bar);
        }
        __syncwarp();
        if (G == 1) {                                     // the sequence's rows are contiguous
            if (lane == 0) {
                ptx::bulk_g2s(ptx::smem_u32(Cs), Cg, (uint32_t)T * kRowBytes, bar);
                ptx::bulk_g2s(ptx::smem_u32(Bs), Bg, (uint32_t)T * kRowBytes, bar);
            }
        } else {
            for (int i = lane; i < T; i += 32) {
                ptx::bulk_g2s(ptx::smem_u32(Cs + i * kN), Cg + (size_t)i * brow, kRowBytes, bar);
                ptx::bulk_g2s(ptx::smem_u32(Bs + i * kN), Bg + (size_t)i * brow, kRowBytes, bar);
            }
        }
        for (int i = lane; i < T; i += 32)
            ptx::bulk_g2s(ptx::smem_u32(xs + i * kRows), Xg + (size_t)i * xrow, kXBytes, bar);
    }

    bool okb = true, commit = false;
    int len = 0;
    float4 hv[8];                                         // root warps: rows 8 w + r, columns 4 lane + c
    if (tree_warp) {
        // ------------------------------------------------------------ 2. tree (tree group)
        if (ttid < T) {
            dts[ttid] = in_to_f(dt_raw);
            par[ttid] = par_v;
        }
        if (do_commit && ttid < plim) praw[ttid] = path_v;
        if (ttid == 0) {
            misc[S_BADI] = INT_MAX;
            misc[S_BADQ] = INT_MAX;
            misc[S_MAXD] = 0;
            misc[S_TREEOK] = ok_v;
            misc[S_LEN] = len_v;
            miscf[S_A] = A_v;
            miscf[S_D] = D_v;
        }
        named_sync(kBarTree, kTreeThreads);
        if (p.parent && ttid < T && (ttid == 0 ? par_v != -1 : (par_v < 0 || par_v >= ttid))) {
            atomicMin(&misc[S_BADI], ttid);
            misc[S_TREEOK] = 0;
        }
        named_sync(kBarTree, kTreeThreads);
        okb = misc[S_TREEOK] != 0;
        len = misc[S_LEN];
        const float Ah = miscf[S_A];
        if (okb && ttid < T) {
            uint32_t a0 = anc_v0, a1 = anc_v1;
            int d = dep_v;
            if (p.parent) {
                d = -1;
                for (int j = ttid; j >= 0; j = par[j]) {
                    if (j < 32) a0 |= 1u << j; else a1 |= 1u << (j - 32);
                    ++d;
                }
            }
            // Sum over the ancestors in increasing index order.
            float sum = 0.f;
            for (uint32_t bits = a0; bits; bits &= bits - 1) sum += dts[__ffs(bits) - 1];
            for (uint32_t bits = a1; bits; bits &= bits - 1) sum += dts[32 + __ffs(bits) - 1];
            const float L = Ah * sum;
            ancs[2 * ttid] = a0;
            ancs[2 * ttid + 1] = a1;
            dep[ttid] = d;
            atomicMax(&misc[S_MAXD], d);
            Ls[ttid] = L;
            eLs[ttid] = expf(L);
        }
        if (leader && p.parent) {
            // The sequence's tree for later calls (zeros and a cleared flag when invalid).
            if (ttid < T) {
                if (p.anc_out) {
                    p.anc_out[((size_t)b * T + ttid) * W] = okb ? ancs[2 * ttid] : 0u;
                    if (W > 1) p.anc_out[((size_t)b * T + ttid) * W + 1] = okb ? ancs[2 * ttid + 1] : 0u;
                }
                if (p.depth_out) p.depth_out[(size_t)b * T + ttid] = okb ? dep[ttid] : 0;
            }
            if (ttid == 0) {
                if (p.ok_out) p.ok_out[b] = okb ? 1 : 0;
                if (!okb) {
                    const int i = misc[S_BADI];
                    latch_error(p.err, STREE_ERR_BAD_TREE, b, i, par[i]);
                }
            }
        }
        named_sync(kBarTree, kTreeThreads);

        // ------------------------------------------------------------ 3. accepted path
        // Position q must hold the depth-q ancestor of the last node.
        if (okb && do_commit) {
            if (len < 0 || len > p.maxlen || len > T) {
                if (leader && ttid == 0) latch_error(p.err, STREE_ERR_BAD_PATH, b, -1, len);
            } else {
                if (ttid == 0) misc[S_PATHOK] = 1;
                named_sync(kBarTree, kTreeThreads);
                if (ttid < len) {
                    const int leaf = praw[len - 1];
                    const int j = praw[ttid];
                    const bool good = leaf >= 0 && leaf < T && j >= 0 && j < T &&
                                      ((ancs[2 * leaf + (j >> 5)] >> (j & 31)) & 1u) && dep[j] == ttid;
                    if (!good) {
                        atomicMin(&misc[S_BADQ], ttid);
                        misc[S_PATHOK] = 0;
                    }
                    pnode[ttid] = good ? j : 0;
                    wq[ttid] = good ? expf(Ls[leaf] - Ls[j]) * dts[j] : 0.f;
                }
                named_sync(kBarTree, kTreeThreads);
                commit = misc[S_PATHOK] != 0;
                if (!commit && leader && ttid == 0) {
                    const int q = misc[S_BADQ];
                    latch_error(p.err, STREE_ERR_BAD_PATH, b, q, praw[q]);
                }
            }
        }

        // ------------------------------------------------------------ 4. masked decay (tree group)
        // M[i][j] = exp(L_i - L_j) (C_i . B_j) dt_j for j in anc(i), plus D_h on the
        // diagonal.  Slot (i, k) pairs i with its depth-k ancestor (the k-th set bit
        // of its row); four lanes take a slot, 32 state columns each.
        const bool data_ok = ptx::mbar_wait(bar, 0);
        if (!data_ok) {
            misc[S_DATAOK] = 0;
            latch_error(p.err, STREE_ERR_TIMEOUT, b, h, slice);
        }
        if (okb && data_ok) {
            const float Dh = miscf[S_D];
            int lgD = 0;
            while ((1 << lgD) < misc[S_MAXD] + 1) ++lgD;
            const int nslots = T << lgD, quarter = lane & 3;
            for (int base = (warp - kRootWarps) * 8; base < nslots; base += kTreeThreads / 4) {
                const int q = base + (lane >> 2);
                const int i = min(q >> lgD, T - 1), k = q & ((1 << lgD) - 1);
                const bool valid = q < nslots && k <= dep[i];
                uint32_t a0 = ancs[2 * i], a1 = ancs[2 * i + 1];
                for (int t = 0; t < k && (a0 | a1); ++t) {       // drop the k lowest ancestors
                    if (a0) a0 &= a0 - 1; else a1 &= a1 - 1;
                }
                const int j = valid ? (a0 ? __ffs(a0) - 1 : 32 + __ffs(a1) - 1) : i;
                float d = dot32(Cs, Bs, i, j, quarter, dot32_rot<In>(lane));
                d += __shfl_xor_sync(0xffffffffu, d, 1);
                d += __shfl_xor_sync(0xffffffffu, d, 2);
                if (valid && quarter == 0) Ms[i * T + j] = expf(Ls[i] - Ls[j]) * d * dts[j] + (i == j ? Dh : 0.f);
            }
        }
        if (ttid == 0) misc[S_COMMIT] = commit ? 1 : 0;
    } else {
        // ------------------------------------------------------------ 5. root term (root group)
        // R[i][row] = h0[row] . C_i for the warp's 8 rows: per 4 rows and 16 nodes, each
        // lane multiplies its 4 columns, and a reduce-scatter over the warp leaves
        // it two (row, node) sums.
        if (ptx::mbar_wait(bar, 0)) {
#pragma unroll
            for (int r = 0; r < 8; ++r) hv[r] = *reinterpret_cast<const float4 *>(h0s + (8 * warp + r) * kN + 4 * lane);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                for (int n0 = 0; n0 < T; n0 += 16) {
                    float v[64];
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        const float4 ci = row4(Cs, min(n0 + n, T - 1), lane);
#pragma unroll
                        for (int r = 0; r < 4; ++r) v[r * 16 + n] = dot4(hv[4 * half + r], ci);
                    }
                    reduce_scatter64(v, lane);
                    const int row = 8 * warp + 4 * half + (lane >> 3);
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int i = n0 + 2 * (lane & 7) + u;
                        if (i < T) Rs[i * kRows + row] = v[u];
                    }
                }
            }
        } else {
            misc[S_DATAOK] = 0;
            latch_error(p.err, STREE_ERR_TIMEOUT, b, h, slice);
        }
    }
    __syncthreads();
    if (!misc[S_TREEOK] || !misc[S_DATAOK]) {
        // Invalid tree or copies that never landed: no output; the copies get one
        // more bounded wait, so that none lands after the CTA has exited.
        ptx::mbar_wait(bar, 0);
        return;
    }

    // ---------------------------------------------------------------- 6. y = exp(L) R + M x
    for (int q = tid; q < T * kRows; q += kThreadsS) {
        const int i = q / kRows, row = q - i * kRows;
        float acc = eLs[i] * Rs[q];
        const float *Mi = Ms + i * T;
        for (int wd = 0; wd < W; ++wd)
            for (uint32_t bits = ancs[2 * i + wd]; bits; bits &= bits - 1) {
                const int j = (wd << 5) + __ffs(bits) - 1;
                acc = fmaf(Mi[j], in_to_f(xs[j * kRows + row]), acc);
            }
        ys[q] = f_to_in<In>(acc);
    }

    // ---------------------------------------------------------------- 7. commit (root group)
    if (!tree_warp && misc[S_COMMIT]) {
        len = misc[S_LEN];
        const float al = len > 0 ? eLs[pnode[len - 1]] : 1.f;
        float4 acc[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r] = make_float4(al * hv[r].x, al * hv[r].y, al * hv[r].z, al * hv[r].w);
        for (int q = 0; q < len; ++q) {
            const int j = pnode[q];
            const float4 bq = row4(Bs, j, lane);
            const float w = wq[q];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float cf = w * in_to_f(xs[j * kRows + 8 * warp + r]);
                acc[r].x = fmaf(cf, bq.x, acc[r].x);
                acc[r].y = fmaf(cf, bq.y, acc[r].y);
                acc[r].z = fmaf(cf, bq.z, acc[r].z);
                acc[r].w = fmaf(cf, bq.w, acc[r].w);
            }
        }
        float *hn = p.h_new + (((size_t)b * H + h) * P + p0 + 8 * warp) * kN + 4 * lane;
#pragma unroll
        for (int r = 0; r < 8; ++r) __stcs(reinterpret_cast<float4 *>(hn + r * kN), acc[r]);
    }

    // ---------------------------------------------------------------- 8. y
    __syncthreads();
    constexpr int kEl16 = 16 / (int)sizeof(In), kXChunks = kRows / kEl16;
    In *Yg = static_cast<In *>(p.y) + ((size_t)b * T * H + h) * P + p0;
    for (int q = tid; q < T * kXChunks; q += kThreadsS) {
        const int i = q / kXChunks, c = q % kXChunks;
        *reinterpret_cast<uint4 *>(Yg + (size_t)i * xrow + c * kEl16) =
            *reinterpret_cast<const uint4 *>(ys + i * kRows + c * kEl16);
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
