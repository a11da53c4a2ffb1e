// k_gdn.cu -- the gated delta rule (linear attention) over the packed draft tree,
// with the commit of the accepted path, sm_100a.
//
// Method ("TreeWY" abstract: Gated DeltaNet layers; every draft node's output from
// one triangular solve, and only the accepted state rebuilt on commit from a small
// pseudo-value matrix instead of per-node states; "Bole" abstract: the
// tree-structured closed form of the linear-attention recurrence).  Per sequence
// and value head, with state S [d_v, d_k], write strength beta and erase strength a
// (a = beta for the gated delta rule; apart, the decoupled erase and write of
// Gated DeltaNet-2; a = 0, gated linear attention):
//   S_i = alpha_i S_p(i) (I - a_i k_i k_i^T) + beta_i v_i k_i^T,  S_p(root) = S0,  o_i = S_i q_i.
// Writing S_t = alpha_t S_{t-1} + u_t k_t^T with u_t = beta_t v_t - a_t alpha_t S_{t-1} k_t
// and gamma_i for the product of alpha over the root path of i:
//   u_j   = beta_j v_j - a_j gamma_j S0 k_j - sum_{l strict ancestor of j} a_j (gamma_j / gamma_l) (k_j . k_l) u_l
//   o_i   = gamma_i S0 q_i + sum_{j in anc(i)} (gamma_i / gamma_j) (q_i . k_j) u_j
//   S_new = gamma_leaf S0 + sum_{j on path} (gamma_leaf / gamma_j) u_j k_j^T
// The system for u is lower triangular over the ancestor relation: nodes of one
// depth depend only on shallower ones, so it is solved level by level.
//
// Design: the small-batch layout of the SSM scan (k_scan_small.cu), because the
// state plays the part of h0 (rows d_v, 128 columns d_k) and a decode step is a
// few MB: one CTA per (sequence, value head, 32 rows of d_v), every global read
// issued at entry (the root group's rows of S0 into registers, bulk copies of q, k
// and the CTA's v columns, the scalars); the tree group rebuilds the tree (log
// gamma as a tree cumsum), checks the path and forms both pair matrices (q_i . k_j
// on ancestor pairs for the outputs, k_j . k_l for the solve; four lanes per pair)
// while the root group forms S0 q_i and S0 k_i (reduce-scatter over the warp);
// then all threads solve for u level by level, form the outputs, and the root
// group rebuilds the accepted state from its S0 registers.  CUDA cores, fp32.
#include <climits>
#include <mutex>

#include "stree_internal.cuh"
#include "tc_ptx.cuh"
#include "warp_tiles.cuh"

namespace stree {
namespace {

using namespace tiles;

constexpr int kK = 128;                     // d_k
constexpr int kRows = 32;                   // d_v rows per CTA
constexpr int kWarpsG = 8;
constexpr int kThreadsG = kWarpsG * 32;
constexpr int kRootWarps = 4;               // warps 0-3: S0 q, S0 k and the commit, 8 rows each
constexpr int kTreeThreads = (kWarpsG - kRootWarps) * 32;
constexpr int kBarTree = 1;
constexpr int kMaxGdnNodes = 64;
constexpr int kMaxDevices = 64;

struct GdnParams {
    const void *q, *k, *v;
    const float *alpha, *beta, *erase, *S0;          // erase NULL: a = beta
    const int32_t *parent, *path, *path_len;
    int maxlen;
    void *o;
    float *S_new;                           // NULL: no commit
    int32_t *err;
    int T, Hv, Hk, dv, slices;
};

enum GdnMisc { G_BADI = 0, G_BADQ, G_LEN, G_TREEOK, G_PATHOK, G_COMMIT, G_DATAOK, G_MAXD, kGdnMisc };

struct GdnLayout {
    uint32_t q, k, v, o, rq, rk, u, mq, ak, lg, eg, be, er, la, par, dep, anc, praw, pnode, wq, misc, bar, total;
    __host__ __device__ GdnLayout(int T, int e)
    {
        uint32_t off = 0;
        auto take = [&](uint32_t bytes) {
            const uint32_t at = off;
            off = (off + bytes + 15u) & ~15u;
            return at;
        };
        q = take((uint32_t)T * kK * e);
        k = take((uint32_t)T * kK * e);
        v = take((uint32_t)T * kRows * e);
        o = take((uint32_t)T * kRows * e);
        rq = take((uint32_t)T * kRows * 4);
        rk = take((uint32_t)T * kRows * 4);
        u = take((uint32_t)T * kRows * 4);
        mq = take((uint32_t)T * T * 4);
        ak = take((uint32_t)T * T * 4);
        lg = take((uint32_t)T * 4);
        eg = take((uint32_t)T * 4);
        be = take((uint32_t)T * 4);
        er = take((uint32_t)T * 4);
        la = take((uint32_t)T * 4);
        par = take((uint32_t)T * 4);
        dep = take((uint32_t)T * 4);
        anc = take((uint32_t)T * 8);
        praw = take((uint32_t)T * 4);
        pnode = take((uint32_t)T * 4);
        wq = take((uint32_t)T * 4);
        misc = take(kGdnMisc * 4);
        bar = take(8);
        total = off;
    }
};

// The call's error word is optional.
__device__ __forceinline__ void latch_if(int32_t *err, int code, int b, int pos, int detail)
{
    if (err) latch_error(err, code, b, pos, detail);
}

template <typename In>
__global__ void __launch_bounds__(kThreadsG, 2) gdn_tree_kernel(const GdnParams p)
{
    extern __shared__ __align__(16) uint8_t sm[];
    const int T = p.T, Hv = p.Hv, Hk = p.Hk, dv = p.dv;
    const GdnLayout ly(T, (int)sizeof(In));
    In *qs = reinterpret_cast<In *>(sm + ly.q);          // [T][128] q rows of the key head
    In *ks = reinterpret_cast<In *>(sm + ly.k);          // [T][128] k rows
    In *vs = reinterpret_cast<In *>(sm + ly.v);          // [T][32]  v columns of the CTA
    In *os = reinterpret_cast<In *>(sm + ly.o);          // [T][32]  output staging
    float *Rq = reinterpret_cast<float *>(sm + ly.rq);   // [T][32]  S0 q_i
    float *Rk = reinterpret_cast<float *>(sm + ly.rk);   // [T][32]  S0 k_i
    float *U = reinterpret_cast<float *>(sm + ly.u);     // [T][32]  pseudo-values
    float *Mq = reinterpret_cast<float *>(sm + ly.mq);   // [T][T]   (gamma_i / gamma_j) q_i . k_j
    float *Ak = reinterpret_cast<float *>(sm + ly.ak);   // [T][T]   beta_i (gamma_i / gamma_j) k_i . k_j
    float *lg = reinterpret_cast<float *>(sm + ly.lg);   // log gamma
    float *eg = reinterpret_cast<float *>(sm + ly.eg);   // gamma
    float *bes = reinterpret_cast<float *>(sm + ly.be);  // beta (write)
    float *ers = reinterpret_cast<float *>(sm + ly.er);  // erase strength
    float *las = reinterpret_cast<float *>(sm + ly.la);  // log alpha
    int32_t *par = reinterpret_cast<int32_t *>(sm + ly.par);
    int32_t *dep = reinterpret_cast<int32_t *>(sm + ly.dep);
    uint32_t *ancs = reinterpret_cast<uint32_t *>(sm + ly.anc);
    int32_t *praw = reinterpret_cast<int32_t *>(sm + ly.praw);
    int32_t *pnode = reinterpret_cast<int32_t *>(sm + ly.pnode);
    float *wq = reinterpret_cast<float *>(sm + ly.wq);
    int32_t *misc = reinterpret_cast<int32_t *>(sm + ly.misc);
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sm + ly.bar);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool tree_warp = warp >= kRootWarps;
    const int ttid = tid - kRootWarps * 32;
    const int slice = blockIdx.x % p.slices;
    const int h = (blockIdx.x / p.slices) % Hv;
    const int b = blockIdx.x / (p.slices * Hv);
    const int g = h / (Hv / Hk);
    const int p0 = slice * kRows;
    const bool leader = h == 0 && slice == 0;
    const bool do_commit = p.S_new != nullptr;
    const uint32_t bar = ptx::smem_u32(mbar);

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---------------------------------------------------------------- 1. loads
    const int plim = min(p.maxlen, T);
    int par_v = 0, path_v = 0, len_v = 0;
    float al_v = 1.f, be_v = 0.f, er_v = 0.f;
    float4 hv[8];                                         // root warps: rows 8 w + r of S0
    if (tree_warp) {
        if (ttid < T) {
            par_v = p.parent[(size_t)b * T + ttid];
            al_v = p.alpha[((size_t)b * T + ttid) * Hv + h];
            be_v = p.beta[((size_t)b * T + ttid) * Hv + h];
            er_v = p.erase ? p.erase[((size_t)b * T + ttid) * Hv + h] : be_v;
        }
        if (do_commit && ttid < plim) path_v = p.path[(size_t)b * p.maxlen + ttid];
        if (do_commit && ttid == 0) len_v = p.path_len[b];
    } else {
        const float *sr = p.S0 + (((size_t)b * Hv + h) * dv + p0 + 8 * warp) * kK + 4 * lane;
#pragma unroll
        for (int r = 0; r < 8; ++r)
            asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(hv[r].x), "=f"(hv[r].y), "=f"(hv[r].z), "=f"(hv[r].w)
                         : "l"(sr + r * kK)
                         : "memory");
    }
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
        misc[G_DATAOK] = 1;
    }
    __syncthreads();
    constexpr uint32_t kRowBytes = kK * sizeof(In), kVBytes = kRows * sizeof(In);
    const In *Qg = static_cast<const In *>(p.q) + ((size_t)b * T * Hk + g) * kK;   // row i at + i * Hk * kK
    const In *Kg = static_cast<const In *>(p.k) + ((size_t)b * T * Hk + g) * kK;
    const In *Vg = static_cast<const In *>(p.v) + ((size_t)b * T * Hv + h) * dv + p0;
    const size_t krow = (size_t)Hk * kK, vrow = (size_t)Hv * dv;
    if (warp == 0) {
        if (lane == 0) ptx::mbar_expect_tx(bar, (uint32_t)T * (2u * kRowBytes + kVBytes));
        __syncwarp();
        if (Hk == 1) {
            if (lane == 0) {
                ptx::bulk_g2s(ptx::smem_u32(qs), Qg, (uint32_t)T * kRowBytes, bar);
                ptx::bulk_g2s(ptx::smem_u32(ks), Kg, (uint32_t)T * kRowBytes, bar);
            }
        } else {
            for (int i = lane; i < T; i += 32) {
                ptx::bulk_g2s(ptx::smem_u32(qs + i * kK), Qg + (size_t)i * krow, kRowBytes, bar);
                ptx::bulk_g2s(ptx::smem_u32(ks + i * kK), Kg + (size_t)i * krow, kRowBytes, bar);
            }
        }
        for (int i = lane; i < T; i += 32)
            ptx::bulk_g2s(ptx::smem_u32(vs + i * kRows), Vg + (size_t)i * vrow, kVBytes, bar);
    }

    if (tree_warp) {
        // ------------------------------------------------------------ 2. tree (tree group)
        if (ttid < T) {
            par[ttid] = par_v;
            las[ttid] = logf(al_v);
            bes[ttid] = be_v;
            ers[ttid] = er_v;
        }
        if (do_commit && ttid < plim) praw[ttid] = path_v;
        if (ttid == 0) {
            misc[G_BADI] = INT_MAX;
            misc[G_BADQ] = INT_MAX;
            misc[G_MAXD] = 0;
            misc[G_TREEOK] = 1;
            misc[G_LEN] = len_v;
            misc[G_PATHOK] = 0;
        }
        named_sync(kBarTree, kTreeThreads);
        if (ttid < T && (ttid == 0 ? par_v != -1 : (par_v < 0 || par_v >= ttid))) {
            atomicMin(&misc[G_BADI], ttid);
            misc[G_TREEOK] = 0;
        }
        named_sync(kBarTree, kTreeThreads);
        const bool okb = misc[G_TREEOK] != 0;
        const int len = misc[G_LEN];
        if (okb && ttid < T) {
            uint32_t a0 = 0u, a1 = 0u;
            int d = -1;
            for (int j = ttid; j >= 0; j = par[j]) {
                if (j < 32) a0 |= 1u << j; else a1 |= 1u << (j - 32);
                ++d;
            }
            float sum = 0.f;                              // ancestors in increasing index order
            for (uint32_t bits = a0; bits; bits &= bits - 1) sum += las[__ffs(bits) - 1];
            for (uint32_t bits = a1; bits; bits &= bits - 1) sum += las[32 + __ffs(bits) - 1];
            ancs[2 * ttid] = a0;
            ancs[2 * ttid + 1] = a1;
            dep[ttid] = d;
            atomicMax(&misc[G_MAXD], d);
            lg[ttid] = sum;
            eg[ttid] = expf(sum);
        }
        if (!okb && leader && ttid == 0) {
            const int i = misc[G_BADI];
            latch_if(p.err, STREE_ERR_BAD_TREE, b, i, par[i]);
        }
        named_sync(kBarTree, kTreeThreads);
        if (okb && do_commit) {
            if (len < 0 || len > p.maxlen || len > T) {
                if (leader && ttid == 0) latch_if(p.err, STREE_ERR_BAD_PATH, b, -1, len);
            } else {
                if (ttid == 0) misc[G_PATHOK] = 1;
                named_sync(kBarTree, kTreeThreads);
                if (ttid < len) {
                    const int leaf = praw[len - 1];
                    const int j = praw[ttid];
                    const bool good = leaf >= 0 && leaf < T && j >= 0 && j < T &&
                                      ((ancs[2 * leaf + (j >> 5)] >> (j & 31)) & 1u) && dep[j] == ttid;
                    if (!good) {
                        atomicMin(&misc[G_BADQ], ttid);
                        misc[G_PATHOK] = 0;
                    }
                    pnode[ttid] = good ? j : 0;
                    wq[ttid] = good ? expf(lg[leaf] - lg[j]) : 0.f;
                }
                named_sync(kBarTree, kTreeThreads);
                if (!misc[G_PATHOK] && leader && ttid == 0) {
                    const int q = misc[G_BADQ];
                    latch_if(p.err, STREE_ERR_BAD_PATH, b, q, praw[q]);
                }
            }
        }

        // ------------------------------------------------------------ 3. pair matrices (tree group)
        // Slot (i, k) pairs i with its depth-k ancestor j; four lanes per slot.
        const bool data_ok = ptx::mbar_wait(bar, 0);
        if (!data_ok) {
            misc[G_DATAOK] = 0;
            latch_if(p.err, STREE_ERR_TIMEOUT, b, h, slice);
        }
        if (okb && data_ok) {
            int lgD = 0;
            while ((1 << lgD) < misc[G_MAXD] + 1) ++lgD;
            const int nslots = T << lgD, quarter = lane & 3;
            for (int base = (warp - kRootWarps) * 8; base < nslots; base += kTreeThreads / 4) {
                const int q = base + (lane >> 2);
                const int i = min(q >> lgD, T - 1), kk = q & ((1 << lgD) - 1);
                const bool valid = q < nslots && kk <= dep[i];
                uint32_t a0 = ancs[2 * i], a1 = ancs[2 * i + 1];
                for (int t = 0; t < kk && (a0 | a1); ++t) {
                    if (a0) a0 &= a0 - 1; else a1 &= a1 - 1;
                }
                const int j = valid ? (a0 ? __ffs(a0) - 1 : 32 + __ffs(a1) - 1) : i;
                float dq = dot32(qs, ks, i, j, quarter, dot32_rot<In>(lane));
                float dk = dot32(ks, ks, i, j, quarter, dot32_rot<In>(lane));
                dq += __shfl_xor_sync(0xffffffffu, dq, 1);
                dk += __shfl_xor_sync(0xffffffffu, dk, 1);
                dq += __shfl_xor_sync(0xffffffffu, dq, 2);
                dk += __shfl_xor_sync(0xffffffffu, dk, 2);
                if (valid && quarter == 0) {
                    const float r = expf(lg[i] - lg[j]);
                    Mq[i * T + j] = r * dq;
                    if (j != i) Ak[i * T + j] = ers[i] * r * dk;
                }
            }
        }
        if (ttid == 0) misc[G_COMMIT] = misc[G_PATHOK];
    } else {
        // ------------------------------------------------------------ 4. S0 q_i and S0 k_i (root group)
        if (ptx::mbar_wait(bar, 0)) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const In *X = which == 0 ? qs : ks;
                float *R = which == 0 ? Rq : Rk;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    for (int n0 = 0; n0 < T; n0 += 16) {
                        float vv[64];
#pragma unroll
                        for (int n = 0; n < 16; ++n) {
                            const float4 xi = row4(X, min(n0 + n, T - 1), lane);
#pragma unroll
                            for (int r = 0; r < 4; ++r) vv[r * 16 + n] = dot4(hv[4 * half + r], xi);
                        }
                        reduce_scatter64(vv, lane);
                        const int row = 8 * warp + 4 * half + (lane >> 3);
#pragma unroll
                        for (int u2 = 0; u2 < 2; ++u2) {
                            const int i = n0 + 2 * (lane & 7) + u2;
                            if (i < T) R[i * kRows + row] = vv[u2];
                        }
                    }
                }
            }
        } else {
            misc[G_DATAOK] = 0;
            latch_if(p.err, STREE_ERR_TIMEOUT, b, h, slice);
        }
    }
    __syncthreads();
    if (!misc[G_TREEOK] || !misc[G_DATAOK]) {
        ptx::mbar_wait(bar, 0);                           // no copy may land after exit
        return;
    }

    // ---------------------------------------------------------------- 5. pseudo-values, level by level
    const int maxd = misc[G_MAXD];
    for (int d = 0; d <= maxd; ++d) {
        for (int e = tid; e < T * kRows; e += kThreadsG) {
            const int j = e / kRows, row = e - j * kRows;
            if (dep[j] != d) continue;
            float u = p.erase ? bes[j] * in_to_f(vs[e]) - ers[j] * eg[j] * Rk[e]
                              : bes[j] * (in_to_f(vs[e]) - eg[j] * Rk[e]);
            const float *Aj = Ak + j * T;
            for (int wd = 0; wd < 2; ++wd)
                for (uint32_t bits = ancs[2 * j + wd]; bits; bits &= bits - 1) {
                    const int l = (wd << 5) + __ffs(bits) - 1;
                    if (l != j) u = fmaf(-Aj[l], U[l * kRows + row], u);
                }
            U[e] = u;
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- 6. outputs
    for (int e = tid; e < T * kRows; e += kThreadsG) {
        const int i = e / kRows, row = e - i * kRows;
        float acc = eg[i] * Rq[e];
        const float *Mi = Mq + i * T;
        for (int wd = 0; wd < 2; ++wd)
            for (uint32_t bits = ancs[2 * i + wd]; bits; bits &= bits - 1) {
                const int j = (wd << 5) + __ffs(bits) - 1;
                acc = fmaf(Mi[j], U[j * kRows + row], acc);
            }
        os[e] = f_to_in<In>(acc);
    }

    // ---------------------------------------------------------------- 7. commit (root group)
    if (!tree_warp && misc[G_COMMIT]) {
        const int len = misc[G_LEN];
        const float gl = len > 0 ? eg[pnode[len - 1]] : 1.f;
        float4 acc[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r] = make_float4(gl * hv[r].x, gl * hv[r].y, gl * hv[r].z, gl * hv[r].w);
        for (int q = 0; q < len; ++q) {
            const int j = pnode[q];
            const float4 kq = row4(ks, j, lane);
            const float w = wq[q];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float cf = w * U[j * kRows + 8 * warp + r];
                acc[r].x = fmaf(cf, kq.x, acc[r].x);
                acc[r].y = fmaf(cf, kq.y, acc[r].y);
                acc[r].z = fmaf(cf, kq.z, acc[r].z);
                acc[r].w = fmaf(cf, kq.w, acc[r].w);
            }
        }
        float *sn = p.S_new + (((size_t)b * Hv + h) * dv + p0 + 8 * warp) * kK + 4 * lane;
#pragma unroll
        for (int r = 0; r < 8; ++r) __stcs(reinterpret_cast<float4 *>(sn + r * kK), acc[r]);
    }

    // ---------------------------------------------------------------- 8. outputs to HBM
    __syncthreads();
    constexpr int kEl16 = 16 / (int)sizeof(In), kOChunks = kRows / kEl16;
    In *Og = static_cast<In *>(p.o) + ((size_t)b * T * Hv + h) * dv + p0;
    for (int e = tid; e < T * kOChunks; e += kThreadsG) {
        const int i = e / kOChunks, c = e % kOChunks;
        *reinterpret_cast<uint4 *>(Og + (size_t)i * vrow + c * kEl16) =
            *reinterpret_cast<const uint4 *>(os + i * kRows + c * kEl16);
    }
}

std::mutex g_gdn_mutex;
bool g_gdn_prepared[kMaxDevices] = {};

cudaError_t prepare_gdn()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_gdn_mutex);
    if (g_gdn_prepared[dev]) return cudaSuccess;
    const int most = (int)GdnLayout(kMaxGdnNodes, 4).total;
    if ((e = cudaFuncSetAttribute(gdn_tree_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, most)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(gdn_tree_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  most)) != cudaSuccess)
        return e;
    g_gdn_prepared[dev] = true;
    return cudaSuccess;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace stree

using namespace stree;

extern "C" stree_status stree_gdn_tree_scan_commit(const void *q, const void *k, const void *v, const float *alpha,
                                                   const float *beta, const float *erase, const float *S0,
                                                   const int32_t *parent,
                                                   int n_nodes, int batch, int heads_v, int heads_k, int dk, int dv,
                                                   stree_dtype dtype, const int32_t *accepted_path,
                                                   const int32_t *path_len, int maxlen, void *o, float *S_new,
                                                   int32_t *err_out, void *stream)
{
    if (batch < 0 || n_nodes < 1 || heads_v < 1 || heads_k < 1 || dk < 1 || dv < 1) return STREE_ERR_UNSUPPORTED;
    if (n_nodes > kMaxGdnNodes || dk != kK || dv % kRows != 0 || dv > kMaxDim || heads_v % heads_k != 0)
        return STREE_ERR_UNSUPPORTED;
    if (dtype != STREE_F32 && dtype != STREE_BF16) return STREE_ERR_UNSUPPORTED;
    const bool commit = accepted_path != nullptr || path_len != nullptr || S_new != nullptr;
    if (batch == 0) return (!commit || maxlen >= 0) ? STREE_OK : STREE_ERR_INVALID_ARG;
    if (!q || !k || !v || !alpha || !beta || !S0 || !parent || !o) return STREE_ERR_INVALID_ARG;
    if (commit && (!accepted_path || !path_len || !S_new || maxlen < 1)) return STREE_ERR_INVALID_ARG;
    const void *ptrs16[] = {q, k, v, S0, o};
    for (const void *ptr : ptrs16)
        if (!aligned(ptr, 16)) return STREE_ERR_MISALIGNED;
    if (commit && !aligned(S_new, 16)) return STREE_ERR_MISALIGNED;
    if (!aligned(alpha, 4) || !aligned(beta, 4) || !aligned(erase, 4) || !aligned(parent, 4) || !aligned(err_out, 4) ||
        (commit && (!aligned(accepted_path, 4) || !aligned(path_len, 4))))
        return STREE_ERR_MISALIGNED;
    const long long grid = (long long)batch * heads_v * (dv / kRows);
    if (grid > 0x7fffffffLL) return STREE_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *err = err_out;
    // The tensor-core kernel: one CTA per (sequence, value head); its state rows and
    // node positions are 32-bit TMA coordinates.
    if (gdn_tc_supported(n_nodes, dk, dv, dtype) && (long long)batch * heads_v * dv <= 0x7fffffffLL &&
        (long long)batch * n_nodes <= 0x7fffffffLL) {
        if (err && cudaMemsetAsync(err, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return STREE_ERR_CUDA;
        return launch_gdn_tc(q, k, v, alpha, beta, erase, S0, parent, n_nodes, batch, heads_v, heads_k,
                             commit ? accepted_path : nullptr, commit ? path_len : nullptr, commit ? maxlen : 0, o,
                             commit ? S_new : nullptr, err, s) == cudaSuccess
                   ? STREE_OK
                   : STREE_ERR_CUDA;
    }
    if (prepare_gdn() != cudaSuccess) return STREE_ERR_CUDA;
    if (err && cudaMemsetAsync(err, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return STREE_ERR_CUDA;
    GdnParams p{};
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta; p.erase = erase; p.S0 = S0;
    p.parent = parent;
    p.path = commit ? accepted_path : nullptr;
    p.path_len = commit ? path_len : nullptr;
    p.maxlen = commit ? maxlen : 0;
    p.o = o;
    p.S_new = commit ? S_new : nullptr;
    p.err = err;
    p.T = n_nodes; p.Hv = heads_v; p.Hk = heads_k; p.dv = dv;
    p.slices = dv / kRows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreadsG);
    cfg.dynamicSmemBytes = GdnLayout(n_nodes, dtype == STREE_BF16 ? 2 : 4).total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = dtype == STREE_BF16 ? cudaLaunchKernelEx(&cfg, gdn_tree_kernel<__nv_bfloat16>, p)
                                        : cudaLaunchKernelEx(&cfg, gdn_tree_kernel<float>, p);
    return e == cudaSuccess ? STREE_OK : STREE_ERR_CUDA;
}
