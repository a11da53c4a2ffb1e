// k_scan_tc.cu -- tensor-core (tcgen05) packed tree scan with fused commit, sm_100a.
//
// Method ("STree: Speculative Tree Decoding for Hybrid State Space Models",
// scime.ai summary, "Approach"): every node's exact per-path output comes from
// one scan over the packed tree with the accumulated transition A_tree = L.logA,
// and the accepted path's state is rebuilt by activation replay:
//   L_i   = A_h * sum_{j in anc(i)} dt_j
//   y_i   = exp(L_i) (h0 . C_i) + sum_{j in anc(i)} exp(L_i - L_j) cb_ij dt_j x_j + D_h x_i
//   h_new = exp(L_leaf) h0 + sum_{j on path} exp(L_leaf - L_j) dt_j x_j (outer) B_j
//
// Design (B200): the state h0 [b, H*P, N] is streamed through the SMs in tiles of
// RB rows of the flattened (head, headdim) axis.  Per tile:
//   * TMA brings the fp32 h0 tile (128-byte swizzled, 4 boxes of 32 columns) and
//     the bf16 x tile [T nodes x RB] into a double-buffered stage;
//   * one thread issues tcgen05.mma kind::tf32 (M = 128, N = T_pad, K = 128):
//     R[row, i] = h0[row, :] . C_i[:] into tensor memory -- the root term, the
//     only dense contraction of the path (C is staged once per sequence/group);
//   * the commit (fp32 FMA, exact h0) is written in place over the h0 tile and
//     the outputs y in place over the x tile; TMA stores both back;
//   * the sparse tree term runs on the CUDA cores over the ancestor pairs only
//     (lanes of a warp share a head: each lane builds one pair's decayed weight
//     and the warp broadcasts them), so exp never sees a positive argument.
// The load of tile k+1 and the stores of tile k-1 overlap the work on tile k.
// Only the tf32 rounding of h0 inside the root-term MMA departs from fp32
// arithmetic; it is below the bf16 rounding of the output y.
#include <cuda.h>

#include <mutex>

#include "stree_internal.cuh"
#include "tc_ptx.cuh"

namespace stree {
namespace {

constexpr int kThreads = 128;
constexpr int kDstate = 128;               // dstate of the tensor-core path
constexpr int kMaxTcNodes = 128;           // T_pad <= 128 (TMEM columns, smem)
constexpr size_t kSmemLimit = 232448;      // 227 KB opt-in dynamic shared memory

enum Misc { M_TMEM = 0, M_ABORT, M_LEN, M_STATE, M_INSMEM, M_TOTAL, kMiscWords = 8 };

struct TcParams {
    const __nv_bfloat16 *dt, *B, *C;
    const float *A, *D;
    const int32_t *path, *path_len;
    const float *cb;
    TreeView tree;
    int32_t *err;
    int T, T_pad, H, P, G, RB, tps, ntiles, maxlen, do_commit, hpt, pair_cap;
    uint32_t tmem_cols;
    uint32_t off_x, x_stage, off_c, off_anc, off_poff, off_dts, off_L, off_eL, off_w, off_alpha, off_pnode,
        off_bar, off_misc, off_pcb, off_pj;
};

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ int nth_set_bit(const uint32_t *row, int W, int n)
{
    for (int w = 0; w < W; ++w) {
        int c = __popc(row[w]);
        if (n < c) return (w << 5) + __fns(row[w], 0, n + 1);
        n -= c;
    }
    return -1;
}

__global__ void __launch_bounds__(kThreads, 1)
scan_tc_kernel(const __grid_constant__ CUtensorMap tm_h0, const __grid_constant__ CUtensorMap tm_hn,
               const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
               const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.T, RB = p.RB, P = p.P, H = p.H, G = p.G, W = p.tree.W, HP = H * P;
    const int hpg = H / G;

    uint8_t *h0s = smem;                                            // 2 x [4 atoms][RB rows][128 B]
    uint8_t *xs = smem + p.off_x;                                   // 2 x [T][RB] bf16
    uint8_t *cs = smem + p.off_c;                                   // [4 atoms][T_pad rows][128 B]
    uint32_t *ancs = reinterpret_cast<uint32_t *>(smem + p.off_anc);  // [T][W]
    int32_t *poff = reinterpret_cast<int32_t *>(smem + p.off_poff);   // [T+1]
    float *dts = reinterpret_cast<float *>(smem + p.off_dts);         // [hpt][T]
    float *Ls = reinterpret_cast<float *>(smem + p.off_L);            // [hpt][T]
    float *eLs = reinterpret_cast<float *>(smem + p.off_eL);          // [hpt][T]
    float *wts = reinterpret_cast<float *>(smem + p.off_w);           // [hpt][T]
    float *alpha = reinterpret_cast<float *>(smem + p.off_alpha);     // [hpt]
    int16_t *pnode = reinterpret_cast<int16_t *>(smem + p.off_pnode); // [T]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + p.off_bar);  // full[2], mma
    int32_t *misc = reinterpret_cast<int32_t *>(smem + p.off_misc);
    float *pcb = reinterpret_cast<float *>(smem + p.off_pcb);         // [pair_cap]
    uint8_t *pj = smem + p.off_pj;                                    // [pair_cap]

    const uint32_t bar_full0 = ptx::smem_u32(&bars[0]);
    const uint32_t bar_mma = ptx::smem_u32(&bars[2]);
    const uint32_t h0_stage_bytes = (uint32_t)RB * 512u;
    const uint32_t tx_bytes = h0_stage_bytes + (uint32_t)T * RB * 2u;
    const uint32_t idesc = ptx::idesc_tf32(128, p.T_pad);

    if (tid == 0) {
        ptx::prefetch_tensormap(&tm_h0);
        ptx::prefetch_tensormap(&tm_x);
        ptx::prefetch_tensormap(&tm_hn);
        ptx::prefetch_tensormap(&tm_y);
        ptx::mbar_init(bar_full0, 1);
        ptx::mbar_init(bar_full0 + 8, 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::fence_mbar_init();
        for (int k = 0; k < kMiscWords; ++k) misc[k] = 0;
    }
    // Rows the MMA reads past an RB-row atom alias the next atom or the x
    // region; give every byte a defined value once.
    for (uint32_t o = tid * 16u; o < p.off_c; o += kThreads * 16u)
        *reinterpret_cast<float4 *>(smem + o) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(&misc[M_TMEM]), p.tmem_cols);
        ptx::tmem_relinquish();
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = static_cast<uint32_t>(misc[M_TMEM]);

    const int start = (int)((long long)blockIdx.x * p.ntiles / gridDim.x);
    const int end = (int)((long long)(blockIdx.x + 1) * p.ntiles / gridDim.x);
    auto tile_ok = [&](int t) { return __ldg(&p.tree.ok[t / p.tps]) != 0; };
    auto next_valid = [&](int t) {
        while (t < end && !tile_ok(t)) ++t;
        return t;
    };
    auto issue_load = [&](int t, int stage) {
        const int b = t / p.tps, r0 = (t % p.tps) * RB;
        const uint32_t bar = bar_full0 + 8u * stage;
        ptx::mbar_expect_tx(bar, tx_bytes);
        const uint32_t dst = ptx::smem_u32(h0s + stage * h0_stage_bytes);
        for (int kb = 0; kb < 4; ++kb)
            ptx::tma_load_2d(dst + kb * RB * 128, &tm_h0, kb * 32, b * HP + r0, bar);
        ptx::tma_load_2d(ptx::smem_u32(xs + stage * p.x_stage), &tm_x, r0, b * T, bar);
    };

    int t = next_valid(start);
    if (tid == 0 && t < end) issue_load(t, 0);
    int cur_key = -1, cur_b = -1;
    uint32_t k = 0;
    bool pending_load = (t < end);

    while (t < end) {
        const int b = t / p.tps, r0 = (t % p.tps) * RB;
        const int hfirst = r0 / P;
        const int g = hfirst / hpg;
        const int key = b * G + g;
        const int stage = k & 1;

        // ---------------------------------------------------- per (sequence, group)
        if (key != cur_key) {
            if (b != cur_b) {
                for (int q = tid; q < T * W; q += kThreads) ancs[q] = __ldg(&p.tree.anc[(size_t)b * T * W + q]);
                __syncthreads();
                if (tid == 0) {
                    int len = 0, state = 0;
                    if (p.do_commit) {
                        len = __ldg(&p.path_len[b]);
                        state = 1;
                        if (len < 0 || len > p.maxlen || len > T) {
                            state = 0;
                            latch_error(p.err, STREE_ERR_BAD_PATH, b, -1, len);
                        } else if (len > 0) {
                            const int32_t *pb = p.path + (size_t)b * p.maxlen;
                            const int leaf = __ldg(&pb[len - 1]);
                            if (leaf < 0 || leaf >= T || __ldg(&p.tree.depth[(size_t)b * T + leaf]) != len - 1) {
                                state = 0;
                                latch_error(p.err, STREE_ERR_BAD_PATH, b, len - 1, leaf);
                            } else {
                                for (int q = 0; q < len; ++q) {
                                    const int j = __ldg(&pb[q]);
                                    const bool good = j >= 0 && j < T && ((ancs[leaf * W + (j >> 5)] >> (j & 31)) & 1u) &&
                                                      __ldg(&p.tree.depth[(size_t)b * T + j]) == q;
                                    if (!good) {
                                        state = 0;
                                        latch_error(p.err, STREE_ERR_BAD_PATH, b, q, j);
                                        break;
                                    }
                                    pnode[q] = (int16_t)j;
                                }
                            }
                        }
                    }
                    misc[M_LEN] = len;
                    misc[M_STATE] = state;
                    int acc = 0;
                    for (int i = 0; i < T; ++i) {
                        poff[i] = acc;
                        for (int w = 0; w < W; ++w) acc += __popc(ancs[i * W + w]);
                    }
                    poff[T] = acc;
                    misc[M_TOTAL] = acc;
                    misc[M_INSMEM] = acc <= p.pair_cap;
                }
                cur_b = b;
            }
            // C operand: rows i < T_pad, fp32 in the 128-byte swizzled K-major layout.
            for (int q = tid; q < p.T_pad * 32; q += kThreads) {
                const int i = q >> 5, c = q & 31;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < T) {
                    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p.C + (((size_t)b * T + i) * G + g) * kDstate + c * 4));
                    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
                    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
                    v = make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
                }
                const int kb = c >> 3, ch = c & 7;
                *reinterpret_cast<float4 *>(cs + kb * p.T_pad * 128 + i * 128 + ((ch ^ (i & 7)) << 4)) = v;
            }
            __syncthreads();
            if (misc[M_INSMEM]) {
                const int total = misc[M_TOTAL];
                const float *cbg = p.cb + ((size_t)b * G + g) * T * T;
                for (int q = tid; q < total; q += kThreads) {
                    int lo = 0, hi = T;                   // poff[lo] <= q < poff[hi]
                    while (hi - lo > 1) {
                        const int mid = (lo + hi) >> 1;
                        if (poff[mid] <= q) lo = mid; else hi = mid;
                    }
                    const int j = nth_set_bit(ancs + lo * W, W, q - poff[lo]);
                    pj[q] = (uint8_t)j;
                    pcb[q] = __ldg(&cbg[(size_t)lo * T + j]);
                }
            }
            ptx::fence_proxy_async_smem();
            __syncthreads();
            cur_key = key;
        }

        const int nt = next_valid(t + 1);

        // ---------------------------------------------------- MMA + prefetch (one thread)
        if (tid == 0) {
            if (!ptx::mbar_wait(bar_full0 + 8u * stage, (k >> 1) & 1)) {
                latch_error(p.err, STREE_ERR_TIMEOUT, b, r0, 1);
                misc[M_ABORT] = 1;
            } else {
                pending_load = false;
                ptx::tc_fence_after();
                const uint32_t a0 = ptx::smem_u32(h0s + stage * h0_stage_bytes);
                const uint32_t b0 = ptx::smem_u32(cs);
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        ptx::mma_tf32(tmem, ptx::desc_kmajor_sw128(a0 + kb * RB * 128 + kk * 32),
                                      ptx::desc_kmajor_sw128(b0 + kb * p.T_pad * 128 + kk * 32), idesc,
                                      (kb | kk) != 0);
                ptx::mma_commit(bar_mma);
                if (nt < end) {
                    ptx::bulk_wait_read_all();            // tile k-1's stores have left the other stage
                    issue_load(nt, stage ^ 1);
                    pending_load = true;
                }
            }
        }

        // ---------------------------------------------------- per-tile coefficients
        const int hpt = p.hpt;
        const int len = misc[M_LEN];
        const bool commit = p.do_commit && misc[M_STATE];
        for (int q = tid; q < hpt * T; q += kThreads) {
            const int hh = q / T, i = q - hh * T;
            dts[q] = bf2f(p.dt[((size_t)b * T + i) * H + hfirst + hh]);
        }
        __syncthreads();
        for (int q = tid; q < hpt * T; q += kThreads) {
            const int hh = q / T, i = q - hh * T;
            float s = 0.f;
            for (int w = 0; w < W; ++w) {
                uint32_t bits = ancs[i * W + w];
                while (bits) {
                    const int j = (w << 5) + __ffs(bits) - 1;
                    bits &= bits - 1;
                    s += dts[hh * T + j];
                }
            }
            const float L = __ldg(&p.A[hfirst + hh]) * s;
            Ls[q] = L;
            eLs[q] = expf(L);
        }
        __syncthreads();
        if (commit) {
            const int leaf = len > 0 ? pnode[len - 1] : 0;
            for (int q = tid; q < hpt * len; q += kThreads) {
                const int hh = q / len, kk = q - hh * len;
                const int j = pnode[kk];
                wts[hh * T + kk] = expf(Ls[hh * T + leaf] - Ls[hh * T + j]) * dts[hh * T + j];
            }
            if (tid < hpt) alpha[tid] = len > 0 ? eLs[tid * T + leaf] : 1.f;
        }

        // ---------------------------------------------------- wait for the MMA
        if (!misc[M_ABORT]) {
            if (!ptx::mbar_wait(bar_mma, k & 1)) {
                latch_error(p.err, STREE_ERR_TIMEOUT, b, r0, 2);
                misc[M_ABORT] = 1;
            }
        }
        __syncthreads();
        if (misc[M_ABORT]) break;
        ptx::tc_fence_after();

        uint8_t *h0t = h0s + stage * h0_stage_bytes;
        __nv_bfloat16 *xt = reinterpret_cast<__nv_bfloat16 *>(xs + stage * p.x_stage);

        // ---------------------------------------------------- commit, in place over h0
        if (commit) {
            const int row = tid % RB, seg = tid / RB;     // RB columns per thread
            const int hh = (r0 + row) / P - hfirst;
            const float al = alpha[hh];
            const float *wh = wts + hh * T;
            for (int c4 = 0; c4 < RB / 4; ++c4) {
                const int n = seg * RB + c4 * 4;
                const int kb = n >> 5, ch = (n & 31) >> 2;
                float4 *ptr = reinterpret_cast<float4 *>(h0t + kb * RB * 128 + row * 128 + ((ch ^ (row & 7)) << 4));
                float4 v = *ptr;
                v.x *= al; v.y *= al; v.z *= al; v.w *= al;
                for (int q = 0; q < len; ++q) {
                    const int j = pnode[q];
                    const float coef = wh[q] * bf2f(xt[j * RB + row]);
                    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p.B + (((size_t)b * T + j) * G + g) * kDstate + n));
                    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
                    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
                    v.x = fmaf(coef, __low2float(lo), v.x);
                    v.y = fmaf(coef, __high2float(lo), v.y);
                    v.z = fmaf(coef, __low2float(hi), v.z);
                    v.w = fmaf(coef, __high2float(hi), v.w);
                }
                *ptr = v;
            }
        }
        __syncthreads();                                   // x rows of the path are read

        // ---------------------------------------------------- y, in place over x
        if (warp < RB / 32) {
            const int row = warp * 32 + lane;
            const int hh = (r0 + row) / P - hfirst;       // same for the whole warp (P >= 32)
            const float Dh = __ldg(&p.D[hfirst + hh]);
            const float *Lh = Ls + hh * T, *eLh = eLs + hh * T, *dth = dts + hh * T;
            const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
            const bool insmem = misc[M_INSMEM] != 0;
            const float *cbg = p.cb + ((size_t)b * G + g) * T * T;
            __nv_bfloat16 *xc = xt + row;
            for (int c0 = ((T - 1) >> 4) << 4; c0 >= 0; c0 -= 16) {
                float v[16];
                ptx::tmem_ld16(tl + (uint32_t)c0, v);
#pragma unroll
                for (int u = 15; u >= 0; --u) {
                    const int i = c0 + u;
                    if (i < T) {
                        const float Li = Lh[i];
                        float tree = 0.f;
                        const int q0 = poff[i], cnt = poff[i + 1] - q0;
                        for (int base = 0; base < cnt; base += 32) {
                            int jl = 0;
                            float ml = 0.f;
                            if (base + lane < cnt) {
                                float cbv;
                                if (insmem) {
                                    jl = pj[q0 + base + lane];
                                    cbv = pcb[q0 + base + lane];
                                } else {
                                    jl = nth_set_bit(ancs + i * W, W, base + lane);
                                    cbv = __ldg(&cbg[(size_t)i * T + jl]);
                                }
                                ml = expf(Li - Lh[jl]) * cbv * dth[jl];
                            }
                            const int nn = min(32, cnt - base);
                            for (int s = 0; s < nn; ++s) {
                                const float ms = __shfl_sync(0xffffffffu, ml, s);
                                const int js = __shfl_sync(0xffffffffu, jl, s);
                                tree = fmaf(ms, bf2f(xc[js * RB]), tree);
                            }
                        }
                        const float yv = eLh[i] * v[u] + tree + Dh * bf2f(xc[i * RB]);
                        xc[i * RB] = __float2bfloat16_rn(yv);
                    }
                }
            }
        }
        ptx::tc_fence_before();
        ptx::fence_proxy_async_smem();
        __syncthreads();

        // ---------------------------------------------------- stores (one thread)
        if (tid == 0) {
            ptx::tma_store_2d(&tm_y, r0, b * T, ptx::smem_u32(xt));
            if (commit) {
                const uint32_t src = ptx::smem_u32(h0t);
                for (int kb = 0; kb < 4; ++kb)
                    ptx::tma_store_2d(&tm_hn, kb * 32, b * HP + r0, src + kb * RB * 128);
            }
            ptx::bulk_commit();
        }
        ++k;
        t = nt;
    }

    if (tid == 0) {
        ptx::bulk_wait_all();
        if (misc[M_ABORT] && pending_load) {
            // A load may still land in this CTA's shared memory: give it a bounded wait.
            ptx::mbar_wait(bar_full0 + 8u * (k & 1), (k >> 1) & 1);
            ptx::mbar_wait(bar_full0 + 8u * ((k + 1) & 1), ((k + 1) >> 1) & 1);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, p.tmem_cols);
    }
}

// ------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

uint32_t round_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

struct TcPlan {
    TcParams p;
    size_t smem;
    int grid;
};

// Shared-memory layout for a tile height RB; returns false if it does not fit.
bool layout(const ScanArgs &a, int RB, TcParams &p, size_t &smem)
{
    const int T = a.T, T_pad = (T + 15) / 16 * 16, W = (T + 31) / 32;
    const int hpt = a.P >= RB ? 1 : RB / a.P;
    uint32_t off = 2u * RB * 512u;                            // h0 stages
    p.off_x = off;
    p.x_stage = round_up((uint32_t)T * RB * 2u, 1024u);
    uint32_t xreg = 2u * p.x_stage;
    const uint32_t spill = (uint32_t)(128 - RB) * 128u;      // MMA rows past the last h0 stage
    if (xreg < spill) xreg = spill;
    off = round_up(off + xreg, 1024u);
    p.off_c = off;
    off += (uint32_t)T_pad * 512u;
    p.off_anc = off;   off = round_up(off + (uint32_t)T * W * 4u, 16u);
    p.off_poff = off;  off = round_up(off + (uint32_t)(T + 1) * 4u, 16u);
    p.off_dts = off;   off = round_up(off + (uint32_t)hpt * T * 4u, 16u);
    p.off_L = off;     off = round_up(off + (uint32_t)hpt * T * 4u, 16u);
    p.off_eL = off;    off = round_up(off + (uint32_t)hpt * T * 4u, 16u);
    p.off_w = off;     off = round_up(off + (uint32_t)hpt * T * 4u, 16u);
    p.off_alpha = off; off = round_up(off + (uint32_t)hpt * 4u, 16u);
    p.off_pnode = off; off = round_up(off + (uint32_t)T * 2u, 16u);
    p.off_bar = off;   off = round_up(off + 3u * 8u, 16u);
    p.off_misc = off;  off = round_up(off + kMiscWords * 4u, 16u);
    p.off_pcb = off;
    const size_t fixed = (size_t)off + 1024;                  // + alignment slack of the dynamic base
    if (fixed + 5 * 64 > kSmemLimit) return false;
    const int all_pairs = T * (T + 1) / 2;
    int cap = (int)((kSmemLimit - fixed) / 5);
    if (cap > all_pairs) cap = all_pairs;
    p.pair_cap = cap;
    p.off_pj = round_up(p.off_pcb + (uint32_t)cap * 4u, 16u);
    smem = (size_t)p.off_pj + cap + 1024;
    smem = (smem + 15) / 16 * 16;
    if (smem > kSmemLimit) return false;
    p.T = T;
    p.T_pad = T_pad;
    p.RB = RB;
    p.hpt = hpt;
    uint32_t cols = 32;
    while (cols < (uint32_t)T_pad) cols <<= 1;
    p.tmem_cols = cols;
    return true;
}

bool rb_valid(const ScanArgs &a, int RB)
{
    const int HP = a.H * a.P, hpg = a.H / a.G;
    if (HP % RB != 0) return false;
    if (a.P >= RB) return a.P % RB == 0;
    return RB % a.P == 0 && hpg % (RB / a.P) == 0;
}

bool plan(const ScanArgs &a, TcPlan &pl)
{
    if (a.dtype != STREE_BF16 || a.N != kDstate || a.T > kMaxTcNodes || a.P % 32 != 0) return false;
    if (a.batch <= 0 || a.H % a.G != 0) return false;
    if (!encode_fn()) return false;
    const int sms = num_sms();
    int chosen = -1;
    TcParams best{};
    size_t best_smem = 0;
    for (int RB : {128, 64, 32}) {
        TcParams p{};
        size_t smem = 0;
        if (!rb_valid(a, RB) || !layout(a, RB, p, smem)) continue;
        const long long ntiles = (long long)a.batch * (a.H * a.P / RB);
        if (ntiles > 0x7fffffff) continue;
        chosen = RB;
        best = p;
        best_smem = smem;
        if (ntiles >= sms) break;                  // largest tile that still fills the GPU
    }
    if (chosen < 0) return false;
    best.H = a.H;
    best.P = a.P;
    best.G = a.G;
    best.tps = a.H * a.P / chosen;
    best.ntiles = a.batch * best.tps;
    pl.p = best;
    pl.smem = best_smem;
    return true;
}

}  // namespace

bool tc_supported(const ScanArgs &a)
{
    TcPlan pl;
    return plan(a, pl);
}

cudaError_t launch_scan_tc(const ScanArgs &a, cudaStream_t s)
{
    TcPlan pl;
    if (!plan(a, pl)) return cudaErrorNotSupported;
    TcParams p = pl.p;
    p.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    p.B = static_cast<const __nv_bfloat16 *>(a.B);
    p.C = static_cast<const __nv_bfloat16 *>(a.C);
    p.A = a.A;
    p.D = a.D;
    p.path = a.path;
    p.path_len = a.path_len;
    p.maxlen = a.maxlen;
    p.do_commit = a.path != nullptr && a.h_new != nullptr;
    p.cb = a.cb;
    p.tree = a.tree;
    p.err = a.err;

    EncodeTiledFn enc = encode_fn();
    const int HP = a.H * a.P;
    CUtensorMap m_h0, m_hn, m_x, m_y;
    {
        cuuint64_t dims[2] = {(cuuint64_t)kDstate, (cuuint64_t)a.batch * HP};
        cuuint64_t strides[1] = {(cuuint64_t)kDstate * 4};
        cuuint32_t box[2] = {32, (cuuint32_t)p.RB};
        cuuint32_t es[2] = {1, 1};
        if (enc(&m_h0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(a.h0), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        float *hn = p.do_commit ? a.h_new : const_cast<float *>(a.h0);
        if (enc(&m_hn, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, hn, dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)HP, (cuuint64_t)a.batch * a.T};
        cuuint64_t strides[1] = {(cuuint64_t)HP * 2};
        cuuint32_t box[2] = {(cuuint32_t)p.RB, (cuuint32_t)a.T};
        cuuint32_t es[2] = {1, 1};
        if (enc(&m_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.x), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        if (enc(&m_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.y, dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
    if (e != cudaSuccess) return e;
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, scan_tc_kernel, kThreads, pl.smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    // Tensor memory: every resident CTA holds tmem_cols of the SM's 512 columns.
    const int tmem_fit = 512 / (int)p.tmem_cols;
    if (per_sm > tmem_fit) per_sm = tmem_fit;
    long long grid = (long long)num_sms() * per_sm;
    if (grid > p.ntiles) grid = p.ntiles;
    scan_tc_kernel<<<(unsigned)grid, kThreads, pl.smem, s>>>(m_h0, m_hn, m_x, m_y, p);
    return cudaGetLastError();
}

}  // namespace stree
