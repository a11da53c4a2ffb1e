// k_scan_tc.cu -- tensor-core (tcgen05) packed tree scan with fused commit, sm_100a.
//
// Method ("STree: Speculative Tree Decoding for Hybrid State Space Models",
// scime.ai summary, "Approach"): every node's exact per-path output comes from
// one scan over the packed tree with the accumulated transition A_tree = L.logA,
// and the accepted path's state is rebuilt by activation replay:
//   L_i   = A_h * sum_{j in anc(i)} dt_j
//   y_i   = exp(L_i) (h0 . C_i) + sum_{j in anc(i)} exp(L_i - L_j) (C_i . B_j) dt_j x_j + D_h x_i
//   h_new = exp(L_leaf) h0 + sum_{j on path} exp(L_leaf - L_j) dt_j x_j (outer) B_j
//
// Design (B200).  The state h0 [b, H*P, N=128] streams through the SMs in tiles
// of RB rows of the flattened (head, headdim) axis; a persistent CTA walks a
// contiguous range of tiles with warp-specialised roles joined by mbarriers:
//   * producer warp: TMA loads of the fp32 h0 tile (128-byte swizzled, 4 boxes
//     of 32 columns), the bf16 x tile (64-column swizzled boxes) and the dt box
//     into a 2-stage ring;
//   * MMA warp (one thread): the root term R[row, i] = h0[row, :] . C_i as
//     tcgen05.mma kind::tf32 (M = 128, N = T_pad, K = 128) and the tree term
//     Y[row, i] = sum_j x[j, row] M_h[i, j] as kind::f16 with x as an MN-major
//     operand straight from the stage, into a 2-deep tensor-memory ring;
//   * prep warps: per tile and head the tree cumsum L, exp(L) and the masked
//     decay matrix M_h[i][j] = exp(L_i - L_j) (C_i . B_j) dt_j over ancestor
//     pairs only (bf16, K-major swizzled), plus the commit weights;
//   * epilogue warps: the commit in exact fp32 FMA, written in place over the
//     h0 tile, then y = exp(L_i) R + Y + D x in place over the x tile, then TMA
//     stores of both and the release of the stage.
// C (fp32 operand of the root MMA), the ancestor pairs' C.B and the accepted
// path's rows of B are staged once per (sequence, group).  Roles only block on
// bounded mbarrier waits; a timeout latches STREE_ERR_TIMEOUT and the CTA runs
// to its end without further work.  Precision: the root term rounds h0 to tf32
// and the masked decay matrix to bf16 inside the MMAs (fp32 accumulation); the
// commit and every other step are fp32.
#include <cuda.h>

#include <mutex>

#include "stree_internal.cuh"
#include "tc_ptx.cuh"

namespace stree {
namespace {

constexpr int kDstate = 128;               // dstate of the tensor-core path
constexpr int kMaxTcNodes = 128;           // T_pad <= 128 (TMEM columns, smem)
constexpr int kPathRows = 8;               // accepted-path rows of B staged in smem (fp32)
constexpr size_t kSmemLimit = 232448;      // 227 KB opt-in dynamic shared memory

constexpr int kProducerWarp = 0, kMmaWarp = 1, kPrepWarp0 = 2, kPrepWarps = 4, kEpiWarp0 = 6, kEpiWarps = 8;
constexpr int kMaxStages = 3;
constexpr int kMaxSmemHeads = 1024;        // A and D are staged in shared memory
constexpr int kWarps = kEpiWarp0 + kEpiWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kPrepThreads = kPrepWarps * 32, kEpiThreads = kEpiWarps * 32;
constexpr int kBarEpi = 1, kBarPrep = 2;   // named barriers (0 is __syncthreads)

enum Misc { M_TMEM = 0, M_ABORT, M_LEN, M_STATE, M_INSMEM, M_TOTAL, M_SDESC = 8, M_WSUM = 8 + 2 * kMaxStages,
            kMiscWords = M_WSUM + kWarps };
// mbarriers: TMA stage full / epilogue done with a stage (ring of S), tensor-memory
// accumulator full / empty (ring of 2), masked-decay matrix full / empty, and
// per-tile coefficients full / empty (ring of 2).
enum Bars { B_FULL = 0, B_EPID = kMaxStages, B_ACCF = 2 * kMaxStages, B_ACCE = B_ACCF + 2, B_MHF = B_ACCE + 2,
            B_MHE = B_MHF + 1, B_COEFF = B_MHE + 1, B_COEFE = B_COEFF + 2, kNumBars = B_COEFE + 2 };

struct TcParams {
    const __nv_bfloat16 *__restrict__ dt;
    const __nv_bfloat16 *__restrict__ B;
    const __nv_bfloat16 *__restrict__ C;
    const float *__restrict__ A;
    const float *__restrict__ D;
    const int32_t *__restrict__ path;
    const int32_t *__restrict__ path_len;
    TreeView tree;
    int32_t *err;
    int T, T_pad, KA, H, P, G, RB, NB, S, tps, ntiles, maxlen, do_commit, hpt, pair_cap, acc_cols;
    uint32_t tmem_cols;
    uint32_t off_x, x_stage, off_c, off_mh, mh_head, off_bp, off_anc, off_poff, off_coef, coef_slot,
        off_pnode, off_bar, off_misc, off_ad, off_pcb, off_pj, off_pi;
};

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ void unpack4(uint2 raw, float &a, float &b, float &c, float &d)
{
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    a = __low2float(lo);
    b = __high2float(lo);
    c = __low2float(hi);
    d = __high2float(hi);
}

__device__ __forceinline__ int nth_set_bit(const uint32_t *row, int W, int n)
{
    for (int w = 0; w < W; ++w) {
        int c = __popc(row[w]);
        if (n < c) return (w << 5) + __fns(row[w], 0, n + 1);
        n -= c;
    }
    return -1;
}

// Index i with poff[i] <= q < poff[i+1] (poff non-decreasing, poff[0] = 0).
__device__ __forceinline__ int pair_row(const int32_t *poff, int T, int q)
{
    int lo = 0, hi = T;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (poff[mid] <= q) lo = mid; else hi = mid;
    }
    return lo;
}

// C_i . B_j: C from the staged fp32 MMA operand (swizzled), B_j from global memory.
__device__ __forceinline__ float dot_cb(const uint8_t *cs, int T_pad, const __nv_bfloat16 *Bj, int i)
{
    float acc = 0.f;
    const uint8_t *crow = cs + i * 128;
    const uint2 *brow = reinterpret_cast<const uint2 *>(Bj);
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
        const float4 cv = *reinterpret_cast<const float4 *>(crow + (c >> 3) * T_pad * 128 + (((c & 7) ^ (i & 7)) << 4));
        float b0, b1, b2, b3;
        unpack4(__ldg(brow + c), b0, b1, b2, b3);
        acc = fmaf(cv.x, b0, acc);
        acc = fmaf(cv.y, b1, acc);
        acc = fmaf(cv.z, b2, acc);
        acc = fmaf(cv.w, b3, acc);
    }
    return acc;
}

// C_i . B_j over the quarter `part` (32 of the 128 state columns); four lanes of
// a warp combine their parts with shuffles.
__device__ __forceinline__ float dot_cb_part(const uint8_t *cs, int T_pad, const __nv_bfloat16 *Bj, int i, int part)
{
    float acc = 0.f;
    const uint8_t *crow = cs + part * T_pad * 128 + i * 128;     // K-atom `part` holds columns 32*part..
    const uint2 *brow = reinterpret_cast<const uint2 *>(Bj) + part * 8;
    uint2 raw[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) raw[c] = __ldg(brow + c);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 cv = *reinterpret_cast<const float4 *>(crow + ((c ^ (i & 7)) << 4));
        float b0, b1, b2, b3;
        unpack4(raw[c], b0, b1, b2, b3);
        acc = fmaf(cv.x, b0, acc);
        acc = fmaf(cv.y, b1, acc);
        acc = fmaf(cv.z, b2, acc);
        acc = fmaf(cv.w, b3, acc);
    }
    return acc;
}

// Byte offset of bf16 element (row, k) in a K-major 128-byte swizzled operand of
// `rows` rows: 64 K-columns per atom, atoms rows*128 bytes apart.
__device__ __forceinline__ uint32_t k_off(int row, int kcol, int rows)
{
    return (uint32_t)(kcol >> 6) * (uint32_t)rows * 128u + (uint32_t)row * 128u +
           ((uint32_t)(((kcol & 63) >> 3) ^ (row & 7)) << 4) + (uint32_t)(kcol & 7) * 2u;
}

// Column `m` of an MN-major 128-byte swizzled bf16 stack (64 columns per block,
// blocks xbs bytes apart): element (k, m) sits at base + k*128 + ((chunk ^ (k&7)) << 4).
struct MnCol {
    uint32_t base, chunk;
    __device__ __forceinline__ MnCol(int m, uint32_t xbs)
        : base((uint32_t)(m >> 6) * xbs + (uint32_t)(m & 7) * 2u), chunk((uint32_t)((m & 63) >> 3)) {}
    __device__ __forceinline__ uint32_t at(int k) const
    {
        return base + (uint32_t)k * 128u + ((chunk ^ (uint32_t)(k & 7)) << 4);
    }
};

// Commit of one tile row segment: h_new = alpha h0 + sum_q coef_q B[pnode_q] (fp32),
// coef_q = w_q x[pnode_q][row].  The first kPathRows path rows of B come from shared
// memory (fp32, fully unrolled), later ones from global memory.
template <int CPT>
__device__ __forceinline__ void commit_rows(uint8_t *h0t, const uint8_t *xt, const MnCol &xc, const float *Bp,
                                            const __nv_bfloat16 *Bseq, size_t brow, const int16_t *pnode,
                                            const float *wh, float al, int len, int RB, int row, int c_lo)
{
    float acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[c] = 0.f;
    float cf[kPathRows];
#pragma unroll
    for (int q = 0; q < kPathRows; ++q) {
        // Only path positions q < len hold node indices; others address node 0.
        const int j = q < len ? (int)pnode[q] : 0;
        const float xv = bf2f(*reinterpret_cast<const __nv_bfloat16 *>(xt + xc.at(j)));
        cf[q] = q < len ? wh[q] * xv : 0.f;
    }
#pragma unroll
    for (int q = 0; q < kPathRows; ++q) {
        if (q < len) {
            const float4 *src = reinterpret_cast<const float4 *>(Bp + q * kDstate + c_lo);
#pragma unroll
            for (int c = 0; c < CPT / 4; ++c) {
                const float4 bv = src[c];
                acc[4 * c + 0] = fmaf(cf[q], bv.x, acc[4 * c + 0]);
                acc[4 * c + 1] = fmaf(cf[q], bv.y, acc[4 * c + 1]);
                acc[4 * c + 2] = fmaf(cf[q], bv.z, acc[4 * c + 2]);
                acc[4 * c + 3] = fmaf(cf[q], bv.w, acc[4 * c + 3]);
            }
        }
    }
    for (int q = kPathRows; q < len; ++q) {
        const int j = pnode[q];
        const float coef = wh[q] * bf2f(*reinterpret_cast<const __nv_bfloat16 *>(xt + xc.at(j)));
        const uint2 *src = reinterpret_cast<const uint2 *>(Bseq + (size_t)j * brow + c_lo);
#pragma unroll
        for (int c = 0; c < CPT / 4; ++c) {
            float b0, b1, b2, b3;
            unpack4(__ldg(src + c), b0, b1, b2, b3);
            acc[4 * c + 0] = fmaf(coef, b0, acc[4 * c + 0]);
            acc[4 * c + 1] = fmaf(coef, b1, acc[4 * c + 1]);
            acc[4 * c + 2] = fmaf(coef, b2, acc[4 * c + 2]);
            acc[4 * c + 3] = fmaf(coef, b3, acc[4 * c + 3]);
        }
    }
#pragma unroll
    for (int c0 = 0; c0 < CPT / 4; c0 += 4) {
        float4 h[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int n = c_lo + 4 * (c0 + c);
            const int kb = n >> 5, ch = (n & 31) >> 2;
            h[c] = *reinterpret_cast<const float4 *>(h0t + kb * RB * 128 + row * 128 + ((ch ^ (row & 7)) << 4));
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int n = c_lo + 4 * (c0 + c);
            const int kb = n >> 5, ch = (n & 31) >> 2;
            float4 v;
            v.x = fmaf(al, h[c].x, acc[4 * (c0 + c) + 0]);
            v.y = fmaf(al, h[c].y, acc[4 * (c0 + c) + 1]);
            v.z = fmaf(al, h[c].z, acc[4 * (c0 + c) + 2]);
            v.w = fmaf(al, h[c].w, acc[4 * (c0 + c) + 3]);
            *reinterpret_cast<float4 *>(h0t + kb * RB * 128 + row * 128 + ((ch ^ (row & 7)) << 4)) = v;
        }
    }
}

#ifdef STREE_TRACE
// Profiling builds only: wall-clock stamps of pipeline events for four CTAs.
__device__ unsigned long long g_trace[4 * 32 * 24];
__device__ __forceinline__ void trace_event(uint32_t k, int ev)
{
    const int slot = blockIdx.x == 0 ? 0 : blockIdx.x == 37 ? 1 : blockIdx.x == 74 ? 2 : blockIdx.x == 111 ? 3 : -1;
    if (slot >= 0 && k < 32) g_trace[(slot * 32 + k) * 24 + ev] = ptx::globaltimer();
}
#define STREE_TR(k, ev) trace_event((k), (ev))
#else
#define STREE_TR(k, ev) ((void)0)
#endif

// Eight 16-bit shared-memory loads issued back to back (addresses in the shared window).
__device__ __forceinline__ void lds_u16x8(const uint32_t (&a)[8], uint16_t (&v)[8])
{
    asm volatile(
        "ld.shared.u16 %0, [%8];\n\t"
        "ld.shared.u16 %1, [%9];\n\t"
        "ld.shared.u16 %2, [%10];\n\t"
        "ld.shared.u16 %3, [%11];\n\t"
        "ld.shared.u16 %4, [%12];\n\t"
        "ld.shared.u16 %5, [%13];\n\t"
        "ld.shared.u16 %6, [%14];\n\t"
        "ld.shared.u16 %7, [%15];"
        : "=h"(v[0]), "=h"(v[1]), "=h"(v[2]), "=h"(v[3]), "=h"(v[4]), "=h"(v[5]), "=h"(v[6]), "=h"(v[7])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7])
        : "memory");
}

__device__ __forceinline__ void lds_f32x8(const uint32_t (&a)[8], float (&v)[8])
{
    asm volatile(
        "ld.shared.f32 %0, [%8];\n\t"
        "ld.shared.f32 %1, [%9];\n\t"
        "ld.shared.f32 %2, [%10];\n\t"
        "ld.shared.f32 %3, [%11];\n\t"
        "ld.shared.f32 %4, [%12];\n\t"
        "ld.shared.f32 %5, [%13];\n\t"
        "ld.shared.f32 %6, [%14];\n\t"
        "ld.shared.f32 %7, [%15];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7])
        : "memory");
}

__device__ __forceinline__ void sts_u16x8(const uint32_t (&a)[8], const uint16_t (&v)[8])
{
    asm volatile(
        "st.shared.u16 [%0], %8;\n\t"
        "st.shared.u16 [%1], %9;\n\t"
        "st.shared.u16 [%2], %10;\n\t"
        "st.shared.u16 [%3], %11;\n\t"
        "st.shared.u16 [%4], %12;\n\t"
        "st.shared.u16 [%5], %13;\n\t"
        "st.shared.u16 [%6], %14;\n\t"
        "st.shared.u16 [%7], %15;"
        :: "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
           "h"(v[0]), "h"(v[1]), "h"(v[2]), "h"(v[3]), "h"(v[4]), "h"(v[5]), "h"(v[6]), "h"(v[7])
        : "memory");
}

__device__ __forceinline__ void named_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
scan_tc_kernel(const __grid_constant__ CUtensorMap tm_h0, const __grid_constant__ CUtensorMap tm_hn,
               const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
               const TcParams p)
{
    // 1024-byte aligned base.  Offsetting the __shared__ array itself (rather than
    // rounding an integer address) keeps every derived pointer in the shared state
    // space, so accesses compile to shared-memory instructions, not generic ones.
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.T, T_pad = p.T_pad, RB = p.RB, P = p.P, H = p.H, G = p.G, W = p.tree.W, HP = H * P;
    const int hpg = H / G, hpt = p.hpt, S = p.S;
    const uint32_t xbs = (uint32_t)T_pad * 128u;                      // x: bytes per 64-column block

    uint8_t *h0s = smem;                                              // S x [4 atoms][RB rows][128 B] fp32
    uint8_t *xs = smem + p.off_x;                                     // S x {NB x [T_pad rows][128 B] x, dt}
    uint8_t *cs = smem + p.off_c;                                     // [4 atoms][T_pad rows][128 B] fp32
    uint8_t *mh = smem + p.off_mh;                                    // hpt x [KA atoms][T_pad rows][128 B] bf16
    float *Bp = reinterpret_cast<float *>(smem + p.off_bp);           // [kPathRows][128] fp32
    uint32_t *ancs = reinterpret_cast<uint32_t *>(smem + p.off_anc);  // [T][W]
    int32_t *poff = reinterpret_cast<int32_t *>(smem + p.off_poff);   // [T+1]
    int16_t *pnode = reinterpret_cast<int16_t *>(smem + p.off_pnode); // [T]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    volatile int32_t *misc = reinterpret_cast<volatile int32_t *>(smem + p.off_misc);
    float *Ash = reinterpret_cast<float *>(smem + p.off_ad);          // [H] A, then [H] D
    float *Dsh = Ash + H;
    float *pcb = reinterpret_cast<float *>(smem + p.off_pcb);         // [pair_cap] C_i . B_j
    uint8_t *pj = smem + p.off_pj;                                    // [pair_cap] j
    uint8_t *pi = smem + p.off_pi;                                    // [pair_cap] i
    // Per-tile coefficients, two slots: dts, L, exp(L), commit weights [hpt][T] each, alpha [hpt].
    auto coef = [&](int slot, int which) {
        return reinterpret_cast<float *>(smem + p.off_coef + slot * p.coef_slot) + which * hpt * T;
    };
    auto bar = [&](int i) { return ptx::smem_u32(&bars[i]); };

    const uint32_t h0_stage_bytes = (uint32_t)RB * 512u;
    const uint32_t tx_bytes = h0_stage_bytes + (uint32_t)T * RB * 2u;

    if (tid == 0) {
        ptx::prefetch_tensormap(&tm_h0);
        ptx::prefetch_tensormap(&tm_x);
        ptx::prefetch_tensormap(&tm_hn);
        ptx::prefetch_tensormap(&tm_y);
        for (int s = 0; s < kMaxStages; ++s) {
            ptx::mbar_init(bar(B_FULL + s), 1);
            ptx::mbar_init(bar(B_EPID + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(bar(B_ACCF + s), 1);
            ptx::mbar_init(bar(B_ACCE + s), kEpiWarps);
            ptx::mbar_init(bar(B_COEFF + s), kPrepThreads);
            ptx::mbar_init(bar(B_COEFE + s), kEpiWarps);
        }
        ptx::mbar_init(bar(B_MHF), kPrepThreads);
        ptx::mbar_init(bar(B_MHE), 1);
        ptx::fence_mbar_init();
        for (int q = 0; q < kMiscWords; ++q) misc[q] = 0;
    }
    __syncthreads();                                  // misc cleared before the allocation writes it
    // Operand rows the MMAs read past the valid tile (rows >= RB, nodes >= T)
    // must hold finite values: clear the staging regions once.
    for (uint32_t o = tid * 16u; o < p.off_mh; o += kThreads * 16u)
        *reinterpret_cast<float4 *>(smem + o) = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int h = tid; h < H; h += kThreads) {
        Ash[h] = __ldg(&p.A[h]);
        Dsh[h] = __ldg(&p.D[h]);
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(const_cast<int32_t *>(&misc[M_TMEM])), p.tmem_cols);
        ptx::tmem_relinquish();
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = static_cast<uint32_t>(misc[M_TMEM]);

    // Bounded wait that turns a timeout into a CTA-wide abort; after an abort
    // every wait returns false at once and no role does further work.
    auto wait = [&](uint32_t b, uint32_t parity, int where) -> bool {
        if (misc[M_ABORT]) return false;
        if (ptx::mbar_wait(b, parity)) return true;
        latch_error(p.err, STREE_ERR_TIMEOUT, blockIdx.x, where, (int)parity);
        misc[M_ABORT] = 1;
        return false;
    };

    // Launched as a programmatic dependent of the tree builder: everything above
    // overlapped it; the tree masks, depths and flags are read only after this.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int start = (int)((long long)blockIdx.x * p.ntiles / gridDim.x);
    const int end = (int)((long long)(blockIdx.x + 1) * p.ntiles / gridDim.x);
    uint32_t loads_issued = 0, stores_issued = 0;

    // Producer: TMA stores of tile q once its epilogue is done (descriptor in misc).
    auto store_tile = [&](uint32_t q) {
        const int s = q % S;
        if (!wait(bar(B_EPID + s), (q / S) & 1, 11)) return;
        const int t = misc[M_SDESC + 2 * s], commit = misc[M_SDESC + 2 * s + 1];
        const int b = t / p.tps, r0 = (t % p.tps) * RB;
        const uint32_t xsrc = ptx::smem_u32(xs + s * p.x_stage);
        for (int nb = 0; nb < p.NB; ++nb) ptx::tma_store_2d(&tm_y, r0 + nb * 64, b * T, xsrc + nb * xbs);
        if (commit) {
            const uint32_t src = ptx::smem_u32(h0s + s * h0_stage_bytes);
            ptx::tma_store_3d(&tm_hn, 0, b * HP + r0, 0, src);
        }
        ptx::bulk_commit();
        stores_issued = q + 1;
        STREE_TR(q, 10);
    };
    // Producer: TMA loads of tile k into stage k % S once tile k - S has left it.
    auto produce = [&](uint32_t k, int t) {
        const int s = k % S;
        if (k >= (uint32_t)S) {
            store_tile(k - S);
            ptx::bulk_wait_read_all();
            STREE_TR(k - S, 11);
        }
        if (misc[M_ABORT]) return;
        const int b = t / p.tps, r0 = (t % p.tps) * RB;
        const uint32_t fb = bar(B_FULL + s);
        ptx::mbar_expect_tx(fb, tx_bytes);
        const uint32_t dst = ptx::smem_u32(h0s + s * h0_stage_bytes);
        ptx::tma_load_3d(dst, &tm_h0, 0, b * HP + r0, 0, fb);    // [4 column groups][RB rows][32]
        const uint32_t xdst = ptx::smem_u32(xs + s * p.x_stage);
        for (int nb = 0; nb < p.NB; ++nb) ptx::tma_load_2d(xdst + nb * xbs, &tm_x, r0 + nb * 64, b * T, fb);
        loads_issued = k + 1;
        STREE_TR(k, 0);
    };

    int cur_key = -1, cur_b = -1;
    uint32_t k = 0;
    for (int t = start; t < end; ++t) {
        const int b = t / p.tps;
        if (!__ldg(&p.tree.ok[b])) continue;                     // invalid tree: skipped by every role
        const int r0 = (t % p.tps) * RB;
        const int hfirst = r0 / P;
        const int g = hfirst / hpg;
        const int key = b * G + g;
        const int s = k % S;
        const uint32_t sph = (k / S) & 1;                        // phase parity of this stage use
        const __nv_bfloat16 *Bseq = p.B + ((size_t)b * T * G + g) * kDstate;   // row j at + j * G * 128
        const size_t brow = (size_t)G * kDstate;
        bool produced = false;

        // ------------------------------------------------------------ (sequence, group) switch
        if (key != cur_key) {
            if (warp == kProducerWarp && lane == 0) {          // keep the stream going meanwhile
                produce(k, t);
                produced = true;
            }
            __syncthreads();                                   // every earlier tile is consumed
            if (tid == 0) STREE_TR(k, 12);
            const bool new_b = (b != cur_b);
            // Phase 1: independent loads.
            for (int q = tid; q < T_pad * 32; q += kThreads) {
                const int i = q >> 5, c = q & 31;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < T) {
                    float c0, c1, c2, c3;
                    unpack4(__ldg(reinterpret_cast<const uint2 *>(p.C + (((size_t)b * T + i) * G + g) * kDstate + c * 4)),
                            c0, c1, c2, c3);
                    v = make_float4(c0, c1, c2, c3);
                }
                const int kb = c >> 3, ch = c & 7;
                *reinterpret_cast<float4 *>(cs + kb * T_pad * 128 + i * 128 + ((ch ^ (i & 7)) << 4)) = v;
            }
            if (new_b) {
                for (int q = tid; q < T * W; q += kThreads) ancs[q] = __ldg(&p.tree.anc[(size_t)b * T * W + q]);
                for (uint32_t o = tid * 16u; o < (uint32_t)hpt * p.mh_head; o += kThreads * 16u)
                    *reinterpret_cast<float4 *>(mh + o) = make_float4(0.f, 0.f, 0.f, 0.f);
                if (tid == 0) {
                    misc[M_LEN] = p.do_commit ? __ldg(&p.path_len[b]) : 0;
                    misc[M_STATE] = p.do_commit;
                }
            }
            __syncthreads();
            if (new_b) {
                // Phase 2: the accepted path -- position q must hold the depth-q ancestor
                // of the last node -- and the pair offsets (prefix sum of ancestor counts).
                const int len = misc[M_LEN];
                if (p.do_commit) {
                    if (len < 0 || len > p.maxlen || len > T) {
                        if (tid == 0) {
                            misc[M_STATE] = 0;
                            latch_error(p.err, STREE_ERR_BAD_PATH, b, -1, len);
                        }
                    } else if (len > 0) {
                        const int leaf = __ldg(&p.path[(size_t)b * p.maxlen + len - 1]);
                        const bool leaf_ok = leaf >= 0 && leaf < T;
                        for (int q = tid; q < len; q += kThreads) {
                            const int j = __ldg(&p.path[(size_t)b * p.maxlen + q]);
                            const bool good = leaf_ok && j >= 0 && j < T &&
                                              ((ancs[leaf * W + (j >> 5)] >> (j & 31)) & 1u) &&
                                              __ldg(&p.tree.depth[(size_t)b * T + j]) == q &&
                                              (q != len - 1 || __ldg(&p.tree.depth[(size_t)b * T + leaf]) == len - 1);
                            if (!good) {
                                misc[M_STATE] = 0;
                                latch_error(p.err, STREE_ERR_BAD_PATH, b, q, j);
                            }
                            pnode[q] = (int16_t)(good ? j : 0);
                        }
                    }
                }
                int cnt = 0;
                if (tid < T)
                    for (int w = 0; w < W; ++w) cnt += __popc(ancs[tid * W + w]);
                int incl = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += v;
                }
                if (lane == 31) misc[M_WSUM + warp] = incl;
                __syncthreads();
                int add = 0;
                for (int w = 0; w < warp; ++w) add += misc[M_WSUM + w];
                if (tid < T) poff[tid + 1] = add + incl;
                if (tid == 0) {
                    poff[0] = 0;
                    int total = 0;
                    for (int w = 0; w < kWarps; ++w) total += misc[M_WSUM + w];
                    misc[M_TOTAL] = total;
                    misc[M_INSMEM] = total <= p.pair_cap;
                }
                cur_b = b;
            }
            __syncthreads();
            // Phase 3: path rows of B (fp32) for the commit, C_i . B_j of every ancestor pair.
            if (misc[M_STATE]) {
                const int nrows = min((int)misc[M_LEN], kPathRows);
                for (int q = tid; q < nrows * 32; q += kThreads) {
                    float b0, b1, b2, b3;
                    unpack4(__ldg(reinterpret_cast<const uint2 *>(Bseq + (size_t)pnode[q >> 5] * brow) + (q & 31)),
                            b0, b1, b2, b3);
                    reinterpret_cast<float4 *>(Bp)[q] = make_float4(b0, b1, b2, b3);
                }
            }
            if (misc[M_INSMEM]) {
                const int total = misc[M_TOTAL];
                // Node i's pairs: its ancestors in increasing order.
                for (int i = tid; i < T; i += kThreads) {
                    int q = poff[i];
                    for (int w = 0; w < W; ++w) {
                        uint32_t bits = ancs[i * W + w];
                        while (bits) {
                            pj[q] = (uint8_t)((w << 5) + __ffs(bits) - 1);
                            pi[q] = (uint8_t)i;
                            bits &= bits - 1;
                            ++q;
                        }
                    }
                }
                __syncthreads();
                // Four lanes per pair, a quarter of the state columns each.
                const int part = lane & 3;
                for (int q0 = (tid >> 2); q0 < ((total + 7) & ~7); q0 += kThreads / 4) {
                    const int q = q0 < total ? q0 : total - 1;
                    const int i = pi[q], j = pj[q];
                    float v = dot_cb_part(cs, T_pad, Bseq + (size_t)j * brow, i, part);
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    if (part == 0 && q0 < total) pcb[q] = v;
                }
            }
            ptx::fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) STREE_TR(k, 13);
            cur_key = key;
        }
        const int len = misc[M_LEN];
        const bool commit = p.do_commit && misc[M_STATE];
        uint8_t *h0t = h0s + s * h0_stage_bytes;
        uint8_t *xt = xs + s * p.x_stage;

        if (warp == kProducerWarp) {
            // ------------------------------------------------------------ producer
            if (lane == 0 && !produced) produce(k, t);
        } else if (warp == kMmaWarp) {
            // ------------------------------------------------------------ MMA issue
            if (lane == 0) {
                const int a = k & 1;
                const uint32_t acc = tmem + (uint32_t)(a * p.acc_cols);
                bool ok = wait(bar(B_FULL + s), sph, 20);
                if (ok && k >= 2) ok = wait(bar(B_ACCE + a), ((k >> 1) - 1) & 1, 21);
                STREE_TR(k, 1);
                if (ok) {
                    ptx::tc_fence_after();
                    const uint32_t a0 = ptx::smem_u32(h0t), b0 = ptx::smem_u32(cs);
                    const uint32_t idesc_root = ptx::idesc_tf32(RB, T_pad);
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            ptx::mma_tf32(acc, ptx::desc_kmajor_sw128(a0 + kb * RB * 128 + kk * 32),
                                          ptx::desc_kmajor_sw128(b0 + kb * T_pad * 128 + kk * 32), idesc_root,
                                          (kb | kk) != 0);
                    ok = wait(bar(B_MHF), k & 1, 22);
                    STREE_TR(k, 2);
                }
                if (ok) {
                    ptx::tc_fence_after();
                    const uint32_t xa = ptx::smem_u32(xt);
                    const uint32_t idesc_tree = ptx::idesc_bf16_amn(RB, T_pad);
                    for (int hh = 0; hh < hpt; ++hh) {
                        const uint32_t mb = ptx::smem_u32(mh + hh * p.mh_head);
                        const uint32_t dcol = acc + (uint32_t)(T_pad * (1 + hh));
                        for (int ks = 0; ks < T_pad / 16; ++ks)
                            ptx::mma_f16(dcol, ptx::desc_mnmajor_sw128(xa + ks * 2048, xbs, 1024),
                                         ptx::desc_kmajor_sw128(mb + (ks >> 2) * T_pad * 128 + (ks & 3) * 32),
                                         idesc_tree, ks != 0);
                    }
                    ptx::mma_commit(bar(B_ACCF + a));
                    ptx::mma_commit(bar(B_MHE));
                    STREE_TR(k, 3);
                }
            }
        } else if (warp < kEpiWarp0) {
            // ------------------------------------------------------------ prep warps
            const int ptid = tid - kPrepWarp0 * 32;
            const int c = k & 1;
            // Prep needs only dt, A and the topology -- not the tile's TMA stage -- so
            // it runs ahead of the load.  One thread polls; the others sleep on the
            // named barrier.
            if (ptid == 0 && k >= 2) wait(bar(B_COEFE + c), ((k >> 1) - 1) & 1, 31);
            named_sync(kBarPrep, kPrepThreads);
            bool ok = !misc[M_ABORT];
            float *dts = coef(c, 0), *Ls = coef(c, 1), *eLs = coef(c, 2), *wts = coef(c, 3);
            float *alpha = coef(c, 4);
            if (ptid == 0) STREE_TR(k, 4);
            if (ok) {
                for (int q = ptid; q < hpt * T; q += kPrepThreads) {
                    const int hh = q / T, i = q - hh * T;
                    dts[q] = bf2f(p.dt[((size_t)b * T + i) * H + hfirst + hh]);
                }
            }
            named_sync(kBarPrep, kPrepThreads);
            if (ok && !misc[M_ABORT]) {
                for (int q = ptid; q < hpt * T; q += kPrepThreads) {
                    const int hh = q / T, i = q - hh * T;
                    const float *dh = dts + hh * T;
                    float sum = 0.f;
                    for (int w = 0; w < W; ++w) {
                        uint32_t bits = ancs[i * W + w];
                        while (bits) {
                            sum += dh[(w << 5) + __ffs(bits) - 1];
                            bits &= bits - 1;
                        }
                    }
                    const float L = Ash[hfirst + hh] * sum;
                    Ls[q] = L;
                    eLs[q] = expf(L);
                }
            }
            named_sync(kBarPrep, kPrepThreads);
            if (ok && !misc[M_ABORT]) {
                if (commit) {
                    const int leaf = len > 0 ? pnode[len - 1] : 0;
                    for (int q = ptid; q < hpt * len; q += kPrepThreads) {
                        const int hh = q / len, kk = q - hh * len;
                        const int j = pnode[kk];
                        wts[hh * T + kk] = expf(Ls[hh * T + leaf] - Ls[hh * T + j]) * dts[hh * T + j];
                    }
                    if (ptid < hpt) alpha[ptid] = len > 0 ? eLs[ptid * T + leaf] : 1.f;
                }
                mbar_arrive(bar(B_COEFF + c));
                if (ptid == 0) STREE_TR(k, 5);
                // Masked decay matrix of every head of the tile (bf16, K-major swizzled):
                // M_h[i][j] = exp(L_i - L_j) (C_i . B_j) dt_j for j an ancestor-or-self of i.
                if (ptid == 0 && k > 0) wait(bar(B_MHE), (k - 1) & 1, 32);
                named_sync(kBarPrep, kPrepThreads);
                ok = !misc[M_ABORT];
                if (ok) {
                    const int total = misc[M_TOTAL];
                    if (misc[M_INSMEM]) {
                        for (int q = ptid; q < hpt * total; q += kPrepThreads) {
                            const int hh = q / total, qq = q - hh * total;
                            const int i = pi[qq], j = pj[qq];
                            const float m = expf(Ls[hh * T + i] - Ls[hh * T + j]) * pcb[qq] * dts[hh * T + j];
                            *reinterpret_cast<__nv_bfloat16 *>(mh + hh * p.mh_head + k_off(i, j, T_pad)) =
                                __float2bfloat16_rn(m);
                        }
                    } else {
                        for (int q = ptid; q < hpt * total; q += kPrepThreads) {
                            const int hh = q / total, qq = q - hh * total;
                            const int i = pair_row(poff, T, qq);
                            const int j = nth_set_bit(ancs + i * W, W, qq - poff[i]);
                            const float m = expf(Ls[hh * T + i] - Ls[hh * T + j]) *
                                            dot_cb(cs, T_pad, Bseq + (size_t)j * brow, i) * dts[hh * T + j];
                            *reinterpret_cast<__nv_bfloat16 *>(mh + hh * p.mh_head + k_off(i, j, T_pad)) =
                                __float2bfloat16_rn(m);
                        }
                    }
                    ptx::fence_proxy_async_smem();
                    mbar_arrive(bar(B_MHF));
                    if (ptid == 0) STREE_TR(k, 6);
                }
            }
        } else {
            // ------------------------------------------------------------ epilogue warps
            const int etid = tid - kEpiWarp0 * 32, ewarp = warp - kEpiWarp0;
            const int a = k & 1, c = k & 1;
            // One thread polls the barriers; the others sleep on the named barrier.
            if (etid == 0) {
                bool w = wait(bar(B_FULL + s), sph, 40);
                if (w) w = wait(bar(B_COEFF + c), (k >> 1) & 1, 41);
                if (w) w = wait(bar(B_ACCF + a), (k >> 1) & 1, 42);
            }
            named_sync(kBarEpi, kEpiThreads);
            // Warp-uniform decision (tcgen05.ld below is a warp-collective instruction).
            const bool run = __all_sync(0xffffffffu, !misc[M_ABORT]);
            if (etid == 0) STREE_TR(k, 7);
            if (run) ptx::tc_fence_after();
            const float *eLs = coef(c, 2), *wts = coef(c, 3), *alpha = coef(c, 4);
            if (run && commit) {
                const int tpr = kEpiThreads / RB;                  // threads per row: 2 or 4
                const int row = etid % RB, part = etid / RB;
                const int hh = (r0 + row) / P - hfirst;
                const MnCol xc(row, xbs);
                const int cols = kDstate / tpr;
                for (int c_lo = part * cols; c_lo < (part + 1) * cols; c_lo += 32)
                    commit_rows<32>(h0t, xt, xc, Bp, Bseq, brow, pnode, wts + hh * T, alpha[hh], len, RB, row, c_lo);
            }
            if (warp == 8 && lane == 0) STREE_TR(k, 19);
            named_sync(kBarEpi, kEpiThreads);                  // x rows of the path are read
            if (etid == 0) STREE_TR(k, 8);
            // A warp reads only its own quarter of the tensor-memory lanes: 32 * (warp % 4).
            // M = 128 puts tile row r in lane r; M = 64 puts rows 16q..16q+15 in
            // lanes 32q..32q+15, so every quarter (and every SM sub-partition) gets rows.
            const int quad = warp & 3, half = ewarp >> 2;
            // With M = 64 lanes 16..31 of a quarter hold no rows: those threads load
            // (tcgen05.ld is warp-collective) but do not store.
            const bool active = RB == 128 || lane < 16;
            const int row = RB == 128 ? quad * 32 + lane : quad * 16 + (lane & 15);
            if (run) {
                const int hh = (r0 + row) / P - hfirst;           // same for the whole warp (P >= 32)
                const float Dh = Dsh[hfirst + hh];
                const float *eLh = eLs + hh * T;
                const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * p.acc_cols);
                const uint32_t ty = tl + (uint32_t)(T_pad * (1 + hh));
                const MnCol xc(row, xbs);
                const uint32_t xbase = ptx::smem_u32(xt), ebase = ptx::smem_u32(eLh);
                // Chunks of 8 nodes; the next chunk's tensor-memory values are loaded
                // while the current one is computed.
                uint32_t R[8], Y[8], Rn[8], Yn[8];
                int c0 = half * 8;
                if (c0 < T) {
                    ptx::tmem_ld8_nowait(tl + (uint32_t)c0, R);
                    ptx::tmem_ld8_nowait(ty + (uint32_t)c0, Y);
                    ptx::tmem_wait_ld();
                }
                for (; c0 < T; c0 += 16) {
                    const bool more = c0 + 16 < T;
                    if (more) {
                        ptx::tmem_ld8_nowait(tl + (uint32_t)(c0 + 16), Rn);
                        ptx::tmem_ld8_nowait(ty + (uint32_t)(c0 + 16), Yn);
                    }
                    // Nodes past T read row T-1 and their results are dropped (every
                    // address stays inside the stage).
                    uint32_t xa[8], ea[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int i = min(c0 + u, T - 1);
                        xa[u] = xbase + xc.at(i);
                        ea[u] = ebase + (uint32_t)i * 4u;
                    }
                    uint16_t Xh[8];
                    float E[8];
                    lds_u16x8(xa, Xh);
                    lds_f32x8(ea, E);
                    uint16_t Yh[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float xv = __uint_as_float((uint32_t)Xh[u] << 16);
                        const float yv = fmaf(E[u], __uint_as_float(R[u]), fmaf(Dh, xv, __uint_as_float(Y[u])));
                        Yh[u] = __bfloat16_as_ushort(__float2bfloat16_rn(yv));
                    }
                    if (active && c0 + 8 <= T) {
                        sts_u16x8(xa, Yh);
                    } else if (active) {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            if (c0 + u < T)
                                asm volatile("st.shared.u16 [%0], %1;" ::"r"(xa[u]), "h"(Yh[u]) : "memory");
                    }
                    if (more) {
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            R[u] = Rn[u];
                            Y[u] = Yn[u];
                        }
                    }
                }
            }
            if (warp == 8 && lane == 0) STREE_TR(k, 16);
            ptx::tc_fence_before();
            __syncwarp();
            if (run && lane == 0) {
                mbar_arrive(bar(B_ACCE + a));
                mbar_arrive(bar(B_COEFE + c));
            }
            ptx::fence_proxy_async_smem();
            if (warp == 8 && lane == 0) STREE_TR(k, 17);
            if (warp == 6 && lane == 0) STREE_TR(k, 18);
            named_sync(kBarEpi, kEpiThreads);
            if (etid == 0) STREE_TR(k, 9);
            if (run && etid == 0) {
                misc[M_SDESC + 2 * s] = t;                     // the producer issues the stores
                misc[M_SDESC + 2 * s + 1] = commit ? 1 : 0;
                mbar_arrive(bar(B_EPID + s));
            }
        }
        ++k;
    }

    // ---------------------------------------------------------------- teardown
    if (warp == kProducerWarp && lane == 0) {
        for (uint32_t q = stores_issued; q < k && !misc[M_ABORT]; ++q) store_tile(q);
        ptx::bulk_wait_all();
        if (misc[M_ABORT]) {
            // Loads issued but never consumed may still land in this CTA's shared
            // memory: give them a bounded wait before the CTA exits.
            for (uint32_t q = loads_issued >= (uint32_t)S ? loads_issued - S : 0; q < loads_issued; ++q)
                ptx::mbar_wait(bar(B_FULL + q % S), (q / S) & 1);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
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

// Shared-memory layout for a tile height RB and S stages; false if it does not fit.
bool layout(const ScanArgs &a, int RB, int S, TcParams &p, size_t &smem)
{
    const int T = a.T, T_pad = (T + 15) / 16 * 16, W = (T + 31) / 32;
    const int hpt = a.P >= RB ? 1 : RB / a.P;
    const int NB = RB / 64, KA = (T_pad + 63) / 64;
    uint32_t off = (uint32_t)S * RB * 512u;                   // h0 stages
    p.off_x = off;
    p.x_stage = round_up((uint32_t)NB * T_pad * 128u, 1024u);
    off += (uint32_t)S * p.x_stage;
    // MMA rows past the tile (h0 rows >= RB, the second x block when RB = 64)
    // read whatever follows; keep that inside the allocation.
    const uint32_t spill = (uint32_t)(128 - RB) * 128u > (uint32_t)T_pad * 128u ? (uint32_t)(128 - RB) * 128u
                                                                               : (uint32_t)T_pad * 128u;
    p.off_c = round_up(off, 1024u);
    off = p.off_c + (uint32_t)T_pad * 512u;
    if (off < p.off_c + spill) off = p.off_c + spill;
    p.off_mh = round_up(off, 1024u);
    p.mh_head = (uint32_t)KA * T_pad * 128u;
    off = p.off_mh + (uint32_t)hpt * p.mh_head;
    p.off_bp = round_up(off, 16u);     off = p.off_bp + (uint32_t)kPathRows * kDstate * 4u;
    p.off_anc = round_up(off, 16u);    off = p.off_anc + (uint32_t)T * W * 4u;
    p.off_poff = round_up(off, 16u);   off = p.off_poff + (uint32_t)(T + 1) * 4u;
    p.coef_slot = round_up((uint32_t)(4 * hpt * T + hpt) * 4u, 16u);
    p.off_coef = round_up(off, 16u);   off = p.off_coef + 2u * p.coef_slot;
    p.off_pnode = round_up(off, 16u);  off = p.off_pnode + (uint32_t)T * 2u;
    p.off_bar = round_up(off, 16u);    off = p.off_bar + kNumBars * 8u;
    p.off_misc = round_up(off, 16u);   off = p.off_misc + kMiscWords * 4u;
    p.off_ad = round_up(off, 16u);     off = p.off_ad + 2u * a.H * 4u;
    p.off_pcb = round_up(off, 16u);
    const size_t fixed = (size_t)p.off_pcb + 1024;            // + alignment slack of the dynamic base
    if (fixed + 6 * 64 + 32 > kSmemLimit) return false;
    const int all_pairs = T * (T + 1) / 2;
    int cap = (int)((kSmemLimit - fixed - 32) / 6);
    if (cap > all_pairs) cap = all_pairs;
    p.pair_cap = cap;
    p.off_pj = round_up(p.off_pcb + (uint32_t)cap * 4u, 16u);
    p.off_pi = round_up(p.off_pj + (uint32_t)cap, 16u);
    smem = (size_t)p.off_pi + cap + 1024;
    smem = (smem + 15) / 16 * 16;
    if (smem > kSmemLimit) return false;
    p.T = T;
    p.T_pad = T_pad;
    p.KA = KA;
    p.RB = RB;
    p.NB = NB;
    p.S = S;
    p.hpt = hpt;
    p.acc_cols = (1 + hpt) * T_pad;
    uint32_t cols = 32;
    while (cols < (uint32_t)(2 * p.acc_cols)) cols <<= 1;
    if (cols > 512) return false;
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
    if (a.batch <= 0 || a.H % a.G != 0 || a.H > kMaxSmemHeads) return false;
    if (!encode_fn()) return false;
    const int sms = num_sms();
    // Preference: three stages (loads two tiles ahead), then the tallest tile
    // that still gives every SM work.
    const int cand[4][2] = {{128, 3}, {128, 2}, {64, 3}, {64, 2}};
    int chosen = -1;
    long long chosen_tiles = -1;
    TcParams best{};
    size_t best_smem = 0;
    for (const auto &c : cand) {
        const int RB = c[0], S = c[1];
        TcParams p{};
        size_t smem = 0;
        if (!rb_valid(a, RB) || !layout(a, RB, S, p, smem)) continue;
        const int all_pairs = a.T * (a.T + 1) / 2;
        if (p.pair_cap < all_pairs && p.pair_cap < 4 * a.T) continue;   // typical trees must fit
        const long long ntiles = (long long)a.batch * (a.H * a.P / RB);
        if (ntiles > 0x7fffffff) continue;
        if (ntiles >= sms) {
            chosen = RB;
            best = p;
            best_smem = smem;
            break;
        }
        if (ntiles > chosen_tiles) {
            chosen = RB;
            chosen_tiles = ntiles;
            best = p;
            best_smem = smem;
        }
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
    p.tree = a.tree;
    p.err = a.err;

    EncodeTiledFn enc = encode_fn();
    const int HP = a.H * a.P;
    CUtensorMap m_h0, m_hn, m_x, m_y;
    {
        // h0 / h_new as [4 groups of 32 columns][rows][32 columns]: one box is a
        // whole tile in the K-major layout of the MMA (four 128-byte-swizzled atoms).
        cuuint64_t dims[3] = {32, (cuuint64_t)a.batch * HP, kDstate / 32};
        cuuint64_t strides[2] = {(cuuint64_t)kDstate * 4, 128};
        cuuint32_t box[3] = {32, (cuuint32_t)p.RB, kDstate / 32};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&m_h0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(a.h0), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        float *hn = p.do_commit ? a.h_new : const_cast<float *>(a.h0);
        if (enc(&m_hn, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, hn, dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)HP, (cuuint64_t)a.batch * a.T};
        cuuint64_t strides[1] = {(cuuint64_t)HP * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)a.T};
        cuuint32_t es[2] = {1, 1};
        if (enc(&m_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.x), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        if (enc(&m_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.y, dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, scan_tc_kernel, kThreads, pl.smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    // Tensor memory: every resident CTA holds tmem_cols of the SM's 512 columns.
    const int tmem_fit = 512 / (int)p.tmem_cols;
    if (per_sm > tmem_fit) per_sm = tmem_fit;
    long long grid = (long long)num_sms() * per_sm;
    if (grid > p.ntiles) grid = p.ntiles;
    // Programmatic dependent launch: the prologue (barriers, tensor memory, A/D)
    // overlaps the preceding kernel, normally the tree builder.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, scan_tc_kernel, m_h0, m_hn, m_x, m_y, p);
}

}  // namespace stree

#ifdef STREE_TRACE
extern "C" int stree_debug_trace(unsigned long long *host, size_t n)
{
    return (int)cudaMemcpyFromSymbol(host, stree::g_trace, n * sizeof(unsigned long long));
}
extern "C" int stree_debug_trace_clear(void)
{
    static unsigned long long zero[4 * 32 * 24];
    return (int)cudaMemcpyToSymbol(stree::g_trace, zero, sizeof(zero));
}
#endif
