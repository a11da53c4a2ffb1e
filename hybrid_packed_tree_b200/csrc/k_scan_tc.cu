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
//   * producer warp: TMA loads of the fp32 h0 tile (one 3-D box: four 128-byte
//     swizzled atoms of 32 columns) and the bf16 x tile (64-column swizzled
//     boxes) into an S-stage ring (S = 2 or 3), and the TMA stores of y and h_new;
//   * MMA warp (one thread): the root term R[row, i] = h0[row, :] . C_i as
//     tcgen05.mma kind::tf32 (M = 128, N = T_pad, K = 128) and the tree term
//     Y[row, i] = sum_j x[j, row] M_h[i, j] as kind::f16 with x as an MN-major
//     operand straight from the stage, into a 2-deep tensor-memory ring;
//   * prep warps: per tile and head the tree cumsum L, exp(L) and the masked
//     decay matrix M_h[i][j] = exp(L_i - L_j) (C_i . B_j) dt_j over ancestor
//     pairs only, with D_h added on the diagonal (bf16, K-major swizzled), plus
//     the commit weights;
//   * epilogue warps: the commit in exact fp32 FMA, written in place over the
//     h0 tile, then y = exp(L_i) R + Y in place over the x tile (Y already holds
//     the skip term), and the release of the stage to the producer's stores.
// C (fp32 operand of the root MMA), the ancestor pairs' C.B and the accepted
// path's rows of B are staged once per (sequence, group), all of its global
// reads issued together.  When the call passes parent[] the kernel builds the
// tree masks itself in shared memory and requests its first tiles at entry, so
// it never waits for the tree builder launched beside it.  Roles only block on
// bounded mbarrier waits; a timeout latches STREE_ERR_TIMEOUT and the CTA runs
// to its end without further work.  Precision: the root term rounds h0 to tf32
// and the masked decay matrix (D_h on its diagonal included) to bf16 inside the
// MMAs (fp32 accumulation); on trees whose ancestor pairs overflow the fp32 pair
// table (deep trees: up to three times as many pairs are kept) C_i . B_j is held
// in bf16 before that product; the commit and every other step are fp32.
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

// Sixteen warps at 128 registers fill the register file: producer, MMA issuer,
// six prep warps, eight epilogue warps (two per tensor-memory lane quarter).
constexpr int kProducerWarp = 0, kMmaWarp = 1, kPrepWarp0 = 2, kPrepWarps = 6;
constexpr int kEpiWarp0 = kPrepWarp0 + kPrepWarps, kEpiWarps = 8;
constexpr int kMaxStages = 3;
constexpr int kMaxSmemHeads = 1024;        // A and D are staged in shared memory
constexpr int kWarps = kEpiWarp0 + kEpiWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kPrepThreads = kPrepWarps * 32, kEpiThreads = kEpiWarps * 32;
constexpr int kBarEpi = 1, kBarPrep = 2;   // named barriers (0 is __syncthreads)

enum Misc { M_TMEM = 0, M_ABORT, M_LEN, M_STATE, M_INSMEM, M_TOTAL, M_OK, M_DTK, M_SDESC = 8, M_WSUM = 8 + 2 * kMaxStages,
            kMiscWords = M_WSUM + kWarps };
// mbarriers: TMA stage full / epilogue done with a stage (ring of S), tensor-memory
// accumulator full / empty (ring of 2), masked-decay matrix full / empty,
// per-tile coefficients full / empty (ring of 2), for the tensor-core commit its
// coefficient operand written and its (single) product read, and the MMA drain
// after an abort.
enum Bars { B_FULL = 0, B_EPID = kMaxStages, B_ACCF = 2 * kMaxStages, B_ACCE = B_ACCF + 2, B_MHF = B_ACCE + 2,
            B_MHE = B_MHF + 1, B_COEFF = B_MHE + 1, B_COEFE = B_COEFF + 2, B_CFF = B_COEFE + 2, B_CME = B_CFF + 1,
            B_DRAIN = B_CME + 1, kNumBars = B_DRAIN + 1 };

struct TcParams {
    const __nv_bfloat16 *__restrict__ dt;
    const __nv_bfloat16 *__restrict__ B;
    const __nv_bfloat16 *__restrict__ C;
    const float *__restrict__ A;
    const float *__restrict__ D;
    const int32_t *__restrict__ path;
    const int32_t *__restrict__ path_len;
    const int32_t *__restrict__ parent;    // non-NULL: masks built in-kernel, inputs complete at launch
    TreeView tree;
    uint32_t *tree_anc;                    // with parent: the tree written here for later calls (or NULL)
    int32_t *tree_depth, *tree_ok;
    int32_t *err;
    unsigned long long wait_ns;            // limit of every bounded wait
    int fault;                             // test hook: 1 withholds the first tile's coefficient hand-off
    int T, T_pad, KA, H, P, G, RB, NB, S, tps, ntiles, maxlen, do_commit, pre, bs_mh, tc_commit, hpt, pair_cap,
        acc_cols, cm_col;
    int tpg, sw_milli;                     // tiles per (sequence, group); cost of a switch in tiles x 1000
    float *pcb_g;                          // trees whose pairs overflow shared memory: C_i . B_j of the
    int pair_max;                          //   pairs in a global region of pair_max floats per CTA
    uint32_t tmem_cols;
    uint32_t off_x, x_stage, off_c, off_mh, mh_head, off_bp, off_anc, off_poff, off_coef, coef_slot,
        off_pnode, off_praw, off_par, off_dep, off_bs, off_cf, off_bt, off_bar, off_misc, off_ad, off_pcb, off_pj,
        off_pi;
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

// C_i . B_j over all 128 state columns by one lane.  The lane walks the 32
// four-column chunks starting at chunk `rot` (its lane index), so the lanes of a
// warp read 32 different chunks of their B rows (rows lie 256 bytes apart,
// unswizzled: without the rotation they would all hit the same banks) and spread
// their C reads over the swizzle's eight 16-byte bank groups.  Four accumulators,
// one per column of the chunk.
template <bool kStaged>
__device__ __forceinline__ float dot_cb_lane(const uint8_t *cs, int T_pad, const __nv_bfloat16 *Bj, int i, int rot)
{
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    const uint2 *brow = reinterpret_cast<const uint2 *>(Bj);
    const uint8_t *crow = cs + i * 128;
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
        const int g = (c + rot) & 31;
        const float4 cv = *reinterpret_cast<const float4 *>(crow + (g >> 3) * T_pad * 128 + (((g & 7) ^ (i & 7)) << 4));
        float b0, b1, b2, b3;
        unpack4(kStaged ? brow[g] : __ldg(brow + g), b0, b1, b2, b3);
        a0 = fmaf(cv.x, b0, a0);
        a1 = fmaf(cv.y, b1, a1);
        a2 = fmaf(cv.z, b2, a2);
        a3 = fmaf(cv.w, b3, a3);
    }
    return (a0 + a1) + (a2 + a3);
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

// Two fp32 fused multiply-adds in one instruction (lane-wise a * b + c, each
// rounded once, exactly as two scalar fmaf).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<const unsigned long long *>(&a)), "l"(*reinterpret_cast<const unsigned long long *>(&b)),
          "l"(*reinterpret_cast<const unsigned long long *>(&c)));
    return *reinterpret_cast<float2 *>(&d);
}

// Commit of one tile row segment on CUDA cores: h_new = alpha h0 + sum_q coef_q B[pnode_q]
// (fp32), coef_q = w_q x[pnode_q][row], written in place over the h0 tile.  The
// first `nsm` (<= kPathRows) path rows of B come from shared memory (fp32), the
// others from global memory.
template <int CPT>
__device__ __forceinline__ void commit_rows(uint8_t *h0t, const uint8_t *xt, const MnCol &xc, const float *Bp, int nsm,
                                            const __nv_bfloat16 *Bseq, size_t brow, const int16_t *pnode,
                                            const float *wh, float al, int len, int RB, int row, int c_lo)
{
    float2 acc[CPT / 2];
#pragma unroll
    for (int c = 0; c < CPT / 2; ++c) acc[c] = make_float2(0.f, 0.f);
    const int lsm = min(len, nsm);
    float cf[kPathRows];
#pragma unroll
    for (int q = 0; q < kPathRows; ++q) {
        // Only path positions q < lsm are used here; others address node 0.
        const int j = q < lsm ? (int)pnode[q] : 0;
        const float xv = bf2f(*reinterpret_cast<const __nv_bfloat16 *>(xt + xc.at(j)));
        cf[q] = q < lsm ? wh[q] * xv : 0.f;
    }
#pragma unroll
    for (int q = 0; q < kPathRows; ++q) {
        if (q < lsm) {
            const float4 *src = reinterpret_cast<const float4 *>(Bp + q * kDstate + c_lo);
            const float2 cq = make_float2(cf[q], cf[q]);
#pragma unroll
            for (int c = 0; c < CPT / 4; ++c) {
                const float4 bv = src[c];
                acc[2 * c + 0] = ffma2(cq, make_float2(bv.x, bv.y), acc[2 * c + 0]);
                acc[2 * c + 1] = ffma2(cq, make_float2(bv.z, bv.w), acc[2 * c + 1]);
            }
        }
    }
    for (int q = lsm; q < len; ++q) {
        const int j = pnode[q];
        const float coef = wh[q] * bf2f(*reinterpret_cast<const __nv_bfloat16 *>(xt + xc.at(j)));
        const float2 cq = make_float2(coef, coef);
        const uint2 *src = reinterpret_cast<const uint2 *>(Bseq + (size_t)j * brow + c_lo);
#pragma unroll
        for (int c = 0; c < CPT / 4; ++c) {
            float b0, b1, b2, b3;
            unpack4(__ldg(src + c), b0, b1, b2, b3);
            acc[2 * c + 0] = ffma2(cq, make_float2(b0, b1), acc[2 * c + 0]);
            acc[2 * c + 1] = ffma2(cq, make_float2(b2, b3), acc[2 * c + 1]);
        }
    }
    const float2 a2 = make_float2(al, al);
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
            const float2 lo = ffma2(a2, make_float2(h[c].x, h[c].y), acc[2 * (c0 + c) + 0]);
            const float2 hi = ffma2(a2, make_float2(h[c].z, h[c].w), acc[2 * (c0 + c) + 1]);
            *reinterpret_cast<float4 *>(h0t + kb * RB * 128 + row * 128 + ((ch ^ (row & 7)) << 4)) =
                make_float4(lo.x, lo.y, hi.x, hi.y);
        }
    }
}

// Byte offset of fp32 element (row, k), k < 8, in a K-major operand without
// swizzle: 8-row x 16-byte core matrices of 128 contiguous bytes, the two
// K-halves of a row group 128 bytes apart, row groups 256 bytes apart.
__device__ __forceinline__ uint32_t k8_off(int row, int k)
{
    return (uint32_t)(row >> 3) * 256u + (uint32_t)(k >> 2) * 128u + (uint32_t)(row & 7) * 16u + (uint32_t)(k & 3) * 4u;
}

// Eight 32-bit shared-memory loads issued back to back (addresses in the shared window).
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
    const int T = p.T, T_pad = p.T_pad, RB = p.RB, P = p.P, H = p.H, G = p.G, HP = H * P;
    const int W = (T + 31) / 32;
    const int hpg = H / G, hpt = p.hpt, S = p.S;
    const uint32_t xbs = (uint32_t)T_pad * 128u;                      // x: bytes per 64-column block

    uint8_t *h0s = smem;                                              // S x [4 atoms][RB rows][128 B] fp32
    uint8_t *xs = smem + p.off_x;                                     // S x NB x [T_pad rows][128 B] bf16
    uint8_t *cs = smem + p.off_c;                                     // [4 atoms][T_pad rows][128 B] fp32
    uint8_t *mh = smem + p.off_mh;                                    // hpt x [KA atoms][T_pad rows][128 B] bf16
    float *Bp = reinterpret_cast<float *>(smem + p.off_bp);           // [kPathRows][128] fp32
    uint32_t *ancs = reinterpret_cast<uint32_t *>(smem + p.off_anc);  // [T][W]
    int32_t *poff = reinterpret_cast<int32_t *>(smem + p.off_poff);   // [T+1]
    int16_t *pnode = reinterpret_cast<int16_t *>(smem + p.off_pnode); // [T] validated accepted path
    int32_t *praw = reinterpret_cast<int32_t *>(smem + p.off_praw);   // [T] accepted path as given
    int32_t *par = reinterpret_cast<int32_t *>(smem + p.off_par);     // [T] parent as given
    int32_t *dep = reinterpret_cast<int32_t *>(smem + p.off_dep);     // [T] depth
    __nv_bfloat16 *Bs = reinterpret_cast<__nv_bfloat16 *>(smem + p.off_bs);   // [T][128] B rows, when staged
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    volatile int32_t *misc = reinterpret_cast<volatile int32_t *>(smem + p.off_misc);
    float *Ash = reinterpret_cast<float *>(smem + p.off_ad);          // [H] A, then [H] D
    float *Dsh = Ash + H;
    float *pcb = reinterpret_cast<float *>(smem + p.off_pcb);         // [pair_cap] C_i . B_j
    uint8_t *pj = smem + p.off_pj;                                    // [pair_cap] j
    uint8_t *pi = smem + p.off_pi;                                    // [pair_cap] i
    // Deep trees whose pairs overflow the fp32 table: the same region as bf16 values
    // in row order (node i's pairs at poff[i] .., its ancestors in increasing order).
    __nv_bfloat16 *pcb16 = reinterpret_cast<__nv_bfloat16 *>(smem + p.off_pcb);   // [3 pair_cap]
    const bool b_staged = p.off_bs != 0;
    uint8_t *cfs = smem + p.off_cf;                                   // [RB][8] fp32 commit coefficients (MMA A)
    uint8_t *bts = smem + p.off_bt;                                   // [128][8] fp32 path rows of B^T (MMA B)
    // Per-tile coefficients, two slots: dts, L, exp(L), commit weights [hpt][T] each, alpha [hpt].
    auto coef = [&](int slot, int which) {
        return reinterpret_cast<float *>(smem + p.off_coef + slot * p.coef_slot) + which * hpt * T;
    };
    auto bar = [&](int i) { return ptx::smem_u32(&bars[i]); };

    const uint32_t h0_stage_bytes = (uint32_t)RB * 512u;
    const uint32_t tx_bytes = h0_stage_bytes + (uint32_t)T * RB * 2u;
    // Tile range of this CTA: equal shares of a cost line on which every tile costs
    // one unit and every (sequence, group) start costs sw_milli / 1000 more (the
    // switch), so that a range crossing a group boundary takes fewer tiles.
    int start, end;
    {
        const long long per = (long long)p.tpg * 1000 + p.sw_milli;
        const long long total = (long long)(p.ntiles / p.tpg) * per;
        auto tile_at = [&](long long c) -> int {
            if (c >= total) return p.ntiles;
            const long long q = c / per, r = c - q * per;
            long long t = q * p.tpg + (r <= p.sw_milli ? 0 : (r - p.sw_milli + 999) / 1000);
            if (t > (q + 1) * p.tpg) t = (q + 1) * p.tpg;
            return (int)t;
        };
        start = tile_at((long long)blockIdx.x * total / gridDim.x);
        end = tile_at((long long)(blockIdx.x + 1) * total / gridDim.x);
    }
    // With p.pre the first S tiles are requested before anything else, once the
    // preceding grid (the kernel is a programmatic dependent) has completed.
    const uint32_t npre = p.pre ? (uint32_t)min(S, end - start) : 0u;
    uint32_t loads_issued = 0, stores_issued = 0;

    // Bounded wait that turns a timeout into a CTA-wide abort; after an abort
    // every wait returns false at once and no role does further work.
    auto wait = [&](uint32_t b, uint32_t parity, int where) -> bool {
        if (misc[M_ABORT]) return false;
        if (ptx::mbar_wait(b, parity, p.wait_ns)) return true;
        latch_error(p.err, STREE_ERR_TIMEOUT, blockIdx.x, where, (int)parity);
        misc[M_ABORT] = 1;
        return false;
    };
    // Producer: TMA stores of tile q once its epilogue is done (descriptor in misc:
    // the tile, and bit 0 = store y, bit 1 = store h_new).
    auto store_tile = [&](uint32_t q) {
        const int s = q % S;
        if (!wait(bar(B_EPID + s), (q / S) & 1, 11)) return;
        const int t = misc[M_SDESC + 2 * s], what = misc[M_SDESC + 2 * s + 1];
        const int b = t / p.tps, r0 = (t % p.tps) * RB;
        if (what & 1) {
            const uint32_t xsrc = ptx::smem_u32(xs + s * p.x_stage);
            for (int nb = 0; nb < p.NB; ++nb) ptx::tma_store_2d(&tm_y, r0 + nb * 64, b * T, xsrc + nb * xbs);
        }
        if (what & 2) ptx::tma_store_3d(&tm_hn, 0, b * HP + r0, 0, ptx::smem_u32(h0s + s * h0_stage_bytes));
        ptx::bulk_commit();
        stores_issued = q + 1;
    };
    // Producer: TMA loads of tile k into stage k % S once tile k - S has left it.
    auto produce = [&](uint32_t k, int t) {
        const int s = k % S;
        if (k >= (uint32_t)S) {
            store_tile(k - S);
            ptx::bulk_wait_read_all();
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
    };

    if (p.pre) asm volatile("griddepcontrol.wait;" ::: "memory");
    // A later launch on the stream (the next layer) may be scheduled onto SMs as
    // this grid's CTAs leave; it waits for this grid's completion before it reads
    // anything, so only its set-up overlaps this grid's tail.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
        ptx::mbar_init(bar(B_CFF), kPrepThreads);
        ptx::mbar_init(bar(B_CME), kEpiWarps);
        ptx::mbar_init(bar(B_DRAIN), 1);
        ptx::fence_mbar_init();
        for (int q = 0; q < kMiscWords; ++q) misc[q] = 0;
        for (uint32_t q = 0; q < npre; ++q) produce(q, start + (int)q);
    }
    // x rows T..T_pad-1 of every stage are never written by the TMA but enter the
    // tree MMA (times zero weights): keep them finite.  The TMA writes only rows < T.
    {
        const int padrows = T_pad - T, nchunks = S * p.NB * padrows * 8;
        for (int q = tid; q < nchunks; q += kThreads) {
            const int c16 = q & 7, r = (q >> 3) % padrows, blk = (q >> 3) / padrows;
            uint8_t *dst = xs + (blk / p.NB) * p.x_stage + (blk % p.NB) * xbs + (T + r) * 128 + c16 * 16;
            *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // Without p.pre the inputs or the context's tree may come from the preceding
    // launch: nothing global is read before it has completed.
    if (!p.pre) asm volatile("griddepcontrol.wait;" ::: "memory");
    __syncthreads();                                  // misc cleared before the allocation writes it
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(const_cast<int32_t *>(&misc[M_TMEM])), p.tmem_cols);
        ptx::tmem_relinquish();
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = static_cast<uint32_t>(misc[M_TMEM]);

    int cur_key = -1, cur_b = -1;
    // Prep warps: dt of the next tile, requested while the current one is prepared.
    __nv_bfloat16 dnext[4];
    int dnext_k = -1;
    uint32_t ncm = 0;                                 // tiles committed on the tensor cores so far
    uint32_t k = 0;
    for (int t = start; t < end; ++t, ++k) {
        const int b = t / p.tps;
        const int r0 = (t % p.tps) * RB;
        const int hfirst = r0 / P;
        const int g = hfirst / hpg;
        const int key = b * G + g;
        const int s = k % S;
        const uint32_t sph = (k / S) & 1;                        // phase parity of this stage use
        const __nv_bfloat16 *Bseq = p.B + ((size_t)b * T * G + g) * kDstate;   // row j at + j * G * 128
        const size_t brow = (size_t)G * kDstate;
        bool produced = k < npre;

        // ------------------------------------------------------------ (sequence, group) switch
        if (key != cur_key) {
            if (warp == kProducerWarp && lane == 0 && !produced) produce(k, t);   // keep the stream going
            produced = true;
            __syncthreads();                                   // every earlier tile is consumed
            const bool new_b = (b != cur_b);
            // Phase 1: every global read of this (sequence, group) in flight at once:
            // asynchronous copies for the B rows, parent, path, A and D (or the
            // context's tree), plain loads for dt and C (C is widened to fp32).
            if (b_staged)
                for (int q = tid; q < T * 32; q += kThreads)
                    ptx::cp_async8(ptx::smem_u32(Bs) + (uint32_t)q * 8u, Bseq + (size_t)(q >> 5) * brow + (q & 31) * 4);
            if (cur_key < 0)
                for (int h = tid; h < H; h += kThreads) {
                    ptx::cp_async4(ptx::smem_u32(Ash + h), p.A + h);
                    ptx::cp_async4(ptx::smem_u32(Dsh + h), p.D + h);
                }
            int plen = 0, okv = 1;
            if (new_b) {
                if (p.parent) {
                    for (int i = tid; i < T; i += kThreads) ptx::cp_async4(ptx::smem_u32(par + i), p.parent + (size_t)b * T + i);
                } else {
                    for (int q = tid; q < T * W; q += kThreads)
                        ptx::cp_async4(ptx::smem_u32(ancs + q), p.tree.anc + (size_t)b * T * W + q);
                    for (int i = tid; i < T; i += kThreads) ptx::cp_async4(ptx::smem_u32(dep + i), p.tree.depth + (size_t)b * T + i);
                    if (tid == 0) okv = __ldg(&p.tree.ok[b]);
                }
                if (p.do_commit) {
                    for (int q = tid; q < min(p.maxlen, T); q += kThreads)
                        ptx::cp_async4(ptx::smem_u32(praw + q), p.path + (size_t)b * p.maxlen + q);
                    if (tid == 0) plen = __ldg(&p.path_len[b]);
                }
            }
            // dt of this tile for the prep warps (hpt * T <= 512 values).
            __nv_bfloat16 dtv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int q = tid + u * kThreads, hh = q / T, i = q - hh * T;
                if (q < hpt * T) dtv[u] = p.dt[((size_t)b * T + i) * H + hfirst + hh];
            }
            // All of this thread's C loads are issued here and first used after the
            // tree is rebuilt, so their latency overlaps that work.
            constexpr int kCItems = (kMaxTcNodes * 32 + kThreads - 1) / kThreads;
            uint2 craw[kCItems];
#pragma unroll
            for (int u = 0; u < kCItems; ++u) {
                const int q = tid + u * kThreads, i = q >> 5, c = q & 31;
                craw[u] = make_uint2(0u, 0u);
                if (i < T)
                    craw[u] = __ldg(reinterpret_cast<const uint2 *>(p.C + (((size_t)b * T + i) * G + g) * kDstate + c * 4));
            }
            if (new_b && !p.bs_mh)
                for (uint32_t o = tid * 16u; o < (uint32_t)hpt * p.mh_head; o += kThreads * 16u)
                    *reinterpret_cast<float4 *>(mh + o) = make_float4(0.f, 0.f, 0.f, 0.f);
            if (tid == 0) {
                misc[M_DTK] = (int)k + 1;
                if (new_b) {
                    misc[M_LEN] = plen;
                    misc[M_STATE] = p.do_commit;
                    if (!p.parent) misc[M_OK] = okv;
                }
            }
            ptx::cp_async_wait_all();
            __syncthreads();
            if (new_b) {
                bool okb;
                if (p.parent) {
                    // Phase 2a: the tree itself -- node 0 the only root, every other
                    // parent an earlier node -- then each node's ancestor-or-self row
                    // (built in registers) and depth by walking its root path.  An
                    // invalid tree is reported by the CTA holding the sequence's first
                    // tile; its tiles flow through the pipeline with empty masks and
                    // are not stored.
                    int bad = 0;
                    for (int i = tid; i < T; i += kThreads) {
                        const int v = par[i];
                        bad |= (i == 0) ? (v != -1) : (v < 0 || v >= i);
                    }
                    okb = !__syncthreads_or(bad);
                    for (int i = tid; i < T; i += kThreads) {
                        uint32_t a4[4] = {0u, 0u, 0u, 0u};                // W <= 4 (T <= 128)
                        int d = -1;
                        if (okb)
                            for (int j = i; j >= 0; j = par[j]) {
                                const uint32_t bit = 1u << (j & 31), wq = (uint32_t)j >> 5;
#pragma unroll
                                for (int u = 0; u < 4; ++u) a4[u] |= wq == (uint32_t)u ? bit : 0u;
                                ++d;
                            }
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (u < W) ancs[i * W + u] = a4[u];
                        dep[i] = okb ? d : 0;
                    }
                    if (tid == 0) misc[M_OK] = okb;
                    __syncthreads();
                    if (t % p.tps == 0) {
                        // The CTA holding the sequence's first tile keeps its tree for
                        // later calls and reports an invalid one (first bad node).
                        if (p.tree_anc)
                            for (int q = tid; q < T * W; q += kThreads) p.tree_anc[(size_t)b * T * W + q] = ancs[q];
                        if (p.tree_depth)
                            for (int i = tid; i < T; i += kThreads) p.tree_depth[(size_t)b * T + i] = dep[i];
                        if (tid == 0) {
                            if (p.tree_ok) p.tree_ok[b] = okb ? 1 : 0;
                            for (int i = 0; i < T && !okb; ++i) {
                                const int v = par[i];
                                if ((i == 0) ? (v != -1) : (v < 0 || v >= i)) {
                                    latch_error(p.err, STREE_ERR_BAD_TREE, b, i, v);
                                    break;
                                }
                            }
                        }
                    }
                } else {
                    okb = misc[M_OK] != 0;
                }
                // Phase 2b: the accepted path -- position q must hold the depth-q
                // ancestor of the last node -- and the pair offsets (prefix sum of
                // ancestor counts).
                const int len = misc[M_LEN];
                if (!okb) {
                    if (tid == 0) misc[M_STATE] = 0;
                } else if (p.do_commit) {
                    if (len < 0 || len > p.maxlen || len > T) {
                        if (tid == 0) {
                            misc[M_STATE] = 0;
                            latch_error(p.err, STREE_ERR_BAD_PATH, b, -1, len);
                        }
                    } else if (len > 0) {
                        const int leaf = praw[len - 1];
                        const bool leaf_ok = leaf >= 0 && leaf < T;
                        for (int q = tid; q < len; q += kThreads) {
                            const int j = praw[q];
                            const bool good = leaf_ok && j >= 0 && j < T &&
                                              ((ancs[leaf * W + (j >> 5)] >> (j & 31)) & 1u) && dep[j] == q &&
                                              (q != len - 1 || dep[leaf] == len - 1);
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
                    misc[M_INSMEM] = total <= p.pair_cap ? 1 : total <= 3 * p.pair_cap ? 2 : 0;
                }
                cur_b = b;
            }
            // C widened to fp32 into the root MMA's operand layout, and this tile's dt.
#pragma unroll
            for (int u = 0; u < kCItems; ++u) {
                const int q = tid + u * kThreads, i = q >> 5, c = q & 31;
                if (q < T_pad * 32) {
                    float4 v;
                    unpack4(craw[u], v.x, v.y, v.z, v.w);
                    *reinterpret_cast<float4 *>(cs + (c >> 3) * T_pad * 128 + i * 128 + (((c & 7) ^ (i & 7)) << 4)) = v;
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u)
                if (tid + u * kThreads < hpt * T) coef(k & 1, 0)[tid + u * kThreads] = bf2f(dtv[u]);
            __syncthreads();
            // Phase 3: path rows of B (fp32) for the commit, C_i . B_j of every ancestor pair.
            if (misc[M_STATE] && p.tc_commit && misc[M_LEN] <= kPathRows) {
                // B^T of the path rows, K-major fp32 (zeros past the path), for the commit MMA.
                const int len = misc[M_LEN];
                for (int it = tid; it < kDstate * 2; it += kThreads) {
                    const int n = it & (kDstate - 1), kc = it >> 7;
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int q = 4 * kc + e;
                        const int j = q < len ? (int)pnode[q] : 0;
                        const float bv = b_staged ? bf2f(Bs[j * kDstate + n]) : bf2f(Bseq[(size_t)j * brow + n]);
                        v[e] = q < len ? bv : 0.f;
                    }
                    *reinterpret_cast<float4 *>(bts + k8_off(n, 4 * kc)) = make_float4(v[0], v[1], v[2], v[3]);
                }
            } else if (misc[M_STATE] && !p.tc_commit) {
                const int nrows = min((int)misc[M_LEN], kPathRows);
                for (int q = tid; q < nrows * 32; q += kThreads) {
                    const int j = pnode[q >> 5];
                    const uint2 raw = b_staged ? reinterpret_cast<const uint2 *>(Bs + j * kDstate)[q & 31]
                                               : __ldg(reinterpret_cast<const uint2 *>(Bseq + (size_t)j * brow) + (q & 31));
                    float b0, b1, b2, b3;
                    unpack4(raw, b0, b1, b2, b3);
                    reinterpret_cast<float4 *>(Bp)[q] = make_float4(b0, b1, b2, b3);
                }
            }
            if (misc[M_INSMEM] == 1) {
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
                // One lane per pair.
                for (int q = tid; q < total; q += kThreads) {
                    const int i = pi[q], j = pj[q];
                    pcb[q] = b_staged ? dot_cb_lane<true>(cs, T_pad, Bs + j * kDstate, i, lane)
                                      : dot_cb_lane<false>(cs, T_pad, Bseq + (size_t)j * brow, i, lane);
                }
            } else if (misc[M_INSMEM] == 2 || p.pcb_g) {
                // Too many pairs for the fp32 table (deep trees): the products rounded
                // to bf16 in the same region (row order), else in this CTA's own region
                // of a global scratch (fp32), read back by the prep warps.
                const bool h16 = misc[M_INSMEM] == 2;
                const int total = h16 ? (int)misc[M_TOTAL] : min((int)misc[M_TOTAL], p.pair_max);
                float *pg = h16 ? nullptr : p.pcb_g + (size_t)blockIdx.x * p.pair_max;
                for (int q = tid; q < total; q += kThreads) {
                    const int i = pair_row(poff, T, q);
                    const int j = nth_set_bit(ancs + i * W, W, q - poff[i]);
                    const float v = b_staged ? dot_cb_lane<true>(cs, T_pad, Bs + j * kDstate, i, lane)
                                             : dot_cb_lane<false>(cs, T_pad, Bseq + (size_t)j * brow, i, lane);
                    if (h16) pcb16[q] = __float2bfloat16_rn(v);
                    else pg[q] = v;
                }
            }
            if (p.bs_mh) {                                     // B rows read: clear the region for M_h
                __syncthreads();
                for (uint32_t o = tid * 16u; o < (uint32_t)hpt * p.mh_head; o += kThreads * 16u)
                    *reinterpret_cast<float4 *>(mh + o) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            ptx::fence_proxy_async_smem();
            __syncthreads();
            cur_key = key;
        }
        const int len = misc[M_LEN];
        const bool commit = p.do_commit && misc[M_STATE];
        const bool tcc = commit && p.tc_commit && len <= kPathRows;   // commit product on the tensor cores
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
                    if (tcc) {
                        // Commit product D[row][n] = sum_q cf[row][q] B_q[n] (K = 8, tf32) once the
                        // prep warps have written cf and the epilogue has read the previous
                        // product (D has one buffer).
                        ok = (ncm == 0 || wait(bar(B_CME), (ncm - 1) & 1, 24)) && wait(bar(B_CFF), ncm & 1, 23);
                        if (ok) {
                            ptx::tc_fence_after();
                            ptx::mma_tf32(tmem + (uint32_t)p.cm_col,
                                          ptx::desc_kmajor_none(ptx::smem_u32(cfs), 128, 256),
                                          ptx::desc_kmajor_none(ptx::smem_u32(bts), 128, 256),
                                          ptx::idesc_tf32(RB, kDstate), 0);
                        }
                    }
                    if (ok) {
                        // Tile accumulators (and the commit product) full; M_h and cf free.
                        ptx::mma_commit(bar(B_ACCF + a));
                        ptx::mma_commit(bar(B_MHE));
                    }
                }
                if (tcc) ++ncm;
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
            if (ok && misc[M_DTK] != (int)k + 1) {             // not already read by the switch
                if (dnext_k == (int)k) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (ptid + u * kPrepThreads < hpt * T) dts[ptid + u * kPrepThreads] = bf2f(dnext[u]);
                } else {
                    for (int q = ptid; q < hpt * T; q += kPrepThreads) {
                        const int hh = q / T, i = q - hh * T;
                        dts[q] = bf2f(p.dt[((size_t)b * T + i) * H + hfirst + hh]);
                    }
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
                // (The failure-path test hook withholds this arrival for the first
                // tile, so that the epilogue's bounded wait runs out.)
                if (!(p.fault == 1 && k == 0)) mbar_arrive(bar(B_COEFF + c));
                // Masked decay matrix of every head of the tile (bf16, K-major swizzled):
                // M_h[i][j] = exp(L_i - L_j) (C_i . B_j) dt_j for j an ancestor-or-self of i,
                // plus D_h on the diagonal, so that the tree MMA also yields the skip term.
                if (ptid == 0 && k > 0) wait(bar(B_MHE), (k - 1) & 1, 32);
                named_sync(kBarPrep, kPrepThreads);
                ok = !misc[M_ABORT];
                if (ok) {
                    const int total = misc[M_TOTAL];
                    if (misc[M_INSMEM] == 1) {
                        for (int q = ptid; q < hpt * total; q += kPrepThreads) {
                            const int hh = q / total, qq = q - hh * total;
                            const int i = pi[qq], j = pj[qq];
                            float m = expf(Ls[hh * T + i] - Ls[hh * T + j]) * pcb[qq] * dts[hh * T + j];
                            if (i == j) m += Dsh[hfirst + hh];            // skip term D_h x_i
                            *reinterpret_cast<__nv_bfloat16 *>(mh + hh * p.mh_head + k_off(i, j, T_pad)) =
                                __float2bfloat16_rn(m);
                        }
                    } else if (misc[M_INSMEM] == 2) {
                        // Row order: kRowParts threads per (head, node) take every
                        // kRowParts-th of its ancestors (no per-pair index search).
                        constexpr int kRowParts = 3;
                        for (int it = ptid; it < hpt * T * kRowParts; it += kPrepThreads) {
                            const int hh = it / (T * kRowParts), rem = it - hh * T * kRowParts;
                            const int i = rem / kRowParts, part = rem - i * kRowParts;
                            const float Li = Ls[hh * T + i];
                            int q = poff[i], k = 0;
                            for (int w = 0; w < W; ++w) {
                                uint32_t bits = ancs[i * W + w];
                                while (bits) {
                                    const int j = (w << 5) + __ffs(bits) - 1;
                                    bits &= bits - 1;
                                    if (k == part) {
                                        float m = expf(Li - Ls[hh * T + j]) * __bfloat162float(pcb16[q]) *
                                                  dts[hh * T + j];
                                        if (i == j) m += Dsh[hfirst + hh];
                                        *reinterpret_cast<__nv_bfloat16 *>(mh + hh * p.mh_head +
                                                                           k_off(i, j, T_pad)) = __float2bfloat16_rn(m);
                                    }
                                    ++q;
                                    k = k == kRowParts - 1 ? 0 : k + 1;
                                }
                            }
                        }
                    } else {
                        const float *pg = p.pcb_g ? p.pcb_g + (size_t)blockIdx.x * p.pair_max : nullptr;
                        for (int q = ptid; q < hpt * total; q += kPrepThreads) {
                            const int hh = q / total, qq = q - hh * total;
                            const int i = pair_row(poff, T, qq);
                            const int j = nth_set_bit(ancs + i * W, W, qq - poff[i]);
                            const float cb = pg ? (qq < p.pair_max ? pg[qq] : 0.f)
                                                : dot_cb(cs, T_pad, Bseq + (size_t)j * brow, i);
                            float m = expf(Ls[hh * T + i] - Ls[hh * T + j]) * cb * dts[hh * T + j];
                            if (i == j) m += Dsh[hfirst + hh];
                            *reinterpret_cast<__nv_bfloat16 *>(mh + hh * p.mh_head + k_off(i, j, T_pad)) =
                                __float2bfloat16_rn(m);
                        }
                    }
                    ptx::fence_proxy_async_smem();
                    mbar_arrive(bar(B_MHF));
                    // dt of the next tile when it belongs to the same (sequence, group)
                    // (a switch reads its own); hpt * T <= 512 values.
                    const int t1 = t + 1, b1 = t1 / p.tps, hf1 = (t1 % p.tps) * RB / P;
                    if (t1 < end && b1 * G + hf1 / hpg == key) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int q = ptid + u * kPrepThreads, hh = q / T, i = q - hh * T;
                            if (q < hpt * T) dnext[u] = p.dt[((size_t)b1 * T + i) * H + hf1 + hh];
                        }
                        dnext_k = (int)k + 1;
                    }
                    if (tcc) {
                        // Coefficients of the commit product, once the tile's x has landed:
                        // cf[row][q] = w_q x[pnode_q][row] for q < len, 0 past the path
                        // (K-major fp32, no swizzle).  The previous product was read by its
                        // MMA before this tile's M_h region was released.
                        if (ptid == 0) wait(bar(B_FULL + s), sph, 33);
                        named_sync(kBarPrep, kPrepThreads);
                        if (!misc[M_ABORT]) {
                            for (int it = ptid; it < RB * 2; it += kPrepThreads) {
                                const int row = it % RB, kc = it / RB;
                                const int hh = (r0 + row) / P - hfirst;
                                const MnCol xc(row, xbs);
                                float v[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int q = 4 * kc + e;
                                    const int j = q < len ? (int)pnode[q] : 0;
                                    const float xv = bf2f(*reinterpret_cast<const __nv_bfloat16 *>(xt + xc.at(j)));
                                    v[e] = q < len ? wts[hh * T + q] * xv : 0.f;
                                }
                                *reinterpret_cast<float4 *>(cfs + k8_off(row, 4 * kc)) = make_float4(v[0], v[1], v[2], v[3]);
                            }
                            ptx::fence_proxy_async_smem();
                            mbar_arrive(bar(B_CFF));
                        }
                    }
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
            if (run) ptx::tc_fence_after();
            const float *eLs = coef(c, 2), *wts = coef(c, 3), *alpha = coef(c, 4);
            if (run && commit && !tcc) {
                const int tpr = kEpiThreads / RB;                  // threads per row: 2 or 4
                const int row = etid % RB, part = etid / RB;
                const int hh = (r0 + row) / P - hfirst;
                const MnCol xc(row, xbs);
                const int cols = kDstate / tpr;
                for (int c_lo = part * cols; c_lo < (part + 1) * cols; c_lo += 32)
                    commit_rows<32>(h0t, xt, xc, Bp, p.tc_commit ? 0 : kPathRows, Bseq, brow, pnode, wts + hh * T,
                                    alpha[hh], len, RB, row, c_lo);
            }
            named_sync(kBarEpi, kEpiThreads);                  // x rows of the path are read
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
                    float E[8];
                    lds_f32x8(ea, E);
                    uint16_t Yh[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float yv = fmaf(E[u], __uint_as_float(R[u]), __uint_as_float(Y[u]));
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
            if (tcc && run) {
                // h_new = alpha h0 + D, D read from tensor memory (same lane mapping as y).
                {
                    ptx::tc_fence_after();
                    const int hh = (r0 + row) / P - hfirst;
                    const float2 a2 = make_float2(alpha[hh], alpha[hh]);
                    const uint32_t td = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(p.cm_col + half * 64);
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 32) {
                        uint32_t d0[16], d1[16];
                        ptx::tmem_ld16_nowait(td + (uint32_t)c0, d0);
                        ptx::tmem_ld16_nowait(td + (uint32_t)(c0 + 16), d1);
                        ptx::tmem_wait_ld();
                        if (active) {
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const int n = half * 64 + c0 + 4 * u;
                                const int kb = n >> 5, ch = (n & 31) >> 2;
                                float4 *hp = reinterpret_cast<float4 *>(h0t + kb * RB * 128 + row * 128 +
                                                                        ((ch ^ (row & 7)) << 4));
                                const float4 h = *hp;
                                const uint32_t *dv = u < 4 ? d0 + 4 * u : d1 + 4 * (u - 4);
                                const float2 lo = ffma2(a2, make_float2(h.x, h.y),
                                                        make_float2(__uint_as_float(dv[0]), __uint_as_float(dv[1])));
                                const float2 hi = ffma2(a2, make_float2(h.z, h.w),
                                                        make_float2(__uint_as_float(dv[2]), __uint_as_float(dv[3])));
                                *hp = make_float4(lo.x, lo.y, hi.x, hi.y);
                            }
                        }
                    }
                }
                // This warp's reads of the commit product are done: the next one may be issued.
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_CME));
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (run && lane == 0) {
                mbar_arrive(bar(B_ACCE + a));
                mbar_arrive(bar(B_COEFE + c));
            }
            ptx::fence_proxy_async_smem();
            named_sync(kBarEpi, kEpiThreads);
            if (run && etid == 0) {
                misc[M_SDESC + 2 * s] = t;                     // the producer issues the stores
                misc[M_SDESC + 2 * s + 1] = (misc[M_OK] ? 1 : 0) | (commit ? 2 : 0);
                mbar_arrive(bar(B_EPID + s));
            }
        }
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
    if (warp == kMmaWarp && lane == 0 && misc[M_ABORT]) {
        // After an abort some issued MMAs may have no commit: wait (bounded) until
        // every MMA of this thread has completed before the tensor memory is freed.
        ptx::mma_commit(bar(B_DRAIN));
        ptx::mbar_wait(bar(B_DRAIN), 0);
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

constexpr int kMaxDevices = 64;

// Per-device facts looked up once: the SM count, and whether the kernel's
// shared-memory limit has been raised on that device.
struct DeviceInfo {
    int sms = 0;
    bool prepared = false;
};
std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < kMaxDevices) {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        if (g_dev[dev].sms > 0) return g_dev[dev].sms;
    }
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    if (dev >= 0 && dev < kMaxDevices) {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        g_dev[dev].sms = n;
    }
    return n;
}

// Raises the dynamic shared-memory limit of the kernel to the largest layout
// (once per device; later launches need no attribute call).
cudaError_t prepare_device()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (g_dev[dev].prepared) return cudaSuccess;
    e = cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    g_dev[dev].prepared = true;
    return cudaSuccess;
}

uint32_t round_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

struct TcPlan {
    TcParams p;
    size_t smem;
    int grid;
};

// Shared-memory and tensor-memory layout for a tile height RB, S stages, (stage_b)
// the B rows of a (sequence, group) kept in shared memory and (tcc) the commit
// product on the tensor cores; false if it does not fit.
bool layout(const ScanArgs &a, int RB, int S, bool stage_b, bool tcc, TcParams &p, size_t &smem)
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
    p.off_bp = 0;                      // fp32 path rows of B for the CUDA-core commit
    if (!tcc) {
        p.off_bp = round_up(off, 16u);
        off = p.off_bp + (uint32_t)kPathRows * kDstate * 4u;
    }
    p.off_anc = round_up(off, 16u);    off = p.off_anc + (uint32_t)T * W * 4u;
    p.off_poff = round_up(off, 16u);   off = p.off_poff + (uint32_t)(T + 1) * 4u;
    p.coef_slot = round_up((uint32_t)(4 * hpt * T + hpt) * 4u, 16u);
    p.off_coef = round_up(off, 16u);   off = p.off_coef + 2u * p.coef_slot;
    p.off_pnode = round_up(off, 16u);  off = p.off_pnode + (uint32_t)T * 2u;
    p.off_praw = round_up(off, 16u);   off = p.off_praw + (uint32_t)T * 4u;
    p.off_par = round_up(off, 16u);    off = p.off_par + (uint32_t)T * 4u;
    p.off_dep = round_up(off, 16u);    off = p.off_dep + (uint32_t)T * 4u;
    // B rows of a (sequence, group), bf16: a region of their own, else (when it
    // is large enough) the masked-decay region, which is free during a switch.
    p.off_bs = 0;
    p.bs_mh = 0;
    if (stage_b) {
        p.off_bs = round_up(off, 16u);
        off = p.off_bs + (uint32_t)T * kDstate * 2u;
    } else if ((uint32_t)hpt * p.mh_head >= (uint32_t)T * kDstate * 2u) {
        p.off_bs = p.off_mh;
        p.bs_mh = 1;
    }
    p.off_cf = p.off_bt = 0;           // operands of the commit MMA (K = 8, fp32)
    if (tcc) {
        p.off_cf = round_up(off, 128u);
        off = p.off_cf + (uint32_t)RB * 32u;
        p.off_bt = round_up(off, 128u);
        off = p.off_bt + (uint32_t)kDstate * 32u;
    }
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
    // Tensor memory: two accumulator sets (root term, tree term of each head), then
    // the commit product (128 columns) when it runs on the tensor cores.
    p.acc_cols = (1 + hpt) * T_pad;
    p.cm_col = 2 * p.acc_cols;
    p.tc_commit = tcc ? 1 : 0;
    const uint32_t need = (uint32_t)p.cm_col + (tcc ? (uint32_t)kDstate : 0u);
    uint32_t cols = 32;
    while (cols < need) cols <<= 1;
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
        if (!rb_valid(a, RB)) continue;
        const int all_pairs = a.T * (a.T + 1) / 2;
        TcParams p{};
        size_t smem = 0;
        bool fits = false;
        // Preference: the commit product on the tensor cores, then B rows in a
        // shared-memory region of their own.
        for (int tcc = 1; tcc >= 0 && !fits; --tcc)
            for (int stage_b = 1; stage_b >= 0 && !fits; --stage_b)
                fits = layout(a, RB, S, stage_b != 0, tcc != 0, p, smem) &&
                       (p.pair_cap >= all_pairs || p.pair_cap >= 4 * a.T);
        if (!fits) continue;                                      // typical trees must fit
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
    best.tpg = (a.H / a.G) * a.P / chosen;          // whole tiles: rb_valid keeps groups tile-aligned
    best.sw_milli = 1500;                           // a switch costs about one and a half tiles
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

size_t tc_pair_scratch_floats(const ScanArgs &a)
{
    TcPlan pl;
    if (!plan(a, pl)) return 0;
    const long long pairs = (long long)a.T * (a.T + 1) / 2;
    if (pl.p.pair_cap >= pairs) return 0;
    long long grid = num_sms();
    if (grid > pl.p.ntiles) grid = pl.p.ntiles;
    return (size_t)grid * (size_t)pairs;
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
    p.parent = a.parent;
    p.pre = a.parent != nullptr;
    p.tree = a.tree;
    p.tree_anc = a.tree_anc;
    p.tree_depth = a.tree_depth;
    p.tree_ok = a.tree_ok;
    p.wait_ns = a.wait_ns ? a.wait_ns : ptx::kWaitLimitNs;
    p.fault = a.fault;
    p.err = a.err;
    if (a.pair_scratch && tc_pair_scratch_floats(a) > 0) {
        p.pcb_g = a.pair_scratch;
        p.pair_max = a.T * (a.T + 1) / 2;
    }

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
    cudaError_t e = prepare_device();
    if (e != cudaSuccess) return e;
    // 512 threads at 128 registers leave room for one CTA per SM.
    long long grid = num_sms();
    if (grid > p.ntiles) grid = p.ntiles;
    // Programmatic dependent launch: the kernel waits for the preceding grid
    // before its first global read (at entry with parent[] given, after the
    // barrier and tensor-memory set-up otherwise), so that much overlaps the
    // preceding grid's tail.
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
