// k_gdn_tc.cu -- the gated delta rule over the packed draft tree on tcgen05, for
// bf16 q/k/v with d_k = d_v = 128 and up to 64 nodes, sm_100a.
//
// The rule and its packed form are those of k_gdn.cu ("TreeWY" abstract: every
// draft node's output from one triangular solve, only the accepted state rebuilt on
// commit from the pseudo-values; "Bole" abstract: the tree-structured closed form):
//   u_j   = beta_j v_j - a_j gamma_j S0 k_j - sum_{l strict ancestor of j} a_j (gamma_j / gamma_l) (k_j . k_l) u_l
//   o_i   = gamma_i S0 q_i + sum_{j in anc(i)} (gamma_i / gamma_j) (q_i . k_j) u_j
//   S_new = gamma_leaf S0 + sum_{j on path} (gamma_leaf / gamma_j) u_j k_j^T
// with gamma_i the product of alpha over the root path of i and a the erase
// strength (a = beta unless given).
//
// Design (B200).  One CTA per (sequence, value head) holds the whole state S0
// [128 x 128] fp32 (one TMA box, the 128-byte-swizzled K-major operand layout); q, k
// and v arrive as bf16 TMA boxes beside it.  Every dense contraction of the rule
// runs as one tf32 product on the tensor cores into tensor memory: R = S0 [Q;K]^T
// (the root terms S0 q_i and S0 k_i of every node; M = 128 state rows, N = 128),
// P = [Q;K] K^T (q_i . k_j and k_i . k_j of every node pair; M = 128, N = 64), q and
// k widened to fp32 in the same operand layout (bf16 values are exact in tf32, so
// only S0 is rounded, as in the SSM scan's root term).  The pair products are
// weighted and masked to the ancestor relation: the q weights as a K-major operand
// (row i), the k weights as [l][j] (row l holds node l's weight in every later node)
// for the solve.  Then each of the 128 threads owns one state row and solves for its
// column of the pseudo-values in blocks of up to 32 nodes held in registers,
// right-looking (node l's value is final once the earlier nodes of its block are
// folded in, and is then folded into the later ones with two-wide fp32 FMAs); the
// first block reaches the second through one more tf32 product.  The outputs are a
// fourth product, U^T x (the q weights)^T, beside which the threads rebuild their
// rows of the accepted state in place over the S0 tile; outputs and state leave by
// TMA stores.  Waits are bounded; a timeout latches STREE_ERR_TIMEOUT and the CTA
// drains its copies and products before it exits.
#include <cuda.h>

#include <climits>
#include <mutex>

#include "stree_internal.cuh"
#include "tc_ptx.cuh"

namespace stree {
namespace {

constexpr int kD = 128;                      // d_k = d_v
constexpr int kTP = 64;                      // nodes padded to 64 (N of P, half of M)
constexpr int kGThreads = 128;               // one thread per state row
constexpr int kMaxDevices = 64;
constexpr uint32_t kRowBytes = kD * 2;       // one bf16 row of q, k or v
// Tensor-memory columns (256 allocated): R = [S0 q_i | S0 k_j], then P, reused for
// the output product, then the second solve block's sums from the first.
constexpr uint32_t kColRq = 0, kColRk = kTP, kColP = 2 * kTP, kColAcc = 3 * kTP;

struct GdnTcLayout {
    static constexpr uint32_t s0 = 0;                            // [4 atoms][128 rows][128 B] fp32
    static constexpr uint32_t qk = s0 + 65536;                   // [4 atoms][128 rows: q 0-63, k 64-127][128 B]
    static constexpr uint32_t u = qk + 65536;                    // [2 atoms][128 rows][128 B] U^T; first the bf16 q, k boxes
    static constexpr uint32_t mq = u + kTP * kD * 4;             // [2 atoms][64 i][128 B] (gamma_i/gamma_l) q_i . k_l, l in anc(i)
    static constexpr uint32_t ak = mq + kTP * kTP * 4;           // [64 l][64 j] (gamma_j/gamma_l) k_j . k_l, l strict anc of j
    static constexpr uint32_t ak2 = ak + kTP * kTP * 4;          // [32 j - 32][128 B: l < 32] the same, K-major
    static constexpr uint32_t v = ak2 + 32 * 128;                // [64 nodes][128] bf16
    static constexpr uint32_t nodef = v + kTP * kD * 2;          // 6 x [64] fp32: las, lg, eg, be, er, wq
    static constexpr uint32_t nodei = nodef + 6 * kTP * 4;       // 6 x [64] int32: par, dep, praw, pnode, anc0, anc1
    static constexpr uint32_t misc = nodei + 6 * kTP * 4;        // [16] int32
    static constexpr uint32_t bars = misc + 16 * 4;              // 5 mbarriers
    static constexpr uint32_t total = bars + 5 * 8 + 1024;       // + alignment slack
};
static_assert(GdnTcLayout::total <= 232448, "shared memory of the gated-delta-rule CTA");
static_assert(2 * kTP * kRowBytes <= kTP * kD * 4, "the q and k boxes fit in the pseudo-value region");

enum GMisc { T_TMEM = 0, T_OK, T_LEN, T_PATHOK, T_BADI, T_BADQ, T_ABORT };

struct GdnTcParams {
    const float *alpha, *beta, *erase;
    const int32_t *parent, *path, *path_len;
    int maxlen;
    int32_t *err;
    int T, Hv, Hk, do_commit;
};

__device__ __forceinline__ void latch_opt(int32_t *err, int code, int b, int pos, int detail)
{
    if (err) latch_error(err, code, b, pos, detail);
}

// fp32 element (row, c) of a [4 atoms][rows][128 B] K-major swizzled operand: the
// 16-byte chunk of four columns starting at 4 * (c / 4).
__device__ __forceinline__ uint32_t kmaj_chunk(int row, int chunk, int rows)
{
    return (uint32_t)(chunk >> 3) * (uint32_t)rows * 128u + (uint32_t)row * 128u +
           ((uint32_t)((chunk & 7) ^ (row & 7)) << 4);
}

// N consecutive tensor-memory columns of this thread's lane.
template <int N>
__device__ __forceinline__ void tmem_cols(uint32_t taddr, uint32_t (&r)[N])
{
    static_assert(N == 16 || N == 32 || N == 64, "column count");
    if constexpr (N == 16) {
        ptx::tmem_ld16_nowait(taddr, r);
        ptx::tmem_wait_ld();
    } else if constexpr (N == 32) {
        ptx::tmem_ld32(taddr, r);
    } else {
        ptx::tmem_ld64(taddr, r);
    }
}

// TB: the node count rounded up to 16, 32 or 64 (registers of the right-looking solve).
template <int TB>
__global__ void __launch_bounds__(kGThreads, 1)
gdn_tc_kernel(const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_sn,
              const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const GdnTcParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s0t = sm + GdnTcLayout::s0;
    uint8_t *qkt = sm + GdnTcLayout::qk;
    uint8_t *Ub = sm + GdnTcLayout::u;
    const uint8_t *qk16 = sm + GdnTcLayout::u;                   // bf16 q rows, then k rows at +kTP rows
    uint8_t *Mqb = sm + GdnTcLayout::mq;
    float *AkT = reinterpret_cast<float *>(sm + GdnTcLayout::ak);
    uint8_t *Ak2b = sm + GdnTcLayout::ak2;
    __nv_bfloat16 *vs = reinterpret_cast<__nv_bfloat16 *>(sm + GdnTcLayout::v);
    float *las = reinterpret_cast<float *>(sm + GdnTcLayout::nodef);
    float *lg = las + kTP, *eg = lg + kTP, *bes = eg + kTP, *ers = bes + kTP, *wq = ers + kTP;
    int32_t *par = reinterpret_cast<int32_t *>(sm + GdnTcLayout::nodei);
    int32_t *dep = par + kTP, *praw = dep + kTP, *pnode = praw + kTP;
    uint32_t *anc0 = reinterpret_cast<uint32_t *>(pnode + kTP), *anc1 = anc0 + kTP;
    volatile int32_t *misc = reinterpret_cast<volatile int32_t *>(sm + GdnTcLayout::misc);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + GdnTcLayout::bars);
    const uint32_t bar_s0 = ptx::smem_u32(&bars[0]), bar_mma = ptx::smem_u32(&bars[1]);
    const uint32_t bar_in = ptx::smem_u32(&bars[2]), bar_acc = ptx::smem_u32(&bars[3]);
    const uint32_t bar_out = ptx::smem_u32(&bars[4]);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.T, Hv = p.Hv, Hk = p.Hk;
    const int h = blockIdx.x % Hv, b = blockIdx.x / Hv;
    const int g = h / (Hv / Hk);
    const bool leader = h == 0;
    const int srow = (b * Hv + h) * kD;                          // first row of this state in S0 / S_new

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // The per-node scalars first: their latency overlaps the set-up below.
    const int plim = min(p.maxlen, T);
    int pv = 0, pr = 0, plen = 0;
    float al = 1.f, be = 0.f, er = 0.f;
    if (tid < T) {
        const size_t n = (size_t)b * T + tid;
        pv = p.parent[n];
        al = p.alpha[n * Hv + h];
        be = p.beta[n * Hv + h];
        er = p.erase ? p.erase[n * Hv + h] : be;
    }
    if (p.do_commit && tid < plim) pr = p.path[(size_t)b * p.maxlen + tid];
    if (p.do_commit && tid == 0) plen = p.path_len[b];

    if (tid == 0) {
        ptx::prefetch_tensormap(&tm_s0);
        ptx::prefetch_tensormap(&tm_sn);
        ptx::prefetch_tensormap(&tm_o);
        ptx::mbar_init(bar_s0, 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::mbar_init(bar_in, 1);
        ptx::mbar_init(bar_acc, 1);
        ptx::mbar_init(bar_out, 1);
        ptx::fence_mbar_init();
        misc[T_ABORT] = 0;
        misc[T_BADI] = INT_MAX;
        misc[T_BADQ] = INT_MAX;
        misc[T_PATHOK] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        ptx::mbar_expect_tx(bar_s0, 65536u);
        ptx::tma_load_3d(ptx::smem_u32(s0t), &tm_s0, 0, srow, 0, bar_s0);
        ptx::mbar_expect_tx(bar_in, 3u * (uint32_t)T * kRowBytes);
        ptx::tma_load_3d(ptx::smem_u32(qk16), &tm_q, 0, g, b * T, bar_in);
        ptx::tma_load_3d(ptx::smem_u32(qk16 + kTP * kRowBytes), &tm_k, 0, g, b * T, bar_in);
        ptx::tma_load_3d(ptx::smem_u32(vs), &tm_v, 0, h, b * T, bar_in);
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(const_cast<int32_t *>(&misc[T_TMEM])), 256);
        ptx::tmem_relinquish();
    }

    // ---------------------------------------------------------------- 1. per-node scalars
    if (tid < kTP) {
        par[tid] = pv;
        las[tid] = logf(al);
        bes[tid] = be;
        ers[tid] = er;
        lg[tid] = 0.f;
        eg[tid] = 0.f;
        praw[tid] = pr;
    }
    if (tid == 0) misc[T_LEN] = plen;
    __syncthreads();

    // ---------------------------------------------------------------- 2. tree and path
    int bad = 0;
    if (tid < T) {
        const int v = par[tid];
        bad = (tid == 0) ? (v != -1) : (v < 0 || v >= tid);
        if (bad) atomicMin(const_cast<int32_t *>(&misc[T_BADI]), tid);
    }
    const bool okb = !__syncthreads_or(bad);
    if (tid < kTP) {
        uint32_t a0 = 0u, a1 = 0u;
        int d = -1;
        if (okb && tid < T) {
            for (int j = tid; j >= 0; j = par[j]) {
                if (j < 32) a0 |= 1u << j;
                else a1 |= 1u << (j - 32);
                ++d;
            }
            float sum = 0.f;                                      // ancestors in increasing index order
            for (uint32_t bits = a0; bits; bits &= bits - 1) sum += las[__ffs(bits) - 1];
            for (uint32_t bits = a1; bits; bits &= bits - 1) sum += las[32 + __ffs(bits) - 1];
            lg[tid] = sum;
            eg[tid] = expf(sum);
        }
        anc0[tid] = a0;                                           // nodes past T: no ancestors
        anc1[tid] = a1;
        dep[tid] = d;
    }
    if (!okb && leader && tid == 0) latch_opt(p.err, STREE_ERR_BAD_TREE, b, misc[T_BADI], par[misc[T_BADI]]);
    __syncthreads();
    const int len = misc[T_LEN];
    if (okb && p.do_commit) {
        if (len < 0 || len > p.maxlen || len > T) {
            if (leader && tid == 0) latch_opt(p.err, STREE_ERR_BAD_PATH, b, -1, len);
        } else {
            if (tid == 0) misc[T_PATHOK] = 1;
            __syncthreads();
            if (tid < len) {
                const int leaf = praw[len - 1];
                const int j = praw[tid];
                const bool good = leaf >= 0 && leaf < T && j >= 0 && j < T &&
                                  ((((j < 32) ? anc0[leaf] : anc1[leaf]) >> (j & 31)) & 1u) && dep[j] == tid;
                if (!good) {
                    atomicMin(const_cast<int32_t *>(&misc[T_BADQ]), tid);
                    misc[T_PATHOK] = 0;
                }
                pnode[tid] = good ? j : 0;
                wq[tid] = good ? expf(lg[leaf] - lg[j]) : 0.f;
            }
            __syncthreads();
            if (!misc[T_PATHOK] && leader && tid == 0)
                latch_opt(p.err, STREE_ERR_BAD_PATH, b, misc[T_BADQ], praw[misc[T_BADQ]]);
        }
    }

    // ---------------------------------------------------------------- 3. q and k widened to fp32
    bool in_ok = true;
    if (tid == 0) {
        in_ok = ptx::mbar_wait(bar_in, 0);
        if (!in_ok) {
            latch_opt(p.err, STREE_ERR_TIMEOUT, b, h, 2);
            misc[T_ABORT] = 1;
        }
    }
    __syncthreads();
    const bool go = okb && !misc[T_ABORT];
    if (go) {
        // Rows past T stay zero (their products are never read, but are kept finite).
#pragma unroll 8
        for (int e = tid; e < 2 * kTP * 32; e += kGThreads) {
            const int m = e >> 11, i = (e >> 5) & (kTP - 1), c = e & 31;
            float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < T) {
                const uint2 raw = *reinterpret_cast<const uint2 *>(qk16 + (m * kTP + i) * kRowBytes + 8 * c);
                const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
                const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
                f = make_float4(lo.x, lo.y, hi.x, hi.y);
            }
            *reinterpret_cast<float4 *>(qkt + kmaj_chunk(m * kTP + i, c, 2 * kTP)) = f;
        }
    }

    // ---------------------------------------------------------------- 4. the two products
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = static_cast<uint32_t>(misc[T_TMEM]);
    bool mma_issued = false;
    if (go && tid == 0) {
        if (ptx::mbar_wait(bar_s0, 0)) {
            ptx::tc_fence_after();
            const uint32_t a0 = ptx::smem_u32(s0t), q0 = ptx::smem_u32(qkt);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    ptx::mma_tf32(tmem, ptx::desc_kmajor_sw128(a0 + kb * kD * 128 + kk * 32),
                                  ptx::desc_kmajor_sw128(q0 + kb * 2 * kTP * 128 + kk * 32), ptx::idesc_tf32(kD, 2 * kTP),
                                  (kb | kk) != 0);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    ptx::mma_tf32(tmem + 2 * kTP, ptx::desc_kmajor_sw128(q0 + kb * 2 * kTP * 128 + kk * 32),
                                  ptx::desc_kmajor_sw128(q0 + kb * 2 * kTP * 128 + kTP * 128 + kk * 32),
                                  ptx::idesc_tf32(2 * kTP, kTP), (kb | kk) != 0);
            ptx::mma_commit(bar_mma);
            mma_issued = true;
        } else {
            latch_opt(p.err, STREE_ERR_TIMEOUT, b, h, 0);
            misc[T_ABORT] = 1;
        }
    }
    bool run = go;
    if (go) {
        if (lane == 0) {
            run = !misc[T_ABORT];
            if (run && !ptx::mbar_wait(bar_mma, 0)) {
                latch_opt(p.err, STREE_ERR_TIMEOUT, b, h, 1);
                misc[T_ABORT] = 1;
                run = false;
            }
        }
        run = __shfl_sync(0xffffffffu, run ? 1 : 0, 0) != 0;
        __syncthreads();
        run = run && !misc[T_ABORT];
    }
    if (run) ptx::tc_fence_after();
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;       // this warp's tensor-memory lanes
    const int row = tid;
    // A product's completion seen by every warp (lane 0 waits, bounded); false for the
    // whole CTA once any wait has run out.
    auto wait_all = [&](uint32_t bar, int where) -> bool {
        bool ok = true;
        if (lane == 0 && !ptx::mbar_wait(bar, 0)) {
            latch_opt(p.err, STREE_ERR_TIMEOUT, b, h, where);
            misc[T_ABORT] = 1;
            ok = false;
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        __syncthreads();
        ok = ok && !misc[T_ABORT];
        if (ok) ptx::tc_fence_after();
        return ok;
    };

    // ---------------------------------------------------------------- 5. pair weights
    // Thread t holds row t of P: q_i . k_l (t = i < 64) or k_j . k_l (t = 64 + j), and
    // weights and masks it to the ancestor relation: row i of Mq in the K-major
    // operand layout (16-byte chunks of its own row), column j of AkT [l][j] for the
    // solve (consecutive threads, consecutive words) and, with two blocks, row j - 32
    // of the first block's columns in the K-major layout for the product between them.
    if (run) {
        uint32_t pv[TB];
        tmem_cols<TB>(tmem + kColP + lane_base, pv);
        const int i = row & (kTP - 1);
        const bool is_k = row >= kTP;
        uint32_t a0 = anc0[i], a1 = anc1[i];                      // zero past T
        if (is_k) {                                               // strict ancestors for the solve
            if (i < 32) a0 &= ~(1u << i);
            else a1 &= ~(1u << (i - 32));
        }
        const float li = lg[i];
#pragma unroll
        for (int c = 0; c < TB / 4; ++c) {
            float w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int l = 4 * c + e;
                const bool anc = ((l < 32 ? a0 : a1) >> (l & 31)) & 1u;
                const float x = anc ? li - lg[l] : -INFINITY;     // exp(-inf) = 0 off the relation
                w[e] = expf(x) * __uint_as_float(pv[l]);
            }
            if (!is_k) {
                *reinterpret_cast<float4 *>(Mqb + kmaj_chunk(i, c, kTP)) = make_float4(w[0], w[1], w[2], w[3]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) AkT[(4 * c + e) * kTP + i] = w[e];
                if (TB == kTP && i >= 32 && c < 8)
                    *reinterpret_cast<float4 *>(Ak2b + kmaj_chunk(i - 32, c, 32)) = make_float4(w[0], w[1], w[2], w[3]);
            }
        }
    }

    // ---------------------------------------------------------------- 6. solve (one state row per thread)
    // Blocks of BS nodes in registers, right-looking: node l's pseudo-value is final once
    // every earlier node of its block has been folded in (earlier blocks arrive through
    // one tensor-core product, D_acc = U[block 0] x AkT[block 0][block 1]), and is then
    // folded into the pending sums of the later nodes of the block.  Pseudo-values of
    // nodes past T are zero (the output product runs over whole 8-node groups).
    constexpr int BS = TB < 32 ? TB : 32;
    constexpr int NB = TB / BS;
    bool acc_issued = false, out_issued = false;
    if (run) {
        const bool erase = p.erase != nullptr;
        for (int blk = 0; blk < NB; ++blk) {
            const int jb0 = blk * BS;
            if (blk > 0) {
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                __syncthreads();
                if (tid == 0) {
                    ptx::tc_fence_after();
#pragma unroll
                    for (int s = 0; s < BS / 8; ++s)             // K = the first block's 32 nodes, one atom
                        ptx::mma_tf32(tmem + kColAcc, ptx::desc_kmajor_sw128(ptx::smem_u32(Ub) + s * 32),
                                      ptx::desc_kmajor_sw128(ptx::smem_u32(Ak2b) + s * 32), ptx::idesc_tf32(kD, BS),
                                      s != 0);
                    ptx::mma_commit(bar_acc);
                    acc_issued = true;
                }
                if (!wait_all(bar_acc, 3)) break;
            }
            float2 acc[BS / 2];
            {
                uint32_t r[BS];
                tmem_cols<BS>(tmem + kColRk + jb0 + lane_base, r);   // S0 k_j
#pragma unroll
                for (int j = 0; j < BS; j += 2)
                    acc[j / 2] = make_float2(eg[jb0 + j] * __uint_as_float(r[j]), eg[jb0 + j + 1] * __uint_as_float(r[j + 1]));
                if (blk > 0) {
                    tmem_cols<BS>(tmem + kColAcc + lane_base, r);
#pragma unroll
                    for (int j = 0; j < BS; j += 2)
                        acc[j / 2] = make_float2(acc[j / 2].x + __uint_as_float(r[j]), acc[j / 2].y + __uint_as_float(r[j + 1]));
                }
            }
            float ub[4];
#pragma unroll
            for (int ll = 0; ll < BS; ++ll) {
                const int l = jb0 + ll;
                const float vl = __bfloat162float(vs[l * kD + row]);
                const float al = (ll & 1) ? acc[ll / 2].y : acc[ll / 2].x;
                float ul = erase ? bes[l] * vl - ers[l] * al : bes[l] * (vl - al);
                ul = l < T ? ul : 0.f;
                ub[ll & 3] = ul;
                if ((ll & 3) == 3)                                // row `row` of U^T, K-major, 4 nodes a chunk
                    *reinterpret_cast<float4 *>(Ub + kmaj_chunk(row, l >> 2, kD)) = make_float4(ub[0], ub[1], ub[2], ub[3]);
                const float2 u2 = make_float2(ul, ul);
                // Entries with j <= l are zero, so whole aligned 4-node chunks are folded in.
#pragma unroll
                for (int jj = (ll / 4) * 4; jj < BS; jj += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(AkT + l * kTP + jb0 + jj);
                    acc[jj / 2] = ptx::ffma2(make_float2(a4.x, a4.y), u2, acc[jj / 2]);
                    acc[jj / 2 + 1] = ptx::ffma2(make_float2(a4.z, a4.w), u2, acc[jj / 2 + 1]);
                }
            }
        }
        run = !misc[T_ABORT];
    }

    // ---------------------------------------------------------------- 7. outputs on the tensor cores
    // D_out = U^T Mq^T over whole 8-node groups: M = 128 state rows, N = TB outputs.
    if (run) {
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            ptx::tc_fence_after();
            const int ks = (T + 7) / 8;
            for (int s = 0; s < ks; ++s)
                ptx::mma_tf32(tmem + kColP, ptx::desc_kmajor_sw128(ptx::smem_u32(Ub) + (s >> 2) * kD * 128 + (s & 3) * 32),
                              ptx::desc_kmajor_sw128(ptx::smem_u32(Mqb) + (s >> 2) * kTP * 128 + (s & 3) * 32),
                              ptx::idesc_tf32(kD, TB), s != 0);
            ptx::mma_commit(bar_out);
            out_issued = true;
        }

        // ------------------------------------------------------------ 8. commit (in place over S0), beside the product
        if (misc[T_PATHOK]) {
            const float gl = len > 0 ? eg[pnode[len - 1]] : 1.f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float2 s[32];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float4 h4 = *reinterpret_cast<const float4 *>(s0t + kmaj_chunk(row, 16 * half + c, kD));
                    s[2 * c] = make_float2(gl * h4.x, gl * h4.y);
                    s[2 * c + 1] = make_float2(gl * h4.z, gl * h4.w);
                }
                for (int q = 0; q < len; ++q) {
                    const int j = pnode[q];
                    const float cf = wq[q] * *reinterpret_cast<const float *>(Ub + kmaj_chunk(row, j >> 2, kD) + (j & 3) * 4);
                    const float2 c2 = make_float2(cf, cf);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float4 kq =
                            *reinterpret_cast<const float4 *>(qkt + kmaj_chunk(kTP + j, 16 * half + c, 2 * kTP));
                        s[2 * c] = ptx::ffma2(make_float2(kq.x, kq.y), c2, s[2 * c]);
                        s[2 * c + 1] = ptx::ffma2(make_float2(kq.z, kq.w), c2, s[2 * c + 1]);
                    }
                }
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    *reinterpret_cast<float4 *>(s0t + kmaj_chunk(row, 16 * half + c, kD)) =
                        make_float4(s[2 * c].x, s[2 * c].y, s[2 * c + 1].x, s[2 * c + 1].y);
            }
        }

        // ------------------------------------------------------------ 9. outputs: gamma_i S0 q_i + D_out
        // Staged as [T][128] bf16 over v (read by the solve only), stored by one TMA box.
        if (wait_all(bar_out, 4)) {
#pragma unroll
            for (int i0 = 0; i0 < TB; i0 += BS) {
                uint32_t rq[BS], d[BS];
                tmem_cols<BS>(tmem + kColRq + i0 + lane_base, rq);
                tmem_cols<BS>(tmem + kColP + i0 + lane_base, d);
#pragma unroll
                for (int ii = 0; ii < BS; ++ii) {
                    const int i = i0 + ii;
                    if (i < T)
                        vs[i * kD + row] =
                            __float2bfloat16_rn(fmaf(eg[i], __uint_as_float(rq[ii]), __uint_as_float(d[ii])));
                }
            }
        }
        run = !misc[T_ABORT];
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        if (run) {
            ptx::tma_store_3d(&tm_o, 0, h, b * T, ptx::smem_u32(vs));
            if (misc[T_PATHOK]) ptx::tma_store_3d(&tm_sn, 0, srow, 0, ptx::smem_u32(s0t));
            ptx::bulk_commit();
            ptx::bulk_wait_read_all();
        }
        if (!in_ok) ptx::mbar_wait(bar_in, 0);                    // the input boxes may still land
        if (!mma_issued) ptx::mbar_wait(bar_s0, 0);               // and the state box
        if (misc[T_ABORT]) {                                      // and products still in flight
            if (mma_issued) ptx::mbar_wait(bar_mma, 0);
            if (acc_issued) ptx::mbar_wait(bar_acc, 0);
            if (out_issued) ptx::mbar_wait(bar_out, 0);
        }
    }
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 256);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn gdn_encode_fn()
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

// A [rows][128] fp32 state as [4 groups of 32 columns][rows][32]: one box is a
// whole 128-row state in the K-major layout of the MMA (four 128-byte-swizzled atoms).
bool encode_state(EncodeTiledFn enc, CUtensorMap *m, const float *base, long long rows)
{
    cuuint64_t dims[3] = {32, (cuuint64_t)rows, kD / 32};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 4, 128};
    cuuint32_t box[3] = {32, (cuuint32_t)kD, kD / 32};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A [positions][heads][128] bf16 tensor; one box is the T rows of one head of one
// sequence, landing as [T][128] (row-major, unswizzled).
bool encode_rows(EncodeTiledFn enc, CUtensorMap *m, const void *base, long long positions, int heads, int T)
{
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)heads, (cuuint64_t)positions};
    cuuint64_t strides[2] = {(cuuint64_t)kRowBytes, (cuuint64_t)heads * kRowBytes};
    cuuint32_t box[3] = {(cuuint32_t)kD, 1, (cuuint32_t)T};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::mutex g_mutex;
bool g_prepared[kMaxDevices] = {};

cudaError_t prepare()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_prepared[dev]) return cudaSuccess;
    const int bytes = (int)GdnTcLayout::total;
    if ((e = cudaFuncSetAttribute(gdn_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
            cudaSuccess ||
        (e = cudaFuncSetAttribute(gdn_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
            cudaSuccess ||
        (e = cudaFuncSetAttribute(gdn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
            cudaSuccess)
        return e;
    g_prepared[dev] = true;
    return cudaSuccess;
}

}  // namespace

bool gdn_tc_supported(int n_nodes, int dk, int dv, stree_dtype dtype)
{
    return dtype == STREE_BF16 && dk == kD && dv == kD && n_nodes >= 1 && n_nodes <= kTP && gdn_encode_fn() != nullptr;
}

cudaError_t launch_gdn_tc(const void *q, const void *k, const void *v, const float *alpha, const float *beta,
                          const float *erase, const float *S0, const int32_t *parent, int n_nodes, int batch,
                          int heads_v, int heads_k, const int32_t *path, const int32_t *path_len, int maxlen, void *o,
                          float *S_new, int32_t *err, cudaStream_t s)
{
    EncodeTiledFn enc = gdn_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const long long rows = (long long)batch * heads_v * kD;
    const long long positions = (long long)batch * n_nodes;
    CUtensorMap m_s0, m_sn, m_q, m_k, m_v, m_o;
    if (!encode_state(enc, &m_s0, S0, rows) || !encode_state(enc, &m_sn, S_new ? S_new : S0, rows) ||
        !encode_rows(enc, &m_q, q, positions, heads_k, n_nodes) ||
        !encode_rows(enc, &m_k, k, positions, heads_k, n_nodes) ||
        !encode_rows(enc, &m_v, v, positions, heads_v, n_nodes) ||
        !encode_rows(enc, &m_o, o, positions, heads_v, n_nodes))
        return cudaErrorInvalidValue;
    cudaError_t e = prepare();
    if (e != cudaSuccess) return e;
    GdnTcParams p{};
    p.alpha = alpha;
    p.beta = beta;
    p.erase = erase;
    p.parent = parent;
    p.path = path;
    p.path_len = path_len;
    p.maxlen = maxlen;
    p.err = err;
    p.T = n_nodes;
    p.Hv = heads_v;
    p.Hk = heads_k;
    p.do_commit = S_new != nullptr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(batch * heads_v));
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = GdnTcLayout::total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (n_nodes <= 16) return cudaLaunchKernelEx(&cfg, gdn_tc_kernel<16>, m_s0, m_sn, m_q, m_k, m_v, m_o, p);
    if (n_nodes <= 32) return cudaLaunchKernelEx(&cfg, gdn_tc_kernel<32>, m_s0, m_sn, m_q, m_k, m_v, m_o, p);
    return cudaLaunchKernelEx(&cfg, gdn_tc_kernel<64>, m_s0, m_sn, m_q, m_k, m_v, m_o, p);
}

}  // namespace stree
