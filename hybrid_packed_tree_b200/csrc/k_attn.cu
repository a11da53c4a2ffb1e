// k_attn.cu -- tree-masked attention over the packed draft tree, tcgen05, sm_100a.
//
// The Transformer layers of a hybrid model verify the same packed tree as its SSM
// layers ("STree: Speculative Tree Decoding for Hybrid State Space Models":
// abstract, hybrid SSM and Transformer layers; scime.ai summary, "Approach": the
// packed tree sequence with a tree mask): node i attends to the whole valid
// cached context and to the tree nodes on its own root path,
//   o_i = sum_j softmax_j(scale q_i . k_j) v_j,   j in context[0, ctx_len) and anc(i).
//
// Design (B200).  The rows of a query tile are (node, query head of the group)
// pairs, so the group's heads share every key and value tile; the keys come in
// blocks of 128 -- the context blocks, then one block holding the tree's own
// keys.  One CTA takes one (sequence, key/value head, tile of 128 query rows) and
// a contiguous range of its key blocks (a split): with few sequences a long
// context is spread over several CTAs so that the grid fills the SMs, each CTA
// leaving its unnormalised partial output, row maximum and row sum in a caller
// workspace, and a second launch merging the splits (the log-sum-exp merge of
// the online softmax).  Inside a CTA, warp roles joined by bounded mbarrier waits:
//   * producer (one thread): TMA loads of the query tile (once) and of the key
//     and value blocks into two-stage rings;
//   * MMA (one thread): S = Q K^T into a double-buffered tensor-memory tile
//     (kind::f16, M = N = K-block = 128), then O += P V with V as an MN-major
//     operand (its rows are the keys), one key block behind, so that S of the
//     next block is computed while the softmax works on this one;
//   * softmax (four warps, one query row per thread, each warp on its own
//     tensor-memory lane quarter): the whole 128-score row in registers from one
//     tensor-memory load (the S buffer is released at once), the masked row
//     maximum, P = 2^(S scale log2(e) - m) in bf16 into shared memory for the
//     next MMA, the running row sum.  The reference maximum m moves only when a
//     block's maximum exceeds it by more than 2^8 (the running output and sum are
//     then rescaled together); P values stay below 256 and the quotient O / l is
//     the same softmax, so the rarely taken rescale costs no accuracy.
// The mask is applied before any maximum or exponential (masked scores are
// -inf), so nothing read past a valid length reaches the softmax; the value rows
// past the valid length of a block are zeroed in shared memory before the PV MMA
// (0 x a stale non-finite value would otherwise poison the product).
#include <cuda.h>

#include <climits>
#include <mutex>

#include "stree_internal.cuh"
#include "tc_ptx.cuh"

namespace stree {
namespace {

constexpr int kD = 128;                      // head dim
constexpr int kKB = 128;                     // keys per block
constexpr int kMRows = 128;                  // query rows per CTA
constexpr int kAttnWarps = 6;                // producer, MMA, four softmax warps
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kMaxAttnNodes = 128;
constexpr int kMaxDevices = 64;
constexpr uint32_t kTileBytes = kMRows * kD * 2;   // 32 KB: a 128 x 128 bf16 tile
constexpr uint32_t kHalfBytes = kTileBytes / 2;    // one 64-column swizzled half
constexpr float kLazyLog2 = 8.f;             // reference maximum moves when exceeded by 2^8
constexpr int kCombineThreads = 256;
constexpr int kCombineRows = 32;             // rows per combine CTA

enum AttnBars { A_QF = 0, A_KF = 1, A_KE = 3, A_VF = 5, A_VE = 7, A_SF = 9, A_SE = 11, A_PF = 13, A_OF = 14,
                A_DRAIN = 15, kAttnBars = 16 };
enum AttnMisc { AM_TMEM = 0, AM_ABORT, kAttnMisc };

struct AttnParams {
    const int32_t *ctx_len, *parent;
    __nv_bfloat16 *o;
    float *part_o;                           // [item * nsplit + split][128 rows][128] (nsplit > 1)
    float2 *part_ml;                         // [item * nsplit + split][128 rows]: (reference max, row sum)
    int32_t *err;
    int T, S, Hq, Hkv, G, TQ, mtiles;
    int nsplit, bps;                         // splits per query tile, key blocks per split
    float scale_log2;                        // scale * log2(e)
};

// Shared-memory layout (offsets from a 1024-byte aligned base).
struct AttnLayout {
    static constexpr uint32_t q = 0;
    static constexpr uint32_t k = q + kTileBytes;            // 2 stages
    static constexpr uint32_t v = k + 2 * kTileBytes;        // 2 stages
    static constexpr uint32_t pp = v + 2 * kTileBytes;       // P (bf16, K-major)
    static constexpr uint32_t anc = pp + kTileBytes;         // [128 nodes][4 words]
    static constexpr uint32_t par = anc + kMaxAttnNodes * 16;
    static constexpr uint32_t bars = par + kMaxAttnNodes * 4;
    static constexpr uint32_t misc = bars + kAttnBars * 8;
    static constexpr uint32_t total = misc + kAttnMisc * 4 + 1024;   // + alignment slack
};

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// parent[] of one sequence is a packed tree: parent[0] = -1, 0 <= parent[i] < i.
__device__ __forceinline__ bool tree_row_ok(const int32_t *par, int T, int tid, int nthreads)
{
    int bad = 0;
    for (int i = tid; i < T; i += nthreads) {
        const int v = par[i];
        bad |= (i == 0) ? (v != -1) : (v < 0 || v >= i);
    }
    return !__syncthreads_or(bad);
}

__global__ void __launch_bounds__(kAttnThreads, 1)
tree_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                      const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kt,
                      const __grid_constant__ CUtensorMap tm_vt, const AttnParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint32_t *ancs = reinterpret_cast<uint32_t *>(smem + AttnLayout::anc);
    int32_t *par = reinterpret_cast<int32_t *>(smem + AttnLayout::par);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + AttnLayout::bars);
    volatile int32_t *misc = reinterpret_cast<volatile int32_t *>(smem + AttnLayout::misc);
    auto bar = [&](int i) { return ptx::smem_u32(&bars[i]); };

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.T, G = p.G, TQ = p.TQ;
    const int sp = blockIdx.x % p.nsplit;
    const int item = blockIdx.x / p.nsplit;
    const int mt = item % p.mtiles;
    const int g = (item / p.mtiles) % p.Hkv;
    const int b = item / (p.mtiles * p.Hkv);
    const int node0 = mt * TQ;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int L = min(max(__ldg(p.ctx_len + b), 0), p.S);
    const int nctx = (L + kKB - 1) / kKB;
    const int nb = nctx + 1;                                  // context blocks, then the tree block
    const int j0 = sp * p.bps;                                // this split's key blocks: j0 .. j0 + nloc - 1
    const int nloc = max(0, min(nb, j0 + p.bps) - j0);

    auto wait = [&](uint32_t bb, uint32_t parity, int where) -> bool {
        if (misc[AM_ABORT]) return false;
        if (ptx::mbar_wait(bb, parity)) return true;
        latch_error(p.err, STREE_ERR_TIMEOUT, b, where, (int)parity);
        misc[AM_ABORT] = 1;
        return false;
    };

    if (tid == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_kc);
        ptx::prefetch_tensormap(&tm_vc);
        ptx::prefetch_tensormap(&tm_kt);
        ptx::prefetch_tensormap(&tm_vt);
        // The softmax warps arrive once each on "S read" and "P written".
        for (int i = 0; i < kAttnBars; ++i)
            ptx::mbar_init(bar(i), (i == A_SE || i == A_SE + 1 || i == A_PF) ? 4 : 1);
        ptx::fence_mbar_init();
        misc[AM_ABORT] = 0;
    }
    // The tree: parent[] of the sequence, validated, then one ancestor row per node.
    for (int i = tid; i < T; i += kAttnThreads) par[i] = __ldg(p.parent + (size_t)b * T + i);
    __syncthreads();
    const bool okb = tree_row_ok(par, T, tid, kAttnThreads);
    for (int i = tid; i < kMaxAttnNodes; i += kAttnThreads) {
        uint32_t w0 = 0u, w1 = 0u, w2 = 0u, w3 = 0u;
        if (okb && i < T)
            for (int j = i; j >= 0; j = par[j]) {
                const uint32_t bit = 1u << (j & 31), q = (uint32_t)j >> 5;
                w0 |= q == 0 ? bit : 0u;
                w1 |= q == 1 ? bit : 0u;
                w2 |= q == 2 ? bit : 0u;
                w3 |= q == 3 ? bit : 0u;
            }
        *reinterpret_cast<uint4 *>(ancs + 4 * i) = make_uint4(w0, w1, w2, w3);
    }
    if (!okb) {
        if (tid == 0 && g == 0 && mt == 0 && sp == 0) latch_error(p.err, STREE_ERR_BAD_TREE, b, -1, 0);
        return;                                               // no copy issued yet; o untouched
    }
    if (nloc == 0) {
        // A split past this sequence's last key block: an empty partial.
        if (tid < kMRows) p.part_ml[(size_t)blockIdx.x * kMRows + tid] = make_float2(-INFINITY, 0.f);
        return;
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(const_cast<int32_t *>(&misc[AM_TMEM])), 512);
        ptx::tmem_relinquish();
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = static_cast<uint32_t>(misc[AM_TMEM]);
    const uint32_t t_s = tmem, t_o = tmem + 2 * kKB;          // S: columns 0..255 (two buffers), O: 256..383

    int loads_k = 0, loads_v = 0;                             // producer: blocks whose loads were issued
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            ptx::mbar_expect_tx(bar(A_QF), kTileBytes);
            for (int hh = 0; hh < 2; ++hh)
                ptx::tma_load_3d(ptx::smem_u32(smem + AttnLayout::q + hh * kHalfBytes), &tm_q, hh * 64, g * G,
                                 b * T + node0, bar(A_QF));
            for (int i = 0; i < nloc; ++i) {
                const int j = j0 + i, s = i & 1;
                const uint32_t ph = ((i >> 1) - 1) & 1;
                if (i >= 2 && !wait(bar(A_KE + s), ph, 1)) break;
                const bool tree = j == nctx;
                const CUtensorMap *mk = tree ? &tm_kt : &tm_kc;
                const CUtensorMap *mv = tree ? &tm_vt : &tm_vc;
                const int row = tree ? b * T : b * p.S + j * kKB;
                ptx::mbar_expect_tx(bar(A_KF + s), kTileBytes);
                for (int hh = 0; hh < 2; ++hh)
                    ptx::tma_load_3d(ptx::smem_u32(smem + AttnLayout::k + s * kTileBytes + hh * kHalfBytes), mk,
                                     hh * 64, g, row, bar(A_KF + s));
                loads_k = i + 1;
                if (i >= 2 && !wait(bar(A_VE + s), ph, 2)) break;
                ptx::mbar_expect_tx(bar(A_VF + s), kTileBytes);
                for (int hh = 0; hh < 2; ++hh)
                    ptx::tma_load_3d(ptx::smem_u32(smem + AttnLayout::v + s * kTileBytes + hh * kHalfBytes), mv,
                                     hh * 64, g, row, bar(A_VF + s));
                loads_v = i + 1;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        const uint32_t id_s = ptx::idesc_bf16_kk(kMRows, kKB), id_o = ptx::idesc_bf16_bmn(kMRows, kD);
        const uint32_t q0 = ptx::smem_u32(smem + AttnLayout::q), p0 = ptx::smem_u32(smem + AttnLayout::pp);
        bool ok = wait(bar(A_QF), 0, 10);
        // O += P V for local key block i (P written by the softmax warps; V rows
        // past the block's valid keys zeroed first by this warp).
        auto pv = [&](int i) -> bool {
            const int s = i & 1, j = j0 + i;
            if (!wait(bar(A_PF), i & 1, 11) || !wait(bar(A_VF + s), (i >> 1) & 1, 12)) return false;
            const int valid = j == nctx ? T : min(kKB, L - j * kKB);
            if (valid < kKB) {
                uint8_t *vt = smem + AttnLayout::v + s * kTileBytes;
                for (int e = lane; e < (kKB - valid) * 16; e += 32) {      // 16-byte chunks of both halves
                    const int r = valid + e / 16, c = e % 16;
                    *reinterpret_cast<uint4 *>(vt + (c >> 3) * kHalfBytes + r * 128 + (c & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                ptx::fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                ptx::tc_fence_after();
                const uint32_t v0 = ptx::smem_u32(smem + AttnLayout::v + s * kTileBytes);
#pragma unroll
                for (int kk = 0; kk < kKB / 16; ++kk)
                    ptx::mma_f16(t_o, ptx::desc_kmajor_sw128(p0 + (kk >> 2) * kHalfBytes + (kk & 3) * 32),
                                 ptx::desc_mnmajor_sw128(v0 + kk * 2048, kHalfBytes, 1024), id_o, (i | kk) != 0);
                ptx::mma_commit(bar(A_OF));                   // O ready, P buffer free
                ptx::mma_commit(bar(A_VE + s));               // value stage free
            }
            __syncwarp();
            return true;
        };
        for (int i = 0; i < nloc && ok; ++i) {
            const int s = i & 1;
            if (lane == 0) {
                ok = wait(bar(A_KF + s), (i >> 1) & 1, 13);
                if (ok && i >= 2) ok = wait(bar(A_SE + s), ((i >> 1) - 1) & 1, 14);
                if (ok) {
                    ptx::tc_fence_after();
                    const uint32_t k0 = ptx::smem_u32(smem + AttnLayout::k + s * kTileBytes);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        ptx::mma_f16(t_s + s * kKB, ptx::desc_kmajor_sw128(q0 + (kk >> 2) * kHalfBytes + (kk & 3) * 32),
                                     ptx::desc_kmajor_sw128(k0 + (kk >> 2) * kHalfBytes + (kk & 3) * 32), id_s,
                                     kk != 0);
                    ptx::mma_commit(bar(A_SF + s));
                    ptx::mma_commit(bar(A_KE + s));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (ok && i >= 1) ok = pv(i - 1);
        }
        if (ok) pv(nloc - 1);
    } else {
        // ------------------------------------------------------------ softmax
        const int quad = warp & 3;
        const int r = quad * 32 + lane;                       // query row = tensor-memory lane
        const int node = node0 + r / G, hq = g * G + r % G;
        const bool real = node < T;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const uint4 aw = *reinterpret_cast<const uint4 *>(ancs + 4 * (real ? node : 0));
        const uint32_t awv[4] = {real ? aw.x : 0u, real ? aw.y : 0u, real ? aw.z : 0u, real ? aw.w : 0u};
        uint8_t *prow = smem + AttnLayout::pp + r * 128;
        float m_ref = -INFINITY, l = 0.f;
        bool run = true;
        for (int i = 0; i < nloc && run; ++i) {
            const int s = i & 1, j = j0 + i;
            if (lane == 0) run = wait(bar(A_SF + s), (i >> 1) & 1, 20);
            run = __shfl_sync(0xffffffffu, run ? 1 : 0, 0) != 0;
            if (!run) break;
            ptx::tc_fence_after();
            uint32_t sv[kKB];
            ptx::tmem_ld128(t_s + s * kKB + lane_base, sv);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(A_SE + s));        // S buffer read
            // The mask: masked scores become -inf (full context blocks need none).
            const int kbase = j * kKB;
            if (j == nctx) {
#pragma unroll
                for (int key = 0; key < kKB; ++key)
                    if (!((awv[key >> 5] >> (key & 31)) & 1u)) sv[key] = 0xff800000u;
            } else if (kbase + kKB > L) {
                const int lim = L - kbase;
#pragma unroll
                for (int key = 0; key < kKB; ++key)
                    if (key >= lim) sv[key] = 0xff800000u;
            }
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int key = 0; key < kKB; ++key) mx4[key & 3] = fmaxf(mx4[key & 3], __uint_as_float(sv[key]));
            const float m_blk = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * p.scale_log2;
            bool need = false;
            float alpha = 1.f;
            if (i == 0) {
                m_ref = m_blk;
            } else if (m_blk > m_ref + kLazyLog2) {
                need = true;
                alpha = ptx::ex2_approx(m_ref - m_blk);
                m_ref = m_blk;
            }
            const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
            // The previous block's P V must be complete: it reads the P buffer, and
            // a rescale of the running output must not race its accumulation.
            if (i >= 1) {
                if (lane == 0) run = wait(bar(A_OF), (i - 1) & 1, 21);
                run = __shfl_sync(0xffffffffu, run ? 1 : 0, 0) != 0;
                if (!run) break;
                ptx::tc_fence_after();
            }
            // P = 2^(S scale log2(e) - m) in bf16 into the K-major swizzled P tile.
            float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < kKB / 32; ++c) {
                uint32_t packed[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float p0 = ptx::ex2_approx(fmaf(__uint_as_float(sv[c * 32 + e]), p.scale_log2, -m_use));
                    const float p1 = ptx::ex2_approx(fmaf(__uint_as_float(sv[c * 32 + e + 1]), p.scale_log2, -m_use));
                    rs4[(e >> 1) & 3] += p0 + p1;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    packed[e >> 1] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                // Keys c*32 .. c*32+31: half c/2 of the tile, 16-byte chunks 4(c&1) .. 4(c&1)+3.
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int chunk = 4 * (c & 1) + q;
                    *reinterpret_cast<uint4 *>(prow + (c >> 1) * kHalfBytes + ((chunk ^ (r & 7)) << 4)) =
                        make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                }
            }
            // tcgen05.ld / st are warp-collective: the rescale runs for the whole
            // warp when any row needs it (alpha is 1 for the others).
            if (__any_sync(0xffffffffu, need)) {
                uint32_t ov[32];
#pragma unroll
                for (int c = 0; c < kD / 32; ++c) {
                    ptx::tmem_ld32(t_o + lane_base + c * 32, ov);
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                    ptx::tmem_st32(t_o + lane_base + c * 32, ov);
                }
                ptx::tmem_wait_st();
            }
            l = l * alpha + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(A_PF));            // P written, O rescaled
        }
        // Epilogue: O / l in bf16 (one split), else the partial (O, m, l) in fp32;
        // rows of real nodes only.
        if (run) {
            if (lane == 0) run = wait(bar(A_OF), (nloc - 1) & 1, 22);
            run = __shfl_sync(0xffffffffu, run ? 1 : 0, 0) != 0;
        }
        if (run) {
            ptx::tc_fence_after();
            uint32_t ov[kD];
            ptx::tmem_ld128(t_o + lane_base, ov);
            if (real && p.nsplit == 1) {
                const float inv = l > 0.f ? 1.f / l : 0.f;
                __nv_bfloat16 *orow = p.o + (((size_t)b * T + node) * p.Hq + hq) * kD;
#pragma unroll
                for (int q = 0; q < kD / 8; ++q) {
                    uint32_t w4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(ov[8 * q + 2 * u]) * inv,
                                                                        __uint_as_float(ov[8 * q + 2 * u + 1]) * inv);
                        w4[u] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    *reinterpret_cast<uint4 *>(orow + 8 * q) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            } else if (real) {
                const size_t prow_i = (size_t)blockIdx.x * kMRows + r;
                float4 *dst = reinterpret_cast<float4 *>(p.part_o + prow_i * kD);
#pragma unroll
                for (int q = 0; q < kD / 4; ++q)
                    dst[q] = make_float4(__uint_as_float(ov[4 * q]), __uint_as_float(ov[4 * q + 1]),
                                         __uint_as_float(ov[4 * q + 2]), __uint_as_float(ov[4 * q + 3]));
                p.part_ml[prow_i] = make_float2(m_ref, l);
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    if (warp == 1 && lane == 0 && misc[AM_ABORT]) {
        ptx::mma_commit(bar(A_DRAIN));                        // every issued MMA completes first
        ptx::mbar_wait(bar(A_DRAIN), 0);
    }
    if (warp == 0 && lane == 0 && misc[AM_ABORT]) {
        // Loads that may still land: one more bounded wait on the last two issued
        // blocks of each ring (earlier ones completed before their stage was reused).
        for (int j = max(0, loads_k - 2); j < loads_k; ++j) ptx::mbar_wait(bar(A_KF + (j & 1)), (j >> 1) & 1);
        for (int j = max(0, loads_v - 2); j < loads_v; ++j) ptx::mbar_wait(bar(A_VF + (j & 1)), (j >> 1) & 1);
        ptx::mbar_wait(bar(A_QF), 0);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

// The merge of the splits: for each real row, M = max_s m_s and
//   o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// (empty splits carry m = -inf and are skipped).  CTA per (query tile, 32 rows);
// one warp per row at a time, four columns per lane.  A sequence whose tree is
// invalid was skipped by the first launch and is skipped here (o untouched).
__global__ void __launch_bounds__(kCombineThreads)
tree_attention_combine_kernel(const AttnParams p)
{
    __shared__ int32_t par[kMaxAttnNodes];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = blockIdx.x % (kMRows / kCombineRows);
    const int item = blockIdx.x / (kMRows / kCombineRows);
    const int mt = item % p.mtiles;
    const int g = (item / p.mtiles) % p.Hkv;
    const int b = item / (p.mtiles * p.Hkv);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i = tid; i < p.T; i += kCombineThreads) par[i] = __ldg(p.parent + (size_t)b * p.T + i);
    __syncthreads();
    if (!tree_row_ok(par, p.T, tid, kCombineThreads)) return;
    const size_t base = (size_t)item * p.nsplit;
    for (int rr = warp; rr < kCombineRows; rr += kCombineThreads / 32) {
        const int r = quarter * kCombineRows + rr;
        const int node = mt * p.TQ + r / p.G, hq = g * p.G + r % p.G;
        if (node >= p.T) continue;
        float M = -INFINITY;
        for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, p.part_ml[(base + s) * kMRows + r].x);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float den = 0.f;
        for (int s = 0; s < p.nsplit; ++s) {
            const float2 ml = p.part_ml[(base + s) * kMRows + r];
            if (ml.x == -INFINITY) continue;
            const float w = ptx::ex2_approx(ml.x - M);
            const float4 v = reinterpret_cast<const float4 *>(p.part_o + ((base + s) * kMRows + r) * kD)[lane];
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
            den = fmaf(w, ml.y, den);
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
        __nv_bfloat16 *orow = p.o + (((size_t)b * p.T + node) * p.Hq + hq) * kD;
        reinterpret_cast<uint2 *>(orow)[lane] =
            make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
    }
}

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

// A [rows, heads, 128] bf16 tensor as a 3-D map with boxes of 64 columns x `bh`
// heads x `br` rows (128-byte swizzle: each box row is one swizzled 128-byte row).
bool encode3(EncodeTiledFn enc, CUtensorMap *m, const void *base, long long rows, int heads, int bh, int br)
{
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)heads * kD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)bh, (cuuint32_t)br};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::mutex g_attn_mutex;
bool g_attn_prepared[kMaxDevices] = {};
int g_attn_sms[kMaxDevices] = {};

// Per-device setup (once): the kernel's shared-memory opt-in and the SM count.
cudaError_t prepare_attn(int *sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_attn_mutex);
    if (!g_attn_prepared[dev]) {
        if ((e = cudaFuncSetAttribute(tree_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)AttnLayout::total)) != cudaSuccess)
            return e;
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        g_attn_sms[dev] = n > 0 ? n : 1;
        g_attn_prepared[dev] = true;
    }
    *sms = g_attn_sms[dev];
    return cudaSuccess;
}

// How the key blocks are spread over CTAs.  One CTA per SM (its shared memory);
// a CTA spends about one key-block time on its set-up and, when split, one more
// on its partial and the merge.  The plan takes the split count with the least
// estimated time, waves x (blocks per CTA + overhead), preferring fewer splits.
struct AttnPlan {
    int G, TQ, mtiles, items, nsplit, bps;
    size_t ws_bytes;
};

AttnPlan attn_plan(int n_nodes, int batch, int ctx_cap, int heads_q, int heads_kv, int sms)
{
    AttnPlan pl{};
    pl.G = heads_q / heads_kv;
    pl.TQ = kMRows / pl.G;
    pl.mtiles = (n_nodes + pl.TQ - 1) / pl.TQ;
    pl.items = batch * heads_kv * pl.mtiles;
    const int nb = (ctx_cap + kKB - 1) / kKB + 1;
    auto waves = [&](long long ctas) { return (ctas + sms - 1) / sms; };
    long long best = waves(pl.items) * (nb + 1);
    pl.nsplit = 1;
    pl.bps = nb;
    for (int ns = 2; ns <= nb; ++ns) {
        const int bps = (nb + ns - 1) / ns;
        if ((nb + bps - 1) / bps != ns) continue;             // same blocks per split as a smaller count
        const long long cost = waves((long long)pl.items * ns) * (bps + 2);
        if (cost < best) {
            best = cost;
            pl.nsplit = ns;
            pl.bps = bps;
        }
    }
    pl.ws_bytes = pl.nsplit > 1 ? (size_t)pl.items * pl.nsplit * kMRows * (kD * sizeof(float) + sizeof(float2)) : 0;
    return pl;
}

bool attn_shape_ok(int n_nodes, int batch, int ctx_cap, int heads_q, int heads_kv, int head_dim)
{
    if (batch < 0 || n_nodes < 1 || n_nodes > kMaxAttnNodes || ctx_cap < 0 || heads_q < 1 || heads_kv < 1)
        return false;
    if (head_dim != kD || heads_q % heads_kv != 0) return false;
    const int G = heads_q / heads_kv;
    return G <= kMRows && kMRows % G == 0;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace stree

using namespace stree;

extern "C" stree_status stree_tree_attention_workspace_size(int n_nodes, int batch, int ctx_cap, int heads_q,
                                                            int heads_kv, int head_dim, size_t *bytes)
{
    if (!bytes) return STREE_ERR_INVALID_ARG;
    if (!attn_shape_ok(n_nodes, batch, ctx_cap, heads_q, heads_kv, head_dim)) return STREE_ERR_UNSUPPORTED;
    int sms = 0;
    if (prepare_attn(&sms) != cudaSuccess) return STREE_ERR_CUDA;
    *bytes = batch == 0 ? 0 : attn_plan(n_nodes, batch, ctx_cap, heads_q, heads_kv, sms).ws_bytes;
    return STREE_OK;
}

extern "C" stree_status stree_tree_attention(const void *q, const void *k_ctx, const void *v_ctx, const void *k_tree,
                                             const void *v_tree, const int32_t *ctx_len, const int32_t *parent,
                                             int n_nodes, int batch, int ctx_cap, int heads_q, int heads_kv,
                                             int head_dim, float scale, stree_dtype dtype, void *o, void *workspace,
                                             size_t workspace_bytes, int32_t *err_out, void *stream)
{
    if (!attn_shape_ok(n_nodes, batch, ctx_cap, heads_q, heads_kv, head_dim) || dtype != STREE_BF16)
        return STREE_ERR_UNSUPPORTED;
    if (!(scale > 0.f)) return STREE_ERR_INVALID_ARG;
    if (batch == 0) return STREE_OK;
    if (!q || !k_tree || !v_tree || !ctx_len || !parent || !o || !err_out) return STREE_ERR_INVALID_ARG;
    if (ctx_cap > 0 && (!k_ctx || !v_ctx)) return STREE_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k_tree, v_tree, o};
    for (const void *ptr : ptrs)
        if (!aligned(ptr, 16)) return STREE_ERR_MISALIGNED;
    if (ctx_cap > 0 && (!aligned(k_ctx, 16) || !aligned(v_ctx, 16))) return STREE_ERR_MISALIGNED;
    if (!aligned(ctx_len, 4) || !aligned(parent, 4) || !aligned(err_out, 4)) return STREE_ERR_MISALIGNED;
    if (workspace && !aligned(workspace, 16)) return STREE_ERR_MISALIGNED;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return STREE_ERR_CUDA;
    int sms = 0;
    if (prepare_attn(&sms) != cudaSuccess) return STREE_ERR_CUDA;
    AttnPlan pl = attn_plan(n_nodes, batch, ctx_cap, heads_q, heads_kv, sms);
    if (pl.nsplit > 1 && (!workspace || workspace_bytes < pl.ws_bytes)) {
        pl.nsplit = 1;                                        // no room for partials: one CTA per tile
        pl.bps = (ctx_cap + kKB - 1) / kKB + 1;
    }
    const long long grid = (long long)pl.items * pl.nsplit;
    if (grid > 0x7fffffffLL) return STREE_ERR_UNSUPPORTED;
    CUtensorMap m_q, m_kc, m_vc, m_kt, m_vt;
    // Context maps need a non-empty tensor; with no context they alias the tree's
    // and are never used (every sequence has no context block).
    const void *kc = ctx_cap > 0 ? k_ctx : k_tree, *vc = ctx_cap > 0 ? v_ctx : v_tree;
    const long long crows = ctx_cap > 0 ? (long long)batch * ctx_cap : (long long)batch * n_nodes;
    if (!encode3(enc, &m_q, q, (long long)batch * n_nodes, heads_q, pl.G, pl.TQ) ||
        !encode3(enc, &m_kc, kc, crows, heads_kv, 1, kKB) || !encode3(enc, &m_vc, vc, crows, heads_kv, 1, kKB) ||
        !encode3(enc, &m_kt, k_tree, (long long)batch * n_nodes, heads_kv, 1, kKB) ||
        !encode3(enc, &m_vt, v_tree, (long long)batch * n_nodes, heads_kv, 1, kKB))
        return STREE_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(err_out, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return STREE_ERR_CUDA;
    AttnParams p{};
    p.ctx_len = ctx_len;
    p.parent = parent;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.err = err_out;
    if (pl.nsplit > 1) {
        p.part_o = static_cast<float *>(workspace);
        p.part_ml = reinterpret_cast<float2 *>(static_cast<uint8_t *>(workspace) +
                                               (size_t)grid * kMRows * kD * sizeof(float));
    }
    p.T = n_nodes;
    p.S = ctx_cap;
    p.Hq = heads_q;
    p.Hkv = heads_kv;
    p.G = pl.G;
    p.TQ = pl.TQ;
    p.mtiles = pl.mtiles;
    p.nsplit = pl.nsplit;
    p.bps = pl.bps;
    p.scale_log2 = scale * 1.4426950408889634f;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = AttnLayout::total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, tree_attention_kernel, m_q, m_kc, m_vc, m_kt, m_vt, p) != cudaSuccess)
        return STREE_ERR_CUDA;
    if (pl.nsplit == 1) return STREE_OK;
    cfg.gridDim = dim3((unsigned)(pl.items * (kMRows / kCombineRows)));
    cfg.blockDim = dim3(kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, tree_attention_combine_kernel, p) == cudaSuccess ? STREE_OK : STREE_ERR_CUDA;
}
