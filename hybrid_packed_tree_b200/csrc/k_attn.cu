// k_attn.cu -- tree-masked attention over the packed draft tree, tcgen05, sm_100a.
//
// The Transformer layers of a hybrid model verify the same packed tree as its SSM
// layers ("STree: Speculative Tree Decoding for Hybrid State Space Models":
// abstract, hybrid SSM and Transformer layers; scime.ai summary, "Approach": the
// packed tree sequence with a tree mask): node i attends to the whole valid
// cached context and to the tree nodes on its own root path,
//   o_i = sum_j softmax_j(scale q_i . k_j) v_j,   j in context[0, ctx_len) and anc(i).
//
// Design (B200).  One CTA per (sequence, key/value head, tile of 128 query rows):
// the rows are (node, query head of the group) pairs, so the group's heads share
// every key and value tile.  The keys are streamed in blocks of 128 -- the
// context blocks, then one block holding the tree's own keys -- with an online
// softmax, in warp roles joined by bounded mbarrier waits:
//   * producer (one thread): TMA loads of the query tile (once) and of the key
//     and value blocks into two-stage rings;
//   * MMA (one thread): S = Q K^T into a double-buffered tensor-memory tile
//     (kind::f16, M = N = K-block = 128), then O += P V with V as an MN-major
//     operand (its rows are the keys), one key block behind, so that S of the
//     next block is computed while the softmax works on this one;
//   * softmax (four warps, one query row per thread, each warp on its own
//     tensor-memory lane quarter): the masked row maximum, the rescale of the
//     running output in tensor memory when the maximum grows, P = exp(S - m) in
//     bf16 into shared memory for the next MMA, the running row sum; at the end
//     O / l in bf16 to HBM.
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

enum AttnBars { A_QF = 0, A_KF = 1, A_KE = 3, A_VF = 5, A_VE = 7, A_SF = 9, A_SE = 11, A_PF = 13, A_OF = 14,
                A_DRAIN = 15, kAttnBars = 16 };
enum AttnMisc { AM_TMEM = 0, AM_ABORT, kAttnMisc };

struct AttnParams {
    const int32_t *ctx_len, *parent;
    __nv_bfloat16 *o;
    int32_t *err;
    int T, S, Hq, Hkv, G, TQ, mtiles;
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
    const int mt = blockIdx.x % p.mtiles;
    const int g = (blockIdx.x / p.mtiles) % p.Hkv;
    const int b = blockIdx.x / (p.mtiles * p.Hkv);
    const int node0 = mt * TQ;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int L = min(max(__ldg(p.ctx_len + b), 0), p.S);
    const int nctx = (L + kKB - 1) / kKB;
    const int nb = nctx + 1;                                  // context blocks, then the tree block

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
    int bad = 0;
    for (int i = tid; i < T; i += kAttnThreads) {
        const int v = par[i];
        bad |= (i == 0) ? (v != -1) : (v < 0 || v >= i);
    }
    const bool okb = !__syncthreads_or(bad);
    for (int i = tid; i < kMaxAttnNodes; i += kAttnThreads) {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if (okb && i < T)
            for (int j = i; j >= 0; j = par[j]) w[j >> 5] |= 1u << (j & 31);
        *reinterpret_cast<uint4 *>(ancs + 4 * i) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (!okb) {
        if (tid == 0 && g == 0 && mt == 0) latch_error(p.err, STREE_ERR_BAD_TREE, b, -1, 0);
        return;                                               // no copy issued yet; o untouched
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
            for (int j = 0; j < nb; ++j) {
                const int s = j & 1;
                const uint32_t ph = ((j >> 1) - 1) & 1;
                if (j >= 2 && !wait(bar(A_KE + s), ph, 1)) break;
                const bool tree = j == nctx;
                const CUtensorMap *mk = tree ? &tm_kt : &tm_kc;
                const CUtensorMap *mv = tree ? &tm_vt : &tm_vc;
                const int row = tree ? b * T : b * p.S + j * kKB;
                ptx::mbar_expect_tx(bar(A_KF + s), kTileBytes);
                for (int hh = 0; hh < 2; ++hh)
                    ptx::tma_load_3d(ptx::smem_u32(smem + AttnLayout::k + s * kTileBytes + hh * kHalfBytes), mk,
                                     hh * 64, g, row, bar(A_KF + s));
                loads_k = j + 1;
                if (j >= 2 && !wait(bar(A_VE + s), ph, 2)) break;
                ptx::mbar_expect_tx(bar(A_VF + s), kTileBytes);
                for (int hh = 0; hh < 2; ++hh)
                    ptx::tma_load_3d(ptx::smem_u32(smem + AttnLayout::v + s * kTileBytes + hh * kHalfBytes), mv,
                                     hh * 64, g, row, bar(A_VF + s));
                loads_v = j + 1;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        const uint32_t id_s = ptx::idesc_bf16_kk(kMRows, kKB), id_o = ptx::idesc_bf16_bmn(kMRows, kD);
        const uint32_t q0 = ptx::smem_u32(smem + AttnLayout::q), p0 = ptx::smem_u32(smem + AttnLayout::pp);
        bool ok = wait(bar(A_QF), 0, 10);
        // O += P V for key block j (P written by the softmax warps; V rows past the
        // block's valid keys zeroed first by this warp).
        auto pv = [&](int j) -> bool {
            const int s = j & 1;
            if (!wait(bar(A_PF), j & 1, 11) || !wait(bar(A_VF + s), (j >> 1) & 1, 12)) return false;
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
                                 ptx::desc_mnmajor_sw128(v0 + kk * 2048, kHalfBytes, 1024), id_o, (j | kk) != 0);
                ptx::mma_commit(bar(A_OF));                   // O ready, P buffer free
                ptx::mma_commit(bar(A_VE + s));               // value stage free
            }
            __syncwarp();
            return true;
        };
        for (int j = 0; j < nb && ok; ++j) {
            const int s = j & 1;
            if (lane == 0) {
                ok = wait(bar(A_KF + s), (j >> 1) & 1, 13);
                if (ok && j >= 2) ok = wait(bar(A_SE + s), ((j >> 1) - 1) & 1, 14);
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
            if (ok && j >= 1) ok = pv(j - 1);
        }
        if (ok) pv(nb - 1);
    } else {
        // ------------------------------------------------------------ softmax
        const int quad = warp & 3;
        const int r = quad * 32 + lane;                       // query row = tensor-memory lane
        const int node = node0 + r / G, hq = g * G + r % G;
        const bool real = node < T;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const uint32_t *myanc = ancs + 4 * (real ? node : 0);
        uint8_t *prow = smem + AttnLayout::pp + r * 128;
        float m = -INFINITY, l = 0.f;
        bool run = true;
        for (int j = 0; j < nb && run; ++j) {
            const int s = j & 1;
            if (lane == 0) run = wait(bar(A_SF + s), (j >> 1) & 1, 20);
            run = __shfl_sync(0xffffffffu, run ? 1 : 0, 0) != 0;
            if (!run) break;
            ptx::tc_fence_after();
            const bool tree = j == nctx;
            const int kbase = j * kKB;
            // Pass 1: the masked maximum of the row (scaled to log2 units).
            float mx = -INFINITY;
            uint32_t sv[32];
#pragma unroll
            for (int c = 0; c < kKB / 32; ++c) {
                ptx::tmem_ld32(t_s + s * kKB + lane_base + c * 32, sv);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int key = c * 32 + e;
                    const bool vis = tree ? (real && ((myanc[key >> 5] >> (key & 31)) & 1u)) : (kbase + key < L);
                    if (vis) mx = fmaxf(mx, __uint_as_float(sv[e]) * p.scale_log2);
                }
            }
            const float m_new = fmaxf(m, mx);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = exp2f(m - m_use);             // 0 on the first block (m = -inf)
            // The previous block's P V must be complete: it reads the P buffer, and
            // the running output is rescaled before this block's P V adds to it.
            if (j >= 1) {
                if (lane == 0) run = wait(bar(A_OF), (j - 1) & 1, 21);
                run = __shfl_sync(0xffffffffu, run ? 1 : 0, 0) != 0;
                if (!run) break;
                ptx::tc_fence_after();
                // tcgen05.ld / st are warp-collective: the rescale runs for the whole
                // warp when any row needs it (alpha is 1 for the others).
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
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
            }
            // Pass 2: P = exp2(S scale - m) in bf16 into the K-major swizzled P tile.
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < kKB / 32; ++c) {
                ptx::tmem_ld32(t_s + s * kKB + lane_base + c * 32, sv);
                uint32_t packed[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float pe[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int key = c * 32 + e + u;
                        const bool vis =
                            tree ? (real && ((myanc[key >> 5] >> (key & 31)) & 1u)) : (kbase + key < L);
                        pe[u] = vis ? exp2f(__uint_as_float(sv[e + u]) * p.scale_log2 - m_use) : 0.f;
                        rs += pe[u];
                    }
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(pe[0], pe[1]);
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
            l = l * alpha + rs;
            m = m_new;
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(A_SE + s));                   // S buffer read
                mbar_arrive(bar(A_PF));                       // P written, O rescaled
            }
        }
        // Epilogue: O / l in bf16, rows of real nodes only.
        if (run) {
            if (lane == 0) run = wait(bar(A_OF), (nb - 1) & 1, 22);
            run = __shfl_sync(0xffffffffu, run ? 1 : 0, 0) != 0;
        }
        if (run) {
            ptx::tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = p.o + (((size_t)b * T + (real ? node : 0)) * p.Hq + hq) * kD;
            uint32_t ov[32];
#pragma unroll
            for (int c = 0; c < kD / 32; ++c) {
                ptx::tmem_ld32(t_o + lane_base + c * 32, ov);
                if (real) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w4[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(ov[8 * q + 2 * u]) * inv,
                                                                            __uint_as_float(ov[8 * q + 2 * u + 1]) * inv);
                            w4[u] = *reinterpret_cast<const uint32_t *>(&h2);
                        }
                        *reinterpret_cast<uint4 *>(orow + c * 32 + 8 * q) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
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

cudaError_t prepare_attn()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_attn_mutex);
    if (g_attn_prepared[dev]) return cudaSuccess;
    if ((e = cudaFuncSetAttribute(tree_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)AttnLayout::total)) != cudaSuccess)
        return e;
    g_attn_prepared[dev] = true;
    return cudaSuccess;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace stree

using namespace stree;

extern "C" stree_status stree_tree_attention(const void *q, const void *k_ctx, const void *v_ctx, const void *k_tree,
                                             const void *v_tree, const int32_t *ctx_len, const int32_t *parent,
                                             int n_nodes, int batch, int ctx_cap, int heads_q, int heads_kv,
                                             int head_dim, float scale, stree_dtype dtype, void *o, int32_t *err_out,
                                             void *stream)
{
    if (batch < 0 || n_nodes < 1 || n_nodes > kMaxAttnNodes || ctx_cap < 0 || heads_q < 1 || heads_kv < 1)
        return STREE_ERR_UNSUPPORTED;
    if (head_dim != kD || dtype != STREE_BF16 || heads_q % heads_kv != 0) return STREE_ERR_UNSUPPORTED;
    const int G = heads_q / heads_kv;
    if (G > kMRows || kMRows % G != 0) return STREE_ERR_UNSUPPORTED;
    if (!(scale > 0.f)) return STREE_ERR_INVALID_ARG;
    if (batch == 0) return STREE_OK;
    if (!q || !k_tree || !v_tree || !ctx_len || !parent || !o || !err_out) return STREE_ERR_INVALID_ARG;
    if (ctx_cap > 0 && (!k_ctx || !v_ctx)) return STREE_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k_tree, v_tree, o};
    for (const void *ptr : ptrs)
        if (!aligned(ptr, 16)) return STREE_ERR_MISALIGNED;
    if (ctx_cap > 0 && (!aligned(k_ctx, 16) || !aligned(v_ctx, 16))) return STREE_ERR_MISALIGNED;
    if (!aligned(ctx_len, 4) || !aligned(parent, 4) || !aligned(err_out, 4)) return STREE_ERR_MISALIGNED;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return STREE_ERR_CUDA;
    const int TQ = kMRows / G;
    const int mtiles = (n_nodes + TQ - 1) / TQ;
    const long long grid = (long long)batch * heads_kv * mtiles;
    if (grid > 0x7fffffffLL) return STREE_ERR_UNSUPPORTED;
    CUtensorMap m_q, m_kc, m_vc, m_kt, m_vt;
    // Context maps need a non-empty tensor; with no context they alias the tree's
    // and are never used (every sequence has no context block).
    const void *kc = ctx_cap > 0 ? k_ctx : k_tree, *vc = ctx_cap > 0 ? v_ctx : v_tree;
    const long long crows = ctx_cap > 0 ? (long long)batch * ctx_cap : (long long)batch * n_nodes;
    if (!encode3(enc, &m_q, q, (long long)batch * n_nodes, heads_q, G, TQ) ||
        !encode3(enc, &m_kc, kc, crows, heads_kv, 1, kKB) || !encode3(enc, &m_vc, vc, crows, heads_kv, 1, kKB) ||
        !encode3(enc, &m_kt, k_tree, (long long)batch * n_nodes, heads_kv, 1, kKB) ||
        !encode3(enc, &m_vt, v_tree, (long long)batch * n_nodes, heads_kv, 1, kKB))
        return STREE_ERR_UNSUPPORTED;
    if (prepare_attn() != cudaSuccess) return STREE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(err_out, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return STREE_ERR_CUDA;
    AttnParams p{};
    p.ctx_len = ctx_len;
    p.parent = parent;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.err = err_out;
    p.T = n_nodes;
    p.S = ctx_cap;
    p.Hq = heads_q;
    p.Hkv = heads_kv;
    p.G = G;
    p.TQ = TQ;
    p.mtiles = mtiles;
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
    return cudaLaunchKernelEx(&cfg, tree_attention_kernel, m_q, m_kc, m_vc, m_kt, m_vt, p) == cudaSuccess
               ? STREE_OK
               : STREE_ERR_CUDA;
}
