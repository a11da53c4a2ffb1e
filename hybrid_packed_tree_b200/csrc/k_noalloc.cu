// k_noalloc.cu -- the fused scan + commit for callers that must not allocate.
//
// Some callers cannot call cudaMalloc at the point where they run the scan: a
// serving runtime that owns all device memory through its own pool and forbids
// stray allocations, code running under a memory cap that is already reached,
// or a hot loop whose allocator calls would synchronise the device.  This entry
// point runs the same kernels as stree_tree_scan_commit, but takes its scratch
// (tree masks, depths, per-sequence flags, the C.B pair scratch of the CUDA-core
// kernel and, when the caller gives none, the error word) from one file-scope
// device array instead of a context's workspace.
//
// That array is a static __device__ object: every GPU that loads the library
// holds its kNoAllocScratch bytes until the process exits (with lazy module
// loading the array is placed on a device when the library's module is first
// loaded there, at the latest by the first call of this entry point on it).
// Host code may not pass the array's name to a kernel -- on the host it is only
// a stand-in -- so the device address is looked up with cudaGetSymbolAddress,
// with the device current, on the first call made on it; a call that finds a new
// CUDA context on the device (after cudaDeviceReset) looks it up again.
#include <cuda.h>

#include <mutex>
#include <string.h>

#include "stree_internal.cuh"

namespace stree {
namespace {

constexpr size_t kNoAllocScratch = size_t(8) << 20;   // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratch];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct ScratchSlot {
    uint8_t *ptr = nullptr;
    unsigned long long ctx_id = 0;
};

std::mutex g_mutex;
ScratchSlot g_scratch[kMaxDevices];

// Identifier of the current CUDA context; 0 when the thread has none yet, 1
// when the driver cannot tell contexts apart (then the lookup is kept per device).
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    if (!get_current || !get_id) return 1;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch on the current device: looked up on the first
// call on the device (with the device current) and again when the device has a
// new context.
cudaError_t scratch_address(uint8_t **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(g_mutex);
    ScratchSlot &slot = g_scratch[dev];
    if (!slot.ptr || id == 0 || slot.ctx_id != id) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        slot.ptr = static_cast<uint8_t *>(p);
        slot.ctx_id = current_context_id();         // the lookup has made the context current
    }
    *out = slot.ptr;
    return cudaSuccess;
}

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace stree

using namespace stree;

extern "C" stree_status stree_tree_scan_commit_noalloc(
    const void *x, const void *dt, const float *A, const void *B, const void *C, const float *D, const float *h0,
    const int32_t *parent, int n_nodes, int batch, int nheads, int headdim, int dstate, int ngroups,
    stree_dtype dtype, const int32_t *accepted_path, const int32_t *path_len, int maxlen, void *y, float *h_new,
    int32_t *err_out, void *stream)
{
    ScanArgs a{};
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D; a.h0 = h0;
    a.T = n_nodes; a.batch = batch; a.H = nheads; a.P = headdim; a.N = dstate; a.G = ngroups;
    a.dtype = dtype;
    a.y = y;
    a.path = accepted_path;
    a.path_len = path_len;
    a.maxlen = maxlen;
    a.h_new = h_new;

    // The shape rules and batch-0 behaviour of stree_tree_scan_commit.
    if (batch < 0 || n_nodes < 1 || nheads < 1 || ngroups < 1 || headdim < 1 || dstate < 1) return STREE_ERR_UNSUPPORTED;
    if (batch == 0) return maxlen >= 0 ? STREE_OK : STREE_ERR_INVALID_ARG;
    if (n_nodes > kMaxNodes || headdim > kMaxDim || dstate > kMaxDim) return STREE_ERR_UNSUPPORTED;
    if (headdim % 8 != 0 || dstate % 8 != 0 || nheads % ngroups != 0 || nheads > 65535) return STREE_ERR_UNSUPPORTED;
    if (dtype != STREE_F32 && dtype != STREE_BF16) return STREE_ERR_UNSUPPORTED;
    if (!x || !dt || !A || !B || !C || !D || !h0 || !y || !parent || !accepted_path || !path_len || !h_new)
        return STREE_ERR_INVALID_ARG;
    if (maxlen < 1) return STREE_ERR_INVALID_ARG;
    const void *ptrs[] = {x, dt, A, B, C, D, h0, y, h_new};
    for (const void *p : ptrs)
        if (!aligned16(p)) return STREE_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(parent) & 3u) || (reinterpret_cast<uintptr_t>(accepted_path) & 3u) ||
        (reinterpret_cast<uintptr_t>(path_len) & 3u) || (reinterpret_cast<uintptr_t>(err_out) & 3u))
        return STREE_ERR_MISALIGNED;

    // Scratch layout: error word, masks, depths, flags, then the C.B pair
    // scratch of the CUDA-core kernel, or of the tensor-core kernel on trees with
    // more ancestor pairs than its shared memory holds.  Sizes beyond the array
    // are rejected (the tensor-core pair scratch is optional).
    const size_t T = (size_t)n_nodes, W = (T + 31) / 32, nb = (size_t)batch;
    const size_t off_err = 0;
    const size_t off_anc = 256;
    const size_t off_depth = off_anc + round256(nb * T * W * sizeof(uint32_t));
    const size_t off_ok = off_depth + round256(nb * T * sizeof(int32_t));
    const size_t off_cb = off_ok + round256(nb * sizeof(int32_t));
    if (off_cb > kNoAllocScratch) return STREE_ERR_UNSUPPORTED;
    // The kernel choice needs the device; look the scratch up first.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return STREE_ERR_CUDA;
    ScanPath path;
    if (!select_path(STREE_KERNEL_AUTO, a, &path)) return STREE_ERR_UNSUPPORTED;
    size_t need = off_cb;
    if (path == ScanPath::Simt) need += round256(nb * (size_t)ngroups * T * T * sizeof(float));
    if (need > kNoAllocScratch) return STREE_ERR_UNSUPPORTED;
    // The tensor-core kernel's pair scratch for deep trees, when it fits (without
    // it the kernel recomputes those products per tile: same result, slower).
    const size_t pair_bytes = path == ScanPath::Tc ? round256(tc_pair_scratch_floats(a) * sizeof(float)) : 0;
    const bool use_pairs = pair_bytes > 0 && off_cb + pair_bytes <= kNoAllocScratch;

    int32_t *err = err_out ? err_out : reinterpret_cast<int32_t *>(base + off_err);
    uint32_t *anc = reinterpret_cast<uint32_t *>(base + off_anc);
    int32_t *depth = reinterpret_cast<int32_t *>(base + off_depth);
    int32_t *ok = reinterpret_cast<int32_t *>(base + off_ok);
    // The error word must start at zero; masks, depths, flags and the pair
    // scratch are fully rewritten by the kernels below.
    if (cudaMemsetAsync(err, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return STREE_ERR_CUDA;
    a.tree.anc = anc;
    a.tree.depth = depth;
    a.tree.ok = ok;
    a.tree.T = n_nodes;
    a.tree.W = (int)W;
    a.tree.batch = batch;
    a.parent = parent;                       // the launch rebuilds the tree into the scratch
    a.tree_anc = anc;
    a.tree_depth = depth;
    a.tree_ok = ok;
    a.err = err;
    if (path == ScanPath::Simt) a.cb = reinterpret_cast<float *>(base + off_cb);
    if (use_pairs) a.pair_scratch = reinterpret_cast<float *>(base + off_cb);
    int64_t launches = 0;
    return launch_scan(path, a, s, &launches) == cudaSuccess ? STREE_OK : STREE_ERR_CUDA;
}
