// k_scan_tc.cu -- tensor-core (tcgen05) packed tree scan: not built yet.
#include "stree_internal.cuh"

namespace stree {

bool tc_supported(const ScanArgs &) { return false; }

cudaError_t launch_scan_tc(const ScanArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace stree
