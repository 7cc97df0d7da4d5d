// Placeholder until the tensor-core kernels land: reports "not supported" so
// the CUDA-core kernels run every shape.
#include "mm_internal.cuh"

namespace mm {
bool scan_tc_supported(const ScanArgs&) { return false; }
size_t scan_tc_workspace(const ScanArgs&) { return 0; }
int scan_tc_kernel_count(const ScanArgs&) { return 0; }
cudaError_t launch_scan_tc(const ScanArgs&, void*, size_t, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace mm
