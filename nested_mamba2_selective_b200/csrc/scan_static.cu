// ssd_scan_static: the selective scan with its scratch space in a fixed
// device array owned by this library instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory for a call: an engine whose
// allocator reserves all device memory up front and hands out nothing else, a
// plugin that is given only its input and output buffers, or a latency-
// critical loop that must not risk the device-wide synchronisation that
// cudaMalloc / cudaFree can cause.  This entry point needs no workspace: the
// scan's segment states live in g_scan_scratch below, which every GPU that
// loads the library holds until the process exits.
//
// Rules of use:
//  - The array holds kScanScratchBytes (MM_SCAN_STATIC_SCRATCH_BYTES); a call
//    whose scan needs more is rejected with MM_ERR_WORKSPACE before anything
//    is launched: ssd_scan compares the need of these very arguments with the
//    array's size.
//  - All calls on a device share the one array and it keeps whatever the last
//    call left in it.  The scan writes every scratch byte before reading it,
//    so nothing has to start at zero, but calls that overlap on the GPU (two
//    streams, or two host threads) race on the array and give wrong results:
//    serialise them.
//  - The first call on a device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current) and caches it; make
//    that first call before any stream capture.
#include <atomic>

#include "mm_internal.cuh"

namespace {

constexpr size_t kScanScratchBytes = MM_SCAN_STATIC_SCRATCH_BYTES;

// In host code this name is only a stand-in for the device array; kernels are
// given the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_scan_scratch[kScanScratchBytes];

// Device address of g_scan_scratch on the current device (looked up once per
// device); nullptr if the runtime cannot resolve it.
void* scratch_address()
{
    static std::atomic<void*> addr[64] = {};  // host threads may look it up at the same time
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    void* a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        if (cudaGetSymbolAddress(&a, g_scan_scratch) != cudaSuccess) return nullptr;
        addr[dev].store(a, std::memory_order_release);
    }
    return a;
}

}  // namespace

extern "C" int ssd_scan_static(int dtype, const void* x, int64_t x_stride, const float* dt, int64_t dt_stride,
                               const float* A, const void* B, int64_t B_stride, const void* C, int64_t C_stride,
                               const float* D, int batch, int L, int h, int P, int N, int G, int heads_per_group,
                               int chunk, const float* init_state, int64_t state_stride, void* y, int64_t y_stride,
                               float* final_state, void* stream)
{
    // ssd_scan validates the arguments and rejects, before any launch, a scan whose scratch need
    // (worked out from these very arguments) exceeds the array
    void* scratch = scratch_address();
    if (!scratch) return MM_ERR_CUDA;
    return ssd_scan(dtype, x, x_stride, dt, dt_stride, A, B, B_stride, C, C_stride, D, batch, L, h, P, N, G,
                    heads_per_group, chunk, init_state, state_stride, y, y_stride, final_state, scratch,
                    kScanScratchBytes, stream);
}
