// m2_scan_static.cu -- the fixed device scratch of m2_chunk_scan_varlen_static.
//
// A split variable-length scan (vllm.cpp issue #1311 "NemotronH runs the
// PREFILL mamba kernels at decode", section "The divergence": the chunk scan
// at prefill) keeps one fp32 P x N state per (sequence, segment, head) plus one
// decay each between its passes. This translation unit holds that scratch as
// a file-scope device array, so the entry point that uses it allocates
// nothing. The array's 16 MiB is reserved on every device where the library's
// module is loaded: under lazy module loading (the CUDA default) a device on
// which a libm2 call has run, with CUDA_MODULE_LOADING=EAGER every device the
// process initialises. The address looked up per device is cached for the
// life of the process; it does not survive a cudaDeviceReset.
#include <cuda_runtime.h>

#include <mutex>

#include "m2_internal.cuh"

namespace m2 {
namespace {

// A split plan keeps at most one (sequence, segment, head) state of 32 KB
// (P = 64, N = 128) and one decay per SM: 4.6 MiB on a 148-SM B200; 16 MiB
// covers GPUs of up to 511 SMs.
constexpr size_t kStaticScanScratchBytes = size_t{16} << 20;

__device__ __align__(256) unsigned char g_static_scan_scratch[kStaticScanScratchBytes];

}  // namespace

cudaError_t static_scan_scratch(void** ptr, size_t* bytes) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scan_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    *bytes = kStaticScanScratchBytes;
    return cudaSuccess;
}

}  // namespace m2
