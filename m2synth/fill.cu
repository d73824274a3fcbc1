// fill.cu -- device twin of the seeded input generator in m2synth/__init__.py.
//
// Test and benchmark infrastructure: it fills device buffers with the same
// bits the host generator produces for the same (key, element index), so that
// multi-GiB synthetic caches need not cross PCIe. It holds none of the
// method's arithmetic. Definition (identical on both sides):
//   word(key, i) = SplitMix64 finaliser of key + (i + 1) * 0x9E3779B97F4A7C15
//   n_i = (sum of the 32-bit halves of words 6i .. 6i+5 - 6 * 2^32) / 2^32
//   v_i = mean + std * n_i   (float64, one rounding per operation, no FMA)
//   stored as float32 (round to nearest even), or bf16 from that float32
//   (round to nearest even on the bit pattern).
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void fill_normal_kernel(void* dst, int bf16, int64_t n, uint64_t key, int64_t start,
                                   double mean, double stdev) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        const uint64_t c = static_cast<uint64_t>(start + i) * 6ull;
        uint64_t sum = 0;
#pragma unroll
        for (int j = 0; j < 6; ++j) {
            const uint64_t w = mix64(key + (c + j + 1) * 0x9E3779B97F4A7C15ull);
            sum += (w >> 32) + (w & 0xFFFFFFFFull);
        }
        const double nv = (static_cast<double>(sum) - 6.0 * 4294967296.0) / 4294967296.0;
        const double v = __dadd_rn(mean, __dmul_rn(stdev, nv));
        const float f = __double2float_rn(v);
        if (bf16) {
            const uint32_t u = __float_as_uint(f);
            static_cast<uint16_t*>(dst)[i] = static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
        } else {
            static_cast<float*>(dst)[i] = f;
        }
    }
}

}  // namespace

extern "C" int m2s_fill_normal(void* dst, int bf16, int64_t n, uint64_t key, int64_t start,
                               double mean, double stdev, cudaStream_t stream) {
    if (n <= 0) return 0;
    int blocks = static_cast<int>((n + 255) / 256);
    if (blocks > 148 * 64) blocks = 148 * 64;
    fill_normal_kernel<<<blocks, 256, 0, stream>>>(dst, bf16, n, key, start, mean, stdev);
    return static_cast<int>(cudaGetLastError());
}
