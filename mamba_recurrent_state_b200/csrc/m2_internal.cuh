// m2_internal.cuh -- declarations shared by the libm2 translation units.
// Not installed; the public ABI is include/m2.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "m2.h"

namespace m2 {

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point (no
// -lcuda); nullptr when the driver does not provide it.
using TensorMapEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                       const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                       CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                       CUtensorMapFloatOOBfill);
TensorMapEncodeFn tensor_map_encoder();

// Runs a kernel's one-time function-attribute setup once per device (the
// attributes belong to the device's context). Concurrent first calls may both
// run the setup, which is harmless; a failure is returned and retried.
struct AttrOnce {
    static constexpr int kMaxDevices = 64;
    std::atomic<int> done[kMaxDevices] = {};
    template <typename F>
    cudaError_t ensure(F&& setup) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
        e = setup();
        if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(1, std::memory_order_release);
        return e;
    }
};

// Everything a decode-step launch needs (host-validated).
struct StateUpdateArgs {
    void* ssm;
    void* conv;
    int32_t* error;
    int64_t num_slots;
    int H, P, N, G, K;
    int64_t conv_dim;
    int state_bf16, act_bf16;
    int x_dtype;  // m2_dtype of xBC when it is post-conv (the unfused path)
    const float* A_log;
    const float* dt_bias;
    const float* D;
    const void* conv_w;
    const void* conv_b;
    int activation;
    int fused;
    int batch;
    const void* xBC;
    int64_t xBC_stride;
    const void* dt;
    int64_t dt_stride;
    const void* z;
    int64_t z_stride;
    void* y;
    int64_t y_stride;
    const int32_t* slot_idx;
    const void* norm_w;  // gated RMSNorm weight [H*P] act dtype, or NULL (fused launches only)
    float norm_eps;
};

struct ConvArgs {
    void* conv;
    int32_t* error;
    int64_t num_slots;
    int K;
    int64_t conv_dim;
    int act_bf16;
    int out_dtype;  // m2_dtype of the post-conv output
    const void* w;
    const void* b;
    int activation;
    int batch, seqlen;
    const void* x;
    int64_t x_stride;
    void* out;
    int64_t out_stride;
    const int32_t* slot_idx;
    // variable-length batches: sequence b is packed rows cu_seqlens[b] ..
    // cu_seqlens[b+1]-1 (NULL: rows b*seqlen ..); seqlen then bounds the grid
    const int32_t* cu_seqlens;
    int64_t total_rows;  // rows of x (batch * seqlen, or the packed total)
};

struct ZeroArgs {
    void* ssm;
    void* conv;
    int32_t* error;
    int64_t num_slots;
    int64_t ssm_bytes_per_slot;
    int64_t conv_bytes_per_slot;
    int n;
    const int32_t* slot_idx;
};

struct ScanArgs {
    void* ssm;
    int32_t* error;
    int64_t num_slots;
    int H, P, N, G;
    int state_bf16, act_bf16;
    int x_dtype;  // m2_dtype of the post-conv xBC
    const float* A_log;
    const float* dt_bias;
    const float* D;
    int batch, seqlen, chunk;
    const void* xBC;
    int64_t xBC_stride;
    const void* dt;
    int64_t dt_stride;
    const void* z;
    int64_t z_stride;
    void* y;
    int64_t y_stride;
    const int32_t* slot_idx;
    const uint8_t* has_init;
    // variable-length batches: sequence b is packed rows cu_seqlens[b] ..
    // cu_seqlens[b+1]-1 (NULL: rows b*seqlen .. of a [batch, seqlen] layout)
    const int32_t* cu_seqlens;
    int64_t total_tokens;  // rows of the packed xBC / dt / z / y
    // split sequences (tensor-core path): nseg segments of seg_chunks chunks
    // per sequence in the grid; nseg = 1 runs every sequence in one CTA per head
    int nseg, seg_chunks;
    float* seg_state;  // [batch][nseg][H][P][N] fp32 scratch (nseg > 1)
    float* seg_decay;  // [batch][nseg][H] fp32 scratch (nseg > 1)
};

// Multi-token decode (speculative drafts): T tokens per row from slot_idx[b],
// the state and conv window after token t stored into token_slots[b*T + t].
constexpr int kMaxDraftTokens = 16;
struct MtArgs {
    void* ssm;
    void* conv;
    int32_t* error;
    int64_t num_slots;
    int H, P, N, G, K, T;
    int64_t conv_dim;
    int state_bf16, act_bf16;
    const float* A_log;
    const float* dt_bias;
    const float* D;
    const void* conv_w;
    const void* conv_b;
    int activation;
    int batch;
    const void* xBC;  // [batch, T, conv_dim] raw, token rows xBC_stride apart
    int64_t xBC_stride;
    const void* dt;   // [batch, T, H]
    int64_t dt_stride;
    const void* z;    // [batch, T, H*P] or NULL
    int64_t z_stride;
    void* y;          // [batch, T, H*P]
    int64_t y_stride;
    const int32_t* slot_idx;     // [batch], read only
    const int32_t* token_slots;  // [batch, T], written
};
m2_status plan_multi_token(int H, int P, int N, int G, int K, int T);
cudaError_t launch_state_update_mt(const MtArgs& a, cudaStream_t stream);

// Launch-shape query for the decode kernels: M2_OK and the shape, or
// M2_ERR_UNSUPPORTED. Pure host arithmetic.
struct DecodePlan {
    int loads;        // 16-byte loads per thread
    int tile_rows;    // state rows (of N elements) per CTA
    int ctas_per_seq; // H*P / tile_rows
    int cluster;      // CTAs per group when the conv is fused (1 otherwise)
};
m2_status plan_state_update(int H, int P, int N, int G, int state_bf16, int fused,
                            DecodePlan* plan);

cudaError_t launch_state_update(const StateUpdateArgs& a, const DecodePlan& plan,
                                cudaStream_t stream);
cudaError_t launch_conv1d_update(const ConvArgs& a, cudaStream_t stream);
cudaError_t launch_zero_slots(const ZeroArgs& a, cudaStream_t stream);
m2_status plan_chunk_scan(int H, int P, int N, int G, int chunk);
// Address and size of the fixed scratch array of m2_chunk_scan_varlen_static
// on the current device (looked up once per device with cudaGetSymbolAddress).
cudaError_t static_scan_scratch(void** ptr, size_t* bytes);
cudaError_t launch_chunk_scan(const ScanArgs& a, cudaStream_t stream);
// Tensor-core (tcgen05) scan: bf16 state, activations and xBC, P = 64, N = 128.
bool chunk_scan_tc_supported(const ScanArgs& a);
cudaError_t launch_chunk_scan_tc(const ScanArgs& a, cudaStream_t stream);

// Records `code` in the error word unless an earlier error is already there.
__device__ __forceinline__ void record_error(int32_t* error, int32_t code) {
    if (error) atomicCAS(error, 0, code);
}

}  // namespace m2
