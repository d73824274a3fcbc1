// m2_chunk_scan.cu -- prefill scan over seqlen tokens per row, landing on the
// same state as seqlen sequential selective_state_update steps.
//
// Operation: vllm.cpp issue #1311 "NemotronH runs the PREFILL mamba kernels at
// decode", section "The divergence" (the chunk scan that follows the prefill
// conv), and section "Confirm or refute" (the state-update arm and the chunk
// scan must agree, T = 1 included, for n_groups = 8). For every token t:
//   S <- S*exp(dt_t*A) + (dt_t*x_t) B_t^T,   y_t = S C_t + D x_t,  y_t *= silu(z_t)
// from the slot's state (or zero), with the final S stored back once.
//
// bf16 state and activations at P = 64, N = 128 go to the tensor-core kernel
// (m2_chunk_scan_tc.cu). This file holds the token-sequential kernel on the
// CUDA cores used for the other dtypes and shapes: one CTA per
// (sequence, head), the head's P x N state in registers (TPR threads per state
// row), inputs staged through shared memory a tile of tokens at a time. It
// allocates nothing and keeps the state on chip for the whole sequence.
#include <cuda_runtime.h>

#include "m2_device.cuh"
#include "m2_internal.cuh"

namespace m2 {
namespace {

constexpr int kScanThreads = 128;
constexpr int kTok = 16;  // tokens staged per tile

template <typename ST, typename AT, typename XT, int P, int N>
__global__ void __launch_bounds__(kScanThreads) scan_seq_kernel(const ScanArgs a) {
    constexpr int TPR = kScanThreads / P;  // threads per state row
    constexpr int CPT = N / TPR;           // state columns per thread
    static_assert(kScanThreads % P == 0 && N % TPR == 0 && CPT % 4 == 0, "layout");

    __shared__ __align__(16) float s_x[kTok][P];
    __shared__ __align__(16) float s_B[kTok][N];
    __shared__ __align__(16) float s_C[kTok][N];
    __shared__ __align__(16) float s_z[kTok][P];
    __shared__ __align__(16) float s_y[kTok][P];
    __shared__ float s_dt[kTok];
    __shared__ float s_dA[kTok];

    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    const int p = tid / TPR;
    const int n0 = (tid % TPR) * CPT;
    const int H = a.H;
    const int g = h / (H / a.G);
    const int64_t HP = static_cast<int64_t>(H) * P;
    // this sequence's rows of the packed token arrays
    const int64_t row0 = a.cu_seqlens ? static_cast<int64_t>(a.cu_seqlens[b]) : static_cast<int64_t>(b) * a.seqlen;
    const int T = a.cu_seqlens ? a.cu_seqlens[b + 1] - a.cu_seqlens[b] : a.seqlen;
    if (T <= 0) return;  // an empty sequence leaves its cache slot untouched
    const int32_t slot = a.slot_idx[b];
    AT* y = static_cast<AT*>(a.y);
    if (slot < 0) {
        for (int64_t i = tid; i < static_cast<int64_t>(T) * P; i += kScanThreads) {
            const int64_t t = i / P;
            y[(row0 + t) * a.y_stride + h * P + (i % P)] = from_f32<AT>(0.f);
        }
        return;
    }
    if (slot >= a.num_slots) {
        if (tid == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }

    ST* state = static_cast<ST*>(a.ssm) + (static_cast<int64_t>(slot) * HP + static_cast<int64_t>(h) * P + p) * N + n0;
    float S[CPT];
    const bool init = a.has_init != nullptr && a.has_init[b] != 0;
#pragma unroll
    for (int c = 0; c < CPT; ++c) S[c] = init ? to_f32(state[c]) : 0.f;

    const float A = -expf(a.A_log[h]);
    const float dtb = a.dt_bias[h];
    const float Dh = a.D[h];
    const XT* xbc = static_cast<const XT*>(a.xBC);
    const AT* dtp = static_cast<const AT*>(a.dt);
    const AT* zp = static_cast<const AT*>(a.z);
    const int64_t cB = HP + static_cast<int64_t>(g) * N;
    const int64_t cC = HP + static_cast<int64_t>(a.G) * N + static_cast<int64_t>(g) * N;

    for (int t0 = 0; t0 < T; t0 += kTok) {
        const int nt = min(kTok, T - t0);
        // stage the tile
        for (int i = tid; i < nt * P; i += kScanThreads) {
            const int j = i / P, q = i % P;
            const int64_t r = row0 + t0 + j;
            s_x[j][q] = to_f32(xbc[r * a.xBC_stride + h * P + q]);
            s_z[j][q] = zp ? to_f32(zp[r * a.z_stride + h * P + q]) : 0.f;
        }
        for (int i = tid; i < nt * N; i += kScanThreads) {
            const int j = i / N, n = i % N;
            const int64_t r = row0 + t0 + j;
            s_B[j][n] = to_f32(xbc[r * a.xBC_stride + cB + n]);
            s_C[j][n] = to_f32(xbc[r * a.xBC_stride + cC + n]);
        }
        if (tid < nt) {
            const float dt = softplus_f32(to_f32(dtp[(row0 + t0 + tid) * a.dt_stride + h]) + dtb);
            s_dt[tid] = dt;
            s_dA[tid] = expf(dt * A);
        }
        __syncthreads();
        for (int j = 0; j < nt; ++j) {
            const float xv = s_x[j][p];
            const float dtx = s_dt[j] * xv;
            const float dA = s_dA[j];
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; c += 4) {
                const float4 Bq = *reinterpret_cast<const float4*>(&s_B[j][n0 + c]);
                const float4 Cq = *reinterpret_cast<const float4*>(&s_C[j][n0 + c]);
                S[c + 0] = fmaf(S[c + 0], dA, dtx * Bq.x);
                S[c + 1] = fmaf(S[c + 1], dA, dtx * Bq.y);
                S[c + 2] = fmaf(S[c + 2], dA, dtx * Bq.z);
                S[c + 3] = fmaf(S[c + 3], dA, dtx * Bq.w);
                acc = fmaf(S[c + 0], Cq.x, acc);
                acc = fmaf(S[c + 1], Cq.y, acc);
                acc = fmaf(S[c + 2], Cq.z, acc);
                acc = fmaf(S[c + 3], Cq.w, acc);
            }
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if ((tid % TPR) == 0) {
                float yv = fmaf(Dh, xv, acc);
                if (zp) yv *= silu_f32(s_z[j][p]);
                s_y[j][p] = yv;
            }
        }
        __syncthreads();
        for (int i = tid; i < nt * P; i += kScanThreads) {
            const int j = i / P, q = i % P;
            y[(row0 + t0 + j) * a.y_stride + h * P + q] = from_f32<AT>(s_y[j][q]);
        }
        // the next tile's staging overwrites s_x/s_B/...; s_y is read above
        __syncthreads();
    }
#pragma unroll
    for (int c = 0; c < CPT; ++c) state[c] = from_f32<ST>(S[c]);
}

template <typename ST, typename AT, typename XT>
cudaError_t scan_by_shape(const ScanArgs& a, cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>(a.H), static_cast<unsigned>(a.batch));
    if (a.P == 64 && a.N == 128) scan_seq_kernel<ST, AT, XT, 64, 128><<<grid, kScanThreads, 0, s>>>(a);
    else if (a.P == 64 && a.N == 64) scan_seq_kernel<ST, AT, XT, 64, 64><<<grid, kScanThreads, 0, s>>>(a);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

template <typename ST, typename AT>
cudaError_t scan_by_x(const ScanArgs& a, cudaStream_t s) {
    if (a.x_dtype == M2_BF16) return scan_by_shape<ST, AT, bf16_t>(a, s);
    if (a.x_dtype == M2_F16) return scan_by_shape<ST, AT, f16_t>(a, s);
    return scan_by_shape<ST, AT, float>(a, s);
}

}  // namespace

m2_status plan_chunk_scan(int H, int P, int N, int G, int chunk) {
    (void)H; (void)G;
    if (chunk <= 0) return M2_ERR_INVALID_ARG;
    if (P == 64 && (N == 128 || N == 64)) return M2_OK;
    return M2_ERR_UNSUPPORTED;
}

cudaError_t launch_chunk_scan(const ScanArgs& a, cudaStream_t s) {
    if (a.batch == 0 || a.total_tokens == 0) return cudaSuccess;
    if (chunk_scan_tc_supported(a)) return launch_chunk_scan_tc(a, s);
    if (a.state_bf16) return a.act_bf16 ? scan_by_x<bf16_t, bf16_t>(a, s) : scan_by_x<bf16_t, float>(a, s);
    return a.act_bf16 ? scan_by_x<float, bf16_t>(a, s) : scan_by_x<float, float>(a, s);
}

}  // namespace m2
