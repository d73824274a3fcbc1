// m2_state_update_mt.cu -- multi-token decode for speculative decoding: T draft
// tokens of one sequence in one launch, with the state after every token kept.
//
// Operation: T consecutive selective_state_update steps with the
// causal_conv1d_update tap (vllm.cpp issue #1311 "NemotronH runs the PREFILL
// mamba kernels at decode", section "The divergence"), from the state and conv
// window of slot_idx[b]. Speculative decoding verifies the T drafts afterwards
// and keeps only an accepted prefix (the Nemotron-H-8B-Base-8K record notes
// the engines serve NemotronH with MTP / EAGLE speculative decoding), so the
// state and conv window after token t are stored into cache slot
// token_slots[b*T + t] of the same cache, and the input slot is only read:
// after verification the caller adopts the slot of the last accepted token.
//
// Work decomposition: one CTA of 256 threads per 64 state rows (the rows of
// 64/P heads) of one sequence. The CTA stages its state tile (16 KB for bf16,
// N = 128) and the conv rows of its x channels and of the group's B/C channels
// with bulk copies, loads the T raw inputs, and then, token by token, runs the
// conv tap (one thread per 16-byte channel vector; the group's B/C conv is
// computed by every CTA of the group), the state update on the tile in shared
// memory (rounded to the storage dtype after every token, exactly as T
// separate decode steps store it), the y reduction, and the stores of the
// token's state and conv rows. The first CTA of each group writes the group's
// B/C conv rows; no CTA writes the input slot, so nothing races with the reads.
#include <cuda_runtime.h>

#include "m2_device.cuh"
#include "m2_internal.cuh"

namespace m2 {
namespace {

constexpr int kMtThreads = 256;
constexpr int kMtRows = 64;   // state rows per CTA
constexpr int kMtMaxHeads = kMtRows / 8 + 1;
constexpr uint64_t kMtWaitNs = 1000000000ull;

template <typename ST, typename AT, int N>
__global__ void __launch_bounds__(kMtThreads) mt_decode_kernel(const MtArgs a) {
    constexpr int EPV = Vec16<ST>::n;        // state elements per 16-byte vector
    constexpr int LPR = N / EPV;             // lanes per state row
    static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row must fit a warp");
    constexpr int VPT = kMtRows * LPR / kMtThreads;  // vectors per thread per token
    static_assert(VPT >= 1 && kMtRows * LPR == VPT * kMtThreads, "whole passes");
    constexpr uint32_t TILE_BYTES = kMtRows * N * sizeof(ST);
    constexpr int AV = Vec16<AT>::n;         // activation elements per 16-byte vector
    constexpr int XV = kMtRows / AV;         // x-channel vectors of the tile
    constexpr int BV = N / AV;               // vectors of one B (or C) segment

    const int T = a.T;
    const int K = a.K;
    const int W = K - 1 + T;                 // window rows: K-1 cached, then T raw inputs
    extern __shared__ __align__(128) uint8_t s_dyn[];
    uint8_t* s_state = s_dyn;                                        // [64][N] ST
    AT* s_xw = reinterpret_cast<AT*>(s_dyn + TILE_BYTES);            // [W][64] raw x window
    AT* s_bcw = s_xw + static_cast<size_t>(W) * kMtRows;              // [W][2N] raw B|C window
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ __align__(16) float s_x[kMtRows];                     // post-conv x of the token
    __shared__ __align__(16) float s_B[N];
    __shared__ __align__(16) float s_C[N];
    __shared__ float s_y[kMtRows];
    __shared__ float s_dt[kMtMaxHeads];
    __shared__ float s_dA[kMtMaxHeads];
    __shared__ float s_D[kMtMaxHeads];
    __shared__ int s_fail;

    const int tid = threadIdx.x;
    const int b = blockIdx.y;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kMtRows;   // first row h*P + p
    const int P = a.P;
    const int64_t HP = static_cast<int64_t>(a.H) * P;
    const int hpg = a.H / a.G;
    const int h_first = static_cast<int>(r0 / P);
    const int g = h_first / hpg;
    const int n_heads = (kMtRows + P - 1) / P;
    const int64_t cd = a.conv_dim;
    const int64_t cB = HP + static_cast<int64_t>(g) * N;
    const int64_t cC = HP + static_cast<int64_t>(a.G) * N + static_cast<int64_t>(g) * N;
    const bool bc_writer = (r0 % (static_cast<int64_t>(hpg) * P)) == 0;  // first CTA of the group
    const AT* xbase = static_cast<const AT*>(a.xBC) + static_cast<int64_t>(b) * T * a.xBC_stride;
    AT* ybase = static_cast<AT*>(a.y) + static_cast<int64_t>(b) * T * a.y_stride;

    const int32_t slot = a.slot_idx[b];
    if (slot < 0) {  // padding row: y = 0 for every token, no state stored
        for (int i = tid; i < T * kMtRows; i += kMtThreads)
            ybase[static_cast<int64_t>(i / kMtRows) * a.y_stride + r0 + i % kMtRows] = from_f32<AT>(0.f);
        return;
    }
    if (slot >= a.num_slots) {
        if (tid == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }

    // ---- stage the input slot's state tile and conv rows; load the raw inputs
    const ST* tile = static_cast<const ST*>(a.ssm) + (static_cast<int64_t>(slot) * HP + r0) * N;
    const AT* conv_in = static_cast<const AT*>(a.conv) + static_cast<int64_t>(slot) * (K - 1) * cd;
    if (tid == 0) {
        s_fail = 0;
        mbar_init(&s_bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&s_bar, TILE_BYTES + static_cast<uint32_t>(K - 1) * (kMtRows + 2 * N) * sizeof(AT));
        bulk_g2s(s_state, tile, TILE_BYTES, &s_bar);
        for (int k = 0; k < K - 1; ++k) {
            bulk_g2s(s_xw + k * kMtRows, conv_in + k * cd + r0, kMtRows * sizeof(AT), &s_bar);
            bulk_g2s(s_bcw + k * 2 * N, conv_in + k * cd + cB, N * sizeof(AT), &s_bar);
            bulk_g2s(s_bcw + k * 2 * N + N, conv_in + k * cd + cC, N * sizeof(AT), &s_bar);
        }
    }
    __syncthreads();  // the barrier is initialised before any thread waits on it
    // raw inputs of the T tokens (x channels of the tile, the group's B and C)
    for (int i = tid; i < T * (XV + 2 * BV); i += kMtThreads) {
        const int t = i / (XV + 2 * BV);
        const int v = i % (XV + 2 * BV);
        const AT* row = xbase + static_cast<int64_t>(t) * a.xBC_stride;
        if (v < XV) {
            *reinterpret_cast<uint4*>(s_xw + (K - 1 + t) * kMtRows + v * AV) =
                *reinterpret_cast<const uint4*>(row + r0 + v * AV);
        } else {
            const int u = v - XV;  // 0 .. 2*BV-1: B then C
            const int64_t c0 = (u < BV ? cB : cC - BV * AV) + u * AV;
            *reinterpret_cast<uint4*>(s_bcw + (K - 1 + t) * 2 * N + u * AV) =
                *reinterpret_cast<const uint4*>(row + c0);
        }
    }
    // this thread's conv channel vector (fixed for all tokens): weights and bias
    const int nvec = XV + 2 * BV;
    const bool conv_thread = tid < nvec;
    int64_t c_vec = 0;
    const AT* win = nullptr;   // window column of the vector in shared memory
    int win_pitch = 0;
    float wt[AV][8];
    float bias[AV];
    if (conv_thread) {
        if (tid < XV) {
            c_vec = r0 + tid * AV;
            win = s_xw + tid * AV;
            win_pitch = kMtRows;
        } else {
            const int u = tid - XV;
            c_vec = (u < BV ? cB : cC - BV * AV) + u * AV;
            win = s_bcw + u * AV;
            win_pitch = 2 * N;
        }
        const AT* wp = static_cast<const AT*>(a.conv_w) + c_vec * K;
#pragma unroll
        for (int e = 0; e < AV; ++e) {
#pragma unroll
            for (int k = 0; k < 8; ++k) wt[e][k] = k < K ? to_f32(wp[e * K + k]) : 0.f;
            bias[e] = a.conv_b ? to_f32(static_cast<const AT*>(a.conv_b)[c_vec + e]) : 0.f;
        }
    }
    const bool wait_ok = mbar_wait_bounded(&s_bar, 0, kMtWaitNs);
    if (!wait_ok) s_fail = 1;
    __syncthreads();
    if (s_fail) {
        if (tid == 0) record_error(a.error, M2_ERR_TIMEOUT);
        mbar_wait_bounded(&s_bar, 0, kMtWaitNs);  // this CTA's copies land before it leaves
        return;
    }

    const int lane = tid & 31;
    const int e0 = (lane % LPR) * EPV;
    const int64_t HPN = HP * N;
    for (int t = 0; t < T; ++t) {
        // ---- conv tap of token t (window rows t .. t+K-1) and the head scalars
        if (conv_thread) {
            float out[AV];
#pragma unroll
            for (int e = 0; e < AV; ++e) out[e] = bias[e];
            for (int k = 0; k < K; ++k) {
                float rv[AV];
                unpack16<AT>(*reinterpret_cast<const uint4*>(win + (t + k) * win_pitch), rv);
#pragma unroll
                for (int e = 0; e < AV; ++e) out[e] = fmaf(wt[e][k], rv[e], out[e]);
            }
#pragma unroll
            for (int e = 0; e < AV; ++e) {
                const float o = a.activation ? silu_f32(out[e]) : out[e];
                if (tid < XV) {
                    s_x[tid * AV + e] = o;
                } else {
                    const int u = tid - XV;
                    if (u < BV) s_B[u * AV + e] = o;
                    else s_C[(u - BV) * AV + e] = o;
                }
            }
        } else if (tid >= 224 && tid - 224 < n_heads) {
            const int hl = tid - 224;
            const int h = h_first + hl;
            const float dtr = to_f32(static_cast<const AT*>(a.dt)[(static_cast<int64_t>(b) * T + t) * a.dt_stride + h]);
            const float dt = softplus_f32(dtr + a.dt_bias[h]);
            s_dt[hl] = dt;
            s_dA[hl] = expf(dt * -expf(a.A_log[h]));
            s_D[hl] = a.D[h];
        }
        __syncthreads();

        // ---- state update of the tile, y partial sums, token state stores
        const int32_t dest = a.token_slots[static_cast<int64_t>(b) * T + t];
        const bool store = dest >= 0 && dest < a.num_slots;
        if (dest >= a.num_slots && tid == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        ST* dtile = store ? static_cast<ST*>(a.ssm) + static_cast<int64_t>(dest) * HPN + r0 * N : nullptr;
        float Bv[EPV], Cv[EPV];
#pragma unroll
        for (int e = 0; e < EPV; ++e) {
            Bv[e] = s_B[e0 + e];
            Cv[e] = s_C[e0 + e];
        }
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = i * kMtThreads + tid;
            const int row = v / LPR;
            const int hl = static_cast<int>((r0 + row) / P) - h_first;
            const float dtx = s_dt[hl] * s_x[row];
            const float dA = s_dA[hl];
            uint4* sp = reinterpret_cast<uint4*>(s_state + static_cast<uint32_t>(v) * 16u);
            float st[EPV];
            unpack16<ST>(*sp, st);
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < EPV; ++e) {
                st[e] = fmaf(st[e], dA, dtx * Bv[e]);
                acc = fmaf(st[e], Cv[e], acc);
            }
            const uint4 packed = pack16<ST>(st);  // the stored state, rounded once per token
            *sp = packed;
            if (store) st_stream(dtile + static_cast<int64_t>(row) * N + e0, packed);
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if ((lane % LPR) == 0) s_y[row] = acc + s_D[hl] * s_x[row];
        }
        __syncthreads();

        // ---- gated y of the token; the token's conv window into the destination slot
        if (tid < kMtRows) {
            float yv = s_y[tid];
            if (a.z) {
                const AT* zr = static_cast<const AT*>(a.z) + (static_cast<int64_t>(b) * T + t) * a.z_stride;
                yv *= silu_f32(to_f32(zr[r0 + tid]));
            }
            ybase[static_cast<int64_t>(t) * a.y_stride + r0 + tid] = from_f32<AT>(yv);
        }
        if (store && conv_thread && (tid < XV || bc_writer)) {
            // new row k of the destination = window row t+1+k (raw inputs, exact copies)
            AT* conv_out = static_cast<AT*>(a.conv) + static_cast<int64_t>(dest) * (K - 1) * cd;
            for (int k = 0; k < K - 1; ++k)
                *reinterpret_cast<uint4*>(conv_out + k * cd + c_vec) =
                    *reinterpret_cast<const uint4*>(win + (t + 1 + k) * win_pitch);
        }
        // the next token's conv overwrites s_x / s_B / s_C read above
        __syncthreads();
    }
}

template <typename ST, typename AT>
cudaError_t mt_by_n(const MtArgs& a, cudaStream_t s) {
    const size_t smem_max = static_cast<size_t>(kMtRows) * 256 * sizeof(ST) +
                            static_cast<size_t>(7 + kMaxDraftTokens) * (kMtRows + 2 * 256) * sizeof(AT);
    const size_t tile = static_cast<size_t>(kMtRows) * a.N * sizeof(ST);
    const size_t smem = tile + static_cast<size_t>(a.K - 1 + a.T) * (kMtRows + 2 * a.N) * sizeof(AT);
    const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(a.H) * a.P / kMtRows), static_cast<unsigned>(a.batch));
    auto launch = [&](auto kern) -> cudaError_t {
        static AttrOnce attrs;
        const cudaError_t e = attrs.ensure([&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_max));
        });
        if (e != cudaSuccess) return e;
        kern<<<grid, kMtThreads, smem, s>>>(a);
        return cudaGetLastError();
    };
    switch (a.N) {
        case 64: return launch(mt_decode_kernel<ST, AT, 64>);
        case 128: return launch(mt_decode_kernel<ST, AT, 128>);
        case 256:
            if constexpr (sizeof(ST) == 2) return launch(mt_decode_kernel<ST, AT, 256>);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

m2_status plan_multi_token(int H, int P, int N, int G, int K, int T) {
    if (T < 1 || T > kMaxDraftTokens || K < 2 || K > 8) return M2_ERR_UNSUPPORTED;
    if (N != 64 && N != 128 && N != 256) return M2_ERR_UNSUPPORTED;
    const int64_t group_rows = static_cast<int64_t>(H / G) * P;
    // 64-row tiles that never straddle a group (the group's first CTA writes its B/C rows)
    if (group_rows % kMtRows != 0 || P % 8 != 0) return M2_ERR_UNSUPPORTED;
    return M2_OK;
}

cudaError_t launch_state_update_mt(const MtArgs& a, cudaStream_t stream) {
    if (a.state_bf16) return a.act_bf16 ? mt_by_n<bf16_t, bf16_t>(a, stream) : mt_by_n<bf16_t, float>(a, stream);
    if (a.N == 256) return cudaErrorInvalidValue;
    return a.act_bf16 ? mt_by_n<float, bf16_t>(a, stream) : mt_by_n<float, float>(a, stream);
}

}  // namespace m2
