// m2_state_update.cu -- the one-token decode step: selective_state_update,
// optionally with the causal_conv1d_update tap fused into the same launch.
//
// Operation: vllm.cpp issue #1311 "NemotronH runs the PREFILL mamba kernels at
// decode", section "The divergence" (both decode kernels read and write the
// cache in place at the slot; no gather/scatter) and section "Confirm or
// refute" (hpg = H/G head grouping). Per head h, group g = h/(H/G):
//   dt = softplus(dt_raw + dt_bias), dA = exp(dt * -exp(A_log))
//   S' = S*dA + (dt*x)*B[g],  y = sum_n S'*C[g] + D*x,  y *= silu(z)
//
// Work decomposition (HBM-bound: ~96% of the bytes are the state stream).
//  * A sequence's state [H, P, N] is a run of H*P rows of N elements. One CTA
//    of 256 threads owns TILE = 8 warps x RPW rows x LOADS consecutive rows, so
//    its slice of the cache is one contiguous block (64 KB with LOADS = 16).
//  * A row is read by LPR = N*sizeof(state)/16 lanes, one 16-byte vector each,
//    so every lane keeps the same EPV state columns n for all of its rows and
//    holds B[g, n] and C[g, n] for those columns in registers. A warp load
//    instruction covers 512 contiguous bytes.
//  * Each thread issues all LOADS 16-byte loads of the tile before any
//    arithmetic (up to 64 KB in flight per CTA), then updates, stores and
//    reduces y over its LPR lanes with xor shuffles.
//  * Fused conv: the CTA computes the conv tap for its own x channels (and
//    rolls their conv-cache rows, which no other CTA touches) and for the
//    group's B and C channels, which every CTA of the group needs. Those CTAs
//    form one thread-block cluster; each arrives on the cluster barrier after
//    reading the B/C conv rows, and only cluster rank 0 writes the rolled B/C
//    rows, after waiting on the barrier at the very end.
#include <cuda_runtime.h>

#include "m2_device.cuh"
#include "m2_internal.cuh"

namespace m2 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxK = 8;
constexpr int kMaxHeadsPerTile = 33;

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}

// Conv tap for channel c of one row: reads the K-1 cached raw inputs and the
// new raw input, returns the post-conv value (bias, activation) and leaves the
// raw window in win[] (oldest first, newest at K-1).
template <typename AT>
__device__ __forceinline__ float conv_tap(const AT* conv_row0, int64_t conv_dim, int K,
                                          const AT* w, const AT* bias, int activation,
                                          AT new_in, int64_t c, AT* win) {
    float acc = bias ? to_f32(bias[c]) : 0.f;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
        if (k < K) {
            const AT v = (k < K - 1) ? conv_row0[static_cast<int64_t>(k) * conv_dim + c] : new_in;
            win[k] = v;
            acc = fmaf(to_f32(w[c * K + k]), to_f32(v), acc);
        }
    }
    return activation ? silu_f32(acc) : acc;
}

// Roll: conv[k] <- win[k+1] for k < K-1 (exact copies of raw inputs).
template <typename AT>
__device__ __forceinline__ void conv_roll(AT* conv_row0, int64_t conv_dim, int K, int64_t c,
                                          const AT* win) {
#pragma unroll
    for (int k = 0; k < kMaxK - 1; ++k) {
        if (k < K - 1) conv_row0[static_cast<int64_t>(k) * conv_dim + c] = win[k + 1];
    }
}

template <typename ST, typename AT, typename XT, int N, int LOADS, bool FUSED>
__global__ void __launch_bounds__(kThreads)
state_update_kernel(const StateUpdateArgs a) {
    constexpr int EPV = Vec16<ST>::n;       // state elements per 16-byte vector
    constexpr int LPR = N / EPV;            // lanes per state row
    static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "row must fit a warp");
    constexpr int RPW = 32 / LPR;           // rows per warp load instruction
    constexpr int TILE = kWarps * RPW * LOADS;

    __shared__ float s_x[TILE];
    __shared__ float s_B[N];
    __shared__ float s_C[N];
    __shared__ float s_y[TILE];
    __shared__ float s_dt[kMaxHeadsPerTile];
    __shared__ float s_dA[kMaxHeadsPerTile];
    __shared__ float s_D[kMaxHeadsPerTile];

    const int tid = threadIdx.x;
    const int b = blockIdx.y;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * TILE;  // first row (h*P + p)
    const int P = a.P;
    const int H = a.H;
    const int64_t HP = static_cast<int64_t>(H) * P;
    const int hpg = H / a.G;
    const int h_first = static_cast<int>(r0 / P);
    const int g = h_first / hpg;
    const int n_heads_tile = static_cast<int>((r0 + TILE - 1) / P) - h_first + 1;

    const int32_t slot = a.slot_idx[b];
    const AT* zrow = a.z ? static_cast<const AT*>(a.z) + b * a.z_stride : nullptr;
    AT* yrow = static_cast<AT*>(a.y) + b * a.y_stride;

    if (slot < 0) {  // padding row: y = 0, caches untouched (uniform per cluster)
        for (int i = tid; i < TILE; i += kThreads) yrow[r0 + i] = from_f32<AT>(0.f);
        return;
    }
    if (slot >= a.num_slots) {  // bad slot: record, skip, write nothing
        if (tid == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }

    // ---- phase 1: per-head scalars, post-conv x / B / C into shared memory
    if (tid < n_heads_tile) {
        const int h = h_first + tid;
        const float dtr = to_f32(static_cast<const AT*>(a.dt)[b * a.dt_stride + h]);
        const float dt = softplus_f32(dtr + a.dt_bias[h]);
        const float A = -expf(a.A_log[h]);
        s_dt[tid] = dt;
        s_dA[tid] = expf(dt * A);
        s_D[tid] = a.D[h];
    }

    const int64_t cd = a.conv_dim;
    const int64_t cB = HP + static_cast<int64_t>(g) * N;                        // first B channel
    const int64_t cC = HP + static_cast<int64_t>(a.G) * N + static_cast<int64_t>(g) * N;
    // raw windows of this thread's (at most two) B/C channels, kept for the roll
    AT bc_win[2][kMaxK];

    if constexpr (FUSED) {
        const AT* xrow = static_cast<const AT*>(a.xBC) + b * a.xBC_stride;
        AT* conv0 = static_cast<AT*>(a.conv) + static_cast<int64_t>(slot) * (a.K - 1) * cd;
        const AT* w = static_cast<const AT*>(a.conv_w);
        const AT* bias = static_cast<const AT*>(a.conv_b);
        for (int i = tid; i < TILE; i += kThreads) {  // private x channels
            const int64_t c = r0 + i;
            AT win[kMaxK];
            s_x[i] = conv_tap(conv0, cd, a.K, w, bias, a.activation, xrow[c], c, win);
            conv_roll(conv0, cd, a.K, c, win);
        }
        static_assert(2 * N <= 2 * kThreads, "B/C channels: at most two per thread");
#pragma unroll
        for (int q = 0; q < 2; ++q) {  // shared B / C channels
            const int j = tid + q * kThreads;
            if (j < 2 * N) {
                const int64_t c = j < N ? cB + j : cC + (j - N);
                const float v =
                    conv_tap(conv0, cd, a.K, w, bias, a.activation, xrow[c], c, bc_win[q]);
                if (j < N) s_B[j] = v; else s_C[j - N] = v;
            }
        }
        // every CTA of the group has read the B/C conv rows once it arrives here
        cluster_arrive();
    } else {
        const XT* xrow = static_cast<const XT*>(a.xBC) + b * a.xBC_stride;
        for (int i = tid; i < TILE; i += kThreads) s_x[i] = to_f32(xrow[r0 + i]);
        for (int j = tid; j < N; j += kThreads) {
            s_B[j] = to_f32(xrow[cB + j]);
            s_C[j] = to_f32(xrow[cC + j]);
        }
    }
    __syncthreads();

    // ---- phase 2: stream the state tile
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int sub = lane / LPR;          // row within a warp load
    const int e0 = (lane % LPR) * EPV;   // first state column of this lane
    float Bv[EPV], Cv[EPV];
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
        Bv[e] = s_B[e0 + e];
        Cv[e] = s_C[e0 + e];
    }

    ST* tile = static_cast<ST*>(a.ssm) + (static_cast<int64_t>(slot) * HP + r0) * N;
    uint4 v[LOADS];
#pragma unroll
    for (int i = 0; i < LOADS; ++i) {
        const int row = (i * kWarps + warp) * RPW + sub;
        v[i] = ld_stream(tile + static_cast<int64_t>(row) * N + e0);
    }
#pragma unroll
    for (int i = 0; i < LOADS; ++i) {
        const int row = (i * kWarps + warp) * RPW + sub;
        const int hl = static_cast<int>((r0 + row) / P) - h_first;
        const float xv = s_x[row];
        const float dtx = s_dt[hl] * xv;
        const float dA = s_dA[hl];
        float s[EPV];
        unpack16<ST>(v[i], s);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPV; ++e) {
            s[e] = fmaf(s[e], dA, dtx * Bv[e]);
            acc = fmaf(s[e], Cv[e], acc);
        }
        st_stream(tile + static_cast<int64_t>(row) * N + e0, pack16<ST>(s));
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if ((lane % LPR) == 0) s_y[row] = fmaf(s_D[hl], xv, acc);
    }
    __syncthreads();

    // ---- y (gated), contiguous over the tile's rows
    for (int i = tid; i < TILE; i += kThreads) {
        float yv = s_y[i];
        if (zrow) yv *= silu_f32(to_f32(zrow[r0 + i]));
        yrow[r0 + i] = from_f32<AT>(yv);
    }

    if constexpr (FUSED) {
        // ---- phase 3: cluster rank 0 rolls the shared B/C conv rows
        cluster_wait();
        if (cluster_rank() == 0) {
            AT* conv0 = static_cast<AT*>(a.conv) + static_cast<int64_t>(slot) * (a.K - 1) * cd;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int j = tid + q * kThreads;
                if (j < 2 * N) {
                    const int64_t c = j < N ? cB + j : cC + (j - N);
                    conv_roll(conv0, cd, a.K, c, bc_win[q]);
                }
            }
        }
    }
}

template <typename ST, typename AT, typename XT, int N, int LOADS, bool FUSED>
cudaError_t launch_one(const StateUpdateArgs& a, const DecodePlan& plan, cudaStream_t stream) {
    auto kern = state_update_kernel<ST, AT, XT, N, LOADS, FUSED>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.ctas_per_seq, a.batch, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = FUSED ? plan.cluster : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (FUSED && plan.cluster > 8) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename ST, typename AT, typename XT, int N, bool FUSED>
cudaError_t by_loads(const StateUpdateArgs& a, const DecodePlan& p, cudaStream_t s) {
    switch (p.loads) {
        case 16: return launch_one<ST, AT, XT, N, 16, FUSED>(a, p, s);
        case 4: return launch_one<ST, AT, XT, N, 4, FUSED>(a, p, s);
        case 1: return launch_one<ST, AT, XT, N, 1, FUSED>(a, p, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename ST, typename AT, typename XT, bool FUSED>
cudaError_t by_n(const StateUpdateArgs& a, const DecodePlan& p, cudaStream_t s) {
    switch (a.N) {
        case 64: return by_loads<ST, AT, XT, 64, FUSED>(a, p, s);
        case 128: return by_loads<ST, AT, XT, 128, FUSED>(a, p, s);
        case 256:
            if constexpr (sizeof(ST) == 2) return by_loads<ST, AT, XT, 256, FUSED>(a, p, s);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

template <typename ST, typename AT>
cudaError_t by_mode(const StateUpdateArgs& a, const DecodePlan& p, cudaStream_t s) {
    if (a.fused) return by_n<ST, AT, AT, true>(a, p, s);
    if (a.x_bf16) return by_n<ST, AT, bf16_t, false>(a, p, s);
    return by_n<ST, AT, float, false>(a, p, s);
}

}  // namespace

m2_status plan_state_update(int H, int P, int N, int G, int state_bf16, int fused,
                            DecodePlan* plan) {
    if (N != 64 && N != 128 && N != 256) return M2_ERR_UNSUPPORTED;
    if (!state_bf16 && N == 256) return M2_ERR_UNSUPPORTED;
    if (P < 8 || P > 256 || P % 8 != 0) return M2_ERR_UNSUPPORTED;
    const int epv = state_bf16 ? 8 : 4;
    const int lpr = N / epv;
    const int rpw = 32 / lpr;
    const int64_t group_rows = static_cast<int64_t>(H / G) * P;
    static const int kLoads[3] = {16, 4, 1};
    for (int li = 0; li < 3; ++li) {
        const int tile = kWarps * rpw * kLoads[li];
        if (group_rows % tile != 0) continue;
        const int64_t cluster = group_rows / tile;
        if (fused && cluster > 16) return M2_ERR_UNSUPPORTED;  // group too large for a cluster
        if ((tile + P - 1) / P + 1 > kMaxHeadsPerTile) continue;
        plan->loads = kLoads[li];
        plan->tile_rows = tile;
        plan->ctas_per_seq = static_cast<int>(static_cast<int64_t>(H) * P / tile);
        plan->cluster = fused ? static_cast<int>(cluster) : 1;
        return M2_OK;
    }
    return M2_ERR_UNSUPPORTED;
}

cudaError_t launch_state_update(const StateUpdateArgs& a, const DecodePlan& plan,
                                cudaStream_t stream) {
    if (a.state_bf16) {
        return a.act_bf16 ? by_mode<bf16_t, bf16_t>(a, plan, stream)
                          : by_mode<bf16_t, float>(a, plan, stream);
    }
    return a.act_bf16 ? by_mode<float, bf16_t>(a, plan, stream)
                      : by_mode<float, float>(a, plan, stream);
}

}  // namespace m2
