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
//    of 256 threads owns TILE consecutive rows, one contiguous block of the
//    cache (64 KB in the main configuration), split in CHUNKS chunks.
//  * Right after reading its slot index, one thread issues the slot's conv
//    rows (fused: three 2-D TMA boxes, the tile's x rows and the group's B and
//    C rows, where the shared-memory layout allows; else row by row) and the
//    whole tile as bulk asynchronous copies (cp.async.bulk) into shared
//    memory, one mbarrier per chunk, so the tile's bytes are in flight while
//    the CTA runs the conv tap and the per-head scalars. Registers are not used as the
//    staging buffer, which lets three CTAs share an SM.
//  * A state row is handled by LPR = N*sizeof(state)/16 lanes, one 16-byte
//    vector each, so every lane keeps the same EPV state columns n for all of
//    its rows and holds B[g, n] and C[g, n] for those columns in registers.
//    Shared-memory reads are linear (conflict free); the new state goes
//    straight from registers to global memory with 16-byte streaming stores.
//    y is reduced over the LPR lanes with xor shuffles.
//  * Waits on the copies are bounded (one second of %globaltimer); on a
//    timeout the CTA records M2_ERR_TIMEOUT, waits once more (bounded) for its
//    copies and skips the rest of its tile.
//  * Fused conv: the CTA computes the conv tap for its own x channels (and
//    rolls their conv-cache rows, which no other CTA touches) and for the
//    group's B and C channels, which every CTA of the group needs. Those CTAs
//    form one thread-block cluster; each arrives on the cluster barrier after
//    reading the B/C conv rows, and only cluster rank 0 waits on it (at the
//    very end) and then writes the rolled B/C rows.
#include <cuda_runtime.h>

#include <climits>

#include "m2_device.cuh"
#include "m2_internal.cuh"

namespace m2 {
namespace {

// Tuning knobs (compile-time): resident CTAs per SM the register budget is
// sized for, and 16 KB chunks per CTA tile in the main configuration.
#ifndef M2_DECODE_MIN_BLOCKS
#define M2_DECODE_MIN_BLOCKS 3
#endif
#ifndef M2_DECODE_MAIN_CHUNKS
#define M2_DECODE_MAIN_CHUNKS 4
#endif

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxHeadsPerTile = 33;

// Relaxed arrive: the only cross-CTA hazard it orders is WAR on the group's
// B/C conv rows, and those rows were read by bulk copies whose completion every
// reading thread has already observed on its mbarrier before arriving.
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;\n" : "=r"(n));
    return n;
}
// Release arrive: this CTA's shared-memory writes before it become visible to
// the cluster threads that complete the matching wait.
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
// Stores v into the shared memory of cluster CTA `rank`, at the offset of `local`.
__device__ __forceinline__ void st_cluster_f32(float* local, uint32_t rank, float v) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;\n" ::"r"(remote), "f"(v) : "memory");
}

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bounded waits: one second


// Slot-independent inputs of one conv vector (AV channels c0..): the raw
// input, the bias and, for K = 4, the AV x K weight block, which is exactly
// four 16-byte vectors with (e, k) at e*K + k. Loaded before the slot index
// is known, so their latency overlaps the slot read and the bulk copies.
struct ConvIn {
    uint4 xin;
    uint4 bias;
    uint4 w[4];
};

template <typename AT>
__device__ __forceinline__ ConvIn load_conv_in(const AT* xrow, const AT* w, const AT* bias, int64_t c0, int K) {
    ConvIn in;
    in.xin = *reinterpret_cast<const uint4*>(xrow + c0);
    in.bias = bias ? __ldg(reinterpret_cast<const uint4*>(bias + c0)) : make_uint4(0, 0, 0, 0);
    if (K == 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) in.w[q] = __ldg(reinterpret_cast<const uint4*>(w + c0 * 4) + q);
    }
    return in;
}

// K = 4 conv inputs of one quarter of a 16-byte channel vector: CQ = AV / 4
// consecutive channels c0.. (two bf16 or one fp32), i.e. 4 bytes of raw input
// and bias and the CQ x 4 weight block, one 16-byte vector ((e, k) at e*4 + k).
struct QuadIn {
    uint4 w;
    uint32_t xin;
    uint32_t bias;
};

template <typename AT>
__device__ __forceinline__ QuadIn load_quad_in(const AT* xrow, const AT* w, const AT* bias, int64_t c0) {
    QuadIn in;
    in.xin = *reinterpret_cast<const uint32_t*>(xrow + c0);
    in.bias = bias ? __ldg(reinterpret_cast<const uint32_t*>(bias + c0)) : 0u;
    in.w = __ldg(reinterpret_cast<const uint4*>(w + c0 * 4));
    return in;
}

// The 4 bytes of a quarter vector as floats: two bf16 (lo, hi) or one fp32.
template <typename AT>
__device__ __forceinline__ void unpack4(uint32_t u, float* out);
template <>
__device__ __forceinline__ void unpack4<bf16_t>(uint32_t u, float* out) {
    out[0] = __uint_as_float(u << 16);
    out[1] = __uint_as_float(u & 0xFFFF0000u);
}
template <>
__device__ __forceinline__ void unpack4<float>(uint32_t u, float* out) { out[0] = __uint_as_float(u); }

// Conv tap of AV consecutive channels c0.. for one row: the K-1 cached raw
// inputs (staged in shared memory at `rows`, row pitch `pitch` elements,
// oldest first) and the raw input; tap K-1 multiplies the newest input.
// Returns false if the bounded wait for the staged rows ran out.
template <typename AT, int AV>
__device__ __forceinline__ bool conv_vec_k4(const ConvIn& in, const AT* rows, int64_t pitch, int activation,
                                            uint64_t* bar, float (&out)[AV]) {
    constexpr int K = 4;
    float wf[AV * K];
#pragma unroll
    for (int q = 0; q < K; ++q) unpack16<AT>(in.w[q], wf + q * AV);
    unpack16<AT>(in.bias, out);
    if (!mbar_wait_bounded(bar, 0, kWaitLimitNs)) return false;
    const uint4& xin = in.xin;
    float xv[AV];
    unpack16<AT>(xin, xv);
#pragma unroll
    for (int k = 0; k < K - 1; ++k) {
        float rv[AV];
        unpack16<AT>(*reinterpret_cast<const uint4*>(rows + k * pitch), rv);
#pragma unroll
        for (int e = 0; e < AV; ++e) out[e] = fmaf(wf[e * K + k], rv[e], out[e]);
    }
#pragma unroll
    for (int e = 0; e < AV; ++e) {
        out[e] = fmaf(wf[e * K + K - 1], xv[e], out[e]);
        if (activation) out[e] = silu_f32(out[e]);
    }
    return true;
}

// Same for any width K (2..8): weights read one by one (cached).
template <typename AT, int AV>
__device__ __forceinline__ bool conv_vec_any(const ConvIn& in, const AT* w, int64_t c0, int K,
                                             const AT* rows, int64_t pitch, int activation,
                                             uint64_t* bar, float (&out)[AV]) {
    unpack16<AT>(in.bias, out);
    if (!mbar_wait_bounded(bar, 0, kWaitLimitNs)) return false;
    const uint4& xin = in.xin;
    float xv[AV];
    unpack16<AT>(xin, xv);
#pragma unroll
    for (int e = 0; e < AV; ++e) {
        for (int k = 0; k < K; ++k) {
            const float in = (k < K - 1) ? to_f32(rows[k * pitch + e]) : xv[e];
            out[e] = fmaf(to_f32(__ldg(w + (c0 + e) * K + k)), in, out[e]);
        }
        if (activation) out[e] = silu_f32(out[e]);
    }
    return true;
}

// NORM (fused only): the gated y goes through the gated RMSNorm before it is
// stored. The norm's channel group (the hpg*P rows of an SSM group) is exactly
// the CTA cluster, so the group's sum of squares is exchanged through
// distributed shared memory.
// map_cx / map_cbc (fused, use_tma): the conv cache as (channel, slot*(K-1) + k)
// with boxes of TILE and of N channels x K-1 rows, for the tile's x rows and
// the group's B and C rows; use_tma = 0: every row is a bulk copy.
template <typename ST, typename AT, typename XT, int N, int CHUNKS, int VPT, bool FUSED, bool NORM>
__global__ void __launch_bounds__(kThreads, M2_DECODE_MIN_BLOCKS)
state_update_kernel(const __grid_constant__ CUtensorMap map_cx, const __grid_constant__ CUtensorMap map_cbc,
                    const StateUpdateArgs a, const int use_tma) {
    static_assert(FUSED || !NORM, "the norm exchange needs the group cluster of the fused launch");
    constexpr int EPV = Vec16<ST>::n;       // state elements per 16-byte vector
    constexpr int LPR = N / EPV;            // lanes per state row
    static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "row must fit a warp");
    constexpr int RPP = kThreads / LPR;     // rows per pass of the CTA
    constexpr int RC = RPP * VPT;           // rows per chunk
    constexpr int TILE = RC * CHUNKS;       // rows per CTA
    constexpr uint32_t CHUNK_BYTES = RC * N * sizeof(ST);
    constexpr uint32_t TILE_BYTES = CHUNK_BYTES * CHUNKS;
    static_assert(CHUNK_BYTES % 16 == 0, "bulk copies move multiples of 16 bytes");
    constexpr int AV = Vec16<AT>::n;        // activation elements per 16-byte vector
    constexpr int XV = TILE / AV;           // 16-byte vectors of x channels in the tile
    constexpr int BV = N / AV;              // 16-byte vectors of one B (or C) segment
    static_assert(TILE % AV == 0 && N % AV == 0, "whole activation vectors");
    constexpr uint32_t XROW_BYTES = TILE * sizeof(AT);
    constexpr uint32_t BROW_BYTES = N * sizeof(AT);
    constexpr int kHalf = kThreads / 2;     // x-conv threads | B/C-conv threads

    // dynamic: [state tile | conv rows of the tile's x channels | conv rows of B, then of C]
    extern __shared__ __align__(128) uint8_t s_dyn[];
    uint8_t* s_tile = s_dyn;
    const AT* s_cx = reinterpret_cast<const AT*>(s_dyn + TILE_BYTES);                 // [K-1][TILE]
    const AT* s_cbc = reinterpret_cast<const AT*>(s_dyn + TILE_BYTES + (a.K - 1) * XROW_BYTES);  // [2][K-1][N]
    __shared__ __align__(8) uint64_t s_bar[CHUNKS + 1];  // one per state chunk, one for the conv rows
    __shared__ __align__(16) float4 s_rp[TILE];          // per row: dt*x, dA, D*x
    __shared__ __align__(16) float s_B[N];
    __shared__ __align__(16) float s_C[N];
    // (fused, K = 4) the raw B and C inputs of this step, for cluster rank 0's roll
    __shared__ __align__(16) uint32_t s_rawbc[2 * N * sizeof(AT) / 4];
    __shared__ float s_y[TILE];
    __shared__ float s_dt[kMaxHeadsPerTile];
    __shared__ float s_dA[kMaxHeadsPerTile];
    __shared__ float s_D[kMaxHeadsPerTile];
    __shared__ int s_fail;
    __shared__ float s_red[kWarps];  // (NORM) per-warp sums of squares
    __shared__ float s_parts[16];    // (NORM) every cluster CTA's sum of squares, pushed by each
    __shared__ float s_rstd;         // (NORM) 1 / sqrt(mean square + eps) of the group

    const int tid = threadIdx.x;
    const int b = blockIdx.y;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * TILE;  // first row (h*P + p)
    const int P = a.P;
    const int H = a.H;
    const int K = a.K;
    const int64_t HP = static_cast<int64_t>(H) * P;
    const int hpg = H / a.G;
    const int h_first = static_cast<int>(r0 / P);
    // r0's row within its head: head offsets below use 32-bit arithmetic
    const int rr0 = static_cast<int>(r0 - static_cast<int64_t>(h_first) * P);
    const int g = h_first / hpg;
    const int n_heads_tile = static_cast<int>((r0 + TILE - 1) / P) - h_first + 1;
    const int64_t cd = a.conv_dim;
    const int64_t cB = HP + static_cast<int64_t>(g) * N;                        // first B channel
    const int64_t cC = HP + static_cast<int64_t>(a.G) * N + static_cast<int64_t>(g) * N;

    const AT* zrow = a.z ? static_cast<const AT*>(a.z) + b * a.z_stride : nullptr;
    AT* yrow = static_cast<AT*>(a.y) + b * a.y_stride;

    // Launched as a programmatic dependent of the previous kernel on the stream:
    // nothing here may read global memory before that kernel has completed and
    // its writes are visible (the inputs, the slots and the cache may all come
    // from it). Only the launch and the CTA set-up overlap its tail.
    asm volatile("griddepcontrol.wait;\n" ::: "memory");

    // ---- slot-independent inputs first: under a saturated memory system every
    // dependent round trip costs microseconds, so these loads are issued before
    // the slot read and overlap it and the bulk copies.
    // (a) this thread's first conv vector (fused) or x value and B/C column (unfused)
    const bool first_half = tid < kHalf;
    const int v_first = first_half ? tid : tid - kHalf;
    ConvIn cin_first{};
    QuadIn qin_first{};
    float x_first = 0.f, b_first = 0.f, c_first = 0.f;
    // K = 4: every thread takes a quarter of a channel vector (vector tid / 4)
    constexpr int CQ = AV / 4;           // channels per quarter vector
    constexpr int NVC = XV + 2 * BV;     // conv vectors: the tile's x channels, the group's B and C
    auto quad_channel = [&](int q, bool& is_x, int& v, int& sub) -> int64_t {
        v = q >> 2;
        sub = q & 3;
        is_x = v < XV;
        if (is_x) return r0 + static_cast<int64_t>(v) * AV + sub * CQ;
        const int u = v - XV;
        return ((u / BV) ? cC : cB) + (u % BV) * AV + sub * CQ;
    };
    if constexpr (FUSED) {
        const int nvec = first_half ? XV : 2 * BV;
        if (K == 4) {
            if (tid < 4 * NVC) {
                bool is_x;
                int v, sub;
                const int64_t c0 = quad_channel(tid, is_x, v, sub);
                qin_first = load_quad_in<AT>(static_cast<const AT*>(a.xBC) + b * a.xBC_stride,
                                             static_cast<const AT*>(a.conv_w), static_cast<const AT*>(a.conv_b), c0);
            }
        } else if (v_first < nvec) {
            const int64_t c0 = first_half ? r0 + static_cast<int64_t>(v_first) * AV
                                          : ((v_first / BV) ? cC : cB) + (v_first % BV) * AV;
            cin_first = load_conv_in<AT>(static_cast<const AT*>(a.xBC) + b * a.xBC_stride,
                                         static_cast<const AT*>(a.conv_w), static_cast<const AT*>(a.conv_b),
                                         c0, K);
        }
    } else {
        const XT* xrow = static_cast<const XT*>(a.xBC) + b * a.xBC_stride;
        if (tid < TILE) x_first = to_f32(xrow[r0 + tid]);
        if (tid < N) {
            b_first = to_f32(xrow[cB + tid]);
            c_first = to_f32(xrow[cC + tid]);
        }
    }
    // (b) the raw per-head scalars
    float hs_dtr = 0.f, hs_bias = 0.f, hs_alog = 0.f, hs_D = 0.f;
    if (tid < n_heads_tile) {
        const int h = h_first + tid;
        hs_dtr = to_f32(static_cast<const AT*>(a.dt)[b * a.dt_stride + h]);
        hs_bias = a.dt_bias[h];
        hs_alog = a.A_log[h];
        hs_D = a.D[h];
    }
    // (c) z of this thread's first y row (and its norm weight)
    float z_first = 0.f;
    if (zrow && tid < TILE) z_first = to_f32(zrow[r0 + tid]);
    float nw_first = 0.f;
    if constexpr (NORM) {
        if (tid < TILE) nw_first = to_f32(static_cast<const AT*>(a.norm_w)[r0 + tid]);
    }

    const int32_t slot = a.slot_idx[b];

    if (slot < 0) {  // padding row: y = 0, caches untouched (uniform per cluster)
        for (int i = tid; i < TILE; i += kThreads) yrow[r0 + i] = from_f32<AT>(0.f);
        return;
    }
    if (slot >= a.num_slots) {  // bad slot: record, skip, write nothing
        if (tid == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }

    // ---- phase 0: the slot's conv rows, then the whole state tile, go in flight
    ST* tile = static_cast<ST*>(a.ssm) + (static_cast<int64_t>(slot) * HP + r0) * N;
    AT* conv0 = static_cast<AT*>(a.conv) + static_cast<int64_t>(slot) * (K - 1) * cd;
    uint64_t* bar_conv = &s_bar[CHUNKS];
    if (tid == 0) {
        s_fail = 0;
#pragma unroll
        for (int c = 0; c <= CHUNKS; ++c) mbar_init(&s_bar[c], 1);
        fence_mbar_init();
        if constexpr (FUSED) {
            mbar_arrive_expect_tx(bar_conv, (K - 1) * (XROW_BYTES + 2 * BROW_BYTES));
            uint8_t* dst = s_dyn + TILE_BYTES;
            uint8_t* dbc = dst + (K - 1) * XROW_BYTES;
            if (use_tma) {  // three 2-D boxes: the x rows, the B rows, the C rows
                const int crow = slot * (K - 1);
                tma_load_tile_2d(dst, &map_cx, static_cast<int>(r0), crow, bar_conv);
                tma_load_tile_2d(dbc, &map_cbc, static_cast<int>(cB), crow, bar_conv);
                tma_load_tile_2d(dbc + (K - 1) * BROW_BYTES, &map_cbc, static_cast<int>(cC), crow, bar_conv);
            } else {
                for (int k = 0; k < K - 1; ++k) {
                    bulk_g2s(dst + k * XROW_BYTES, conv0 + k * cd + r0, XROW_BYTES, bar_conv);
                    bulk_g2s(dbc + k * BROW_BYTES, conv0 + k * cd + cB, BROW_BYTES, bar_conv);
                    bulk_g2s(dbc + (K - 1 + k) * BROW_BYTES, conv0 + k * cd + cC, BROW_BYTES, bar_conv);
                }
            }
        }
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
            mbar_arrive_expect_tx(&s_bar[c], CHUNK_BYTES);
            bulk_g2s(s_tile + c * CHUNK_BYTES, reinterpret_cast<const uint8_t*>(tile) + c * CHUNK_BYTES,
                     CHUNK_BYTES, &s_bar[c]);
        }
    }
    // every CTA of this grid has its copies in flight: the next kernel on the
    // stream may be scheduled (it waits for this grid's completion before it
    // reads anything)
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    // per-head scalars (n_heads_tile <= kMaxHeadsPerTile < kThreads: one per thread)
    if (tid < n_heads_tile) {
        const float dt = softplus_f32(hs_dtr + hs_bias);
        const float A = -expf(hs_alog);
        s_dt[tid] = dt;
        s_dA[tid] = expf(dt * A);
        s_D[tid] = hs_D;
    }
    __syncthreads();  // barrier initialisation and head scalars visible to all threads

    // ---- phase 1: post-conv x (into the row parameters) and B, C
    if constexpr (FUSED) {
        const AT* xrow = static_cast<const AT*>(a.xBC) + b * a.xBC_stride;
        const AT* w = static_cast<const AT*>(a.conv_w);
        const AT* bias = static_cast<const AT*>(a.conv_b);
        const int nvec = first_half ? XV : 2 * BV;
        if (K == 4) {
            // every thread: a quarter of a 16-byte channel vector (CQ channels),
            // so the conv's FMA and SiLU chains are short and no warp idles; per
            // channel the same operations in the same order as conv_vec_k4
            QuadIn qin = qin_first;  // the first quarter's inputs were loaded up front
            for (int q = tid; q < 4 * NVC; q += kThreads) {
                bool is_x;
                int v, sub;
                const int64_t c0 = quad_channel(q, is_x, v, sub);
                const AT* rows;
                int row_pitch;
                if (is_x) {
                    rows = s_cx + v * AV + sub * CQ;
                    row_pitch = TILE;
                } else {
                    const int u = v - XV;
                    rows = s_cbc + (u / BV) * (K - 1) * N + (u % BV) * AV + sub * CQ;
                    row_pitch = N;
                }
                if (q != tid) qin = load_quad_in<AT>(xrow, w, bias, c0);
                float wf[4 * CQ], out[CQ], xv[CQ];
                {
                    float w8[8];
                    unpack16<AT>(qin.w, w8);  // (e, k) at e*4 + k
#pragma unroll
                    for (int i = 0; i < 4 * CQ; ++i) wf[i] = w8[i];
                }
                unpack4<AT>(qin.bias, out);
                if (!mbar_wait_bounded(bar_conv, 0, kWaitLimitNs)) {
                    record_error(a.error, M2_ERR_TIMEOUT);
                    s_fail = 1;
                    break;
                }
                unpack4<AT>(qin.xin, xv);
                uint32_t rr[3];
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    rr[k] = *reinterpret_cast<const uint32_t*>(rows + k * row_pitch);
                    float rv[CQ];
                    unpack4<AT>(rr[k], rv);
#pragma unroll
                    for (int e = 0; e < CQ; ++e) out[e] = fmaf(wf[e * 4 + k], rv[e], out[e]);
                }
#pragma unroll
                for (int e = 0; e < CQ; ++e) {
                    out[e] = fmaf(wf[e * 4 + 3], xv[e], out[e]);
                    if (a.activation) out[e] = silu_f32(out[e]);
                }
                if (is_x) {
                    // roll the private x rows: row k <- row k+1, last row <- raw input
                    *reinterpret_cast<uint32_t*>(conv0 + c0) = rr[1];
                    *reinterpret_cast<uint32_t*>(conv0 + cd + c0) = rr[2];
                    *reinterpret_cast<uint32_t*>(conv0 + 2 * cd + c0) = qin.xin;
                    // the rows of one vector lie in one head (r0 and P are multiples of 8)
                    const int hl = (rr0 + v * AV) / P;
                    const float dtv = s_dt[hl], dAv = s_dA[hl], Dv = s_D[hl];
#pragma unroll
                    for (int e = 0; e < CQ; ++e)
                        s_rp[v * AV + sub * CQ + e] = make_float4(dtv * out[e], dAv, Dv * out[e], 0.f);
                } else {
                    const int u = v - XV;
                    float* dstf = (u / BV) ? s_C : s_B;
#pragma unroll
                    for (int e = 0; e < CQ; ++e) dstf[(u % BV) * AV + sub * CQ + e] = out[e];
                    s_rawbc[((u / BV) * N + (u % BV) * AV + sub * CQ) * sizeof(AT) / 4] = qin.xin;
                }
            }
        } else {
        ConvIn cin = cin_first;  // the first vector's inputs were loaded up front
        for (int v = v_first; v < nvec; v += kHalf) {
            // channel c0 .. c0+AV-1 and where its cached rows sit in shared memory
            int64_t c0;
            const AT* rows;
            int64_t row_pitch;
            if (first_half) {
                c0 = r0 + static_cast<int64_t>(v) * AV;
                rows = s_cx + v * AV;
                row_pitch = TILE;
            } else {
                const int seg = v / BV;                        // 0 = B, 1 = C
                const int j0 = (v % BV) * AV;
                c0 = (seg ? cC : cB) + j0;
                rows = s_cbc + seg * (K - 1) * N + j0;
                row_pitch = N;
            }
            if (v != v_first) cin = load_conv_in<AT>(xrow, w, bias, c0, K);
            const uint4 xin = cin.xin;
            float out[AV];
            bool got;
            if (K == 4) {
                got = conv_vec_k4<AT, AV>(cin, rows, row_pitch, a.activation, bar_conv, out);
            } else {
                got = conv_vec_any<AT, AV>(cin, w, c0, K, rows, row_pitch, a.activation, bar_conv, out);
            }
            if (!got) {
                record_error(a.error, M2_ERR_TIMEOUT);
                s_fail = 1;
                break;
            }
            if (first_half) {
                // roll the private x rows: row k <- row k+1, last row <- raw input
                for (int k = 0; k < K - 1; ++k) {
                    const uint4 nv = (k < K - 2) ? *reinterpret_cast<const uint4*>(rows + (k + 1) * row_pitch) : xin;
                    *reinterpret_cast<uint4*>(conv0 + k * cd + c0) = nv;
                }
                // the AV rows of one vector lie in one head (r0 and P are multiples of 8)
                const int hl = (rr0 + v * AV) / P;
                const float dtv = s_dt[hl], dAv = s_dA[hl], Dv = s_D[hl];
#pragma unroll
                for (int e = 0; e < AV; ++e) s_rp[v * AV + e] = make_float4(dtv * out[e], dAv, Dv * out[e], 0.f);
            } else {
                float* dstf = (v / BV) ? s_C : s_B;
#pragma unroll
                for (int e = 0; e < AV; ++e) dstf[(v % BV) * AV + e] = out[e];
            }
        }
        }
        // every CTA of the group has read the B/C conv rows once it arrives here
        cluster_arrive();
    } else {
        const XT* xrow = static_cast<const XT*>(a.xBC) + b * a.xBC_stride;
        for (int i = tid; i < TILE; i += kThreads) {
            const int hl = (rr0 + i) / P;
            const float xv = (i == tid) ? x_first : to_f32(xrow[r0 + i]);
            s_rp[i] = make_float4(s_dt[hl] * xv, s_dA[hl], s_D[hl] * xv, 0.f);
        }
        for (int j = tid; j < N; j += kThreads) {
            s_B[j] = (j == tid) ? b_first : to_f32(xrow[cB + j]);
            s_C[j] = (j == tid) ? c_first : to_f32(xrow[cC + j]);
        }
    }
    __syncthreads();
    bool ok = s_fail == 0;

    // ---- phase 2: update the tile chunk by chunk as the copies land
    const int lane = tid & 31;
    const int e0 = (lane % LPR) * EPV;   // first state column of this thread (same in every pass)
    static_assert(EPV % 2 == 0, "pairs of state columns");
    float2 B2[EPV / 2], C2[EPV / 2];
#pragma unroll
    for (int e = 0; e < EPV / 2; ++e) {
        B2[e] = make_float2(s_B[e0 + 2 * e], s_B[e0 + 2 * e + 1]);
        C2[e] = make_float2(s_C[e0 + 2 * e], s_C[e0 + 2 * e + 1]);
    }
#pragma unroll 1
    for (int c = 0; c < CHUNKS && ok; ++c) {
        if (!mbar_wait_bounded(&s_bar[c], 0, kWaitLimitNs)) {
            record_error(a.error, M2_ERR_TIMEOUT);
            ok = false;
            break;
        }
        const uint8_t* src = s_tile + c * CHUNK_BYTES;
        float acc[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = i * kThreads + tid;          // vector index within the chunk
            const int row = c * RC + v / LPR;          // row within the tile
            const float4 rp = s_rp[row];
            const float2 dtx2 = make_float2(rp.x, rp.x);
            const float2 dA2 = make_float2(rp.y, rp.y);
            float st[EPV];
            unpack16<ST>(*reinterpret_cast<const uint4*>(src + static_cast<uint32_t>(v) * 16u), st);
            float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < EPV / 2; ++e) {
                float2 s2 = make_float2(st[2 * e], st[2 * e + 1]);
                s2 = __ffma2_rn(s2, dA2, __fmul2_rn(dtx2, B2[e]));  // S*dA + (dt*x)*B
                a2 = __ffma2_rn(s2, C2[e], a2);                      // partial sum of S'*C
                st[2 * e] = s2.x;
                st[2 * e + 1] = s2.y;
            }
            st_stream(tile + static_cast<int64_t>(row) * N + e0, pack16<ST>(st));
            acc[i] = a2.x + a2.y;
        }
        int which;
        const float sum = reduce_rows<LPR, VPT>(acc, lane, which);
        if ((lane % (LPR / VPT)) == 0) {
            const int row = c * RC + which * RPP + tid / LPR;
            s_y[row] = sum + s_rp[row].z;
        }
    }
    if (!ok) {
        // let this CTA's own copies land (bounded) before its shared memory is released
        for (int c = 0; c <= CHUNKS; ++c) mbar_wait_bounded(&s_bar[c], 0, kWaitLimitNs);
    }
    __syncthreads();

    // ---- y (gated), contiguous over the tile's rows
    if constexpr (!NORM) {
        if (ok) {
            for (int i = tid; i < TILE; i += kThreads) {
                float yv = s_y[i];
                if (zrow) yv *= silu_f32(i == tid ? z_first : to_f32(zrow[r0 + i]));
                yrow[r0 + i] = from_f32<AT>(yv);
            }
        }
    } else {
        // gated RMSNorm: v = y silu(z) over the group's hpg*P channels (this
        // cluster), out = v / sqrt(mean(v^2) + eps) * w
        float ss = 0.f;
        for (int i = tid; i < TILE; i += kThreads) {
            float yv = s_y[i];
            if (zrow) yv *= silu_f32(i == tid ? z_first : to_f32(zrow[r0 + i]));
            s_y[i] = yv;
            ss = fmaf(yv, yv, ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if ((tid & 31) == 0) s_red[tid >> 5] = ss;
        __syncthreads();
        // barrier phases (every thread, in order): the wait of the phase-1
        // arrive (after it every cluster CTA is past its conv reads), then each
        // CTA pushes its partial into every CTA's s_parts[own rank] and the
        // release/acquire phase makes them visible. Nothing reads another CTA's
        // shared memory afterwards, so a CTA may exit as soon as it is done.
        cluster_wait();
        const uint32_t cs = cluster_size();
        if (tid < static_cast<int>(cs)) {
            float part = 0.f;
            for (int w = 0; w < kWarps; ++w) part += s_red[w];
            st_cluster_f32(&s_parts[cluster_rank()], static_cast<uint32_t>(tid), part);
        }
        cluster_arrive_release();
        cluster_wait();
        if (tid == 0) {
            float total = 0.f;
            for (uint32_t q = 0; q < cs; ++q) total += s_parts[q];
            s_rstd = rsqrtf(total / static_cast<float>(hpg * P) + a.norm_eps);
        }
        __syncthreads();
        if (ok) {
            const AT* nw = static_cast<const AT*>(a.norm_w);
            const float rstd = s_rstd;
            for (int i = tid; i < TILE; i += kThreads)
                yrow[r0 + i] = from_f32<AT>(s_y[i] * rstd * (i == tid ? nw_first : to_f32(nw[r0 + i])));
        }
    }

    if constexpr (FUSED) {
        // ---- phase 3: cluster rank 0 rolls the shared B/C conv rows (from the
        // staged copy of the old rows and the raw inputs). Only rank 0 writes
        // after the barrier, so only rank 0 waits; the other CTAs have arrived
        // and may exit (exited threads never hold up a cluster wait).
        if (!NORM && cluster_rank() == 0) cluster_wait();  // NORM: that phase completed above
        if (ok && cluster_rank() == 0) {
            const AT* xrow = static_cast<const AT*>(a.xBC) + b * a.xBC_stride;
            for (int v = tid; v < 2 * BV; v += kThreads) {
                const int seg = v / BV;
                const int j0 = (v % BV) * AV;
                const int64_t c0 = (seg ? cC : cB) + j0;
                const AT* rows = s_cbc + seg * (K - 1) * N + j0;
                for (int k = 0; k < K - 1; ++k) {
                    // the newest row is this step's raw input: staged by the K = 4 conv
                    const uint4 nv =
                        (k < K - 2) ? *reinterpret_cast<const uint4*>(rows + (k + 1) * N)
                        : (K == 4)  ? *reinterpret_cast<const uint4*>(&s_rawbc[(seg * N + j0) * sizeof(AT) / 4])
                                    : *reinterpret_cast<const uint4*>(xrow + c0);
                    *reinterpret_cast<uint4*>(conv0 + k * cd + c0) = nv;
                }
            }
        }
    }
}

template <typename ST, typename AT, typename XT, int N, int CHUNKS, int VPT, bool FUSED, bool NORM>
cudaError_t launch_one(const StateUpdateArgs& a, const DecodePlan& plan, cudaStream_t stream) {
    auto kern = state_update_kernel<ST, AT, XT, N, CHUNKS, VPT, FUSED, NORM>;
    constexpr int LPR = N / Vec16<ST>::n;
    constexpr int TILE = CHUNKS * (kThreads / LPR) * VPT;
    size_t smem = static_cast<size_t>(TILE) * N * sizeof(ST);
    if (FUSED) smem += static_cast<size_t>(a.K - 1) * (TILE + 2 * N) * sizeof(AT);
    // function attributes once per instantiation and device, sized for the
    // widest conv (K = 8), so the launch path makes no extra driver calls
    static AttrOnce attrs;
    const cudaError_t attr_err = attrs.ensure([&] {
        size_t smem_max = static_cast<size_t>(TILE) * N * sizeof(ST);
        if (FUSED) smem_max += static_cast<size_t>(7) * (TILE + 2 * N) * sizeof(AT);
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem_max));
        if (e == cudaSuccess && FUSED)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        return e;
    });
    if (attr_err != cudaSuccess) return attr_err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.ctas_per_seq, a.batch, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = FUSED ? plan.cluster : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic dependent launch: the grid may be scheduled while the
    // previous kernel on the stream finishes (the kernel waits for it with
    // griddepcontrol.wait before any global read)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    // fused: the slot's conv rows by three 2-D TMA boxes where the cache allows
    // it (16-byte row pitch, row coordinates in 32 bits) and each box lands on
    // a 128-byte boundary of shared memory, as a tensor copy requires (the B
    // rows follow K-1 x rows of TILE channels, the C rows K-1 B rows);
    // otherwise row by row
    CUtensorMap map_cx{}, map_cbc{};
    int use_tma = 0;
    if constexpr (FUSED) {
        const TensorMapEncodeFn enc = tensor_map_encoder();
        const int64_t as = sizeof(AT);
        const int64_t rows = a.num_slots * (a.K - 1);
        const int64_t off_b = static_cast<int64_t>(TILE) * N * sizeof(ST) + (a.K - 1) * TILE * as;
        const int64_t off_c = off_b + (a.K - 1) * N * as;
        if (enc && (a.conv_dim * as) % 16 == 0 && rows <= INT32_MAX && off_b % 128 == 0 && off_c % 128 == 0) {
            const CUtensorMapDataType dt =
                sizeof(AT) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
            const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.conv_dim), static_cast<cuuint64_t>(rows)};
            const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.conv_dim * as)};
            const cuuint32_t estr[2] = {1, 1};
            const cuuint32_t box_x[2] = {static_cast<cuuint32_t>(TILE), static_cast<cuuint32_t>(a.K - 1)};
            const cuuint32_t box_bc[2] = {static_cast<cuuint32_t>(N), static_cast<cuuint32_t>(a.K - 1)};
            use_tma = enc(&map_cx, dt, 2, a.conv, dims, strides, box_x, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS &&
                      enc(&map_cbc, dt, 2, a.conv, dims, strides, box_bc, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        }
    }
    return cudaLaunchKernelEx(&cfg, kern, map_cx, map_cbc, a, use_tma);
}

template <typename ST, typename AT, typename XT, int N, bool FUSED, bool NORM>
cudaError_t by_loads_norm(const StateUpdateArgs& a, const DecodePlan& p, cudaStream_t s) {
    // loads = 16-byte vectors per thread per tile = CHUNKS * VPT
    switch (p.loads) {
        case 4 * M2_DECODE_MAIN_CHUNKS:
            return launch_one<ST, AT, XT, N, M2_DECODE_MAIN_CHUNKS, 4, FUSED, NORM>(a, p, s);
        case 4: return launch_one<ST, AT, XT, N, 1, 4, FUSED, NORM>(a, p, s);
        case 1: return launch_one<ST, AT, XT, N, 1, 1, FUSED, NORM>(a, p, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename ST, typename AT, typename XT, int N, bool FUSED>
cudaError_t by_loads(const StateUpdateArgs& a, const DecodePlan& p, cudaStream_t s) {
    if constexpr (FUSED) {
        if (a.norm_w) return by_loads_norm<ST, AT, XT, N, true, true>(a, p, s);
    }
    return by_loads_norm<ST, AT, XT, N, FUSED, false>(a, p, s);
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
    if (a.x_dtype == M2_BF16) return by_n<ST, AT, bf16_t, false>(a, p, s);
    if (a.x_dtype == M2_F16) return by_n<ST, AT, f16_t, false>(a, p, s);
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
    static const int kLoads[3] = {4 * M2_DECODE_MAIN_CHUNKS, 4, 1};
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
