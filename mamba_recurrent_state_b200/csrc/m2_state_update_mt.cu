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
// 64/P heads) of one sequence, four CTAs per SM. The CTA stages its state tile (16 KB for bf16,
// N = 128) with a bulk copy, and the conv rows of its x channels and of the
// group's B/C channels with their T raw input rows as 64-channel segments, two
// 2-D TMA boxes per segment (the K-1 cached rows, the T raw rows: 10 copies
// instead of 21 row copies for N = 128, 153.4 us instead of 155.7 us for 64
// Nemotron-H sequences x 4 drafts), computes the conv tap of every
// (token, 16-byte channel vector) at once (the group's B/C conv is computed by
// every CTA of the group), and then runs the T state updates on the tile in
// shared memory (rounded to the storage dtype after every token, exactly as T
// separate decode steps store it): each thread keeps the same state vectors for
// all tokens, so the token loop needs no barrier. y and every token's conv
// rows are stored at the end. The first CTA of each group writes the group's
// B/C conv rows; no CTA writes the input slot, so nothing races with the reads.
#include <cuda_runtime.h>

#include <climits>

#include "m2_device.cuh"
#include "m2_internal.cuh"

namespace m2 {
namespace {

// Resident CTAs per SM the register budget is sized for (compile-time knob):
// four (64 registers) where N <= 128 -- the phases between the block barriers
// leave a CTA idle much of its time, and a fourth CTA per SM covers it
// (Nemotron-H, 64 x 4 drafts: 155.7 us against 169.2 us at three) -- three for
// N = 256, whose wider rows would spill at 64 registers.
#ifndef M2_MT_MIN_BLOCKS
#define M2_MT_MIN_BLOCKS 4
#endif

constexpr int kMtThreads = 256;
constexpr int kMtRows = 64;   // state rows per CTA
constexpr int kMtSeg = 64;    // channels per staged window segment
constexpr int kMtMaxHeads = kMtRows / 8 + 1;
constexpr uint64_t kMtWaitNs = 1000000000ull;

// map_x: xBC as (channel, token row), boxes of 64 channels x T rows;
// map_conv: the conv cache as (channel, slot * (K-1) + k), boxes of 64 channels
// x K-1 rows; use_tma = 0: both unused, every row segment is a bulk copy.
template <typename ST, typename AT, int N>
__global__ void __launch_bounds__(kMtThreads, N <= 128 ? M2_MT_MIN_BLOCKS : 3)
    mt_decode_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_conv,
                     const MtArgs a, const int use_tma) {
    constexpr int EPV = Vec16<ST>::n;        // state elements per 16-byte vector
    constexpr int LPR = N / EPV;             // lanes per state row
    static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "row must fit a warp");
    constexpr int VPT = kMtRows * LPR / kMtThreads;  // vectors per thread per token
    static_assert(VPT >= 1 && kMtRows * LPR == VPT * kMtThreads, "whole passes");
    constexpr uint32_t TILE_BYTES = kMtRows * N * sizeof(ST);
    constexpr int AV = Vec16<AT>::n;         // activation elements per 16-byte vector
    constexpr int XV = kMtRows / AV;         // x-channel vectors of the tile
    constexpr int BV = N / AV;               // vectors of one B (or C) segment
    constexpr int NVEC = XV + 2 * BV;        // conv vectors per token
    constexpr int SEGV = kMtSeg / AV;        // vectors per 64-channel window segment
    constexpr int NSEG = 1 + 2 * N / kMtSeg; // window segments: x, then B, then C
    static_assert(kMtRows == kMtSeg && N % kMtSeg == 0, "64-channel segments");

    const int T = a.T;
    const int K = a.K;
    const int W = K - 1 + T;                 // window rows: K-1 cached, then T raw inputs
    // dynamic shared memory: [state tile | raw window, NSEG segments of 64
    //   channels (the tile's x, then the group's B, then C) x W rows |
    //   per (token, row) dt*x, dA, D*x | post-conv B, C of every token | y (fp32)]
    extern __shared__ __align__(128) uint8_t s_dyn[];
    uint8_t* s_state = s_dyn;                                        // [64][N] ST
    AT* s_win = reinterpret_cast<AT*>(s_dyn + TILE_BYTES);           // [NSEG][W][64]
    float4* s_rp = reinterpret_cast<float4*>(s_win + static_cast<size_t>(NSEG) * W * kMtSeg);  // [T][64]
    float* s_B = reinterpret_cast<float*>(s_rp + T * kMtRows);       // [T][N]
    float* s_C = s_B + T * N;                                        // [T][N]
    float* s_y = s_C + T * N;                                        // [T][64]
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ float s_dt[kMaxDraftTokens][kMtMaxHeads];
    __shared__ float s_dA[kMaxDraftTokens][kMtMaxHeads];
    __shared__ float s_D[kMtMaxHeads];
    __shared__ int32_t s_tok[kMaxDraftTokens];  // destination slot of every token
    __shared__ int s_fail;

    const int tid = threadIdx.x;
    const int b = blockIdx.y;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kMtRows;   // first row h*P + p
    const int P = a.P;
    const int64_t HP = static_cast<int64_t>(a.H) * P;
    const int hpg = a.H / a.G;
    const int h_first = static_cast<int>(r0 / P);
    // r0's row within its head: head offsets below use 32-bit arithmetic
    const int rr0 = static_cast<int>(r0 - static_cast<int64_t>(h_first) * P);
    const int g = h_first / hpg;
    const int n_heads = (rr0 + kMtRows - 1) / P + 1;  // heads the tile's rows touch
    const int64_t cd = a.conv_dim;
    const int64_t cB = HP + static_cast<int64_t>(g) * N;
    const int64_t cC = HP + static_cast<int64_t>(a.G) * N + static_cast<int64_t>(g) * N;
    const bool bc_writer = (r0 % (static_cast<int64_t>(hpg) * P)) == 0;  // first CTA of the group
    const AT* xbase = static_cast<const AT*>(a.xBC) + static_cast<int64_t>(b) * T * a.xBC_stride;
    AT* ybase = static_cast<AT*>(a.y) + static_cast<int64_t>(b) * T * a.y_stride;
    // channel of conv vector u (0 .. NVEC-1) and where its window column sits
    auto vec_channel = [&](int u) -> int64_t {
        return u < XV ? r0 + u * AV : (u - XV < BV ? cB + (u - XV) * AV : cC + (u - XV - BV) * AV);
    };
    // first channel of window segment sg
    auto seg_channel = [&](int sg) -> int64_t {
        return sg == 0 ? r0 : (sg <= N / kMtSeg ? cB + (sg - 1) * kMtSeg : cC + (sg - 1 - N / kMtSeg) * kMtSeg);
    };
    auto vec_window = [&](int u, int& pitch) -> const AT* {
        pitch = kMtSeg;
        return s_win + static_cast<size_t>(u / SEGV) * W * kMtSeg + (u % SEGV) * AV;
    };

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
        // the state tile, the K-1 cached rows and the T raw input rows of the
        // window (x channels of the tile, the group's B and C), all row segments
        mbar_arrive_expect_tx(&s_bar, TILE_BYTES + static_cast<uint32_t>(NSEG * W * kMtSeg) * sizeof(AT));
        bulk_g2s(s_state, tile, TILE_BYTES, &s_bar);
        for (int sg = 0; sg < NSEG; ++sg) {
            AT* dst = s_win + static_cast<size_t>(sg) * W * kMtSeg;
            const int64_t c = seg_channel(sg);
            if (use_tma) {
                // two 2-D boxes per segment: the K-1 cached rows, the T raw rows
                tma_load_tile_2d(dst, &map_conv, static_cast<int>(c), slot * (K - 1), &s_bar);
                tma_load_tile_2d(dst + (K - 1) * kMtSeg, &map_x, static_cast<int>(c), b * T, &s_bar);
            } else {
                for (int k = 0; k < K - 1; ++k)
                    bulk_g2s(dst + k * kMtSeg, conv_in + k * cd + c, kMtSeg * sizeof(AT), &s_bar);
                for (int t = 0; t < T; ++t)
                    bulk_g2s(dst + (K - 1 + t) * kMtSeg, xbase + static_cast<int64_t>(t) * a.xBC_stride + c,
                             kMtSeg * sizeof(AT), &s_bar);
            }
        }
    }
    __syncthreads();  // the barrier is initialised before any thread waits on it
    // the head scalars of every token, while the copies land
    if (tid < T) s_tok[tid] = a.token_slots[static_cast<int64_t>(b) * T + tid];
    for (int i = tid; i < T * n_heads; i += kMtThreads) {
        const int t = i / n_heads;
        const int hl = i % n_heads;
        const int h = h_first + hl;
        const float dtr = to_f32(static_cast<const AT*>(a.dt)[(static_cast<int64_t>(b) * T + t) * a.dt_stride + h]);
        const float dt = softplus_f32(dtr + a.dt_bias[h]);
        s_dt[t][hl] = dt;
        s_dA[t][hl] = expf(dt * -expf(a.A_log[h]));
        if (t == 0) s_D[hl] = a.D[h];
    }
    const bool wait_ok = mbar_wait_bounded(&s_bar, 0, kMtWaitNs);
    if (!wait_ok) s_fail = 1;
    __syncthreads();
    if (s_fail) {
        if (tid == 0) record_error(a.error, M2_ERR_TIMEOUT);
        mbar_wait_bounded(&s_bar, 0, kMtWaitNs);  // this CTA's copies land before it leaves
        return;
    }

    // ---- the conv tap of every (token, channel vector) at once: token t's
    // window is rows t .. t+K-1
    for (int i = tid; i < T * NVEC; i += kMtThreads) {
        const int t = i / NVEC;
        const int u = i % NVEC;
        int pitch;
        const AT* win = vec_window(u, pitch);
        const int64_t c = vec_channel(u);
        const AT* wp = static_cast<const AT*>(a.conv_w) + c * K;
        float out[AV];
        if (a.conv_b) {
            unpack16<AT>(__ldg(reinterpret_cast<const uint4*>(static_cast<const AT*>(a.conv_b) + c)), out);
        } else {
#pragma unroll
            for (int e = 0; e < AV; ++e) out[e] = 0.f;
        }
        if (K == 4) {
            // the AV x 4 weight block is four 16-byte vectors, (e, k) at e*4 + k
            float wf[AV * 4];
#pragma unroll
            for (int q = 0; q < 4; ++q) unpack16<AT>(__ldg(reinterpret_cast<const uint4*>(wp) + q), wf + q * AV);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float rv[AV];
                unpack16<AT>(*reinterpret_cast<const uint4*>(win + (t + k) * pitch), rv);
#pragma unroll
                for (int e = 0; e < AV; ++e) out[e] = fmaf(wf[e * 4 + k], rv[e], out[e]);
            }
        } else {
            for (int k = 0; k < K; ++k) {
                float rv[AV];
                unpack16<AT>(*reinterpret_cast<const uint4*>(win + (t + k) * pitch), rv);
#pragma unroll
                for (int e = 0; e < AV; ++e) out[e] = fmaf(to_f32(wp[e * K + k]), rv[e], out[e]);
            }
        }
        if (a.activation) {
#pragma unroll
            for (int e = 0; e < AV; ++e) out[e] = silu_f32(out[e]);
        }
        if (u < XV) {
            // x: the row parameters of token t; the AV rows of one vector lie in
            // one head (r0 and P are multiples of 8)
            const int hl = (rr0 + u * AV) / P;
            const float dtv = s_dt[t][hl], dAv = s_dA[t][hl], Dv = s_D[hl];
#pragma unroll
            for (int e = 0; e < AV; ++e)
                s_rp[t * kMtRows + u * AV + e] = make_float4(dtv * out[e], dAv, Dv * out[e], 0.f);
        } else {
            float* dst = u - XV < BV ? s_B + t * N + (u - XV) * AV : s_C + t * N + (u - XV - BV) * AV;
#pragma unroll
            for (int e = 0; e < AV; e += 4)
                *reinterpret_cast<float4*>(dst + e) = make_float4(out[e], out[e + 1], out[e + 2], out[e + 3]);
        }
    }
    __syncthreads();

    // ---- the T tokens: every thread keeps the same VPT state vectors in
    // registers for all of them (carrying the stored, rounded value), so the
    // token loop needs no barrier
    constexpr int RPP = kMtThreads / LPR;  // rows per pass
    const int lane = tid & 31;
    const int e0 = (lane % LPR) * EPV;
    const int64_t HPN = HP * N;
    float st[VPT][EPV];
#pragma unroll
    for (int i = 0; i < VPT; ++i)
        unpack16<ST>(*reinterpret_cast<const uint4*>(s_state + static_cast<uint32_t>(i * kMtThreads + tid) * 16u), st[i]);
    for (int t = 0; t < T; ++t) {
        const int32_t dest = s_tok[t];
        const bool store = dest >= 0 && dest < a.num_slots;
        if (dest >= a.num_slots && tid == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        ST* dtile = store ? static_cast<ST*>(a.ssm) + static_cast<int64_t>(dest) * HPN + r0 * N : nullptr;
        float2 B2[EPV / 2], C2[EPV / 2];
#pragma unroll
        for (int e = 0; e < EPV; e += 4) {
            const float4 b4 = *reinterpret_cast<const float4*>(s_B + t * N + e0 + e);
            const float4 c4 = *reinterpret_cast<const float4*>(s_C + t * N + e0 + e);
            B2[e / 2] = make_float2(b4.x, b4.y);
            B2[e / 2 + 1] = make_float2(b4.z, b4.w);
            C2[e / 2] = make_float2(c4.x, c4.y);
            C2[e / 2 + 1] = make_float2(c4.z, c4.w);
        }
        float acc[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int row = i * RPP + tid / LPR;
            const float4 rp = s_rp[t * kMtRows + row];
            const float dtx = rp.x;
            const float dA = rp.y;
            // packed f32x2: per element the rounded product dt*x*B, then one FMA
            // (the arithmetic of the single-step kernel, element for element)
            const float2 dtx2 = make_float2(dtx, dtx);
            const float2 dA2 = make_float2(dA, dA);
            float2 a2v = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < EPV / 2; ++e) {
                float2 s2 = make_float2(st[i][2 * e], st[i][2 * e + 1]);
                s2 = __ffma2_rn(s2, dA2, __fmul2_rn(dtx2, B2[e]));
                a2v = __ffma2_rn(s2, C2[e], a2v);
                st[i][2 * e] = s2.x;
                st[i][2 * e + 1] = s2.y;
            }
            const float a2 = a2v.x + a2v.y;
            const uint4 packed = pack16<ST>(st[i]);  // the stored state, rounded once per token
            unpack16<ST>(packed, st[i]);              // ... and carried as stored
            if (store) st_stream(dtile + static_cast<int64_t>(row) * N + e0, packed);
            acc[i] = a2;
        }
        if constexpr (VPT == 4 && LPR >= 4) {
            int which;
            const float sum = reduce_rows<LPR, 4>(acc, lane, which);
            if ((lane % (LPR / 4)) == 0) {
                const int row = which * RPP + tid / LPR;
                s_y[t * kMtRows + row] = sum + s_rp[t * kMtRows + row].z;
            }
        } else {
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float v = acc[i];
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if ((lane % LPR) == 0) {
                    const int row = i * RPP + tid / LPR;
                    s_y[t * kMtRows + row] = v + s_rp[t * kMtRows + row].z;
                }
            }
        }
    }
    __syncthreads();

    // ---- gated y of every token; every token's conv window into its destination
    for (int i = tid; i < T * kMtRows; i += kMtThreads) {
        const int t = i / kMtRows;
        const int row = i % kMtRows;
        float yv = s_y[i];
        if (a.z) {
            const AT* zr = static_cast<const AT*>(a.z) + (static_cast<int64_t>(b) * T + t) * a.z_stride;
            yv *= silu_f32(to_f32(zr[r0 + row]));
        }
        ybase[static_cast<int64_t>(t) * a.y_stride + r0 + row] = from_f32<AT>(yv);
    }
    const int nwrite = bc_writer ? NVEC : XV;  // the group's first CTA also writes B/C
    for (int i = tid; i < T * nwrite * (K - 1); i += kMtThreads) {
        const int k = i % (K - 1);
        const int u = (i / (K - 1)) % nwrite;
        const int t = i / ((K - 1) * nwrite);
        const int32_t dest = s_tok[t];
        if (dest < 0 || dest >= a.num_slots) continue;
        int pitch;
        const AT* win = vec_window(u, pitch);
        // new row k of the destination = window row t+1+k (raw inputs, exact copies)
        AT* conv_out = static_cast<AT*>(a.conv) + static_cast<int64_t>(dest) * (K - 1) * cd;
        *reinterpret_cast<uint4*>(conv_out + k * cd + vec_channel(u)) =
            *reinterpret_cast<const uint4*>(win + (t + 1 + k) * pitch);
    }
}

// One kernel instantiation with its own once-per-device attribute setup.
template <typename ST, typename AT, int N>
cudaError_t mt_launch(const CUtensorMap& map_x, const CUtensorMap& map_conv, int use_tma, const MtArgs& a,
                      size_t smem, size_t smem_max, dim3 grid, cudaStream_t s) {
    static AttrOnce attrs;
    const cudaError_t e = attrs.ensure([&] {
        return cudaFuncSetAttribute(mt_decode_kernel<ST, AT, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem_max));
    });
    if (e != cudaSuccess) return e;
    mt_decode_kernel<ST, AT, N><<<grid, kMtThreads, smem, s>>>(map_x, map_conv, a, use_tma);
    return cudaGetLastError();
}

template <typename ST, typename AT>
cudaError_t mt_by_n(const MtArgs& a, cudaStream_t s) {
    // tile + raw windows + per token: row parameters (4 floats), fp32 B, C and y
    // (the largest N, K and T)
    const size_t smem_max = static_cast<size_t>(kMtRows) * 256 * sizeof(ST) +
                            static_cast<size_t>(7 + kMaxDraftTokens) * (kMtRows + 2 * 256) * sizeof(AT) +
                            static_cast<size_t>(kMaxDraftTokens) * (5 * kMtRows + 2 * 256) * sizeof(float);
    const size_t tile = static_cast<size_t>(kMtRows) * a.N * sizeof(ST);
    const size_t smem = tile + static_cast<size_t>(a.K - 1 + a.T) * (kMtRows + 2 * a.N) * sizeof(AT) +
                        static_cast<size_t>(a.T) * (5 * kMtRows + 2 * a.N) * sizeof(float);
    const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(a.H) * a.P / kMtRows), static_cast<unsigned>(a.batch));
    // the raw window by 2-D TMA boxes where both tensors allow it (16-byte row
    // pitches, row coordinates in 32 bits); otherwise segment by segment
    CUtensorMap map_x{}, map_conv{};
    int use_tma = 0;
    const TensorMapEncodeFn enc = tensor_map_encoder();
    const int64_t as = sizeof(AT);
    const int64_t x_rows = static_cast<int64_t>(a.batch) * a.T;
    const int64_t c_rows = a.num_slots * (a.K - 1);
    if (enc && (a.xBC_stride * as) % 16 == 0 && (a.conv_dim * as) % 16 == 0 && x_rows <= INT32_MAX &&
        c_rows <= INT32_MAX) {
        const CUtensorMapDataType dt = sizeof(AT) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
        const cuuint32_t estr[2] = {1, 1};
        const cuuint64_t xd[2] = {static_cast<cuuint64_t>(a.conv_dim), static_cast<cuuint64_t>(x_rows)};
        const cuuint64_t xs[1] = {static_cast<cuuint64_t>(a.xBC_stride * as)};
        const cuuint32_t xb[2] = {static_cast<cuuint32_t>(kMtSeg), static_cast<cuuint32_t>(a.T)};
        const cuuint64_t cdm[2] = {static_cast<cuuint64_t>(a.conv_dim), static_cast<cuuint64_t>(c_rows)};
        const cuuint64_t cs[1] = {static_cast<cuuint64_t>(a.conv_dim * as)};
        const cuuint32_t cb[2] = {static_cast<cuuint32_t>(kMtSeg), static_cast<cuuint32_t>(a.K - 1)};
        use_tma = enc(&map_x, dt, 2, const_cast<void*>(a.xBC), xd, xs, xb, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS &&
                  enc(&map_conv, dt, 2, a.conv, cdm, cs, cb, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    switch (a.N) {
        case 64: return mt_launch<ST, AT, 64>(map_x, map_conv, use_tma, a, smem, smem_max, grid, s);
        case 128: return mt_launch<ST, AT, 128>(map_x, map_conv, use_tma, a, smem, smem_max, grid, s);
        case 256:
            if constexpr (sizeof(ST) == 2)
                return mt_launch<ST, AT, 256>(map_x, map_conv, use_tma, a, smem, smem_max, grid, s);
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
