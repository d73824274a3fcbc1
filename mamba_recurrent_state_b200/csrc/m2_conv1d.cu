// m2_conv1d.cu -- causal_conv1d_update over seqlen >= 1 tokens per row, and the
// slot-zeroing kernel of the cache lifecycle.
//
// Operation: vllm.cpp issue #1311 "NemotronH runs the PREFILL mamba kernels at
// decode", section "The divergence": causal_conv1d_update reads and writes the
// conv cache in place at conv_state_indices; with seqlen > 1 it is the prefill
// conv (CausalConv1dFwd) that feeds the chunk scan. For channel c and token t:
//   window = (raw inputs t-K+1 .. t), older ones from the cache,
//   out[t, c] = bias[c] + sum_k w[c, k] * window[k],  SiLU if requested,
// and afterwards the cache holds the last K-1 raw inputs (exact copies).
//
// Layout: a thread owns VEC = 16 bytes of consecutive channels and TT
// consecutive tokens; the raw-input history it needs before its first token
// comes from the input itself (t >= 0) or from the cache (t < 0). Only the
// CTAs of the first token tile read the cache, and those same CTAs write the
// new cache rows afterwards, so no other CTA can observe a half-rolled cache.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <type_traits>

#include "m2_device.cuh"
#include "m2_internal.cuh"

namespace m2 {
namespace {

// Tuning knobs (compile-time): tokens per thread and the resident CTAs per SM
// the prefill path's register budget is sized for. Measured on the 8 x 2048
// Nemotron-H prefill conv: 16 tokens at 3 CTAs/SM 239 us; 8 at 4 263 us; 8 at
// 3 284 us; 4 at 4 390 us.
#ifndef M2_CONV_TT
#define M2_CONV_TT 16
#endif
#ifndef M2_CONV_MIN_BLOCKS
#define M2_CONV_MIN_BLOCKS 3
#endif

constexpr int kConvThreads = 128;
constexpr int kTT = M2_CONV_TT;  // tokens per thread

// Store VEC floats as OT at p (VEC * sizeof(OT) is 16 or 32 bytes, or 8 for
// four bf16 outputs of fp32 inputs).
template <typename OT, int VEC>
__device__ __forceinline__ void store_vec(OT* p, const float* o) {
    if constexpr (sizeof(OT) == 2 && VEC == 4) {
        float t[8] = {o[0], o[1], o[2], o[3], 0.f, 0.f, 0.f, 0.f};
        const uint4 v = pack16<OT>(t);
        *reinterpret_cast<uint2*>(p) = make_uint2(v.x, v.y);
    } else {
        constexpr int OVEC = Vec16<OT>::n;
        static_assert(VEC % OVEC == 0, "whole 16-byte output vectors");
#pragma unroll
        for (int v = 0; v < VEC; v += OVEC) *reinterpret_cast<uint4*>(p + v) = pack16<OT>(o + v);
    }
}

// Variable-length batches (cu_seqlens): sequence b is packed rows
// cu_seqlens[b] .. cu_seqlens[b+1]-1 and the CTA walks the sequence's token
// tiles blockIdx.y, blockIdx.y + gridDim.y, ..., so a sequence longer than
// the grid was planned for is still covered; tile 0 (the only one that reads
// the cache) is always its blockIdx.y == 0 CTA's first.
// The prefill path (K <= 4, 16-bit post-conv output) is held to three CTAs
// per SM (168 registers, no spills); the tile loop would otherwise take ~200.
template <typename AT, typename OT, int K>
__global__ void __launch_bounds__(kConvThreads, (sizeof(OT) == 2 && K <= 4) ? M2_CONV_MIN_BLOCKS : 1)
conv1d_kernel(const ConvArgs a) {
    constexpr int VEC = Vec16<AT>::n;
    const int b = blockIdx.z;
    const int64_t c0 = (static_cast<int64_t>(blockIdx.x) * kConvThreads + threadIdx.x) * VEC;
    if (c0 >= a.conv_dim) return;
    const int64_t row0 = a.cu_seqlens ? static_cast<int64_t>(a.cu_seqlens[b]) : static_cast<int64_t>(b) * a.seqlen;
    const int T = a.cu_seqlens ? a.cu_seqlens[b + 1] - a.cu_seqlens[b] : a.seqlen;
    if (T <= 0) return;  // an empty sequence leaves its cache slot untouched

    const int32_t slot = a.slot_idx[b];
    const AT* xb = static_cast<const AT*>(a.x) + row0 * a.x_stride;
    OT* ob = static_cast<OT*>(a.out) + row0 * a.out_stride;
    if (slot < 0) {  // padding row: zero output, cache untouched
        float zeros[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) zeros[v] = 0.f;
        for (int t0 = blockIdx.y * kTT; t0 < T; t0 += gridDim.y * kTT)
            for (int t = t0; t < min(t0 + kTT, T); ++t) store_vec<OT, VEC>(ob + t * a.out_stride + c0, zeros);
        return;
    }
    if (slot >= a.num_slots) {
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }
    AT* cache = static_cast<AT*>(a.conv) + static_cast<int64_t>(slot) * (K - 1) * a.conv_dim;

    // weights and bias of the VEC channels, as float
    float w[VEC][K];
    float bias[VEC];
    {
        const AT* wp = static_cast<const AT*>(a.w) + c0 * K;
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
#pragma unroll
            for (int k = 0; k < K; ++k) w[v][k] = to_f32(wp[v * K + k]);
            bias[v] = a.b ? to_f32(static_cast<const AT*>(a.b)[c0 + v]) : 0.f;
        }
    }

    float out_max = 0.f;  // largest post-conv magnitude (checked for fp16 outputs)
#pragma unroll 1
    for (int t0 = blockIdx.y * kTT; t0 < T; t0 += gridDim.y * kTT) {
    const int t_end = min(t0 + kTT, T);
    // history: raw vectors of tokens t0-K+1 .. t0-1 (oldest first)
    uint4 hist_raw[K - 1];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int t = t0 - (K - 1) + j;
        hist_raw[j] = t >= 0 ? *reinterpret_cast<const uint4*>(xb + t * a.x_stride + c0)
                             : *reinterpret_cast<const uint4*>(cache + (K - 1 + t) * a.conv_dim + c0);
    }
    float hist[K - 1][VEC];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) unpack16<AT>(hist_raw[j], hist[j]);

    // all of the tile's raw inputs are loaded before any output is stored, so
    // the loads are in flight together (the output may alias nothing, but the
    // compiler cannot know that)
    uint4 raw[kTT];
#pragma unroll
    for (int i = 0; i < kTT; ++i) {
        const int t = t0 + i;
        raw[i] = t < t_end ? *reinterpret_cast<const uint4*>(xb + t * a.x_stride + c0) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kTT; ++i) {
        const int t = t0 + i;
        if (t < t_end) {
            float cur[VEC];
            unpack16<AT>(raw[i], cur);
            float o[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                float acc = bias[v];
#pragma unroll
                for (int k = 0; k < K - 1; ++k) acc = fmaf(w[v][k], hist[k][v], acc);
                acc = fmaf(w[v][K - 1], cur[v], acc);
                o[v] = a.activation ? silu_f32(acc) : acc;
            }
            if constexpr (std::is_same<OT, f16_t>::value) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) out_max = fmaxf(out_max, fabsf(o[v]));
            }
            store_vec<OT, VEC>(ob + t * a.out_stride + c0, o);
#pragma unroll
            for (int k = 0; k < K - 2; ++k) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) hist[k][v] = hist[k + 1][v];
            }
#pragma unroll
            for (int v = 0; v < VEC; ++v) hist[K - 2][v] = cur[v];
        }
    }
    }

    if (out_max >= 65520.f) record_error(a.error, M2_ERR_RANGE);  // beyond fp16 (rounds to inf)
    if (blockIdx.y == 0) {
        // new cache row k holds the raw input of token T-(K-1)+k: from the input
        // when that token exists, else old cache row k + T (only when
        // T < K-1; rows are written in increasing k and row k + T > k is read
        // before row k + T is written, so every read sees an old row)
#pragma unroll
        for (int k = 0; k < K - 1; ++k) {
            const int t = T - (K - 1) + k;
            const uint4 v = t >= 0 ? *reinterpret_cast<const uint4*>(xb + t * a.x_stride + c0)
                                   : *reinterpret_cast<const uint4*>(cache + (k + T) * a.conv_dim + c0);
            *reinterpret_cast<uint4*>(cache + k * a.conv_dim + c0) = v;
        }
    }
}

// ---- prefill conv with the input tile staged in shared memory ---------------
//
// For long sequences of 16-bit activations: a CTA of 128 threads owns 256
// channels x 32 tokens. The 32 + K-1 input rows of a tile (512 bytes each)
// arrive in shared memory as one 2-D TMA box of x; the first tile of a
// sequence, whose rows before the sequence start come from the slot's conv
// cache, is staged row by row with bulk copies by warp 0 (as is every tile
// when the box does not apply). One box instead of 35 row copies per tile:
// 132-134 us instead of 151.6 us for 8 x 2048 Nemotron-H tokens, whose
// 35 copies of 512 bytes per tile kept the copy engine, not DRAM, busy (the
// copies alone, with no arithmetic, took 84 us). Every thread then computes 8
// tokens of one 16-byte channel vector from shared memory, two channels at a
// time with packed f32x2 FMAs (per channel the same FMA chain as the other
// conv kernels, so the outputs agree bit for bit). A CTA walks several tiles of
// its sequence with two buffers: the next tile's rows land while the current
// one is computed. There is no block barrier between tiles: each warp arrives
// on the buffer's "empty" mbarrier when it is done with it, and warp 0 refills
// the buffer once all four have arrived. Small tiles keep five CTAs on an SM
// (96 registers), which the latency of the conv's FMA and SiLU chains needs.
constexpr int kTileThreads = 128;
constexpr int kTileCh = 256;   // channels per CTA
// Tuning knobs (compile-time): tokens per tile, tile buffers in flight per
// CTA, resident CTAs per SM the register budget is sized for, tiles a CTA walks
// at most. Measured on the 8 x 2048 Nemotron-H prefill with one box per tile
// and the tanh-form SiLU (the warps wait mostly for the next tile): 32 tokens,
// 3 buffers, 4 CTAs per SM, 8 tiles 118.8 us; 32, 2, 5: 120.9 us; 64, 2, 3:
// 120.8 us; 16, 4, 5: 125 us; 16 tiles 129 us; 16, 3, 6: 199 us (spills).
// With the two-SFU SiLU, bound by its arithmetic, 32, 2, 5 was best
// (132-134 us; 32, 3, 4: 144 us).
#ifndef M2_CONV_TILE_TOK
#define M2_CONV_TILE_TOK 32
#endif
#ifndef M2_CONV_NBUF
#define M2_CONV_NBUF 3
#endif
#ifndef M2_CONV_MINB
#define M2_CONV_MINB 4
#endif
#ifndef M2_CONV_MAXTILES
#define M2_CONV_MAXTILES 8
#endif
constexpr int kTileTok = M2_CONV_TILE_TOK;   // tokens per tile
constexpr int kTileBufs = M2_CONV_NBUF;      // tile buffers in flight per CTA
constexpr int kTileMinBlocks = M2_CONV_MINB;
constexpr int kMaxTilesPerCta = M2_CONV_MAXTILES;  // token tiles a CTA walks (at most)
constexpr uint64_t kTileWaitNs = 1000000000ull;

// (wider convs keep more taps per channel in registers: three CTAs per SM)
template <typename OT, int K>
__global__ void __launch_bounds__(kTileThreads, K <= 4 ? kTileMinBlocks : 3)
    conv1d_tile_kernel(const __grid_constant__ CUtensorMap tmap_x, const ConvArgs a, const int use_tma) {
    using AT = bf16_t;
    constexpr int VEC = Vec16<AT>::n;                    // 8 channels per vector
    constexpr int NV = kTileCh / VEC;                    // 32 vectors per row
    constexpr int TPT = kTileTok / (kTileThreads / NV);  // 8 tokens per thread
    constexpr int ROWS = kTileTok + K - 1;
    // two tile buffers (dynamic shared memory): the next tile's rows land while
    // this one is computed
    extern __shared__ __align__(128) uint8_t s_conv_dyn[];
    AT (*s_buf)[ROWS][kTileCh] = reinterpret_cast<AT (*)[ROWS][kTileCh]>(s_conv_dyn);
    __shared__ __align__(8) uint64_t s_bar[kTileBufs];
    __shared__ __align__(8) uint64_t s_empty[kTileBufs];  // arrivals of the 4 warps done with buffer q

    const int tid = threadIdx.x;
    const int b = blockIdx.z;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTileCh;
    const int nch = static_cast<int>(a.conv_dim - c0 < kTileCh ? a.conv_dim - c0 : kTileCh);
    const int64_t row0 = a.cu_seqlens ? static_cast<int64_t>(a.cu_seqlens[b]) : static_cast<int64_t>(b) * a.seqlen;
    const int T = a.cu_seqlens ? a.cu_seqlens[b + 1] - a.cu_seqlens[b] : a.seqlen;
    if (T <= 0) return;  // an empty sequence leaves its cache slot untouched
    const int v = tid % NV;             // this thread's channel vector
    const int tg = tid / NV;            // its token group within the tile
    const bool vec_ok = v * VEC < nch;
    const int32_t slot = a.slot_idx[b];
    const AT* xb = static_cast<const AT*>(a.x) + row0 * a.x_stride;
    OT* ob = static_cast<OT*>(a.out) + row0 * a.out_stride;
    if (slot < 0) {  // padding row: zero output, cache untouched
        float zeros[VEC] = {};
        for (int t0 = blockIdx.y * kTileTok; t0 < T; t0 += gridDim.y * kTileTok)
            for (int i = 0; i < TPT; ++i) {
                const int t = t0 + tg * TPT + i;
                if (t < T && vec_ok) store_vec<OT, VEC>(ob + t * a.out_stride + c0 + v * VEC, zeros);
            }
        return;
    }
    if (slot >= a.num_slots) {
        if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }
    AT* cache = static_cast<AT*>(a.conv) + static_cast<int64_t>(slot) * (K - 1) * a.conv_dim;

    // weights and bias of the thread's 8 channels
    float w[VEC][K];
    float bias[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        const int64_t c = c0 + v * VEC + e;
        const bool ok = vec_ok;
#pragma unroll
        for (int k = 0; k < K; ++k) w[e][k] = ok ? to_f32(static_cast<const AT*>(a.w)[c * K + k]) : 0.f;
        bias[e] = (ok && a.b) ? to_f32(static_cast<const AT*>(a.b)[c]) : 0.f;
    }
    if (tid == 0) {
#pragma unroll
        for (int q = 0; q < kTileBufs; ++q) {
            mbar_init(&s_bar[q], 1);
            mbar_init(&s_empty[q], kTileThreads / 32);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // this CTA's tiles: t0 = (blockIdx.y + j * gridDim.y) * 64, j = 0, 1, ...
    const int stride = gridDim.y * kTileTok;
    // stage rows t0-K+1 .. t0+63 of a tile into buffer q (only rows inside the
    // sequence or, before its start, in the conv cache; rows past the end are
    // never read); warp 0: lane 0 sets the byte count, then the lanes issue rows
    auto issue = [&](int t0, int q) {
        if (use_tma && t0 >= K - 1) {
            // every row of the tile lies inside the packed rows of x: one 2-D
            // TMA box of ROWS rows x 256 channels (channels past conv_dim and
            // rows past the last packed row arrive as zeros and are not read)
            if (tid == 0) {
                mbar_arrive_expect_tx(&s_bar[q], static_cast<uint32_t>(ROWS) * kTileCh * sizeof(AT));
                tma_load_tile_2d(&s_buf[q][0][0], &tmap_x, static_cast<int>(c0),
                                 static_cast<int>(row0 + t0 - (K - 1)), &s_bar[q]);
            }
            return;
        }
        if (tid < 32) {
            const int r_end = min(ROWS, T - t0 + K - 1);
            if (tid == 0) mbar_arrive_expect_tx(&s_bar[q], static_cast<uint32_t>(r_end) * nch * sizeof(AT));
            __syncwarp();
            for (int r = tid; r < r_end; r += 32) {
                const int t = t0 - (K - 1) + r;
                const AT* src = t >= 0 ? xb + t * a.x_stride + c0 : cache + (K - 1 + t) * a.conv_dim + c0;
                bulk_g2s(&s_buf[q][r][0], src, static_cast<uint32_t>(nch) * sizeof(AT), &s_bar[q]);
            }
        }
    };
    const int first = blockIdx.y * kTileTok;
#pragma unroll
    for (int q = 0; q < kTileBufs; ++q)
        if (first + q * stride < T) issue(first + q * stride, q);
    // tiles j+1 .. j+kTileBufs-1 may be in flight into the other buffers: a
    // warp that leaves early lets them land first (bounded)
    auto drain = [&](int j, int t0) {
        for (int i = 1; i < kTileBufs; ++i)
            if (t0 + i * stride < T)
                mbar_wait_bounded(&s_bar[(j + i) % kTileBufs], ((j + i) / kTileBufs) & 1, kTileWaitNs);
    };

    __half2 hmax = __float2half2_rn(0.f);  // largest |fp16 output| (packed)
#pragma unroll 1
    for (int j = 0, t0 = first; t0 < T; ++j, t0 += stride) {
        const int q = j % kTileBufs;
        const uint32_t par = (j / kTileBufs) & 1;  // tile j is buffer q's (j / kTileBufs)-th fill
        const bool ok = mbar_wait_bounded(&s_bar[q], par, kTileWaitNs);
        if (!__all_sync(0xffffffffu, ok)) {
            if ((tid & 31) == 0) record_error(a.error, M2_ERR_TIMEOUT);
            if (!ok) mbar_wait_bounded(&s_bar[q], par, kTileWaitNs);
            drain(j, t0);
            return;
        }
        AT (*s_rows)[kTileCh] = s_buf[q];
        if (vec_ok) {
            // window of token t0 + tg*8 + i: staged rows tg*8 + i .. tg*8 + i + K-1
            float hist[K - 1][VEC];
#pragma unroll
            for (int j = 0; j < K - 1; ++j) unpack16<AT>(*reinterpret_cast<const uint4*>(&s_rows[tg * TPT + j][v * VEC]), hist[j]);
#pragma unroll
            for (int i = 0; i < TPT; ++i) {
                const int t = t0 + tg * TPT + i;
                if (t >= T) break;
                OT* const optr = ob + t * a.out_stride + c0 + v * VEC;
                float cur[VEC];
                unpack16<AT>(*reinterpret_cast<const uint4*>(&s_rows[tg * TPT + i + K - 1][v * VEC]), cur);
                float o[VEC];
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {  // channel pairs: per channel bias, then taps 0..K-1
                    float2 acc = make_float2(bias[e], bias[e + 1]);
#pragma unroll
                    for (int k = 0; k < K - 1; ++k)
                        acc = __ffma2_rn(make_float2(w[e][k], w[e + 1][k]), make_float2(hist[k][e], hist[k][e + 1]), acc);
                    acc = __ffma2_rn(make_float2(w[e][K - 1], w[e + 1][K - 1]), make_float2(cur[e], cur[e + 1]), acc);
                    if (a.activation) {
                        if constexpr (std::is_same<OT, float>::value)
                            acc = silu2_f32(acc);
                        else
                            acc = silu2_tanh_f32(acc);
                    }
                    o[e] = acc.x;
                    o[e + 1] = acc.y;
                }
                if constexpr (std::is_same<OT, f16_t>::value) {
                    // the range check on the packed halves: |v| >= 65520 rounds to inf
                    const uint4 pk = pack16<OT>(o);
                    const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) hmax = __hmax2(hmax, __habs2(*reinterpret_cast<const __half2*>(&pw[e])));
                    *reinterpret_cast<uint4*>(optr) = pk;
                } else {
                    store_vec<OT, VEC>(optr, o);
                }
#pragma unroll
                for (int k = 0; k < K - 2; ++k) {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) hist[k][e] = hist[k + 1][e];
                }
#pragma unroll
                for (int e = 0; e < VEC; ++e) hist[K - 2][e] = cur[e];
            }
        }
        // this warp is done with buffer q; warp 0 refills it once all four are
        // (no block barrier: a warp that finishes early goes on to the next tile)
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive(&s_empty[q]);
        if (tid < 32 && t0 + kTileBufs * stride < T) {
            const bool eok = mbar_wait_bounded(&s_empty[q], (j / kTileBufs) & 1, kTileWaitNs);
            if (!__all_sync(0xffffffffu, eok)) {
                if (tid == 0) record_error(a.error, M2_ERR_TIMEOUT);
                drain(j, t0);
                return;
            }
            issue(t0 + kTileBufs * stride, q);  // tile j + kTileBufs lands in buffer q
        }
    }
    if (fmaxf(__low2float(hmax), __high2float(hmax)) >= 65520.f)
        record_error(a.error, M2_ERR_RANGE);  // beyond fp16 (rounds to inf)
    if (blockIdx.y == 0 && tg == 0 && vec_ok) {
        // new cache row k = raw input of token T-(K-1)+k: from the input when
        // that token exists, else old cache row k + T (read before it is written)
#pragma unroll
        for (int k = 0; k < K - 1; ++k) {
            const int t = T - (K - 1) + k;
            const int64_t c = c0 + v * VEC;
            const uint4 val = t >= 0 ? *reinterpret_cast<const uint4*>(xb + t * a.x_stride + c)
                                     : *reinterpret_cast<const uint4*>(cache + (k + T) * a.conv_dim + c);
            *reinterpret_cast<uint4*>(cache + k * a.conv_dim + c) = val;
        }
    }
}

template <typename OT, int K>
cudaError_t conv_tile_launch(const CUtensorMap& map, int use_tma, const ConvArgs& a, dim3 grid, cudaStream_t s) {
    constexpr size_t smem = kTileBufs * static_cast<size_t>(kTileTok + K - 1) * kTileCh * sizeof(bf16_t);
    static AttrOnce attrs;
    const cudaError_t e = attrs.ensure([] {
        return cudaFuncSetAttribute(conv1d_tile_kernel<OT, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem));
    });
    if (e != cudaSuccess) return e;
    conv1d_tile_kernel<OT, K><<<grid, kTileThreads, smem, s>>>(map, a, use_tma);
    return cudaGetLastError();
}

template <typename OT>
cudaError_t conv_tile_by_k(const ConvArgs& a, cudaStream_t s) {
    // Each CTA walks up to 8 token tiles of its sequence, double-buffered, as
    // long as the grid keeps about two waves of resident CTAs per SM.
    // Measured on the 8 x 2048 Nemotron-H prefill with 64-token tiles at three
    // CTAs per SM: one tile per CTA 221 us, 2 tiles 205 us, 4 tiles 196 us,
    // 8 tiles 192 us; with 32-token tiles at five CTAs per SM and 8 tiles, 154 us.
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    const int64_t ch_blocks = (a.conv_dim + kTileCh - 1) / kTileCh;
    const int64_t tiles = std::max<int64_t>((a.seqlen + kTileTok - 1) / kTileTok, 1);
    const int64_t per_cta = std::clamp<int64_t>(ch_blocks * a.batch * tiles / (2LL * kTileMinBlocks * sms), 1,
                                                kMaxTilesPerCta);
    const int64_t ctas_y = std::min<int64_t>((tiles + per_cta - 1) / per_cta, 65535);
    const dim3 grid(static_cast<unsigned>(ch_blocks), static_cast<unsigned>(ctas_y), static_cast<unsigned>(a.batch));
    // x as a 2-D tensor (channel, packed row) for one TMA box per tile, where
    // the rows are 16-byte aligned and the row count fits the 32-bit
    // coordinates; otherwise the rows are copied one by one
    CUtensorMap map{};
    int use_tma = 0;
    const TensorMapEncodeFn enc = tensor_map_encoder();
    if (enc && (a.x_stride * 2) % 16 == 0 && a.total_rows > 0 && a.total_rows <= INT32_MAX) {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.conv_dim), static_cast<cuuint64_t>(a.total_rows)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.x_stride) * 2};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileCh), static_cast<cuuint32_t>(kTileTok + a.K - 1)};
        const cuuint32_t estr[2] = {1, 1};
        use_tma = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.x), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    switch (a.K) {
        case 2: return conv_tile_launch<OT, 2>(map, use_tma, a, grid, s);
        case 3: return conv_tile_launch<OT, 3>(map, use_tma, a, grid, s);
        case 4: return conv_tile_launch<OT, 4>(map, use_tma, a, grid, s);
        case 5: return conv_tile_launch<OT, 5>(map, use_tma, a, grid, s);
        case 6: return conv_tile_launch<OT, 6>(map, use_tma, a, grid, s);
        case 7: return conv_tile_launch<OT, 7>(map, use_tma, a, grid, s);
        case 8: return conv_tile_launch<OT, 8>(map, use_tma, a, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename AT, typename OT>
cudaError_t conv_by_k(const ConvArgs& a, cudaStream_t s) {
    constexpr int VEC = Vec16<AT>::n;
    // token tiles per sequence: at least one, at most 65535 (the CTAs loop)
    const int64_t tiles = std::min<int64_t>(std::max<int64_t>((a.seqlen + kTT - 1) / kTT, 1), 65535);
    const dim3 grid(static_cast<unsigned>((a.conv_dim / VEC + kConvThreads - 1) / kConvThreads),
                    static_cast<unsigned>(tiles), static_cast<unsigned>(a.batch));
    switch (a.K) {
        case 2: conv1d_kernel<AT, OT, 2><<<grid, kConvThreads, 0, s>>>(a); break;
        case 3: conv1d_kernel<AT, OT, 3><<<grid, kConvThreads, 0, s>>>(a); break;
        case 4: conv1d_kernel<AT, OT, 4><<<grid, kConvThreads, 0, s>>>(a); break;
        case 5: conv1d_kernel<AT, OT, 5><<<grid, kConvThreads, 0, s>>>(a); break;
        case 6: conv1d_kernel<AT, OT, 6><<<grid, kConvThreads, 0, s>>>(a); break;
        case 7: conv1d_kernel<AT, OT, 7><<<grid, kConvThreads, 0, s>>>(a); break;
        case 8: conv1d_kernel<AT, OT, 8><<<grid, kConvThreads, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// Zero the SSM and conv regions of n slots; one CTA row per slot.
__global__ void __launch_bounds__(256) zero_slots_kernel(const ZeroArgs a) {
    const int32_t slot = a.slot_idx[blockIdx.y];
    if (slot < 0) return;
    if (slot >= a.num_slots) {
        if (threadIdx.x == 0 && blockIdx.x == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }
    const uint4 zero = make_uint4(0, 0, 0, 0);
    uint4* ssm = reinterpret_cast<uint4*>(static_cast<char*>(a.ssm) + slot * a.ssm_bytes_per_slot);
    uint4* conv = reinterpret_cast<uint4*>(static_cast<char*>(a.conv) + slot * a.conv_bytes_per_slot);
    const int64_t n_ssm = a.ssm_bytes_per_slot / 16;
    const int64_t n_conv = a.conv_bytes_per_slot / 16;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_ssm; i += stride)
        st_stream(ssm + i, zero);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_conv; i += stride)
        conv[i] = zero;
}

}  // namespace

cudaError_t launch_conv1d_update(const ConvArgs& a, cudaStream_t s) {
    // long sequences of bf16 activations: the shared-memory tile kernel
    if (a.act_bf16 && a.seqlen >= kTileTok) {
        if (a.out_dtype == M2_BF16) return conv_tile_by_k<bf16_t>(a, s);
        if (a.out_dtype == M2_F16) return conv_tile_by_k<f16_t>(a, s);
        return conv_tile_by_k<float>(a, s);
    }
    if (a.act_bf16) {
        if (a.out_dtype == M2_BF16) return conv_by_k<bf16_t, bf16_t>(a, s);
        if (a.out_dtype == M2_F16) return conv_by_k<bf16_t, f16_t>(a, s);
        return conv_by_k<bf16_t, float>(a, s);
    }
    if (a.out_dtype == M2_BF16) return conv_by_k<float, bf16_t>(a, s);
    if (a.out_dtype == M2_F16) return conv_by_k<float, f16_t>(a, s);
    return conv_by_k<float, float>(a, s);
}

cudaError_t launch_zero_slots(const ZeroArgs& a, cudaStream_t s) {
    if (a.n == 0) return cudaSuccess;
    const dim3 grid(32, static_cast<unsigned>(a.n));
    zero_slots_kernel<<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace m2
