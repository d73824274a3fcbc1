// m2_device.cuh -- small device helpers shared by the libm2 kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace m2 {

// Storage types: bf16 is carried as its raw 16-bit pattern; fp16 (IEEE
// binary16) as the CUDA __half type, so the two stay distinct C++ types.
using bf16_t = uint16_t;
using f16_t = __half;

__device__ __forceinline__ float bf16_to_f32(bf16_t v) {
    return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

// Round to nearest even (the hardware conversion).
__device__ __forceinline__ bf16_t f32_to_bf16(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Two floats -> one 32-bit word of two bf16 (lo = a, hi = b), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<bf16_t>(bf16_t v) { return bf16_to_f32(v); }

template <>
__device__ __forceinline__ float to_f32<f16_t>(f16_t v) { return __half2float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ bf16_t from_f32<bf16_t>(float v) { return f32_to_bf16(v); }
template <>
__device__ __forceinline__ f16_t from_f32<f16_t>(float v) { return __float2half_rn(v); }

// Elements of T per 16-byte vector.
template <typename T>
struct Vec16 {
    static constexpr int n = 16 / sizeof(T);
};

// Unpack a 16-byte vector into floats.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& v, float* out);
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& v, float* out) {
    out[0] = __uint_as_float(v.x);
    out[1] = __uint_as_float(v.y);
    out[2] = __uint_as_float(v.z);
    out[3] = __uint_as_float(v.w);
}
template <>
__device__ __forceinline__ void unpack16<bf16_t>(const uint4& v, float* out) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(w[i] << 16);
        out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Pack floats into a 16-byte vector, rounding to nearest even for bf16.
template <typename T>
__device__ __forceinline__ uint4 pack16(const float* in);
template <>
__device__ __forceinline__ uint4 pack16<float>(const float* in) {
    return make_uint4(__float_as_uint(in[0]), __float_as_uint(in[1]), __float_as_uint(in[2]),
                      __float_as_uint(in[3]));
}
template <>
__device__ __forceinline__ uint4 pack16<bf16_t>(const float* in) {
    return make_uint4(pack_bf16x2(in[0], in[1]), pack_bf16x2(in[2], in[3]),
                      pack_bf16x2(in[4], in[5]), pack_bf16x2(in[6], in[7]));
}

// Eight fp16 values <-> one 16-byte vector (round to nearest even).
__device__ __forceinline__ void unpack16_f16(const uint4& v, float* out) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
        out[2 * i] = f.x;
        out[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ uint4 pack16_f16(const float* in) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 h = __floats2half2_rn(in[2 * i], in[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <>
__device__ __forceinline__ void unpack16<f16_t>(const uint4& v, float* out) { unpack16_f16(v, out); }
template <>
__device__ __forceinline__ uint4 pack16<f16_t>(const float* in) { return pack16_f16(in); }

// Streaming 16-byte global load / store (data touched once per call).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_stream(void* p, const uint4& v) {
    __stcs(reinterpret_cast<uint4*>(p), v);
}

// ---- bulk asynchronous copies and mbarriers (shared memory addresses are
// 32-bit offsets in the shared window)

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Makes barrier initialisation visible to the async proxy and the cluster.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n" ::"r"(
                     smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// One 2-D TMA tile load (no multicast) of the box at element coordinates
// (x, y) of `map` into shared memory at `dst`, completing the box's bytes on
// `bar`. x times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_tile_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];\n" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}

// Plain arrive (release): one of the barrier's expected arrivals.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}

// One bulk copy global -> shared, completing `bytes` transactions on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}

// Waits for phase `parity` of `bar` for at most `limit_ns`; false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// Sums VPT row partials over the LPR lanes that share each row. For VPT = 4
// the first two levels exchange only the halves each lane keeps
// (reduce-scatter), so 4 rows cost 5 shuffles instead of 16. On return the
// lanes with (lane % (LPR/VPT)) == 0 hold the sum of row `which`.
template <int LPR, int VPT>
__device__ __forceinline__ float reduce_rows(const float (&acc)[VPT], int lane, int& which) {
    static_assert(VPT == 1 || VPT == 4, "one or four rows per thread");
    static_assert(LPR >= VPT, "reduce-scatter needs at least one lane per row");
    if constexpr (VPT == 1) {
        float v = acc[0];
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        which = 0;
        return v;
    } else {
        const bool hi1 = (lane & (LPR / 2)) != 0;   // keeps rows 2,3 instead of 0,1
        const float s0 = hi1 ? acc[0] : acc[2];
        const float s1 = hi1 ? acc[1] : acc[3];
        const float k0 = (hi1 ? acc[2] : acc[0]) + __shfl_xor_sync(0xffffffffu, s0, LPR / 2);
        const float k1 = (hi1 ? acc[3] : acc[1]) + __shfl_xor_sync(0xffffffffu, s1, LPR / 2);
        const bool hi2 = (lane & (LPR / 4)) != 0;   // keeps the odd row of the pair
        float v = (hi2 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, hi2 ? k0 : k1, LPR / 4);
#pragma unroll
        for (int off = LPR / 8; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        which = (hi1 ? 2 : 0) + (hi2 ? 1 : 0);
        return v;
    }
}

// softplus(v) = log(1 + exp(v)), v itself above 20.
__device__ __forceinline__ float softplus_f32(float v) {
    return v > 20.f ? v : log1pf(expf(v));
}

// 2^x and 1/x on the special-function unit (ex2.approx / rcp.approx, flush to
// zero; a couple of ulp each).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kNegLog2E = -1.4426950408889634f;  // -log2(e): exp(-v) = 2^(v * -log2 e)

// silu(v) = v / (1 + exp(-v)): exp(-v) = 2^(v * -log2 e) and the reciprocal of
// 1 + exp(-v) on the special-function unit, about 3 ulp in all. The limits
// come out right: for v -> -inf the exponential overflows to inf and its
// reciprocal to 0, for v -> +inf it underflows to 0. silu2_f32 is the same
// arithmetic on a pair, with packed f32x2 multiplies and adds (bit for bit
// silu_f32 of each half; the conv kernels, bound by instruction issue, take
// SiLUs in pairs). Every decode-side kernel uses these, so fused and unfused
// decode paths agree bit for bit; the prefill tile conv takes the tanh form
// below for its 16-bit outputs and these for fp32 outputs.
__device__ __forceinline__ float silu_f32(float v) {
    const float d = 1.f + ex2_approx(v * kNegLog2E);
    return v * rcp_approx(d);
}
// silu on a pair in the tanh form: silu(v) = h + h tanh(h), h = v / 2, with
// the hardware tanh (PTX tanh.approx, one special-function operation per
// value instead of two; relative error about 2^-11). For outputs rounded to a
// 16-bit type, whose own rounding is of that size.
__device__ __forceinline__ float2 silu2_tanh_f32(float2 v) {
    const float2 h = __fmul2_rn(v, make_float2(0.5f, 0.5f));
    float ta, tb;
    asm("tanh.approx.f32 %0, %1;" : "=f"(ta) : "f"(h.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(tb) : "f"(h.y));
    return __ffma2_rn(h, make_float2(ta, tb), h);
}
__device__ __forceinline__ float2 silu2_f32(float2 v) {
    const float2 t = __fmul2_rn(v, make_float2(kNegLog2E, kNegLog2E));
    const float2 d = __fadd2_rn(make_float2(1.f, 1.f), make_float2(ex2_approx(t.x), ex2_approx(t.y)));
    return __fmul2_rn(v, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

}  // namespace m2
