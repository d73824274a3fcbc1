// m2_chunk_scan_tc.cu -- chunked prefill scan on the 5th-generation tensor
// cores (tcgen05 + TMEM, operands staged by TMA), bf16 state and activations.
//
// Operation: vllm.cpp issue #1311 "NemotronH runs the PREFILL mamba kernels at
// decode", section "The divergence" (the chunk scan that follows the prefill
// conv) and section "Confirm or refute" (it must land on the state of the
// sequential updates). The Mamba-2 recurrence over a chunk of Q = 128 tokens
// t = 0..Q-1 of one head, with c_t = sum_{r<=t} dt_r * A (A = -exp(A_log)),
// written in its chunked (state-space dual) form:
//   Y      = (C B^T o L o dt_u) X + diag(exp(c_t)) C S^T + D x      (y before the gate)
//   S_next = exp(c_end) S + X^T (w o B),   w_u = exp(c_end - c_u) dt_u
// with L[t,u] = exp(c_t - c_u) for u <= t, else 0. The four products run as
// tcgen05 MMAs (M = 128, fp16 operands, fp32 accumulators in TMEM):
//   MMA1  CB     [t,u] = C . B^T        A = C (K-major), B = B (K-major)
//   MMA3  Yoff   [t,p] = C . S^T        A = C (K-major), B = S (K-major, fp16 copy)
//   MMA2  Ydiag  [t,p] = M . X          A = M = CB o L o dt + D I (K-major), B = X (MN-major)
//   MMA4  dS^T   [n,p] = W^T . X        A = W = w o B (MN-major), B = X (MN-major)
//         (the pipelined kernel below forms the same sum as B^T . (w o X): x
//         scaled per token into its own tile, B as loaded)
// The state itself is carried exactly in fp32 registers (thread n holds column
// n of S) and rounded once when the sequence ends. Only the chunk-to-chunk carry
// is sequential. D x rides on the diagonal of M, so once MMA2 and MMA4 are
// done no operand tile is read again and the next chunk's TMA loads overlap
// the output epilogue.
//
// Operand precision. The intra-chunk terms dt_u (C_t . B_u) x_u are often an
// order of magnitude larger than y itself, so rounding M, W and the state copy
// to bf16 (8-bit significand) leaves absolute errors of a few percent of
// rms(y). The MMAs therefore take fp16 operands (11-bit significand, the same
// A/B type in every MMA): an fp16 post-conv buffer is used as loaded, a bf16 one
// is converted exactly in shared memory after each load, and M, W, S are
// rounded once to fp16. Any value outside the fp16 range (|v| >= 65520)
// records M2_ERR_RANGE.
//
// One CTA of 256 threads per (sequence, head). Thread t owns TMEM lane
// r = t % 128 (row r of every accumulator; warps w and w+4 share a lane quarter)
// and the column half h2 = t / 128 of that row. Shared memory (1024-byte
// aligned, 128-byte swizzle):
//   C tile  32 KB [2 atoms of 64 n][128 t][128 B]   later overwritten by M
//   B tile  32 KB [2 atoms of 64 n][128 u][128 B]   later scaled in place to W
//   X tile  16 KB [128 u][64 p]
//   S copy  16 KB [2 atoms of 64 n][64 p][128 B]    fp16 state for MMA3
// TMEM (256 columns): CB at 0..127 (then dS^T at 0..63), Yoff at 128..191,
// Ydiag at 192..255. Tokens past the sequence end arrive as zeros from TMA and
// get dt = 0, so they neither decay nor feed the state.
//
// Every wait is bounded (one second of %globaltimer); the CTA takes the
// timeout decision together (__syncthreads_and), records M2_ERR_TIMEOUT, waits
// once more for its own copies and MMAs, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <type_traits>

#include "m2_device.cuh"
#include "m2_internal.cuh"

namespace m2 {
namespace {

constexpr int kQ = 128;   // tokens per chunk = MMA M
constexpr int kP = 64;    // head dim
constexpr int kN = 128;   // state dim
constexpr int kTC = 256;  // threads per CTA: two threads per TMEM lane (row)
constexpr uint32_t kOffC = 0, kOffB = 32768, kOffX = 65536, kOffS = 81920, kSmemUsed = 98304;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColCB = 0, kColDS = 0, kColYoff = 128, kColYdiag = 192;
constexpr uint64_t kLimitNs = 1000000000ull;

// ---- tcgen05 / TMA helpers -----------------------------------------------

// Shared-memory matrix descriptor, 128-byte swizzle, sm100 version field.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // descriptor version (sm100)
    d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: fp16 A and B (format 0), fp32 D, dense.
constexpr uint32_t idesc_f16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane. The wait for the
// load sits in the same asm statement, so no use of the registers can be
// scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive fp32 columns of this thread's TMEM lane (load and wait as above).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Two blocks of 16 consecutive fp32 columns of this thread's TMEM lane (at
// taddr_a and taddr_b), with one wait for both loads.
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr_a, uint32_t taddr_b, float (&va)[16], float (&vb)[16]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr_a), "r"(taddr_b)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        va[i] = __uint_as_float(r[i]);
        vb[i] = __uint_as_float(r[16 + i]);
    }
}

// 2^x with the hardware approximation (PTX ex2.approx, relative error about
// 2^-22); the decay sums are kept in log2 units so exp(c) = 2^(c log2 e).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// silu(v) = v sigmoid(v) = h + h tanh(h) with h = v/2, on a pair, with the
// hardware tanh (PTX tanh.approx, relative error about 2^-11: below half an
// ulp of the bf16 y it feeds). One MUFU operation per element instead of two.
__device__ __forceinline__ float2 silu2_tanh(float a, float b) {
    const float2 hh = __fmul2_rn(make_float2(a, b), make_float2(0.5f, 0.5f));
    float ta, tb;
    asm("tanh.approx.f32 %0, %1;\n" : "=f"(ta) : "f"(hh.x));
    asm("tanh.approx.f32 %0, %1;\n" : "=f"(tb) : "f"(hh.y));
    return __ffma2_rn(hh, make_float2(ta, tb), hh);
}

// Generic-proxy shared-memory writes become visible to the async proxy
// (tensor cores, TMA).
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}

// One 2-D TMA tile store (no multicast) from shared memory at `src` to the box
// at element coordinates (x, y) of `map`, in the thread's bulk group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(src)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
}
// Waits until every bulk store of this thread has read its shared memory.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }

// Byte offset of 16-byte chunk j of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t j) { return r * 128u + ((j ^ (r & 7u)) << 4); }

constexpr float kF16Limit = 65520.f;  // smallest magnitude that rounds to fp16 infinity

// Converts a 16-byte chunk of 8 bf16 values in shared memory to fp16 in place;
// returns the largest magnitude seen.
__device__ __forceinline__ float bf16_chunk_to_f16(uint8_t* p) {
    float v[8];
    unpack16<bf16_t>(*reinterpret_cast<const uint4*>(p), v);
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(v[e]));
    *reinterpret_cast<uint4*>(p) = pack16_f16(v);
    return mx;
}

// Segments a sequence of nchunks chunks is cut into: seg_chunks chunks each,
// at most nseg (the grid's segments per sequence), 1 when unsplit.
__device__ __forceinline__ int segments_of(int nchunks, int nseg, int seg_chunks) {
    if (nseg <= 1 || nchunks <= seg_chunks) return 1;
    return min(nseg, (nchunks + seg_chunks - 1) / seg_chunks);
}

// XT: element type of the post-conv xBC tiles (bf16_t: converted to fp16 in
// shared memory after each load; f16_t: used as loaded).
// STATE_ONLY: the first pass of a split sequence. The CTA runs one segment of
// chunks from a zero state and stores only its final state (fp32, scratch)
// and the segment's total decay: no C tile, no y, only the dS^T MMA.
// Otherwise the CTA scans its segment (the whole sequence when unsplit) from
// its initial state and writes y; the last segment stores the state.
template <typename ST, typename XT, bool STATE_ONLY>
__global__ void __launch_bounds__(kTC, 2)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const ScanArgs a) {
    extern __shared__ uint8_t s_raw[];
    __shared__ __align__(8) uint64_t s_bar_ld;
    __shared__ __align__(8) uint64_t s_bar_mma;
    __shared__ uint32_t s_tmem;
    // c_t in log2 units and dt_t, double-buffered by chunk parity: the next
    // chunk's are computed while this chunk's second MMA pair runs
    __shared__ __align__(16) float s_cum[2][kQ];
    __shared__ __align__(16) float s_dt[2][kQ];
    // g_u^(b) = exp(c_{32b} - c_u) dt_u for row blocks b = 1..3 and u < 32b,
    // at offsets 0, 32, 96
    __shared__ __align__(16) float s_gam[192];
    __shared__ float s_wsum[kQ / 32];

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int r = tid & (kQ - 1);   // TMEM lane / tile row of this thread
    const int h2 = tid >> 7;        // column half of this thread
    const int h = blockIdx.x;
    const int nseg = a.nseg;  // segments per sequence in the grid (1: unsplit)
    const int b = blockIdx.y / nseg;
    const int seg = blockIdx.y - b * nseg;
    const int H = a.H;
    const int G = a.G;
    const int g = h / (H / G);
    const int64_t HP = static_cast<int64_t>(H) * kP;
    // this sequence's rows of the packed token arrays, and its chunk range
    const int64_t row0 = a.cu_seqlens ? static_cast<int64_t>(a.cu_seqlens[b]) : static_cast<int64_t>(b) * a.seqlen;
    const int T = a.cu_seqlens ? a.cu_seqlens[b + 1] - a.cu_seqlens[b] : a.seqlen;
    if (T <= 0) return;  // an empty sequence leaves its cache slot untouched
    const int nchunks_seq = (T + kQ - 1) / kQ;
    const int nseg_s = segments_of(nchunks_seq, nseg, a.seg_chunks);
    const bool split = nseg_s > 1;
    if (seg >= nseg_s) return;                                  // empty segment
    if (STATE_ONLY && (!split || seg == nseg_s - 1)) return;   // nothing to summarise
    // the last segment runs to the end of the sequence (also when the sequence
    // is longer than the grid was planned for)
    const int c_begin = split ? seg * a.seg_chunks : 0;
    const int c_end = (split && seg < nseg_s - 1) ? c_begin + a.seg_chunks : nchunks_seq;
    const int32_t slot = a.slot_idx[b];
    bf16_t* y = static_cast<bf16_t*>(a.y);

    if (slot < 0) {  // padding row: y = 0 over this segment's tokens, cache untouched
        if constexpr (!STATE_ONLY) {
            const int64_t tb = static_cast<int64_t>(c_begin) * kQ;
            const int64_t te = min(static_cast<int64_t>(c_end) * kQ, static_cast<int64_t>(T));
            for (int64_t i = tb * (kP / 8) + tid; i < te * (kP / 8); i += kTC) {
                const int64_t t = i / (kP / 8);
                *reinterpret_cast<uint4*>(y + (row0 + t) * a.y_stride + h * kP + (i % (kP / 8)) * 8) =
                    make_uint4(0, 0, 0, 0);
            }
        }
        return;
    }
    if (slot >= a.num_slots) {
        if (tid == 0 && !STATE_ONLY) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }

    // 1024-byte aligned base for the swizzled tiles
    const uint32_t raw_addr = smem_addr(s_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* sm = s_raw + (base - raw_addr);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_addr(&s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&s_bar_ld, 1);
        mbar_init(&s_bar_mma, 1);
        fence_mbar_init();
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;  // this warp's TMEM lanes

    const float A = -expf(a.A_log[h]);
    const float A2 = A * 1.4426950408889634f;  // A log2(e)
    const float dt_bias = a.dt_bias[h];
    const float Dh = a.D[h];
    const int xcol = h * kP;
    const int bcol = static_cast<int>(HP) + g * kN;
    const int ccol = static_cast<int>(HP) + G * kN + g * kN;

    // running state: thread (n = r, h2) holds S[p][n] for p = 32*h2 .. 32*h2+31 (fp32)
    constexpr int kPH = kP / 2;
    const int n = r;
    const int p0 = h2 * kPH;
    ST* state = static_cast<ST*>(a.ssm) + (static_cast<int64_t>(slot) * HP + static_cast<int64_t>(h) * kP) * kN;
    float S[kPH];
    float range_max = 0.f;  // largest magnitude handed to an fp16 operand (fp32 side)
    __half2 hmax = __float2half2_rn(0.f);  // the same for values already rounded to fp16
    // scratch slot j of (sequence b, head h): [batch][nseg][H][P][N] fp32
    auto seg_slot = [&](int j) {
        return a.seg_state + ((static_cast<int64_t>(b) * nseg + j) * H + h) * (kP * kN);
    };
    if (STATE_ONLY) {
#pragma unroll
        for (int i = 0; i < kPH; ++i) S[i] = 0.f;
    } else if (split) {  // initial state of this segment, from the combine pass
        const float* src = seg_slot(seg);
#pragma unroll
        for (int i = 0; i < kPH; ++i) S[i] = src[(p0 + i) * kN + n];
    } else {
        const bool init = a.has_init != nullptr && a.has_init[b] != 0;
#pragma unroll
        for (int i = 0; i < kPH; ++i) S[i] = init ? to_f32(state[(p0 + i) * kN + n]) : 0.f;
    }
    // fp16 copy for MMA3: element (p, n) of the K-major [2 atoms][64 p][64 n] tile
    auto write_state_copy = [&]() {
        uint8_t* sS = sm + kOffS + (n >> 6) * 8192;
        const uint32_t j = (n & 63) >> 3;
#pragma unroll
        for (int i = 0; i < kPH; i += 2) {
            const __half2 hv = __floats2half2_rn(S[i], S[i + 1]);
            hmax = __hmax2(hmax, __habs2(hv));
            *reinterpret_cast<__half*>(sS + sw128(p0 + i, j) + (n & 7) * 2) = __low2half(hv);
            *reinterpret_cast<__half*>(sS + sw128(p0 + i + 1, j) + (n & 7) * 2) = __high2half(hv);
        }
    };
    if (!STATE_ONLY) write_state_copy();

    const uint32_t id_cb = idesc_f16(128, 128, false, false);
    const uint32_t id_yoff = idesc_f16(128, 64, false, false);
    const uint32_t id_ydiag = idesc_f16(128, 64, false, true);
    const uint32_t id_ds = idesc_f16(128, 64, true, true);
    // chunk c of the sequence = packed rows row0 + 128c ..; rows past the end
    // of the buffer arrive as zeros, rows of the next sequence get dt = 0
    auto issue_loads = [&](int c) {
        const int ty = static_cast<int>(row0 + static_cast<int64_t>(c) * kQ);
        mbar_arrive_expect_tx(&s_bar_ld, (STATE_ONLY ? 3u : 5u) * 16384u);
        tma_load_2d(base + kOffX, &tmap_x, xcol, ty, &s_bar_ld);
        tma_load_2d(base + kOffB, &tmap_x, bcol, ty, &s_bar_ld);
        tma_load_2d(base + kOffB + 16384, &tmap_x, bcol + 64, ty, &s_bar_ld);
        if (!STATE_ONLY) {
            tma_load_2d(base + kOffC, &tmap_x, ccol, ty, &s_bar_ld);
            tma_load_2d(base + kOffC + 16384, &tmap_x, ccol + 64, ty, &s_bar_ld);
        }
    };
    if (tid == 0 && c_begin < c_end) issue_loads(c_begin);

    bool ok = true;
    int loads_issued = c_begin < c_end ? 1 : 0, loads_done = 0, mma_issued = 0, mma_done = 0;
    const int t = r;  // token (row) of this thread within a chunk
    // raw dt bits of this thread's token in the chunk to be prepared next: kept
    // unconverted so the load stays in flight until that chunk needs it
    bf16_t dt_raw_next = 0;
    if (tid < kQ && c_begin * kQ + tid < T) dt_raw_next = static_cast<const bf16_t*>(a.dt)[(row0 + c_begin * kQ + tid) * a.dt_stride + h];
    float seg_log2 = 0.f;  // total decay of the chunks done so far, log2 units
    // dt and the cumulative decay c_t of chunk cn, in two parts around a block
    // barrier (warps 0..3, thread = token): the in-warp scan, then the
    // cross-warp prefix and the store into buffer cn & 1.
    auto cum_scan = [&](int cn, float& dt, float& cum) {
        const int vn = min(kQ, T - cn * kQ);
        dt = (t < vn) ? softplus_f32(to_f32(dt_raw_next) + dt_bias) : 0.f;
        if (cn + 1 < c_end && t < min(kQ, T - (cn + 1) * kQ))  // prefetch the following chunk's raw dt
            dt_raw_next = static_cast<const bf16_t*>(a.dt)[(row0 + (cn + 1) * kQ + t) * a.dt_stride + h];
        cum = dt * A2;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, cum, off);
            if (lane >= off) cum += o;
        }
        if (lane == 31) s_wsum[warp] = cum;
    };
    auto cum_store = [&](int cn, float dt, float cum) {
        for (int w = 0; w < warp; ++w) cum += s_wsum[w];
        s_cum[cn & 1][t] = cum;
        s_dt[cn & 1][t] = dt;
    };
    {
        float dt0 = 0.f, cum0 = 0.f;
        if (h2 == 0 && c_begin < c_end) cum_scan(c_begin, dt0, cum0);
        __syncthreads();
        if (h2 == 0 && c_begin < c_end) cum_store(c_begin, dt0, cum0);
    }
    for (int c = c_begin; c < c_end; ++c) {
        const int t0 = c * kQ;
        const int valid = min(kQ, T - t0);
        const float* cum_c = s_cum[c & 1];
        const float* dt_c = s_dt[c & 1];

        // ---- wait for X, B, C; MMA1 (CB) and MMA3 (Yoff)
        bool got = mbar_wait_bounded(&s_bar_ld, loads_done & 1, kLimitNs);
        if (!__syncthreads_and(got)) { ok = false; break; }
        ++loads_done;
        if constexpr (std::is_same<XT, bf16_t>::value) {
            // bf16 -> fp16 in place (exact within range): row t of C and B
            // (atom h2) and half of row t of X. Chunks are visited in swizzled
            // order (any order converts the whole row), so the eight rows a
            // quarter-warp touches fall in different banks.
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (!STATE_ONLY)
                    range_max = fmaxf(range_max, bf16_chunk_to_f16(sm + kOffC + h2 * 16384 + sw128(t, j)));
                range_max = fmaxf(range_max, bf16_chunk_to_f16(sm + kOffB + h2 * 16384 + sw128(t, j)));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                range_max = fmaxf(range_max, bf16_chunk_to_f16(sm + kOffX + sw128(t, 4 * h2 + j)));
            fence_proxy_async();
            __syncthreads();
        }
        const float cum_end = cum_c[kQ - 1];
        seg_log2 += cum_end;
        if constexpr (!STATE_ONLY) {
        if (tid < 192) {  // decay factors of the off-diagonal blocks of M (read after the MMA wait)
            const int bq = tid < 32 ? 1 : (tid < 96 ? 2 : 3);
            const int u = tid - (bq == 1 ? 0 : (bq == 2 ? 32 : 96));
            s_gam[tid] = ex2(cum_c[32 * bq] - cum_c[u]) * dt_c[u];
        }
        if (tid == 0) {
            tc_fence_after();
            for (int k = 0; k < kN / 16; ++k) {
                const uint32_t koff = (k >> 2) * 16384u + (k & 3) * 32u;
                mma_f16(tmem + kColCB, sw128_desc(base + kOffC + koff, 16, 1024),
                         sw128_desc(base + kOffB + koff, 16, 1024), id_cb, k > 0);
            }
            for (int k = 0; k < kN / 16; ++k) {
                const uint32_t koff = (k >> 2) * 16384u + (k & 3) * 32u;
                const uint32_t soff = (k >> 2) * 8192u + (k & 3) * 32u;
                mma_f16(tmem + kColYoff, sw128_desc(base + kOffC + koff, 16, 1024),
                         sw128_desc(base + kOffS + soff, 16, 1024), id_yoff, k > 0);
            }
            mma_commit(&s_bar_mma);
        }
        ++mma_issued;
        got = mbar_wait_bounded(&s_bar_mma, mma_done & 1, kLimitNs);
        if (!__syncthreads_and(got)) { ok = false; break; }
        ++mma_done;
        tc_fence_after();
        }  // !STATE_ONLY

        // ---- epilogue 1: M = CB o L o dt + D I (row t, fp16, into the C tile)
        // and W = w o B (row u = t of the B tile, scaled in place)
        {
            const float cum_t = cum_c[t];
            if constexpr (!STATE_ONLY) {
            const int wq = warp & 3;  // this warp's rows are t = 32*wq .. 32*wq+31
            // Off-diagonal blocks (u < 32 wq <= t) factor through the decay at
            // the block start: L[t,u] = exp(c_t - c_{32wq}) exp(c_{32wq} - c_u),
            // both factors <= 1 since c is non-increasing, so M = CB * alpha_t * g_u.
            const float alpha = ex2(cum_t - cum_c[32 * wq]);
            const float2 alpha2 = make_float2(alpha, alpha);
            const float* gam = s_gam + (wq == 1 ? 0 : (wq == 2 ? 32 : 96));
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                // this thread's columns u = 32q + 16 h2 .. +15: chunks j0, j0+1 of atom q/2
                uint8_t* dst = sm + kOffC + (q >> 1) * 16384;
                const uint32_t j0 = (q & 1) * 4 + 2 * h2;
                const int u0 = q * 32 + 16 * h2;
                if (q > wq) {  // every u > t: the causal mask zeroes the block (warp-uniform)
                    *reinterpret_cast<uint4*>(dst + sw128(t, j0)) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(dst + sw128(t, j0 + 1)) = make_uint4(0, 0, 0, 0);
                    continue;
                }
                float m[16];
                tmem_ld16(tmem + lane_base + kColCB + u0, m);
                if (q < wq) {
                    const float4* g4 = reinterpret_cast<const float4*>(gam + u0);
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const float4 g = g4[i4];
                        float2 lo = __fmul2_rn(make_float2(m[4 * i4], m[4 * i4 + 1]), make_float2(g.x, g.y));
                        float2 hi = __fmul2_rn(make_float2(m[4 * i4 + 2], m[4 * i4 + 3]), make_float2(g.z, g.w));
                        lo = __fmul2_rn(lo, alpha2);
                        hi = __fmul2_rn(hi, alpha2);
                        m[4 * i4] = lo.x;
                        m[4 * i4 + 1] = lo.y;
                        m[4 * i4 + 2] = hi.x;
                        m[4 * i4 + 3] = hi.y;
                    }
                } else {  // diagonal block: exact per-element decay, mask u > t, D x_t rides on u = t
                    const float4* cu4 = reinterpret_cast<const float4*>(cum_c + u0);
                    const float4* du4 = reinterpret_cast<const float4*>(dt_c + u0);
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const float4 cu = cu4[i4], du = du4[i4];
                        const float cuv[4] = {cu.x, cu.y, cu.z, cu.w};
                        const float duv[4] = {du.x, du.y, du.z, du.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int u = u0 + 4 * i4 + e;
                            float v = m[4 * i4 + e] * ex2(cum_t - cuv[e]) * duv[e];
                            if (u > t) v = 0.f;
                            if (u == t) v += Dh;
                            m[4 * i4 + e] = v;
                        }
                    }
                }
                uint32_t hw[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const __half2 hv = __floats2half2_rn(m[2 * i], m[2 * i + 1]);
                    hmax = __hmax2(hmax, __habs2(hv));
                    hw[i] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                *reinterpret_cast<uint4*>(dst + sw128(t, j0)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(dst + sw128(t, j0 + 1)) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
            }
            }  // !STATE_ONLY
            // W row t = w_t * B row t, multiplied in fp16 pairs (w rounded once to fp16)
            const float wu = (t < valid) ? ex2(cum_end - cum_t) * dt_c[t] : 0.f;
            const __half2 w2 = __float2half2_rn(wu);
            hmax = __hmax2(hmax, __habs2(w2));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                // swizzled chunk order: conflict-free across the quarter-warp's rows
                uint4* p = reinterpret_cast<uint4*>(sm + kOffB + h2 * 16384 + sw128(t, j));
                uint4 v = *p;
                uint32_t* vw = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half2 r2 = __hmul2(*reinterpret_cast<const __half2*>(&vw[e]), w2);
                    hmax = __hmax2(hmax, __habs2(r2));
                    vw[e] = *reinterpret_cast<const uint32_t*>(&r2);
                }
                *p = v;
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- MMA2 (Ydiag = M X) and MMA4 (dS^T = W^T X)
        if (tid == 0) {
            tc_fence_after();
            if (!STATE_ONLY) {
                for (int k = 0; k < kQ / 16; ++k) {
                    const uint32_t koff = (k >> 2) * 16384u + (k & 3) * 32u;
                    mma_f16(tmem + kColYdiag, sw128_desc(base + kOffC + koff, 16, 1024),
                             sw128_desc(base + kOffX + k * 2048u, 16384, 1024), id_ydiag, k > 0);
                }
            }
            for (int k = 0; k < kQ / 16; ++k) {
                mma_f16(tmem + kColDS, sw128_desc(base + kOffB + k * 2048u, 16384, 1024),
                         sw128_desc(base + kOffX + k * 2048u, 16384, 1024), id_ds, k > 0);
            }
            mma_commit(&s_bar_mma);
        }
        ++mma_issued;
        // z of this thread's row half (used in epilogue 2): its latency
        // overlaps the MMAs
        uint4 zpre[4];
        {
            const bool zok = !STATE_ONLY && a.z != nullptr && t < valid;
            const bf16_t* zr = zok ? static_cast<const bf16_t*>(a.z) + (row0 + t0 + t) * a.z_stride + xcol + 32 * h2
                                   : nullptr;
#pragma unroll
            for (int j = 0; j < 4; ++j) zpre[j] = zok ? *reinterpret_cast<const uint4*>(zr + 8 * j) : make_uint4(0, 0, 0, 0);
        }
        // the next chunk's dt and decay sums, while the MMAs run
        float dt_n = 0.f, cum_n = 0.f;
        if (h2 == 0 && c + 1 < c_end) cum_scan(c + 1, dt_n, cum_n);
        got = mbar_wait_bounded(&s_bar_mma, mma_done & 1, kLimitNs);
        if (!__syncthreads_and(got)) { ok = false; break; }
        ++mma_done;
        tc_fence_after();
        if (h2 == 0 && c + 1 < c_end) cum_store(c + 1, dt_n, cum_n);
        // C, B and X are dead now (epilogue 2 reads TMEM and writes only the
        // state copy): the next chunk's tiles stream in underneath it
        if (tid == 0 && c + 1 < c_end) {
            issue_loads(c + 1);
            ++loads_issued;
        }

        // ---- epilogue 2: y row t, then the state carry (thread n = t)
        {
            const float cum_t_e2 = cum_c[t];
            const float et = ex2(cum_t_e2);
            const bool row_ok = t < valid;
            const bool gate = a.z != nullptr;
            bf16_t* yrow = y + (row0 + t0 + t) * a.y_stride + xcol;
            if constexpr (!STATE_ONLY) {
                const int q = h2;  // columns p = 32*h2 .. 32*h2+31, in two passes of 16
                const float2 et2 = make_float2(et, et);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float yd[16], yo[16];
                    tmem_ld16(tmem + lane_base + kColYdiag + q * 32 + 16 * hh, yd);
                    tmem_ld16(tmem + lane_base + kColYoff + q * 32 + 16 * hh, yo);
#pragma unroll
                    for (int jh = 0; jh < 2; ++jh) {
                        const int jj = 2 * hh + jh;
                        const uint32_t j = q * 4 + jj;  // chunk of 8 p values
                        float out[8];
                        float zv[8];
                        unpack16<bf16_t>(zpre[jj], zv);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            // D x is in Ydiag
                            float2 v = __ffma2_rn(et2, make_float2(yo[8 * jh + e], yo[8 * jh + e + 1]),
                                                  make_float2(yd[8 * jh + e], yd[8 * jh + e + 1]));
                            if (gate) v = __fmul2_rn(v, silu2_tanh(zv[e], zv[e + 1]));
                            out[e] = v.x;
                            out[e + 1] = v.y;
                        }
                        if (row_ok) *reinterpret_cast<uint4*>(yrow + 8 * j) = pack16<bf16_t>(out);
                    }
                }
            }
            const float eend = ex2(cum_end);
            {
                float ds[32];
                tmem_ld32(tmem + lane_base + kColDS + p0, ds);
#pragma unroll
                for (int i = 0; i < kPH; ++i) S[i] = fmaf(eend, S[i], ds[i]);
            }
            if (!STATE_ONLY) write_state_copy();
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
    }
    if (ok) {
        if constexpr (STATE_ONLY) {  // segment summary for the combine pass
            float* dst = seg_slot(seg + 1);
#pragma unroll
            for (int i = 0; i < kPH; ++i) dst[(p0 + i) * kN + n] = S[i];
            if (tid == 0) a.seg_decay[(static_cast<int64_t>(b) * nseg + seg) * H + h] = ex2(seg_log2);
        } else if (!split || seg == nseg_s - 1) {  // the sequence's final state, in place
#pragma unroll
            for (int i = 0; i < kPH; ++i) state[(p0 + i) * kN + n] = from_f32<ST>(S[i]);
        }
        range_max = fmaxf(range_max, fmaxf(__low2float(hmax), __high2float(hmax)));  // inf if rounded out of range
        if (range_max >= kF16Limit) record_error(a.error, M2_ERR_RANGE);
    } else {
        if (tid == 0) record_error(a.error, M2_ERR_TIMEOUT);
        // let this CTA's own copies and MMAs finish (bounded) before freeing
        if (loads_done < loads_issued) mbar_wait_bounded(&s_bar_ld, loads_done & 1, kLimitNs);
        if (mma_done < mma_issued) mbar_wait_bounded(&s_bar_mma, mma_done & 1, kLimitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// Pipelined variant: warp-specialised, two chunks in flight (fp16 post-conv
// input). The per-chunk chain of the kernel above is latency-bound (load, CB,
// epilogue 1, M X and the state MMA, epilogue 2, one after the other). Only
// epilogue 2 and C S^T depend on the carried state, so here they form the
// sequential chain while epilogue 1 of the next chunk runs beside them:
//   warp 0        TMA producer: stage (c & 1) <- x, B, C tiles of chunk c
//   warp 1        MMA issuer: C S^T, M X, dS^T = B^T (w o X), then CB of the
//                 next chunk
//   warps 2..9    epilogue 1 (256 threads): dt and decay sums, M (into TMEM
//                 in place of CB, as the A operand of M X, so the C tile
//                 stays intact for C S^T) and w o x (the x tile scaled by
//                 the decay-to-chunk-end weights w_t = exp(cum_end - cum_t) dt_t)
//   warps 10..17  epilogue 2 (256 threads): the fp32 state carry of chunk c
//                 and its fp16 copy for C S^T of chunk c+1 first, then y of
//                 chunk c
//   warp 18       mover: the y tile of chunk c out and the z tile of chunk
//                 c+1 in (TMA), off the epilogue-2 chain
// Per chunk the issuer runs C S^T as soon as the state entering the chunk is
// ready (normally while epilogue 1 still works on M), then M X as soon as
// every epilogue-1 thread has written its rows of M (the last of them are
// still scaling x), then B^T (w o X) once w o x is built, after which the
// stage's tiles are free for the load of chunk c+2, then CB of chunk c+1
// (once M X of chunk c has read M). MMAs complete in issue order, so once dS
// of chunk c is in, C S^T of chunk c has read the state copy and epilogue 2
// overwrites it with the state leaving chunk c; y leaves the chain.
// One CTA per SM: two shared-memory stages of 80 KB, a 16 KB fp16 state copy
// (n-major like the x tile), the 16 KB w o x tile (fp16) and a 16 KB z / y
// tile. TMEM holds two rings with their own lifetimes:
//   ring A (columns 0..127, one stage): CB, then M in place of it. Each
//     epilogue-1 thread writes the fp16 pairs of M's K-step k (its columns
//     u = 16k..16k+15) into the first 8 of the 16 columns it read CB from,
//     so no thread overwrites a column another thread has still to read.
//     Free once M X has completed, which CB of the next chunk waits for.
//   ring B (columns 128..511, two stages of 192): Ydiag at 0..63, dS^T at
//     64..127, Yoff at 128..191 of a stage; free once every epilogue-2
//     thread has read it.
// Every hand-off is an mbarrier; every wait is bounded and a timeout ends all
// roles with M2_ERR_TIMEOUT.
#ifndef M2_SCAN_PIPELINED
#define M2_SCAN_PIPELINED 1
#endif
constexpr int kP2Threads = 608;
constexpr uint32_t kP2Stage = 81920;                       // C 32 KB | B 32 KB | X 16 KB
constexpr uint32_t kP2OffS = 2 * kP2Stage;                 // the fp16 state copy (16 KB)
constexpr uint32_t kP2OffXw = kP2OffS + 16384;             // w o x of a chunk (fp16, 16 KB)
constexpr uint32_t kP2OffZ = kP2OffXw + 16384;             // the z tile of a chunk (bf16, 16 KB)
constexpr uint32_t kP2Smem = kP2OffZ + 16384 + 1024;       // + alignment slack
constexpr uint32_t kP2TmemCols = 512;

// D (TMEM) = A (TMEM, K-major fp16 pairs) . B (shared memory descriptor)
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 8 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// Barrier of one 256-thread role (named barrier `id`) that also ORs `flag`
// over the role: every thread gets the same answer.
__device__ __forceinline__ bool role_sync_or(int id, bool flag) {
    uint32_t out;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
        " bar.red.or.pred q, %2, 256, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(out)
        : "r"(flag ? 1u : 0u), "r"(id)
        : "memory");
    return out != 0;
}

// Waits for phase `parity` of `bar`, giving up after the time limit or as soon
// as another role has aborted.
__device__ __forceinline__ bool p2_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag || global_ns() - t0 > kLimitNs) return false;
    }
    return true;
}

__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}

template <typename ST>
__global__ void __launch_bounds__(kP2Threads, 1)
chunk_scan_p2_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_z,
                     const __grid_constant__ CUtensorMap tmap_y, const ScanArgs a) {
    extern __shared__ uint8_t s_raw[];
    __shared__ __align__(8) uint64_t s_full[2], s_cb[2], s_m[2], s_d[2], s_yoff[2], s_free[2], s_tfree[2];
    __shared__ __align__(8) uint64_t s_w[2];  // W of stage q is built (every epilogue-1 thread arrives)
    __shared__ __align__(8) uint64_t s_sready[2];  // state copy (i & 1) holds the state entering chunk i
    __shared__ __align__(8) uint64_t s_drain;
    __shared__ __align__(8) uint64_t s_mx;  // M X of the last chunk has completed (TMEM ring A is free)
    __shared__ __align__(8) uint64_t s_z;  // the z tile of the next chunk has landed
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ __align__(16) float s_cum[4][kQ];  // ring of 4 chunks (E2 reads c & 3 while E1 writes ahead)
    __shared__ __align__(16) float s_dt[4][kQ];
    __shared__ __align__(16) float s_gam[192];
    __shared__ float s_wsum[kQ / 32];
    __shared__ float s_dt0[kQ / 32];  // dt of the first row of each quarter of the chunk
    volatile int* abort_flag = &s_abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int h = blockIdx.x;
    const int nseg = a.nseg;
    const int b = blockIdx.y / nseg;
    const int seg = blockIdx.y - b * nseg;
    const int H = a.H;
    const int G = a.G;
    const int g = h / (H / G);
    const int64_t HP = static_cast<int64_t>(H) * kP;
    const int64_t row0 = a.cu_seqlens ? static_cast<int64_t>(a.cu_seqlens[b]) : static_cast<int64_t>(b) * a.seqlen;
    const int T = a.cu_seqlens ? a.cu_seqlens[b + 1] - a.cu_seqlens[b] : a.seqlen;
    if (T <= 0) return;
    const int nchunks_seq = (T + kQ - 1) / kQ;
    const int nseg_s = segments_of(nchunks_seq, nseg, a.seg_chunks);
    const bool split = nseg_s > 1;
    if (seg >= nseg_s) return;
    const int c_begin = split ? seg * a.seg_chunks : 0;
    const int c_end = (split && seg < nseg_s - 1) ? c_begin + a.seg_chunks : nchunks_seq;
    const int nloc = c_end - c_begin;
    const int32_t slot = a.slot_idx[b];
    bf16_t* y = static_cast<bf16_t*>(a.y);
    if (slot < 0) {  // padding row: y = 0 over this segment's tokens, cache untouched
        const int64_t tb = static_cast<int64_t>(c_begin) * kQ;
        const int64_t te = min(static_cast<int64_t>(c_end) * kQ, static_cast<int64_t>(T));
        for (int64_t i = tb * (kP / 8) + tid; i < te * (kP / 8); i += kP2Threads) {
            const int64_t t = i / (kP / 8);
            *reinterpret_cast<uint4*>(y + (row0 + t) * a.y_stride + h * kP + (i % (kP / 8)) * 8) = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    if (slot >= a.num_slots) {
        if (tid == 0) record_error(a.error, M2_ERR_BAD_SLOT);
        return;
    }

    const uint32_t raw_addr = smem_addr(s_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* sm = s_raw + (base - raw_addr);
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(&s_tmem)),
                     "r"(kP2TmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    if (tid == 32) {
        s_abort = 0;
        for (int q = 0; q < 2; ++q) {
            mbar_init(&s_full[q], 1);
            mbar_init(&s_cb[q], 1);
            mbar_init(&s_m[q], 256);  // every epilogue-1 thread, once its rows of M are in TMEM
            mbar_init(&s_w[q], 256);
            mbar_init(&s_d[q], 1);
            mbar_init(&s_yoff[q], 1);
            mbar_init(&s_free[q], 1);
            mbar_init(&s_tfree[q], 256);  // every epilogue-2 thread, once it has read the stage's TMEM
        }
        mbar_init(&s_sready[0], 1);
        mbar_init(&s_sready[1], 1);
        mbar_init(&s_drain, 1);
        mbar_init(&s_mx, 1);
        mbar_init(&s_z, 1);
        fence_mbar_init();
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    const float A = -expf(a.A_log[h]);
    const float A2 = A * 1.4426950408889634f;
    const float dt_bias = a.dt_bias[h];
    const float Dh = a.D[h];
    const int xcol = h * kP;
    const int bcol = static_cast<int>(HP) + g * kN;
    const int ccol = static_cast<int>(HP) + G * kN + g * kN;
    float range_max = 0.f;
    __half2 hmax = __float2half2_rn(0.f);
    int loads_issued = 0;  // producer bookkeeping (lane 0 of warp 0)
    int z_issued = 0;      // z tiles issued (the mover)

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            for (int i = 0; i < nloc; ++i) {
                const int q = i & 1;
                if (i >= 2 && !p2_wait(&s_free[q], ((i >> 1) - 1) & 1, abort_flag)) {
                    s_abort = 1;
                    break;
                }
                const int ty = static_cast<int>(row0 + static_cast<int64_t>(c_begin + i) * kQ);
                const uint32_t st = base + q * kP2Stage;
                mbar_arrive_expect_tx(&s_full[q], 5u * 16384u);
                tma_load_2d(st + 65536, &tmap_x, xcol, ty, &s_full[q]);
                tma_load_2d(st + 32768, &tmap_x, bcol, ty, &s_full[q]);
                tma_load_2d(st + 32768 + 16384, &tmap_x, bcol + 64, ty, &s_full[q]);
                tma_load_2d(st, &tmap_x, ccol, ty, &s_full[q]);
                tma_load_2d(st + 16384, &tmap_x, ccol + 64, ty, &s_full[q]);
                ++loads_issued;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t id_cb = idesc_f16(128, 128, false, false);
            const uint32_t id_yoff = idesc_f16(128, 64, false, true);
            const uint32_t id_ydiag = idesc_f16(128, 64, false, true);
            const uint32_t id_ds = idesc_f16(128, 64, true, true);
            // CB = C . B^T of chunk j into stage j & 1, once its tiles have landed
            // and epilogue 2 is done with that stage's TMEM (chunk j - 2)
            auto issue_cb = [&](int j) -> bool {
                const int q = j & 1;
                bool ok = p2_wait(&s_full[q], (j >> 1) & 1, abort_flag);
                if (ok && j >= 1) ok = p2_wait(&s_mx, (j - 1) & 1, abort_flag);  // M of chunk j-1 read
                if (!ok) return false;
                tc_fence_after();
                const uint32_t st = base + q * kP2Stage;
                for (int k = 0; k < kN / 16; ++k) {
                    const uint32_t koff = (k >> 2) * 16384u + (k & 3) * 32u;
                    mma_f16(tmem, sw128_desc(st + koff, 16, 1024), sw128_desc(st + 32768 + koff, 16, 1024),
                            id_cb, k > 0);
                }
                mma_commit(&s_cb[q]);
                return true;
            };
            // Per chunk: C S^T as soon as the state entering it is ready (well
            // before epilogue 1 is done with M), then M X and W^T X, which free
            // the stage, then CB of the next chunk.
            bool ok = nloc <= 0 || issue_cb(0);
            for (int i = 0; ok && i < nloc; ++i) {
                const int q = i & 1;
                const uint32_t par = (i >> 1) & 1;
                const uint32_t st = base + q * kP2Stage;
                const uint32_t tq = tmem + 128 + q * 192;  // ring B: Ydiag, dS^T, Yoff
                // ring-B stage q: epilogue 2 has read chunk i - 2's
                if (i >= 2 && !p2_wait(&s_tfree[q], ((i >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
                // the state entering chunk i, in copy q
                if (!p2_wait(&s_sready[q], par, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int k = 0; k < kN / 16; ++k) {  // Yoff = C . S^T
                    const uint32_t koff = (k >> 2) * 16384u + (k & 3) * 32u;
                    mma_f16(tq + 128, sw128_desc(st + koff, 16, 1024),
                            sw128_desc(base + kP2OffS + k * 2048u, 16384, 1024), id_yoff, k > 0);
                }
                mma_commit(&s_yoff[q]);
                if (!p2_wait(&s_m[q], par, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int k = 0; k < kQ / 16; ++k)  // Ydiag = M . X (M from TMEM ring A), while W is built
                    mma_f16_ta(tq + 0, tmem + k * 16, sw128_desc(st + 65536 + k * 2048u, 16384, 1024), id_ydiag,
                               k > 0);
                mma_commit(&s_mx);
                if (!p2_wait(&s_w[q], par, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int k = 0; k < kQ / 16; ++k)  // dS^T = B^T . (w o X)
                    mma_f16(tq + 64, sw128_desc(st + 32768 + k * 2048u, 16384, 1024),
                            sw128_desc(base + kP2OffXw + k * 2048u, 16384, 1024), id_ds, k > 0);
                mma_commit(&s_d[q]);
                mma_commit(&s_free[q]);
                if (i + 1 < nloc && !issue_cb(i + 1)) { ok = false; break; }
            }
            if (!ok) s_abort = 1;
        }
    } else if (warp < 10) {
        // ------------------------------------------------------- epilogue 1
        const int e1 = tid - 64;
        const int quarter = warp & 3;           // TMEM lane quarter of this warp
        const int t = quarter * 32 + lane;      // row (token) of this thread
        const int h2 = e1 >> 7;                 // column half
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        // the next chunk's dt_raw stays in its bf16 bits until it is used, so the
        // load is waited for a chunk later, not where it is issued
        bf16_t dt_raw_next = 0;
        if (h2 == 0 && c_begin * kQ + t < T)
            dt_raw_next = static_cast<const bf16_t*>(a.dt)[(row0 + c_begin * kQ + t) * a.dt_stride + h];
        bool cb_fail = false;
        for (int i = 0; i < nloc; ++i) {
            const int c = c_begin + i;
            const int q = i & 1;
            const uint32_t par = (i >> 1) & 1;
            const int ring = i & 3;
            const int valid = min(kQ, T - c * kQ);
            // dt and the cumulative decay (log2 units) of chunk c
            float dt = 0.f, cum = 0.f;
            if (h2 == 0) {
                dt = (t < valid) ? softplus_f32(to_f32(dt_raw_next) + dt_bias) : 0.f;
                if (c + 1 < c_end && t < min(kQ, T - (c + 1) * kQ))
                    dt_raw_next = static_cast<const bf16_t*>(a.dt)[(row0 + (c + 1) * kQ + t) * a.dt_stride + h];
                cum = dt * A2;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float o = __shfl_up_sync(0xffffffffu, cum, off);
                    if (lane >= off) cum += o;
                }
                if (lane == 31) s_wsum[quarter] = cum;
                if (lane == 0) s_dt0[quarter] = dt;
            }
            // a failed wait of the previous chunk is decided here, by all together
            if (role_sync_or(1, cb_fail)) { s_abort = 1; break; }
            if (h2 == 0) {
                for (int w = 0; w < quarter; ++w) cum += s_wsum[w];
                s_cum[ring][t] = cum;
                s_dt[ring][t] = dt;
                // the factored decay of column t for the row quarters below it:
                // exp(c_32bq - c_t) dt_t, c_32bq summed in the same order as row 32bq's own
                for (int bq = quarter + 1; bq < 4; ++bq) {
                    float cq = s_dt0[bq] * A2;
                    for (int w = 0; w < bq; ++w) cq += s_wsum[w];
                    s_gam[(bq == 1 ? 0 : (bq == 2 ? 32 : 96)) + t] = ex2(cq - cum) * dt;
                }
            }
            role_sync_or(1, false);
            const float* cum_c = s_cum[ring];
            const float* dt_c = s_dt[ring];
            if (!p2_wait(&s_cb[q], par, abort_flag)) {  // the next chunk's first barrier decides
                s_abort = 1;
                cb_fail = true;
                continue;
            }
            tc_fence_after();
            const uint32_t ta = tmem;  // ring A: CB, then M in place
            const uint8_t* stX = sm + q * kP2Stage + 65536;
            const float cum_t = cum_c[t];
            const float cum_end = cum_c[kQ - 1];
            const int wq = quarter;
            const float alpha = ex2(cum_t - cum_c[32 * wq]);
            const float2 alpha2 = make_float2(alpha, alpha);
            const float* gam = s_gam + (wq == 1 ? 0 : (wq == 2 ? 32 : 96));
#pragma unroll 1
            for (int qb = 0; qb < 4; ++qb) {
                const int u0 = qb * 32 + 16 * h2;  // this thread's 16 columns of M
                float m[16];
                if (qb > wq) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) m[e] = 0.f;
                } else {
                    tmem_ld16(ta + lane_base + u0, m);
                    if (qb < wq) {
                        const float4* g4 = reinterpret_cast<const float4*>(gam + u0);
#pragma unroll
                        for (int i4 = 0; i4 < 4; ++i4) {
                            const float4 gv = g4[i4];
                            float2 lo = __fmul2_rn(make_float2(m[4 * i4], m[4 * i4 + 1]), make_float2(gv.x, gv.y));
                            float2 hi = __fmul2_rn(make_float2(m[4 * i4 + 2], m[4 * i4 + 3]), make_float2(gv.z, gv.w));
                            lo = __fmul2_rn(lo, alpha2);
                            hi = __fmul2_rn(hi, alpha2);
                            m[4 * i4] = lo.x;
                            m[4 * i4 + 1] = lo.y;
                            m[4 * i4 + 2] = hi.x;
                            m[4 * i4 + 3] = hi.y;
                        }
                    } else {
                        const float4* cu4 = reinterpret_cast<const float4*>(cum_c + u0);
                        const float4* du4 = reinterpret_cast<const float4*>(dt_c + u0);
                        const float2 ct2 = make_float2(cum_t, cum_t);
#pragma unroll
                        for (int i4 = 0; i4 < 4; ++i4) {
                            const float4 cu = cu4[i4], du = du4[i4];
#pragma unroll
                            for (int hp = 0; hp < 2; ++hp) {  // a pair of columns, packed
                                const float2 x = __fadd2_rn(ct2, hp ? make_float2(-cu.z, -cu.w) : make_float2(-cu.x, -cu.y));
                                float2 v = __fmul2_rn(make_float2(m[4 * i4 + 2 * hp], m[4 * i4 + 2 * hp + 1]),
                                                      make_float2(ex2(x.x), ex2(x.y)));
                                v = __fmul2_rn(v, hp ? make_float2(du.z, du.w) : make_float2(du.x, du.y));
                                const float vv[2] = {v.x, v.y};
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const int u = u0 + 4 * i4 + 2 * hp + e;
                                    float w = vv[e];
                                    if (u > t) w = 0.f;
                                    if (u == t) w += Dh;
                                    m[4 * i4 + 2 * hp + e] = w;
                                }
                            }
                        }
                    }
                }
                uint32_t hw[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const __half2 hv = __floats2half2_rn(m[2 * j], m[2 * j + 1]);
                    hmax = __hmax2(hmax, __habs2(hv));
                    hw[j] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                // M row t, columns u0 .. u0+15 as fp16 pairs, into the first 8 of
                // the 16 TMEM columns this thread read them from
                tmem_st8(ta + lane_base + u0, hw);
            }
            // this thread's rows of M are in TMEM: M . X may start while W is built
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive1(&s_m[q]);
            // (w o x) row t = w_t * x row t (fp16 pairs; this thread's 32 of the 64
            // channels) into the one w o x buffer, once dS of the previous chunk
            // has read it. B stays as loaded: dS^T = B^T (w o X) is the same sum
            // as W^T X with W = w o B, and x has half the elements of B.
            if (i >= 1 && !p2_wait(&s_d[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag)) {
                s_abort = 1;
                cb_fail = true;  // decided at the next chunk's first barrier
                continue;
            }
            const float wu = (t < valid) ? ex2(cum_end - cum_t) * dt_c[t] : 0.f;
            const __half2 w2 = __float2half2_rn(wu);
            hmax = __hmax2(hmax, __habs2(w2));
            // w <= 1 cannot take a finite fp16 x past the range: the products are
            // checked only where it is larger
            const bool wcheck = wu > 1.f;
            uint8_t* xw = sm + kP2OffXw;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = 4 * h2 + jj;
                uint4 v = *reinterpret_cast<const uint4*>(stX + sw128(t, j));
                uint32_t* vw = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half2 r2 = __hmul2(*reinterpret_cast<const __half2*>(&vw[e]), w2);
                    vw[e] = *reinterpret_cast<const uint32_t*>(&r2);
                }
                if (wcheck) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) hmax = __hmax2(hmax, __habs2(*reinterpret_cast<const __half2*>(&vw[e])));
                }
                *reinterpret_cast<uint4*>(xw + sw128(t, j)) = v;
            }
            // w o x visible to the tensor cores; the next chunk's first role barrier
            // orders this chunk's reads of s_gam and the decay sums before their reuse
            fence_proxy_async();
            mbar_arrive1(&s_w[q]);
        }
    } else if (warp == 18) {
        // --------------------------------------------------- y / z mover
        // Chunk c's y tile leaves (one TMA store, in place of its z tile) and
        // chunk c+1's z tile is loaded into the same buffer, once every
        // epilogue-2 thread is done with chunk c (its TMEM-free arrival), so
        // no epilogue-2 thread waits for the copies.
        if (lane == 0 && a.z != nullptr) {
            auto load_z = [&](int c) {
                mbar_arrive_expect_tx(&s_z, 16384u);
                tma_load_2d(base + kP2OffZ, &tmap_z, xcol, static_cast<int>(row0 + static_cast<int64_t>(c) * kQ),
                            &s_z);
                ++z_issued;
            };
            if (nloc > 0) load_z(c_begin);
            for (int i = 0; i < nloc; ++i) {
                const int c = c_begin + i;
                const bool ytile = T - c * kQ >= kQ;  // a whole chunk: y leaves as one tile
                if (!ytile && i + 1 >= nloc) break;
                if (!p2_wait(&s_tfree[i & 1], (i >> 1) & 1, abort_flag)) {
                    s_abort = 1;
                    break;
                }
                if (ytile) {
                    tma_store_2d(&tmap_y, xcol, static_cast<int>(row0 + static_cast<int64_t>(c) * kQ), base + kP2OffZ);
                    bulk_wait_read();  // the tile is read out before z of the next chunk lands in it
                }
                if (i + 1 < nloc) load_z(c + 1);
            }
        }
    } else {
        // ------------------------------------------------------- epilogue 2
        const int e2 = tid - 320;
        const int quarter = warp & 3;
        const int t = quarter * 32 + lane;   // row t (y) and state column n = t
        const int h2 = e2 >> 7;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        constexpr int kPH = kP / 2;
        const int n = t;
        const int p0 = h2 * kPH;
        ST* state = static_cast<ST*>(a.ssm) + (static_cast<int64_t>(slot) * HP + static_cast<int64_t>(h) * kP) * kN;
        float S[kPH];
        if (split) {
            const float* src = a.seg_state + ((static_cast<int64_t>(b) * nseg + seg) * H + h) * (kP * kN);
#pragma unroll
            for (int k = 0; k < kPH; ++k) S[k] = src[(p0 + k) * kN + n];
        } else {
            const bool init = a.has_init != nullptr && a.has_init[b] != 0;
#pragma unroll
            for (int k = 0; k < kPH; ++k) S[k] = init ? to_f32(state[(p0 + k) * kN + n]) : 0.f;
        }
        // fp16 copy of the state as the B operand of C S^T, n-major like the x
        // tile (row n: the 64 p values, 128-byte swizzle): four 16-byte stores
        auto write_state_copy = [&]() {
            uint8_t* sS = sm + kP2OffS;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half2 hv = __floats2half2_rn(S[8 * jj + 2 * e], S[8 * jj + 2 * e + 1]);
                    hmax = __hmax2(hmax, __habs2(hv));
                    w[e] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                *reinterpret_cast<uint4*>(sS + sw128(n, 4 * h2 + jj)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        };
        // the z tile of chunk c (128 tokens x 64 channels, 128-byte swizzle)
        // arrives by TMA in one shared buffer; the mover warp issues it
        const bool gate = a.z != nullptr;
        uint8_t* zt = sm + kP2OffZ;
        bool e2_fail = false;
        write_state_copy();
        fence_proxy_async();
        role_sync_or(2, false);
        if (e2 == 0) mbar_arrive1(&s_sready[0]);
        bool ok = true;
        for (int i = 0; i < nloc; ++i) {
            const int c = c_begin + i;
            const int q = i & 1;
            const uint32_t par = (i >> 1) & 1;
            const int ring = i & 3;
            const int t0 = c * kQ;
            const int valid = min(kQ, T - t0);
            // s_m: epilogue 1 of chunk c is done (its decay sums, read below, are
            // published by that release); s_d: dS and Ydiag are in TMEM
            bool got = p2_wait(&s_m[q], par, abort_flag);
            if (got) got = p2_wait(&s_d[q], par, abort_flag);
            // also decides, together, a failed wait of the previous chunk's y phase
            if (role_sync_or(2, !got || e2_fail)) { s_abort = 1; ok = false; break; }
            tc_fence_after();
            const uint32_t tq = tmem + 128 + q * 192;
            {
                const float eend = ex2(s_cum[ring][kQ - 1]);
                float ds[32];
                tmem_ld32(tq + lane_base + 64 + p0, ds);
#pragma unroll
                for (int k = 0; k < kPH; k += 2) {
                    const float2 r = __ffma2_rn(make_float2(eend, eend), make_float2(S[k], S[k + 1]),
                                                make_float2(ds[k], ds[k + 1]));
                    S[k] = r.x;
                    S[k + 1] = r.y;
                }
            }
            // the state leaving chunk c, for C S^T of chunk c+1, in the one copy:
            // its last reader, C S^T of chunk c, was issued before dS of chunk c
            // and has completed with it (s_d, above)
            if (i + 1 < nloc) {
                write_state_copy();
                fence_proxy_async();
                role_sync_or(2, false);
                if (e2 == 0) mbar_arrive1(&s_sready[(i + 1) & 1]);
            }
            got = p2_wait(&s_yoff[q], par, abort_flag);
            if (got && gate) got = p2_wait(&s_z, i & 1, abort_flag);
            if (!got) {  // decided at the next chunk's first barrier
                s_abort = 1;
                e2_fail = true;
                ok = false;
                continue;
            }
            tc_fence_after();
            const float et = ex2(s_cum[ring][t]);
            const bool row_ok = t < valid;
            // a whole chunk with a gate: y goes in place of z into the tile and
            // out as one TMA store (a partial chunk's rows past the sequence are
            // another sequence's, so those chunks store row by row)
            const bool ytile = gate && valid == kQ;
            bf16_t* yrow = y + (row0 + t0 + t) * a.y_stride + xcol;
            const float2 et2 = make_float2(et, et);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float yd[16], yo[16];
                tmem_ld16x2(tq + lane_base + h2 * 32 + 16 * hh, tq + lane_base + 128 + h2 * 32 + 16 * hh, yd, yo);
#pragma unroll
                for (int jh = 0; jh < 2; ++jh) {
                    const int jj = 2 * hh + jh;
                    float out[8];
                    float zv[8];
                    if (gate) unpack16<bf16_t>(*reinterpret_cast<const uint4*>(zt + sw128(t, 4 * h2 + jj)), zv);
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        float2 v = __ffma2_rn(et2, make_float2(yo[8 * jh + e], yo[8 * jh + e + 1]),
                                              make_float2(yd[8 * jh + e], yd[8 * jh + e + 1]));
                        if (gate) v = __fmul2_rn(v, silu2_tanh(zv[e], zv[e + 1]));
                        out[e] = v.x;
                        out[e + 1] = v.y;
                    }
                    if (ytile)
                        *reinterpret_cast<uint4*>(zt + sw128(t, 4 * h2 + jj)) = pack16<bf16_t>(out);
                    else if (row_ok)
                        *reinterpret_cast<uint4*>(yrow + 8 * (h2 * 4 + jj)) = pack16<bf16_t>(out);
                }
            }
            if (ytile) fence_proxy_async();  // the y tile, for the TMA store
            // this thread has read TMEM stage q and the z tile (and written its y
            // rows): chunk c+2 may reuse the stage, the tile may go out and chunk
            // c+1's z land, once all have
            tc_fence_before();
            mbar_arrive1(&s_tfree[q]);
        }
        if (ok && (!split || seg == nseg_s - 1)) {  // the sequence's final state, in place
#pragma unroll
            for (int k = 0; k < kPH; ++k) state[(p0 + k) * kN + n] = from_f32<ST>(S[k]);
        }
    }

    // every role is done (or aborted): settle outstanding MMAs and copies, free TMEM
    if (tid == 32) {  // the MMA issuer: one more commit arrives once all its MMAs have completed
        mma_commit(&s_drain);
        mbar_wait_bounded(&s_drain, 0, kLimitNs);
    }
    if (tid == 0) {  // the producer: the last load of each stage has landed
        for (int q = 0; q < 2; ++q) {
            const int uses = (loads_issued - q + 1) / 2;
            if (uses > 0) mbar_wait_bounded(&s_full[q], (uses - 1) & 1, kLimitNs);
        }
    }
    if (tid == 576) {  // the mover: the last z tile has landed and the last y tile has been read out
        if (z_issued > 0) mbar_wait_bounded(&s_z, (z_issued - 1) & 1, kLimitNs);
        bulk_wait_read();
    }
    __syncthreads();
    range_max = fmaxf(range_max, fmaxf(__low2float(hmax), __high2float(hmax)));
    if (s_abort) {
        if (tid == 0) record_error(a.error, M2_ERR_TIMEOUT);
    } else if (range_max >= kF16Limit) {
        record_error(a.error, M2_ERR_RANGE);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kP2TmemCols) : "memory");
    }
}

}  // namespace

TensorMapEncodeFn tensor_map_encoder() {
    static std::once_flag once;
    static TensorMapEncodeFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TensorMapEncodeFn>(p);
        cudaGetLastError();
    });
    return fn;
}

bool chunk_scan_tc_supported(const ScanArgs& a) {
    return a.P == kP && a.N == kN && a.state_bf16 && a.act_bf16 &&
           (a.x_dtype == M2_BF16 || a.x_dtype == M2_F16) && (a.xBC_stride * 2) % 16 == 0;
}

// Combine pass of a split sequence (CUDA cores, fp32): scratch slot 0 <- the
// initial state (the cache's, or zero), then slot j+1 <- decay_j * slot j +
// slot j+1, where slot j+1 held segment j's summary (its final state from a
// zero start). Afterwards slot j is the state entering segment j.
template <typename ST>
__global__ void __launch_bounds__(256) seg_combine_kernel(const ScanArgs a) {
    constexpr int kPN = kP * kN;
    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int H = a.H;
    const int T = a.cu_seqlens ? a.cu_seqlens[b + 1] - a.cu_seqlens[b] : a.seqlen;
    const int nseg_s = segments_of((T + kQ - 1) / kQ, a.nseg, a.seg_chunks);
    if (nseg_s <= 1) return;
    const int32_t slot = a.slot_idx[b];
    if (slot < 0 || slot >= a.num_slots) return;  // the scan pass handles both
    const bool init = a.has_init != nullptr && a.has_init[b] != 0;
    const ST* st = static_cast<const ST*>(a.ssm) +
                   (static_cast<int64_t>(slot) * H + h) * static_cast<int64_t>(kPN);
    float* slot0 = a.seg_state + (static_cast<int64_t>(b) * a.nseg * H + h) * kPN;
    const int64_t slot_stride = static_cast<int64_t>(H) * kPN;
    const float* decay = a.seg_decay + static_cast<int64_t>(b) * a.nseg * H + h;
    for (int e = threadIdx.x; e < kPN; e += blockDim.x) {
        float v = init ? to_f32(st[e]) : 0.f;
        slot0[e] = v;
        for (int j = 0; j + 1 < nseg_s; ++j) {
            float* nxt = slot0 + (j + 1) * slot_stride + e;
            v = fmaf(decay[static_cast<int64_t>(j) * H], v, *nxt);
            *nxt = v;
        }
    }
}

cudaError_t launch_chunk_scan_tc(const ScanArgs& a, cudaStream_t stream) {
    TensorMapEncodeFn enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    // xBC as a 2-D tensor (channel, packed token row), 64 x 128 boxes of 16-bit
    // elements, 128-byte swizzle; rows past the end of the buffer read as zeros
    CUtensorMap map;
    const int64_t cd = static_cast<int64_t>(a.H) * a.P + 2LL * a.G * a.N;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cd), static_cast<cuuint64_t>(a.total_tokens)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.xBC_stride) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kQ)};
    const cuuint32_t estr[2] = {1, 1};
    const bool f16_in = a.x_dtype == M2_F16;
    if (enc(&map, f16_in ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(a.xBC), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    static AttrOnce attrs;
    const cudaError_t attr_err = attrs.ensure([] {
        const void* kerns[4] = {
            reinterpret_cast<const void*>(chunk_scan_tc_kernel<bf16_t, f16_t, false>),
            reinterpret_cast<const void*>(chunk_scan_tc_kernel<bf16_t, bf16_t, false>),
            reinterpret_cast<const void*>(chunk_scan_tc_kernel<bf16_t, f16_t, true>),
            reinterpret_cast<const void*>(chunk_scan_tc_kernel<bf16_t, bf16_t, true>)};
        for (const void* k : kerns) {
            const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       static_cast<int>(kSmemBytes));
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int nseg = a.nseg > 1 ? a.nseg : 1;
    const dim3 grid(static_cast<unsigned>(a.H), static_cast<unsigned>(a.batch) * static_cast<unsigned>(nseg));
    if (nseg > 1) {  // pass 1: segment summaries; pass 2: carry them across segments
        auto summ = f16_in ? chunk_scan_tc_kernel<bf16_t, f16_t, true> : chunk_scan_tc_kernel<bf16_t, bf16_t, true>;
        summ<<<grid, kTC, kSmemBytes, stream>>>(map, a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        seg_combine_kernel<bf16_t><<<dim3(static_cast<unsigned>(a.H), static_cast<unsigned>(a.batch)), 256, 0,
                                     stream>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
#if M2_SCAN_PIPELINED
    if (f16_in) {  // the pipelined, warp-specialised scan (one CTA per SM)
        static AttrOnce attrs_p2;
        const cudaError_t e = attrs_p2.ensure([] {
            return cudaFuncSetAttribute(chunk_scan_p2_kernel<bf16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kP2Smem));
        });
        if (e != cudaSuccess) return e;
        // z (bf16) as (channel, packed token row), boxes of 64 x 128, 128-byte swizzle
        CUtensorMap map_z{};
        if (a.z) {
            const cuuint64_t zd[2] = {static_cast<cuuint64_t>(a.H) * kP, static_cast<cuuint64_t>(a.total_tokens)};
            const cuuint64_t zs[1] = {static_cast<cuuint64_t>(a.z_stride) * 2};
            const cuuint32_t zb[2] = {64, static_cast<cuuint32_t>(kQ)};
            if (enc(&map_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.z), zd, zs, zb, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        // y (bf16), the same boxes, for the TMA stores of whole gated chunks
        CUtensorMap map_y{};
        if (a.z) {
            const cuuint64_t yd[2] = {static_cast<cuuint64_t>(a.H) * kP, static_cast<cuuint64_t>(a.total_tokens)};
            const cuuint64_t ys[1] = {static_cast<cuuint64_t>(a.y_stride) * 2};
            const cuuint32_t yb[2] = {64, static_cast<cuuint32_t>(kQ)};
            if (enc(&map_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.y, yd, ys, yb, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        chunk_scan_p2_kernel<bf16_t><<<grid, kP2Threads, kP2Smem, stream>>>(map, map_z, map_y, a);
        return cudaGetLastError();
    }
#endif
    auto kern = f16_in ? chunk_scan_tc_kernel<bf16_t, f16_t, false> : chunk_scan_tc_kernel<bf16_t, bf16_t, false>;
    kern<<<grid, kTC, kSmemBytes, stream>>>(map, a);
    return cudaGetLastError();
}

}  // namespace m2
