// m2_api.cu -- the extern "C" entry points of libm2 (include/m2.h).
//
// Host-side only: argument validation, launch planning and error mapping. No
// entry point on the hot path allocates, synchronises or reads device memory
// on the host (the allocator and the error query are not hot-path calls).
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "m2_internal.cuh"

namespace {

// Storage dtypes of caches and activations; the post-conv buffer may also be fp16.
bool valid_dtype(int32_t d) { return d == M2_F32 || d == M2_BF16; }
bool valid_buffer_dtype(int32_t d) { return valid_dtype(d) || d == M2_F16; }
int dsize(int32_t d) { return d == M2_F32 ? 4 : 2; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride_ok(int64_t stride_elems, int elem_size, int64_t min_elems) {
    return stride_elems >= min_elems && (stride_elems * elem_size) % 16 == 0;
}

m2_status shape_status(const m2_shape* s) {
    if (!s) return M2_ERR_INVALID_ARG;
    if (s->nheads <= 0 || s->head_dim <= 0 || s->d_state <= 0 || s->ngroups <= 0 || s->d_conv <= 0)
        return M2_ERR_INVALID_ARG;
    if (s->nheads % s->ngroups != 0) return M2_ERR_INVALID_ARG;
    if (!valid_dtype(s->state_dtype) || !valid_dtype(s->act_dtype)) return M2_ERR_INVALID_ARG;
    if (s->d_conv < 2 || s->d_conv > 8) return M2_ERR_UNSUPPORTED;
    const int a = dsize(s->act_dtype);
    const int64_t hp = static_cast<int64_t>(s->nheads) * s->head_dim;
    const int64_t gn = static_cast<int64_t>(s->ngroups) * s->d_state;
    // 16-byte vectors must tile the x, B and C segments of a row
    if ((hp * a) % 16 != 0 || (gn * a) % 16 != 0 || (static_cast<int64_t>(s->head_dim) * a) % 16 != 0)
        return M2_ERR_UNSUPPORTED;
    m2::DecodePlan plan;
    return m2::plan_state_update(s->nheads, s->head_dim, s->d_state, s->ngroups,
                                 s->state_dtype == M2_BF16, 0, &plan);
}

m2_status cache_status(const m2_cache* c) {
    if (!c || !c->ssm || !c->conv || c->num_slots <= 0) return M2_ERR_INVALID_ARG;
    return shape_status(&c->shape);
}

m2_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return M2_OK;
    if (e == cudaErrorMemoryAllocation) return M2_ERR_OOM;
    return M2_ERR_CUDA;
}

// M2_VALIDATE=1: copy the slot indices to the host (synchronising) and reject
// duplicates. Debug aid only; never used on a captured stream.
bool validate_mode() {
    const char* v = std::getenv("M2_VALIDATE");
    return v && v[0] == '1';
}

m2_status validate_slots(const int32_t* slot_idx, int32_t n, int64_t num_slots, cudaStream_t s) {
    std::vector<int32_t> h(static_cast<size_t>(n));
    if (cudaMemcpyAsync(h.data(), slot_idx, sizeof(int32_t) * n, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return M2_ERR_CUDA;
    std::vector<char> seen(static_cast<size_t>(num_slots), 0);
    for (int32_t v : h) {
        if (v < 0 || v >= num_slots) continue;  // padding / device-reported
        if (seen[v]) return M2_ERR_INVALID_ARG;
        seen[v] = 1;
    }
    return M2_OK;
}

}  // namespace

extern "C" {

int64_t m2_conv_dim(const m2_shape* s) {
    if (!s || s->nheads <= 0 || s->head_dim <= 0 || s->d_state <= 0 || s->ngroups <= 0) return -1;
    return static_cast<int64_t>(s->nheads) * s->head_dim + 2LL * s->ngroups * s->d_state;
}

m2_status m2_shape_check(const m2_shape* s) { return shape_status(s); }

m2_status m2_cache_bytes(const m2_shape* s, int64_t num_slots, int64_t* ssm_bytes,
                         int64_t* conv_bytes) {
    const m2_status st = shape_status(s);
    if (st == M2_ERR_INVALID_ARG) return st;
    if (num_slots <= 0) return M2_ERR_INVALID_ARG;
    const int64_t per_ssm = static_cast<int64_t>(s->nheads) * s->head_dim * s->d_state * dsize(s->state_dtype);
    const int64_t per_conv = static_cast<int64_t>(s->d_conv - 1) * m2_conv_dim(s) * dsize(s->act_dtype);
    if (ssm_bytes) *ssm_bytes = per_ssm * num_slots;
    if (conv_bytes) *conv_bytes = per_conv * num_slots;
    return M2_OK;
}

m2_status m2_cache_alloc(const m2_shape* s, int64_t num_slots, m2_stream stream, m2_cache* out) {
    if (!out) return M2_ERR_INVALID_ARG;
    const m2_status st = shape_status(s);
    if (st != M2_OK) return st;
    int64_t ssm_b = 0, conv_b = 0;
    if (m2_cache_bytes(s, num_slots, &ssm_b, &conv_b) != M2_OK) return M2_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return M2_ERR_CUDA;
    void* ssm = nullptr;
    void* conv = nullptr;
    void* err = nullptr;
    cudaError_t e = cudaMalloc(&ssm, static_cast<size_t>(ssm_b));
    if (e == cudaSuccess) e = cudaMalloc(&conv, static_cast<size_t>(conv_b));
    if (e == cudaSuccess) e = cudaMalloc(&err, sizeof(int32_t));
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(ssm, 0, static_cast<size_t>(ssm_b), cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(conv, 0, static_cast<size_t>(conv_b), cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(err, 0, sizeof(int32_t), cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) {
        cudaFree(ssm);
        cudaFree(conv);
        cudaFree(err);
        cudaGetLastError();
        return from_cuda(e);
    }
    std::memset(out, 0, sizeof(*out));
    out->ssm = ssm;
    out->conv = conv;
    out->error = static_cast<int32_t*>(err);
    out->num_slots = num_slots;
    out->shape = *s;
    out->owned = 1;
    out->device = dev;
    return M2_OK;
}

m2_status m2_cache_wrap(const m2_shape* s, int64_t num_slots, void* ssm, void* conv,
                        int32_t* error_word, m2_cache* out) {
    if (!out || !ssm || !conv || num_slots <= 0) return M2_ERR_INVALID_ARG;
    if (!aligned16(ssm) || !aligned16(conv)) return M2_ERR_INVALID_ARG;
    if (error_word && (reinterpret_cast<uintptr_t>(error_word) & 3u)) return M2_ERR_INVALID_ARG;
    const m2_status st = shape_status(s);
    if (st != M2_OK) return st;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaGetLastError();
    std::memset(out, 0, sizeof(*out));
    out->ssm = ssm;
    out->conv = conv;
    out->error = error_word;
    out->num_slots = num_slots;
    out->shape = *s;
    out->owned = 0;
    out->device = dev;
    return M2_OK;
}

m2_status m2_cache_free(m2_cache* c, m2_stream stream) {
    if (!c) return M2_ERR_INVALID_ARG;
    m2_status st = M2_OK;
    if (c->owned) {
        if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) st = M2_ERR_CUDA;
        cudaFree(c->ssm);
        cudaFree(c->conv);
        cudaFree(c->error);
    }
    std::memset(c, 0, sizeof(*c));
    return st;
}

m2_status m2_cache_zero_slots(const m2_cache* c, int32_t n, const int32_t* slot_idx, m2_stream stream) {
    const m2_status st = cache_status(c);
    if (st != M2_OK) return st;
    if (n < 0 || (n > 0 && !slot_idx)) return M2_ERR_INVALID_ARG;
    if (n == 0) return M2_OK;
    m2::ZeroArgs a{};
    a.ssm = c->ssm;
    a.conv = c->conv;
    a.error = c->error;
    a.num_slots = c->num_slots;
    m2_cache_bytes(&c->shape, 1, &a.ssm_bytes_per_slot, &a.conv_bytes_per_slot);
    a.n = n;
    a.slot_idx = slot_idx;
    return from_cuda(m2::launch_zero_slots(a, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {

m2_status conv1d_impl(const m2_cache* c, const m2_conv_params* conv, int32_t batch, int32_t seqlen,
                      const int32_t* cu_seqlens, int64_t total_rows, const void* xBC, int64_t xBC_row_stride,
                      void* xBC_out,
                      int32_t out_dtype, int64_t out_row_stride, const int32_t* slot_idx, m2_stream stream) {
    const m2_status st = cache_status(c);
    if (st != M2_OK) return st;
    if (!conv || !conv->weight || batch < 0 || seqlen < 0 || !valid_buffer_dtype(out_dtype))
        return M2_ERR_INVALID_ARG;
    if (conv->activation != 0 && conv->activation != 1) return M2_ERR_INVALID_ARG;
    if (batch == 0 || seqlen == 0) return M2_OK;
    if (!xBC || !xBC_out || !slot_idx) return M2_ERR_INVALID_ARG;
    const m2_shape& s = c->shape;
    const int64_t cd = m2_conv_dim(&s);
    const int as = dsize(s.act_dtype);
    if (!aligned16(xBC) || !aligned16(xBC_out) || !stride_ok(xBC_row_stride, as, cd) ||
        !stride_ok(out_row_stride, dsize(out_dtype), cd) || !aligned16(conv->weight) ||
        (conv->bias && !aligned16(conv->bias)))
        return M2_ERR_INVALID_ARG;
    if (validate_mode()) {
        const m2_status v = validate_slots(slot_idx, batch, c->num_slots, reinterpret_cast<cudaStream_t>(stream));
        if (v != M2_OK) return v;
    }
    m2::ConvArgs a{};
    a.conv = c->conv;
    a.error = c->error;
    a.num_slots = c->num_slots;
    a.K = s.d_conv;
    a.conv_dim = cd;
    a.act_bf16 = s.act_dtype == M2_BF16;
    a.out_dtype = out_dtype;
    a.w = conv->weight;
    a.b = conv->bias;
    a.activation = conv->activation;
    a.batch = batch;
    a.seqlen = seqlen;
    a.x = xBC;
    a.x_stride = xBC_row_stride;
    a.out = xBC_out;
    a.out_stride = out_row_stride;
    a.slot_idx = slot_idx;
    a.cu_seqlens = cu_seqlens;
    a.total_rows = total_rows;
    return from_cuda(m2::launch_conv1d_update(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

m2_status m2_conv1d_update(const m2_cache* c, const m2_conv_params* conv, int32_t batch, int32_t seqlen,
                           const void* xBC, int64_t xBC_row_stride, void* xBC_out, int32_t out_dtype,
                           int64_t out_row_stride, const int32_t* slot_idx, m2_stream stream) {
    return conv1d_impl(c, conv, batch, seqlen, nullptr, static_cast<int64_t>(batch) * seqlen, xBC, xBC_row_stride,
                       xBC_out, out_dtype, out_row_stride, slot_idx, stream);
}

m2_status m2_conv1d_update_varlen(const m2_cache* c, const m2_conv_params* conv, int32_t nseq,
                                  const int32_t* cu_seqlens, int64_t total_tokens, int32_t max_seqlen,
                                  const void* xBC, int64_t xBC_row_stride, void* xBC_out, int32_t out_dtype,
                                  int64_t out_row_stride, const int32_t* slot_idx, m2_stream stream) {
    if (nseq < 0 || total_tokens < 0 || max_seqlen < 0) return M2_ERR_INVALID_ARG;
    if (total_tokens > INT32_MAX) return M2_ERR_UNSUPPORTED;
    if (nseq > 0 && total_tokens > 0 && !cu_seqlens) return M2_ERR_INVALID_ARG;
    // no tokens: validate and return, as a zero-length fixed call does
    const int32_t len = (nseq == 0 || total_tokens == 0) ? 0 : std::max(max_seqlen, 1);
    return conv1d_impl(c, conv, nseq, len, cu_seqlens, total_tokens, xBC, xBC_row_stride, xBC_out, out_dtype,
                       out_row_stride, slot_idx, stream);
}

namespace {

// check_only: validate the arguments and the launch plan, enqueue nothing.
m2_status state_update_impl(const m2_cache* c, const m2_ssm_params* ssm, const m2_conv_params* conv,
                            const m2_norm_params* norm, int32_t batch, const void* xBC, int32_t xBC_dtype,
                            int64_t xBC_row_stride, const void* dt, int64_t dt_row_stride, const void* z,
                            int64_t z_row_stride, void* y, int64_t y_row_stride, const int32_t* slot_idx,
                            m2_stream stream, bool check_only = false) {
    const m2_status st = cache_status(c);
    if (st != M2_OK) return st;
    if (!ssm || !ssm->A_log || !ssm->dt_bias || !ssm->D || batch < 0 || !valid_buffer_dtype(xBC_dtype))
        return M2_ERR_INVALID_ARG;
    if (batch == 0) return M2_OK;
    if (!xBC || !dt || !y || !slot_idx) return M2_ERR_INVALID_ARG;
    const m2_shape& s = c->shape;
    const int as = dsize(s.act_dtype);
    const int64_t cd = m2_conv_dim(&s);
    const int64_t hp = static_cast<int64_t>(s.nheads) * s.head_dim;
    if (conv) {
        if (!conv->weight || (conv->activation != 0 && conv->activation != 1)) return M2_ERR_INVALID_ARG;
        if (!aligned16(conv->weight) || (conv->bias && !aligned16(conv->bias))) return M2_ERR_INVALID_ARG;
        if (xBC_dtype != s.act_dtype) return M2_ERR_INVALID_ARG;
    }
    if (!aligned16(xBC) || !aligned16(y) || !stride_ok(xBC_row_stride, dsize(xBC_dtype), cd) ||
        !stride_ok(y_row_stride, as, hp) || dt_row_stride < s.nheads)
        return M2_ERR_INVALID_ARG;
    if (z && (!aligned16(z) || !stride_ok(z_row_stride, as, hp))) return M2_ERR_INVALID_ARG;
    if (norm) {  // the fused launch's group cluster carries the norm's reduction
        if (!conv) return M2_ERR_UNSUPPORTED;
        if (!norm->weight || !aligned16(norm->weight) || !(norm->eps >= 0.f)) return M2_ERR_INVALID_ARG;
    }
    m2::DecodePlan plan;
    const m2_status ps = m2::plan_state_update(s.nheads, s.head_dim, s.d_state, s.ngroups,
                                               s.state_dtype == M2_BF16, conv != nullptr, &plan);
    if (ps != M2_OK) return ps;
    if (check_only) return M2_OK;
    if (validate_mode()) {
        const m2_status v = validate_slots(slot_idx, batch, c->num_slots, reinterpret_cast<cudaStream_t>(stream));
        if (v != M2_OK) return v;
    }
    m2::StateUpdateArgs a{};
    a.ssm = c->ssm;
    a.conv = c->conv;
    a.error = c->error;
    a.num_slots = c->num_slots;
    a.H = s.nheads;
    a.P = s.head_dim;
    a.N = s.d_state;
    a.G = s.ngroups;
    a.K = s.d_conv;
    a.conv_dim = cd;
    a.state_bf16 = s.state_dtype == M2_BF16;
    a.act_bf16 = s.act_dtype == M2_BF16;
    a.x_dtype = xBC_dtype;
    a.A_log = ssm->A_log;
    a.dt_bias = ssm->dt_bias;
    a.D = ssm->D;
    a.conv_w = conv ? conv->weight : nullptr;
    a.conv_b = conv ? conv->bias : nullptr;
    a.activation = conv ? conv->activation : 0;
    a.fused = conv != nullptr;
    a.batch = batch;
    a.xBC = xBC;
    a.xBC_stride = xBC_row_stride;
    a.dt = dt;
    a.dt_stride = dt_row_stride;
    a.z = z;
    a.z_stride = z_row_stride;
    a.y = y;
    a.y_stride = y_row_stride;
    a.slot_idx = slot_idx;
    a.norm_w = norm ? norm->weight : nullptr;
    a.norm_eps = norm ? norm->eps : 0.f;
    return from_cuda(m2::launch_state_update(a, plan, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

m2_status m2_state_update(const m2_cache* c, const m2_ssm_params* ssm, const m2_conv_params* conv,
                          int32_t batch, const void* xBC, int32_t xBC_dtype, int64_t xBC_row_stride,
                          const void* dt, int64_t dt_row_stride, const void* z, int64_t z_row_stride,
                          void* y, int64_t y_row_stride, const int32_t* slot_idx, m2_stream stream) {
    return state_update_impl(c, ssm, conv, nullptr, batch, xBC, xBC_dtype, xBC_row_stride, dt, dt_row_stride, z,
                             z_row_stride, y, y_row_stride, slot_idx, stream);
}

m2_status m2_state_update_norm(const m2_cache* c, const m2_ssm_params* ssm, const m2_conv_params* conv,
                               const m2_norm_params* norm, int32_t batch, const void* xBC,
                               int64_t xBC_row_stride, const void* dt, int64_t dt_row_stride, const void* z,
                               int64_t z_row_stride, void* y, int64_t y_row_stride, const int32_t* slot_idx,
                               m2_stream stream) {
    if (!norm || !conv) return M2_ERR_INVALID_ARG;
    const m2_status st = cache_status(c);
    if (st != M2_OK) return st;
    return state_update_impl(c, ssm, conv, norm, batch, xBC, c->shape.act_dtype, xBC_row_stride, dt,
                             dt_row_stride, z, z_row_stride, y, y_row_stride, slot_idx, stream);
}

namespace {

// Shared by the fixed-length and the variable-length scan entry points:
// validation and argument marshalling (cu_seqlens NULL: [batch, seqlen] rows).
m2_status scan_args(const m2_cache* c, const m2_ssm_params* ssm, int32_t batch, int32_t chunk_size,
                    const void* xBC, int32_t xBC_dtype, int64_t xBC_row_stride, const void* dt,
                    int64_t dt_row_stride, const void* z, int64_t z_row_stride, void* y, int64_t y_row_stride,
                    const int32_t* slot_idx, const uint8_t* has_initial_state, m2_stream stream,
                    m2::ScanArgs* out) {
    const m2_status st = cache_status(c);
    if (st != M2_OK) return st;
    if (!ssm || !ssm->A_log || !ssm->dt_bias || !ssm->D || batch < 0 || chunk_size <= 0 ||
        !valid_buffer_dtype(xBC_dtype))
        return M2_ERR_INVALID_ARG;
    if (!xBC || !dt || !y || !slot_idx) return M2_ERR_INVALID_ARG;
    const m2_shape& s = c->shape;
    const int as = dsize(s.act_dtype);
    const int64_t cd = m2_conv_dim(&s);
    const int64_t hp = static_cast<int64_t>(s.nheads) * s.head_dim;
    if (!aligned16(xBC) || !aligned16(y) || !stride_ok(xBC_row_stride, dsize(xBC_dtype), cd) ||
        !stride_ok(y_row_stride, as, hp) || dt_row_stride < s.nheads)
        return M2_ERR_INVALID_ARG;
    if (z && (!aligned16(z) || !stride_ok(z_row_stride, as, hp))) return M2_ERR_INVALID_ARG;
    const m2_status ps = m2::plan_chunk_scan(s.nheads, s.head_dim, s.d_state, s.ngroups, chunk_size);
    if (ps != M2_OK) return ps;
    if (validate_mode()) {
        const m2_status v = validate_slots(slot_idx, batch, c->num_slots, reinterpret_cast<cudaStream_t>(stream));
        if (v != M2_OK) return v;
    }
    m2::ScanArgs a{};
    a.ssm = c->ssm;
    a.error = c->error;
    a.num_slots = c->num_slots;
    a.H = s.nheads;
    a.P = s.head_dim;
    a.N = s.d_state;
    a.G = s.ngroups;
    a.state_bf16 = s.state_dtype == M2_BF16;
    a.act_bf16 = s.act_dtype == M2_BF16;
    a.x_dtype = xBC_dtype;
    a.A_log = ssm->A_log;
    a.dt_bias = ssm->dt_bias;
    a.D = ssm->D;
    a.batch = batch;
    a.chunk = chunk_size;
    a.xBC = xBC;
    a.xBC_stride = xBC_row_stride;
    a.dt = dt;
    a.dt_stride = dt_row_stride;
    a.z = z;
    a.z_stride = z_row_stride;
    a.y = y;
    a.y_stride = y_row_stride;
    a.slot_idx = slot_idx;
    a.has_init = has_initial_state;
    a.nseg = 1;
    *out = a;
    return M2_OK;
}

// The split scan's stream-ordered memory pool on the current device, created
// once per device. It keeps freed memory (release threshold: never), so after
// the first split call on a device the scratch costs no driver allocation;
// the device's default pool, whose memory goes back to the driver at every
// synchronisation, cost up to milliseconds per call.
cudaError_t scratch_pool(cudaMemPool_t* out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static cudaMemPool_t pools[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (pools[dev] == nullptr) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        e = cudaMemPoolCreate(&p, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = UINT64_MAX;
        e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) {
            cudaMemPoolDestroy(p);
            return e;
        }
        pools[dev] = p;
    }
    *out = pools[dev];
    return cudaSuccess;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        n = 148;
    return n > 0 ? n : 148;
}

// Split plan of a variable-length scan (tensor-core path). The scan of a
// chunk is latency-bound inside its CTA: on B200 a CTA alone on its SM takes
// about 5.6 us per 128-token chunk, two CTAs sharing an SM about 8.7 us each,
// and the summary pass of a split about 4.9 us per chunk. Splitting therefore
// only pays when whole extra SMs can be put to work: sequences are cut into
// nseg segments so that the (sequence, segment, head) CTAs of the scan pass
// are at most one per SM, and only when at least three segments fit. Returns
// the scratch bytes (state slots, then decays; 0 without a split) and sets
// a->nseg / a->seg_chunks.
size_t plan_split(m2::ScanArgs* a, int32_t nseq, int32_t max_seqlen, size_t* state_bytes) {
    a->nseg = 1;
    a->seg_chunks = 0;
    *state_bytes = 0;
    const int64_t pairs = static_cast<int64_t>(nseq) * a->H;
    const int max_chunks = (max_seqlen + 127) / 128;
    if (!m2::chunk_scan_tc_supported(*a) || pairs <= 0 || max_chunks < 3) return 0;
    int nseg = static_cast<int>(std::min<int64_t>({sm_count() / pairs, max_chunks, 64}));
    if (nseg < 3) return 0;
    const int seg_chunks = (max_chunks + nseg - 1) / nseg;
    nseg = (max_chunks + seg_chunks - 1) / seg_chunks;
    if (nseg <= 1) return 0;
    a->nseg = nseg;
    a->seg_chunks = seg_chunks;
    *state_bytes = static_cast<size_t>(nseq) * nseg * a->H * a->P * a->N * sizeof(float);
    return *state_bytes + static_cast<size_t>(nseq) * nseg * a->H * sizeof(float);
}

}  // namespace

m2_status m2_chunk_scan(const m2_cache* c, const m2_ssm_params* ssm, int32_t batch, int32_t seqlen,
                        int32_t chunk_size, const void* xBC, int32_t xBC_dtype, int64_t xBC_row_stride,
                        const void* dt, int64_t dt_row_stride, const void* z, int64_t z_row_stride,
                        void* y, int64_t y_row_stride, const int32_t* slot_idx,
                        const uint8_t* has_initial_state, m2_stream stream) {
    if (seqlen < 0 || batch < 0) return M2_ERR_INVALID_ARG;
    if (batch == 0 || seqlen == 0) {
        const m2_status st = cache_status(c);
        return st != M2_OK ? st : (ssm && chunk_size > 0 ? M2_OK : M2_ERR_INVALID_ARG);
    }
    if (static_cast<int64_t>(batch) * seqlen > INT32_MAX) return M2_ERR_UNSUPPORTED;
    m2::ScanArgs a{};
    const m2_status st = scan_args(c, ssm, batch, chunk_size, xBC, xBC_dtype, xBC_row_stride, dt, dt_row_stride,
                                   z, z_row_stride, y, y_row_stride, slot_idx, has_initial_state, stream, &a);
    if (st != M2_OK) return st;
    a.seqlen = seqlen;
    a.total_tokens = static_cast<int64_t>(batch) * seqlen;
    return from_cuda(m2::launch_chunk_scan(a, reinterpret_cast<cudaStream_t>(stream)));
}

m2_status m2_chunk_scan_varlen(const m2_cache* c, const m2_ssm_params* ssm, int32_t nseq,
                               const int32_t* cu_seqlens, int64_t total_tokens, int32_t max_seqlen,
                               int32_t chunk_size, const void* xBC, int32_t xBC_dtype, int64_t xBC_row_stride,
                               const void* dt, int64_t dt_row_stride, const void* z, int64_t z_row_stride,
                               void* y, int64_t y_row_stride, const int32_t* slot_idx,
                               const uint8_t* has_initial_state, m2_stream stream) {
    if (nseq < 0 || total_tokens < 0 || max_seqlen < 0) return M2_ERR_INVALID_ARG;
    if (total_tokens > INT32_MAX) return M2_ERR_UNSUPPORTED;
    if (nseq == 0 || total_tokens == 0) {
        const m2_status st = cache_status(c);
        return st != M2_OK ? st : (ssm && chunk_size > 0 ? M2_OK : M2_ERR_INVALID_ARG);
    }
    if (!cu_seqlens) return M2_ERR_INVALID_ARG;
    m2::ScanArgs a{};
    const m2_status st = scan_args(c, ssm, nseq, chunk_size, xBC, xBC_dtype, xBC_row_stride, dt, dt_row_stride,
                                   z, z_row_stride, y, y_row_stride, slot_idx, has_initial_state, stream, &a);
    if (st != M2_OK) return st;
    a.cu_seqlens = cu_seqlens;
    a.seqlen = max_seqlen;
    a.total_tokens = total_tokens;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    size_t state_bytes = 0;
    const size_t scratch_bytes = plan_split(&a, nseq, max_seqlen, &state_bytes);
    if (scratch_bytes > 0) {
        cudaMemPool_t pool = nullptr;
        const cudaError_t pe = scratch_pool(&pool);
        if (pe != cudaSuccess) return from_cuda(pe);
        void* scratch = nullptr;
        if (cudaMallocFromPoolAsync(&scratch, scratch_bytes, pool, cs) != cudaSuccess) {
            cudaGetLastError();
            return M2_ERR_OOM;
        }
        a.seg_state = static_cast<float*>(scratch);
        a.seg_decay = reinterpret_cast<float*>(static_cast<char*>(scratch) + state_bytes);
        const cudaError_t e = m2::launch_chunk_scan(a, cs);
        const cudaError_t f = cudaFreeAsync(scratch, cs);
        return from_cuda(e != cudaSuccess ? e : f);
    }
    return from_cuda(m2::launch_chunk_scan(a, cs));
}

m2_status m2_chunk_scan_varlen_static(const m2_cache* c, const m2_ssm_params* ssm, int32_t nseq,
                                      const int32_t* cu_seqlens, int64_t total_tokens, int32_t max_seqlen,
                                      int32_t chunk_size, const void* xBC, int32_t xBC_dtype,
                                      int64_t xBC_row_stride, const void* dt, int64_t dt_row_stride,
                                      const void* z, int64_t z_row_stride, void* y, int64_t y_row_stride,
                                      const int32_t* slot_idx, const uint8_t* has_initial_state,
                                      m2_stream stream) {
    if (nseq < 0 || total_tokens < 0 || max_seqlen < 0) return M2_ERR_INVALID_ARG;
    if (total_tokens > INT32_MAX) return M2_ERR_UNSUPPORTED;
    if (nseq == 0 || total_tokens == 0) {
        const m2_status st = cache_status(c);
        return st != M2_OK ? st : (ssm && chunk_size > 0 ? M2_OK : M2_ERR_INVALID_ARG);
    }
    if (!cu_seqlens) return M2_ERR_INVALID_ARG;
    m2::ScanArgs a{};
    const m2_status st = scan_args(c, ssm, nseq, chunk_size, xBC, xBC_dtype, xBC_row_stride, dt, dt_row_stride,
                                   z, z_row_stride, y, y_row_stride, slot_idx, has_initial_state, stream, &a);
    if (st != M2_OK) return st;
    a.cu_seqlens = cu_seqlens;
    a.seqlen = max_seqlen;
    a.total_tokens = total_tokens;
    size_t state_bytes = 0;
    const size_t need = plan_split(&a, nseq, max_seqlen, &state_bytes);
    if (need > 0) {  // the same plan as m2_chunk_scan_varlen, on the fixed array
        void* scratch = nullptr;
        size_t capacity = 0;
        const cudaError_t e = m2::static_scan_scratch(&scratch, &capacity);
        if (e != cudaSuccess) return from_cuda(e);
        if (need > capacity) return M2_ERR_UNSUPPORTED;
        a.seg_state = static_cast<float*>(scratch);
        a.seg_decay = reinterpret_cast<float*>(static_cast<char*>(scratch) + state_bytes);
    }
    return from_cuda(m2::launch_chunk_scan(a, reinterpret_cast<cudaStream_t>(stream)));
}

m2_status m2_state_update_multi(const m2_cache* c, const m2_ssm_params* ssm, const m2_conv_params* conv,
                                int32_t batch, int32_t T, const void* xBC, int64_t xBC_row_stride, const void* dt,
                                int64_t dt_row_stride, const void* z, int64_t z_row_stride, void* y,
                                int64_t y_row_stride, const int32_t* slot_idx, const int32_t* token_slots,
                                m2_stream stream) {
    const m2_status st = cache_status(c);
    if (st != M2_OK) return st;
    if (!ssm || !ssm->A_log || !ssm->dt_bias || !ssm->D || !conv || !conv->weight || batch < 0 || T < 0)
        return M2_ERR_INVALID_ARG;
    if (conv->activation != 0 && conv->activation != 1) return M2_ERR_INVALID_ARG;
    if (batch == 0 || T == 0) return M2_OK;
    if (!xBC || !dt || !y || !slot_idx || !token_slots) return M2_ERR_INVALID_ARG;
    const m2_shape& s = c->shape;
    const int as = dsize(s.act_dtype);
    const int64_t cd = m2_conv_dim(&s);
    const int64_t hp = static_cast<int64_t>(s.nheads) * s.head_dim;
    if (!aligned16(xBC) || !aligned16(y) || !stride_ok(xBC_row_stride, as, cd) || !stride_ok(y_row_stride, as, hp) ||
        dt_row_stride < s.nheads || !aligned16(conv->weight) || (conv->bias && !aligned16(conv->bias)))
        return M2_ERR_INVALID_ARG;
    if (z && (!aligned16(z) || !stride_ok(z_row_stride, as, hp))) return M2_ERR_INVALID_ARG;
    const m2_status ps = m2::plan_multi_token(s.nheads, s.head_dim, s.d_state, s.ngroups, s.d_conv, T);
    if (ps != M2_OK) return ps;
    if (s.state_dtype != M2_BF16 && s.d_state == 256) return M2_ERR_UNSUPPORTED;
    if (validate_mode()) {
        // input slots and every token's destination slot: all distinct
        const int64_t n = static_cast<int64_t>(batch) * (T + 1);
        std::vector<int32_t> all(static_cast<size_t>(n));
        const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
        if (cudaMemcpyAsync(all.data(), slot_idx, batch * sizeof(int32_t), cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
            cudaMemcpyAsync(all.data() + batch, token_slots, static_cast<size_t>(batch) * T * sizeof(int32_t),
                            cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
            cudaStreamSynchronize(cs) != cudaSuccess)
            return M2_ERR_CUDA;
        std::vector<int32_t> used;
        for (int32_t v : all)
            if (v >= 0) used.push_back(v);
        std::sort(used.begin(), used.end());
        if (std::adjacent_find(used.begin(), used.end()) != used.end()) return M2_ERR_INVALID_ARG;
    }
    m2::MtArgs a{};
    a.ssm = c->ssm;
    a.conv = c->conv;
    a.error = c->error;
    a.num_slots = c->num_slots;
    a.H = s.nheads;
    a.P = s.head_dim;
    a.N = s.d_state;
    a.G = s.ngroups;
    a.K = s.d_conv;
    a.T = T;
    a.conv_dim = cd;
    a.state_bf16 = s.state_dtype == M2_BF16;
    a.act_bf16 = s.act_dtype == M2_BF16;
    a.A_log = ssm->A_log;
    a.dt_bias = ssm->dt_bias;
    a.D = ssm->D;
    a.conv_w = conv->weight;
    a.conv_b = conv->bias;
    a.activation = conv->activation;
    a.batch = batch;
    a.xBC = xBC;
    a.xBC_stride = xBC_row_stride;
    a.dt = dt;
    a.dt_stride = dt_row_stride;
    a.z = z;
    a.z_stride = z_row_stride;
    a.y = y;
    a.y_stride = y_row_stride;
    a.slot_idx = slot_idx;
    a.token_slots = token_slots;
    return from_cuda(m2::launch_state_update_mt(a, reinterpret_cast<cudaStream_t>(stream)));
}

m2_status m2_mixed_step(const m2_cache* c, const m2_ssm_params* ssm, const m2_conv_params* conv,
                        const m2_decode_rows* decode, const m2_prefill_rows* prefill, m2_stream stream) {
    const m2_status st = cache_status(c);
    if (st != M2_OK) return st;
    if (!ssm || !conv) return M2_ERR_INVALID_ARG;
    const bool has_pre = prefill && prefill->nseq > 0 && prefill->total_tokens > 0;
    const bool has_dec = decode && decode->batch > 0;
    if ((prefill && (prefill->nseq < 0 || prefill->total_tokens < 0)) || (decode && decode->batch < 0))
        return M2_ERR_INVALID_ARG;
    if (has_pre) {
        const m2_prefill_rows& p = *prefill;
        if (p.total_tokens > INT32_MAX) return M2_ERR_UNSUPPORTED;
        if (!p.cu_seqlens || !p.xBC_post) return M2_ERR_INVALID_ARG;
        m2_status r = conv1d_impl(c, conv, p.nseq, std::max(p.max_seqlen, 1), p.cu_seqlens, p.total_tokens,
                                  p.xBC, p.xBC_row_stride, p.xBC_post, p.xBC_post_dtype, p.xBC_post_row_stride,
                                  p.slot_idx, stream);
        if (r != M2_OK) return r;
        m2::ScanArgs a{};
        r = scan_args(c, ssm, p.nseq, 128, p.xBC_post, p.xBC_post_dtype, p.xBC_post_row_stride, p.dt,
                      p.dt_row_stride, p.z, p.z_row_stride, p.y, p.y_row_stride, p.slot_idx, p.has_initial_state,
                      stream, &a);
        if (r != M2_OK) return r;
        a.cu_seqlens = p.cu_seqlens;
        a.seqlen = p.max_seqlen;
        a.total_tokens = p.total_tokens;  // nseg = 1: no split, no scratch
        const cudaError_t e = m2::launch_chunk_scan(a, reinterpret_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return from_cuda(e);
    }
    if (has_dec) {
        const m2_decode_rows& d = *decode;
        return state_update_impl(c, ssm, conv, nullptr, d.batch, d.xBC, c->shape.act_dtype, d.xBC_row_stride,
                                 d.dt, d.dt_row_stride, d.z, d.z_row_stride, d.y, d.y_row_stride, d.slot_idx,
                                 stream);
    }
    return M2_OK;
}

m2_status m2_get_device_error(const m2_cache* c, m2_stream stream, int32_t* out_code) {
    if (!c || !out_code) return M2_ERR_INVALID_ARG;
    *out_code = 0;
    if (!c->error) return M2_OK;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    int32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, c->error, sizeof(h), cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(c->error, 0, sizeof(int32_t), cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return M2_ERR_CUDA;
    *out_code = h;
    return M2_OK;
}

const char* m2_status_string(m2_status s) {
    switch (s) {
        case M2_OK: return "ok";
        case M2_ERR_INVALID_ARG: return "invalid argument";
        case M2_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case M2_ERR_CUDA: return "CUDA error";
        case M2_ERR_OOM: return "out of device memory";
        case M2_ERR_BAD_SLOT: return "slot index out of range";
        case M2_ERR_TIMEOUT: return "bounded wait timed out";
        case M2_ERR_RANGE: return "operand outside the fp16 range of the tensor-core scan";
    }
    return "unknown status";
}

const char* m2_version(void) { return "m2 0.1"; }

// ---------------------------------------------------------------------------
// Host-staged decode steps: a ring of device staging buffers, two copy
// streams and the events that order copy in, step and copy out.
struct m2_host_stage {
    int32_t depth = 0;
    int64_t in_bytes = 0;
    int64_t y_bytes = 0;
    std::vector<void*> d_in, d_y;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    std::vector<cudaEvent_t> in_done, comp_done, out_done;
    cudaEvent_t start = nullptr;
    std::vector<uint8_t> used;
    int64_t next = 0;
    bool fresh = true;  // the next step's copies first wait for the caller's stream
};

m2_status m2_host_stage_destroy(m2_host_stage* hs) {
    if (!hs) return M2_ERR_INVALID_ARG;
    m2_status st = M2_OK;
    auto keep = [&](cudaError_t e) {
        if (e != cudaSuccess && st == M2_OK) st = M2_ERR_CUDA;
    };
    // every step that read a staging buffer and every copy are done before
    // the buffers go
    for (size_t r = 0; r < hs->used.size() && r < hs->comp_done.size(); ++r)
        if (hs->used[r]) keep(cudaEventSynchronize(hs->comp_done[r]));
    if (hs->s_in) keep(cudaStreamSynchronize(hs->s_in));
    if (hs->s_out) keep(cudaStreamSynchronize(hs->s_out));
    for (void* p : hs->d_in) keep(cudaFree(p));
    for (void* p : hs->d_y) keep(cudaFree(p));
    for (auto* v : {&hs->in_done, &hs->comp_done, &hs->out_done})
        for (cudaEvent_t e : *v) keep(cudaEventDestroy(e));
    if (hs->start) keep(cudaEventDestroy(hs->start));
    if (hs->s_in) keep(cudaStreamDestroy(hs->s_in));
    if (hs->s_out) keep(cudaStreamDestroy(hs->s_out));
    delete hs;
    return st;
}

m2_status m2_host_stage_create(int32_t depth, int64_t in_bytes, int64_t y_bytes, m2_host_stage** out) {
    if (!out) return M2_ERR_INVALID_ARG;
    *out = nullptr;
    if (depth < 1 || depth > 64 || in_bytes <= 0 || y_bytes <= 0) return M2_ERR_INVALID_ARG;
    auto* hs = new (std::nothrow) m2_host_stage();
    if (!hs) return M2_ERR_OOM;
    hs->depth = depth;
    hs->in_bytes = in_bytes;
    hs->y_bytes = y_bytes;
    hs->used.assign(static_cast<size_t>(depth), 0);
    auto fail = [&](cudaError_t e) {
        m2_host_stage_destroy(hs);
        return from_cuda(e);
    };
    for (int32_t r = 0; r < depth; ++r) {
        void* p = nullptr;
        cudaError_t e = cudaMalloc(&p, static_cast<size_t>(in_bytes));
        if (e != cudaSuccess) return fail(e);
        hs->d_in.push_back(p);
        p = nullptr;
        e = cudaMalloc(&p, static_cast<size_t>(y_bytes));
        if (e != cudaSuccess) return fail(e);
        hs->d_y.push_back(p);
        for (auto* v : {&hs->in_done, &hs->comp_done, &hs->out_done}) {
            cudaEvent_t ev = nullptr;
            e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
            if (e != cudaSuccess) return fail(e);
            v->push_back(ev);
        }
    }
    cudaError_t e = cudaEventCreateWithFlags(&hs->start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hs->s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hs->s_out, cudaStreamNonBlocking);
    if (e != cudaSuccess) return fail(e);
    *out = hs;
    return M2_OK;
}

m2_status m2_state_update_host(m2_host_stage* hs, const m2_cache* c, const m2_ssm_params* ssm,
                               const m2_conv_params* conv, int32_t batch, const void* host_in,
                               int64_t off_xBC, int64_t xBC_row_stride, int64_t off_dt,
                               int64_t dt_row_stride, int64_t off_z, int64_t z_row_stride, void* host_y,
                               int64_t y_row_stride, const int32_t* slot_idx, m2_stream stream) {
    if (!hs || !host_in || !host_y || batch < 0) return M2_ERR_INVALID_ARG;
    const m2_status cs = cache_status(c);
    if (cs != M2_OK) return cs;
    if (batch == 0) return M2_OK;
    const int64_t as = dsize(c->shape.act_dtype);
    auto block_ok = [&](int64_t off, int64_t stride) {
        return off >= 0 && off % 16 == 0 && stride > 0 && off + batch * stride * as <= hs->in_bytes;
    };
    if (!block_ok(off_xBC, xBC_row_stride) || !block_ok(off_dt, dt_row_stride) ||
        (off_z >= 0 && !block_ok(off_z, z_row_stride)) || y_row_stride <= 0 ||
        batch * y_row_stride * as > hs->y_bytes)
        return M2_ERR_INVALID_ARG;
    const int32_t r = static_cast<int32_t>(hs->next % hs->depth);
    uint8_t* din = static_cast<uint8_t*>(hs->d_in[r]);
    const void* xp = din + off_xBC;
    const void* dtp = din + off_dt;
    const void* zp = off_z >= 0 ? din + off_z : nullptr;
    void* yp = hs->d_y[r];
    m2_status st = state_update_impl(c, ssm, conv, nullptr, batch, xp, c->shape.act_dtype, xBC_row_stride, dtp,
                                     dt_row_stride, zp, z_row_stride, yp, y_row_stride, slot_idx, stream, true);
    if (st != M2_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    auto run = [&](cudaError_t x) {
        if (e == cudaSuccess) e = x;
    };
    if (hs->fresh) {  // the copies follow what the caller enqueued on `stream` before
        run(cudaEventRecord(hs->start, s));
        run(cudaStreamWaitEvent(hs->s_in, hs->start, 0));
        run(cudaStreamWaitEvent(hs->s_out, hs->start, 0));
        hs->fresh = false;
    }
    if (hs->used[r]) run(cudaStreamWaitEvent(hs->s_in, hs->comp_done[r], 0));  // the buffer's last step has run
    run(cudaMemcpyAsync(din, host_in, static_cast<size_t>(hs->in_bytes), cudaMemcpyHostToDevice, hs->s_in));
    run(cudaEventRecord(hs->in_done[r], hs->s_in));
    run(cudaStreamWaitEvent(s, hs->in_done[r], 0));
    if (hs->used[r]) run(cudaStreamWaitEvent(s, hs->out_done[r], 0));  // the buffer's last y has left
    if (e != cudaSuccess) return M2_ERR_CUDA;
    st = state_update_impl(c, ssm, conv, nullptr, batch, xp, c->shape.act_dtype, xBC_row_stride, dtp,
                           dt_row_stride, zp, z_row_stride, yp, y_row_stride, slot_idx, stream);
    if (st != M2_OK) return st;
    run(cudaEventRecord(hs->comp_done[r], s));
    run(cudaStreamWaitEvent(hs->s_out, hs->comp_done[r], 0));
    run(cudaMemcpyAsync(host_y, yp, static_cast<size_t>(batch * y_row_stride * as), cudaMemcpyDeviceToHost,
                        hs->s_out));
    run(cudaEventRecord(hs->out_done[r], hs->s_out));
    hs->used[r] = 1;
    ++hs->next;
    return e == cudaSuccess ? M2_OK : M2_ERR_CUDA;
}

m2_status m2_host_stage_join(m2_host_stage* hs, m2_stream stream) {
    if (!hs) return M2_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    for (int32_t r = 0; r < hs->depth; ++r) {
        if (!hs->used[r]) continue;
        if (cudaStreamWaitEvent(s, hs->out_done[r], 0) != cudaSuccess) return M2_ERR_CUDA;
    }
    hs->fresh = true;
    return M2_OK;
}

}  // extern "C"
