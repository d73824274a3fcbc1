/*
 * m2.h -- C ABI of libm2, the B200 (sm_100a) Mamba-2 recurrent-state library.
 *
 * The library runs the recurrent hot path of a Mamba-2 SSM mixer in hybrid
 * Mamba-Transformer serving: the one-token decode step (causal conv update
 * over a rolling conv cache, then the selective state update) and a chunked
 * prefill scan that lands on the same state. It reads and writes a fixed-size
 * per-sequence state cache in place at slot indices, with no gather/scatter.
 *
 * Passages that define the operations (cited by page title and section):
 *  - vllm.cpp issue #1311 "NemotronH runs the PREFILL mamba kernels at decode",
 *    section "The divergence": decode calls causal_conv1d_update and
 *    selective_state_update, both taking state/conv slot indices and reading
 *    and writing the cache in place at the slot.
 *  - same issue, section "Confirm or refute": heads map to groups with
 *    hpg = H/G, so n_groups = 8 is handled; a state update costs 1 launch and
 *    0 allocations per layer per token (section "Cost, at T=1, ...").
 *  - Nemotron-H-8B-Base-8K model record: ssm_state_size N, mamba_head_dim P,
 *    mamba_num_heads H, n_groups G; 2 MiB of bf16 state per layer per
 *    sequence, constant in context length; a fixed-size recurrent state
 *    allocator.
 *  - TensorRT-LLM issue #16976 (hybrid serving at concurrency 384): decode
 *    must replay as a CUDA graph, so decode calls never allocate, never
 *    synchronise and never read device status on the host.
 *
 * The recurrence, per head h with group g(h) = h / (H/G):
 *     dt = softplus(dt_raw[h] + dt_bias[h]);  A = -exp(A_log[h]);  dA = exp(dt*A)
 *     S[h,p,n] <- S[h,p,n]*dA + (dt*x[h,p]) * B[g,n]
 *     y[h,p]    = sum_n S[h,p,n]*C[g,n] + D[h]*x[h,p],  times silu(z[h,p]) if z
 * where x | B | C are the three parts of the post-conv xBC row
 * (H*P, G*N and G*N channels; conv_dim = H*P + 2*G*N).
 *
 * Conventions for every call:
 *  - Pointers are DEVICE pointers unless stated otherwise, on the device that
 *    is current when the call is made. The caller owns every buffer except the
 *    ones m2_cache_alloc creates.
 *  - Tensor rows are contiguous (unit stride inside a row). Row strides are in
 *    elements; every row start must be 16-byte aligned (pointer and stride).
 *  - Slot indices are int32. A negative index marks a padding row: it is
 *    skipped, its caches are not touched and its y row is written with zeros.
 *    An index >= num_slots is a device error: the row is skipped, nothing is
 *    written for it, and M2_ERR_BAD_SLOT is recorded in the cache's error
 *    word. Slots must be unique within one call (checked on the host only when
 *    the environment variable M2_VALIDATE=1 is set, which synchronises).
 *  - All compute calls are asynchronous on `stream` and never synchronise
 *    (outside M2_VALIDATE mode), so they can be captured in CUDA graphs. They
 *    allocate nothing, except m2_chunk_scan_varlen when it splits sequences
 *    (stream-ordered scratch, see there). Argument errors are returned before
 *    anything is launched.
 *  - There is no CPU fallback: without a usable sm_100 device the compute
 *    calls fail with M2_ERR_CUDA.
 */
#ifndef M2_H_
#define M2_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st* m2_stream;

typedef enum m2_dtype {
    M2_F32 = 0,  /* IEEE binary32 */
    M2_BF16 = 1, /* bfloat16 */
    M2_F16 = 2   /* IEEE binary16: only for the post-conv xBC buffer between
                    m2_conv1d_update (out_dtype) and m2_state_update /
                    m2_chunk_scan (xBC_dtype); its 11-bit significand keeps the
                    post-conv values more precisely than bfloat16 and feeds the
                    tensor-core scan without conversion */
} m2_dtype;

typedef enum m2_status {
    M2_OK = 0,
    M2_ERR_INVALID_ARG = -1, /* NULL pointer, bad size, stride or alignment */
    M2_ERR_UNSUPPORTED = -2, /* valid, but not a shape or dtype the kernels implement */
    M2_ERR_CUDA = -3,        /* a CUDA runtime call or a launch failed */
    M2_ERR_OOM = -4,         /* device allocation failed (m2_cache_alloc only) */
    M2_ERR_BAD_SLOT = -5,    /* device: a slot index >= num_slots was seen */
    M2_ERR_TIMEOUT = -6,     /* device: a bounded wait inside a kernel ran out; only the
                                error word is then meaningful: the launch's outputs (y, the
                                state and conv cache rows it touches) are undefined, and a
                                bulk copy that had still not landed when its CTA gave up
                                may write into shared memory of a later launch, so treat
                                the CUDA context as unreliable from then on */
    M2_ERR_RANGE = -7        /* device: a value exceeded the fp16 range of the tensor-core
                                scan's operands (|v| >= 65520); that row's results are not valid */
} m2_status;

/* Mixer shape (Nemotron-H-8B: H=128, P=64, N=128, G=8, K=4). */
typedef struct m2_shape {
    int32_t nheads;      /* H */
    int32_t head_dim;    /* P */
    int32_t d_state;     /* N */
    int32_t ngroups;     /* G, divides H */
    int32_t d_conv;      /* K, conv width (2..8) */
    int32_t state_dtype; /* m2_dtype of the SSM cache */
    int32_t act_dtype;   /* m2_dtype of activations, conv cache, conv weight/bias, dt_raw, y */
} m2_shape;

/* A slot-indexed cache of one mixer layer. */
typedef struct m2_cache {
    void* ssm;         /* [num_slots, H, P, N] state_dtype, N fastest */
    void* conv;        /* [num_slots, K-1, conv_dim] act_dtype: the last K-1 RAW xBC
                          inputs of each channel, oldest row first */
    int32_t* error;    /* device int32 error word (0 = none), or NULL = not reported */
    int64_t num_slots;
    m2_shape shape;
    int32_t owned;     /* 1 when m2_cache_alloc created ssm/conv/error */
    int32_t device;    /* CUDA device ordinal of the buffers */
} m2_cache;

/* Depthwise causal conv parameters: weight [conv_dim, K] act_dtype (tap K-1
 * multiplies the newest input), bias [conv_dim] act_dtype or NULL,
 * activation 0 = none, 1 = SiLU. weight and bias are device pointers,
 * 16-byte aligned (M2_ERR_INVALID_ARG otherwise). */
typedef struct m2_conv_params {
    const void* weight;
    const void* bias;
    int32_t activation;
} m2_conv_params;

/* Per-head SSM parameters, fp32 [H] each: A = -exp(A_log). */
typedef struct m2_ssm_params {
    const float* A_log;
    const float* dt_bias;
    const float* D;
} m2_ssm_params;

/* conv_dim = H*P + 2*G*N, or -1 for a NULL/invalid shape. Host only. */
int64_t m2_conv_dim(const m2_shape* shape);

/* M2_OK when the kernels implement `shape`; M2_ERR_INVALID_ARG for an
 * inconsistent shape; M2_ERR_UNSUPPORTED otherwise. Host only, no CUDA. */
m2_status m2_shape_check(const m2_shape* shape);

/* Bytes of the SSM and conv caches for num_slots slots (Nemotron-H record:
 * 2 MiB of bf16 state per slot at H=128, P=64, N=128). Host only, no CUDA. */
m2_status m2_cache_bytes(const m2_shape* shape, int64_t num_slots, int64_t* ssm_bytes,
                         int64_t* conv_bytes);

/* The fixed-size recurrent state allocator (Nemotron-H record): allocates
 * the SSM cache, the conv cache and the error word on the current device and
 * zero-fills them on `stream` (then synchronises `stream`; not a hot call).
 * Returns M2_ERR_OOM when the device is out of memory. */
m2_status m2_cache_alloc(const m2_shape* shape, int64_t num_slots, m2_stream stream,
                         m2_cache* out);

/* Describes caller-owned buffers as a cache (for example torch tensors).
 * ssm and conv must be 16-byte aligned; error_word may be NULL. Nothing is
 * allocated or launched. */
m2_status m2_cache_wrap(const m2_shape* shape, int64_t num_slots, void* ssm, void* conv,
                        int32_t* error_word, m2_cache* out);

/* Frees the buffers of a cache made by m2_cache_alloc (after synchronising
 * `stream`); a wrapped cache is only cleared. */
m2_status m2_cache_free(m2_cache* cache, m2_stream stream);

/* Zero the SSM state and conv cache of n slots (start of new sequences) in one
 * launch, without a host synchronisation. Negative indices are skipped; an
 * index >= num_slots is a device error as above. */
m2_status m2_cache_zero_slots(const m2_cache* cache, int32_t n, const int32_t* slot_idx,
                              m2_stream stream);

/*
 * causal_conv1d_update over `seqlen` tokens per row (vllm.cpp issue, "The
 * divergence"; seqlen > 1 is the prefill conv that precedes the chunk scan).
 *   xBC      [batch, seqlen, conv_dim] act_dtype, raw; element (b,t,c) at
 *            xBC[(b*seqlen + t)*xBC_row_stride + c]
 *   xBC_out  [batch, seqlen, conv_dim] out_dtype (M2_F32, M2_BF16 or M2_F16),
 *            post-conv (an fp16 value beyond 65504 records M2_ERR_RANGE)
 *            (bias added, activation applied); same indexing with out_row_stride
 *   slot_idx [batch] int32: row b reads its window history from, and writes
 *            the last K-1 raw inputs back to, cache->conv[slot_idx[b]]
 * The conv cache is rolled in place by exact copies. One launch.
 */
m2_status m2_conv1d_update(const m2_cache* cache, const m2_conv_params* conv, int32_t batch,
                           int32_t seqlen, const void* xBC, int64_t xBC_row_stride,
                           void* xBC_out, int32_t out_dtype, int64_t out_row_stride,
                           const int32_t* slot_idx, m2_stream stream);

/*
 * m2_conv1d_update over nseq sequences packed back to back: sequence b is
 * rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of xBC / xBC_out (cu_seqlens
 * [nseq+1] int32 on the device, cu_seqlens[nseq] = total_tokens) and rolls
 * cache->conv[slot_idx[b]]. max_seqlen (host) sizes the grid; a longer
 * sequence is still covered. An empty sequence leaves its slot untouched.
 * Otherwise as m2_conv1d_update. One launch.
 */
m2_status m2_conv1d_update_varlen(const m2_cache* cache, const m2_conv_params* conv, int32_t nseq,
                                  const int32_t* cu_seqlens, int64_t total_tokens, int32_t max_seqlen,
                                  const void* xBC, int64_t xBC_row_stride, void* xBC_out,
                                  int32_t out_dtype, int64_t out_row_stride, const int32_t* slot_idx,
                                  m2_stream stream);

/*
 * selective_state_update for one token per row (vllm.cpp issue, "The
 * divergence"), in place on cache->ssm at slot_idx[b].
 *   conv     non-NULL: xBC is the RAW row and the conv tap + roll of
 *            causal_conv1d_update run fused in the same launch (xBC_dtype must
 *            then be act_dtype); NULL: xBC is already post-conv, in xBC_dtype
 *            (M2_F32, M2_BF16 or M2_F16)
 *   xBC      [batch, conv_dim], row stride xBC_row_stride
 *   dt       [batch, H] act_dtype (dt_raw, before dt_bias and softplus)
 *   z        [batch, H*P] act_dtype, or NULL for no gate
 *   y        [batch, H*P] act_dtype, out
 *   slot_idx [batch] int32
 * The state is computed in fp32 and stored once, rounded to nearest even; y is
 * computed from the unrounded new state. One launch, no scratch memory.
 */
m2_status m2_state_update(const m2_cache* cache, const m2_ssm_params* ssm,
                          const m2_conv_params* conv, int32_t batch, const void* xBC,
                          int32_t xBC_dtype, int64_t xBC_row_stride, const void* dt,
                          int64_t dt_row_stride, const void* z, int64_t z_row_stride, void* y,
                          int64_t y_row_stride, const int32_t* slot_idx, m2_stream stream);

/* Gated RMSNorm applied to the decode output (the `norm` tensor of the
 * Mamba-2 mixer in the Nemotron-H-8B-Base-8K record): weight [H*P] act_dtype
 * (device, 16-byte aligned), eps >= 0. */
typedef struct m2_norm_params {
    const void* weight;
    float eps;
} m2_norm_params;

/*
 * m2_state_update with the gated RMSNorm fused into the same launch. The
 * gated y, v = y * silu(z) (v = y when z is NULL), is normalised over each
 * group of H*P/G consecutive channels (the heads of one SSM group):
 *     out[c] = v[c] / sqrt(mean over the group of v^2 + eps) * weight[c]
 * and out is written to y. The conv is always fused here (conv must be
 * non-NULL; xBC is the raw row in act_dtype): the group's CTAs are the
 * launch's thread-block cluster and exchange their partial sums of squares
 * through distributed shared memory, so y makes no extra round trip. Other
 * arguments, the state update and the conv cache as for m2_state_update.
 * One launch, no scratch memory.
 */
m2_status m2_state_update_norm(const m2_cache* cache, const m2_ssm_params* ssm,
                               const m2_conv_params* conv, const m2_norm_params* norm, int32_t batch,
                               const void* xBC, int64_t xBC_row_stride, const void* dt,
                               int64_t dt_row_stride, const void* z, int64_t z_row_stride, void* y,
                               int64_t y_row_stride, const int32_t* slot_idx, m2_stream stream);

/*
 * Chunked prefill scan (vllm.cpp issue, "The divergence": the chunk scan that
 * follows CausalConv1dFwd at prefill). For each row, runs `seqlen` tokens of
 * the recurrence starting from cache->ssm[slot_idx[b]] (or from zero when
 * has_initial_state is NULL or has_initial_state[b] == 0), writes y for every
 * token and stores the final state back to the same slot, rounded once.
 *   xBC      [batch, seqlen, conv_dim] xBC_dtype (M2_F32, M2_BF16 or M2_F16),
 *            POST-conv, row stride
 *            xBC_row_stride (token rows of a sequence are consecutive)
 *   dt       [batch, seqlen, H] act_dtype, row stride dt_row_stride
 *   z        [batch, seqlen, H*P] act_dtype or NULL, row stride z_row_stride
 *   y        [batch, seqlen, H*P] act_dtype, row stride y_row_stride
 *   chunk_size  tokens per chunk (the last chunk may be partial)
 * With bf16 state and activations at P = 64, N = 128 the scan runs on the
 * tensor cores in chunks of 128 tokens, with fp16 MMA operands (inputs converted
 * exactly, derived operands rounded once, fp32 accumulation); any operand that
 * leaves the fp16 range sets M2_ERR_RANGE in the error word. The result does
 * not depend on chunk_size, which must be positive (the kernels choose their own
 * tiling). Other dtypes and shapes run token by token on the CUDA cores.
 * No allocation, no scratch memory.
 */
m2_status m2_chunk_scan(const m2_cache* cache, const m2_ssm_params* ssm, int32_t batch,
                        int32_t seqlen, int32_t chunk_size, const void* xBC, int32_t xBC_dtype,
                        int64_t xBC_row_stride, const void* dt, int64_t dt_row_stride,
                        const void* z, int64_t z_row_stride, void* y, int64_t y_row_stride,
                        const int32_t* slot_idx, const uint8_t* has_initial_state,
                        m2_stream stream);

/*
 * Variable-length prefill scan: the same recurrence as m2_chunk_scan over
 * nseq sequences packed back to back (TensorRT-LLM issue #16976: mixed
 * batches of long prompts, ~19K tokens). Sequence b is rows cu_seqlens[b] ..
 * cu_seqlens[b+1]-1 of the packed arrays and runs from
 * cache->ssm[slot_idx[b]] (or zero, as for m2_chunk_scan); its final state is
 * stored back once. An empty sequence (cu_seqlens[b+1] == cu_seqlens[b])
 * leaves its slot untouched.
 *   cu_seqlens    [nseq+1] int32, device, non-decreasing, cu_seqlens[0] = 0,
 *                 cu_seqlens[nseq] = total_tokens
 *   total_tokens  rows of the packed arrays (host value, < 2^31)
 *   max_seqlen    host upper bound on the sequence lengths, used only to plan
 *                 the split below; a longer sequence is still computed
 *                 correctly, with less parallelism
 *   xBC           [total_tokens, conv_dim] xBC_dtype, POST-conv
 *   dt            [total_tokens, H] act_dtype
 *   z, y          [total_tokens, H*P] act_dtype (z may be NULL)
 * Split sequences: on the tensor-core path (bf16 state and activations,
 * P = 64, N = 128), when the nseq * H (sequence, head) pairs leave room for at
 * least three segments per pair at one CTA per SM (nseq * H * 3 <= SMs), each
 * sequence is cut into segments of whole 128-token chunks that run in
 * parallel: a first pass stores every segment's final state from a zero start
 * and its total decay, a combine pass carries the states across segments in
 * fp32 (the recurrence is linear in the state), and the scan pass runs each
 * segment from its carried state. The scratch (at most one 32 KB state and
 * one decay per SM) is allocated stream-ordered on `stream` from a memory pool
 * the library creates once per device and that keeps its memory for reuse,
 * then freed stream-ordered; M2_ERR_OOM if it cannot be had. Without a split
 * the call allocates nothing.
 */
m2_status m2_chunk_scan_varlen(const m2_cache* cache, const m2_ssm_params* ssm, int32_t nseq,
                               const int32_t* cu_seqlens, int64_t total_tokens, int32_t max_seqlen,
                               int32_t chunk_size, const void* xBC, int32_t xBC_dtype,
                               int64_t xBC_row_stride, const void* dt, int64_t dt_row_stride,
                               const void* z, int64_t z_row_stride, void* y, int64_t y_row_stride,
                               const int32_t* slot_idx, const uint8_t* has_initial_state,
                               m2_stream stream);

/*
 * m2_chunk_scan_varlen without any allocation. This entry point has no
 * counterpart in the sources the library follows; it exists for callers that
 * cannot allocate device memory once they are running: a serving runtime that
 * reserves all of its device memory at start-up and must not fail a step on an
 * allocation, or a process in which no stream-ordered memory pool can be used.
 * Same arguments, results and split plan as m2_chunk_scan_varlen (bit for
 * bit); the scratch of a split is a file-scope device array of 16 MiB, enough
 * for every split plan on GPUs of up to 511 SMs (one 32 KB state and one decay
 * per SM at most). A plan that needs more returns M2_ERR_UNSUPPORTED before
 * launching. Nothing in the array needs clearing: every slot the scan pass
 * reads is written earlier in the same call.
 *   - The first call on a device looks up the array's address with
 *     cudaGetSymbolAddress (once per device; its error is returned as
 *     M2_ERR_CUDA) and may load the module that holds it: make that first call
 *     before any stream capture begins on that device. The address is cached
 *     per device for the life of the process; after a cudaDeviceReset the
 *     cached address is stale, so do not call this entry point again in that
 *     process.
 *   - Every GPU on which the library's module is loaded holds the 16 MiB until
 *     the process exits. Under lazy module loading (the CUDA default) that is
 *     only a device where a libm2 call has run; with CUDA_MODULE_LOADING=EAGER
 *     it is every device the process initialises.
 *   - All calls on a device share the one array: two calls whose executions
 *     overlap (other streams, other host threads) race on it and corrupt each
 *     other's results. Serialise them, e.g. on one stream.
 * Without a split the call uses no scratch at all.
 */
m2_status m2_chunk_scan_varlen_static(const m2_cache* cache, const m2_ssm_params* ssm, int32_t nseq,
                                      const int32_t* cu_seqlens, int64_t total_tokens,
                                      int32_t max_seqlen, int32_t chunk_size, const void* xBC,
                                      int32_t xBC_dtype, int64_t xBC_row_stride, const void* dt,
                                      int64_t dt_row_stride, const void* z, int64_t z_row_stride,
                                      void* y, int64_t y_row_stride, const int32_t* slot_idx,
                                      const uint8_t* has_initial_state, m2_stream stream);

/*
 * Multi-token decode for speculative decoding: T draft tokens per sequence in
 * one launch (1 <= T <= 16), each token a decode step with the conv tap fused,
 * starting from the state and conv window of cache slot slot_idx[b]. The
 * state and the conv window after token t are stored into cache slot
 * token_slots[b*T + t] (negative: not stored); the input slot is only read, so
 * after verifying the drafts the caller adopts the slot of the last accepted
 * token and the rejected ones are simply dropped. Every state is rounded to the
 * storage dtype after its token, exactly as T separate m2_state_update calls
 * would store it; y of token t comes from the unrounded state.
 *   xBC          [batch, T, conv_dim] act_dtype, raw; token rows
 *                xBC_row_stride apart, row b*T + t
 *   dt           [batch, T, H] act_dtype;  z [batch, T, H*P] act_dtype or NULL
 *   y            [batch, T, H*P] act_dtype, out
 *   slot_idx     [batch] int32 (negative: padding row, y = 0, nothing stored)
 *   token_slots  [batch, T] int32; every non-negative entry, and every input
 *                slot, must be distinct (checked on the host under
 *                M2_VALIDATE=1); an entry >= num_slots is a device error
 * Supported: H*P/G a multiple of 64, P a multiple of 8, N in {64, 128, 256}
 * (256 only with a bf16 state). One launch, no scratch memory.
 */
m2_status m2_state_update_multi(const m2_cache* cache, const m2_ssm_params* ssm,
                                const m2_conv_params* conv, int32_t batch, int32_t T, const void* xBC,
                                int64_t xBC_row_stride, const void* dt, int64_t dt_row_stride,
                                const void* z, int64_t z_row_stride, void* y, int64_t y_row_stride,
                                const int32_t* slot_idx, const int32_t* token_slots, m2_stream stream);

/* The decode rows of a mixed step: one token each, raw xBC (the conv is
 * fused), as for m2_state_update with conv != NULL. */
typedef struct m2_decode_rows {
    int32_t batch;
    const void* xBC;  /* [batch, conv_dim] act_dtype, raw */
    int64_t xBC_row_stride;
    const void* dt;   /* [batch, H] act_dtype */
    int64_t dt_row_stride;
    const void* z;    /* [batch, H*P] act_dtype or NULL */
    int64_t z_row_stride;
    void* y;          /* [batch, H*P] act_dtype, out */
    int64_t y_row_stride;
    const int32_t* slot_idx;
} m2_decode_rows;

/* The prefill sequences of a mixed step, packed back to back (as for
 * m2_chunk_scan_varlen), with the caller's buffer for the post-conv xBC. */
typedef struct m2_prefill_rows {
    int32_t nseq;
    const int32_t* cu_seqlens;  /* [nseq+1] int32, device */
    int64_t total_tokens;
    int32_t max_seqlen;         /* host bound, sizes the grids */
    const void* xBC;            /* [total_tokens, conv_dim] act_dtype, raw */
    int64_t xBC_row_stride;
    void* xBC_post;             /* [total_tokens, conv_dim] xBC_post_dtype, written */
    int32_t xBC_post_dtype;     /* M2_F32, M2_BF16 or M2_F16 */
    int64_t xBC_post_row_stride;
    const void* dt;             /* [total_tokens, H] act_dtype */
    int64_t dt_row_stride;
    const void* z;              /* [total_tokens, H*P] act_dtype or NULL */
    int64_t z_row_stride;
    void* y;                    /* [total_tokens, H*P] act_dtype, out */
    int64_t y_row_stride;
    const int32_t* slot_idx;    /* [nseq] */
    const uint8_t* has_initial_state;  /* [nseq] or NULL (all start from zero) */
} m2_prefill_rows;

/*
 * One mixed serving step on one slot-indexed cache (TensorRT-LLM issue #16976:
 * iterations that mix prefill chunks and decode tokens, where the decode part
 * should stay graphed): the prefill sequences run the prefill conv
 * (m2_conv1d_update_varlen into xBC_post) and the variable-length chunk scan,
 * and the decode rows run the fused decode step, all enqueued on `stream` in
 * one call (three launches: conv, scan, decode) with no allocation and no
 * synchronisation. The scan does not split sequences here (no scratch). The
 * decode slots and the prefill slots must be disjoint. Either part may be
 * NULL or empty. Results are those of the separate calls, bit for bit.
 */
m2_status m2_mixed_step(const m2_cache* cache, const m2_ssm_params* ssm, const m2_conv_params* conv,
                        const m2_decode_rows* decode, const m2_prefill_rows* prefill,
                        m2_stream stream);

/*
 * Decode steps whose inputs and outputs live in host memory (vllm.cpp issue
 * #1311, section "The divergence": the same fused step as m2_state_update,
 * for a caller that produces the step's rows on the host and reads y back
 * every step). An m2_host_stage owns `depth` device staging buffers of
 * in_bytes and y_bytes, two copy streams and the events that order them; it
 * is created and destroyed off the hot path (cudaMalloc / cudaFree, device of
 * the current context; destroy first waits for every step and copy it issued).
 * M2_ERR_INVALID_ARG for depth < 1 or a zero size, M2_ERR_OOM when the device
 * is out of memory.
 */
typedef struct m2_host_stage m2_host_stage;
m2_status m2_host_stage_create(int32_t depth, int64_t in_bytes, int64_t y_bytes, m2_host_stage** out);
m2_status m2_host_stage_destroy(m2_host_stage* stage);

/*
 * One m2_state_update step (conv fused when conv is non-NULL) whose rows come
 * from host memory. host_in (pinned, in_bytes of the stage) holds the step's
 * xBC rows at byte offset off_xBC (act_dtype, xBC_row_stride elements), its
 * dt rows at off_dt and its z rows at off_z (off_z < 0: no gate); every
 * offset a multiple of 16. y (batch rows of y_row_stride elements, act_dtype)
 * is copied into host_y (pinned) afterwards. slot_idx is on the device.
 * The step takes the next staging buffer of the ring: its copy in (on the
 * stage's input stream) waits until the step that last used the buffer has
 * run, the step on `stream` waits for that copy and for the copy out of the
 * buffer's previous y, and the copy out (on the stage's output stream)
 * follows the step, so consecutive steps overlap their copies with each
 * other's kernels. Everything is asynchronous to the host; host_in may be
 * rewritten and host_y read only after m2_host_stage_join and a
 * synchronisation of `stream`. Validation as for m2_state_update, plus the
 * stage's sizes (M2_ERR_INVALID_ARG) before anything is enqueued.
 */
m2_status m2_state_update_host(m2_host_stage* stage, const m2_cache* cache, const m2_ssm_params* ssm,
                               const m2_conv_params* conv, int32_t batch, const void* host_in,
                               int64_t off_xBC, int64_t xBC_row_stride, int64_t off_dt,
                               int64_t dt_row_stride, int64_t off_z, int64_t z_row_stride, void* host_y,
                               int64_t y_row_stride, const int32_t* slot_idx, m2_stream stream);

/* Makes `stream` wait for every copy the stage has issued so far; the next
 * step's copy in then also waits for `stream`'s work issued before it. */
m2_status m2_host_stage_join(m2_host_stage* stage, m2_stream stream);

/* Debug/test path: synchronises `stream`, copies the cache's error word to
 * *out_code (0 or an m2_status value) and clears it. Not for hot loops. */
m2_status m2_get_device_error(const m2_cache* cache, m2_stream stream, int32_t* out_code);

/* Static description of a status code. */
const char* m2_status_string(m2_status status);

/* Library version string, "m2 <major>.<minor>". */
const char* m2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* M2_H_ */
