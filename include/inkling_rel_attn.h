/*
 * inkling_rel_attn.h -- C ABI of the B200 (sm_100a) learned-relative
 * grouped-query attention library (libinkling_rel_attn.so).
 *
 * The operation is the attention core of Inkling2 as documented on the NVIDIA
 * NeMo AutoModel API pages:
 *   - "nemo_automodel.components.models.inkling2.flex_attention",
 *     Inkling2FlexAttention(head_dim, window) and its forward(q, k, v,
 *     profiles, sink, valid, key_valid, positions, key_positions,
 *     query_offset): argument shapes, defaults and the FP32 result; the class
 *     note that no sequence-by-sequence bias tensor is built and that
 *     gradients reach the profiles and the returned log-sum-exp;
 *   - "nemo_automodel.components.models.inkling2.attention",
 *     Inkling2Attention.forward (the sink as a virtual key whose value row is
 *     zero) and the quadratic reference Inkling2Attention._eager (which leaves
 *     its inputs untouched).
 *
 * Definition (b batch, h query head, g = h / (Hq/Hkv) its KV head, i local
 * query row, i_g = query_offset + i its global column, j key column):
 *   allowed(i,j) = valid[b,i] && key_valid[b,j] && j <= i_g
 *                  && positions[b,i] - key_positions[b,j] == i_g - j  (same document)
 *                  && (window == 0 || i_g - j < window)
 *   d   = positions[b,i] - key_positions[b,j]
 *   z_j = head_dim^-0.5 * <q[b,i,h,:], k[b,j,g,:]> + (d < rel_extent ? profiles[b,h,i,d] : 0)
 *   lse[b,i,h] = log(exp(sink[b,i,h]) + sum_allowed exp(z_j))
 *   out[b,i,h,:] = sum_allowed exp(z_j - lse) * v[b,j,g,:]
 * A row with no allowed key (e.g. an invalid query) gets out = 0, lse = sink.
 *
 * Conventions for every entry point:
 *   - All tensors are dense, row-major, in device memory owned by the caller.
 *     BF16 tensors are passed as their 16-bit patterns (uint16_t).
 *   - The library allocates no device memory; scratch lives in a
 *     caller-provided device workspace whose size comes from
 *     inkling_rel_attn_workspace_size(). Inputs are never written. The state
 *     kept between calls is, per host thread and device, one non-blocking
 *     CUDA stream and four events, created by the first backward call made
 *     outside a stream capture and reused: the backward forks part of its work
 *     onto that stream and joins it back to `stream` with the events before it
 *     returns, so all of it is ordered on `stream` (and captured with it).
 *     One exception: inkling_rel_attn_fwd_noalloc takes no workspace; its
 *     scratch is a static device array inside the library that keeps the last
 *     call's contents, and the library caches that array's address per CUDA
 *     context (see that entry point).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Argument errors are detected on the host before anything is launched and
 *     returned synchronously. fwd/bwd are asynchronous: a device-side failure
 *     (a bounded wait that ran out) is recorded in the workspace and reported
 *     by inkling_rel_attn_last_device_error().
 *   - fwd/bwd assume well-formed positions (see inkling_rel_attn_validate);
 *     on malformed positions they stay memory-safe but their result is
 *     unspecified.
 *   - Masked keys are multiplied by an exact zero weight inside the tensor-core
 *     products, so K/V rows at masked or padded positions must hold finite
 *     values (NaN/Inf there would propagate).
 */
#ifndef INKLING_REL_ATTN_H
#define INKLING_REL_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    INKLING_OK = 0,
    INKLING_ERR_INVALID_ARG = 1,          /* null / misaligned pointer, bad size, workspace too small */
    INKLING_ERR_UNSUPPORTED = 2,          /* valid request outside what the kernels implement */
    INKLING_ERR_MALFORMED_POSITIONS = 3,  /* validate(): masks / positions break the preconditions */
    INKLING_ERR_TIMEOUT = 4,              /* a device-side bounded wait ran out */
    INKLING_ERR_CUDA = 5                  /* a CUDA runtime / driver call failed */
} inkling_status;

/*
 * Problem sizes (Inkling2FlexAttention(head_dim, window) plus the tensor shapes
 * of its forward()):
 *   batch        B
 *   seq_q        S     local query rows
 *   seq_k        Skv   key columns (global under context parallelism; = S otherwise)
 *   heads_q      Hq    query heads
 *   heads_kv     Hkv   key/value heads, Hq % Hkv == 0 (grouped-query attention)
 *   head_dim     D     64 or 128
 *   rel_extent   R     width of each profiles row, a multiple of 8 (0 allowed)
 *   window       W     sliding window (keys with i_g - j < W); 0 = full causal
 *   query_offset       global column of local query row 0; 0 without CP
 * Size limits (INKLING_ERR_UNSUPPORTED beyond them): S, Skv, query_offset, B, R,
 * W < 2^30; Hq < 65536; the tile grids below 2^31 CTAs; and, when R > 0,
 * B * Hq * S below 2^31 - 256 (the backward addresses profile rows as int32).
 */
typedef struct {
    int64_t batch, seq_q, seq_k, heads_q, heads_kv, head_dim, rel_extent, window, query_offset;
} inkling_rel_attn_dims;

/* Bytes of device workspace needed by fwd (backward = 0) or bwd (backward = 1)
 * and by validate. Returns 0 when dims is NULL or malformed. */
size_t inkling_rel_attn_workspace_size(const inkling_rel_attn_dims* dims, int backward);

/*
 * Checks the preconditions that fwd/bwd assume (SYNCHRONOUS: waits on stream).
 *   valid [B,S], key_valid [B,Skv] (uint8 0/1; key_valid NULL = valid, needs
 *   Skv == S and query_offset == 0), positions [B,S], key_positions [B,Skv]
 *   (int32; NULL defaults as in fwd).
 * Conditions (from the forward's argument notes: every batch row holds a slice
 * of one contiguous run of real tokens, their global positions are consecutive,
 * and positions restart at each document):
 *   - the valid columns of each row form one contiguous span (same for key_valid);
 *   - along valid columns each position is the previous one plus one, or 0
 *     (a new document); valid positions are >= 0;
 *   - on the columns the query slice shares with the key stream (key column
 *     query_offset + i), valid and positions agree with key_valid and key_positions.
 * Returns INKLING_OK, INKLING_ERR_MALFORMED_POSITIONS, or an argument / CUDA error.
 */
inkling_status inkling_rel_attn_validate(const inkling_rel_attn_dims* dims,
                                         const uint8_t* valid, const uint8_t* key_valid,
                                         const int32_t* positions, const int32_t* key_positions,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward (ASYNCHRONOUS on stream).
 *   q        [B,S,Hq,D]   bf16        k, v [B,Skv,Hkv,D] bf16
 *   profiles [B,Hq,S,R]   bf16        sink [B,S,Hq] fp32
 *   valid    [B,S] uint8  key_valid [B,Skv] uint8 (NULL = valid)
 *   positions [B,S] int32 (NULL = query_offset + arange(S), one document)
 *   key_positions [B,Skv] int32 (NULL = positions when given, else arange(Skv))
 *   out      [B,S,Hq,D]   fp32 (written)
 *   lse      [B,S,Hq]     fp32 (written; natural log, sink included)
 * q, k, v, profiles, out and the workspace must be 16-byte aligned.
 */
inkling_status inkling_rel_attn_fwd(const inkling_rel_attn_dims* dims,
                                    const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const uint16_t* profiles, const float* sink,
                                    const uint8_t* valid, const uint8_t* key_valid,
                                    const int32_t* positions, const int32_t* key_positions,
                                    float* out, float* lse,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward (ASYNCHRONOUS on stream). Inputs as in fwd plus the forward's out and
 * lse, the upstream gradient dout [B,S,Hq,D] fp32 and an optional upstream
 * gradient of the returned log-sum-exp, dlse [B,S,Hq] fp32 (NULL = zero).
 * Writes (fp32, every element): dq [B,S,Hq,D], dk and dv [B,Skv,Hkv,D],
 * dprofiles [B,Hq,S,R], dsink [B,S,Hq]. dq, dk, dv and dprofiles must be
 * 16-byte aligned.
 */
inkling_status inkling_rel_attn_bwd(const inkling_rel_attn_dims* dims,
                                    const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const uint16_t* profiles, const float* sink,
                                    const uint8_t* valid, const uint8_t* key_valid,
                                    const int32_t* positions, const int32_t* key_positions,
                                    const float* out, const float* lse,
                                    const float* dout, const float* dlse,
                                    float* dq, float* dk, float* dv, float* dprofiles, float* dsink,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward without a caller-provided workspace, for callers that cannot
 * allocate device memory: code that only receives its input and output
 * buffers from a host framework (a plugin or custom-operator interface with no
 * allocator to call), or code that must not call cudaMalloc because it can
 * synchronise the device and stall unrelated work. Same arguments and results
 * as inkling_rel_attn_fwd, minus the workspace; this call allocates nothing
 * (no cudaMalloc / cudaFree, no allocating library routine).
 * Not a counterpart of anything on the Inkling2 pages: an addition of this
 * library.
 *   - Scratch lives in one 4 MiB array of device memory inside the library,
 *     present on every GPU that loads it until the process exits. The forward
 *     needs about 8.5 bytes per (batch, query) token, so B * S up to roughly
 *     480,000 fits; larger problems return INKLING_ERR_UNSUPPORTED.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Every call on a device shares the array and it keeps the last call's
 *     contents: calls that overlap on the GPU (other streams, other host
 *     threads) race on it, so serialise them.
 *   - The address is cached per CUDA context (by the context's
 *     process-unique id), so a context created after cudaDeviceReset, or a
 *     non-primary context the caller made current, gets its own lookup; that
 *     lookup is again a first call and belongs before any stream capture.
 *   - A device-side wait that runs out is recorded at the start of that array;
 *     inkling_rel_attn_fwd_noalloc_last_device_error() reads (and clears) it.
 *     The outputs of such a call are unspecified.
 */
inkling_status inkling_rel_attn_fwd_noalloc(const inkling_rel_attn_dims* dims,
                                            const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                            const uint16_t* profiles, const float* sink,
                                            const uint8_t* valid, const uint8_t* key_valid,
                                            const int32_t* positions, const int32_t* key_positions,
                                            float* out, float* lse, void* stream);

/*
 * Context parallelism (the forward's query_offset / key_valid / key_positions
 * arguments, whose key side is global under CP, on the Inkling2FlexAttention
 * page): merges a second result for the same query rows, computed over a key
 * set disjoint from the first one, into the first (ASYNCHRONOUS on stream):
 *   lse = log(exp(lse) + exp(lse_part))
 *   out = out * exp(lse_old - lse) + out_part * exp(lse_part - lse)
 * out, out_part: [rows, head_dim] fp32 (rows = B * S * Hq, 16-byte aligned);
 * lse, lse_part: [rows] fp32, natural log. out / lse are updated in place; the
 * sink must be counted in exactly one of the two parts (the other passes a sink
 * of -inf). A row with both lse at -inf stays out = 0, lse = -inf.
 * head_dim 64 or 128; INKLING_ERR_INVALID_ARG for null or misaligned pointers.
 */
inkling_status inkling_rel_attn_merge(int64_t rows, int64_t head_dim, float* out, float* lse,
                                      const float* out_part, const float* lse_part, void* stream);

/* SYNCHRONOUS: waits on stream, returns INKLING_ERR_TIMEOUT if a kernel of the
 * last fwd/bwd call on this workspace gave up a bounded wait (and clears the
 * record), INKLING_OK otherwise. */
inkling_status inkling_rel_attn_last_device_error(void* workspace, void* stream);

/* SYNCHRONOUS: the same check for inkling_rel_attn_fwd_noalloc, whose device
 * error word lives in the library's static scratch array of the current CUDA
 * context: waits on stream, returns INKLING_ERR_TIMEOUT if a kernel of the last
 * no-allocation forward gave up a bounded wait (and clears the record),
 * INKLING_OK otherwise. Like that entry point, it allocates nothing and has no
 * counterpart on the Inkling2 pages. */
inkling_status inkling_rel_attn_fwd_noalloc_last_device_error(void* stream);

/* Diagnostic: runs one kernel whose bounded wait is on an mbarrier that nothing
 * arrives on, with a limit of `timeout_us` microseconds, and returns the
 * status the host reads back (INKLING_ERR_TIMEOUT when the guard works).
 * SYNCHRONOUS. Needs 16 bytes of workspace. */
inkling_status inkling_rel_attn_selftest_wait_timeout(uint32_t timeout_us, void* workspace,
                                                      size_t workspace_bytes, void* stream);

/* Diagnostic: sets the limit of the attention kernels' pipeline waits (every wait
 * of a CTA on its copies, its tensor-core products and its other warps) for the
 * fwd / bwd calls that follow, in nanoseconds; 0 restores the default (2 s).
 * When a wait runs out, the CTA records the site in the workspace's error word
 * (read by inkling_rel_attn_last_device_error), stops, and drains what it has in
 * flight before it exits; those drain waits always keep the default limit.
 * Limits below 20 us are polled without sleeping, so a limit of 1 ns makes every
 * wait that does not succeed at its first test run out (a CTA's first wait, for
 * its Q tile, always does) and exercises that path. Host-side, not thread-safe. */
inkling_status inkling_rel_attn_set_wait_timeout_ns(uint64_t timeout_ns);

/* Diagnostic: evaluates, on the device, the FMA-pipe power of two the forward
 * kernel uses for a share of its softmax exponentials (range reduction
 * t = n + f, a fitted cubic for 2^f, n added to the exponent field):
 * out[k] = 2^t[k] for k < n, inputs clamped to >= -125. `t` and `out` are device
 * buffers of n floats owned by the caller. Returns INKLING_ERR_INVALID_ARG for
 * null pointers or n < 0, INKLING_ERR_CUDA on a launch error; asynchronous. */
inkling_status inkling_rel_attn_selftest_exp2(const float* t, float* out, int64_t n, void* stream);

/*
 * Diagnostic timing hook. While `events` is non-NULL, each later fwd/bwd call
 * records events[2k] just before and events[2k+1] just after its k-th kernel
 * launch (k < n_pairs) on the call's stream; `events` holds cudaEvent_t
 * handles owned by the caller. Kernel order: fwd = key span, row bounds,
 * attention; bwd = key span, row bounds, preprocessing, dprofiles zeroing,
 * dK/dV/dprofiles, dQ. Pass NULL to switch it off. Host-side only, not
 * thread-safe; returns INKLING_ERR_INVALID_ARG when n_pairs < 0.
 */
inkling_status inkling_rel_attn_set_timing_events(void* const* events, int n_pairs);

/* Description of the last CUDA runtime error an entry point of the calling
 * thread ran into (behind an INKLING_ERR_CUDA status); "no error" if none. */
const char* inkling_rel_attn_last_cuda_error(void);

/* Static description of a status code. */
const char* inkling_status_string(inkling_status status);

#ifdef __cplusplus
}
#endif

#endif /* INKLING_REL_ATTN_H */
