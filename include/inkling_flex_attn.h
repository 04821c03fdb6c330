/*
 * inkling_flex_attn.h -- C ABI of the generic FlexAttention variant in
 * libinkling_rel_attn.so (same library, same status codes and conventions as
 * inkling_rel_attn.h).
 *
 * The operation is the one documented on the NVIDIA NeMo AutoModel API page
 * "nemo_automodel.components.attention.flex_attention": the FlexAttention
 * module with attn_mask_type "causal" or "block_causal" (blocks delimited by
 * an EOS token), fixed_block_size, and forward(q, k, v, scale, sink_weights,
 * sliding_window, enable_gqa) on [B, H, S, D] tensors, returning an output of
 * q's dtype. It is the learned-relative attention of inkling_rel_attn.h with
 * no relative profiles, all tokens valid, one sink logit per head and the
 * documents derived from the tokens; it runs on the same kernels.
 *
 * Definition (b batch, h query head, g = h / (Hq / Hkv), i query, j key):
 *   doc(i)   = number of EOS tokens in tokens[b, 0 .. i-1]      (block_causal;
 *              the EOS belongs to the document it closes), 0 for "causal"
 *   allowed  = j <= i && doc(i) == doc(j)
 *              && (fixed_block_size == 0 || i / fixed_block_size == j / fixed_block_size)
 *              && (sliding_window == 0 || i - j < sliding_window)
 *   z_j      = scale * <q[b,h,i,:], k[b,g,j,:]>
 *   lse[b,h,i] = log(exp(sink_weights[h]) + sum_allowed exp(z_j))  (no sink term when NULL)
 *   out[b,h,i,:] = sum_allowed exp(z_j - lse) * v[b,g,j,:]
 * sliding_window counts the tokens a query sees including itself (the
 * forward describes it as a count of causal tokens per query); the page's
 * sliding-window mask mod (q_idx - kv_idx <= window) is sliding_window =
 * window + 1. The page applies `scale` when sink_weights is not set: with
 * sink weights the scale is head_dim^-0.5, and scale <= 0 also means
 * head_dim^-0.5. With enable_gqa == 0, heads_q must equal heads_kv.
 *
 * Layouts (dense, row-major, device memory owned by the caller):
 *   q, out, dout      [B, Hq, S, D]   BF16 bit patterns (uint16_t)
 *   k, v              [B, Hkv, S, D]  BF16
 *   sink_weights      [Hq]            FP32, or NULL (no sink)
 *   tokens            [B, S]          int64 token ids (block_causal only; else may be NULL)
 *   lse               [B, Hq, S]      FP32 (written by fwd, read by bwd)
 *   dq                [B, Hq, S, D]   FP32
 *   dk, dv            [B, Hkv, S, D]  FP32
 *   dsink_weights     [Hq]            FP32 (NULL when sink_weights is NULL)
 * Every tensor pointer must be 16-byte aligned.
 *
 * Errors: as in inkling_rel_attn.h. INKLING_ERR_INVALID_ARG for a null or
 * misaligned pointer, an unknown mask type, block_causal without tokens,
 * heads_q % heads_kv != 0, heads_q != heads_kv without enable_gqa, negative
 * sizes or a workspace that is too small; INKLING_ERR_UNSUPPORTED for head_dim
 * other than 64 / 128 or sizes beyond the limits of inkling_rel_attn.h.
 * fwd / bwd are asynchronous; device-side timeouts are read with
 * inkling_rel_attn_last_device_error() on the same workspace.
 */
#ifndef INKLING_FLEX_ATTN_H
#define INKLING_FLEX_ATTN_H

#include <stddef.h>
#include <stdint.h>

#include "inkling_rel_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    INKLING_FLEX_CAUSAL = 0,        /* attn_mask_type "causal" */
    INKLING_FLEX_BLOCK_CAUSAL = 1   /* attn_mask_type "block_causal": documents closed by eos_id */
} inkling_flex_mask_type;

typedef struct {
    int64_t batch;             /* B */
    int64_t seq;               /* S (queries and keys) */
    int64_t heads_q;           /* Hq */
    int64_t heads_kv;          /* Hkv */
    int64_t head_dim;          /* D: 64 or 128 */
    int64_t mask_type;         /* inkling_flex_mask_type */
    int64_t fixed_block_size;  /* 0 = none */
    int64_t sliding_window;    /* 0 = full causal history */
    int64_t eos_id;            /* block_causal only */
    int64_t enable_gqa;        /* nonzero: heads_q may be a multiple of heads_kv */
    double scale;              /* <= 0: head_dim^-0.5; ignored when sink_weights is given */
} inkling_flex_attn_dims;

/* Device workspace bytes for fwd (backward = 0) or bwd (backward = 1); 0 on bad dims. */
size_t inkling_flex_attn_workspace_size(const inkling_flex_attn_dims* dims, int backward);

/* Forward: out (BF16) and lse. Asynchronous on `stream`. */
inkling_status inkling_flex_attn_fwd(const inkling_flex_attn_dims* dims, const uint16_t* q, const uint16_t* k,
                                     const uint16_t* v, const float* sink_weights, const int64_t* tokens,
                                     uint16_t* out, float* lse, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* Backward of sum(dout * out): dq, dk, dv and dsink_weights (FP32), from the forward's
 * out and lse. Asynchronous on `stream`. */
inkling_status inkling_flex_attn_bwd(const inkling_flex_attn_dims* dims, const uint16_t* q, const uint16_t* k,
                                     const uint16_t* v, const float* sink_weights, const int64_t* tokens,
                                     const uint16_t* out, const float* lse, const uint16_t* dout, float* dq,
                                     float* dk, float* dv, float* dsink_weights, void* workspace,
                                     size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* INKLING_FLEX_ATTN_H */
