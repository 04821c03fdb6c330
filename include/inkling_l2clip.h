/*
 * inkling_l2clip.h -- C ABI of L2Clip in libinkling_rel_attn.so (same library,
 * status codes and conventions as inkling_rel_attn.h).
 *
 * The operation is the per-head clipping that Inkling2 applies to q and k
 * ahead of the attention, as documented on the NVIDIA NeMo AutoModel API page
 * "nemo_automodel.components.models.inkling2.layers": L2Clip(heads, width,
 * threshold, learned_scale) clips each head's vector by its L2 norm, with
 * optional learned per-channel scales before the clip, and L2Clip.forward(x
 * [batch, sequence, heads, head_dim], tau [batch, sequence]) applies the
 * optional tau as a length scaling after the clip and returns x's dtype. The
 * page prints no formula; the library computes the plainest reading, per
 * (b, s, h) vector:
 *   z = x * scale[h, :]                       (scale NULL: z = x)
 *   y = z * min(1, threshold / ||z||_2) * tau[b, s]   (tau NULL: no length scaling)
 * in FP32, y rounded to BF16 (round to nearest even).
 * The backward returns the gradients of sum(dy * y):
 *   c = min(1, threshold / ||z||); at ||z|| > threshold
 *   dz = tau * c * (dy - ((z . dy) / ||z||^2) z), else dz = tau * dy;
 *   dx = dz * scale;  dscale[h, :] = sum over (b, s) of dz * x;
 *   dtau[b, s] = sum over (h, d) of dy * z * c.
 * dscale and dtau are summed in a fixed order (deterministic).
 *
 * Layouts (dense, row-major, device memory owned by the caller; every tensor
 * pointer 16-byte aligned): x, y [B, S, H, D] BF16 bit patterns; dy, dx
 * [B, S, H, D] FP32; scale, dscale [H, D] FP32; tau, dtau [B, S] FP32.
 * Errors: INKLING_ERR_INVALID_ARG for null / misaligned pointers, negative
 * sizes, a threshold that is negative or not a number, dscale without scale or
 * the reverse (likewise dtau / tau), or a workspace that is too small;
 * INKLING_ERR_UNSUPPORTED for head_dim other than 64 / 128 or B * S * H >= 2^40.
 * Both calls are asynchronous on `stream`.
 */
#ifndef INKLING_L2CLIP_H
#define INKLING_L2CLIP_H

#include <stddef.h>
#include <stdint.h>

#include "inkling_rel_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int64_t batch;     /* B */
    int64_t seq;       /* S */
    int64_t heads;     /* H */
    int64_t head_dim;  /* D: 64 or 128 */
    double threshold;  /* clipping radius, >= 0 */
} inkling_l2clip_dims;

/* Device workspace bytes of the backward (the forward needs none); 0 on bad dims. */
size_t inkling_l2clip_workspace_size(const inkling_l2clip_dims* dims);

inkling_status inkling_l2clip_fwd(const inkling_l2clip_dims* dims, const uint16_t* x, const float* scale,
                                  const float* tau, uint16_t* y, void* stream);

inkling_status inkling_l2clip_bwd(const inkling_l2clip_dims* dims, const uint16_t* x, const float* scale,
                                  const float* tau, const float* dy, float* dx, float* dscale, float* dtau,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * L2Clip of q fused into the learned-relative attention (inkling_rel_attn.h): the
 * clipping Inkling2 applies to q ahead of the attention (the q_l2_clip attribute of
 * Inkling2Attention on the "nemo_automodel.components.models.inkling2.attention"
 * page; L2Clip.forward(x, tau) on the "...inkling2.layers" page), done inside the
 * attention kernels instead of as a pass of its own. Same arithmetic as
 * inkling_l2clip_fwd / _bwd above with H = heads_q, D = head_dim:
 *
 * inkling_rel_attn_fwd_qclip: x [B,S,Hq,D] BF16 is the unclipped q. Each query tile
 *   is clipped in shared memory as soon as it is loaded, y = z min(1, threshold /
 *   |z|) tau (z = x * clip_scale), rounded to BF16, and used for the attention; y is
 *   also stored to q_clipped [B,S,Hq,D] BF16 for the backward. Every other argument
 *   and result as in inkling_rel_attn_fwd.
 * inkling_rel_attn_bwd_qclip: takes x and the forward's q_clipped; the attention
 *   gradients are those of inkling_rel_attn_bwd with q = q_clipped, except that the
 *   dQ kernel turns the query gradient into the gradient of x through the clip
 *   (written to dx [B,S,Hq,D] FP32), and writes the parts of dclip_scale [Hq,D] and
 *   dtau [B,S] that a final fixed-order sum adds up (each NULL exactly when its
 *   parameter is NULL).
 * clip_scale [Hq,D] and tau [B,S] FP32 or NULL; threshold >= 0 and finite.
 * Workspace: inkling_rel_attn_qclip_workspace_size(dims, backward) bytes (the
 * forward's equals inkling_rel_attn_workspace_size's). Errors as in the unfused
 * calls, plus INKLING_ERR_INVALID_ARG for a bad threshold or a NULL q_clipped / x.
 * Both asynchronous on `stream`.
 */
size_t inkling_rel_attn_qclip_workspace_size(const inkling_rel_attn_dims* dims, int backward);

inkling_status inkling_rel_attn_fwd_qclip(const inkling_rel_attn_dims* dims, double threshold,
                                          const float* clip_scale, const float* tau, const uint16_t* x,
                                          const uint16_t* k, const uint16_t* v, const uint16_t* profiles,
                                          const float* sink, const uint8_t* valid, const uint8_t* key_valid,
                                          const int32_t* positions, const int32_t* key_positions,
                                          uint16_t* q_clipped, float* out, float* lse, void* workspace,
                                          size_t workspace_bytes, void* stream);

inkling_status inkling_rel_attn_bwd_qclip(const inkling_rel_attn_dims* dims, double threshold,
                                          const float* clip_scale, const float* tau, const uint16_t* x,
                                          const uint16_t* q_clipped, const uint16_t* k, const uint16_t* v,
                                          const uint16_t* profiles, const float* sink, const uint8_t* valid,
                                          const uint8_t* key_valid, const int32_t* positions,
                                          const int32_t* key_positions, const float* out, const float* lse,
                                          const float* dout, const float* dlse, float* dx, float* dk, float* dv,
                                          float* dprofiles, float* dsink, float* dclip_scale, float* dtau,
                                          void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* INKLING_L2CLIP_H */
