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

#ifdef __cplusplus
}
#endif

#endif /* INKLING_L2CLIP_H */
