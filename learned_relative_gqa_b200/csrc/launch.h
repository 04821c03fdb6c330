// launch.h -- host-side launchers of the CUDA path (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace ira {

cudaError_t launch_kspan(const uint8_t* key_valid, int B, int Skv, int2* kspan, cudaStream_t st);
cudaError_t launch_bounds(const uint8_t* valid, const int32_t* positions, const int2* kspan, int B, int S,
                          int q_off, int W, int2* row_bounds, TileBounds* tiles, cudaStream_t st);
cudaError_t launch_validate(const uint8_t* valid, const uint8_t* key_valid, const int32_t* positions,
                            const int32_t* key_positions, int B, int S, int Skv, int q_off,
                            int key_pos_from_query, int* ctl, int* edges, cudaStream_t st);
cudaError_t launch_bwd_prep(int D, const float* out, const float* lse, const float* sink, const float* dout,
                            const float* dlse, int B, int S, int Hq, float* dsink, __nv_bfloat16* dout_bf16,
                            float* lse2t, float* dvt, cudaStream_t st);
cudaError_t launch_dprof_zero(const int2* row_bounds, int B, int S, int Hq, int R, int q_off, float* dprof,
                              cudaStream_t st);
cudaError_t launch_selftest_wait(uint64_t timeout_ns, int* err, cudaStream_t st);
// Context parallelism: merges a partial result (out_part, lse_part) over a disjoint key
// set into (out, lse), rows = B * S * Hq of D floats.
cudaError_t launch_merge(float* out, float* lse, const float* out_part, const float* lse_part, int64_t rows, int D,
                         cudaStream_t st);

// Generic FlexAttention variant: block positions from EOS tokens / fixed blocks, the
// backward preprocessing of BF16 [B, H, S, D] out / dout rows, and the per-head sum of
// the per-row sink gradients ([B, Hq, S] -> [Hq]).
cudaError_t launch_flex_positions(const int64_t* tokens, int64_t eos_id, int B, int S, int fbs, int32_t* positions,
                                  cudaStream_t st);
cudaError_t launch_flex_bwd_prep(int D, const uint16_t* out, const uint16_t* dout, const float* lse, const float* sink,
                                 int64_t sink_sb, int64_t sink_ss, int64_t sink_sh, int B, int S, int Hq,
                                 float* dsink_rows, float* lse2t, float* dvt, cudaStream_t st);
cudaError_t launch_flex_dsink_reduce(const float* dsink_rows, int B, int S, int Hq, float* dsink_weights,
                                     cudaStream_t st);
cudaError_t launch_selftest_exp2(const float* t, float* out, int64_t n, cudaStream_t st);
// L2Clip backward reduction (l2clip.cu): dtau[t] = sum_h dtau_part[t, h], dscale[j] = sum
// over chunks of dscale_part[chunk, j]; fixed order, null outputs skipped.
cudaError_t launch_l2clip_reduce(const float* dtau_part, int64_t T, int H, float* dtau, const float* dscale_part,
                                 int64_t nchunks, int64_t HD, float* dscale, cudaStream_t st);

// Forward attention. tm_q: {D, Hq, S, B} box {64,1,128,1}; tm_k / tm_v: {D, Hkv, Skv, B} box {64,1,64,1}.
cudaError_t launch_fwd(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                       const AttnParams& p, cudaStream_t st);
// The same with the L2Clip of q fused in (p.q_clipped set): tm_q maps the unclipped q,
// tm_qc the clipped q it stores (same geometry).
cudaError_t launch_fwd_qclip(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const CUtensorMap& tm_qc, const AttnParams& p, cudaStream_t st);

// Backward attention. dkdv: tm_k / tm_v box {64,1,128,1}, tm_q / tm_do box {64,1,64,1},
// tm_band: profiles as {R, B*Hq*S} with box {136, 8} (unused when R == 0).
cudaError_t launch_bwd_dkdv(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                            const CUtensorMap& tm_do, const CUtensorMap& tm_band, const AttnParams& p,
                            cudaStream_t st);
// dq: tm_q / tm_do box {64,1,128,1}, tm_k / tm_v box {64,1,64,1}.
cudaError_t launch_bwd_dq(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const CUtensorMap& tm_do, const AttnParams& p, cudaStream_t st);

}  // namespace ira
