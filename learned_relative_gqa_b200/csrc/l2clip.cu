// l2clip.cu -- L2Clip (include/inkling_l2clip.h): per-head clipping of q / k head
// vectors, with optional learned per-channel scales before the clip and a per-token
// length scale after it ("nemo_automodel.components.models.inkling2.layers",
// L2Clip and L2Clip.forward), forward and backward, and their C entry points.
//
// Both kernels are HBM-bound streams: one warp per head vector of D = 64 / 128
// values (2 or 4 per lane), the norm and the dot product reduced with shuffles; the
// forward loads four vectors before it reduces any, the backward one vector ahead.
// Forward: 2 bytes read + 2 bytes written per element. Backward: x (2 B) and dy
// (4 B) read, dx (4 B) written per element; each warp walks one head over a chunk
// of tokens, so its share of dscale stays in registers; per-(token, head) parts of
// dtau and per-(chunk, head) parts of dscale go to the workspace and a second
// kernel sums them in a fixed order.
#include <cmath>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "inkling_l2clip.h"

namespace ira {
cudaError_t note_cuda_error(cudaError_t e);  // host.cu: keeps the error for inkling_rel_attn_last_cuda_error
}

namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kTargetWarps = 148 * 64;  // enough warps in flight to cover HBM latency

template <int PER>
__device__ __forceinline__ void load_bf16(const uint16_t* p, float (&v)[PER]) {
    if constexpr (PER == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xFFFF0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
        v[0] = __uint_as_float(u << 16);
        v[1] = __uint_as_float(u & 0xFFFF0000u);
    }
}

template <int PER>
__device__ __forceinline__ void load_f32(const float* p, float (&v)[PER]) {
    if constexpr (PER == 4) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    } else {
        const float2 u = *reinterpret_cast<const float2*>(p);
        v[0] = u.x; v[1] = u.y;
    }
}

template <int PER>
__device__ __forceinline__ void store_f32(float* p, const float (&v)[PER]) {
    if constexpr (PER == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    }
}

__device__ __forceinline__ uint32_t pack_rne(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&b);
}

template <int PER>
__device__ __forceinline__ void store_bf16(uint16_t* p, const float (&v)[PER]) {
    if constexpr (PER == 4) {
        *reinterpret_cast<uint2*>(p) = make_uint2(pack_rne(v[0], v[1]), pack_rne(v[2], v[3]));
    } else {
        *reinterpret_cast<uint32_t*>(p) = pack_rne(v[0], v[1]);
    }
}

constexpr int kRows = 4;  // head vectors a warp loads before it reduces any (forward)

// y = (x * scale) * min(1, thr / ||x * scale||) * tau. One warp per token: it walks the
// token's H head vectors (contiguous in memory), kRows at a time, so neither the head
// nor the token index is ever divided out of a row index.
template <int D>
__global__ void l2clip_fwd_kernel(const uint16_t* __restrict__ x, const float* __restrict__ scale,
                                  const float* __restrict__ tau, float thr, int64_t T, int H,
                                  uint16_t* __restrict__ y) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t nw = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t t = blockIdx.x * int64_t(blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nw) {
        const float tv = tau ? tau[t] : 1.f;
        const uint16_t* xt = x + t * H * D + lane * PER;
        uint16_t* yt = y + t * H * D + lane * PER;
        for (int h0 = 0; h0 < H; h0 += kRows) {
            float z[kRows][PER];
#pragma unroll
            for (int u = 0; u < kRows; ++u)
                if (h0 + u < H) load_bf16<PER>(xt + (h0 + u) * D, z[u]);
            float ss[kRows];
#pragma unroll
            for (int u = 0; u < kRows; ++u) {
                ss[u] = 0.f;
                if (h0 + u >= H) continue;
                if (scale) {
                    float s[PER];
                    load_f32<PER>(scale + size_t(h0 + u) * D + lane * PER, s);
#pragma unroll
                    for (int e = 0; e < PER; ++e) z[u][e] *= s[e];
                }
#pragma unroll
                for (int e = 0; e < PER; ++e) ss[u] = fmaf(z[u][e], z[u][e], ss[u]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int u = 0; u < kRows; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
#pragma unroll
            for (int u = 0; u < kRows; ++u) {
                if (h0 + u >= H) continue;
                const float n = sqrtf(ss[u]);
                const float c = (n > thr ? thr / n : 1.f) * tv;
#pragma unroll
                for (int e = 0; e < PER; ++e) z[u][e] *= c;
                store_bf16<PER>(yt + (h0 + u) * D, z[u]);
            }
        }
    }
}

// Backward: warp (chunk, h) walks tokens [chunk * tpc, (chunk + 1) * tpc) of head h.
// Writes dx, the per-(token, head) part of dtau (= c * (z . dy)) and the warp's part
// of dscale[h, :] (= sum of dz * x over its tokens).
template <int D>
__global__ void l2clip_bwd_kernel(const uint16_t* __restrict__ x, const float* __restrict__ scale,
                                  const float* __restrict__ tau, float thr, const float* __restrict__ dy,
                                  int64_t T, int H, int64_t tpc, int64_t nchunks, float* __restrict__ dx,
                                  float* __restrict__ dtau_part, float* __restrict__ dscale_part) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t gw = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (gw >= nchunks * H) return;  // whole warps leave together
    const int h = int(gw % H);
    const int64_t chunk = gw / H;
    const int64_t t0 = chunk * tpc;
    const int64_t t1 = t0 + tpc < T ? t0 + tpc : T;
    float s[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) s[e] = 1.f;
    if (scale) load_f32<PER>(scale + size_t(h) * D + lane * PER, s);
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    // software pipeline: the next token's x and dy are loaded before this one is reduced
    float xn[PER], gn[PER];
    if (t0 < t1) {
        load_bf16<PER>(x + (t0 * H + h) * D + lane * PER, xn);
        load_f32<PER>(dy + (t0 * H + h) * D + lane * PER, gn);
    }
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t r = t * H + h;
        float xv[PER], g[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) { xv[e] = xn[e]; g[e] = gn[e]; }
        if (t + 1 < t1) {
            load_bf16<PER>(x + (r + H) * D + lane * PER, xn);
            load_f32<PER>(dy + (r + H) * D + lane * PER, gn);
        }
        float z[PER], ss = 0.f, zg = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            z[e] = xv[e] * s[e];
            ss = fmaf(z[e], z[e], ss);
            zg = fmaf(z[e], g[e], zg);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            zg += __shfl_xor_sync(0xffffffffu, zg, o);
        }
        const float n = sqrtf(ss);
        const bool clipped = n > thr;
        const float c = clipped ? thr / n : 1.f;
        const float k = clipped ? zg / (n * n) : 0.f;  // n > thr >= 0 when clipped
        const float tv = tau ? tau[t] : 1.f;
        float d[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const float dz = tv * c * (g[e] - k * z[e]);
            d[e] = dz * s[e];
            acc[e] = fmaf(dz, xv[e], acc[e]);
        }
        store_f32<PER>(dx + r * D + lane * PER, d);
        if (dtau_part && lane == 0) dtau_part[r] = c * zg;
    }
    if (dscale_part) store_f32<PER>(dscale_part + (chunk * H + h) * D + lane * PER, acc);
}

// dtau[t] = sum over h of the parts (threads [0, T)); dscale[j] = sum over chunks of
// the parts (threads [T, T + H * D)); fixed summation order, four partial sums per
// thread so that four loads are in flight.
__global__ void l2clip_reduce_kernel(const float* __restrict__ dtau_part, int64_t T, int H,
                                     float* __restrict__ dtau, const float* __restrict__ dscale_part,
                                     int64_t nchunks, int64_t HD, float* __restrict__ dscale) {
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < T) {
        if (dtau) {
            const float* q = dtau_part + i * H;
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            int h = 0;
            for (; h + 3 < H; h += 4) {
                a0 += q[h];
                a1 += q[h + 1];
                a2 += q[h + 2];
                a3 += q[h + 3];
            }
            for (; h < H; ++h) a0 += q[h];
            dtau[i] = (a0 + a1) + (a2 + a3);
        }
    } else if (i - T < HD) {
        if (dscale) {
            const float* q = dscale_part + (i - T);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            int64_t c = 0;
            for (; c + 3 < nchunks; c += 4) {
                a0 += q[c * HD];
                a1 += q[(c + 1) * HD];
                a2 += q[(c + 2) * HD];
                a3 += q[(c + 3) * HD];
            }
            for (; c < nchunks; ++c) a0 += q[c * HD];
            dscale[i - T] = (a0 + a1) + (a2 + a3);
        }
    }
}

// Work split of the backward: chunks of tokens per head.
struct Split {
    int64_t T, tpc, nchunks;
    size_t dtau_off, dscale_off, total;
};

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

Split split_of(const inkling_l2clip_dims* d) {
    Split sp{};
    sp.T = d->batch * d->seq;
    const int64_t want = (kTargetWarps + d->heads - 1) / d->heads;
    const int64_t n = sp.T < want ? sp.T : want;
    sp.tpc = n > 0 ? (sp.T + n - 1) / n : 1;
    sp.nchunks = sp.T > 0 ? (sp.T + sp.tpc - 1) / sp.tpc : 0;
    sp.dtau_off = 0;
    sp.dscale_off = up256(size_t(sp.T) * d->heads * 4);
    sp.total = sp.dscale_off + up256(size_t(sp.nchunks) * d->heads * d->head_dim * 4);
    if (sp.total == 0) sp.total = 256;
    return sp;
}

inkling_status check(const inkling_l2clip_dims* d) {
    if (!d) return INKLING_ERR_INVALID_ARG;
    if (d->batch < 0 || d->seq < 0 || d->heads <= 0 || !(d->threshold >= 0.0)) return INKLING_ERR_INVALID_ARG;
    if (d->head_dim != 64 && d->head_dim != 128) return INKLING_ERR_UNSUPPORTED;
    if (d->heads >= (int64_t(1) << 20) || d->batch >= (int64_t(1) << 30) || d->seq >= (int64_t(1) << 30) ||
        d->batch * d->seq * d->heads >= (int64_t(1) << 40))
        return INKLING_ERR_UNSUPPORTED;
    return INKLING_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A named NVTX range over an entry point (a no-op when no profiler is attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

inkling_status status_of(cudaError_t e) { return ira::note_cuda_error(e) == cudaSuccess ? INKLING_OK : INKLING_ERR_CUDA; }

}  // namespace

namespace ira {
// dtau[t] = sum over h of dtau_part[t, h] (t < T) and dscale[j] = sum over chunks of
// dscale_part[chunk, j] (j < HD), in a fixed order; either output may be null. Used by the
// L2Clip of q fused into the attention backward as well.
cudaError_t launch_l2clip_reduce(const float* dtau_part, int64_t T, int H, float* dtau, const float* dscale_part,
                                 int64_t nchunks, int64_t HD, float* dscale, cudaStream_t st) {
    const int64_t n = T + HD;
    if (n == 0) return cudaSuccess;
    l2clip_reduce_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(dtau_part, T, H, dtau, dscale_part, nchunks, HD,
                                                                   dscale);
    return cudaGetLastError();
}
}  // namespace ira

extern "C" {

size_t inkling_l2clip_workspace_size(const inkling_l2clip_dims* dims) {
    if (check(dims) != INKLING_OK) return 0;
    return split_of(dims).total;
}

inkling_status inkling_l2clip_fwd(const inkling_l2clip_dims* dims, const uint16_t* x, const float* scale,
                                  const float* tau, uint16_t* y, void* stream) {
    NvtxRange nvtx_range("inkling_l2clip_fwd");
    inkling_status s = check(dims);
    if (s != INKLING_OK) return s;
    const int64_t rows = dims->batch * dims->seq * dims->heads;
    if (rows > 0 && (!x || !y)) return INKLING_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(scale) || !aligned16(tau)) return INKLING_ERR_INVALID_ARG;
    if (rows == 0) return INKLING_OK;
    const int64_t T = dims->batch * dims->seq;
    const int64_t want = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int blocks = int(want < 148 * 16 ? want : 148 * 16);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float thr = float(dims->threshold);
    if (dims->head_dim == 128)
        l2clip_fwd_kernel<128><<<blocks, 32 * kWarpsPerBlock, 0, st>>>(x, scale, tau, thr, T, int(dims->heads), y);
    else
        l2clip_fwd_kernel<64><<<blocks, 32 * kWarpsPerBlock, 0, st>>>(x, scale, tau, thr, T, int(dims->heads), y);
    return status_of(cudaGetLastError());
}

inkling_status inkling_l2clip_bwd(const inkling_l2clip_dims* dims, const uint16_t* x, const float* scale,
                                  const float* tau, const float* dy, float* dx, float* dscale, float* dtau,
                                  void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("inkling_l2clip_bwd");
    inkling_status s = check(dims);
    if (s != INKLING_OK) return s;
    if ((scale == nullptr) != (dscale == nullptr) || (tau == nullptr) != (dtau == nullptr))
        return INKLING_ERR_INVALID_ARG;
    const int64_t rows = dims->batch * dims->seq * dims->heads;
    if (rows > 0 && (!x || !dy || !dx)) return INKLING_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || !aligned16(scale) || !aligned16(tau) ||
        !aligned16(dscale) || !aligned16(dtau))
        return INKLING_ERR_INVALID_ARG;
    const Split sp = split_of(dims);
    if (!workspace || !aligned16(workspace) || workspace_bytes < sp.total) return INKLING_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t HD = dims->heads * dims->head_dim;
    if (rows == 0) {  // no tokens: zero gradient for the learned scales
        return dscale ? status_of(cudaMemsetAsync(dscale, 0, size_t(HD) * 4, st)) : INKLING_OK;
    }
    auto* base = static_cast<uint8_t*>(workspace);
    float* dtau_part = dtau ? reinterpret_cast<float*>(base + sp.dtau_off) : nullptr;
    float* dscale_part = dscale ? reinterpret_cast<float*>(base + sp.dscale_off) : nullptr;
    const int64_t warps = sp.nchunks * dims->heads;
    const unsigned blocks = unsigned((warps + kWarpsPerBlock - 1) / kWarpsPerBlock);
    const float thr = float(dims->threshold);
    if (dims->head_dim == 128)
        l2clip_bwd_kernel<128><<<blocks, 32 * kWarpsPerBlock, 0, st>>>(x, scale, tau, thr, dy, sp.T, int(dims->heads),
                                                                      sp.tpc, sp.nchunks, dx, dtau_part, dscale_part);
    else
        l2clip_bwd_kernel<64><<<blocks, 32 * kWarpsPerBlock, 0, st>>>(x, scale, tau, thr, dy, sp.T, int(dims->heads),
                                                                     sp.tpc, sp.nchunks, dx, dtau_part, dscale_part);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess && (dtau || dscale)) {
        const int64_t n = sp.T + HD;
        l2clip_reduce_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(dtau_part, sp.T, int(dims->heads), dtau,
                                                                       dscale_part, sp.nchunks, HD, dscale);
        e = cudaGetLastError();
    }
    return status_of(e);
}

}  // extern "C"
