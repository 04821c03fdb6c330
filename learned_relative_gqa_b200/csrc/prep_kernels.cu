// prep_kernels.cu -- the O(B*S) kernels around the attention kernels:
//   * key span (first / last valid key column of each batch row),
//   * per-row allowed key range [lo, hi] and per-64-row tile summaries,
//   * the precondition checker behind inkling_rel_attn_validate,
//   * the backward preprocessing (row dot products, dsink, BF16 copy of dout,
//     log2-scaled lse),
//   * zeroing of the dprofiles entries that no allowed key reaches.
//
// Row range. Under the preconditions (one contiguous valid span per row,
// positions consecutive inside a document and restarting at 0), the keys a
// valid query row i (global column i_g) may attend form one interval:
//   lo = max(i_g - positions[i], first valid key, i_g - W + 1 if W > 0)
//   hi = min(i_g, last valid key)
// i_g - positions[i] is the column where the row's document starts
// (positions restart at every document, per the Inkling2FlexAttention.forward
// page), so the interval is exactly the causal, same-document, in-window,
// valid keys of the definition.
#include <algorithm>

#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace ira {

namespace {

__device__ __forceinline__ int warp_min(int v) {
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ int warp_max(int v) {
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ int warp_sum(int v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Merge of two results for the same query rows over disjoint key sets (context
// parallelism: the local keys first, the keys of the ranks before later), each
// normalised over its own keys with its own log-sum-exp:
//   lse = log(exp(lse_a) + exp(lse_b)),
//   out = out_a exp(lse_a - lse) + out_b exp(lse_b - lse),
// written over (out_a, lse_a). One warp per row, float4 accesses. A row whose
// parts are both empty (both lse -inf) keeps out = 0 and lse = -inf.
__global__ void merge_kernel(float* __restrict__ out_a, float* __restrict__ lse_a, const float* __restrict__ out_b,
                             const float* __restrict__ lse_b, int64_t rows, int D) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    for (int64_t r = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
        const float la = lse_a[r], lb = lse_b[r];
        const float m = fmaxf(la, lb);
        float wa = 0.f, wb = 0.f, l = m;
        if (m > -INFINITY) {
            const float ea = expf(la - m), eb = expf(lb - m);
            const float sum = ea + eb;
            wa = ea / sum;
            wb = eb / sum;
            l = m + logf(sum);
        }
        float4* oa = reinterpret_cast<float4*>(out_a + r * D);
        const float4* ob = reinterpret_cast<const float4*>(out_b + r * D);
        for (int c = lane; c < D / 4; c += 32) {
            float4 x = oa[c];
            const float4 y = ob[c];
            x.x = fmaf(x.x, wa, y.x * wb);
            x.y = fmaf(x.y, wa, y.y * wb);
            x.z = fmaf(x.z, wa, y.z * wb);
            x.w = fmaf(x.w, wa, y.w * wb);
            oa[c] = x;
        }
        __syncwarp();
        if (lane == 0) lse_a[r] = l;
    }
}

}  // namespace

// Bit 7 of each byte of the result is set where that byte of x is nonzero.
__device__ __forceinline__ uint32_t nonzero_bytes(uint32_t x) {
    return (((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x) & 0x80808080u;
}

// grid (B), block 512. Rows whose start is 16-byte aligned are read 16 bytes per
// thread and load (the whole row of a 8192-key batch in one round trip); the
// rest of a row (and unaligned rows) byte by byte.
__global__ void kspan_kernel(const uint8_t* __restrict__ key_valid, int Skv, int2* __restrict__ kspan) {
    const int b = blockIdx.x;
    const uint8_t* row = key_valid + size_t(b) * Skv;
    int first = 0x7FFFFFFF, last = -1;
    const int vec_end = (reinterpret_cast<uintptr_t>(row) & 15) == 0 ? (Skv & ~15) : 0;
#pragma unroll 4
    for (int j0 = threadIdx.x * 16; j0 < vec_end; j0 += blockDim.x * 16) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + j0));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t m = nonzero_bytes(w[u]);
            if (m) {  // little endian: byte t of the word is bits 8t..8t+7
                first = min(first, j0 + 4 * u + ((__ffs(int(m)) - 1) >> 3));
                last = max(last, j0 + 4 * u + ((31 - __clz(int(m))) >> 3));
            }
        }
    }
    for (int j = vec_end + threadIdx.x; j < Skv; j += blockDim.x) {
        if (row[j]) {
            first = min(first, j);
            last = max(last, j);
        }
    }
    __shared__ int sf[32], sl[32];
    first = warp_min(first);
    last = warp_max(last);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) { sf[w] = first; sl[w] = last; }
    __syncthreads();
    if (w == 0) {
        const int nw = blockDim.x >> 5;
        first = lane < nw ? sf[lane] : 0x7FFFFFFF;
        last = lane < nw ? sl[lane] : -1;
        first = warp_min(first);
        last = warp_max(last);
        if (lane == 0) kspan[b] = make_int2(first, last);
    }
}

// grid (ceil(S/64), B), block 64
__global__ void bounds_kernel(const uint8_t* __restrict__ valid, const int32_t* __restrict__ positions,
                              const int2* __restrict__ kspan, int S, int q_off, int W,
                              int2* __restrict__ row_bounds, TileBounds* __restrict__ tiles) {
    const int b = blockIdx.y, tile = blockIdx.x, r = threadIdx.x;
    const int i = tile * 64 + r;
    const int2 ks = kspan[b];
    int lo = kEmptyLo, hi = kEmptyHi;
    const bool in_range = i < S;
    if (in_range && valid[size_t(b) * S + i] && ks.x <= ks.y) {
        const int ig = q_off + i;
        const int pos = positions ? positions[size_t(b) * S + i] : ig;
        int l = max(ig - pos, ks.x);
        if (W > 0) l = max(l, ig - W + 1);
        const int h = min(ig, ks.y);
        if (l <= h) { lo = l; hi = h; }
    }
    if (in_range) row_bounds[size_t(b) * S + i] = make_int2(lo, hi);
    const bool ne = lo <= hi;
    int a_min_lo = ne ? lo : 0x7FFFFFFF, a_max_hi = ne ? hi : -0x7FFFFFFF;
    int a_max_lo = ne ? lo : -0x7FFFFFFF, a_min_hi = ne ? hi : 0x7FFFFFFF;
    int cnt = ne ? 1 : 0;
    a_min_lo = warp_min(a_min_lo);
    a_max_hi = warp_max(a_max_hi);
    a_max_lo = warp_max(a_max_lo);
    a_min_hi = warp_min(a_min_hi);
    cnt = warp_sum(cnt);
    __shared__ int red[2][5];
    const int w = r >> 5;
    if ((r & 31) == 0) {
        red[w][0] = a_min_lo; red[w][1] = a_max_hi; red[w][2] = a_max_lo; red[w][3] = a_min_hi; red[w][4] = cnt;
    }
    __syncthreads();
    if (r == 0) {
        TileBounds t;
        t.min_lo = min(red[0][0], red[1][0]);
        t.max_hi = max(red[0][1], red[1][1]);
        t.max_lo = max(red[0][2], red[1][2]);
        t.min_hi = min(red[0][3], red[1][3]);
        t.n_nonempty = red[0][4] + red[1][4];
        t.n_rows = min(64, S - tile * 64);
        t.pad0 = t.pad1 = 0;
        tiles[size_t(b) * gridDim.x + tile] = t;
    }
}

// Precondition checker. grid-stride over (b, column) of the longer of the two
// streams; counts violations in ctl[1] and rising edges of the valid masks.
__global__ void validate_kernel(const uint8_t* __restrict__ valid, const uint8_t* __restrict__ key_valid,
                                const int32_t* __restrict__ positions, const int32_t* __restrict__ key_positions,
                                int B, int S, int Skv, int q_off, int key_pos_from_query,
                                int* __restrict__ ctl, int* __restrict__ edges) {
    const int64_t T = S > Skv ? S : Skv;
    const int64_t n = int64_t(B) * T;
    int bad = 0;
    for (int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; t < n; t += int64_t(gridDim.x) * blockDim.x) {
        const int b = int(t / T), c = int(t % T);
        // query side
        if (c < S) {
            const size_t o = size_t(b) * S + c;
            const bool v = valid[o] != 0;
            const bool vp = c > 0 && valid[o - 1] != 0;
            if (v && !vp) atomicAdd(&edges[2 * b + 0], 1);
            const int p = positions ? positions[o] : q_off + c;
            if (v) {
                if (p < 0) ++bad;
                if (vp) {
                    const int pp = positions ? positions[o - 1] : q_off + c - 1;
                    if (!(p == pp + 1 || p == 0)) ++bad;
                }
            }
            const int j = q_off + c;
            if (j < Skv) {
                const size_t ok = size_t(b) * Skv + j;
                const bool kv = key_valid[ok] != 0;
                if (kv != v) ++bad;
                if (v) {
                    const int kp = key_positions ? key_positions[ok] : (key_pos_from_query ? p : j);
                    if (kp != p) ++bad;
                }
            } else if (v) {
                ++bad;  // a valid query outside the key stream
            }
        }
        // key side
        if (c < Skv) {
            const size_t o = size_t(b) * Skv + c;
            const bool v = key_valid[o] != 0;
            const bool vp = c > 0 && key_valid[o - 1] != 0;
            if (v && !vp) atomicAdd(&edges[2 * b + 1], 1);
            if (v) {
                auto kpos = [&](int col) {
                    if (key_positions) return key_positions[size_t(b) * Skv + col];
                    if (key_pos_from_query) return positions ? positions[size_t(b) * S + col] : q_off + col;
                    return col;
                };
                const int p = kpos(c);
                if (p < 0) ++bad;
                if (vp) {
                    const int pp = kpos(c - 1);
                    if (!(p == pp + 1 || p == 0)) ++bad;
                }
            }
        }
    }
    if (bad) atomicAdd(&ctl[1], bad);
}

// Backward preprocessing: one warp per (b, i, h) row.
template <int D>
__global__ void bwd_prep_kernel(const float* __restrict__ out, const float* __restrict__ lse,
                                const float* __restrict__ sink, const float* __restrict__ dout,
                                const float* __restrict__ dlse, int B, int S, int Hq,
                                float* __restrict__ dsink, __nv_bfloat16* __restrict__ dout_bf16,
                                float* __restrict__ lse2t, float* __restrict__ dvt) {
    constexpr int PER = D / 32;
    const int64_t nrows = int64_t(B) * S * Hq;
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t row = blockIdx.x * int64_t(blockDim.x >> 5) + (threadIdx.x >> 5); row < nrows; row += warps) {
        const float* o = out + row * D + lane * PER;
        const float* g = dout + row * D + lane * PER;
        float acc = 0.f;
        float gv[PER];
        if constexpr (PER == 4) {
            const float4 a = *reinterpret_cast<const float4*>(o);
            const float4 c = *reinterpret_cast<const float4*>(g);
            gv[0] = c.x; gv[1] = c.y; gv[2] = c.z; gv[3] = c.w;
            acc = a.x * c.x + a.y * c.y + a.z * c.z + a.w * c.w;
        } else {
            const float2 a = *reinterpret_cast<const float2*>(o);
            const float2 c = *reinterpret_cast<const float2*>(g);
            gv[0] = c.x; gv[1] = c.y;
            acc = a.x * c.x + a.y * c.y;
        }
        for (int of = 16; of > 0; of >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, of);
        __nv_bfloat16* gb = dout_bf16 + row * D + lane * PER;
        if constexpr (PER == 4) {
            __nv_bfloat162 p0 = __floats2bfloat162_rn(gv[0], gv[1]);
            __nv_bfloat162 p1 = __floats2bfloat162_rn(gv[2], gv[3]);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t*>(&p0);
            u.y = *reinterpret_cast<uint32_t*>(&p1);
            *reinterpret_cast<uint2*>(gb) = u;
        } else {
            __nv_bfloat162 p0 = __floats2bfloat162_rn(gv[0], gv[1]);
            *reinterpret_cast<__nv_bfloat162*>(gb) = p0;
        }
        if (lane == 0) {
            const float dv = acc - (dlse ? dlse[row] : 0.f);
            const float l = lse[row], s = sink[row];
            float ps = 0.f;
            if (isfinite(l)) ps = expf(s - l);
            else if (l == INFINITY && s == INFINITY) ps = 1.f;
            dsink[row] = -ps * dv;
            const int h = int(row % Hq);
            const int64_t bi = row / Hq;
            const int i = int(bi % S), b = int(bi / S);
            const size_t t = (size_t(b) * Hq + h) * S + i;
            lse2t[t] = l * kLog2e;
            dvt[t] = dv;
        }
    }
}

// ---------------------------------------------------------------------------
// generic FlexAttention variant ([B, H, S, D] tensors, BF16 out / dout,
// per-head sink weights, EOS-delimited documents and fixed blocks)
// ---------------------------------------------------------------------------

// positions[b, i] = i - (start of the block holding token i), where a block starts at
// token 0, after every EOS token (block_causal: the EOS closes its document) and, when
// fixed_block_size F > 0, at every multiple of F. The attention kernels then see one
// document per block. grid (B), block 1024: each thread takes a contiguous chunk of
// the row, the block combines the chunks' latest starts with a max-scan.
__global__ void flex_positions_kernel(const int64_t* __restrict__ tokens, int64_t eos_id, int S, int fbs,
                                      int32_t* __restrict__ positions) {
    const int b = blockIdx.x;
    const int nt = blockDim.x, t = threadIdx.x;
    const int chunk = (S + nt - 1) / nt;
    const int c0 = min(S, t * chunk), c1 = min(S, c0 + chunk);
    const int64_t* row = tokens ? tokens + size_t(b) * S : nullptr;
    auto starts_block = [&](int c) {
        return c == 0 || (row && row[c - 1] == eos_id) || (fbs > 0 && c % fbs == 0);
    };
    int last = -1;  // latest block start inside this thread's chunk
    for (int c = c0; c < c1; ++c)
        if (starts_block(c)) last = c;
    // inclusive max-scan over the threads (starts only grow with c)
    __shared__ int warp_last[32];
    const int lane = t & 31, w = t >> 5;
    int v = last;
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v = max(v, u);
    }
    if (lane == 31) warp_last[w] = v;
    __syncthreads();
    if (w == 0) {
        int x = lane < (nt >> 5) ? warp_last[lane] : -1;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x = max(x, u);
        }
        warp_last[lane] = x;
    }
    __syncthreads();
    // latest start before this thread's chunk: the scan up to the previous thread
    int prev = __shfl_up_sync(0xffffffffu, v, 1);
    if (lane == 0) prev = -1;
    if (w > 0) prev = max(prev, warp_last[w - 1]);
    int start = prev;
    for (int c = c0; c < c1; ++c) {
        if (starts_block(c)) start = c;
        positions[size_t(b) * S + c] = c - start;
    }
}

// Backward preprocessing of the generic variant: one warp per (b, h, i) row, rows in
// [B, H, S] order (consecutive rows are consecutive in memory). Reads the BF16 output
// and output gradient rows, writes Dv = sum_d dO.O, the per-row sink gradient
// -exp(sigma - lse) Dv and the transposed lse * log2(e) / Dv of the attention kernels.
template <int D>
__global__ void flex_bwd_prep_kernel(const uint16_t* __restrict__ out, const uint16_t* __restrict__ dout,
                                     const float* __restrict__ lse, const float* __restrict__ sink, int64_t sink_sb,
                                     int64_t sink_ss, int64_t sink_sh, int B, int S, int Hq,
                                     float* __restrict__ dsink_rows, float* __restrict__ lse2t,
                                     float* __restrict__ dvt) {
    constexpr int PER = D / 32;  // BF16 values per lane: 4 (8 bytes) or 2 (4 bytes)
    const int64_t nrows = int64_t(B) * Hq * S;
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t row = blockIdx.x * int64_t(blockDim.x >> 5) + (threadIdx.x >> 5); row < nrows; row += warps) {
        const uint16_t* o = out + row * D + lane * PER;
        const uint16_t* g = dout + row * D + lane * PER;
        float acc = 0.f;
        if constexpr (PER == 4) {
            const uint2 a = *reinterpret_cast<const uint2*>(o);
            const uint2 c = *reinterpret_cast<const uint2*>(g);
            acc = __uint_as_float(a.x << 16) * __uint_as_float(c.x << 16) +
                  __uint_as_float(a.x & 0xFFFF0000u) * __uint_as_float(c.x & 0xFFFF0000u) +
                  __uint_as_float(a.y << 16) * __uint_as_float(c.y << 16) +
                  __uint_as_float(a.y & 0xFFFF0000u) * __uint_as_float(c.y & 0xFFFF0000u);
        } else {
            const uint32_t a = *reinterpret_cast<const uint32_t*>(o);
            const uint32_t c = *reinterpret_cast<const uint32_t*>(g);
            acc = __uint_as_float(a << 16) * __uint_as_float(c << 16) +
                  __uint_as_float(a & 0xFFFF0000u) * __uint_as_float(c & 0xFFFF0000u);
        }
        for (int of = 16; of > 0; of >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, of);
        if (lane == 0) {
            const int i = int(row % S);
            const int64_t bh = row / S;
            const int h = int(bh % Hq), b = int(bh / Hq);
            const float l = lse[row];
            const float sg = sink ? sink[b * sink_sb + i * sink_ss + h * sink_sh] : -INFINITY;  // no sink: -inf
            float ps = 0.f;
            if (isfinite(l)) ps = expf(sg - l);
            dsink_rows[row] = -ps * acc;
            lse2t[row] = l * kLog2e;
            dvt[row] = acc;
        }
    }
}

// dsink_weights[h] = sum over (b, i) of the per-row sink gradients, in a fixed order
// (no atomics: the result does not depend on scheduling). grid (Hq), block 1024; each
// thread keeps four partial sums so that four loads are in flight.
__global__ void flex_dsink_reduce_kernel(const float* __restrict__ dsink_rows, int B, int S, int Hq,
                                         float* __restrict__ dsink_weights) {
    const int h = blockIdx.x;
    const int nt = blockDim.x;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int b = 0; b < B; ++b) {
        const float* r = dsink_rows + (size_t(b) * Hq + h) * S;
        int i = threadIdx.x;
        for (; i + 3 * nt < S; i += 4 * nt) {
            a0 += r[i];
            a1 += r[i + nt];
            a2 += r[i + 2 * nt];
            a3 += r[i + 3 * nt];
        }
        for (; i < S; i += nt) a0 += r[i];
    }
    float acc = (a0 + a1) + (a2 + a3);
    __shared__ float part[32];
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        float x = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.f;
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (threadIdx.x == 0) dsink_weights[h] = x;
    }
}

// Zero the dprofiles entries of each (b, h, i) row that no allowed key
// reaches: everything outside the visited distances [i_g - hi, i_g - lo].
// One warp per 32 consecutive rows of one (b, h): lane l reads the bounds of row
// i0 + l, then the warp zeroes row by row (bounds broadcast by shuffles, 16-byte
// stores, rows the attention kernels cover entirely skipped).
__global__ void dprof_zero_kernel(const int2* __restrict__ row_bounds, int B, int S, int Hq, int R, int q_off,
                                  float* __restrict__ dprof) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int segs = (S + 31) >> 5;  // 32-row segments per (b, h)
    const int64_t nseg = int64_t(B) * Hq * segs;
    for (int64_t sg = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; sg < nseg; sg += nwarps) {
        const int64_t bh = sg / segs;
        const int i0 = int(sg - bh * segs) * 32;
        const int b = int(bh / Hq);
        int dlo_l = R, dhi_l = -1;  // visited distances of row i0 + lane (inclusive); none by default
        const int il = i0 + lane;
        if (il < S) {
            const int2 bnd = row_bounds[size_t(b) * S + il];
            if (bnd.x <= bnd.y) {
                dlo_l = max(0, q_off + il - bnd.y);
                dhi_l = min(R - 1, q_off + il - bnd.x);
            }
        }
        const int nrows = min(32, S - i0);
        for (int r = 0; r < nrows; ++r) {
            const int dlo = __shfl_sync(0xffffffffu, dlo_l, r);
            const int dhi = __shfl_sync(0xffffffffu, dhi_l, r);
            if (dlo == 0 && dhi == R - 1) continue;
            float* base = dprof + (bh * S + i0 + r) * int64_t(R);
            for (int e0 = lane * 4; e0 < R; e0 += 128) {
                if (e0 + 3 < dlo || e0 > dhi) {
                    *reinterpret_cast<float4*>(base + e0) = make_float4(0.f, 0.f, 0.f, 0.f);
                } else if (e0 < dlo || e0 + 3 > dhi) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (e0 + u < dlo || e0 + u > dhi) base[e0 + u] = 0.f;
                }
            }
        }
    }
}

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// arrives on; the guard must give up after timeout_ns and record the site.
__global__ void selftest_wait_kernel(uint64_t timeout_ns, int* err) {
    __shared__ uint64_t bar;
    __shared__ CtaControl ctl;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        ctl.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &ctl, err, kErrSelftest, timeout_ns);
    __syncthreads();
}

// Device evaluation of exp2_fma2 (the forward's FMA-pipe power of two), for its accuracy test.
__global__ void selftest_exp2_kernel(const float* __restrict__ t, float* __restrict__ out, int64_t n) {
    const int64_t k = 2 * (int64_t(blockIdx.x) * blockDim.x + threadIdx.x);
    if (k >= n) return;
    const float2 v = exp2_fma2(make_float2(t[k], k + 1 < n ? t[k + 1] : 0.f));
    out[k] = v.x;
    if (k + 1 < n) out[k + 1] = v.y;
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_merge(float* out, float* lse, const float* out_part, const float* lse_part, int64_t rows, int D,
                         cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((rows + 7) / 8, 148 * 16);
    merge_kernel<<<unsigned(blocks), 256, 0, st>>>(out, lse, out_part, lse_part, rows, D);
    return cudaGetLastError();
}

cudaError_t launch_kspan(const uint8_t* key_valid, int B, int Skv, int2* kspan, cudaStream_t st) {
    if (B == 0) return cudaSuccess;
    kspan_kernel<<<B, 512, 0, st>>>(key_valid, Skv, kspan);
    return cudaGetLastError();
}

cudaError_t launch_bounds(const uint8_t* valid, const int32_t* positions, const int2* kspan, int B, int S,
                          int q_off, int W, int2* row_bounds, TileBounds* tiles, cudaStream_t st) {
    if (B == 0 || S == 0) return cudaSuccess;
    dim3 grid((S + 63) / 64, B);
    bounds_kernel<<<grid, 64, 0, st>>>(valid, positions, kspan, S, q_off, W, row_bounds, tiles);
    return cudaGetLastError();
}

cudaError_t launch_validate(const uint8_t* valid, const uint8_t* key_valid, const int32_t* positions,
                            const int32_t* key_positions, int B, int S, int Skv, int q_off,
                            int key_pos_from_query, int* ctl, int* edges, cudaStream_t st) {
    const long long n = (long long)B * (S > Skv ? S : Skv);
    if (n == 0) return cudaSuccess;
    const int blocks = int(n / 256 + 1 < 4096 ? n / 256 + 1 : 4096);
    validate_kernel<<<blocks, 256, 0, st>>>(valid, key_valid, positions, key_positions, B, S, Skv, q_off,
                                            key_pos_from_query, ctl, edges);
    return cudaGetLastError();
}

cudaError_t launch_bwd_prep(int D, const float* out, const float* lse, const float* sink, const float* dout,
                            const float* dlse, int B, int S, int Hq, float* dsink, __nv_bfloat16* dout_bf16,
                            float* lse2t, float* dvt, cudaStream_t st) {
    const long long rows = (long long)B * S * Hq;
    if (rows == 0) return cudaSuccess;
    const int blocks = int(rows / 8 + 1 < 148 * 32 ? rows / 8 + 1 : 148 * 32);
    if (D == 128)
        bwd_prep_kernel<128><<<blocks, 256, 0, st>>>(out, lse, sink, dout, dlse, B, S, Hq, dsink, dout_bf16, lse2t, dvt);
    else
        bwd_prep_kernel<64><<<blocks, 256, 0, st>>>(out, lse, sink, dout, dlse, B, S, Hq, dsink, dout_bf16, lse2t, dvt);
    return cudaGetLastError();
}

cudaError_t launch_dprof_zero(const int2* row_bounds, int B, int S, int Hq, int R, int q_off, float* dprof,
                              cudaStream_t st) {
    const long long segs = (long long)B * Hq * ((S + 31) / 32);
    if (segs == 0 || R == 0) return cudaSuccess;
    const long long want = (segs + 7) / 8;  // 8 warps per block
    const int blocks = int(want < 148 * 16 ? want : 148 * 16);
    dprof_zero_kernel<<<blocks, 256, 0, st>>>(row_bounds, B, S, Hq, R, q_off, dprof);
    return cudaGetLastError();
}

cudaError_t launch_flex_positions(const int64_t* tokens, int64_t eos_id, int B, int S, int fbs, int32_t* positions,
                                  cudaStream_t st) {
    if (B == 0 || S == 0) return cudaSuccess;
    flex_positions_kernel<<<B, 1024, 0, st>>>(tokens, eos_id, S, fbs, positions);
    return cudaGetLastError();
}

cudaError_t launch_flex_bwd_prep(int D, const uint16_t* out, const uint16_t* dout, const float* lse, const float* sink,
                                 int64_t sink_sb, int64_t sink_ss, int64_t sink_sh, int B, int S, int Hq,
                                 float* dsink_rows, float* lse2t, float* dvt, cudaStream_t st) {
    const long long rows = (long long)B * S * Hq;
    if (rows == 0) return cudaSuccess;
    const int blocks = int(rows / 8 + 1 < 148 * 32 ? rows / 8 + 1 : 148 * 32);
    if (D == 128)
        flex_bwd_prep_kernel<128><<<blocks, 256, 0, st>>>(out, dout, lse, sink, sink_sb, sink_ss, sink_sh, B, S, Hq,
                                                          dsink_rows, lse2t, dvt);
    else
        flex_bwd_prep_kernel<64><<<blocks, 256, 0, st>>>(out, dout, lse, sink, sink_sb, sink_ss, sink_sh, B, S, Hq,
                                                         dsink_rows, lse2t, dvt);
    return cudaGetLastError();
}

cudaError_t launch_flex_dsink_reduce(const float* dsink_rows, int B, int S, int Hq, float* dsink_weights,
                                     cudaStream_t st) {
    if (Hq == 0) return cudaSuccess;
    flex_dsink_reduce_kernel<<<Hq, 1024, 0, st>>>(dsink_rows, B, S, Hq, dsink_weights);
    return cudaGetLastError();
}

cudaError_t launch_selftest_exp2(const float* t, float* out, int64_t n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = ((n + 1) / 2 + 255) / 256;
    selftest_exp2_kernel<<<unsigned(blocks), 256, 0, st>>>(t, out, n);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(uint64_t timeout_ns, int* err, cudaStream_t st) {
    selftest_wait_kernel<<<1, 32, 0, st>>>(timeout_ns, err);
    return cudaGetLastError();
}

}  // namespace ira
