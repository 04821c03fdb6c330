// common.cuh -- shared definitions of the CUDA path: kernel parameter blocks,
// workspace layout and constants.
#pragma once

#include <cstddef>
#include <cstdint>

namespace ira {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Lazy-rescale threshold of the online softmax, in log2 units: the running
// maximum is only moved (and O rescaled) when a new row maximum exceeds it by
// more than this, so unnormalised probabilities stay below 2^8.
constexpr float kRescaleThreshold = 8.0f;

// Which column pairs of a softmax thread's step take their exponentials on the FMA
// pipe (bit u set: pair u of a 16-pair group, exp2_fma2) rather than the MUFU: the
// forward, the dK/dV and the dQ kernels. Measured on B200: the forward is fastest
// with a quarter of its pairs on the FMA pipe (the long forward 3 % faster than with
// half, the training-shape forward unchanged; none or three quarters are slower), the
// backward kernels with none.
#ifndef IRA_FWD_FMA_PAIRS
#define IRA_FWD_FMA_PAIRS 0x8888u
#endif
#ifndef IRA_DKDV_FMA_PAIRS
#define IRA_DKDV_FMA_PAIRS 0x0000u
#endif
#ifndef IRA_DQ_FMA_PAIRS
#define IRA_DQ_FMA_PAIRS 0x0000u
#endif

// Default limit of every device-side wait (nanoseconds).
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

// Empty key range marker for a row with no allowed key.
constexpr int kEmptyLo = 0x3FFFFFFF;
constexpr int kEmptyHi = -0x3FFFFFFF;

// Codes recorded in the device error word (first failing wait wins).
enum ErrSite : int {
    kErrNone = 0,
    kErrFwdQ = 101, kErrFwdK, kErrFwdV, kErrFwdS, kErrFwdP, kErrFwdO, kErrFwdKFree, kErrFwdVFree,
    kErrDkdvKV = 201, kErrDkdvQ, kErrDkdvS, kErrDkdvP, kErrDkdvAcc, kErrDkdvQFree,
    kErrDqQ = 301, kErrDqKV, kErrDqS, kErrDqP, kErrDqAcc, kErrDqKVFree,
    kErrSelftest = 901,
    // bounds-checking builds only: an index outside its buffer (the access is skipped)
    kErrBoundsFwdSmem = 951, kErrBoundsFwdGlobal, kErrBoundsDkdvSmem, kErrBoundsDkdvGlobal, kErrBoundsDqSmem,
    kErrBoundsDqGlobal,
};

// Index checks of the bounds-checking build (-DINKLING_BOUNDS_CHECK): IRA_IN_BOUNDS(err,
// code, off, bytes, size) is true when the access [off, off + bytes) lies inside a buffer
// of `size` bytes (or elements, as long as all three agree); otherwise it records `code`
// in the device error word (first one wins) and is false, and the caller skips the
// access. Nothing traps. In ordinary builds it is the constant true.
#ifdef INKLING_BOUNDS_CHECK
__device__ __forceinline__ bool ira_in_bounds(int* err, int code, long long off, long long bytes, long long size) {
    if (off >= 0 && bytes >= 0 && off + bytes <= size) return true;
    if (err) atomicCAS(err, 0, code);
    return false;
}
#define IRA_IN_BOUNDS(err, code, off, bytes, size) \
    ::ira::ira_in_bounds((err), (code), (long long)(off), (long long)(bytes), (long long)(size))
#else
#define IRA_IN_BOUNDS(err, code, off, bytes, size) true
#endif

// Per-64-row query tile summary written by the bounds kernel.
struct TileBounds {
    int min_lo;   // smallest first allowed key over non-empty rows
    int max_hi;   // largest last allowed key over non-empty rows
    int max_lo;   // largest first allowed key over non-empty rows
    int min_hi;   // smallest last allowed key over non-empty rows
    int n_nonempty;
    int n_rows;   // rows of the tile inside [0, S)
    int pad0, pad1;
};

// Byte layout of the caller-provided workspace.
struct WorkspaceLayout {
    size_t ctl;          // int[4]: [0] device error word, [1] validate error count
    size_t kspan;        // int2 [B]: first / last valid key column
    size_t edges;        // int [B][2]: rising edges of valid / key_valid (validate)
    size_t row_bounds;   // int2 [B*S]: (lo, hi) allowed key columns per query row
    size_t tile_bounds;  // TileBounds [B * ceil(S/64)]
    size_t dout_bf16;    // bf16 [B,S,Hq,D] (backward)
    size_t lse2t;        // fp32 [B,Hq,S]: lse * log2(e) (backward)
    size_t dvt;          // fp32 [B,Hq,S]: <dout,out> - dlse (backward)
    size_t total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WorkspaceLayout workspace_layout(int64_t B, int64_t S, int64_t Hq, int64_t D, bool backward) {
    WorkspaceLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = align_up(off + bytes, 256);
        return at;
    };
    const int64_t t64 = (S + 63) / 64;
    L.ctl = take(16);
    L.kspan = take(size_t(B) * 8);
    L.edges = take(size_t(B) * 8);
    L.row_bounds = take(size_t(B) * S * 8);
    L.tile_bounds = take(size_t(B) * t64 * sizeof(TileBounds));
    if (backward) {
        L.dout_bf16 = take(size_t(B) * S * Hq * D * 2);
        L.lse2t = take(size_t(B) * Hq * S * 4);
        L.dvt = take(size_t(B) * Hq * S * 4);
    }
    L.total = off;
    return L;
}

// Sizes and pointers shared by the attention kernels.
struct AttnParams {
    int B, S, Skv, Hq, Hkv, D, R, W, q_off;
    float scale;          // multiplies q.k (head_dim^-0.5 unless the caller gives another)
    float scale_log2;     // scale * log2(e)
    uint64_t timeout_ns;
    const uint16_t* profiles;
    const void* safe_src;  // any valid 16-B aligned global address (source of zero-fill copies)
    const float* sink;    // sink of row (b, i, h): sink[b * sink_sb + i * sink_ss + h * sink_sh]
    int64_t sink_sb, sink_ss, sink_sh;
    // element strides of the (b, i, h) rows of out and dq, of the (b, i, h) entries of
    // lse, and of the (b, j, g) rows of dk / dv (the D values of a row are contiguous)
    int64_t row_sb, row_ss, row_sh;
    int64_t lse_sb, lse_ss, lse_sh;
    int64_t kv_sb, kv_ss, kv_sh;
    const int2* row_bounds;
    const TileBounds* tile_bounds;
    int* err;
    // forward (out_bf16 set: the output is stored as BF16 there, out unused)
    float* out;
    uint16_t* out_bf16;
    float* lse;
    // backward
    const float* lse2t;
    const float* dvt;
    float* dq;
    float* dk;
    float* dv;
    float* dprofiles;
    // L2Clip of q fused into the attention (q_clipped set: the forward clips each Q tile
    // and stores it; q_raw set: the dQ kernel turns dq into the gradient of the unclipped
    // q): z = q_raw * clip_scale[h, :], q = z * min(1, clip_thr / |z|) * clip_tau[b, i]
    float clip_thr;
    const float* clip_scale;   // [Hq, D] or null
    const float* clip_tau;     // [B, S] or null
    uint16_t* q_clipped;       // forward: clipped q [B, S, Hq, D] BF16 (written)
    const uint16_t* q_raw;     // dQ: unclipped q [B, S, Hq, D] BF16
    float* dscale_part;        // dQ: parts of dscale, [B * ceil(S / 128)][Hq][D]
    float* dtau_part;          // dQ: parts of dtau, [B, S, Hq]
    // pipeline timeline of one CTA (only in builds with INKLING_TRACE; null otherwise)
    unsigned long long* trace;
    int trace_cta;
};

}  // namespace ira
