// host.cu -- the C ABI of libinkling_rel_attn.so (declared in
// include/inkling_rel_attn.h): argument checks, workspace carving, TMA
// descriptor encoding and the launch sequence of each entry point.
#include <cstdint>
#include <cmath>
#include <cstring>
#include <functional>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "inkling_flex_attn.h"
#include "inkling_l2clip.h"
#include "inkling_rel_attn.h"
#include "launch.h"

// Scratch of inkling_rel_attn_fwd_noalloc: a fixed-size array in device
// memory that exists on every GPU that loads this library, for as long as the
// process lives. Host code must not take its address directly (the name is a
// host-side stand-in); it asks the runtime for the device address instead.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

using namespace ira;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// BF16 tensor [B, T, H, D] (or, with bhsd, [B, H, T, D]) as a 4-D map {D, H, T, B};
// box {64, 1, rows, 1}; 128-byte swizzle; out-of-range rows read as zero. The kernels
// address (d, head, row, batch) either way: only the strides differ.
bool encode_bhtd(CUtensorMap* m, const void* base, int64_t B, int64_t T, int64_t H, int64_t D, int rows,
                 bool bhsd = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(T), cuuint64_t(B)};
    cuuint64_t strides[3] = {cuuint64_t((bhsd ? T : 1) * D * 2), cuuint64_t((bhsd ? 1 : H) * D * 2),
                             cuuint64_t(T * H * D * 2)};
    cuuint32_t box[4] = {64u, 1u, cuuint32_t(rows), 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Profiles [B, Hq, S, R] as R-long rows, in boxes of 8 rows x 136 entries (the band
// rows of 8 consecutive query columns: 128 distances plus up to 7 of misalignment);
// entries outside [0, R) and rows outside the tensor read 0.
bool encode_band(CUtensorMap* m, const void* base, int64_t rows, int64_t R) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cuuint64_t(R), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(R * 2)};
    cuuint32_t box[2] = {136u, 8u};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Last CUDA error seen by an entry point of this thread (inkling_rel_attn_last_cuda_error).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

cudaError_t note(cudaError_t e) {
    if (e != cudaSuccess) t_last_cuda_error = e;
    return e;
}

#ifdef INKLING_TRACE
// Pipeline timeline of one CTA (diagnostic builds only).
unsigned long long* g_trace_buf = nullptr;
int g_trace_cta = 0;
#endif

// A named NVTX range over an entry point's host work and launches, so that a
// profiler's timeline groups each call's kernels; a no-op when no tool is attached.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// Limit of the attention kernels' pipeline waits for later calls
// (inkling_rel_attn_set_wait_timeout_ns); 0 = the default.
uint64_t g_wait_timeout_ns = 0;

// Optional per-launch timing events (inkling_rel_attn_set_timing_events).
cudaEvent_t const* g_events = nullptr;
int g_event_pairs = 0;

struct LaunchTimer {
    cudaStream_t st;
    int k = 0;
    explicit LaunchTimer(cudaStream_t s) : st(s) {}
    cudaError_t record(int idx) {
        return (g_events && k < g_event_pairs) ? note(cudaEventRecord(g_events[idx], st)) : cudaSuccess;
    }
    template <class F>
    cudaError_t run(F&& f) {
        cudaError_t e = record(2 * k);
        if (e == cudaSuccess) e = note(f());
        if (e == cudaSuccess) e = record(2 * k + 1);
        ++k;
        return e;
    }
    bool active() const { return g_events != nullptr; }
};

// Per host thread and device: a second stream and its events, so that the dK/dV and
// dQ kernels of one backward call can run side by side (each fills the other's last,
// partial wave of CTAs). Fork: the side stream waits for the caller's stream; join:
// the caller's stream waits for the side stream; both are events, so a stream capture
// of the caller's stream takes the side stream's work into the graph. The stream is
// created on the first use outside a capture; a first use inside one gets *out = nullptr
// (the call then runs on the caller's stream alone).
struct SideStream {
    int device = -1;
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, bounds = nullptr, ready = nullptr, join = nullptr;
};
cudaError_t side_stream(SideStream** out, cudaStream_t caller) {
    thread_local SideStream per_dev[16];
    *out = nullptr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 16) return cudaErrorInvalidDevice;
    SideStream& r = per_dev[dev];
    if (r.s == nullptr) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(caller, &cs) != cudaSuccess) {
            (void)cudaGetLastError();  // not sticky; leave no error behind for the launches
            cs = cudaStreamCaptureStatusActive;
        }
        if (cs != cudaStreamCaptureStatusNone) return cudaSuccess;
        e = cudaStreamCreateWithFlags(&r.s, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.bounds, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.ready, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.join, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        r.device = dev;
    }
    *out = &r;
    return cudaSuccess;
}

inkling_status check_dims(const inkling_rel_attn_dims* d) {
    if (!d) return INKLING_ERR_INVALID_ARG;
    if (d->batch < 0 || d->seq_q < 0 || d->seq_k < 0 || d->heads_q <= 0 || d->heads_kv <= 0 ||
        d->rel_extent < 0 || d->window < 0 || d->query_offset < 0)
        return INKLING_ERR_INVALID_ARG;
    if (d->heads_q % d->heads_kv != 0) return INKLING_ERR_INVALID_ARG;
    if (d->head_dim != 64 && d->head_dim != 128) return INKLING_ERR_UNSUPPORTED;
    if (d->rel_extent % 8 != 0) return INKLING_ERR_UNSUPPORTED;
    const int64_t lim = int64_t(1) << 30;
    if (d->seq_q >= lim || d->seq_k >= lim || d->query_offset >= lim || d->batch >= lim || d->heads_q >= 65536 ||
        d->rel_extent >= lim || d->window >= lim)
        return INKLING_ERR_UNSUPPORTED;
    // grid sizes
    const int64_t nqt = (d->seq_q + 127) / 128, nkt = (d->seq_k + 127) / 128;
    if (nqt * d->batch * d->heads_q >= (int64_t(1) << 31) || nkt * d->batch * d->heads_kv >= (int64_t(1) << 31))
        return INKLING_ERR_UNSUPPORTED;
    // the backward's profile-band tensor copies address profile rows b * Hq * S + h * S + i as one int32
    if (d->rel_extent > 0 && d->batch * d->heads_q * d->seq_q >= (int64_t(1) << 31) - 256)
        return INKLING_ERR_UNSUPPORTED;
    return INKLING_OK;
}

struct Ws {
    WorkspaceLayout L;
    uint8_t* base;
    int* ctl() const { return reinterpret_cast<int*>(base + L.ctl); }
    int2* kspan() const { return reinterpret_cast<int2*>(base + L.kspan); }
    int* edges() const { return reinterpret_cast<int*>(base + L.edges); }
    int2* row_bounds() const { return reinterpret_cast<int2*>(base + L.row_bounds); }
    TileBounds* tiles() const { return reinterpret_cast<TileBounds*>(base + L.tile_bounds); }
};

inkling_status get_ws(const inkling_rel_attn_dims* d, bool backward, void* ws, size_t bytes, Ws* out) {
    out->L = workspace_layout(d->batch, d->seq_q, d->heads_q, d->head_dim, backward);
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || bytes < out->L.total) return INKLING_ERR_INVALID_ARG;
    out->base = static_cast<uint8_t*>(ws);
    return INKLING_OK;
}

// key_valid / key_positions defaults (Inkling2FlexAttention.forward: key_valid
// defaults to valid, key positions to the query positions in the single-shard case).
inkling_status resolve_key_side(const inkling_rel_attn_dims* d, const uint8_t* valid, const uint8_t*& key_valid,
                                const int32_t* positions, const int32_t* key_positions, int* key_pos_from_query) {
    const bool single = d->seq_k == d->seq_q && d->query_offset == 0;
    if (!key_valid) {
        if (!single) return INKLING_ERR_INVALID_ARG;
        key_valid = valid;
    }
    *key_pos_from_query = 0;
    if (!key_positions && positions) {
        if (!single) return INKLING_ERR_INVALID_ARG;
        *key_pos_from_query = 1;
    }
    return INKLING_OK;
}

inkling_status cuda_status(cudaError_t e) { return note(e) == cudaSuccess ? INKLING_OK : INKLING_ERR_CUDA; }

AttnParams base_params(const inkling_rel_attn_dims* d, const Ws& w, const uint16_t* profiles, const float* sink) {
    AttnParams p{};
    p.B = int(d->batch);
    p.S = int(d->seq_q);
    p.Skv = int(d->seq_k);
    p.Hq = int(d->heads_q);
    p.Hkv = int(d->heads_kv);
    p.D = int(d->head_dim);
    p.R = int(d->rel_extent);
    p.W = int(d->window);
    p.q_off = int(d->query_offset);
    p.scale = 1.0f / sqrtf(float(d->head_dim));
    p.scale_log2 = p.scale * kLog2e;
    p.timeout_ns = g_wait_timeout_ns ? g_wait_timeout_ns : kDefaultTimeoutNs;
    p.profiles = profiles;
    p.safe_src = w.row_bounds();
    p.sink = sink;
    // [B, S, H, D] tensors, [B, S, H] sink / lse
    const int64_t S = d->seq_q, Hq = d->heads_q, D = d->head_dim;
    p.sink_sb = S * Hq;
    p.sink_ss = Hq;
    p.sink_sh = 1;
    p.row_sb = S * Hq * D;
    p.row_ss = Hq * D;
    p.row_sh = D;
    p.lse_sb = S * Hq;
    p.lse_ss = Hq;
    p.lse_sh = 1;
    p.kv_sb = d->seq_k * d->heads_kv * D;
    p.kv_ss = d->heads_kv * D;
    p.kv_sh = D;
    p.row_bounds = w.row_bounds();
    p.tile_bounds = w.tiles();
    p.err = w.ctl();
#ifdef INKLING_TRACE
    p.trace = g_trace_buf;
    p.trace_cta = g_trace_cta;
#endif
    return p;
}

// Prologue shared by fwd and bwd: clear the error word, key span, row ranges.
inkling_status run_bounds(const inkling_rel_attn_dims* d, const Ws& w, const uint8_t* valid,
                          const uint8_t* key_valid, const int32_t* positions, cudaStream_t st, LaunchTimer& tm) {
    cudaError_t e = cudaMemsetAsync(w.ctl(), 0, 16, st);
    if (e == cudaSuccess)
        e = tm.run([&] { return launch_kspan(key_valid, int(d->batch), int(d->seq_k), w.kspan(), st); });
    if (e == cudaSuccess)
        e = tm.run([&] {
            return launch_bounds(valid, positions, w.kspan(), int(d->batch), int(d->seq_q), int(d->query_offset),
                                 int(d->window), w.row_bounds(), w.tiles(), st);
        });
    return cuda_status(e);
}

// Device address of g_noalloc_scratch in the calling thread's current CUDA
// context, looked up once per context (with that context current) and cached.
// The cache is keyed by the context's process-unique id (cuCtxGetId), so a
// context created after cudaDeviceReset, or a non-primary context made current
// by the caller, gets its own lookup instead of a stale address.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
struct NoAllocSlot {
    unsigned long long ctx_id;
    void* ptr;
};
constexpr int kNoAllocSlots = 64;
std::mutex g_noalloc_mutex;
NoAllocSlot g_noalloc_slots[kNoAllocSlots] = {};
int g_noalloc_used = 0;

inkling_status current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    if (!get_current || !get_id) return INKLING_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return INKLING_ERR_CUDA;
    if (!ctx) {
        // no context on this thread yet: a runtime call that needs one makes the
        // current device's primary context current (and allocates nothing)
        void* p = nullptr;
        if (note(cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess) return INKLING_ERR_CUDA;
        if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return INKLING_ERR_CUDA;
    }
    return get_id(ctx, id) == CUDA_SUCCESS ? INKLING_OK : INKLING_ERR_CUDA;
}

inkling_status noalloc_scratch(void** out) {
    unsigned long long id = 0;
    inkling_status s = current_context_id(&id);
    if (s != INKLING_OK) return s;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    for (int k = 0; k < g_noalloc_used; ++k)
        if (g_noalloc_slots[k].ctx_id == id) {
            *out = g_noalloc_slots[k].ptr;
            return INKLING_OK;
        }
    void* p = nullptr;
    cudaError_t e = note(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    if (e != cudaSuccess || !p) return INKLING_ERR_CUDA;
    // a full table is refilled from the start (its entries only save lookups)
    if (g_noalloc_used == kNoAllocSlots) g_noalloc_used = 0;
    g_noalloc_slots[g_noalloc_used++] = NoAllocSlot{id, p};
    *out = p;
    return INKLING_OK;
}

// Tensor maps of one backward call.
struct BwdMaps {
    CUtensorMap tq64, tq128, tdo64, tdo128, tk128, tv128, tk64, tv64, tband;
};

// The launch sequence of one backward call, for either ABI. `pre_bounds` (optional)
// runs on the stream of the bounds kernels before them; `prep` launches the backward
// preprocessing on the stream it is given.
inkling_status bwd_launches(const inkling_rel_attn_dims* dims, const Ws& w, const AttnParams& p, const BwdMaps& m,
                            const uint8_t* valid, const uint8_t* key_valid, const int32_t* positions, bool has_keys,
                            cudaStream_t st, const std::function<cudaError_t(cudaStream_t)>& pre_bounds,
                            const std::function<cudaError_t(cudaStream_t)>& prep) {
    LaunchTimer tm(st);
    // Two streams, except while the timing hook is on (it wants one kernel at a time):
    //   caller's stream: prep -> (wait row bounds) -> dK/dV
    //   side stream:     key span, row bounds -> dprofiles zeroing -> (wait prep) -> dQ
    // dK/dV and dQ read the same inputs and write disjoint outputs; the zeroing writes the
    // dprofiles entries that dK/dV does not (distances outside a row's visited range).
    SideStream* side = nullptr;
    bool overlap = !tm.active();
    cudaError_t e = cudaSuccess;
    if (overlap) {
        e = side_stream(&side, st);
        if (e != cudaSuccess) return cuda_status(e);
        overlap = side != nullptr;
    }
    if (overlap) {
        e = cudaEventRecord(side->fork, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side->s, side->fork, 0);
        if (e != cudaSuccess) return cuda_status(e);
    }
    cudaStream_t st2 = overlap ? side->s : st;
    auto join = [&](inkling_status r) {  // on the error paths too: no work stays forked off
        if (overlap) {
            cudaError_t e2 = cudaEventRecord(side->join, side->s);
            if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, side->join, 0);
            if (r == INKLING_OK && e2 != cudaSuccess) r = cuda_status(e2);
        }
        return r;
    };
    if (pre_bounds) e = pre_bounds(st2);
    inkling_status s = e == cudaSuccess ? run_bounds(dims, w, valid, key_valid, positions, st2, tm)
                                        : cuda_status(e);
    if (s != INKLING_OK) return join(s);
    if (overlap) e = cudaEventRecord(side->bounds, st2);
    if (e == cudaSuccess)
        e = tm.run([&] { return prep(st); });
    if (e == cudaSuccess && overlap) e = cudaEventRecord(side->ready, st);
    if (e == cudaSuccess)
        e = tm.run([&] {
            return dims->rel_extent > 0 ? launch_dprof_zero(w.row_bounds(), p.B, p.S, p.Hq, p.R, p.q_off,
                                                            p.dprofiles, st2)
                                        : cudaSuccess;
        });
    if (e == cudaSuccess && overlap) e = cudaStreamWaitEvent(st, side->bounds, 0);
    if (e == cudaSuccess)
        e = tm.run([&] { return has_keys ? launch_bwd_dkdv(m.tq64, m.tk128, m.tv128, m.tdo64, m.tband, p, st) : cudaSuccess; });
    if (e == cudaSuccess && overlap) e = cudaStreamWaitEvent(st2, side->ready, 0);
    if (e == cudaSuccess) e = tm.run([&] { return launch_bwd_dq(m.tq128, m.tk64, m.tv64, m.tdo128, p, st2); });
    return join(cuda_status(e));
}

// ---------------------------------------------------------------------------
// generic FlexAttention variant
// ---------------------------------------------------------------------------
// The learned-relative problem it maps to: no profiles, S queries and S keys, the
// sliding window as the window, no query offset.
inkling_status flex_dims(const inkling_flex_attn_dims* f, inkling_rel_attn_dims* d) {
    if (!f) return INKLING_ERR_INVALID_ARG;
    if (f->mask_type != INKLING_FLEX_CAUSAL && f->mask_type != INKLING_FLEX_BLOCK_CAUSAL)
        return INKLING_ERR_INVALID_ARG;
    if (f->fixed_block_size < 0 || f->sliding_window < 0 || f->heads_q <= 0 || f->heads_kv <= 0)
        return INKLING_ERR_INVALID_ARG;
    if (f->heads_q != f->heads_kv && !f->enable_gqa) return INKLING_ERR_INVALID_ARG;
    if (f->fixed_block_size >= (int64_t(1) << 30)) return INKLING_ERR_UNSUPPORTED;
    d->batch = f->batch;
    d->seq_q = f->seq;
    d->seq_k = f->seq;
    d->heads_q = f->heads_q;
    d->heads_kv = f->heads_kv;
    d->head_dim = f->head_dim;
    d->rel_extent = 0;
    d->window = f->sliding_window;
    d->query_offset = 0;
    return check_dims(d);
}

// Workspace: the learned-relative layout, then block positions int32 [B, S], an
// all-ones validity mask u8 [B, S] and (backward) per-row sink gradients f32 [B, Hq, S].
struct FlexWs {
    Ws w;
    int32_t* positions = nullptr;
    uint8_t* valid = nullptr;
    float* dsink_rows = nullptr;
    size_t total = 0;
};
FlexWs flex_layout(const inkling_rel_attn_dims& d, bool backward, uint8_t* base) {
    FlexWs f;
    // the forward sections, then (backward) lse * log2(e) and Dv: the kernels read dO
    // straight from the caller's BF16 tensor, so there is no BF16 copy of it
    f.w.L = workspace_layout(d.batch, d.seq_q, d.heads_q, d.head_dim, false);
    f.w.base = base;
    size_t off = align_up(f.w.L.total, 256);
    if (backward) {
        const size_t rows = size_t(d.batch) * d.heads_q * d.seq_q;
        f.w.L.lse2t = off;
        off = align_up(off + rows * 4, 256);
        f.w.L.dvt = off;
        off = align_up(off + rows * 4, 256);
    }
    const size_t pos_off = off;
    off = align_up(off + size_t(d.batch) * d.seq_q * 4, 256);
    const size_t valid_off = off;
    off = align_up(off + size_t(d.batch) * d.seq_q, 256);
    const size_t dsr_off = off;
    if (backward) off = align_up(off + size_t(d.batch) * d.heads_q * d.seq_q * 4, 256);
    f.total = off;
    if (base) {
        f.positions = reinterpret_cast<int32_t*>(base + pos_off);
        f.valid = base + valid_off;
        f.dsink_rows = backward ? reinterpret_cast<float*>(base + dsr_off) : nullptr;
    }
    return f;
}

// Strides of the [B, H, S, D] tensors, [B, H, S] lse and [Hq] sink weights; the scale.
void flex_params(AttnParams& p, const inkling_flex_attn_dims* f, const float* sink_weights) {
    const int64_t S = f->seq, Hq = f->heads_q, Hkv = f->heads_kv, D = f->head_dim;
    p.scale = (!sink_weights && f->scale > 0) ? float(f->scale) : 1.0f / sqrtf(float(D));
    p.scale_log2 = p.scale * kLog2e;
    p.sink = sink_weights;
    p.sink_sb = 0;
    p.sink_ss = 0;
    p.sink_sh = 1;
    p.row_sb = Hq * S * D;
    p.row_ss = D;
    p.row_sh = S * D;
    p.lse_sb = Hq * S;
    p.lse_ss = 1;
    p.lse_sh = S;
    p.kv_sb = Hkv * S * D;
    p.kv_ss = D;
    p.kv_sh = S * D;
}

// All-ones validity and the block positions, on stream st.
cudaError_t flex_masks(const inkling_flex_attn_dims* f, const int64_t* tokens, const FlexWs& fw, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(fw.valid, 1, size_t(f->batch) * f->seq, st);
    if (e == cudaSuccess)
        e = launch_flex_positions(f->mask_type == INKLING_FLEX_BLOCK_CAUSAL ? tokens : nullptr, f->eos_id,
                                  int(f->batch), int(f->seq), int(f->fixed_block_size), fw.positions, st);
    return note(e);
}

// L2Clip of q fused into the attention (the *_qclip entry points).
struct QClipArgs {
    float thr;
    const float* scale;         // [Hq, D] or null
    const float* tau;           // [B, S] or null
    uint16_t* q_clipped;        // forward: the clipped q (written)
    const uint16_t* q_raw;      // backward: the unclipped q
    float* dscale;              // backward: gradient of scale (or null)
    float* dtau;                // backward: gradient of tau (or null)
};

// Backward workspace of the fused path: the ordinary one, then the dQ kernel's parts of
// dscale [B * ceil(S / 128)][Hq][D] and of dtau [B, S, Hq].
struct QClipLayout {
    size_t dscale_part, dtau_part, total;
    int64_t nchunks;
};
QClipLayout qclip_layout(const inkling_rel_attn_dims* d) {
    QClipLayout q{};
    const size_t base = workspace_layout(d->batch, d->seq_q, d->heads_q, d->head_dim, true).total;
    q.nchunks = d->batch * ((d->seq_q + 127) / 128);
    q.dscale_part = align_up(base, 256);
    q.dtau_part = align_up(q.dscale_part + size_t(q.nchunks) * d->heads_q * d->head_dim * 4, 256);
    q.total = align_up(q.dtau_part + size_t(d->batch) * d->seq_q * d->heads_q * 4, 256);
    return q;
}

// The forward of either ABI; `qc` (optional) fuses the L2Clip of q in: q is then the
// unclipped q, and the clipped q is stored to qc->q_clipped.
inkling_status fwd_impl(const inkling_rel_attn_dims* dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint16_t* profiles, const float* sink, const uint8_t* valid, const uint8_t* key_valid,
                        const int32_t* positions, const int32_t* key_positions, float* out, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream, const QClipArgs* qc) {
    inkling_status s = check_dims(dims);
    if (s != INKLING_OK) return s;
    const int64_t nq = dims->batch * dims->seq_q, nk = dims->batch * dims->seq_k;
    if (nq > 0 && (!q || !sink || !valid || !out || !lse)) return INKLING_ERR_INVALID_ARG;
    if (nq > 0 && dims->rel_extent > 0 && !profiles) return INKLING_ERR_INVALID_ARG;
    if (nk > 0 && (!k || !v)) return INKLING_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(profiles) || !aligned16(out))
        return INKLING_ERR_INVALID_ARG;
    int kpq = 0;
    s = resolve_key_side(dims, valid, key_valid, positions, key_positions, &kpq);
    if (s != INKLING_OK) return s;
    if (nk > 0 && !key_valid) return INKLING_ERR_INVALID_ARG;
    Ws w;
    s = get_ws(dims, false, workspace, workspace_bytes, &w);
    if (s != INKLING_OK) return s;
    if (nq == 0) return INKLING_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // K/V maps need at least one row; with no keys every row is empty and the
    // kernel never reads them, so point them at q.
    const bool no_keys = dims->seq_k == 0;
    CUtensorMap tq, tk, tv;
    if (!encode_bhtd(&tq, q, dims->batch, dims->seq_q, dims->heads_q, dims->head_dim, 128) ||
        !encode_bhtd(&tk, no_keys ? q : k, dims->batch, no_keys ? 1 : dims->seq_k,
                     no_keys ? dims->heads_q : dims->heads_kv, dims->head_dim, 64) ||
        !encode_bhtd(&tv, no_keys ? q : v, dims->batch, no_keys ? 1 : dims->seq_k,
                     no_keys ? dims->heads_q : dims->heads_kv, dims->head_dim, 64))
        return INKLING_ERR_CUDA;

    LaunchTimer tm(st);
    s = run_bounds(dims, w, valid, key_valid, positions, st, tm);
    if (s != INKLING_OK) return s;
    AttnParams p = base_params(dims, w, profiles, sink);
    p.out = out;
    p.lse = lse;
    if (!qc) return cuda_status(tm.run([&] { return launch_fwd(tq, tk, tv, p, st); }));
    p.clip_thr = qc->thr;
    p.clip_scale = qc->scale;
    p.clip_tau = qc->tau;
    p.q_clipped = qc->q_clipped;
    CUtensorMap tqc;
    if (!encode_bhtd(&tqc, qc->q_clipped, dims->batch, dims->seq_q, dims->heads_q, dims->head_dim, 128))
        return INKLING_ERR_CUDA;
    return cuda_status(tm.run([&] { return launch_fwd_qclip(tq, tk, tv, tqc, p, st); }));
}

// The backward of either ABI; `qc` (optional) fuses the L2Clip backward of q in: q is
// then the clipped q the forward stored, dq receives the gradient of the unclipped q
// (qc->q_raw), and qc->dscale / qc->dtau (when set) the clip's parameter gradients.
inkling_status bwd_impl(const inkling_rel_attn_dims* dims, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint16_t* profiles, const float* sink, const uint8_t* valid, const uint8_t* key_valid,
                        const int32_t* positions, const int32_t* key_positions, const float* out, const float* lse,
                        const float* dout, const float* dlse, float* dq, float* dk, float* dv, float* dprofiles,
                        float* dsink, void* workspace, size_t workspace_bytes, void* stream, const QClipArgs* qc) {
    inkling_status s = check_dims(dims);
    if (s != INKLING_OK) return s;
    const int64_t nq = dims->batch * dims->seq_q, nk = dims->batch * dims->seq_k;
    if (nq > 0 && (!q || !sink || !valid || !out || !lse || !dout || !dq || !dsink)) return INKLING_ERR_INVALID_ARG;
    if (nq > 0 && dims->rel_extent > 0 && (!profiles || !dprofiles)) return INKLING_ERR_INVALID_ARG;
    if (nk > 0 && (!k || !v || !dk || !dv)) return INKLING_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(profiles) || !aligned16(out) ||
        !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dprofiles))
        return INKLING_ERR_INVALID_ARG;
    int kpq = 0;
    s = resolve_key_side(dims, valid, key_valid, positions, key_positions, &kpq);
    if (s != INKLING_OK) return s;
    if (nk > 0 && !key_valid) return INKLING_ERR_INVALID_ARG;
    Ws w;
    s = get_ws(dims, true, workspace, workspace_bytes, &w);
    if (s != INKLING_OK) return s;
    const QClipLayout ql = qclip_layout(dims);
    if (qc && workspace_bytes < ql.total) return INKLING_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (nq == 0) {
        // no queries: every key gradient is zero, and so is the clip's scale gradient
        cudaError_t e = cudaSuccess;
        if (nk > 0) {
            const size_t bytes = size_t(nk) * dims->heads_kv * dims->head_dim * 4;
            e = cudaMemsetAsync(dk, 0, bytes, st);
            if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, bytes, st);
        }
        if (e == cudaSuccess && qc && qc->dscale)
            e = cudaMemsetAsync(qc->dscale, 0, size_t(dims->heads_q) * dims->head_dim * 4, st);
        return cuda_status(e);
    }
    const bool no_keys = dims->seq_k == 0;
    auto* dout_bf16 = reinterpret_cast<__nv_bfloat16*>(w.base + w.L.dout_bf16);
    auto* lse2t = reinterpret_cast<float*>(w.base + w.L.lse2t);
    auto* dvt = reinterpret_cast<float*>(w.base + w.L.dvt);
    CUtensorMap tq64, tq128, tdo64, tdo128, tk128, tv128, tk64, tv64;
    const int64_t B = dims->batch, S = dims->seq_q, Hq = dims->heads_q, D = dims->head_dim;
    const int64_t Skv_m = no_keys ? 1 : dims->seq_k, Hkv_m = no_keys ? Hq : dims->heads_kv;
    const void* kb = no_keys ? static_cast<const void*>(q) : k;
    const void* vb = no_keys ? static_cast<const void*>(q) : v;
    if (!encode_bhtd(&tq64, q, B, S, Hq, D, 64) || !encode_bhtd(&tq128, q, B, S, Hq, D, 128) ||
        !encode_bhtd(&tdo64, dout_bf16, B, S, Hq, D, 64) || !encode_bhtd(&tdo128, dout_bf16, B, S, Hq, D, 128) ||
        !encode_bhtd(&tk128, kb, B, Skv_m, Hkv_m, D, 128) || !encode_bhtd(&tv128, vb, B, Skv_m, Hkv_m, D, 128) ||
        !encode_bhtd(&tk64, kb, B, Skv_m, Hkv_m, D, 64) || !encode_bhtd(&tv64, vb, B, Skv_m, Hkv_m, D, 64))
        return INKLING_ERR_CUDA;
    CUtensorMap tband;
    std::memset(&tband, 0, sizeof(tband));
    if (dims->rel_extent > 0 && !encode_band(&tband, profiles, B * Hq * S, dims->rel_extent)) return INKLING_ERR_CUDA;

    AttnParams p = base_params(dims, w, profiles, sink);
    p.lse2t = lse2t;
    p.dvt = dvt;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dprofiles = dprofiles;
    float* dscale_part = nullptr;
    float* dtau_part = nullptr;
    if (qc) {
        dscale_part = reinterpret_cast<float*>(w.base + ql.dscale_part);
        dtau_part = reinterpret_cast<float*>(w.base + ql.dtau_part);
        p.clip_thr = qc->thr;
        p.clip_scale = qc->scale;
        p.clip_tau = qc->tau;
        p.q_raw = qc->q_raw;
        p.dscale_part = dscale_part;
        p.dtau_part = dtau_part;
    }
    BwdMaps mp{tq64, tq128, tdo64, tdo128, tk128, tv128, tk64, tv64, tband};
    s = bwd_launches(dims, w, p, mp, valid, key_valid, positions, nk > 0, st, nullptr,
                     [&](cudaStream_t s0) {
                         return launch_bwd_prep(int(D), out, lse, sink, dout, dlse, int(B), int(S), int(Hq),
                                                dsink, dout_bf16, lse2t, dvt, s0);
                     });
    if (s != INKLING_OK || !qc || (!qc->dscale && !qc->dtau)) return s;
    // the clip's parameter gradients: sums of the dQ kernel's parts, in a fixed order
    return cuda_status(launch_l2clip_reduce(dtau_part, B * S, int(Hq), qc->dtau, dscale_part, ql.nchunks, Hq * D,
                                            qc->dscale, st));
}

}  // namespace

namespace ira {
// Lets the other translation units' entry points record their CUDA errors for
// inkling_rel_attn_last_cuda_error.
cudaError_t note_cuda_error(cudaError_t e) { return note(e); }
}  // namespace ira

extern "C" {

size_t inkling_rel_attn_workspace_size(const inkling_rel_attn_dims* dims, int backward) {
    if (check_dims(dims) != INKLING_OK) return 0;
    return workspace_layout(dims->batch, dims->seq_q, dims->heads_q, dims->head_dim, backward != 0).total;
}

inkling_status inkling_rel_attn_validate(const inkling_rel_attn_dims* dims, const uint8_t* valid,
                                         const uint8_t* key_valid, const int32_t* positions,
                                         const int32_t* key_positions, void* workspace, size_t workspace_bytes,
                                         void* stream) {
    NvtxRange nvtx_range("inkling_rel_attn_validate");
    inkling_status s = check_dims(dims);
    if (s != INKLING_OK) return s;
    if (!valid && dims->batch * dims->seq_q > 0) return INKLING_ERR_INVALID_ARG;
    int kpq = 0;
    s = resolve_key_side(dims, valid, key_valid, positions, key_positions, &kpq);
    if (s != INKLING_OK) return s;
    if (!key_valid && dims->batch * dims->seq_k > 0) return INKLING_ERR_INVALID_ARG;
    Ws w;
    s = get_ws(dims, false, workspace, workspace_bytes, &w);
    if (s != INKLING_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int B = int(dims->batch);
    cudaError_t e = cudaMemsetAsync(w.ctl(), 0, 16, st);
    if (e == cudaSuccess && B > 0) e = cudaMemsetAsync(w.edges(), 0, size_t(B) * 8, st);
    if (e == cudaSuccess)
        e = launch_validate(valid, key_valid, positions, key_positions, B, int(dims->seq_q), int(dims->seq_k),
                            int(dims->query_offset), kpq, w.ctl(), w.edges(), st);
    int ctl[4] = {0, 0, 0, 0};
    if (e == cudaSuccess) e = cudaMemcpyAsync(ctl, w.ctl(), 16, cudaMemcpyDeviceToHost, st);
    int* edges = nullptr;
    if (e == cudaSuccess && B > 0) {
        edges = new int[size_t(B) * 2];
        e = cudaMemcpyAsync(edges, w.edges(), size_t(B) * 8, cudaMemcpyDeviceToHost, st);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        delete[] edges;
        return INKLING_ERR_CUDA;
    }
    bool bad = ctl[1] != 0;
    for (int b = 0; b < B && !bad; ++b) bad = edges[2 * b] > 1 || edges[2 * b + 1] > 1;
    delete[] edges;
    return bad ? INKLING_ERR_MALFORMED_POSITIONS : INKLING_OK;
}

inkling_status inkling_rel_attn_fwd(const inkling_rel_attn_dims* dims, const uint16_t* q, const uint16_t* k,
                                    const uint16_t* v, const uint16_t* profiles, const float* sink,
                                    const uint8_t* valid, const uint8_t* key_valid, const int32_t* positions,
                                    const int32_t* key_positions, float* out, float* lse, void* workspace,
                                    size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("inkling_rel_attn_fwd");
    return fwd_impl(dims, q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, workspace,
                    workspace_bytes, stream, nullptr);
}

inkling_status inkling_rel_attn_bwd(const inkling_rel_attn_dims* dims, const uint16_t* q, const uint16_t* k,
                                    const uint16_t* v, const uint16_t* profiles, const float* sink,
                                    const uint8_t* valid, const uint8_t* key_valid, const int32_t* positions,
                                    const int32_t* key_positions, const float* out, const float* lse,
                                    const float* dout, const float* dlse, float* dq, float* dk, float* dv,
                                    float* dprofiles, float* dsink, void* workspace, size_t workspace_bytes,
                                    void* stream) {
    NvtxRange nvtx_range("inkling_rel_attn_bwd");
    return bwd_impl(dims, q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout, dlse,
                    dq, dk, dv, dprofiles, dsink, workspace, workspace_bytes, stream, nullptr);
}

size_t inkling_rel_attn_qclip_workspace_size(const inkling_rel_attn_dims* dims, int backward) {
    if (check_dims(dims) != INKLING_OK) return 0;
    return backward ? qclip_layout(dims).total
                    : workspace_layout(dims->batch, dims->seq_q, dims->heads_q, dims->head_dim, false).total;
}

inkling_status inkling_rel_attn_fwd_qclip(const inkling_rel_attn_dims* dims, double threshold, const float* clip_scale,
                                          const float* tau, const uint16_t* x, const uint16_t* k, const uint16_t* v,
                                          const uint16_t* profiles, const float* sink, const uint8_t* valid,
                                          const uint8_t* key_valid, const int32_t* positions,
                                          const int32_t* key_positions, uint16_t* q_clipped, float* out, float* lse,
                                          void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("inkling_rel_attn_fwd_qclip");
    if (!(threshold >= 0.0) || !std::isfinite(threshold)) return INKLING_ERR_INVALID_ARG;
    if (dims && dims->batch * dims->seq_q > 0 && !q_clipped) return INKLING_ERR_INVALID_ARG;
    if (!aligned16(q_clipped) || !aligned16(x)) return INKLING_ERR_INVALID_ARG;
    QClipArgs qc{};
    qc.thr = float(threshold);
    qc.scale = clip_scale;
    qc.tau = tau;
    qc.q_clipped = q_clipped;
    return fwd_impl(dims, x, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, workspace,
                    workspace_bytes, stream, &qc);
}

inkling_status inkling_rel_attn_bwd_qclip(const inkling_rel_attn_dims* dims, double threshold, const float* clip_scale,
                                          const float* tau, const uint16_t* x, const uint16_t* q_clipped,
                                          const uint16_t* k, const uint16_t* v, const uint16_t* profiles,
                                          const float* sink, const uint8_t* valid, const uint8_t* key_valid,
                                          const int32_t* positions, const int32_t* key_positions, const float* out,
                                          const float* lse, const float* dout, const float* dlse, float* dx, float* dk,
                                          float* dv, float* dprofiles, float* dsink, float* dclip_scale, float* dtau,
                                          void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("inkling_rel_attn_bwd_qclip");
    if (!(threshold >= 0.0) || !std::isfinite(threshold)) return INKLING_ERR_INVALID_ARG;
    if (dims && dims->batch * dims->seq_q > 0 && !x) return INKLING_ERR_INVALID_ARG;
    if ((dclip_scale != nullptr) != (clip_scale != nullptr) || (dtau != nullptr) != (tau != nullptr))
        return INKLING_ERR_INVALID_ARG;
    if (!aligned16(x)) return INKLING_ERR_INVALID_ARG;
    QClipArgs qc{};
    qc.thr = float(threshold);
    qc.scale = clip_scale;
    qc.tau = tau;
    qc.q_raw = x;
    qc.dscale = dclip_scale;
    qc.dtau = dtau;
    return bwd_impl(dims, q_clipped, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse, dout,
                    dlse, dx, dk, dv, dprofiles, dsink, workspace, workspace_bytes, stream, &qc);
}

inkling_status inkling_rel_attn_fwd_noalloc(const inkling_rel_attn_dims* dims, const uint16_t* q, const uint16_t* k,
                                            const uint16_t* v, const uint16_t* profiles, const float* sink,
                                            const uint8_t* valid, const uint8_t* key_valid,
                                            const int32_t* positions, const int32_t* key_positions, float* out,
                                            float* lse, void* stream) {
    NvtxRange nvtx_range("inkling_rel_attn_fwd_noalloc");
    inkling_status s = check_dims(dims);
    if (s != INKLING_OK) return s;
    if (workspace_layout(dims->batch, dims->seq_q, dims->heads_q, dims->head_dim, false).total >
        kNoAllocScratchBytes)
        return INKLING_ERR_UNSUPPORTED;  // problem needs more scratch than the static array holds
    void* scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != INKLING_OK) return s;
    // the ordinary forward, with the static array as its workspace (it clears the
    // device error word itself and rewrites every other scratch byte it reads)
    return inkling_rel_attn_fwd(dims, q, k, v, profiles, sink, valid, key_valid, positions, key_positions, out, lse,
                                scratch, kNoAllocScratchBytes, stream);
}

inkling_status inkling_rel_attn_fwd_noalloc_last_device_error(void* stream) {
    void* scratch = nullptr;
    inkling_status s = noalloc_scratch(&scratch);
    if (s != INKLING_OK) return s;
    // the device error word sits at the start of the array, as in any workspace
    return inkling_rel_attn_last_device_error(scratch, stream);
}

size_t inkling_flex_attn_workspace_size(const inkling_flex_attn_dims* dims, int backward) {
    inkling_rel_attn_dims d;
    if (flex_dims(dims, &d) != INKLING_OK) return 0;
    return flex_layout(d, backward != 0, nullptr).total;
}

inkling_status inkling_flex_attn_fwd(const inkling_flex_attn_dims* dims, const uint16_t* q, const uint16_t* k,
                                     const uint16_t* v, const float* sink_weights, const int64_t* tokens,
                                     uint16_t* out, float* lse, void* workspace, size_t workspace_bytes,
                                     void* stream) {
    NvtxRange nvtx_range("inkling_flex_attn_fwd");
    inkling_rel_attn_dims d;
    inkling_status s = flex_dims(dims, &d);
    if (s != INKLING_OK) return s;
    const int64_t n = d.batch * d.seq_q;
    if (n > 0 && (!q || !k || !v || !out || !lse)) return INKLING_ERR_INVALID_ARG;
    if (n > 0 && dims->mask_type == INKLING_FLEX_BLOCK_CAUSAL && !tokens) return INKLING_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
        return INKLING_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return INKLING_ERR_INVALID_ARG;
    FlexWs fw = flex_layout(d, false, static_cast<uint8_t*>(workspace));
    if (workspace_bytes < fw.total) return INKLING_ERR_INVALID_ARG;
    if (n == 0) return INKLING_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUtensorMap tq, tk, tv;
    if (!encode_bhtd(&tq, q, d.batch, d.seq_q, d.heads_q, d.head_dim, 128, true) ||
        !encode_bhtd(&tk, k, d.batch, d.seq_k, d.heads_kv, d.head_dim, 64, true) ||
        !encode_bhtd(&tv, v, d.batch, d.seq_k, d.heads_kv, d.head_dim, 64, true))
        return INKLING_ERR_CUDA;
    if (flex_masks(dims, tokens, fw, st) != cudaSuccess) return INKLING_ERR_CUDA;
    LaunchTimer tm(st);
    s = run_bounds(&d, fw.w, fw.valid, fw.valid, fw.positions, st, tm);
    if (s != INKLING_OK) return s;
    AttnParams p = base_params(&d, fw.w, nullptr, sink_weights);
    flex_params(p, dims, sink_weights);
    p.out = nullptr;
    p.out_bf16 = out;
    p.lse = lse;
    return cuda_status(tm.run([&] { return launch_fwd(tq, tk, tv, p, st); }));
}

inkling_status inkling_flex_attn_bwd(const inkling_flex_attn_dims* dims, const uint16_t* q, const uint16_t* k,
                                     const uint16_t* v, const float* sink_weights, const int64_t* tokens,
                                     const uint16_t* out, const float* lse, const uint16_t* dout, float* dq,
                                     float* dk, float* dv, float* dsink_weights, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    NvtxRange nvtx_range("inkling_flex_attn_bwd");
    inkling_rel_attn_dims d;
    inkling_status s = flex_dims(dims, &d);
    if (s != INKLING_OK) return s;
    const int64_t n = d.batch * d.seq_q;
    if (n > 0 && (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv)) return INKLING_ERR_INVALID_ARG;
    if (n > 0 && dims->mask_type == INKLING_FLEX_BLOCK_CAUSAL && !tokens) return INKLING_ERR_INVALID_ARG;
    if (sink_weights && !dsink_weights) return INKLING_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return INKLING_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return INKLING_ERR_INVALID_ARG;
    FlexWs fw = flex_layout(d, true, static_cast<uint8_t*>(workspace));
    if (workspace_bytes < fw.total) return INKLING_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n == 0)  // no tokens: the sink weights get no gradient
        return sink_weights ? cuda_status(cudaMemsetAsync(dsink_weights, 0, size_t(d.heads_q) * 4, st)) : INKLING_OK;
    const int64_t B = d.batch, S = d.seq_q, Hq = d.heads_q, Hkv = d.heads_kv, D = d.head_dim;
    auto* lse2t = reinterpret_cast<float*>(fw.w.base + fw.w.L.lse2t);
    auto* dvt = reinterpret_cast<float*>(fw.w.base + fw.w.L.dvt);
    BwdMaps mp;
    std::memset(&mp, 0, sizeof(mp));
    // dO is read by the tensor maps straight from the caller's BF16 [B, H, S, D] tensor
    if (!encode_bhtd(&mp.tq64, q, B, S, Hq, D, 64, true) || !encode_bhtd(&mp.tq128, q, B, S, Hq, D, 128, true) ||
        !encode_bhtd(&mp.tdo64, dout, B, S, Hq, D, 64, true) || !encode_bhtd(&mp.tdo128, dout, B, S, Hq, D, 128, true) ||
        !encode_bhtd(&mp.tk128, k, B, S, Hkv, D, 128, true) || !encode_bhtd(&mp.tv128, v, B, S, Hkv, D, 128, true) ||
        !encode_bhtd(&mp.tk64, k, B, S, Hkv, D, 64, true) || !encode_bhtd(&mp.tv64, v, B, S, Hkv, D, 64, true))
        return INKLING_ERR_CUDA;
    AttnParams p = base_params(&d, fw.w, nullptr, sink_weights);
    flex_params(p, dims, sink_weights);
    p.lse2t = lse2t;
    p.dvt = dvt;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    return bwd_launches(
        &d, fw.w, p, mp, fw.valid, fw.valid, fw.positions, true, st,
        [&](cudaStream_t s2) { return flex_masks(dims, tokens, fw, s2); },
        [&](cudaStream_t s0) {
            cudaError_t e = launch_flex_bwd_prep(int(D), out, dout, lse, sink_weights, 0, 0, 1, int(B), int(S),
                                                 int(Hq), fw.dsink_rows, lse2t, dvt, s0);
            if (e == cudaSuccess && sink_weights)
                e = launch_flex_dsink_reduce(fw.dsink_rows, int(B), int(S), int(Hq), dsink_weights, s0);
            return e;
        });
}

inkling_status inkling_rel_attn_merge(int64_t rows, int64_t head_dim, float* out, float* lse, const float* out_part,
                                      const float* lse_part, void* stream) {
    NvtxRange nvtx_range("inkling_rel_attn_merge");
    if (rows < 0 || (head_dim != 64 && head_dim != 128)) return INKLING_ERR_INVALID_ARG;
    if (rows > 0 && (!out || !lse || !out_part || !lse_part)) return INKLING_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(out_part)) return INKLING_ERR_INVALID_ARG;
    return cuda_status(launch_merge(out, lse, out_part, lse_part, rows, int(head_dim), static_cast<cudaStream_t>(stream)));
}

inkling_status inkling_rel_attn_last_device_error(void* workspace, void* stream) {
    if (!workspace) return INKLING_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return INKLING_ERR_CUDA;
    if (word != 0) {
        e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        return INKLING_ERR_TIMEOUT;
    }
    return INKLING_OK;
}

inkling_status inkling_rel_attn_selftest_wait_timeout(uint32_t timeout_us, void* workspace, size_t workspace_bytes,
                                                      void* stream) {
    if (!workspace || workspace_bytes < 16 || (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
        return INKLING_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, 16, st);
    if (e == cudaSuccess) e = launch_selftest_wait(uint64_t(timeout_us) * 1000ull, static_cast<int*>(workspace), st);
    if (e != cudaSuccess) return INKLING_ERR_CUDA;
    return inkling_rel_attn_last_device_error(workspace, stream);
}

inkling_status inkling_rel_attn_selftest_exp2(const float* t, float* out, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (!t || !out)) || n > (int64_t(1) << 40)) return INKLING_ERR_INVALID_ARG;
    return cuda_status(note(launch_selftest_exp2(t, out, n, static_cast<cudaStream_t>(stream))));
}

inkling_status inkling_rel_attn_set_wait_timeout_ns(uint64_t timeout_ns) {
    g_wait_timeout_ns = timeout_ns;
    return INKLING_OK;
}

inkling_status inkling_rel_attn_set_timing_events(void* const* events, int n_pairs) {
    if (n_pairs < 0) return INKLING_ERR_INVALID_ARG;
    g_events = reinterpret_cast<cudaEvent_t const*>(events);
    g_event_pairs = events ? n_pairs : 0;
    return INKLING_OK;
}

const char* inkling_rel_attn_last_cuda_error(void) {
    return t_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(t_last_cuda_error);
}

#ifdef INKLING_TRACE
// Diagnostic builds only: record the pipeline timeline of CTA `cta` of the next
// attention kernels (8192 steps x 64 events of 8 bytes, see ira::trace_event) and the
// start / end stamps of every CTA of the forward, dK/dV and dQ kernels (three tables of
// 8192 x 8 words after it, see ira::trace_grid) into the device buffer `buf`, which must
// hold 8192 * 64 + 3 * 65536 words; `cta` = -1 records the CTA tables only.
void inkling_rel_attn_debug_trace(void* buf, int cta) {
    g_trace_buf = static_cast<unsigned long long*>(buf);
    g_trace_cta = cta;
}
#endif

const char* inkling_status_string(inkling_status status) {
    switch (status) {
        case INKLING_OK: return "ok";
        case INKLING_ERR_INVALID_ARG: return "invalid argument";
        case INKLING_ERR_UNSUPPORTED: return "unsupported configuration";
        case INKLING_ERR_MALFORMED_POSITIONS: return "malformed validity masks or positions";
        case INKLING_ERR_TIMEOUT: return "device-side wait timed out";
        case INKLING_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

}  // extern "C"
