// bwd.cu -- backward kernels of learned-relative grouped-query attention (sm_100a).
//
// The backward recomputes probabilities from the forward's log-sum-exp
// (P = exp(z - lse), sink included in lse) and applies the softmax chain rule
//   dP = dout . v,  dz = P (dP - Dv),  Dv = <dout, out> - dlse,
//   dq = scale sum_j dz k_j,  dk = scale sum_i dz q_i,  dv = sum_i P dout_i,
//   dprofiles[b,h,i,d] = dz for the allowed key at distance d < R.
// Dv, dsink, a BF16 copy of dout and lse*log2(e) come from the preprocessing
// kernel; dprofiles entries that no allowed key reaches are zeroed by a kernel of
// their own.
//
// Two kernels, both tensor-core (tcgen05) with TMEM accumulators:
//   * dkdv: one CTA per (batch, KV head, 128-key tile). It walks every query
//     head of the group and every 64-row query tile that sees the key tile,
//     computing S^T = K Q^T and dP^T = V dO^T (keys on TMEM lanes), then
//     dV += P^T dO and dK += dS^T Q with P^T / dS^T taken from TMEM. With keys
//     on the lanes, the dprofiles row of a query is written by 32 consecutive
//     distances per warp store (coalesced), with plain stores: each (i, d)
//     has exactly one allowed key.
//   * dq: one CTA per (batch, query head, 128-row query tile) over 64-key
//     tiles: S = Q K^T, dP = dO V^T, dQ += dS K (dS from TMEM). No atomics.
// In both, four elementwise warpgroups split the columns of every step (16 each)
// and S/dP sit in TMEM, double buffered in dkdv and in three buffers in dq, so the
// MMAs of the next steps run while a step is being processed. dkdv's profile band
// comes by TMA from a producer warp; in dq each warp copies its 32 rows' windows
// for its warpgroup's columns.
#include <cstddef>
#include <type_traits>

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace ira {
namespace bwdk {

__device__ __forceinline__ int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }
__device__ __forceinline__ int ceil_div_i(int a, int b) { return -floor_div(-a, b); }

// =====================================================================================
// dK / dV / dprofiles
// =====================================================================================
namespace kv {

constexpr int BK = 128;              // keys per CTA (TMEM lanes)
constexpr int BQ = 64;               // queries per step
constexpr int NWG = 4;               // elementwise warpgroups
constexpr int COLS = BQ / NWG;       // query columns per elementwise warpgroup
constexpr int BAND_LEN = 136;        // bf16 per band row: 128 distances + up to 7 of misalignment
constexpr int BAND_PITCH = BAND_LEN * 2;
// Band rows of a step, fetched as 9 TMA boxes of 8 rows (2176 B each, so every box
// starts on the 128-byte boundary a tensor copy needs): row dm + c holds column c.
constexpr int BAND_BOXES = BQ / 8 + 1;
constexpr int BAND_BYTES = BAND_BOXES * 8 * BAND_PITCH;
constexpr int NB = 3;                // band / column-info buffers
constexpr int KTILE = BK * 128;      // [128 rows x 64 bf16] box
constexpr int QTILE = BQ * 128;      // [64 rows x 64 bf16] box
constexpr int NST = 3;               // Q / dO stages (two steps of lookahead)

// per query column of a step: allowed key range (lo, hi), -lse*log2(e), -Dv
struct StepInfo {
    int2 rb[BQ];
    float nlse2[BQ];
    float ndv[BQ];
    int full;       // every (key, query) pair of the step is allowed
    int pad[3];
};

template <int D>
struct Layout {
    static constexpr int KB = D / 64;
    static constexpr int K_OFF = 0;
    static constexpr int V_OFF = K_OFF + KB * KTILE;
    static constexpr int Q_OFF = V_OFF + KB * KTILE;             // 2 stages
    static constexpr int DO_OFF = Q_OFF + NST * KB * QTILE;      // NST stages
    static constexpr int BAND_OFF = DO_OFF + NST * KB * QTILE;   // NB buffers
    static constexpr int INFO_OFF = BAND_OFF + NB * BAND_BYTES;  // NB buffers
    static constexpr int BAR_OFF = INFO_OFF + NB * int(sizeof(StepInfo));
    // kv_full, qd_full[NST], qd_empty[NST], s_full[2], p_full[2], acc_full, drain,
    // band_full[NB], band_empty[NB]
    static constexpr int NBARS = 7 + 2 * NST + 2 * NB;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int TOTAL = MISC_OFF + 64;
    static constexpr int ALLOC = TOTAL + 1024;
    static constexpr uint32_t DK_COL = 0;
    static constexpr uint32_t DV_COL = D;
    static constexpr uint32_t s_col(int bb) { return uint32_t(2 * D + 128 * bb); }
    static constexpr uint32_t dp_col(int bb) { return uint32_t(2 * D + 128 * bb + 64); }
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int NWARPS = 4 * NWG + 4;
    // registers per thread at launch, and after the split: control warpgroup / elementwise
    static constexpr int REG_LAUNCH = 96, REG_CTRL = 56, REG_EW = 104;
    static_assert(128 * REG_CTRL + 128 * NWG * REG_EW <= 32 * NWARPS * REG_LAUNCH, "register split");
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    // the epilogue stages 32 x 32 chunks of every warp through the K, V, Q and dO tiles
    static_assert(4 * NWG * 32 * 36 * 4 <= BAND_OFF - K_OFF, "epilogue staging");
};

template <int D>
__global__ void __launch_bounds__(32 * (4 * NWG + 4), 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_band, const AttnParams p, const int num_ktiles) {
    using L = Layout<D>;
    constexpr int KB = L::KB;
    constexpr int CTRL = 4 * NWG;
    constexpr int TMA_WARP = CTRL, MMA_WARP = CTRL + 1, BAND_WARP = CTRL + 2, MMA_WARP_B = CTRL + 3;
    extern __shared__ uint8_t smem_raw[];
    // aligned by pointer arithmetic on the __shared__ array, so the compiler keeps
    // knowing that every pointer derived from it addresses shared memory
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* kv_full = bars + 0;
    uint64_t* qd_full = bars + 1;              // [NST]
    uint64_t* qd_empty = bars + 1 + NST;       // [NST]
    uint64_t* s_full = bars + 1 + 2 * NST;     // [2]
    uint64_t* p_full = bars + 3 + 2 * NST;     // [2]
    uint64_t* acc_full = bars + 5 + 2 * NST;
    uint64_t* drain = bars + 6 + 2 * NST;
    uint64_t* band_full = bars + 7 + 2 * NST;       // [NB]
    uint64_t* band_empty = band_full + NB;          // [NB]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    CtaControl* ctl = reinterpret_cast<CtaControl*>(smem + L::MISC_OFF + 16);
    int* tinfo = reinterpret_cast<int*>(smem + L::MISC_OFF + 32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.Hq / p.Hkv;
    const int kt = int(blockIdx.x) % num_ktiles;
    const int bg = int(blockIdx.x) / num_ktiles;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int j0 = kt * BK;
    const int t64 = (p.S + 63) / 64;
    // buffer extents for the bounds-checking build (elements; shared memory in bytes)
    [[maybe_unused]] const uint32_t smem_base = smem_u32(smem);
    [[maybe_unused]] const long long n_rows = (long long)p.B * p.S * p.Hq;

    if (threadIdx.x == 0) {
        IRA_TRACE_GRID(p, 1, 0);
        mbar_init(kv_full, 1);
        // stage, score and accumulator barriers complete once both MMA issuers committed
        for (int u = 0; u < NST; ++u) {
            mbar_init(&qd_full[u], 1);
            mbar_init(&qd_empty[u], 2);
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(&s_full[u], 2);
            mbar_init(&p_full[u], 4 * NWG);
        }
        mbar_init(acc_full, 2);
        mbar_init(drain, 2);
        for (int u = 0; u < NB; ++u) {
            mbar_init(&band_full[u], 1);
            mbar_init(&band_empty[u], 4 * NWG);  // every elementwise warp
        }
        ctl->abort = 0;
        tinfo[0] = 0x7FFFFFFF;  // first query tile that sees the key tile
        tinfo[1] = -1;          // last
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    // query tiles whose allowed key ranges intersect [j0, j0 + BK)
    for (int t = threadIdx.x; t < t64; t += blockDim.x) {
        if (!IRA_IN_BOUNDS(p.err, kErrBoundsDkdvGlobal, size_t(b) * t64 + t, 1, (long long)p.B * t64)) continue;
        const TileBounds tb = p.tile_bounds[size_t(b) * t64 + t];
        if (tb.n_nonempty > 0 && tb.min_lo <= j0 + BK - 1 && tb.max_hi >= j0) {
            atomicMin(&tinfo[0], t);
            atomicMax(&tinfo[1], t);
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int qt_first = tinfo[0];
    const int n_qt = (tinfo[1] >= tinfo[0]) ? tinfo[1] - tinfo[0] + 1 : 0;
    const int n_steps = n_qt * G;
    if (threadIdx.x == 0) {
        IRA_TRACE_GRID(p, 1, 1);
        IRA_TRACE_GRID_INFO(p, 1, n_steps);
    }

    auto k_smem = [&](int kb) { return smem + L::K_OFF + kb * KTILE; };
    auto v_smem = [&](int kb) { return smem + L::V_OFF + kb * KTILE; };
    auto q_smem = [&](int st, int kb) { return smem + L::Q_OFF + (st * KB + kb) * QTILE; };
    auto do_smem = [&](int st, int kb) { return smem + L::DO_OFF + (st * KB + kb) * QTILE; };
    auto step_h = [&](int n) { return g * G + n / n_qt; };
    auto step_qt = [&](int n) { return qt_first + n % n_qt; };

    // Launched with REG_LAUNCH registers per thread; the control warpgroup (tile producer,
    // two MMA issuers, band producer) gives part of its share to the elementwise
    // warpgroups (checked against the launch total in Layout). Each change sits at the
    // top of its branch.
    // A step whose smallest distance delta - 127 is >= R has no profile entry.
    auto band_used = [&](int n) { return p.R > 0 && p.q_off + step_qt(n) * BQ - j0 - (BK - 1) < p.R; };
    if (warp >= CTRL) {
        setmaxnreg_dec<L::REG_CTRL>();
    if (warp == TMA_WARP) {
        if (lane == 0 && n_steps > 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            prefetch_tensormap(&tm_do);
            mbar_arrive_expect_tx(kv_full, 2 * KB * KTILE);
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_4d(k_smem(kb), &tm_k, kv_full, kb * 64, g, j0, b);
                tma_load_4d(v_smem(kb), &tm_v, kv_full, kb * 64, g, j0, b);
            }
            int last = -1;
            for (int n = 0; n < n_steps; ++n) {
                const int st = n % NST;
                if (!mbar_wait(&qd_empty[st], ((n / NST) & 1) ^ 1, ctl, p.err, kErrDkdvQFree, p.timeout_ns)) break;
                const int h = step_h(n), i0 = step_qt(n) * BQ;
                mbar_arrive_expect_tx(&qd_full[st], 2 * KB * QTILE);
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(q_smem(st, kb), &tm_q, &qd_full[st], kb * 64, h, i0, b);
                    tma_load_4d(do_smem(st, kb), &tm_do, &qd_full[st], kb * 64, h, i0, b);
                }
                IRA_TRACE(p, 21, n);
                last = n;
            }
            mbar_wait_drain(kv_full, 0);
            for (int n = (last >= NST ? last - NST + 1 : 0); n <= last; ++n)
                mbar_wait_drain(&qd_full[n % NST], (n / NST) & 1);
        }
    } else if (warp == BAND_WARP) {
        // ------------------------------------------------------------ band producer
        // Per step: the column info (allowed key range, -lse log2 e, -Dv of the 64
        // query rows) by plain loads, then the band: query column c needs the 136
        // profile entries from distance delta + c - 127 - m, m = (delta + c - 127) mod 8
        // (zero outside [0, R)). The columns with the same start (8 consecutive ones)
        // form one 8-row TMA box. NB buffers run ahead of the elementwise warps.
        if (n_steps > 0) {
            // column info of step n in registers (lane handles columns lane and lane + 32),
            // loaded one step before it is stored so the load latency overlaps the wait
            int2 rb_r[2];
            float l2_r[2], dv_r[2];
            bool full_r = false;
            auto load_info = [&](int n) {
                if (n < n_steps &&
                    IRA_IN_BOUNDS(p.err, kErrBoundsDkdvGlobal, size_t(b) * t64 + step_qt(n), 1, (long long)p.B * t64)) {
                    const TileBounds tb = p.tile_bounds[size_t(b) * t64 + step_qt(n)];
                    full_r = tb.n_nonempty == BQ && tb.max_lo <= j0 && tb.min_hi >= j0 + BK - 1;
                }
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    rb_r[k] = make_int2(kEmptyLo, kEmptyHi);
                    l2_r[k] = 0.f;
                    dv_r[k] = 0.f;
                    const int i = step_qt(n) * BQ + lane + 32 * k;
                    const size_t t = (size_t(b) * p.Hq + step_h(n)) * p.S + i;
                    if (n < n_steps && i < p.S &&
                        IRA_IN_BOUNDS(p.err, kErrBoundsDkdvGlobal, size_t(b) * p.S + i, 1, (long long)p.B * p.S) &&
                        IRA_IN_BOUNDS(p.err, kErrBoundsDkdvGlobal, t, 1, n_rows)) {
                        rb_r[k] = p.row_bounds[size_t(b) * p.S + i];
                        l2_r[k] = p.lse2t[t];
                        dv_r[k] = p.dvt[t];
                    }
                }
            };
            load_info(0);
            int last = -1;
            for (int n = 0; n < n_steps; ++n) {
                const int buf = n % NB;
                if (!warp_wait(&band_empty[buf], ((n / NB) & 1) ^ 1, ctl, p.err, kErrDkdvQFree, p.timeout_ns)) break;
                const int h = step_h(n), i0 = step_qt(n) * BQ;
                StepInfo* info = reinterpret_cast<StepInfo*>(smem + L::INFO_OFF) + buf;
                if (!IRA_IN_BOUNDS(p.err, kErrBoundsDkdvSmem, smem_u32(info) - smem_base, sizeof(StepInfo), L::TOTAL))
                    info = reinterpret_cast<StepInfo*>(smem + L::INFO_OFF);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int c = lane + 32 * k;
                    info->rb[c] = rb_r[k];
                    info->nlse2[c] = -l2_r[k];
                    info->ndv[c] = -dv_r[k];
                }
                if (lane == 0) info->full = full_r ? 1 : 0;
                load_info(n + 1);
                __syncwarp();
                if (lane == 0) {
                    const bool used = band_used(n);
                    mbar_arrive_expect_tx(&band_full[buf], used ? BAND_BYTES : 0);
                    if (used) {
                        const int delta = p.q_off + i0 - j0;
                        const int dm = (delta - 127) & 7;
                        const int x0 = delta - 127 - dm;  // multiple of 8
                        const int row0 = (b * p.Hq + h) * p.S + i0 - dm;
                        uint8_t* band = smem + L::BAND_OFF + buf * BAND_BYTES;
                        // box g: shared rows 8g .. 8g+7 = columns 8g - dm .. 8g - dm + 7
                        for (int g8 = 0; g8 < BAND_BOXES; ++g8)
                            if (IRA_IN_BOUNDS(p.err, kErrBoundsDkdvSmem, smem_u32(band + g8 * 8 * BAND_PITCH) - smem_base,
                                              8 * BAND_PITCH, L::TOTAL))
                                tma_load_2d(band + g8 * 8 * BAND_PITCH, &tm_band, &band_full[buf], x0 + 8 * g8,
                                            row0 + 8 * g8);
                    }
                    IRA_TRACE(p, 34, n);
                }
                last = n;
            }
            // never leave a copy in flight into shared memory of an exiting CTA
            if (lane == 0)
                for (int n = (last >= NB ? last - NB + 1 : 0); n <= last; ++n)
                    mbar_wait_drain(&band_full[n % NB], (n / NB) & 1);
        }
    } else if (warp == MMA_WARP || warp == MMA_WARP_B) {
        // ------------------------------------------------------------ MMA issuers
        // Two issuing threads, one per chain, so that one's waits never starve the
        // tensor core: A issues S^T = K Q^T and dV += P^T dO, B issues dP^T = V dO^T and
        // dK += dS^T Q. Each chain overwrites its TMEM buffer only after its own product
        // that read it (the tensor core runs one thread's MMAs in issue order).
        const bool is_b = warp == MMA_WARP_B;
        if (lane == 0 && n_steps > 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BQ, 0, 0);
            constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t a_base = smem_u32(is_b ? v_smem(0) : k_smem(0));
            const uint32_t prod_col = is_b ? L::DK_COL : L::DV_COL;
            auto col_of = [&](int bb) { return is_b ? L::dp_col(bb) : L::s_col(bb); };
            auto b_base = [&](int st) { return smem_u32(is_b ? do_smem(st, 0) : q_smem(st, 0)); };
            auto c_base = [&](int st) { return smem_u32(is_b ? q_smem(st, 0) : do_smem(st, 0)); };
            auto issue_score = [&](int n) {  // S^T (A) or dP^T (B) of step n
                const int st = n % NST, bb = n & 1;
                const uint32_t bs = b_base(st);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * KTILE + (kk & 3) * 32;
                    const uint32_t boff = (kk >> 2) * QTILE + (kk & 3) * 32;
                    mma_ss(tmem + col_of(bb), sdesc_sw128(a_base + off, 16, 1024), sdesc_sw128(bs + boff, 16, 1024),
                           IDESC_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[bb]);
                IRA_TRACE(p, 22, n);
            };
            bool ok = mbar_wait(kv_full, 0, ctl, p.err, kErrDkdvKV, p.timeout_ns) &&
                      mbar_wait(&qd_full[0], 0, ctl, p.err, kErrDkdvQ, p.timeout_ns);
            if (ok) {
                tc_fence_after();
                issue_score(0);
            }
            for (int n = 0; ok && n < n_steps; ++n) {
                if (n + 1 < n_steps) {
                    ok = mbar_wait(&qd_full[(n + 1) % NST], ((n + 1) / NST) & 1, ctl, p.err, kErrDkdvQ, p.timeout_ns);
                    if (!ok) break;
                    if (!is_b) IRA_TRACE(p, 35, n + 1);
                    tc_fence_after();
                    issue_score(n + 1);
                }
                ok = mbar_wait(&p_full[n & 1], (n >> 1) & 1, ctl, p.err, kErrDkdvP, p.timeout_ns);
                if (!ok) break;
                if (!is_b) IRA_TRACE(p, 23, n);
                tc_fence_after();
                const int st = n % NST, bb = n & 1;
                // P^T / dS^T of query columns [16 w, 16 w + 16) sit, packed, at the
                // start of warpgroup w's own S / dP columns
                const uint32_t cs = c_base(st);
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk) {
                    const uint32_t a_off = COLS * kk;
                    mma_ts(tmem + prod_col, tmem + col_of(bb) + a_off, sdesc_sw128(cs + kk * 2048, QTILE, 1024),
                           IDESC_ACC, (n > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&qd_empty[st]);
                if (!is_b) IRA_TRACE(p, 24, n);
            }
            if (ok) mma_commit(acc_full);
            mma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    }
    } else {
        setmaxnreg_inc<L::REG_EW>();
        // ------------------------------------------------------------ elementwise warpgroups
        const int w = warp >> 2;       // this warpgroup takes query columns [16 w, 16 w + 16) of every step
        const int wq = warp & 3;
        const int r = wq * 32 + lane;  // key row (TMEM lane)
        const int j = j0 + r;
        const uint32_t lane_base = uint32_t(wq * 32) << 16;
        const int tid = threadIdx.x & 127;
        const int cw = COLS * w;       // first query column of this warpgroup

        bool ok = true;
        const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 l2e = make_float2(kLog2e, kLog2e);
        for (int n = 0; n < n_steps; ++n) {
            const int bb = n & 1, buf = n % NB;
            const int h = step_h(n), qt = step_qt(n), i0 = qt * BQ;
            const int delta = p.q_off + i0 - j0;
            const bool used = band_used(n);
            // warp-uniform waits: S / dP of the step, then its band rows and column info
            if (!warp_wait(&s_full[bb], (n >> 1) & 1, ctl, p.err, kErrDkdvS, p.timeout_ns) ||
                !warp_wait(&band_full[buf], (n / NB) & 1, ctl, p.err, kErrDkdvQ, p.timeout_ns)) {
                ok = false;
                break;
            }
            if (tid == 0 && w < 2) IRA_TRACE(p, 25 + 3 * w, n);
            tc_fence_after();
            uint32_t sv[COLS], dp[COLS];
            tmem_ld16(tmem + lane_base + L::s_col(bb) + cw, sv);
            tmem_ld16(tmem + lane_base + L::dp_col(bb) + cw, dp);

            // Band reads. Column c = cw + cl reads element (m + 127 - r) of shared band row
            // dm + c, where m = (dm + c) mod 8 repeats every 8 columns (cw is a multiple
            // of 8): eight per-step shared addresses plus compile-time offsets cover them all.
            const int dm = (delta - 127) & 7;
            const uint32_t band_s = smem_u32(smem + L::BAND_OFF + buf * BAND_BYTES + (dm + cw) * BAND_PITCH);
            const uint32_t info_s = smem_u32(smem + L::INFO_OFF + buf * int(sizeof(StepInfo)));
            const bool info_ok = IRA_IN_BOUNDS(p.err, kErrBoundsDkdvSmem, info_s - smem_base, sizeof(StepInfo), L::TOTAL);
            const bool full = info_ok && lds_s32(info_s + offsetof(StepInfo, full)) != 0;
            // dprofiles[b, h, i0 + c, delta + c - r] for column c = cw + cl: the address of
            // column cl is dbase + cl (R + 1) floats
            const long long dp_at0 = ((long long)(b * p.Hq + h) * p.S + i0 + cw) * p.R + (delta + cw - r);
            [[maybe_unused]] const long long dprof_n = n_rows * p.R;
            char* const dbase = reinterpret_cast<char*>(p.dprofiles + dp_at0);
            const uint32_t dstride4 = 4u * uint32_t(p.R + 1);
            // d = delta + c - r < R  <=>  c < R - delta + r (no limit when the whole step is inside R)
            const bool inside = delta + BQ - 1 < p.R;
            const int cl_lim = (inside ? BQ : p.R - delta + r) - cw;
            tmem_wait_ld();
            if (tid == 0 && w == 0) IRA_TRACE(p, 31, n);
            uint32_t pk[COLS / 2], dk[COLS / 2];
            // USED: the step reads profile entries; PLAIN: every (key, query) pair of the
            // step is allowed and inside R, so there is no mask and no store predicate
            auto math = [&](auto used_c, auto plain_c) {
                constexpr bool USED = decltype(used_c)::value, PLAIN = decltype(plain_c)::value;
#pragma unroll
                for (int c4 = 0; c4 < COLS / 4; ++c4) {
                    // loads of this 4-column chunk: 128-bit broadcast reads of the column info
                    const int c = cw + 4 * c4;
                    const float4 l4 = info_ok ? lds_f32x4(info_s + offsetof(StepInfo, nlse2) + 4 * c)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 v4 = info_ok ? lds_f32x4(info_s + offsetof(StepInfo, ndv) + 4 * c)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float nl_c[4] = {l4.x, l4.y, l4.z, l4.w};
                    const float nv_c[4] = {v4.x, v4.y, v4.z, v4.w};
                    int lo_c[4] = {0, 0, 0, 0}, hi_c[4] = {0, 0, 0, 0};
                    if (!PLAIN && info_ok) {
                        const int4 a4 = lds_s32x4(info_s + offsetof(StepInfo, rb) + 8 * c);
                        const int4 b4 = lds_s32x4(info_s + offsetof(StepInfo, rb) + 8 * c + 16);
                        lo_c[0] = a4.x; hi_c[0] = a4.y; lo_c[1] = a4.z; hi_c[1] = a4.w;
                        lo_c[2] = b4.x; hi_c[2] = b4.y; lo_c[3] = b4.z; hi_c[3] = b4.w;
                    }
                    float bias_c[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int cl = 4 * c4 + u;
                        const uint32_t ba = band_s + (cl & 7) * BAND_PITCH + 2 * (((dm + cl) & 7) + 127 - r) +
                                            BAND_PITCH * 8 * (cl >> 3);
                        bias_c[u] = USED && IRA_IN_BOUNDS(p.err, kErrBoundsDkdvSmem, ba - smem_base, 2, L::TOTAL)
                                        ? __uint_as_float(lds_u16(ba) << 16)
                                        : 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; u += 2) {
                        const int cl = 4 * c4 + u;
                        // log2-domain logit, probability, dS = P (dP - Dv), two columns at a time
                        float2 z = __ffma2_rn(make_float2(__uint_as_float(sv[cl]), __uint_as_float(sv[cl + 1])), sl2,
                                              make_float2(nl_c[u], nl_c[u + 1]));
                        if (USED) z = __ffma2_rn(make_float2(bias_c[u], bias_c[u + 1]), l2e, z);
                        float2 pr = ((IRA_DKDV_FMA_PAIRS >> ((cl >> 1) & 15)) & 1u)
                                        ? exp2_fma2(z)
                                        : make_float2(ex2_approx(z.x), ex2_approx(z.y));
                        bool ok0 = true, ok1 = true;
                        if (!PLAIN) {
                            ok0 = uint32_t(j - lo_c[u]) <= uint32_t(hi_c[u] - lo_c[u]) && cl < cl_lim;
                            ok1 = uint32_t(j - lo_c[u + 1]) <= uint32_t(hi_c[u + 1] - lo_c[u + 1]) && cl + 1 < cl_lim;
                            pr.x = (uint32_t(j - lo_c[u]) <= uint32_t(hi_c[u] - lo_c[u])) ? pr.x : 0.f;
                            pr.y = (uint32_t(j - lo_c[u + 1]) <= uint32_t(hi_c[u + 1] - lo_c[u + 1])) ? pr.y : 0.f;
                        }
                        const float2 ds = __fmul2_rn(
                            pr, __fadd2_rn(make_float2(__uint_as_float(dp[cl]), __uint_as_float(dp[cl + 1])),
                                           make_float2(nv_c[u], nv_c[u + 1])));
                        float* const a0 = reinterpret_cast<float*>(dbase + size_t(uint32_t(cl) * dstride4));
                        float* const a1 = reinterpret_cast<float*>(dbase + size_t(uint32_t(cl + 1) * dstride4));
                        if ((PLAIN || ok0) &&
                            IRA_IN_BOUNDS(p.err, kErrBoundsDkdvGlobal, dp_at0 + (long long)cl * (p.R + 1), 1, dprof_n))
                            __stcs(a0, ds.x);
                        if ((PLAIN || ok1) && IRA_IN_BOUNDS(p.err, kErrBoundsDkdvGlobal,
                                                            dp_at0 + (long long)(cl + 1) * (p.R + 1), 1, dprof_n))
                            __stcs(a1, ds.y);
                        pk[cl >> 1] = pack_bf16x2(pr.x, pr.y);
                        dk[cl >> 1] = pack_bf16x2(ds.x, ds.y);
                    }
                }
            };
            using T_ = std::true_type;
            using F_ = std::false_type;
            if (used) {
                if (full && inside) math(T_{}, T_{}); else math(T_{}, F_{});
            } else {
                if (full && inside) math(F_{}, T_{}); else math(F_{}, F_{});
            }
            if (tid == 0 && w == 0) IRA_TRACE(p, 32, n);
            tmem_st8(tmem + lane_base + L::s_col(bb) + cw, pk);
            tmem_st8(tmem + lane_base + L::dp_col(bb) + cw, dk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&p_full[bb]);
                mbar_arrive(&band_empty[buf]);
            }
            if (tid == 0 && w < 2) IRA_TRACE(p, 26 + 3 * w, n);
        }

        // ---- epilogue: warpgroups 0 and 1 write dK (scaled), 2 and 3 dV, half of the
        // columns each ----
        if (ok && n_steps > 0) {
            ok = warp_wait(acc_full, 0, ctl, p.err, kErrDkdvAcc, p.timeout_ns);
            tc_fence_after();
        }
        if (ok) {
            const bool row_in = j < p.Skv;
            const bool is_dv = w >= 2;
            const int c0 = (w & 1) * (D / 2);  // first of this warpgroup's D / 2 columns
            float* dst = (is_dv ? p.dv : p.dk) + (b * p.kv_sb + j * p.kv_ss + g * p.kv_sh);
            float* const base = (is_dv ? p.dv : p.dk) + (b * p.kv_sb + g * p.kv_sh);
            const float mul = is_dv ? 1.f : p.scale;
            const uint32_t col = (is_dv ? L::DV_COL : L::DK_COL) + c0;
            if (n_steps > 0) {
                // 32 x 32 chunks go out through shared memory (the key / query tiles, idle once
                // every MMA has completed), 144-byte pitch per row: each lane writes its row,
                // then 8 lanes store 128 contiguous bytes of one row, four rows per store
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                float* const stage = reinterpret_cast<float*>(smem + L::K_OFF) + (4 * w + wq) * 32 * 36;
                const int sr = lane >> 3, sc = 4 * (lane & 7);
#pragma unroll 1
                for (int c4 = 0; c4 < D / 64; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + col + 32 * c4, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        if (IRA_IN_BOUNDS(p.err, kErrBoundsDkdvSmem, smem_u32(stage + lane * 36 + 4 * q) - smem_base, 16,
                                          L::TOTAL))
                            *reinterpret_cast<float4*>(stage + lane * 36 + 4 * q) =
                                make_float4(__uint_as_float(o[4 * q]) * mul, __uint_as_float(o[4 * q + 1]) * mul,
                                            __uint_as_float(o[4 * q + 2]) * mul, __uint_as_float(o[4 * q + 3]) * mul);
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int rr = 4 * k + sr;          // row of this warp
                        const int jr = j0 + 32 * wq + rr;   // its key
                        const bool st_ok = IRA_IN_BOUNDS(p.err, kErrBoundsDkdvSmem, smem_u32(stage + rr * 36 + sc) - smem_base,
                                                         16, L::TOTAL);
                        const float4 v = st_ok ? *reinterpret_cast<const float4*>(stage + rr * 36 + sc)
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
                        [[maybe_unused]] const long long at =
                            b * p.kv_sb + g * p.kv_sh + (long long)jr * p.kv_ss + c0 + 32 * c4 + sc;
                        if (jr < p.Skv &&
                            IRA_IN_BOUNDS(p.err, kErrBoundsDkdvGlobal, at, 4, (long long)p.B * p.Skv * p.Hkv * D))
                            *reinterpret_cast<float4*>(base + jr * p.kv_ss + c0 + 32 * c4 + sc) = v;
                    }
                    __syncwarp();
                }
            } else if (row_in && IRA_IN_BOUNDS(p.err, kErrBoundsDkdvGlobal,
                                               b * p.kv_sb + (long long)j * p.kv_ss + g * p.kv_sh + c0, D / 2,
                                               (long long)p.B * p.Skv * p.Hkv * D)) {
                for (int e = c0; e < c0 + D / 2; e += 4)
                    *reinterpret_cast<float4*>(dst + e) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }

    if (threadIdx.x == 0) IRA_TRACE_GRID(p, 1, 4);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
        if (lane == 0) IRA_TRACE_GRID(p, 1, 5);
    }
}

template <int D>
cudaError_t launch(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                   const CUtensorMap& tm_do, const CUtensorMap& tm_band, const AttnParams& p, cudaStream_t st) {
    using L = Layout<D>;
    auto kern = dkdv_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    const int nkt = (p.Skv + BK - 1) / BK;
    const long long grid = (long long)nkt * p.B * p.Hkv;
    if (grid == 0) return cudaSuccess;
    kern<<<dim3(unsigned(grid)), dim3(32 * L::NWARPS), L::ALLOC, st>>>(tm_q, tm_k, tm_v, tm_do, tm_band, p, nkt);
    return cudaGetLastError();
}

}  // namespace kv

// =====================================================================================
// dQ
// =====================================================================================
namespace dqk {

constexpr int BM = 128;               // query rows per CTA (TMEM lanes)
constexpr int BN = 64;                // keys per step
constexpr int NWG = 4;                // elementwise warpgroups
constexpr int COLS = BN / NWG;        // key columns per elementwise warpgroup
constexpr int BAND_CHUNKS = 3;        // 24 bf16 per row window (16 columns + misalignment)
constexpr int BAND_UNITS = BAND_CHUNKS * BM + 2 * (BM / 8);
constexpr int BAND_BYTES = BAND_UNITS * 16;
constexpr int QTILE = BM * 128;       // [128 x 64 bf16]
constexpr int KTILE = BN * 128;       // [64 x 64 bf16]
constexpr int NSB = 3;                // S / dP buffers in TMEM: the MMAs run two steps ahead
constexpr int NSK = 4;                // K stages: K(n) is read by S(n) and, two steps later, by dQ(n)
constexpr int NSV = 2;                // V stages: V(n) is read by dP(n) only

// Row r's window starts at 16-byte unit 3 r + 2 floor(r / 8) of its buffer; with the
// row's misalignment (r + 1) mod 8 the column-wise 32-bit reads of a warp hit 32
// distinct banks.
__host__ __device__ constexpr int band_unit(int r) { return BAND_CHUNKS * r + 2 * (r >> 3); }

template <int D>
struct Layout {
    static constexpr int KB = D / 64;
    static constexpr int Q_OFF = 0;
    static constexpr int DO_OFF = Q_OFF + KB * QTILE;
    static constexpr int K_OFF = DO_OFF + KB * QTILE;          // NSK stages
    static constexpr int V_OFF = K_OFF + NSK * KB * KTILE;     // NSV stages
    static constexpr int BAND_OFF = V_OFF + NSV * KB * KTILE;  // [warpgroup][step parity]
    // fused L2Clip backward: row sums [lane quarter][warpgroup][lane] float2, then column
    // sums [warpgroup][lane quarter][column] floats
    static constexpr int XCH_OFF = BAND_OFF + NWG * 2 * BAND_BYTES;
    static constexpr int XCH_BYTES = 4 * NWG * 32 * 8 + NWG * 4 * 32 * 4;
    static constexpr int BAR_OFF = XCH_OFF + XCH_BYTES;
    // q_full, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV], s_full[NSB], p_full[NSB],
    // acc_full, drain
    static constexpr int NBARS = 3 + 2 * NSK + 2 * NSV + 2 * NSB;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int TOTAL = MISC_OFF + 64;
    static constexpr int ALLOC = TOTAL + 1024;
    static constexpr uint32_t DQ_COL = 0;
    static constexpr uint32_t s_col(int bb) { return uint32_t(D + 128 * bb); }
    static constexpr uint32_t dp_col(int bb) { return uint32_t(D + 128 * bb + 64); }
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int NWARPS = 4 * NWG + 4;
    // registers per thread at launch, and after the split: control warpgroup / elementwise
    static constexpr int REG_LAUNCH = 96, REG_CTRL = 56, REG_EW = 104;
    static_assert(128 * REG_CTRL + 128 * NWG * REG_EW <= 32 * NWARPS * REG_LAUNCH, "register split");
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    // the epilogue stages the D / NWG dQ columns of each warp's 32 rows through the K
    // and V rings (contiguous, idle by then), 4 floats of padding per row
    static constexpr int DC = D / NWG;
    static constexpr int STAGE_PITCH = DC + 4;
    static_assert(4 * NWG * 32 * STAGE_PITCH * 4 <= (NSK + NSV) * KB * KTILE, "epilogue staging");
};

// CLIP: the L2Clip backward of q is fused into the epilogue (dq of the clipped q becomes
// the gradient of the unclipped q, plus this CTA's parts of dscale and dtau).
template <int D, bool CLIP>
__global__ void __launch_bounds__(32 * (4 * NWG + 4), 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const AttnParams p, const int num_qtiles) {
    using L = Layout<D>;
    constexpr int KB = L::KB;
    constexpr int CTRL = 4 * NWG;
    constexpr int TMA_WARP = CTRL, MMA_WARP = CTRL + 1, V_WARP = CTRL + 2, MMA_WARP_B = CTRL + 3;
    extern __shared__ uint8_t smem_raw[];
    // aligned by pointer arithmetic on the __shared__ array, so the compiler keeps
    // knowing that every pointer derived from it addresses shared memory
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;               // [NSK]
    uint64_t* k_empty = k_full + NSK;          // [NSK]
    uint64_t* v_full = k_empty + NSK;          // [NSV]
    uint64_t* v_empty = v_full + NSV;          // [NSV]
    uint64_t* s_full = v_empty + NSV;          // [NSB]
    uint64_t* p_full = s_full + NSB;           // [NSB]
    uint64_t* acc_full = p_full + NSB;
    uint64_t* drain = acc_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    CtaControl* ctl = reinterpret_cast<CtaControl*>(smem + L::MISC_OFF + 16);
    int* tinfo = reinterpret_cast<int*>(smem + L::MISC_OFF + 32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_tile = p.B * p.Hq;
    const int qt = num_qtiles - 1 - int(blockIdx.x) / per_tile;
    const int rem = int(blockIdx.x) % per_tile;
    const int b = rem / p.Hq, h = rem % p.Hq;
    const int g = h / (p.Hq / p.Hkv);
    const int i0 = qt * BM;
    const int i0g = p.q_off + i0;
    const int t64 = (p.S + 63) / 64;
    // buffer extents for the bounds-checking build (elements; shared memory in bytes)
    [[maybe_unused]] const uint32_t smem_base = smem_u32(smem);
    [[maybe_unused]] const long long n_rows = (long long)p.B * p.S * p.Hq;

    if (threadIdx.x == 0) {
        IRA_TRACE_GRID(p, 2, 0);
        mbar_init(q_full, 1);
        // a K stage is free once S (issuer A) and dQ (issuer B) of its step completed,
        // a V stage once dP (issuer B) did
        for (int u = 0; u < NSK; ++u) {
            mbar_init(&k_full[u], 1);
            mbar_init(&k_empty[u], 2);
        }
        for (int u = 0; u < NSV; ++u) {
            mbar_init(&v_full[u], 1);
            mbar_init(&v_empty[u], 1);
        }
        for (int u = 0; u < NSB; ++u) {
            mbar_init(&s_full[u], 2);           // S (issuer A) and dP (issuer B)
            mbar_init(&p_full[u], 4 * NWG);     // every elementwise warp
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 2);
        ctl->abort = 0;
        const TileBounds* tb = p.tile_bounds + size_t(b) * t64 + 2 * qt;
        const bool tb_ok = IRA_IN_BOUNDS(p.err, kErrBoundsDqGlobal, size_t(b) * t64 + 2 * qt,
                                         (2 * qt + 1 < t64) ? 2 : 1, (long long)p.B * t64);
        int min_lo = tb_ok ? tb[0].min_lo : 0, max_hi = tb_ok ? tb[0].max_hi : -1, ne = tb_ok ? tb[0].n_nonempty : 0;
        if (tb_ok && 2 * qt + 1 < t64) {
            min_lo = min(min_lo, tb[1].min_lo);
            max_hi = max(max_hi, tb[1].max_hi);
            ne += tb[1].n_nonempty;
        }
        int t_begin = 0, n_steps = 0;
        if (ne > 0) {
            // step t covers keys [i0g + 64 - 64 t, i0g + 127 - 64 t]
            t_begin = max(0, ceil_div_i(i0g + BN - max_hi, BN));
            const int t_end = floor_div(i0g + 2 * BN - 1 - min_lo, BN);
            n_steps = max(0, t_end - t_begin + 1);
        }
        tinfo[0] = t_begin;
        tinfo[1] = n_steps;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int t_begin = tinfo[0];
    const int n_steps = tinfo[1];
    if (threadIdx.x == 0) {
        IRA_TRACE_GRID(p, 2, 1);
        IRA_TRACE_GRID_INFO(p, 2, n_steps);
    }

    auto q_smem = [&](int kb) { return smem + L::Q_OFF + kb * QTILE; };
    auto do_smem = [&](int kb) { return smem + L::DO_OFF + kb * QTILE; };
    auto k_smem = [&](int n, int kb) { return smem + L::K_OFF + ((n % NSK) * KB + kb) * KTILE; };
    auto v_smem = [&](int n, int kb) { return smem + L::V_OFF + ((n % NSV) * KB + kb) * KTILE; };
    auto key0 = [&](int n) { return i0g + BN - (t_begin + n) * BN; };

    // Launched with REG_LAUNCH registers per thread; the control warpgroup (producers,
    // two MMA issuers) gives part of its share to the elementwise warpgroups (checked
    // against the launch total above). Each change sits at the top of its branch.
    if (warp >= CTRL) {
        setmaxnreg_dec<L::REG_CTRL>();
    if (warp == TMA_WARP || warp == V_WARP) {
        // ------------------------------------------------------------ tile producers:
        // Q and dO once plus the K ring (TMA_WARP), the V ring (V_WARP)
        const bool is_v = warp == V_WARP;
        if (lane == 0 && n_steps > 0) {
            if (!is_v) {
                prefetch_tensormap(&tm_q);
                prefetch_tensormap(&tm_do);
                prefetch_tensormap(&tm_k);
                mbar_arrive_expect_tx(q_full, 2 * KB * QTILE);
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_4d(q_smem(kb), &tm_q, q_full, kb * 64, h, i0, b);
                    tma_load_4d(do_smem(kb), &tm_do, q_full, kb * 64, h, i0, b);
                }
            } else {
                prefetch_tensormap(&tm_v);
            }
            const int ns = is_v ? NSV : NSK;
            uint64_t* full = is_v ? v_full : k_full;
            uint64_t* empty = is_v ? v_empty : k_empty;
            int last = -1;
            for (int n = 0; n < n_steps; ++n) {
                const int st = n % ns;
                if (!mbar_wait(&empty[st], ((n / ns) & 1) ^ 1, ctl, p.err, kErrDqKVFree, p.timeout_ns)) break;
                mbar_arrive_expect_tx(&full[st], KB * KTILE);
                for (int kb = 0; kb < KB; ++kb) {
                    if (is_v)
                        tma_load_4d(v_smem(n, kb), &tm_v, &full[st], kb * 64, g, key0(n), b);
                    else
                        tma_load_4d(k_smem(n, kb), &tm_k, &full[st], kb * 64, g, key0(n), b);
                }
                IRA_TRACE(p, is_v ? 50 : 41, n);
                last = n;
            }
            if (!is_v) mbar_wait_drain(q_full, 0);
            for (int n = (last >= ns ? last - ns + 1 : 0); n <= last; ++n)
                mbar_wait_drain(&full[n % ns], (n / ns) & 1);
        }
    } else if (warp == MMA_WARP || warp == MMA_WARP_B) {
        // ------------------------------------------------------------ MMA issuers
        // Two issuing threads so that one's waits never starve the tensor core:
        // A issues S = Q K^T; B issues dP = dO V^T and dQ += dS K (dS from TMEM). With
        // three S / dP buffers the scores of step n + 2 are issued while the elementwise
        // warps work on step n + 1. Each issuer overwrites a buffer only after the
        // elementwise warps are done with the step that used it, and B's dQ of that
        // step precedes it in B's issue order.
        const bool is_b = warp == MMA_WARP_B;
        if (lane == 0 && n_steps > 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, 0, 0);
            constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t a_base = smem_u32(is_b ? do_smem(0) : q_smem(0));
            auto wait_tile = [&](int n) {  // K(n) for A, V(n) for B
                return is_b ? mbar_wait(&v_full[n % NSV], (n / NSV) & 1, ctl, p.err, kErrDqKV, p.timeout_ns)
                            : mbar_wait(&k_full[n % NSK], (n / NSK) & 1, ctl, p.err, kErrDqKV, p.timeout_ns);
            };
            auto issue_score = [&](int n) {  // S (A) or dP (B) of step n
                const int bb = n % NSB;
                const uint32_t bs = smem_u32(is_b ? v_smem(n, 0) : k_smem(n, 0));
                const uint32_t col = is_b ? L::dp_col(bb) : L::s_col(bb);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t aoff = (kk >> 2) * QTILE + (kk & 3) * 32;
                    const uint32_t boff = (kk >> 2) * KTILE + (kk & 3) * 32;
                    mma_ss(tmem + col, sdesc_sw128(a_base + aoff, 16, 1024), sdesc_sw128(bs + boff, 16, 1024), IDESC_S,
                           kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[bb]);
                // last read of V(n) by B; A's read of K(n)
                mma_commit(is_b ? &v_empty[n % NSV] : &k_empty[n % NSK]);
                IRA_TRACE(p, is_b ? 51 : 42, n);
            };
            bool ok = mbar_wait(q_full, 0, ctl, p.err, kErrDqQ, p.timeout_ns);
            for (int n = 0; ok && n < 2 && n < n_steps; ++n) {
                ok = wait_tile(n);
                if (!ok) break;
                tc_fence_after();
                issue_score(n);
            }
            for (int n = 0; ok && n < n_steps; ++n) {
                // S / dP of step n + 2 go into the buffer of step n - 1, free once the
                // elementwise warps are done with it (P(n-1), awaited last iteration)
                // and, for B, behind dQ(n-1) in issue order
                if (n + 2 < n_steps) {
                    ok = wait_tile(n + 2);
                    if (!ok) break;
                    if (!is_b) IRA_TRACE(p, 49, n + 2);
                    tc_fence_after();
                    issue_score(n + 2);
                }
                ok = mbar_wait(&p_full[n % NSB], (n / NSB) & 1, ctl, p.err, kErrDqP, p.timeout_ns);
                if (!ok) break;
                if (!is_b) continue;
                // K(n) arrived long ago (A issued S(n) on it); B takes the same phase
                // for its own ordering with the copy
                ok = mbar_wait(&k_full[n % NSK], (n / NSK) & 1, ctl, p.err, kErrDqKV, p.timeout_ns);
                if (!ok) break;
                IRA_TRACE(p, 43, n);
                tc_fence_after();
                const int bb = n % NSB;
                const uint32_t ks = smem_u32(k_smem(n, 0));
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // dS of key columns [16 w, 16 w + 16) sits, packed, at the start of
                    // warpgroup w's own 16 dP columns
                    mma_ts(tmem + L::DQ_COL, tmem + L::dp_col(bb) + COLS * kk,
                           sdesc_sw128(ks + kk * 2048, KTILE, 1024), IDESC_DQ, (n > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&k_empty[n % NSK]);
                IRA_TRACE(p, 44, n);
            }
            if (ok && is_b) mma_commit(acc_full);
            mma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    }
    } else {
        setmaxnreg_inc<L::REG_EW>();
        const int w = warp >> 2;       // this warpgroup takes key columns [16 w, 16 w + 16) of every step
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_base = uint32_t(wq * 32) << 16;
        const int cw = COLS * w;
        const int i = i0 + r;
        const size_t trow = (size_t(b) * p.Hq + h) * p.S + i;
        const bool row_in = i < p.S &&
                            IRA_IN_BOUNDS(p.err, kErrBoundsDqGlobal, size_t(b) * p.S + i, 1, (long long)p.B * p.S) &&
                            IRA_IN_BOUNDS(p.err, kErrBoundsDqGlobal, trow, 1, n_rows);
        const int2 rb = row_in ? p.row_bounds[size_t(b) * p.S + i] : make_int2(kEmptyLo, kEmptyHi);
        const bool empty = rb.x > rb.y;
        const float lse2 = row_in ? p.lse2t[trow] : 0.f;
        const float dvr = row_in ? p.dvt[trow] : 0.f;

        // This row's profile window for the warpgroup's columns (copied by the warp, see
        // issue_band), double buffered by step parity: column c = cw + cl of step n has
        // distance delta(n) + r - c; the 16 columns' window starts (r + 1) mod 8
        // elements past a 16-byte boundary.
        const int unit = band_unit(r);
        uint8_t* const band_wg = smem + L::BAND_OFF + w * 2 * BAND_BYTES;
        const int m_r = (r + 1) & 7;
        const int g_r = m_r >> 1;
        const uint32_t fshift = uint32_t(m_r & 1) * 16u;
        [[maybe_unused]] const long long prof_n = n_rows * p.R;
        // step n has distance offset delta = i0g - key0(n) = 64 (t_begin + n) - 64
        auto delta_of = [&](int n) { return BN * (t_begin + n) - BN; };
        // the warp's smallest distance in this warpgroup's columns is delta + 32 wq - cw - 15
        auto band_needed = [&](int n) { return delta_of(n) + wq * 32 - cw - (COLS - 1) < p.R; };
        // The warp copies the windows of its 32 rows together: chunk k = 32 t + lane of its
        // 32 x 3 chunks is chunk k mod 3 of row k / 3, so one copy instruction reads ~11
        // contiguous row segments rather than 32 rows. One cp.async group per call, also
        // when nothing is copied; a row is read only after every lane's wait and a
        // __syncwarp.
        const size_t prof_tile_at = ((size_t(b) * p.Hq + h) * p.S + i0) * size_t(p.R);
        const uint16_t* const prof_tile = p.R > 0 ? p.profiles + prof_tile_at : nullptr;
        auto issue_band = [&](int n) {
            if (n < n_steps && band_needed(n)) {
                uint8_t* const dst_buf = band_wg + (n & 1) * BAND_BYTES;
                const int dl = delta_of(n) - cw - (COLS - 1);
#pragma unroll
                for (int t = 0; t < BAND_CHUNKS; ++t) {
                    const int k = 32 * t + lane;
                    const int rr = wq * 32 + k / BAND_CHUNKS, q = k % BAND_CHUNKS;
                    const int d0 = dl + rr - ((rr + 1) & 7) + 8 * q;
                    const bool inb = prof_tile != nullptr && i0 + rr < p.S && d0 >= 0 && d0 < p.R;
                    const size_t at = size_t(rr) * p.R + d0;
                    const void* src = inb ? static_cast<const void*>(prof_tile + at) : p.safe_src;
                    const uint32_t dst = smem_u32(dst_buf + band_unit(rr) * 16 + 16 * q);
                    if (IRA_IN_BOUNDS(p.err, kErrBoundsDqSmem, dst - smem_base, 16, L::TOTAL) &&
                        IRA_IN_BOUNDS(p.err, kErrBoundsDqGlobal, inb ? prof_tile_at + at : 0, inb ? 8 : 0, prof_n))
                        cp_async_16(dst, src, inb ? 16u : 0u);
                }
            }
            cp_async_commit();
        };

        issue_band(0);
        issue_band(1);
        // the fused clip's epilogue reads this thread's part of its row of x: warm the L2
        if (CLIP && row_in) prefetch_l2(p.q_raw + ((size_t(b) * p.S + i) * p.Hq + h) * D + w * (D / NWG));
        bool ok = true;
        const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 l2e = make_float2(kLog2e, kLog2e);
        const float2 nl2 = make_float2(-lse2, -lse2);
        const float2 nv2 = make_float2(-dvr, -dvr);
        for (int n = 0; n < n_steps; ++n) {
            const int bb = n % NSB;
            const int jk = key0(n) + cw;  // key of this warpgroup's first column
            const bool my_full = empty || (rb.x <= jk && rb.y >= jk + COLS - 1);
            const bool need_mask = !__all_sync(0xffffffffu, my_full);
            const bool use_band = band_needed(n);
            if (!warp_wait(&s_full[bb], (n / NSB) & 1, ctl, p.err, kErrDqS, p.timeout_ns)) {
                ok = false;
                break;
            }
            if (wq == 0 && lane == 0) IRA_TRACE(p, 45 + 2 * (w & 1), n);
            tc_fence_after();
            uint32_t sv[COLS], dp[COLS];
            tmem_ld16(tmem + lane_base + L::s_col(bb) + cw, sv);
            tmem_ld16(tmem + lane_base + L::dp_col(bb) + cw, dp);
            uint32_t wv[COLS / 2 + 1];
            if (use_band) {
                cp_async_wait_group<1>();  // this step's windows (the next step's may fly)
                __syncwarp();              // ... copied by every lane of the warp
                const uint32_t* words = reinterpret_cast<const uint32_t*>(band_wg + (n & 1) * BAND_BYTES + unit * 16) + g_r;
                const bool w_ok = IRA_IN_BOUNDS(p.err, kErrBoundsDqSmem, smem_u32(words) - smem_base,
                                                4 * (COLS / 2 + 1), L::TOTAL);
#pragma unroll
                for (int q = 0; q < COLS / 2 + 1; ++q) wv[q] = w_ok ? words[q] : 0u;
            }
            if (wq == 0 && lane == 0) IRA_TRACE(p, 52 + (w & 1), n);
            // this step's windows are in registers (every lane's: the copies are shared):
            // fetch the ones of step n + 2 into their buffer
            __syncwarp();
            issue_band(n + 2);
            tmem_wait_ld();
            if (wq == 0 && lane == 0) IRA_TRACE(p, 54 + (w & 1), n);
            const int c_lo = rb.x - jk, c_hi = rb.y - jk;  // allowed columns of this row
            uint32_t dk[COLS / 2];
#pragma unroll
            for (int pp = 0; pp < COLS / 2; ++pp) {
                const int c = 2 * pp;
                float2 t = nl2;
                if (use_band) {
                    const uint32_t v = funnel_r(wv[COLS / 2 - 1 - pp], wv[COLS / 2 - pp], fshift);
                    t = __ffma2_rn(make_float2(bf16hi_to_f32(v), bf16lo_to_f32(v)), l2e, nl2);
                }
                const float2 z = __ffma2_rn(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2, t);
                float2 pr = ((IRA_DQ_FMA_PAIRS >> (pp & 15)) & 1u) ? exp2_fma2(z)
                                                                   : make_float2(ex2_approx(z.x), ex2_approx(z.y));
                if (need_mask) {
                    pr.x = (c >= c_lo && c <= c_hi) ? pr.x : 0.f;
                    pr.y = (c + 1 >= c_lo && c + 1 <= c_hi) ? pr.y : 0.f;
                }
                const float2 ds =
                    __fmul2_rn(pr, __fadd2_rn(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), nv2));
                dk[pp] = pack_bf16x2(ds.x, ds.y);
            }
            if (wq == 0 && lane == 0) IRA_TRACE(p, 56 + (w & 1), n);
            tmem_st8(tmem + lane_base + L::dp_col(bb) + cw, dk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[bb]);
            if (wq == 0 && lane == 0) IRA_TRACE(p, 46 + 2 * (w & 1), n);
        }
        cp_async_wait_all();

        // Fused L2Clip backward (CLIP). dy = dq of the clipped q; per row (b, i, h):
        //   z = x * scale, n = |z|, c = min(1, thr / n);
        //   dz = tau c (dy - ((z . dy) / n^2) z) when n > thr, else tau dy;
        //   dx = dz * scale (written where dq goes), dtau part c (z . dy), dscale part dz * x.
        // Each warpgroup holds a quarter of the columns: the row sums z . z and z . dy go
        // through shared memory among the four warps of a lane quarter (barrier 1 + wq), the
        // column sums of dz * x over the CTA's rows among the four warps of a warpgroup
        // (barrier 5 + w); both in a fixed order. Every warp takes both barriers, also after
        // a failed wait; only the stores depend on it.
        auto clip_epilogue = [&](bool ok_out) {
            constexpr int DC = L::DC, STAGE_PITCH = L::STAGE_PITCH;
            const int col = w * DC;
            float dy[DC];
            if (ok_out && n_steps > 0) {
                uint32_t o[DC];
                if constexpr (DC == 32) {
                    tmem_ld32(tmem + lane_base + L::DQ_COL + col, o);
                } else {
                    tmem_ld16(tmem + lane_base + L::DQ_COL + col, o);
                }
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < DC; ++e) dy[e] = empty ? 0.f : __uint_as_float(o[e]) * p.scale;
            } else {
#pragma unroll
                for (int e = 0; e < DC; ++e) dy[e] = 0.f;
            }
            float xv[DC];
            const size_t xrow = ((size_t(b) * p.S + i) * p.Hq + h) * D + col;
#pragma unroll
            for (int e8 = 0; e8 < DC / 8; ++e8) {
                const uint4 u = row_in ? *reinterpret_cast<const uint4*>(p.q_raw + xrow + 8 * e8) : make_uint4(0, 0, 0, 0);
                const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xv[8 * e8 + 2 * e] = bf16lo_to_f32(wv[e]);
                    xv[8 * e8 + 2 * e + 1] = bf16hi_to_f32(wv[e]);
                }
            }
            // the learned scales of this warpgroup's columns (every lane reads the same
            // addresses: broadcast accesses), four at a time
            const float* const scl = p.clip_scale ? p.clip_scale + size_t(h) * D + col : nullptr;
            auto sc4 = [&](int e4) {
                return scl ? *reinterpret_cast<const float4*>(scl + 4 * e4) : make_float4(1.f, 1.f, 1.f, 1.f);
            };
            float zz = 0.f, zd = 0.f;
#pragma unroll
            for (int e4 = 0; e4 < DC / 4; ++e4) {
                const float4 s = sc4(e4);
                const float sv4[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float z = xv[4 * e4 + u] * sv4[u];
                    zz = fmaf(z, z, zz);
                    zd = fmaf(z, dy[4 * e4 + u], zd);
                }
            }
            float2* const xrows = reinterpret_cast<float2*>(smem + L::XCH_OFF);
            float* const csum = reinterpret_cast<float*>(smem + L::XCH_OFF + 4 * NWG * 32 * 8);
            xrows[(wq * NWG + w) * 32 + lane] = make_float2(zz, zd);
            named_bar_sync(1 + wq, 32 * NWG);
            float zz_t = 0.f, zd_t = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < NWG; ++w2) {
                const float2 v = xrows[(wq * NWG + w2) * 32 + lane];
                zz_t += v.x;
                zd_t += v.y;
            }
            const float nrm = sqrtf(zz_t);
            const bool clipped = nrm > p.clip_thr;
            const float c = clipped ? p.clip_thr / nrm : 1.f;
            const float tau = (p.clip_tau && row_in) ? p.clip_tau[size_t(b) * p.S + i] : 1.f;
            const float k2 = clipped ? zd_t / zz_t : 0.f;
            if (ok_out && w == 0 && row_in) p.dtau_part[(size_t(b) * p.S + i) * p.Hq + h] = c * zd_t;
            // dz * x of this warp's rows, summed down the rows (a lane per column), then over
            // the four warps of the warpgroup
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            float* const stage = reinterpret_cast<float*>(smem + L::K_OFF) + (4 * w + wq) * 32 * STAGE_PITCH;
#pragma unroll
            for (int e4 = 0; e4 < DC / 4; ++e4) {  // dy becomes dx
                const float4 s = sc4(e4);
                const float sv4[4] = {s.x, s.y, s.z, s.w};
                float dzx[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = 4 * e4 + u;
                    const float dz = tau * c * (dy[e] - k2 * (xv[e] * sv4[u]));
                    dy[e] = dz * sv4[u];
                    dzx[u] = dz * xv[e];
                }
                *reinterpret_cast<float4*>(stage + lane * STAGE_PITCH + 4 * e4) = make_float4(dzx[0], dzx[1], dzx[2], dzx[3]);
            }
            __syncwarp();
            if (lane < DC) {
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                for (int rr = 0; rr < 32; rr += 4) {
                    a0 += stage[rr * STAGE_PITCH + lane];
                    a1 += stage[(rr + 1) * STAGE_PITCH + lane];
                    a2 += stage[(rr + 2) * STAGE_PITCH + lane];
                    a3 += stage[(rr + 3) * STAGE_PITCH + lane];
                }
                csum[(w * 4 + wq) * 32 + lane] = (a0 + a1) + (a2 + a3);
            }
            named_bar_sync(5 + w, 128);
            if (ok_out && wq == 0 && lane < DC) {
                const float a = (csum[(w * 4 + 0) * 32 + lane] + csum[(w * 4 + 1) * 32 + lane]) +
                                (csum[(w * 4 + 2) * 32 + lane] + csum[(w * 4 + 3) * 32 + lane]);
                p.dscale_part[((size_t(b) * num_qtiles + qt) * p.Hq + h) * D + col + lane] = a;
            }
            __syncwarp();
            // dx leaves through the same staging rows: each lane writes its row, then DC / 4
            // lanes store the row's DC contiguous floats
#pragma unroll
            for (int e = 0; e < DC; e += 4)
                *reinterpret_cast<float4*>(stage + lane * STAGE_PITCH + e) = make_float4(dy[e], dy[e + 1], dy[e + 2], dy[e + 3]);
            __syncwarp();
            constexpr int LPR = DC / 4;       // lanes per row
            constexpr int RPI = 32 / LPR;     // rows per store instruction
            const int sr = lane / LPR, sc = 4 * (lane % LPR);
            float* const base = p.dq + (b * p.row_sb + h * p.row_sh);
            if (ok_out) {
#pragma unroll
                for (int k = 0; k < 32 / RPI; ++k) {
                    const int rr = RPI * k + sr;        // row of this warp
                    const int ir = i0 + 32 * wq + rr;   // its query row
                    const float4 v = *reinterpret_cast<const float4*>(stage + rr * STAGE_PITCH + sc);
                    if (ir < p.S) *reinterpret_cast<float4*>(base + ir * p.row_ss + col + sc) = v;
                }
            }
        };

        // ---- epilogue: each warpgroup writes a quarter of the dQ columns ----
        if (ok && n_steps > 0) {
            ok = warp_wait(acc_full, 0, ctl, p.err, kErrDqAcc, p.timeout_ns);
            tc_fence_after();
        }
        if constexpr (CLIP) {
            clip_epilogue(ok);
        } else if (ok) {
            constexpr int DC = L::DC, STAGE_PITCH = L::STAGE_PITCH;  // dQ columns of this warpgroup
            const int col = w * DC;
            float* dst = p.dq + (b * p.row_sb + i * p.row_ss + h * p.row_sh);
            float* const base = p.dq + (b * p.row_sb + h * p.row_sh);
            if (n_steps > 0) {
                // the rows leave through shared memory (the K / V rings, idle once every MMA
                // has completed): each lane writes its row, then DC / 4 lanes store the row's
                // DC contiguous floats
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                float* const stage = reinterpret_cast<float*>(smem + L::K_OFF) + (4 * w + wq) * 32 * STAGE_PITCH;
                constexpr int LPR = DC / 4;       // lanes per row
                constexpr int RPI = 32 / LPR;     // rows per store instruction
                const int sr = lane / LPR, sc = 4 * (lane % LPR);
                uint32_t o[DC];
                if constexpr (DC == 32) {
                    tmem_ld32(tmem + lane_base + L::DQ_COL + col, o);
                } else {
                    tmem_ld16(tmem + lane_base + L::DQ_COL + col, o);
                }
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < DC / 4; ++q) {
                    float4 v;
                    v.x = empty ? 0.f : __uint_as_float(o[4 * q]) * p.scale;
                    v.y = empty ? 0.f : __uint_as_float(o[4 * q + 1]) * p.scale;
                    v.z = empty ? 0.f : __uint_as_float(o[4 * q + 2]) * p.scale;
                    v.w = empty ? 0.f : __uint_as_float(o[4 * q + 3]) * p.scale;
                    if (IRA_IN_BOUNDS(p.err, kErrBoundsDqSmem, smem_u32(stage + lane * STAGE_PITCH + 4 * q) - smem_base,
                                      16, L::TOTAL))
                        *reinterpret_cast<float4*>(stage + lane * STAGE_PITCH + 4 * q) = v;
                }
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 32 / RPI; ++k) {
                    const int rr = RPI * k + sr;        // row of this warp
                    const int ir = i0 + 32 * wq + rr;   // its query row
                    const bool st_ok = IRA_IN_BOUNDS(p.err, kErrBoundsDqSmem,
                                                     smem_u32(stage + rr * STAGE_PITCH + sc) - smem_base, 16, L::TOTAL);
                    const float4 v = st_ok ? *reinterpret_cast<const float4*>(stage + rr * STAGE_PITCH + sc)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
                    [[maybe_unused]] const long long at = b * p.row_sb + h * p.row_sh + (long long)ir * p.row_ss + col + sc;
                    if (ir < p.S && IRA_IN_BOUNDS(p.err, kErrBoundsDqGlobal, at, 4, n_rows * D))
                        *reinterpret_cast<float4*>(base + ir * p.row_ss + col + sc) = v;
                }
            } else if (row_in && IRA_IN_BOUNDS(p.err, kErrBoundsDqGlobal,
                                               b * p.row_sb + (long long)i * p.row_ss + h * p.row_sh + col, DC,
                                               n_rows * D)) {
                for (int e = col; e < col + DC; e += 4)
                    *reinterpret_cast<float4*>(dst + e) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }

    if (threadIdx.x == 0) IRA_TRACE_GRID(p, 2, 4);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
        if (lane == 0) IRA_TRACE_GRID(p, 2, 5);
    }
}

template <int D, bool CLIP>
cudaError_t launch(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                   const CUtensorMap& tm_do, const AttnParams& p, cudaStream_t st) {
    using L = Layout<D>;
    auto kern = dq_kernel<D, CLIP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    const int nqt = (p.S + BM - 1) / BM;
    const long long grid = (long long)nqt * p.B * p.Hq;
    if (grid == 0) return cudaSuccess;
    kern<<<dim3(unsigned(grid)), dim3(32 * L::NWARPS), L::ALLOC, st>>>(tm_q, tm_k, tm_v, tm_do, p, nqt);
    return cudaGetLastError();
}

}  // namespace dqk
}  // namespace bwdk

cudaError_t launch_bwd_dkdv(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                            const CUtensorMap& tm_do, const CUtensorMap& tm_band, const AttnParams& p,
                            cudaStream_t st) {
    return p.D == 128 ? bwdk::kv::launch<128>(tm_q, tm_k, tm_v, tm_do, tm_band, p, st)
                      : bwdk::kv::launch<64>(tm_q, tm_k, tm_v, tm_do, tm_band, p, st);
}

cudaError_t launch_bwd_dq(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const CUtensorMap& tm_do, const AttnParams& p, cudaStream_t st) {
    if (p.q_raw)
        return p.D == 128 ? bwdk::dqk::launch<128, true>(tm_q, tm_k, tm_v, tm_do, p, st)
                          : bwdk::dqk::launch<64, true>(tm_q, tm_k, tm_v, tm_do, p, st);
    return p.D == 128 ? bwdk::dqk::launch<128, false>(tm_q, tm_k, tm_v, tm_do, p, st)
                      : bwdk::dqk::launch<64, false>(tm_q, tm_k, tm_v, tm_do, p, st);
}

}  // namespace ira
