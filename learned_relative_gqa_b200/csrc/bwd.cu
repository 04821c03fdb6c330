// bwd.cu -- backward kernels of learned-relative grouped-query attention (sm_100a).
//
// The backward recomputes probabilities from the forward's log-sum-exp
// (P = exp(z - lse), sink included in lse) and applies the softmax chain rule
//   dP = dout . v,  dz = P (dP - Dv),  Dv = <dout, out> - dlse,
//   dq = scale sum_j dz k_j,  dk = scale sum_i dz q_i,  dv = sum_i P dout_i,
//   dprofiles[b,h,i,d] = dz for the allowed key at distance d < R.
// Dv, dsink, a BF16 copy of dout and lse*log2(e) come from the preprocessing
// kernel; dprofiles entries that no allowed key reaches are zeroed there too.
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
// In both, S/dP are double buffered in TMEM and the two elementwise warpgroups
// split the columns of every step (each owns half of them, with its own staged
// profile rows), so the MMAs of step n+1 run while step n is being processed.
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
constexpr int HALF = BQ / 2;         // query columns per elementwise warpgroup
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
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_band, const AttnParams p, const int num_ktiles) {
    using L = Layout<D>;
    constexpr int KB = L::KB;
    constexpr int TMA_WARP = 8, MMA_WARP = 9, BAND_WARP = 10, MMA_WARP_B = 11;
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

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        // stage, score and accumulator barriers complete once both MMA issuers committed
        for (int u = 0; u < NST; ++u) {
            mbar_init(&qd_full[u], 1);
            mbar_init(&qd_empty[u], 2);
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(&s_full[u], 2);
            mbar_init(&p_full[u], 8);
        }
        mbar_init(acc_full, 2);
        mbar_init(drain, 2);
        for (int u = 0; u < NB; ++u) {
            mbar_init(&band_full[u], 1);
            mbar_init(&band_empty[u], 8);  // every elementwise warp
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

    auto k_smem = [&](int kb) { return smem + L::K_OFF + kb * KTILE; };
    auto v_smem = [&](int kb) { return smem + L::V_OFF + kb * KTILE; };
    auto q_smem = [&](int st, int kb) { return smem + L::Q_OFF + (st * KB + kb) * QTILE; };
    auto do_smem = [&](int st, int kb) { return smem + L::DO_OFF + (st * KB + kb) * QTILE; };
    auto step_h = [&](int n) { return g * G + n / n_qt; };
    auto step_qt = [&](int n) { return qt_first + n % n_qt; };

    // Launched with 384 x 168 registers; warpgroup 2 (tile producer, two MMA issuers,
    // band producer) gives part of its share to the two elementwise warpgroups
    // (128 x 72 + 256 x 208 <= 384 x 168). Each change sits at the top of its branch.
    // A step whose smallest distance delta - 127 is >= R has no profile entry.
    auto band_used = [&](int n) { return p.R > 0 && p.q_off + step_qt(n) * BQ - j0 - (BK - 1) < p.R; };
    if (warp >= 8) {
        setmaxnreg_dec<72>();
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
            mbar_wait_drain(kv_full, 0, p.timeout_ns);
            for (int n = (last >= NST ? last - NST + 1 : 0); n <= last; ++n)
                mbar_wait_drain(&qd_full[n % NST], (n / NST) & 1, p.timeout_ns);
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
                if (n < n_steps) {
                    const TileBounds tb = p.tile_bounds[size_t(b) * t64 + step_qt(n)];
                    full_r = tb.n_nonempty == BQ && tb.max_lo <= j0 && tb.min_hi >= j0 + BK - 1;
                }
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    rb_r[k] = make_int2(kEmptyLo, kEmptyHi);
                    l2_r[k] = 0.f;
                    dv_r[k] = 0.f;
                    const int i = step_qt(n) * BQ + lane + 32 * k;
                    if (n < n_steps && i < p.S) {
                        rb_r[k] = p.row_bounds[size_t(b) * p.S + i];
                        const size_t t = (size_t(b) * p.Hq + step_h(n)) * p.S + i;
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
                            tma_load_2d(band + g8 * 8 * BAND_PITCH, &tm_band, &band_full[buf], x0 + 8 * g8, row0 + 8 * g8);
                    }
                    IRA_TRACE(p, 34, n);
                }
                last = n;
            }
            // never leave a copy in flight into shared memory of an exiting CTA
            if (lane == 0)
                for (int n = (last >= NB ? last - NB + 1 : 0); n <= last; ++n)
                    mbar_wait_drain(&band_full[n % NB], (n / NB) & 1, p.timeout_ns);
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
                // P^T / dS^T of query columns [32 w, 32 w + 32) sit, packed, at the
                // start of warpgroup w's own S / dP columns
                const uint32_t cs = c_base(st);
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk) {
                    const uint32_t a_off = HALF * (kk >> 1) + 8 * (kk & 1);
                    mma_ts(tmem + prod_col, tmem + col_of(bb) + a_off, sdesc_sw128(cs + kk * 2048, QTILE, 1024),
                           IDESC_ACC, (n > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&qd_empty[st]);
                if (!is_b) IRA_TRACE(p, 24, n);
            }
            if (ok) mma_commit(acc_full);
            mma_commit(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
        }
    }
    } else {
        setmaxnreg_inc<208>();
        // ------------------------------------------------------------ elementwise warpgroups
        const int w = warp >> 2;       // this warpgroup takes query columns [32 w, 32 w + 32) of every step
        const int wq = warp & 3;
        const int r = wq * 32 + lane;  // key row (TMEM lane)
        const int j = j0 + r;
        const uint32_t lane_base = uint32_t(wq * 32) << 16;
        const int tid = threadIdx.x & 127;
        const int cw = HALF * w;       // first query column of this warpgroup

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
            if (tid == 0) IRA_TRACE(p, 25 + 3 * w, n);
            tc_fence_after();
            uint32_t sv[HALF], dp[HALF];
            tmem_ld32(tmem + lane_base + L::s_col(bb) + cw, sv);
            tmem_ld32(tmem + lane_base + L::dp_col(bb) + cw, dp);

            // Band reads. Column c = cw + cl reads element (m + 127 - r) of shared band row
            // dm + c, where m = (dm + c) mod 8 repeats every 8 columns (cw is a multiple
            // of 8): eight per-step shared addresses plus compile-time offsets cover them all.
            const int dm = (delta - 127) & 7;
            const uint32_t band_s = smem_u32(smem + L::BAND_OFF + buf * BAND_BYTES + (dm + cw) * BAND_PITCH);
            uint32_t baddr[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) baddr[u] = band_s + u * BAND_PITCH + 2 * (((dm + u) & 7) + 127 - r);
            const uint32_t info_s = smem_u32(smem + L::INFO_OFF + buf * int(sizeof(StepInfo)));
            const bool full = lds_s32(info_s + offsetof(StepInfo, full)) != 0;
            // dprofiles[b, h, i0 + c, delta + c - r] for column c = cw + cl: the address of
            // column cl is dbase + cl (R + 1) floats
            char* const dbase = reinterpret_cast<char*>(
                p.dprofiles + ((size_t(b) * p.Hq + h) * p.S + i0 + cw) * size_t(p.R) + (delta + cw - r));
            const uint32_t dstride4 = 4u * uint32_t(p.R + 1);
            // d = delta + c - r < R  <=>  c < R - delta + r (no limit when the whole step is inside R)
            const bool inside = delta + BQ - 1 < p.R;
            const int cl_lim = (inside ? BQ : p.R - delta + r) - cw;
            tmem_wait_ld();
            if (tid == 0) IRA_TRACE(p, 31, n);
            uint32_t pk[HALF / 2], dk[HALF / 2];
            // USED: the step reads profile entries; PLAIN: every (key, query) pair of the
            // step is allowed and inside R, so there is no mask and no store predicate
            auto math = [&](auto used_c, auto plain_c) {
                constexpr bool USED = decltype(used_c)::value, PLAIN = decltype(plain_c)::value;
#pragma unroll
                for (int c16 = 0; c16 < HALF / 16; ++c16) {
                    // loads of this 16-column chunk, issued together
                    float nl_c[16], nv_c[16], bias_c[16];
                    int lo_c[16], hi_c[16];
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4) {  // 128-bit broadcast reads of four columns
                        const int c = cw + 16 * c16 + 4 * u4;
                        const float4 l4 = lds_f32x4(info_s + offsetof(StepInfo, nlse2) + 4 * c);
                        const float4 v4 = lds_f32x4(info_s + offsetof(StepInfo, ndv) + 4 * c);
                        nl_c[4 * u4 + 0] = l4.x; nl_c[4 * u4 + 1] = l4.y; nl_c[4 * u4 + 2] = l4.z; nl_c[4 * u4 + 3] = l4.w;
                        nv_c[4 * u4 + 0] = v4.x; nv_c[4 * u4 + 1] = v4.y; nv_c[4 * u4 + 2] = v4.z; nv_c[4 * u4 + 3] = v4.w;
                        if (!PLAIN) {
                            const int4 a4 = lds_s32x4(info_s + offsetof(StepInfo, rb) + 8 * c);
                            const int4 b4 = lds_s32x4(info_s + offsetof(StepInfo, rb) + 8 * c + 16);
                            lo_c[4 * u4 + 0] = a4.x; hi_c[4 * u4 + 0] = a4.y; lo_c[4 * u4 + 1] = a4.z; hi_c[4 * u4 + 1] = a4.w;
                            lo_c[4 * u4 + 2] = b4.x; hi_c[4 * u4 + 2] = b4.y; lo_c[4 * u4 + 3] = b4.z; hi_c[4 * u4 + 3] = b4.w;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int cl = 16 * c16 + u;
                        bias_c[u] = USED ? __uint_as_float(lds_u16(baddr[cl & 7] + BAND_PITCH * 8 * (cl >> 3)) << 16) : 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < 16; u += 2) {
                        const int cl = 16 * c16 + u;
                        // log2-domain logit, probability, dS = P (dP - Dv), two columns at a time
                        float2 z = __ffma2_rn(make_float2(__uint_as_float(sv[cl]), __uint_as_float(sv[cl + 1])), sl2,
                                              make_float2(nl_c[u], nl_c[u + 1]));
                        if (USED) z = __ffma2_rn(make_float2(bias_c[u], bias_c[u + 1]), l2e, z);
                        float2 pr = make_float2(ex2_approx(z.x), ex2_approx(z.y));
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
                        if (PLAIN || ok0) __stcs(a0, ds.x);
                        if (PLAIN || ok1) __stcs(a1, ds.y);
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
            if (tid == 0) IRA_TRACE(p, 32, n);
            tmem_st16(tmem + lane_base + L::s_col(bb) + cw, pk);
            tmem_st16(tmem + lane_base + L::dp_col(bb) + cw, dk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&p_full[bb]);
                mbar_arrive(&band_empty[buf]);
            }
            if (tid == 0) IRA_TRACE(p, 26 + 3 * w, n);
        }

        // ---- epilogue: warpgroup 0 writes dK (scaled), warpgroup 1 writes dV ----
        if (ok && n_steps > 0) {
            ok = warp_wait(acc_full, 0, ctl, p.err, kErrDkdvAcc, p.timeout_ns);
            tc_fence_after();
        }
        if (ok) {
            const bool row_in = j < p.Skv;
            float* dst = (w == 0 ? p.dk : p.dv) + (b * p.kv_sb + j * p.kv_ss + g * p.kv_sh);
            float* const base = (w == 0 ? p.dk : p.dv) + (b * p.kv_sb + g * p.kv_sh);
            const float mul = (w == 0) ? p.scale : 1.f;
            const uint32_t col = (w == 0) ? L::DK_COL : L::DV_COL;
            if (n_steps > 0) {
                // 32 x 32 chunks go out through shared memory (the key / query tiles, idle once
                // every MMA has completed), 144-byte pitch per row: each lane writes its row,
                // then 8 lanes store 128 contiguous bytes of one row, four rows per store
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                float* const stage = reinterpret_cast<float*>(smem + L::K_OFF) + (4 * w + wq) * 32 * 36;
                const int sr = lane >> 3, sc = 4 * (lane & 7);
#pragma unroll 1
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + col + 32 * c4, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4*>(stage + lane * 36 + 4 * q) =
                            make_float4(__uint_as_float(o[4 * q]) * mul, __uint_as_float(o[4 * q + 1]) * mul,
                                        __uint_as_float(o[4 * q + 2]) * mul, __uint_as_float(o[4 * q + 3]) * mul);
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int rr = 4 * k + sr;          // row of this warp
                        const int jr = j0 + 32 * wq + rr;   // its key
                        const float4 v = *reinterpret_cast<const float4*>(stage + rr * 36 + sc);
                        if (jr < p.Skv) *reinterpret_cast<float4*>(base + jr * p.kv_ss + 32 * c4 + sc) = v;
                    }
                    __syncwarp();
                }
            } else if (row_in) {
                for (int e = 0; e < D; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
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
    kern<<<dim3(unsigned(grid)), dim3(384), L::ALLOC, st>>>(tm_q, tm_k, tm_v, tm_do, tm_band, p, nkt);
    return cudaGetLastError();
}

}  // namespace kv

// =====================================================================================
// dQ
// =====================================================================================
namespace dqk {

constexpr int BM = 128;               // query rows per CTA (TMEM lanes)
constexpr int BN = 64;                // keys per step
constexpr int HALF = BN / 2;          // key columns per elementwise warpgroup
constexpr int BAND_CHUNKS = 5;        // 40 bf16 per row window (32 columns + misalignment)
constexpr int BAND_UNITS = BAND_CHUNKS * BM + 2 * (BM / 8);
constexpr int BAND_BYTES = BAND_UNITS * 16;
constexpr int QTILE = BM * 128;       // [128 x 64 bf16]
constexpr int KTILE = BN * 128;       // [64 x 64 bf16]
constexpr int NSB = 3;                // S / dP buffers in TMEM: the MMAs run two steps ahead
constexpr int NSK = 4;                // K stages: K(n) is read by S(n) and, two steps later, by dQ(n)
constexpr int NSV = 2;                // V stages: V(n) is read by dP(n) only

__host__ __device__ constexpr int band_unit(int r) { return BAND_CHUNKS * r + 2 * (r >> 3); }

template <int D>
struct Layout {
    static constexpr int KB = D / 64;
    static constexpr int Q_OFF = 0;
    static constexpr int DO_OFF = Q_OFF + KB * QTILE;
    static constexpr int K_OFF = DO_OFF + KB * QTILE;          // NSK stages
    static constexpr int V_OFF = K_OFF + NSK * KB * KTILE;     // NSV stages
    static constexpr int BAND_OFF = V_OFF + NSV * KB * KTILE;  // [warpgroup][step parity]
    static constexpr int BAR_OFF = BAND_OFF + 4 * BAND_BYTES;
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
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const AttnParams p, const int num_qtiles) {
    using L = Layout<D>;
    constexpr int KB = L::KB;
    constexpr int TMA_WARP = 8, MMA_WARP = 9, V_WARP = 10, MMA_WARP_B = 11;
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

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        // a K / V stage is free, and S / dP of a step ready, once both MMA issuers committed
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
            mbar_init(&s_full[u], 2);
            mbar_init(&p_full[u], 8);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 2);
        ctl->abort = 0;
        const TileBounds* tb = p.tile_bounds + size_t(b) * t64 + 2 * qt;
        int min_lo = tb[0].min_lo, max_hi = tb[0].max_hi, ne = tb[0].n_nonempty;
        if (2 * qt + 1 < t64) {
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

    auto q_smem = [&](int kb) { return smem + L::Q_OFF + kb * QTILE; };
    auto do_smem = [&](int kb) { return smem + L::DO_OFF + kb * QTILE; };
    auto k_smem = [&](int n, int kb) { return smem + L::K_OFF + ((n % NSK) * KB + kb) * KTILE; };
    auto v_smem = [&](int n, int kb) { return smem + L::V_OFF + ((n % NSV) * KB + kb) * KTILE; };
    auto key0 = [&](int n) { return i0g + BN - (t_begin + n) * BN; };

    // Launched with 384 x 168 registers; warpgroup 2 (producer, two MMA issuers, an idle
    // warp) gives part of its share to the two elementwise warpgroups
    // (128 x 80 + 256 x 208 <= 384 x 168). Each change sits at the top of its branch.
    if (warp >= 8) {
        setmaxnreg_dec<80>();
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
                if (!is_v) IRA_TRACE(p, 41, n);
                last = n;
            }
            if (!is_v) mbar_wait_drain(q_full, 0, p.timeout_ns);
            for (int n = (last >= ns ? last - ns + 1 : 0); n <= last; ++n)
                mbar_wait_drain(&full[n % ns], (n / ns) & 1, p.timeout_ns);
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
                if (!is_b) IRA_TRACE(p, 42, n);
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
                    // dS of key columns [32 w, 32 w + 32) sits, packed, at the start of
                    // warpgroup w's own dP columns
                    mma_ts(tmem + L::DQ_COL, tmem + L::dp_col(bb) + HALF * (kk >> 1) + 8 * (kk & 1),
                           sdesc_sw128(ks + kk * 2048, KTILE, 1024), IDESC_DQ, (n > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&k_empty[n % NSK]);
                IRA_TRACE(p, 44, n);
            }
            if (ok && is_b) mma_commit(acc_full);
            mma_commit(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
        }
    }
    } else {
        setmaxnreg_inc<208>();
        const int w = warp >> 2;       // this warpgroup takes key columns [32 w, 32 w + 32) of every step
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_base = uint32_t(wq * 32) << 16;
        const int cw = HALF * w;
        const int i = i0 + r;
        const bool row_in = i < p.S;
        const int2 rb = row_in ? p.row_bounds[size_t(b) * p.S + i] : make_int2(kEmptyLo, kEmptyHi);
        const bool empty = rb.x > rb.y;
        const size_t trow = (size_t(b) * p.Hq + h) * p.S + i;
        const float lse2 = row_in ? p.lse2t[trow] : 0.f;
        const float dvr = row_in ? p.dvt[trow] : 0.f;

        // This thread's profile window for its columns, double buffered by step parity:
        // column c = cw + cl of step n has distance delta(n) + r - c; the 32 columns'
        // window starts (r + 1) mod 8 elements past a 16-byte boundary.
        const int unit = band_unit(r);
        auto band_saddr = [&](int buf) {
            return smem_u32(smem + L::BAND_OFF + (2 * w + buf) * BAND_BYTES) + uint32_t(unit) * 16u;
        };
        const int m_r = (r + 1) & 7;
        const int g_r = m_r >> 1;
        const uint32_t fshift = uint32_t(m_r & 1) * 16u;
        const uint16_t* prof_row =
            (p.R > 0 && row_in && !empty) ? p.profiles + ((size_t(b) * p.Hq + h) * p.S + i) * size_t(p.R) : nullptr;
        // step n has distance offset delta = i0g - key0(n) = 64 (t_begin + n) - 64
        auto delta_of = [&](int n) { return BN * (t_begin + n) - BN; };
        // the warp's smallest distance in this warpgroup's columns is delta + 32 wq - cw - 31
        auto band_needed = [&](int n) { return delta_of(n) + wq * 32 - cw - (HALF - 1) < p.R; };
        // one cp.async group per call, also when nothing is copied
        auto issue_band = [&](int n) {
            if (n < n_steps && band_needed(n)) {
                const int x0 = delta_of(n) + r - cw - (HALF - 1) - m_r;
                const uint32_t dst = band_saddr(n & 1);
#pragma unroll
                for (int q = 0; q < BAND_CHUNKS; ++q) {
                    const int d0 = x0 + 8 * q;
                    const bool inb = prof_row != nullptr && d0 >= 0 && d0 < p.R;
                    const void* src = inb ? static_cast<const void*>(prof_row + d0) : p.safe_src;
                    cp_async_16(dst + 16u * q, src, inb ? 16u : 0u);
                }
            }
            cp_async_commit();
        };

        issue_band(0);
        issue_band(1);
        bool ok = true;
        const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 l2e = make_float2(kLog2e, kLog2e);
        const float2 nl2 = make_float2(-lse2, -lse2);
        const float2 nv2 = make_float2(-dvr, -dvr);
        for (int n = 0; n < n_steps; ++n) {
            const int bb = n % NSB;
            const int jk = key0(n) + cw;  // key of this warpgroup's first column
            const bool my_full = empty || (rb.x <= jk && rb.y >= jk + HALF - 1);
            const bool need_mask = !__all_sync(0xffffffffu, my_full);
            const bool use_band = band_needed(n);
            if (!warp_wait(&s_full[bb], (n / NSB) & 1, ctl, p.err, kErrDqS, p.timeout_ns)) {
                ok = false;
                break;
            }
            if (wq == 0 && lane == 0) IRA_TRACE(p, 45 + 2 * w, n);
            tc_fence_after();
            uint32_t sv[HALF], dp[HALF];
            tmem_ld32(tmem + lane_base + L::s_col(bb) + cw, sv);
            tmem_ld32(tmem + lane_base + L::dp_col(bb) + cw, dp);
            uint32_t wv[17];
            if (use_band) {
                cp_async_wait_group<1>();  // this step's window (the next step's may fly)
                const uint32_t* words =
                    reinterpret_cast<const uint32_t*>(smem + L::BAND_OFF + (2 * w + (n & 1)) * BAND_BYTES + unit * 16) + g_r;
#pragma unroll
                for (int q = 0; q < 17; ++q) wv[q] = words[q];
            }
            // this step's window is in registers: fetch the one of step n + 2 into its buffer
            issue_band(n + 2);
            tmem_wait_ld();
            const int c_lo = rb.x - jk, c_hi = rb.y - jk;  // allowed columns of this row
            uint32_t dk[HALF / 2];
#pragma unroll
            for (int pp = 0; pp < HALF / 2; ++pp) {
                const int c = 2 * pp;
                float2 t = nl2;
                if (use_band) {
                    const uint32_t v = funnel_r(wv[15 - pp], wv[16 - pp], fshift);
                    t = __ffma2_rn(make_float2(bf16hi_to_f32(v), bf16lo_to_f32(v)), l2e, nl2);
                }
                const float2 z = __ffma2_rn(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2, t);
                float2 pr = make_float2(ex2_approx(z.x), ex2_approx(z.y));
                if (need_mask) {
                    pr.x = (c >= c_lo && c <= c_hi) ? pr.x : 0.f;
                    pr.y = (c + 1 >= c_lo && c + 1 <= c_hi) ? pr.y : 0.f;
                }
                const float2 ds =
                    __fmul2_rn(pr, __fadd2_rn(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), nv2));
                dk[pp] = pack_bf16x2(ds.x, ds.y);
            }
            tmem_st16(tmem + lane_base + L::dp_col(bb) + cw, dk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[bb]);
            if (wq == 0 && lane == 0) IRA_TRACE(p, 46 + 2 * w, n);
        }
        cp_async_wait_all();

        // ---- epilogue: each warpgroup writes half of the dQ columns ----
        if (ok && n_steps > 0) {
            ok = warp_wait(acc_full, 0, ctl, p.err, kErrDqAcc, p.timeout_ns);
            tc_fence_after();
        }
        if (ok) {
            float* dst = p.dq + (b * p.row_sb + i * p.row_ss + h * p.row_sh);
            float* const base = p.dq + (b * p.row_sb + h * p.row_sh);
            constexpr int HALF = D / 2;
            if (n_steps > 0) {
                // 32 x 32 chunks go out through shared memory (the K / V rings, idle once every
                // MMA has completed), 144-byte pitch per row: each lane writes its row, then
                // 8 lanes store 128 contiguous bytes of one row, four rows per store
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                float* const stage = reinterpret_cast<float*>(smem + L::K_OFF) + (4 * w + wq) * 32 * 36;
                const int sr = lane >> 3, sc = 4 * (lane & 7);
#pragma unroll 1
                for (int c4 = 0; c4 < HALF / 32; ++c4) {
                    const int col = w * HALF + 32 * c4;
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + L::DQ_COL + col, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 v;
                        v.x = empty ? 0.f : __uint_as_float(o[4 * q]) * p.scale;
                        v.y = empty ? 0.f : __uint_as_float(o[4 * q + 1]) * p.scale;
                        v.z = empty ? 0.f : __uint_as_float(o[4 * q + 2]) * p.scale;
                        v.w = empty ? 0.f : __uint_as_float(o[4 * q + 3]) * p.scale;
                        *reinterpret_cast<float4*>(stage + lane * 36 + 4 * q) = v;
                    }
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int rr = 4 * k + sr;          // row of this warp
                        const int ir = i0 + 32 * wq + rr;   // its query row
                        const float4 v = *reinterpret_cast<const float4*>(stage + rr * 36 + sc);
                        if (ir < p.S) *reinterpret_cast<float4*>(base + ir * p.row_ss + col + sc) = v;
                    }
                    __syncwarp();
                }
            } else if (row_in) {
                for (int e = w * HALF; e < (w + 1) * HALF; e += 4)
                    *reinterpret_cast<float4*>(dst + e) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

template <int D>
cudaError_t launch(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                   const CUtensorMap& tm_do, const AttnParams& p, cudaStream_t st) {
    using L = Layout<D>;
    auto kern = dq_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    const int nqt = (p.S + BM - 1) / BM;
    const long long grid = (long long)nqt * p.B * p.Hq;
    if (grid == 0) return cudaSuccess;
    kern<<<dim3(unsigned(grid)), dim3(384), L::ALLOC, st>>>(tm_q, tm_k, tm_v, tm_do, p, nqt);
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
    return p.D == 128 ? bwdk::dqk::launch<128>(tm_q, tm_k, tm_v, tm_do, p, st)
                      : bwdk::dqk::launch<64>(tm_q, tm_k, tm_v, tm_do, p, st);
}

}  // namespace ira
