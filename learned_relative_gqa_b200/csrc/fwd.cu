// fwd.cu -- forward kernel of learned-relative grouped-query attention (sm_100a).
//
// One CTA handles one 128-row query tile of NH query heads (NH = 2 heads of the
// same KV group when the group size is even, else 1). The K/V tile of each
// step is loaded once by TMA and shared by both heads; the two heads ping-pong
// on the tensor core while the other head's softmax runs:
//
//   warps 0..4*NH-1   softmax, one warpgroup per head (thread = query row =
//                     TMEM lane); also stage the head's profile band
//   warp  4*NH        TMA producer: Q (once), K and V tiles
//   warp  4*NH+1      MMA issuer (one thread): S = Q K^T (SMEM x SMEM -> TMEM),
//                     O += P V (P from TMEM x V from SMEM -> TMEM)
//
// Per KV step the softmax warpgroup reads S from TMEM, adds the learned
// relative logit profiles[b,h,i,d] (d = i_g - j; distances >= R read zeros),
// masks the step's boundary tiles, keeps a lazily rescaled running maximum
// initialised with the sink logit (running sum initialised with exp(0) = 1, so
// the sink enters the denominator with no value row), writes P as BF16 into
// the S columns of TMEM and, when its maximum moved, rescales O in TMEM.
//
// Key tiles are aligned to the query tile: step t covers keys
// [i_g0 - 128 t, i_g0 - 128 t + 127], so the distance offset of the step is
// delta = 128 t and row r needs the profile distances [delta + r - 127,
// delta + r]. Each softmax thread copies exactly that window of its own
// profile row (17 x 16 B, cp.async with zero fill outside [0, R)) into a band
// buffer laid out so that the per-column 32-bit gathers of a warp hit 32
// distinct shared-memory banks: row r starts at 16-byte unit 17 r + 2 (r / 8).
//
// Operation and argument conventions follow the NeMo AutoModel page for
// Inkling2FlexAttention.forward; see include/inkling_rel_attn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace ira {
namespace fwdk {

constexpr int BM = 128;               // query rows per tile (TMEM lanes)
constexpr int BN = 128;               // keys per step
constexpr int BAND_CHUNKS = 17;       // 16-byte chunks per band row (136 bf16)
constexpr int BAND_UNITS = BAND_CHUNKS * BM + 2 * (BM / 8);
constexpr int BAND_BYTES = BAND_UNITS * 16;
constexpr int TILE_BYTES = BM * 128;  // one [128 rows x 64 bf16] 128B-swizzled box

__host__ __device__ constexpr int band_unit(int r) { return BAND_CHUNKS * r + 2 * (r >> 3); }

template <int D, int NH>
struct Layout {
    static constexpr int KB = D / 64;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + NH * KB * TILE_BYTES;
    static constexpr int V_OFF = K_OFF + KB * TILE_BYTES;
    static constexpr int BAND_OFF = V_OFF + KB * TILE_BYTES;
    static constexpr int BAR_OFF = BAND_OFF + NH * BAND_BYTES;
    // q_full, k_full, k_empty, v_full, v_empty, drain, s_full[NH], p_full[NH], o_full[NH]
    static constexpr int NBARS = 6 + 3 * NH;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int TOTAL = MISC_OFF + 64;
    static constexpr int ALLOC = TOTAL + 1024;
    // NH = 2: three full warpgroups (softmax A, softmax B, producer + MMA + 2
    // idle warps) so that registers can be moved between warpgroups.
    static constexpr int NWARPS = (NH == 2) ? 12 : 6;
    static constexpr uint32_t TMEM_COLS = (NH * (128 + D) <= 256) ? 256u : 512u;
    static constexpr uint32_t s_col(int s) { return uint32_t(s * 128); }
    static constexpr uint32_t o_col(int s) { return uint32_t(NH * 128 + s * D); }
};

__device__ __forceinline__ int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }
__device__ __forceinline__ int ceil_div_i(int a, int b) { return -floor_div(-a, b); }

template <int D, int NH>
__global__ void __launch_bounds__(32 * ((NH == 2) ? 12 : 6), 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const AttnParams p, const int num_qtiles) {
    using L = Layout<D, NH>;
    constexpr int KB = L::KB;
    constexpr int TMA_WARP = 4 * NH, MMA_WARP = 4 * NH + 1;

    extern __shared__ uint8_t smem_raw[];
    // aligned by pointer arithmetic on the __shared__ array, so the compiler keeps
    // knowing that every pointer derived from it addresses shared memory
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = bars + 2;
    uint64_t* v_full = bars + 3;
    uint64_t* v_empty = bars + 4;
    uint64_t* drain = bars + 5;
    uint64_t* s_full = bars + 6;
    uint64_t* p_full = bars + 6 + NH;
    uint64_t* o_full = bars + 6 + 2 * NH;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    CtaControl* ctl = reinterpret_cast<CtaControl*>(smem + L::MISC_OFF + 16);
    int* tinfo = reinterpret_cast<int*>(smem + L::MISC_OFF + 32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- work item: longest query tiles are scheduled first ----
    const int pairs = p.Hq / NH;
    const int per_tile = p.B * pairs;
    const int qt = num_qtiles - 1 - int(blockIdx.x) / per_tile;
    const int rem = int(blockIdx.x) % per_tile;
    const int b = rem / pairs;
    const int h0 = (rem % pairs) * NH;
    const int g = h0 / (p.Hq / p.Hkv);
    const int i0 = qt * BM;
    const int i0g = p.q_off + i0;
    const int t64 = (p.S + 63) / 64;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(k_full, 1);
        mbar_init(k_empty, 1);
        mbar_init(v_full, 1);
        mbar_init(v_empty, 1);
        mbar_init(drain, 1);
        for (int s = 0; s < NH; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
            mbar_init(&o_full[s], 1);
        }
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
            t_begin = max(0, ceil_div_i(i0g - max_hi, BN));
            const int t_end = floor_div(i0g + BM - 1 - min_lo, BN);
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

    auto q_smem = [&](int s, int kb) { return smem + L::Q_OFF + (s * KB + kb) * TILE_BYTES; };
    auto k_smem = [&](int kb) { return smem + L::K_OFF + kb * TILE_BYTES; };
    auto v_smem = [&](int kb) { return smem + L::V_OFF + kb * TILE_BYTES; };

    // With NH = 2 the kernel is launched with 384 x 168 registers and the producer
    // warpgroup gives its share to the two softmax warpgroups (128 x 40 + 256 x 232
    // = 384 x 168). Each budget change sits at the top of its role's branch.
    if (warp >= 4 * NH) {
        if constexpr (NH == 2) setmaxnreg_dec<40>();
    if (warp == TMA_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && n_steps > 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            mbar_arrive_expect_tx(q_full, NH * KB * TILE_BYTES);
            for (int s = 0; s < NH; ++s)
                for (int kb = 0; kb < KB; ++kb) tma_load_4d(q_smem(s, kb), &tm_q, q_full, kb * 64, h0 + s, i0, b);
            int nk = -1, nv = -1;
            for (int n = 0; n < n_steps; ++n) {
                const int j0 = i0g - (t_begin + n) * BN;
                if (!mbar_wait(k_empty, (n & 1) ^ 1, ctl, p.err, kErrFwdKFree, p.timeout_ns)) break;
                mbar_arrive_expect_tx(k_full, KB * TILE_BYTES);
                for (int kb = 0; kb < KB; ++kb) tma_load_4d(k_smem(kb), &tm_k, k_full, kb * 64, g, j0, b);
                IRA_TRACE(p, 1, n);
                nk = n;
                if (!mbar_wait(v_empty, (n & 1) ^ 1, ctl, p.err, kErrFwdVFree, p.timeout_ns)) break;
                mbar_arrive_expect_tx(v_full, KB * TILE_BYTES);
                for (int kb = 0; kb < KB; ++kb) tma_load_4d(v_smem(kb), &tm_v, v_full, kb * 64, g, j0, b);
                IRA_TRACE(p, 2, n);
                nv = n;
            }
            // never leave a copy in flight into shared memory of an exiting CTA
            mbar_wait_drain(q_full, 0, p.timeout_ns);
            if (nk >= 0) mbar_wait_drain(k_full, nk & 1, p.timeout_ns);
            if (nv >= 0) mbar_wait_drain(v_full, nv & 1, p.timeout_ns);
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_steps > 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, 0, 0);
            constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);
            auto issue_s = [&](int s) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int kb = kk >> 2, kin = kk & 3;
                    const uint64_t ad = sdesc_sw128(smem_u32(q_smem(s, kb)) + kin * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(smem_u32(k_smem(kb)) + kin * 32, 16, 1024);
                    mma_ss(tmem + L::s_col(s), ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_o = [&](int s, bool acc) {
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bd = sdesc_sw128(smem_u32(v_smem(0)) + kk * 2048, TILE_BYTES, 1024);
                    mma_ts(tmem + L::o_col(s), tmem + L::s_col(s) + kk * 8, bd, IDESC_O,
                           (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(q_full, 0, ctl, p.err, kErrFwdQ, p.timeout_ns) &&
                      mbar_wait(k_full, 0, ctl, p.err, kErrFwdK, p.timeout_ns);
            if (ok) {
                IRA_TRACE(p, 9, 0);
                tc_fence_after();
                for (int s = 0; s < NH; ++s) {
                    issue_s(s);
                    mma_commit(&s_full[s]);
                    IRA_TRACE(p, 3 + s, 0);
                }
                mma_commit(k_empty);
            }
            for (int n = 0; ok && n < n_steps; ++n) {
                ok = mbar_wait(v_full, n & 1, ctl, p.err, kErrFwdV, p.timeout_ns);
                IRA_TRACE(p, 10, n);
                for (int s = 0; ok && s < NH; ++s) {
                    ok = mbar_wait(&p_full[s], n & 1, ctl, p.err, kErrFwdP, p.timeout_ns);
                    if (!ok) break;
                    IRA_TRACE(p, 7 + s, n);
                    tc_fence_after();
                    issue_o(s, n > 0);
                    IRA_TRACE(p, 5 + s, n);
                    if (s == NH - 1) mma_commit(v_empty);
                    if (n + 1 < n_steps) {
                        if (s == 0) {
                            ok = mbar_wait(k_full, (n + 1) & 1, ctl, p.err, kErrFwdK, p.timeout_ns);
                            if (!ok) break;
                            IRA_TRACE(p, 9, n + 1);
                            tc_fence_after();
                        }
                        issue_s(s);
                        mma_commit(&s_full[s]);
                        IRA_TRACE(p, 3 + s, n + 1);
                        if (s == NH - 1) mma_commit(k_empty);
                    }
                }
            }
            if (ok)
                for (int s = 0; s < NH; ++s) mma_commit(&o_full[s]);
            // wait for every issued MMA before TMEM is released
            mma_commit(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
        }
    }
    } else {
        if constexpr (NH == 2) setmaxnreg_inc<232>();
        // ------------------------------------------------------------ softmax
        const int s = warp >> 2;
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_base = uint32_t(wq * 32) << 16;
        const int h = h0 + s;
        const int i = i0 + r;
        const bool row_in = i < p.S;
        const int2 rb = row_in ? p.row_bounds[size_t(b) * p.S + i] : make_int2(kEmptyLo, kEmptyHi);
        const bool empty = rb.x > rb.y;
        const float sigma = row_in ? p.sink[(size_t(b) * p.S + i) * p.Hq + h] : 0.f;
        float m2 = sigma * kLog2e;  // lazily rescaled running maximum, log2 units
        float l = 1.f;              // running denominator; the sink contributes exp(0)

        uint8_t* band = smem + L::BAND_OFF + s * BAND_BYTES;
        const int unit = band_unit(r);
        const uint32_t band_saddr = smem_u32(band) + uint32_t(unit) * 16u;
        const uint32_t* band_words = reinterpret_cast<const uint32_t*>(band + unit * 16);
        const int m_r = (r + 1) & 7;   // misalignment of the row's window start (delta % 8 == 0)
        const int g_r = m_r >> 1;
        const uint32_t fshift = uint32_t(m_r & 1) * 16u;
        const uint16_t* prof_row =
            (p.R > 0 && row_in && !empty) ? p.profiles + ((size_t(b) * p.Hq + h) * p.S + i) * size_t(p.R) : nullptr;

        auto band_needed = [&](int n) { return (t_begin + n) * BN + wq * 32 - 127 < p.R; };
        auto issue_band = [&](int n) {
            const int x0 = (t_begin + n) * BN + r - 127 - m_r;
#pragma unroll
            for (int q = 0; q < BAND_CHUNKS; ++q) {
                const int d0 = x0 + 8 * q;
                const bool inb = prof_row != nullptr && d0 >= 0 && d0 < p.R;
                const void* src = inb ? static_cast<const void*>(prof_row + d0) : p.safe_src;
                cp_async_16(band_saddr + 16u * q, src, inb ? 16u : 0u);
            }
            cp_async_commit();
        };

        if (n_steps > 0 && band_needed(0)) issue_band(0);
        bool ok = true;
        for (int n = 0; n < n_steps; ++n) {
            const int j0 = i0g - (t_begin + n) * BN;
            const bool my_full = empty || (rb.x <= j0 && rb.y >= j0 + BN - 1);
            const bool need_mask = !__all_sync(0xffffffffu, my_full);
            const bool use_band = band_needed(n);
            if (!warp_wait(&s_full[s], n & 1, ctl, p.err, kErrFwdS, p.timeout_ns)) {
                ok = false;
                break;
            }
            if (wq == 0 && lane == 0) IRA_TRACE(p, 11 + 3 * s, n);
            tc_fence_after();
            uint32_t x[128];
            tmem_ld32(tmem + lane_base + L::s_col(s) + 0, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
            tmem_ld32(tmem + lane_base + L::s_col(s) + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
            tmem_ld32(tmem + lane_base + L::s_col(s) + 64, *reinterpret_cast<uint32_t(*)[32]>(&x[64]));
            tmem_ld32(tmem + lane_base + L::s_col(s) + 96, *reinterpret_cast<uint32_t(*)[32]>(&x[96]));
            tmem_wait_ld();

            // pass 1: the row maximum, in the units of `coef` (which turns x into log2 units)
            float mx, coef;
            if (!use_band && !need_mask) {
                // no relative logit and no mask in this step: x stays the raw score and,
                // since scale > 0, max(scale * s) = scale * max(s)
                float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
                for (int c = 0; c < 128; c += 8) {
                    a0 = fmax3(a0, __uint_as_float(x[c + 0]), __uint_as_float(x[c + 1]));
                    a1 = fmax3(a1, __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
                    a2 = fmax3(a2, __uint_as_float(x[c + 4]), __uint_as_float(x[c + 5]));
                    a3 = fmax3(a3, __uint_as_float(x[c + 6]), __uint_as_float(x[c + 7]));
                }
                mx = fmax3(a0, a1, fmaxf(a2, a3));
                coef = p.scale_log2;
            } else {
                // x becomes the logit scale * s + profile bias (natural units), masked
                if (use_band) cp_async_wait_all();
                const int c_lo = rb.x - j0, c_hi = rb.y - j0;  // allowed columns of this row
                const float2 sc2 = make_float2(p.scale, p.scale);
                float a0 = -INFINITY, a1 = -INFINITY;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t w[17];
                    if (use_band) {
#pragma unroll
                        for (int q = 0; q < 17; ++q) w[q] = band_words[g_r + 48 - 16 * c4 + q];
                    }
#pragma unroll
                    for (int pp = 0; pp < 16; ++pp) {
                        const int c = 32 * c4 + 2 * pp;
                        float2 bias = make_float2(0.f, 0.f);
                        if (use_band) {
                            const uint32_t v = funnel_r(w[15 - pp], w[16 - pp], fshift);
                            bias.x = bf16hi_to_f32(v);  // column c
                            bias.y = bf16lo_to_f32(v);  // column c+1
                        }
                        float2 y = __ffma2_rn(make_float2(__uint_as_float(x[c]), __uint_as_float(x[c + 1])), sc2,
                                              bias);
                        if (need_mask) {
                            y.x = (c >= c_lo && c <= c_hi) ? y.x : -INFINITY;
                            y.y = (c + 1 >= c_lo && c + 1 <= c_hi) ? y.y : -INFINITY;
                        }
                        x[c] = __float_as_uint(y.x);
                        x[c + 1] = __float_as_uint(y.y);
                        if (pp & 1)
                            a1 = fmax3(a1, y.x, y.y);
                        else
                            a0 = fmax3(a0, y.x, y.y);
                    }
                }
                mx = fmaxf(a0, a1);
                coef = kLog2e;
                // this row's band buffer is free again: prefetch the next step's window
                // (band_needed is non-increasing in n, so only this path can need it)
                if (n + 1 < n_steps && band_needed(n + 1)) issue_band(n + 1);
            }

            if (wq == 0 && lane == 0) IRA_TRACE(p, 12 + 3 * s, n);
            // running maximum (log2 units): exact on the first step, lazily moved after
            const float mx2 = mx * coef;
            const bool bump = (n == 0) ? (mx2 > m2) : (mx2 > m2 + kRescaleThreshold);
            float alpha = 1.f;
            if (bump) {
                alpha = ex2_approx(m2 - mx2);
                l *= alpha;
                m2 = mx2;
            }
            const float base = (m2 == -INFINITY) ? 0.f : m2;

            // pass 2: probabilities, row sum, BF16 pack, store P over the S columns
            const float2 c2 = make_float2(coef, coef), nb2 = make_float2(-base, -base);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t pk[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int c = 32 * q + 2 * u;
                    const float2 t = __ffma2_rn(make_float2(__uint_as_float(x[c]), __uint_as_float(x[c + 1])), c2, nb2);
                    const float2 pr = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                    pk[u] = pack_bf16x2(pr.x, pr.y);
                    if (u & 1)
                        acc1 = __fadd2_rn(acc1, pr);
                    else
                        acc0 = __fadd2_rn(acc0, pr);
                }
                tmem_st16(tmem + lane_base + L::s_col(s) + 16 * q, pk);
            }
            l += (acc0.x + acc0.y) + (acc1.x + acc1.y);

            // rescale O when a row of this warp moved its maximum (O of step n-1 is complete:
            // the S MMA of this step was committed after it)
            if (n > 0 && __any_sync(0xffffffffu, bump)) {
#pragma unroll 1
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + L::o_col(s) + 32 * c4, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tmem + lane_base + L::o_col(s) + 32 * c4, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[s]);
            if (wq == 0 && lane == 0) IRA_TRACE(p, 13 + 3 * s, n);
        }
        cp_async_wait_all();

        // ---- epilogue: O / l and lse ----
        if (ok && n_steps > 0) {
            ok = warp_wait(&o_full[s], 0, ctl, p.err, kErrFwdO, p.timeout_ns);
            tc_fence_after();
        }
        if (ok) {
            const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
            float* orow = p.out + ((size_t(b) * p.S + i) * p.Hq + h) * size_t(D);
            if (n_steps > 0) {
#pragma unroll 1
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + L::o_col(s) + 32 * c4, o);
                    tmem_wait_ld();
                    if (row_in) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float4 v;
                            v.x = empty ? 0.f : __uint_as_float(o[4 * q + 0]) * inv_l;
                            v.y = empty ? 0.f : __uint_as_float(o[4 * q + 1]) * inv_l;
                            v.z = empty ? 0.f : __uint_as_float(o[4 * q + 2]) * inv_l;
                            v.w = empty ? 0.f : __uint_as_float(o[4 * q + 3]) * inv_l;
                            *reinterpret_cast<float4*>(orow + 32 * c4 + 4 * q) = v;
                        }
                    }
                }
            } else if (row_in) {
                for (int e = 0; e < D; e += 4)
                    *reinterpret_cast<float4*>(orow + e) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (row_in) {
                const float lse = (empty || n_steps == 0) ? sigma : (m2 + log2f(l)) * kLn2;
                p.lse[(size_t(b) * p.S + i) * p.Hq + h] = lse;
            }
        }
    }

    // ---- teardown ----
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

template <int D, int NH>
cudaError_t launch_impl(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                        const AttnParams& p, cudaStream_t st) {
    using L = Layout<D, NH>;
    auto kern = fwd_kernel<D, NH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    const int num_qtiles = (p.S + BM - 1) / BM;
    const long long grid = (long long)num_qtiles * p.B * (p.Hq / NH);
    if (grid == 0) return cudaSuccess;
    kern<<<dim3(unsigned(grid)), dim3(32 * L::NWARPS), L::ALLOC, st>>>(tm_q, tm_k, tm_v, p, num_qtiles);
    return cudaGetLastError();
}

}  // namespace fwdk

cudaError_t launch_fwd(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                       const AttnParams& p, cudaStream_t st) {
    const bool pair = (p.Hq / p.Hkv) % 2 == 0;
    if (p.D == 128) {
        return pair ? fwdk::launch_impl<128, 2>(tm_q, tm_k, tm_v, p, st)
                    : fwdk::launch_impl<128, 1>(tm_q, tm_k, tm_v, p, st);
    }
    return pair ? fwdk::launch_impl<64, 2>(tm_q, tm_k, tm_v, p, st)
                : fwdk::launch_impl<64, 1>(tm_q, tm_k, tm_v, p, st);
}

}  // namespace ira
