// fwd.cu -- forward kernel of learned-relative grouped-query attention (sm_100a).
//
// One CTA handles one 128-row query tile of NH query heads (NH = 2 heads of the
// same KV group when the group size is even, else 1). Each step covers 64 keys;
// its K and V tiles are loaded once by TMA and shared by both heads, K through a
// two-slot ring and V through a three-slot ring, each fed by its own producer.
//
//   warps 0..4*NH-1   softmax, one warpgroup per head (thread = query row =
//                     TMEM lane); each warp also stages its 32 rows' profile
//                     windows (double buffered)
//   warp  4*NH        TMA producer: Q (once), then the K tiles
//   warp  4*NH+1      MMA issuer of head A (one thread): S = Q K^T (SMEM x SMEM
//                     -> TMEM), O += P V (P from TMEM x V from SMEM -> TMEM)
//   warp  4*NH+2      TMA producer: the V tiles
//   warp  4*NH+3      MMA issuer of head B (NH = 2)
//
// S is double buffered per head in TMEM, so the MMAs for step n+2 are queued
// right behind the PV products of step n (P of step n lives in the S buffer it
// aliases) and a softmax warpgroup rarely waits on the tensor core. Each head
// has its own issuing thread, so the tensor core is fed by the other head while
// one issuer waits for its softmax or a tile.
// TMEM: S_A[2], S_B[2] (64 columns each), O_A, O_B (D each).
//
// Per step the softmax warpgroup reads S, adds the learned relative logit
// profiles[b,h,i,d] (d = i_g - j; distances >= R read zeros), masks only the
// steps that cross a document / window / validity boundary, keeps a running
// maximum that starts at the sink logit and is exact on the first step and
// lazily moved afterwards, keeps the running denominator (the sink contributes
// exp(0) = 1, so it enters with no value row), writes P as BF16 over its S
// buffer, and rescales O in TMEM in the rare steps whose maximum moved (after
// the previous PV product is known to be complete).
//
// Key steps are aligned to the query tile: step u covers keys
// [i_g0 + 64 - 64 u, i_g0 + 127 - 64 u], so its distance offset is
// delta = 64 u - 64 and row r needs the distances [delta + r - 63, delta + r].
// That window starts (r + 1) mod 8 elements past a 16-byte boundary for every
// step; each warp copies the windows of its 32 rows (9 x 16 B each, cp.async, zero
// fill outside [0, R); consecutive lanes take consecutive chunks of a row) into a
// buffer whose rows are permuted so that the per-column 32-bit reads of a warp hit
// 32 distinct shared-memory banks.
//
// Operation and argument conventions follow the NeMo AutoModel page for
// Inkling2FlexAttention.forward; see include/inkling_rel_attn.h.
#include <type_traits>

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace ira {
namespace fwdk {

constexpr int BM = 128;               // query rows per tile (TMEM lanes)
constexpr int BN = 64;                // keys per step
// K / V ring slots. A tile copy takes a few thousand cycles from issue to arrival while
// the tensor core and L2 are busy, about a step and a half: K(n+2) is copied once S(n)
// has read K(n) and is needed by S(n+2), issued after step n's probabilities; V(n+3) is
// copied once PV(n) has read V(n) and is needed by PV(n+3), three steps of lead.
constexpr int KSLOTS = 2;
constexpr int VSLOTS = 3;
constexpr int BAND_CHUNKS = 9;        // 16-byte chunks per band row (72 bf16)
constexpr int BAND_PITCH = BAND_CHUNKS * 16;
constexpr int BAND_BYTES = BM * BAND_PITCH;
constexpr int QBOX = BM * 128;        // [128 rows x 64 bf16] 128B-swizzled box
constexpr int KBOX = BN * 128;        // [64 rows x 64 bf16] box

// Row r = 8a + s is stored in slot 8a + ((s + 2a) mod 8): the slot's 16-byte unit
// index is then congruent to (s + 2a) mod 8 (the pitch is 9 units), which spreads
// the 32 rows of a warp over all 32 banks for the column-wise reads below.
__host__ __device__ constexpr int band_slot(int r) { return (r & ~7) | (((r & 7) + 2 * (r >> 3)) & 7); }

template <int D, int NH>
struct Layout {
    static constexpr int KB = D / 64;
    static constexpr int SLOT_BYTES = KB * KBOX;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + NH * KB * QBOX;
    static constexpr int V_OFF = K_OFF + KSLOTS * SLOT_BYTES;
    static constexpr int BAND_OFF = V_OFF + VSLOTS * SLOT_BYTES;
    static constexpr int BAR_OFF = BAND_OFF + NH * 2 * BAND_BYTES;
    // q_full, k_full[KSLOTS], v_full[VSLOTS], k_empty[KSLOTS], v_empty[VSLOTS], drain,
    // s_full[NH][2], p_full[NH][2], o_done[NH], o_full[NH], q_ready[NH]
    static constexpr int NBARS = 2 + 2 * (KSLOTS + VSLOTS) + 7 * NH;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int TOTAL = MISC_OFF + 64;
    static constexpr int ALLOC = TOTAL + 1024;
    // softmax warpgroup(s), then one warpgroup holding the K producer, the MMA
    // issuers and the V producer (whole warpgroups, so that with NH = 2
    // registers can be moved between them)
    static constexpr int NWARPS = 4 * NH + 4;
    static constexpr uint32_t TMEM_COLS = (NH * (128 + D) <= 256) ? 256u : 512u;
    static constexpr uint32_t s_col(int s, int buf) { return uint32_t(s * 128 + buf * 64); }
    static constexpr uint32_t o_col(int s) { return uint32_t(NH * 128 + s * D); }
};

__device__ __forceinline__ int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }
__device__ __forceinline__ int ceil_div_i(int a, int b) { return -floor_div(-a, b); }

// Load K (or V) tiles 0 .. n_steps-1 of this CTA through a ring of NS slots (lane 0 of
// the producer warp): tile n goes to slot n mod NS once the MMAs of every head have
// released it, and completes full[slot]. Before returning, waits for its own copies in
// flight so that none lands in the shared memory of an exiting CTA.
template <int NS, int KB>
__device__ __forceinline__ void produce_ring(const CUtensorMap* tm, uint8_t* ring, uint64_t* full, uint64_t* empty,
                                             int n_steps, int g, int b, int key_first, CtaControl* ctl,
                                             const AttnParams& p, int site, int trace_ev) {
    int last = -1;
    for (int n = 0; n < n_steps; ++n) {
        const int slot = n % NS;
        if (!mbar_wait(&empty[slot], ((n / NS) & 1) ^ 1, ctl, p.err, site, p.timeout_ns)) break;
        mbar_arrive_expect_tx(&full[slot], KB * KBOX);
        for (int kb = 0; kb < KB; ++kb)
            if (IRA_IN_BOUNDS(p.err, kErrBoundsFwdSmem, (slot * KB + kb) * KBOX, KBOX, NS * KB * KBOX))
                tma_load_4d(ring + (slot * KB + kb) * KBOX, tm, &full[slot], kb * 64, g, key_first - n * BN, b);
        IRA_TRACE(p, trace_ev, n);
        last = n;
    }
    for (int n = (last >= NS ? last - NS + 1 : 0); n <= last; ++n) mbar_wait_drain(&full[n % NS], (n / NS) & 1);
}

// CLIP: the L2Clip of q is fused in (each softmax thread clips its row of the Q tile
// in shared memory before the first product and stores the clipped row).
template <int D, int NH, bool CLIP>
__global__ void __launch_bounds__(32 * (4 * NH + 4), 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qc,
               const AttnParams p, const int num_qtiles) {
    using L = Layout<D, NH>;
    constexpr int KB = L::KB;
    constexpr int K_WARP = 4 * NH, MMA_WARP = 4 * NH + 1, V_WARP = 4 * NH + 2, MMA_WARP_B = 4 * NH + 3;

    extern __shared__ uint8_t smem_raw[];
    // aligned by pointer arithmetic on the __shared__ array, so the compiler keeps
    // knowing that every pointer derived from it addresses shared memory
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;                    // [KSLOTS]
    uint64_t* v_full = k_full + KSLOTS;             // [VSLOTS]
    uint64_t* k_empty = v_full + VSLOTS;            // [KSLOTS]
    uint64_t* v_empty = k_empty + KSLOTS;           // [VSLOTS]
    uint64_t* drain = v_empty + VSLOTS;
    uint64_t* s_full = drain + 1;                   // [NH][2]
    uint64_t* p_full = s_full + 2 * NH;             // [NH][2]
    uint64_t* o_done = p_full + 2 * NH;             // [NH]
    uint64_t* o_full = o_done + NH;                 // [NH]
    uint64_t* q_ready = o_full + NH;                // [NH]: Q of head s clipped (CLIP)
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
    // buffer extents for the bounds-checking build (elements; shared memory in bytes)
    [[maybe_unused]] const uint32_t smem_base = smem_u32(smem);
    [[maybe_unused]] const long long n_rows = (long long)p.B * p.S * p.Hq;

    if (threadIdx.x == 0) {
        IRA_TRACE_GRID(p, 0, 0);
        mbar_init(q_full, 1);
        // a K or V slot is free once the MMAs of every head's issuer have read it
        for (int u = 0; u < KSLOTS; ++u) mbar_init(&k_full[u], 1);
        for (int u = 0; u < VSLOTS; ++u) mbar_init(&v_full[u], 1);
        for (int u = 0; u < KSLOTS; ++u) mbar_init(&k_empty[u], NH);
        for (int u = 0; u < VSLOTS; ++u) mbar_init(&v_empty[u], NH);
        mbar_init(drain, NH);
        for (int s = 0; s < NH; ++s) {
            mbar_init(&s_full[2 * s + 0], 1);
            mbar_init(&s_full[2 * s + 1], 1);
            mbar_init(&p_full[2 * s + 0], 4);
            mbar_init(&p_full[2 * s + 1], 4);
            mbar_init(&o_done[s], 1);
            mbar_init(&o_full[s], 1);
            mbar_init(&q_ready[s], 4);  // the head's softmax warps
        }
        ctl->abort = 0;
        const TileBounds* tb = p.tile_bounds + size_t(b) * t64 + 2 * qt;
        const bool tb_ok = IRA_IN_BOUNDS(p.err, kErrBoundsFwdGlobal, size_t(b) * t64 + 2 * qt,
                                         (2 * qt + 1 < t64) ? 2 : 1, (long long)p.B * t64);
        int min_lo = tb_ok ? tb[0].min_lo : 0, max_hi = tb_ok ? tb[0].max_hi : -1, ne = tb_ok ? tb[0].n_nonempty : 0;
        if (tb_ok && 2 * qt + 1 < t64) {
            min_lo = min(min_lo, tb[1].min_lo);
            max_hi = max(max_hi, tb[1].max_hi);
            ne += tb[1].n_nonempty;
        }
        int u_begin = 0, n_steps = 0;
        if (ne > 0) {
            // step u covers keys [i0g + 64 - 64 u, i0g + 127 - 64 u]
            u_begin = max(0, ceil_div_i(i0g + BN - max_hi, BN));
            const int u_end = floor_div(i0g + 2 * BN - 1 - min_lo, BN);
            n_steps = max(0, u_end - u_begin + 1);
        }
        tinfo[0] = u_begin;
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
    const int u_begin = tinfo[0];
    const int n_steps = tinfo[1];
    if (threadIdx.x == 0) {
        IRA_TRACE_GRID(p, 0, 1);
        IRA_TRACE_GRID_INFO(p, 0, n_steps);
    }

    auto q_smem = [&](int s, int kb) { return smem + L::Q_OFF + (s * KB + kb) * QBOX; };
    auto key0 = [&](int n) { return i0g + BN - (u_begin + n) * BN; };

    // With NH = 2 the kernel is launched with 384 x 168 registers and the producer
    // warpgroup gives part of its share to the two softmax warpgroups (128 x 80 +
    // 256 x 208 <= 384 x 168). Each budget change sits at the top of its role's branch.
    if (warp >= 4 * NH) {
        if constexpr (NH == 2) setmaxnreg_dec<80>();
        if (warp == K_WARP) {
            // -------------------------------------------------------- Q and K producer
            if (lane == 0 && n_steps > 0) {
                prefetch_tensormap(&tm_q);
                prefetch_tensormap(&tm_k);
                mbar_arrive_expect_tx(q_full, NH * KB * QBOX);
                for (int s = 0; s < NH; ++s)
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_4d(q_smem(s, kb), &tm_q, q_full, kb * 64, h0 + s, i0, b);
                produce_ring<KSLOTS, KB>(&tm_k, smem + L::K_OFF, k_full, k_empty, n_steps, g, b,
                                               key0(0), ctl, p, kErrFwdKFree, 1);
                mbar_wait_drain(q_full, 0);
            }
        } else if (warp == V_WARP) {
            // -------------------------------------------------------- V producer
            if (lane == 0 && n_steps > 0) {
                prefetch_tensormap(&tm_v);
                produce_ring<VSLOTS, KB>(&tm_v, smem + L::V_OFF, v_full, v_empty, n_steps, g, b,
                                                key0(0), ctl, p, kErrFwdVFree, 2);
            }
        } else if (warp == MMA_WARP || (NH == 2 && warp == MMA_WARP_B)) {
            // -------------------------------------------------------- MMA issuers
            // One issuing thread per head, so that one head's waits never hold back
            // the other head's MMAs. Per step n: O_s += P_s(n) V(n), then
            // S_s(n+2) = Q_s K(n+2)^T into the S buffer that P_s(n) occupied (the
            // tensor core runs one thread's MMAs in issue order). The K and V slots
            // are released once both heads' MMAs that read them have completed.
            const int s = (warp == MMA_WARP) ? 0 : 1;
            if (lane == 0 && n_steps > 0) {
                constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, 0, 0);
                constexpr uint32_t IDESC_O = idesc_bf16_f32(128, D, 0, 1);
                const uint32_t k_base = smem_u32(smem + L::K_OFF), v_base = smem_u32(smem + L::V_OFF);
                const uint32_t q_base = smem_u32(q_smem(s, 0));
                auto wait_k = [&](int n) {  // K(n) has landed
                    return mbar_wait(&k_full[n % KSLOTS], (n / KSLOTS) & 1, ctl, p.err, kErrFwdK, p.timeout_ns);
                };
                auto wait_v = [&](int n) {  // V(n) has landed
                    return mbar_wait(&v_full[n % VSLOTS], (n / VSLOTS) & 1, ctl, p.err, kErrFwdV, p.timeout_ns);
                };
                auto issue_s = [&](int n) {
                    const uint32_t kslot = k_base + (n % KSLOTS) * L::SLOT_BYTES;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * QBOX + (kk & 3) * 32;
                        const uint64_t ad = sdesc_sw128(q_base + off, 16, 1024);
                        const uint64_t bd = sdesc_sw128(kslot + (kk >> 2) * KBOX + (kk & 3) * 32, 16, 1024);
                        mma_ss(tmem + L::s_col(s, n & 1), ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&s_full[2 * s + (n & 1)]);
                    IRA_TRACE(p, 3 + s, n);
                };
                auto issue_o = [&](int n) {
                    const uint32_t vslot = v_base + (n % VSLOTS) * L::SLOT_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        const uint64_t bd = sdesc_sw128(vslot + kk * 2048, KBOX, 1024);
                        mma_ts(tmem + L::o_col(s), tmem + L::s_col(s, n & 1) + kk * 8, bd, IDESC_O,
                               (n > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&o_done[s]);
                    IRA_TRACE(p, 5 + s, n);
                };
                bool ok = mbar_wait(CLIP ? &q_ready[s] : q_full, 0, ctl, p.err, kErrFwdQ, p.timeout_ns);
                if (CLIP && ok) {
                    // the clipped tile goes out to q_clipped by one tensor store (rows
                    // beyond the sequence are not written); waited for before exit
                    for (int kb = 0; kb < KB; ++kb) tma_store_4d(&tm_qc, q_smem(s, kb), kb * 64, h0 + s, i0, b);
                    bulk_commit_group();
                }
                for (int n = 0; ok && n < 2 && n < n_steps; ++n) {
                    ok = wait_k(n);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(n);
                    mma_commit(&k_empty[n % KSLOTS]);
                }
                for (int n = 0; ok && n < n_steps; ++n) {
                    // one barrier per S buffer: the softmax may already have finished
                    // step n + 1 (whose S was issued before this wait)
                    ok = mbar_wait(&p_full[2 * s + (n & 1)], (n >> 1) & 1, ctl, p.err, kErrFwdP, p.timeout_ns);
                    if (!ok) break;
                    IRA_TRACE(p, 7 + s, n);
                    ok = wait_v(n);
                    if (!ok) break;
                    if (s == 0) IRA_TRACE(p, 10, n);
                    tc_fence_after();
                    issue_o(n);
                    mma_commit(&v_empty[n % VSLOTS]);
                    if (n + 2 < n_steps) {
                        ok = wait_k(n + 2);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(n + 2);
                        mma_commit(&k_empty[(n + 2) % KSLOTS]);
                    }
                }
                // O is final once every PV product has completed
                if (ok) mma_commit(&o_full[s]);
                // wait for every MMA of both issuers before TMEM is released
                mma_commit(drain);
                mbar_wait_drain(drain, 0);
                if (CLIP) bulk_wait_all();
            }
        }
    } else {
        if constexpr (NH == 2) setmaxnreg_inc<208>();
        // ------------------------------------------------------------ softmax
        const int s = warp >> 2;
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_base = uint32_t(wq * 32) << 16;
        const int h = h0 + s;
        const int i = i0 + r;
        const bool row_in = i < p.S;
        const int2 rb = row_in && IRA_IN_BOUNDS(p.err, kErrBoundsFwdGlobal, size_t(b) * p.S + i, 1, (long long)p.B * p.S)
                            ? p.row_bounds[size_t(b) * p.S + i]
                            : make_int2(kEmptyLo, kEmptyHi);
        const bool empty = rb.x > rb.y;
        // no sink array: no sink term (a logit of -inf)
        const int64_t sink_at = b * p.sink_sb + i * p.sink_ss + h * p.sink_sh;
        const float sigma = !row_in ? 0.f
                            : !p.sink ? -INFINITY
                            : IRA_IN_BOUNDS(p.err, kErrBoundsFwdGlobal, sink_at, 1,
                                            (p.B - 1) * p.sink_sb + (p.S - 1) * p.sink_ss + (p.Hq - 1) * p.sink_sh + 1)
                                ? p.sink[sink_at]
                                : 0.f;
        float m2 = sigma * kLog2e;  // running maximum, log2 units
        float l = 1.f;              // running denominator; the sink contributes exp(0)
        bool seen = false;          // some earlier step held an unmasked key of this row

        uint8_t* band0 = smem + L::BAND_OFF + (2 * s) * BAND_BYTES;
        const int row_off = band_slot(r) * BAND_PITCH;
        const int m_r = (r + 1) & 7;   // misalignment of the row's window start
        const int g_r = m_r >> 1;
        const uint32_t fshift = uint32_t(m_r & 1) * 16u;
        [[maybe_unused]] const long long prof_n = (long long)p.B * p.Hq * p.S * p.R;
        auto delta_of = [&](int n) { return BN * (u_begin + n) - BN; };
        // the warp's smallest distance is delta + 32 wq - 63: no profile entry if >= R
        auto band_needed = [&](int n) { return delta_of(n) + wq * 32 - (BN - 1) < p.R; };
        // Copy the windows of step n of this warp's 32 rows into band buffer (n & 1). The
        // warp copies its rows together: chunk k = 32 t + lane of the warp's 32 x 9 chunks
        // is chunk k mod 9 of row k / 9, so the lanes of one copy instruction read a few
        // contiguous row segments instead of 32 rows at once. Always commits a group, so
        // that exactly two groups are outstanding at every wait below; a row is read only
        // after every lane's wait and a __syncwarp.
        const uint16_t* const prof_tile =
            p.R > 0 ? p.profiles + ((size_t(b) * p.Hq + h) * p.S + i0) * size_t(p.R) : nullptr;
        auto issue_band = [&](int n) {
            if (n < n_steps && band_needed(n)) {
                uint8_t* const dst_buf = band0 + (n & 1) * BAND_BYTES;
                const int dl = delta_of(n);
#pragma unroll
                for (int t = 0; t < BAND_CHUNKS; ++t) {
                    const int k = 32 * t + lane;
                    const int rr = wq * 32 + k / BAND_CHUNKS, q = k % BAND_CHUNKS;
                    const int d0 = dl + rr - (BN - 1) - ((rr + 1) & 7) + 8 * q;
                    const bool inb = prof_tile != nullptr && i0 + rr < p.S && d0 >= 0 && d0 < p.R;
                    const size_t at = size_t(rr) * p.R + d0;
                    const void* src = inb ? static_cast<const void*>(prof_tile + at) : p.safe_src;
                    const uint32_t dst = smem_u32(dst_buf + band_slot(rr) * BAND_PITCH + 16 * q);
                    if (IRA_IN_BOUNDS(p.err, kErrBoundsFwdSmem, dst - smem_base, 16, L::TOTAL) &&
                        IRA_IN_BOUNDS(p.err, kErrBoundsFwdGlobal,
                                      inb ? ((size_t(b) * p.Hq + h) * p.S + i0) * size_t(p.R) + at : 0, inb ? 8 : 0,
                                      prof_n))
                        cp_async_16(dst, src, inb ? 16u : 0u);
                }
            }
            cp_async_commit();
        };
        if constexpr (CLIP) {
            // L2Clip of this row of q (head h): z = x * scale, y = z * min(1, thr / |z|) * tau,
            // rounded to BF16 and written over the Q tile in shared memory, where the
            // products read it and from where the MMA issuer stores the tile to q_clipped
            // (for the backward). The tile is 128-byte swizzled: 16-byte chunk c of a row
            // of a 64-column box sits at chunk c ^ (r mod 8) of that row.
            const bool q_ok = warp_wait(q_full, 0, ctl, p.err, kErrFwdQ, p.timeout_ns);
            const float* const sc = p.clip_scale ? p.clip_scale + size_t(h) * D : nullptr;
            auto chunk_at = [&](int c) {  // chunk c (8 columns) of the row
                return q_smem(s, c >> 3) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
            };
            auto chunk_z = [&](int c, float (&z)[8]) {
                const uint4 u = *reinterpret_cast<const uint4*>(chunk_at(c));
                const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    z[2 * e] = bf16lo_to_f32(wv[e]);
                    z[2 * e + 1] = bf16hi_to_f32(wv[e]);
                }
                if (sc) {  // every lane reads the same 32 bytes: one broadcast access each
                    const float4 s0 = *reinterpret_cast<const float4*>(sc + 8 * c);
                    const float4 s1 = *reinterpret_cast<const float4*>(sc + 8 * c + 4);
                    z[0] *= s0.x; z[1] *= s0.y; z[2] *= s0.z; z[3] *= s0.w;
                    z[4] *= s1.x; z[5] *= s1.y; z[6] *= s1.z; z[7] *= s1.w;
                }
            };
            if (q_ok) {
                float ss0 = 0.f, ss1 = 0.f;
#pragma unroll 4
                for (int c = 0; c < D / 8; ++c) {
                    float z[8];
                    chunk_z(c, z);
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        ss0 = fmaf(z[e], z[e], ss0);
                        ss1 = fmaf(z[e + 1], z[e + 1], ss1);
                    }
                }
                const float nrm = sqrtf(ss0 + ss1);
                float f = (nrm > p.clip_thr) ? p.clip_thr / nrm : 1.f;
                if (p.clip_tau && row_in) f *= p.clip_tau[size_t(b) * p.S + i];
#pragma unroll 4
                for (int c = 0; c < D / 8; ++c) {
                    float z[8];
                    chunk_z(c, z);
                    *reinterpret_cast<uint4*>(chunk_at(c)) =
                        make_uint4(pack_bf16x2(z[0] * f, z[1] * f), pack_bf16x2(z[2] * f, z[3] * f),
                                   pack_bf16x2(z[4] * f, z[5] * f), pack_bf16x2(z[6] * f, z[7] * f));
                }
                fence_proxy_async_smem();  // the tensor core and the tensor store read these bytes next
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_ready[s]);
        }

        issue_band(0);
        issue_band(1);
        bool ok = true;
        for (int n = 0; n < n_steps; ++n) {
            const int buf = n & 1;
            const int jk = key0(n);
            const bool my_full = empty || (rb.x <= jk && rb.y >= jk + BN - 1);
            const bool need_mask = !__all_sync(0xffffffffu, my_full);
            const bool use_band = band_needed(n);
            if (!warp_wait(&s_full[2 * s + buf], (n >> 1) & 1, ctl, p.err, kErrFwdS, p.timeout_ns)) {
                ok = false;
                break;
            }
            if (wq == 0 && lane == 0) IRA_TRACE(p, 11 + 3 * s, n);
            if (s == 0 && lane == 0) IRA_TRACE(p, 28 + wq, n);  // per-warp S ready (head A)
            if (n == 0 && threadIdx.x == 0) IRA_TRACE_GRID(p, 0, 2);
            tc_fence_after();
            uint32_t x[64];
            tmem_ld32(tmem + lane_base + L::s_col(s, buf) + 0, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
            tmem_ld32(tmem + lane_base + L::s_col(s, buf) + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
            tmem_wait_ld();

            // pass 1: the row maximum, in the units of `coef` (which turns x into log2 units)
            float mx, coef;
            if (!use_band && !need_mask) {
                // no relative logit and no mask in this step: x stays the raw score and,
                // since scale > 0, max(scale * s) = scale * max(s)
                float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
                for (int c = 0; c < 64; c += 8) {
                    a0 = fmax3(a0, __uint_as_float(x[c + 0]), __uint_as_float(x[c + 1]));
                    a1 = fmax3(a1, __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
                    a2 = fmax3(a2, __uint_as_float(x[c + 4]), __uint_as_float(x[c + 5]));
                    a3 = fmax3(a3, __uint_as_float(x[c + 6]), __uint_as_float(x[c + 7]));
                }
                mx = fmax3(a0, a1, fmaxf(a2, a3));
                coef = p.scale_log2;
            } else {
                // x becomes the logit scale * s + profile bias (natural units), masked;
                // specialised on whether the step reads the band and needs the mask
                auto pass1 = [&](auto band_c, auto mask_c) {
                    constexpr bool BAND = decltype(band_c)::value, MASK = decltype(mask_c)::value;
                    uint32_t w[33];
                    if (BAND) {
                        cp_async_wait_group<1>();  // this step's windows (the next step's may fly)
                        __syncwarp();              // ... copied by every lane of the warp
                        if (s == 0 && lane == 0) IRA_TRACE(p, 24 + wq, n);  // per-warp band ready (head A)
                        const uint32_t* words =
                            reinterpret_cast<const uint32_t*>(band0 + buf * BAND_BYTES + row_off) + g_r;
                        const bool w_ok = IRA_IN_BOUNDS(p.err, kErrBoundsFwdSmem, smem_u32(words) - smem_base, 33 * 4,
                                                        L::TOTAL);
#pragma unroll
                        for (int q = 0; q < 33; ++q) w[q] = w_ok ? words[q] : 0u;
                        if (s == 0 && lane == 0) IRA_TRACE(p, 36 + wq, __uint_as_float(w[0]) == 12345.f ? n + 1 : n);
                    }
                    // allowed columns [c_lo, c_lo + c_span] (none for an empty row)
                    const int c_lo = empty ? BN : rb.x - jk, c_span = empty ? 0 : rb.y - rb.x;
                    float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int pp = 0; pp < 32; ++pp) {
                        const int c = 2 * pp;
                        float b0 = 0.f, b1 = 0.f;
                        if (BAND) {
                            const uint32_t v = funnel_r(w[31 - pp], w[32 - pp], fshift);
                            b0 = bf16hi_to_f32(v);  // column c
                            b1 = bf16lo_to_f32(v);  // column c+1
                        }
                        float y0 = fmaf(__uint_as_float(x[c]), p.scale, b0);
                        float y1 = fmaf(__uint_as_float(x[c + 1]), p.scale, b1);
                        if (MASK) {
                            y0 = uint32_t(c - c_lo) <= uint32_t(c_span) ? y0 : -INFINITY;
                            y1 = uint32_t(c + 1 - c_lo) <= uint32_t(c_span) ? y1 : -INFINITY;
                        }
                        x[c] = __float_as_uint(y0);
                        x[c + 1] = __float_as_uint(y1);
                        a[pp & 3] = fmax3(a[pp & 3], y0, y1);
                    }
                    if (s == 0 && lane == 0) IRA_TRACE(p, 32 + wq, n);  // per-warp pass-1 math done (head A)
                    return fmax3(a[0], a[1], fmaxf(a[2], a[3]));
                };
                using T_ = std::true_type;
                using F_ = std::false_type;
                if (use_band && need_mask) mx = pass1(T_{}, T_{});
                else if (use_band) mx = pass1(T_{}, F_{});
                else mx = pass1(F_{}, T_{});
                coef = kLog2e;
            }
            // this step's band buffer is consumed (by every lane: the copies into it are
            // shared): fetch the windows of step n + 2 into it
            __syncwarp();
            issue_band(n + 2);
            if (wq == 0 && lane == 0) IRA_TRACE(p, 12 + 3 * s, n);

            // running maximum (log2 units): exact on the row's first step with an
            // unmasked key (so its largest probability is exactly 1 in BF16), lazily
            // moved after. Until then every P of the row was 0, so its O row is 0 and
            // needs no rescale.
            const float mx2 = mx * coef;
            const bool first = !seen;
            seen = seen || (mx2 > -INFINITY);
            const bool bump = first ? (mx2 > m2) : (mx2 > m2 + kRescaleThreshold);
            float alpha = 1.f;
            if (bump) {
                alpha = ex2_approx(m2 - mx2);
                l *= alpha;
                m2 = mx2;
            }
            const float base = (m2 == -INFINITY) ? 0.f : m2;

            // pass 2: probabilities, row sum, BF16 pack, store P over this step's S buffer
            const float2 c2 = make_float2(coef, coef), nb2 = make_float2(-base, -base);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t pk[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int c = 32 * q + 2 * u;
                    const float2 t =
                        __ffma2_rn(make_float2(__uint_as_float(x[c]), __uint_as_float(x[c + 1])), c2, nb2);
                    // a share of the pairs on the FMA pipe, the rest on the MUFU
                    const float2 pr = ((IRA_FWD_FMA_PAIRS >> u) & 1u) ? exp2_fma2(t)
                                                                       : make_float2(ex2_approx(t.x), ex2_approx(t.y));
                    pk[u] = pack_bf16x2(pr.x, pr.y);
                    if (u & 1)
                        acc1 = __fadd2_rn(acc1, pr);
                    else
                        acc0 = __fadd2_rn(acc0, pr);
                }
                tmem_st16(tmem + lane_base + L::s_col(s, buf) + 16 * q, pk);
            }
            l += (acc0.x + acc0.y) + (acc1.x + acc1.y);
            if (s == 0 && lane == 0) IRA_TRACE(p, 40 + wq, __float_as_uint(l) == 0x7fffffffu ? n + 1 : n);  // pass 2 issued

            // rescale O when a row of this warp moved its maximum; the PV product of
            // step n-1 must be complete first (the one of step n waits for this P).
            // The parity wait is unambiguous: S(n), already waited for, was issued
            // after PV(n-2), and PV(n) cannot start before this warp's arrival.
            if (__any_sync(0xffffffffu, bump && !first)) {
                if (!warp_wait(&o_done[s], (n - 1) & 1, ctl, p.err, kErrFwdO, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
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
            if (s == 0 && lane == 0) IRA_TRACE(p, 44 + wq, n);  // P in TMEM (head A)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[2 * s + buf]);
            if (wq == 0 && lane == 0) IRA_TRACE(p, 13 + 3 * s, n);
            if (s == 0 && lane == 0) IRA_TRACE(p, 20 + wq, n);  // per-warp P done (head A)
        }
        cp_async_wait_all();
        __syncwarp();  // the band rows, reused for staging below, are the warp's own
        if (threadIdx.x == 0) IRA_TRACE_GRID(p, 0, 3);

        // ---- epilogue: O / l and lse ----
        if (ok && n_steps > 0) {
            ok = warp_wait(&o_full[s], 0, ctl, p.err, kErrFwdO, p.timeout_ns);
            tc_fence_after();
        }
        if (ok) {
            const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
            const int64_t orow_at = b * p.row_sb + i * p.row_ss + h * p.row_sh;
            float* orow = p.out + orow_at;
            uint16_t* orow16 = p.out_bf16 ? p.out_bf16 + orow_at : nullptr;
            auto store4 = [&](int e, float4 v) {  // output columns e .. e + 3
                if (orow16) {
                    uint2 u;
                    u.x = pack_bf16x2(v.x, v.y);
                    u.y = pack_bf16x2(v.z, v.w);
                    *reinterpret_cast<uint2*>(orow16 + e) = u;
                } else {
                    *reinterpret_cast<float4*>(orow + e) = v;
                }
            };
            if (n_steps > 0) {
                // 32 x 32 chunks go out through this warp's own 32 band rows (idle now: every
                // copy into them has completed), 144-byte pitch: each lane writes its row,
                // then 8 lanes store 128 contiguous bytes of one row, four rows per store
                float* const stage = reinterpret_cast<float*>(band0 + 32 * wq * BAND_PITCH);
                constexpr int SP = BAND_PITCH / 4;  // staging row pitch in floats
                const int sr = lane >> 3, sc = 4 * (lane & 7);
#pragma unroll 1
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + L::o_col(s) + 32 * c4, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 v;
                        v.x = empty ? 0.f : __uint_as_float(o[4 * q + 0]) * inv_l;
                        v.y = empty ? 0.f : __uint_as_float(o[4 * q + 1]) * inv_l;
                        v.z = empty ? 0.f : __uint_as_float(o[4 * q + 2]) * inv_l;
                        v.w = empty ? 0.f : __uint_as_float(o[4 * q + 3]) * inv_l;
                        if (IRA_IN_BOUNDS(p.err, kErrBoundsFwdSmem, smem_u32(stage + lane * SP + 4 * q) - smem_base,
                                          16, L::TOTAL))
                            *reinterpret_cast<float4*>(stage + lane * SP + 4 * q) = v;
                    }
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int rr = 4 * k + sr;           // row of this warp
                        const int ir = i0 + 32 * wq + rr;    // its query row
                        const bool st_ok = IRA_IN_BOUNDS(p.err, kErrBoundsFwdSmem, smem_u32(stage + rr * SP + sc) - smem_base,
                                                         16, L::TOTAL);
                        const float4 v = st_ok ? *reinterpret_cast<const float4*>(stage + rr * SP + sc)
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
                        const int64_t at = b * p.row_sb + ir * p.row_ss + h * p.row_sh + 32 * c4 + sc;
                        if (ir < p.S && IRA_IN_BOUNDS(p.err, kErrBoundsFwdGlobal, at, 4, n_rows * D)) {
                            if (p.out_bf16) {
                                *reinterpret_cast<uint2*>(p.out_bf16 + at) =
                                    make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
                            } else {
                                *reinterpret_cast<float4*>(p.out + at) = v;
                            }
                        }
                    }
                    __syncwarp();
                }
            } else if (row_in && IRA_IN_BOUNDS(p.err, kErrBoundsFwdGlobal, orow_at, D, n_rows * D)) {
                for (int e = 0; e < D; e += 4) store4(e, make_float4(0.f, 0.f, 0.f, 0.f));
            }
            const int64_t lse_at = b * p.lse_sb + i * p.lse_ss + h * p.lse_sh;
            if (row_in && IRA_IN_BOUNDS(p.err, kErrBoundsFwdGlobal, lse_at, 1, n_rows)) {
                const float lse = (empty || n_steps == 0) ? sigma : (m2 + log2f(l)) * kLn2;
                p.lse[lse_at] = lse;
            }
        }
    }

    // ---- teardown ----
    if (threadIdx.x == 0) IRA_TRACE_GRID(p, 0, 4);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
        if (lane == 0) IRA_TRACE_GRID(p, 0, 5);
    }
}

template <int D, int NH, bool CLIP>
cudaError_t launch_impl(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                        const CUtensorMap& tm_qc, const AttnParams& p, cudaStream_t st) {
    using L = Layout<D, NH>;
    auto kern = fwd_kernel<D, NH, CLIP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
    if (e != cudaSuccess) return e;
    const int num_qtiles = (p.S + BM - 1) / BM;
    const long long grid = (long long)num_qtiles * p.B * (p.Hq / NH);
    if (grid == 0) return cudaSuccess;
    kern<<<dim3(unsigned(grid)), dim3(32 * L::NWARPS), L::ALLOC, st>>>(tm_q, tm_k, tm_v, tm_qc, p, num_qtiles);
    return cudaGetLastError();
}

}  // namespace fwdk

cudaError_t launch_fwd(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                       const AttnParams& p, cudaStream_t st) {
    const bool pair = (p.Hq / p.Hkv) % 2 == 0;
    if (p.D == 128) {
        return pair ? fwdk::launch_impl<128, 2, false>(tm_q, tm_k, tm_v, tm_q, p, st)
                    : fwdk::launch_impl<128, 1, false>(tm_q, tm_k, tm_v, tm_q, p, st);
    }
    return pair ? fwdk::launch_impl<64, 2, false>(tm_q, tm_k, tm_v, tm_q, p, st)
                : fwdk::launch_impl<64, 1, false>(tm_q, tm_k, tm_v, tm_q, p, st);
}

cudaError_t launch_fwd_qclip(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const CUtensorMap& tm_qc, const AttnParams& p, cudaStream_t st) {
    const bool pair = (p.Hq / p.Hkv) % 2 == 0;
    if (p.D == 128) {
        return pair ? fwdk::launch_impl<128, 2, true>(tm_q, tm_k, tm_v, tm_qc, p, st)
                    : fwdk::launch_impl<128, 1, true>(tm_q, tm_k, tm_v, tm_qc, p, st);
    }
    return pair ? fwdk::launch_impl<64, 2, true>(tm_q, tm_k, tm_v, tm_qc, p, st)
                : fwdk::launch_impl<64, 1, true>(tm_q, tm_k, tm_v, tm_qc, p, st);
}

}  // namespace ira
