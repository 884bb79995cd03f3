// Windowed INT8 decode step (the hot path).
//
// LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent
// State Quantization", section "Abstract (arXiv)"): within a window, outputs
// are formed from the fixed low-bit state plus high-precision buffered
// updates, and Compensator Tokens take the update path of real tokens.  With
// G_t the log-gate summed since the window start, gamma_t = exp(G_t),
// x^q = gamma_t * q_t and x^k = gamma_t * k_t:
//   S_{t-1}(alpha_t * k_t) = S~ x^k + sum_{j<t} delta_j (kappa_j . x^k)
//   delta_t = beta_t (v_t - S_{t-1}(alpha_t * k_t))
//   o_t     = S~ x^q + sum_{j<t} delta_j (kappa_j . x^q) + delta_t (k_t . q_t)
// where S~ = sigma Q s + C is the window-start state and kappa_j = k_j/gamma_j.
// For the scalar gate the buffer keeps raw keys and omega_j = exp(-G_j), and
// kappa_j . x^k = gamma_t omega_j (k_j . k_t).  The step reads the INT8 tile
// once, forms both products S~ x^q and S~ x^k in that pass, adds the
// O((n_c + n_buf) d) corrections and appends (delta_t, key_t, omega_t) to the
// buffer.  It writes no state.
//
// Persistent and warp-specialized: four CTAs per SM walk the (sequence, head)
// units in whole rounds (CTA b takes b, b + grid, ...), and the units of the
// last, partial round go to the CTAs that get there first, by a ticket
// counter.  In each CTA one producer thread loads a unit's scalars (beta, the
// scalar gate) and streams its data through a ring of three 16 KB
// shared-memory slots -- a meta segment (row scales, smoothing factors,
// q/k/v, gate, compensators) by 1-D bulk async copies, the INT8 tile by a 2-D
// tensor copy with 128-byte swizzle, then the buffered entries in chunks of up
// to 16 -- and four consumer warps compute.  Each slot has a full mbarrier
// (bytes landed, and for a meta segment the producer's record of the unit) and
// an empty mbarrier that every consumer thread arrives on after its last read,
// so no block-wide barrier is spent on releasing slots; the consumers meet at
// one barrier when a unit's record arrives, one after the operand prep and one
// per chunk.  Each thread keeps its row scale sigma_i in a
// register, so the meta slot goes back before the INT8 pass starts.
//
// The INT8 pass is an exact integer dot product on the tensor cores.  Each
// 32-column block of y^q = s*x^q and y^k = s*x^k is written as
// y = 2^E (d_0 + d_1 2^-7 + d_2 2^-14 + d_3 2^-21) with int8 digits d_p and a
// block exponent E (every step exact in FP32; the dropped remainder is below
// 2^-27 of the block maximum).  The products Q d_p of all 8 (vector, digit)
// columns are exact int32 sums, and the digits are recombined in FP32; no
// per-byte widening is needed.  For d = 128, once the CTAs walk two units or
// more each, one thread issues them on the fifth-generation tensor cores
// (tcgen05.mma kind::i8: per 32-column block an M = 128, N = 16, K = 32
// product from the swizzled tile and the digit rows in shared memory into
// tensor memory, lane i = row i) as soon as the tile has landed, so the pass
// runs while the warps form the compensator terms; each warp then reads its
// 32 rows back.  Otherwise (d = 64, or one unit per CTA, where the tensor
// memory's allocation and the commit round trip would be pure latency) the
// warps use mma.sync m16n8k32.  Both give the same sums and the same FP32
// recombination.
// Every wait is bounded; an expired wait records LQ_DEVERR_TIMEOUT and all
// consumer warps leave together at their next barrier.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "lq_decode_parts.cuh"
#include "lq_kernels.h"

namespace lq {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kConsumers + 32;     // + one producer warp
constexpr int kSlotBytes = 16384;
constexpr int kSlots = 3;
constexpr int kCtasPerSm = 4;
constexpr int kConsumerBarrier = 1;           // named barrier of the consumer warps
constexpr int kPer = 4;                       // buffered entries per warp per chunk
using namespace dec;

__device__ __forceinline__ bool consumer_sync_or(bool pred) { return named_sync_or(kConsumerBarrier, kConsumers, pred); }

// What the producer tells the consumers about the unit whose meta segment
// fills a slot (u < 0: no unit is left).  Scalar gate: G_t = G_{t-1} + g_t and
// gamma_t = exp(G_t).
struct UnitRec {
    double G;
    float gam;
    float beta;
    int u;
    int n_buf;
};

// The unit-ticket counter: a 64-bit word in the error region (int32 index).
constexpr int kTicketWord = 32;

template <int D, bool KDA, typename InT, typename KeyT, bool TCP>
struct Shape {
    static constexpr int KB = (int)sizeof(KeyT);
    static constexpr int ENTRY = 4 * D + KB * D + (KDA ? 0 : 4);   // bytes per buffered entry
    static constexpr int E0 = (kSlotBytes / ENTRY) & ~3;
    static constexpr int E = E0 < kPer * kConsumerWarps ? E0 : kPer * kConsumerWarps;
    static constexpr int C_KEY = 4 * D * E;                        // chunk: deltas, keys, omega_j
    static constexpr int C_GATE = C_KEY + KB * D * E;
    static constexpr int KBLK = D / 32;                            // 32-column blocks (one per prep warp)
    static constexpr int MT = D / 16 / kConsumerWarps;             // 16-row m-tiles per warp
    // the INT8 pass on tcgen05 (one thread issues it, the sums land in tensor
    // memory, lane i = row i; d = 128 only), else on warp-level mma.sync
    static constexpr bool TC = TCP && (D == 128);
    // consumer scratch, in floats: digits (8 x D int8; with the tensor-core pass
    // 16 rows of D in its swizzled operand layout, 8 of them zero), block
    // scales, vectors, products, coefficients (two buffers), compensator dots,
    // reductions
    static constexpr int RED = 1 + 2 * 8;                          // kq, then (k, q) dots of 8 row comps
    static constexpr int S_B8 = 0, S_EXP = S_B8 + (TC ? 4 * D : 2 * D), S_XQ = S_EXP + 8, S_XK = S_XQ + D, S_QR = S_XK + D,
                         S_KR = S_QR + D, S_A = S_KR + D, S_B = S_A + D, S_CF = S_B + D,
                         S_RED = S_CF + 64, S_FLOATS = S_RED + kConsumerWarps * RED;
    static constexpr int OFF_BARS = 4 * S_FLOATS;                  // then the unit records, the ring (1024-aligned)
    static constexpr int OFF_REC = OFF_BARS + 16 * kSlots + 16;    // + MMA barrier, TMEM slot
    static constexpr int OFF_RING = align_up(OFF_REC + (int)sizeof(UnitRec) * kSlots, 1024);
    static constexpr int SMEM = OFF_RING + kSlots * kSlotBytes + 1024;   // + alignment slack
    static_assert(E >= 4 && E <= kPer * kConsumerWarps, "chunk size");
    static_assert(MT >= 1, "m-tiles");
};

template <int D, bool KDA, typename InT, typename KeyT, bool RAGGED, bool TCP>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_window_kernel(DecodeArgs a, const __grid_constant__ CUtensorMap codes_map) {
    using Sh = Shape<D, KDA, InT, KeyT, TCP>;
    constexpr int E = Sh::E, KBLK = Sh::KBLK, MT = Sh::MT;
    const Views &w = a.w;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ncr = w.n_comp_rows, ncc = w.n_comp_cols, cis = w.comp_index_stride, ncomp = ncr + ncc;
    const int units = w.units;
    // Tokens buffered in unit u's window, and whether it takes a token this step:
    // one count and every unit active, or (ragged phases) per-unit counts and
    // per-sequence activity.  The producer and the consumers decide alike.
    auto unit_fill = [&](int u) -> int { return RAGGED ? a.fill[u] : a.n_buf; };
    auto unit_active = [&](int u) -> bool { return !RAGGED || a.active == nullptr || a.active[u / a.heads] != 0; };
    const Meta M = meta_layout<D, KDA, InT>(ncr, ncc, cis);

    extern __shared__ __align__(1024) unsigned char sm_raw[];
    // the swizzled tensor copies need a 1024-byte aligned destination
    unsigned char *sm = sm_raw + ((1024 - (smem_u32(sm_raw) & 1023)) & 1023);
    float *scr = reinterpret_cast<float *>(sm);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + Sh::OFF_BARS);
    uint64_t *empty = full + kSlots;
    uint64_t *mma_bar = empty + kSlots;            // tcgen05 pass complete (d = 128)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_bar + 1);
    UnitRec *rec = reinterpret_cast<UnitRec *>(sm + Sh::OFF_REC);   // one per ring slot
    unsigned char *ring = sm + Sh::OFF_RING;
    unsigned char *dig = sm + Sh::S_B8 * 4;        // digit operand (scratch starts at sm)

    if (tid == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumers);
        }
        mbar_init(mma_bar, 1);
        fence_mbar_init();
    }
    if constexpr (Sh::TC) {
        // the digit operand has 16 rows for N = 16; rows 8..15 stay zero
        for (int i = tid; i < 1024 / 4; i += kThreads) reinterpret_cast<uint32_t *>(dig + 1024)[i] = 0u;
        if (warp == 0) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                         "r"(kTmemCols));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
        tc_fence_before();
    }
    __syncthreads();
    if constexpr (Sh::TC) tc_fence_after();

    // ================================================================ producer
    if (warp == kConsumerWarps) {
        if (lane != 0) return;
        const uint32_t in_b = (uint32_t)sizeof(InT) * D;
        // Units: CTA b walks b, b + grid, ... through the whole rounds; the
        // units of the last, partial round are handed out by ticket (see
        // ticket_unit) to the CTAs that get there first.  Each CTA draws at the
        // start of its last whole-round unit, after the wait for the previous
        // kernel, so no two launches draw at the same time.
        const int grid = (int)gridDim.x;
        const int rounds = units / grid;
        const int n_dyn = units - rounds * grid;
        unsigned long long *tickets = reinterpret_cast<unsigned long long *>(w.err + kTicketWord);
        struct Scalars {
            int n;
            bool act;
            float beta, g;
            double gs;
        };
        auto fetch = [&](int uu, Scalars &s) {   // loads left in flight until the values are used
            s.n = unit_fill(uu);
            s.act = unit_active(uu);
            s.beta = a.beta[uu];
            if (!KDA) {
                s.g = a.g[uu];
                s.gs = w.gate_sum[uu];
            }
        };
        int u = (int)blockIdx.x;
        Scalars cur{};                             // unit u's
        int slot = 0;
        uint32_t ph = 0;
        uint32_t armed = 0;                        // slots filled at least once
        // The record of unit u's meta slot goes out with the slot's arrival,
        // once the unit's INT8 tile is on its way.
        int pend = -1;
        auto publish = [&]() {
            UnitRec &r = rec[pend];
            r.u = u;
            r.n_buf = cur.n;
            r.beta = cur.beta;
            if (!KDA) {
                r.G = cur.gs + (double)cur.g;
                r.gam = exp_of_double(r.G);
            }
            mbar_arrive(&full[pend]);              // releases the record; the phase ends when the bytes land
            pend = -1;
        };
        // a meta slot that will get no unit: it completes (once its copies have
        // landed) as the end of the units
        auto stop = [&](int ms) {
            rec[ms].u = -1;
            mbar_arrive(&full[ms]);
        };
        auto acquire = [&](int uu, int detail) -> unsigned char * {
            if (!mbar_wait(&empty[slot], ph ^ 1u, kWaitBudgetCycles)) {
                report_error(w.err, LQ_DEVERR_TIMEOUT, uu, detail);
                return nullptr;
            }
            armed |= 1u << slot;
            return ring + slot * kSlotBytes;
        };
        auto advance = [&]() {
            if (++slot == kSlots) { slot = 0; ph ^= 1u; }
        };
        // After a timed-out acquire the consumers stop (a meta slot still owed a
        // record gets the end one): wait (bounded) until every copy this thread
        // started has landed, so that no copy still writes into the shared
        // memory of a CTA that has exited.  Slot i was last filled in the round
        // whose parity is ph for i < slot and ph ^ 1 for i >= slot.
        auto fail = [&]() {
            if (pend >= 0) stop(pend);
            for (int i = 0; i < kSlots; ++i)
                if (armed & (1u << i)) mbar_wait(&full[i], i < slot ? ph : (ph ^ 1u), kWaitBudgetCycles);
        };

        // The first unit's code tile takes ring slot 1 of the first round, as the
        // loop below would give it.  With the codes settled it is fetched before
        // the wait for the previous kernel in the stream, which cannot write it.
        const int early_u = (!RAGGED && a.codes_settled) ? u : -1;
        if (early_u >= 0) {
            armed |= 2u;                           // slot 1's empty barrier is in its first phase
            mbar_arrive_expect_tx(&full[1], D * D);
            tma_load_2d(ring + kSlotBytes, &codes_map, 0, early_u * D, &full[1]);
        }
        grid_dependency_wait();
        unsigned long long tk = 0;
        bool draw = n_dyn > 0, drawn = false;
        fetch(u, cur);
        for (int k = 0; u >= 0; ++k) {             // k: units walked
            if (draw && !drawn && k == rounds - 1) {   // the ticket is back by the end of this unit
                tk = atomicAdd(tickets, 1ull);
                drawn = true;
            }
            const int n_buf = cur.n;
            bool issue = true;
            if (RAGGED) {
                if (!cur.act) {
                    issue = false;
                } else if (n_buf >= w.window) {    // ragged phases: the window is full
                    report_error(w.err, LQ_DEVERR_WINDOW_FULL, u, n_buf);
                    issue = false;
                } else if (!in_bounds(w.err, n_buf, 0, w.window, u, -10)) {
                    issue = false;                 // checked build: a negative count (a corrupted workspace)
                }
            }
            if (issue) {
                unsigned char *dst = acquire(u, -1);
                if (dst == nullptr) { fail(); return; }
                pend = slot;
                uint64_t *bar = &full[slot];
                mbar_expect_tx(bar, (uint32_t)M.bytes);   // the arrival comes with the record
                bulk_g2s(dst + M.sig, w.row_scale + (size_t)u * D, 4 * D, bar);
                bulk_g2s(dst + M.s, w.col_smooth + (size_t)u * D, 4 * D, bar);
                bulk_g2s(dst + M.qin, reinterpret_cast<const InT *>(a.q) + (size_t)u * D, in_b, bar);
                bulk_g2s(dst + M.kin, reinterpret_cast<const InT *>(a.k) + (size_t)u * D, in_b, bar);
                bulk_g2s(dst + M.vin, reinterpret_cast<const InT *>(a.v) + (size_t)u * D, in_b, bar);
                if (KDA) {
                    bulk_g2s(dst + M.gin, a.g + (size_t)u * D, 4 * D, bar);
                    bulk_g2s(dst + M.gsum, w.gate_sum + (size_t)u * D, 8 * D, bar);
                }
                if (ncomp > 0) {
                    bulk_g2s(dst + M.cidx, w.comp_index + (size_t)u * cis, 4 * cis, bar);
                    if (ncr > 0) bulk_g2s(dst + M.crow, w.comp_row_vec + (size_t)u * ncr * D, 4 * D * ncr, bar);
                    if (ncc > 0) bulk_g2s(dst + M.ccol, w.comp_col_vec + (size_t)u * ncc * D, 4 * D * ncc, bar);
                }
                advance();
                if (u != early_u) {
                    dst = acquire(u, -2);
                    if (dst == nullptr) { fail(); return; }
                    bar = &full[slot];
                    mbar_arrive_expect_tx(bar, D * D);
                    tma_load_2d(dst, &codes_map, 0, u * D, bar);
                }
                advance();
                publish();
                const int nchunks = (n_buf + E - 1) / E;
                for (int c = 0; c < nchunks; ++c) {
                    dst = acquire(u, -3 - c);
                    if (dst == nullptr) { fail(); return; }
                    const int e0 = c * E, ne = min(E, n_buf - e0);
                    const size_t first = (size_t)u * w.window + e0;
                    const uint32_t bd = 4u * ne * D, bk = (uint32_t)sizeof(KeyT) * ne * D;
                    const uint32_t bg = KDA ? 0u : 4u * (uint32_t)align_up(ne, 4);
                    bar = &full[slot];
                    mbar_arrive_expect_tx(bar, bd + bk + bg);
                    bulk_g2s(dst, w.buf_delta + first * D, bd, bar);
                    bulk_g2s(dst + Sh::C_KEY, reinterpret_cast<const KeyT *>(w.buf_key) + first * D, bk, bar);
                    if (!KDA) bulk_g2s(dst + Sh::C_GATE, w.buf_gate + (size_t)u * w.window_pad + e0, bg, bar);
                    advance();
                }
            }
            // the next unit and its scalars (loads in flight until its record)
            int un = -1;
            if (k + 1 < rounds) {
                un = u + grid;
            } else if (draw) {
                const int r = ticket_unit(tk, n_dyn, grid, tickets, w.err);
                if (r >= 0) {
                    un = rounds * grid + r;
                    tk = atomicAdd(tickets, 1ull);
                } else {
                    draw = false;
                }
            }
            u = un;
            if (u >= 0) fetch(u, cur);
        }
        // no unit left: a record that says so
        if (acquire(-1, -5) == nullptr) { fail(); return; }
        stop(slot);
        return;
    }

    // =============================================================== consumers
    int8_t *sB8 = reinterpret_cast<int8_t *>(scr + Sh::S_B8);   // [8][D] digits: y^q d_0..3, y^k d_0..3
    float *sExp = scr + Sh::S_EXP;                              // 2^E per (vector, 32-column block)
    float *sXq = scr + Sh::S_XQ, *sXk = scr + Sh::S_XK, *sQr = scr + Sh::S_QR, *sKr = scr + Sh::S_KR;
    float *sA = scr + Sh::S_A, *sB = scr + Sh::S_B;
    float2 *sCf = reinterpret_cast<float2 *>(scr + Sh::S_CF);
    float *sRed = scr + Sh::S_RED;                              // [warp][kq, row-comp dots]
    const bool owns_row = tid < D;                 // thread i: state row i and key channel i
    // entry dots: 8 lanes per entry; lane s covers channels 32m + 4s + t (m < D/32, t < 4)
    const int dot_s = lane & 7, dot_e = warp * 4 + (lane >> 3);

    int slot = 0;
    uint32_t ph = 0;
    auto advance = [&]() {
        if (++slot == kSlots) { slot = 0; ph ^= 1u; }
    };
    const uint32_t tmem = Sh::TC ? *tmem_slot : 0u;   // lane i = state row i
    uint32_t mph = 0;                                 // phase of the tcgen05 pass barrier
    bool tc_inflight = false;                         // a pass was issued and not yet seen complete
    grid_dependency_wait();                           // the inputs and the buffer may still be in writing
    if (tid == 0) grid_dependents_launch();
    for (;;) {
        // ------------------------------------------------ A1: operand prep
        bool bad = !mbar_wait(&full[slot], ph, kWaitBudgetCycles);
        const UnitRec r = rec[slot];
        if (consumer_sync_or(bad || r.u < 0)) {   // a timeout, or no unit left
            if (bad) report_error(w.err, LQ_DEVERR_TIMEOUT, -1, -6);
            goto consumers_done;
        }
        const int u = r.u;
        const float beta = r.beta;
        const double Gs = r.G;                     // scalar gate: G_t
        const float gam_s = r.gam;                 // scalar gate: gamma_t
        const int n_buf = r.n_buf;
        const int nchunks = (n_buf + E - 1) / E;
        const unsigned char *mp = ring + slot * kSlotBytes;
        const int meta_slot = slot;
        advance();
        double G_j = 0.0;
        float key_out = 0.0f, v_i = 0.0f, sig_i = 0.0f;
        if (owns_row) {
            const int j = tid;
            float gam;
            if (KDA) {
                G_j = reinterpret_cast<const double *>(mp + M.gsum)[j] + (double)reinterpret_cast<const float *>(mp + M.gin)[j];
                gam = exp_of_double(G_j);
            } else {
                gam = gam_s;
            }
            const float qj = to_f32(reinterpret_cast<const InT *>(mp + M.qin)[j]);
            const float kj = to_f32(reinterpret_cast<const InT *>(mp + M.kin)[j]);
            const float sj = reinterpret_cast<const float *>(mp + M.s)[j];
            v_i = to_f32(reinterpret_cast<const InT *>(mp + M.vin)[j]);
            sig_i = reinterpret_cast<const float *>(mp + M.sig)[j];
            const float xq = gam * qj, xk = gam * kj;
            sXq[j] = xq;
            sXk[j] = xk;
            sQr[j] = qj;
            sKr[j] = kj;
            // exact int8 digits of y^q_j and y^k_j with this warp's block exponents
            const float yq = sj * xq, yk = sj * xk;
            // non-negative floats order like their bit patterns: one integer max
            const float2 eq = block_scale(__uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(yq)))));
            const float2 ek = block_scale(__uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(yk)))));
            const uint32_t dq = digits4(yq, eq.x), dk = digits4(yk, ek.x);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                if constexpr (Sh::TC) {            // digit column n is operand row n
                    dig[sw128_off(p, j)] = (unsigned char)((dq >> (8 * p)) & 0xff);
                    dig[sw128_off(4 + p, j)] = (unsigned char)((dk >> (8 * p)) & 0xff);
                } else {
                    sB8[p * D + j] = (int8_t)((dq >> (8 * p)) & 0xff);
                    sB8[(4 + p) * D + j] = (int8_t)((dk >> (8 * p)) & 0xff);
                }
            }
            if (lane == 0) {
                sExp[warp] = eq.y;
                sExp[4 + warp] = ek.y;
            }
            // k_t . q_t and the row compensators' dots k_c . x, reduced per warp
            // (compensator rows 0..3 together with k.q; rows 4..7, when used, after)
            {
                const float *crow = reinterpret_cast<const float *>(mp + M.crow);
                float kq_p = kj * qj;
                float v[8];                        // (k_c . x^k, k_c . x^q) of rows c < 4
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float kc = (c < ncr) ? crow[c * D + j] : 0.0f;
                    v[2 * c] = kc * xk;
                    v[2 * c + 1] = kc * xq;
                }
                // butterfly reduce-scatter: lane l ends with the warp total of value
                // 4*b4 + 2*b3 + b2 (b = bits of l); k.q by a plain 5-level sum
                const bool hi16 = lane & 16, hi8 = lane & 8, hi4 = lane & 4;
                float h4[4], h2[2], s1;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    h4[i] = (hi16 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, hi16 ? v[i] : v[i + 4], 16);
#pragma unroll
                for (int i = 0; i < 2; ++i)
                    h2[i] = (hi8 ? h4[i + 2] : h4[i]) + __shfl_xor_sync(0xffffffffu, hi8 ? h4[i] : h4[i + 2], 8);
                s1 = (hi4 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, hi4 ? h2[0] : h2[1], 4);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
                kq_p = group_sum<32>(kq_p);
                if ((lane & 3) == 0) sRed[warp * Sh::RED + 1 + (hi16 ? 4 : 0) + (hi8 ? 2 : 0) + (hi4 ? 1 : 0)] = s1;
                if (lane == 0) sRed[warp * Sh::RED] = kq_p;
                if (ncr > 4) {
                    float more[8];
#pragma unroll
                    for (int c = 4; c < 8; ++c) {
                        const float kc = (c < ncr) ? crow[c * D + j] : 0.0f;
                        more[2 * (c - 4)] = kc * xk;
                        more[2 * (c - 4) + 1] = kc * xq;
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                        for (int i = 0; i < 8; ++i) more[i] += __shfl_xor_sync(0xffffffffu, more[i], o);
                    if (lane == 0) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) sRed[warp * Sh::RED + 9 + i] = more[i];
                    }
                }
            }
            if (KDA) {
                if (fabs(G_j) > kMaxAbsGateSum) report_error(w.err, LQ_DEVERR_RANGE, u, j);
                key_out = kj * exp_of_double(-G_j);          // kappa_j
            } else {
                key_out = kj;
            }
        }
        if (!KDA && tid == 0 && fabs(Gs) > kMaxAbsGateSum) report_error(w.err, LQ_DEVERR_RANGE, u, -1);
        if constexpr (Sh::TC) {
            fence_proxy_async_smem();              // the digits are read by the tensor cores
            tc_fence_before();                     // this thread's last tensor-memory loads come first
        }
        if (consumer_sync_or(bad)) {
            if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 0);
            goto consumers_done;
        }

        if constexpr (Sh::TC) {
            tc_inflight = true;
            // One thread starts the INT8 pass as soon as the tile is in: per
            // 32-column block kb an M = 128, N = 16, K = 32 s8 product into
            // tensor-memory columns 16 kb ..  It runs under the compensator terms.
            if (tid == 0) {
                bad = !mbar_wait(&full[slot], ph, kWaitBudgetCycles);
                if (bad) report_error(w.err, LQ_DEVERR_TIMEOUT, u, -4);
                tc_fence_after();
                const uint32_t a0 = smem_u32(ring + slot * kSlotBytes), b0 = smem_u32(dig);
#pragma unroll
                for (int kb = 0; kb < KBLK; ++kb) {
                    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                 "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
                                 ::"r"(tmem + (uint32_t)(16 * kb)), "l"(sw128_desc(a0 + 32 * kb)),
                                 "l"(sw128_desc(b0 + 32 * kb)), "r"(kI8Idesc), "r"(0));
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                             ::"r"(smem_u32(mma_bar)) : "memory");
            }
        }

        // kq, this row's compensator contributions (row and column ones)
        float kq = 0.0f;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) kq += sRed[i * Sh::RED];
        float2 acc = make_float2(0.0f, 0.0f);      // (S_{t-1} x^k, S_{t-1} x^q) parts of this row
        if (owns_row && ncomp > 0) {
            const int32_t *cidx = reinterpret_cast<const int32_t *>(mp + M.cidx);
            const float *ccol = reinterpret_cast<const float *>(mp + M.ccol);
            // column compensators, in order: (C x)_i = sum_c v_c[i] x_{j_c}
#pragma unroll 2
            for (int c = 0; c < ncc; ++c) {
                const int jc = cidx[ncr + c] & (D - 1);      // in range whatever the workspace holds
                const float vc = ccol[c * D + tid];
                acc.x = fmaf(vc, sXk[jc], acc.x);
                acc.y = fmaf(vc, sXq[jc], acc.y);
            }
            int rc = -1;                           // this row's slot among the row compensators
            for (int c = 0; c < ncr; ++c)
                if (cidx[c] == tid) rc = c;
            if (rc >= 0) {
#pragma unroll
                for (int i = 0; i < D / 32; ++i) {
                    acc.x += sRed[i * Sh::RED + 1 + 2 * rc];
                    acc.y += sRed[i * Sh::RED + 2 + 2 * rc];
                }
            }
        }
        // this thread's last read of the meta segment: the slot goes back to the
        // producer before the INT8 pass, so the next copy starts that much earlier
        mbar_arrive(&empty[meta_slot]);

        // ---------------------------- A2: one pass over the INT8 tile
        // sum_j Q_ij y^q_j and sum_j Q_ij y^k_j (sigma_i is applied at emit), as
        // exact int8 products on the tensor cores (see the file comment)
        // (with the tensor-core pass, thread 0 waited for the tile; its completion
        // tells every thread the tile is in and read)
        if constexpr (!Sh::TC) bad = !mbar_wait(&full[slot], ph, kWaitBudgetCycles);
        float p8q = 0.0f, p8k = 0.0f;              // TC: this thread's row of the two products
        if constexpr (Sh::TC) {
            if (mbar_wait(mma_bar, mph, kWaitBudgetCycles)) tc_inflight = false;
            else bad = true;
            mph ^= 1u;
            tc_fence_after();
            __syncwarp();
            // digit columns 0..3 belong to y^q, 4..7 to y^k; the digits combine in
            // the order the warp-level pass uses (digits 0, 1 and 2, 3 in two sums)
            float s01q = 0.0f, s23q = 0.0f, s01k = 0.0f, s23k = 0.0f;
#pragma unroll
            for (int kb = 0; kb < KBLK; ++kb) {
                uint32_t r[8];
                asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                             : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                               "=r"(r[7])
                             : "r"(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(16 * kb)));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                const float sq = sExp[kb], sk = sExp[4 + kb];
                s01q = fmaf(sq, fmaf(i2f_exact((int)r[1]), 0x1p-7f, i2f_exact((int)r[0])), s01q);
                s23q = fmaf(sq, fmaf(i2f_exact((int)r[3]), 0x1p-21f, i2f_exact((int)r[2]) * 0x1p-14f), s23q);
                s01k = fmaf(sk, fmaf(i2f_exact((int)r[5]), 0x1p-7f, i2f_exact((int)r[4])), s01k);
                s23k = fmaf(sk, fmaf(i2f_exact((int)r[7]), 0x1p-21f, i2f_exact((int)r[6]) * 0x1p-14f), s23k);
            }
            p8q = s01q + s23q;
            p8k = s01k + s23k;
        } else {
            const unsigned char *tile = ring + slot * kSlotBytes;
            const int g = lane >> 2, c4 = lane & 3;
            uint32_t bf[KBLK][2];                  // B fragments: digit column g, k = 4*c4 (+16)
#pragma unroll
            for (int kb = 0; kb < KBLK; ++kb) {
                bf[kb][0] = *reinterpret_cast<const uint32_t *>(sB8 + g * D + kb * 32 + 4 * c4);
                bf[kb][1] = *reinterpret_cast<const uint32_t *>(sB8 + g * D + kb * 32 + 16 + 4 * c4);
            }
            // this lane's digit columns: 2*c4 and 2*c4+1, i.e. vector c4/2, digits 2*(c4&1) and +1
            const float w0 = (c4 & 1) ? 0x1p-14f : 1.0f, w1 = w0 * 0x1p-7f;
            float scale[KBLK];
#pragma unroll
            for (int kb = 0; kb < KBLK; ++kb) scale[kb] = sExp[(c4 >> 1) * 4 + kb];
            const uint32_t tile_s = smem_u32(tile);
            const int q = lane >> 3, rr = lane & 7;   // ldmatrix: matrix q, row rr within it
            uint32_t af[MT][KBLK][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int kb = 0; kb < KBLK; ++kb)
                    ldmatrix_x4(tile_s + swz<D>((warp * MT + mt) * 16 + (q & 1) * 8 + rr, kb * 2 + (q >> 1)),
                                af[mt][kb][0], af[mt][kb][1], af[mt][kb][2], af[mt][kb][3]);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int m0 = (warp * MT + mt) * 16;
                float v0 = 0.0f, v1 = 0.0f;        // rows m0 + g and m0 + g + 8
#pragma unroll
                for (int kb = 0; kb < KBLK; ++kb) {
                    int acc4[4] = {0, 0, 0, 0};
                    mma_s8(acc4, af[mt][kb][0], af[mt][kb][1], af[mt][kb][2], af[mt][kb][3], bf[kb][0], bf[kb][1]);
                    v0 = fmaf(scale[kb], fmaf(i2f_exact(acc4[1]), w1, i2f_exact(acc4[0]) * w0), v0);
                    v1 = fmaf(scale[kb], fmaf(i2f_exact(acc4[3]), w1, i2f_exact(acc4[2]) * w0), v1);
                }
                v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
                v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
                if ((c4 & 1) == 0) {
                    float *dst = (c4 == 0) ? sA : sB;
                    dst[m0 + g] = v0;
                    dst[m0 + g + 8] = v1;
                }
            }
        }
        mbar_arrive(&empty[slot]);                 // done with the INT8 tile
        advance();

        // ------------------------------------------- A3: buffered entries
        for (int c = 0; c < nchunks; ++c) {
            bad |= !mbar_wait(&full[slot], ph, kWaitBudgetCycles);
            const unsigned char *cp = ring + slot * kSlotBytes;
            const float *sDelta = reinterpret_cast<const float *>(cp);
            const KeyT *sKey = reinterpret_cast<const KeyT *>(cp + Sh::C_KEY);
            const float *sOmega = reinterpret_cast<const float *>(cp + Sh::C_GATE);
            const int ne = min(E, n_buf - c * E);
            float2 *cf = sCf + (c & 1) * 16;
            // coefficients kappa_e . (x^k, x^q): 8 lanes per entry, 3-level reduction;
            // every lane takes part in the shuffles, lanes past the chunk with zeros
            {
                const bool live_e = dot_e < ne;
                const float *xk = KDA ? sXk : sKr, *xq = KDA ? sXq : sQr;
                float dk0 = 0.0f, dk1 = 0.0f, dq0 = 0.0f, dq1 = 0.0f;
#pragma unroll
                for (int m = 0; m < D / 32 && live_e; ++m) {
                    const int j0 = 32 * m + 4 * dot_s;
                    float kv[4];
                    load_key<KeyT, 4>(sKey + dot_e * D + j0, kv);
                    const float4 a4 = *reinterpret_cast<const float4 *>(xk + j0);
                    const float4 b4 = *reinterpret_cast<const float4 *>(xq + j0);
                    dk0 = fmaf(kv[0], a4.x, dk0); dk1 = fmaf(kv[1], a4.y, dk1);
                    dk0 = fmaf(kv[2], a4.z, dk0); dk1 = fmaf(kv[3], a4.w, dk1);
                    dq0 = fmaf(kv[0], b4.x, dq0); dq1 = fmaf(kv[1], b4.y, dq1);
                    dq0 = fmaf(kv[2], b4.z, dq0); dq1 = fmaf(kv[3], b4.w, dq1);
                }
                float dk = dk0 + dk1, dq = dq0 + dq1;
#pragma unroll
                for (int o = 4; o > 0; o >>= 1) {
                    dk += __shfl_xor_sync(0xffffffffu, dk, o);
                    dq += __shfl_xor_sync(0xffffffffu, dq, o);
                }
                if (live_e && dot_s == 0) {
                    const float f = KDA ? 1.0f : gam_s * sOmega[dot_e];
                    cf[dot_e] = make_float2(f * dk, f * dq);
                }
            }
            if (consumer_sync_or(bad)) {
                if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 1 + c);
                goto consumers_done;
            }
            if (owns_row) {
                float2 p[4] = {acc, make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
                for (int el = 0; el < E; ++el) {
                    const bool live = el < ne;
                    const float d0 = live ? sDelta[el * D + tid] : 0.0f;
                    const float2 cc = live ? cf[el] : make_float2(0.0f, 0.0f);
                    p[el & 3] = __ffma2_rn(make_float2(d0, d0), cc, p[el & 3]);
                }
                acc.x = (p[0].x + p[1].x) + (p[2].x + p[3].x);
                acc.y = (p[0].y + p[1].y) + (p[2].y + p[3].y);
            }
            mbar_arrive(&empty[slot]);             // done with this chunk
            advance();
        }
        if (nchunks == 0 && consumer_sync_or(bad)) {
            if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 0);
            goto consumers_done;
        }

        // ------------------------------------------------ A4: emit and append
        if (owns_row && in_bounds(w.err, n_buf, 0, w.window, u, -12)) {
            const int i = tid;
            // sigma_i times the INT8 products, rounded before the sum as a product of its own
            const float pk = Sh::TC ? p8k : sB[i], pq = Sh::TC ? p8q : sA[i];
            const float sk = acc.x + __fmul_rn(sig_i, pk), so = acc.y + __fmul_rn(sig_i, pq);
            const float delta = beta * (v_i - sk);
            const size_t slot_g = (size_t)u * w.window + n_buf;
            a.o[(size_t)u * D + i] = fmaf(delta, kq, so);
            w.buf_delta[slot_g * D + i] = delta;
            if (KDA) {
                reinterpret_cast<float *>(w.buf_key)[slot_g * D + i] = key_out;
                w.gate_sum[(size_t)u * D + i] = G_j;
            } else {
                reinterpret_cast<KeyT *>(w.buf_key)[slot_g * D + i] = static_cast<KeyT>(key_out);
            }
        }
        // one-thread bookkeeping on lanes of different warps, so that no warp
        // carries all of it into the next unit's barrier
        if (!KDA && tid == 32) {
            w.buf_gate[(size_t)u * w.window_pad + n_buf] = exp_of_double(-Gs);
            w.gate_sum[u] = Gs;
        }
        if (RAGGED && tid == 64) a.fill[u] = n_buf + 1;
    }
consumers_done:
    // every consumer warp gets here (normal end, or a timeout all of them saw at
    // the same barrier).  After a timeout a tensor-core pass may still be in
    // flight: wait for it (bounded) before the tensor memory goes back, once
    // all warps' loads are done.
    if constexpr (Sh::TC) {
        if (tc_inflight) mbar_wait(mma_bar, mph ^ 1u, kWaitBudgetCycles);
        tc_fence_before();
        asm volatile("bar.sync %0, %1;" ::"r"(kConsumerBarrier), "r"(kConsumers) : "memory");
        tc_fence_after();
        if (warp == 0)
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

template <int D, bool KDA, typename InT, typename KeyT, bool RAGGED, bool TCP>
cudaError_t launch_r(const DecodeArgs &a, cudaStream_t s) {
    using Sh = Shape<D, KDA, InT, KeyT, TCP>;
    const Meta M = meta_layout<D, KDA, InT>(a.w.n_comp_rows, a.w.n_comp_cols, a.w.comp_index_stride);
    if (M.bytes > kSlotBytes || D * D > kSlotBytes) return cudaErrorInvalidValue;
    auto kern = decode_window_kernel<D, KDA, InT, KeyT, RAGGED, TCP>;
    // The opt-in shared-memory size is set once per device, so that launches
    // inside a stream capture make no attribute calls.
    const cudaError_t e = opt_in_smem<decode_window_kernel<D, KDA, InT, KeyT, RAGGED, TCP>>(Sh::SMEM);
    if (e != cudaSuccess) return e;
    // A programmatic dependent of the previous kernel in the stream: the CTAs
    // set up (barriers, tensor memory, the first code tile) while it finishes.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(min(a.w.units, kCtasPerSm * sm_count()));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Sh::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, *reinterpret_cast<const CUtensorMap *>(a.codes_map));
}

// Shared window phases compile without the per-unit counts and the active mask.
// The tensor-core pass pays a tensor-memory allocation per CTA and a commit
// round trip per unit; it is the faster one once the CTAs walk two units or
// more each (measured: 1-5 % faster from 2048 units, up to 16 % slower at one
// unit per CTA).  Both passes give the same sums.
template <int D, bool KDA, typename InT, typename KeyT, bool RAGGED>
cudaError_t launch_p(const DecodeArgs &a, cudaStream_t s) {
    if constexpr (D == 128) {
        if (a.w.units >= 2 * kCtasPerSm * sm_count()) return launch_r<D, KDA, InT, KeyT, RAGGED, true>(a, s);
    }
    return launch_r<D, KDA, InT, KeyT, RAGGED, false>(a, s);
}

template <int D, bool KDA, typename InT, typename KeyT>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    return a.fill != nullptr ? launch_p<D, KDA, InT, KeyT, true>(a, s) : launch_p<D, KDA, InT, KeyT, false>(a, s);
}

}  // namespace

cudaError_t make_codes_map(void *map_out, const int8_t *codes, int d, int units) {
    // the driver's entry point, looked up once (first callers serialized)
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> entry{nullptr};
    static std::mutex lookup;
    PFN_cuTensorMapEncodeTiled_v12000 encode = entry.load(std::memory_order_acquire);
    if (encode == nullptr) {
        std::lock_guard<std::mutex> lock(lookup);
        encode = entry.load(std::memory_order_relaxed);
        if (encode == nullptr) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
            if (e != cudaSuccess) return e;
            if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
            encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            entry.store(encode, std::memory_order_release);
        }
    }
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)units * (cuuint64_t)d};
    const cuuint64_t strides[1] = {(cuuint64_t)d};
    const cuuint32_t box[2] = {(cuuint32_t)d, (cuuint32_t)d};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(reinterpret_cast<CUtensorMap *>(map_out), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                              const_cast<int8_t *>(codes), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_decode_window(const DecodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s) {
    const bool kda = (gate == LQ_GATE_CHANNEL);
    const bool bf = (in_dtype == LQ_DTYPE_BF16);
    if (d == 128) {
        if (kda) return bf ? launch_t<128, true, __nv_bfloat16, float>(a, s) : launch_t<128, true, float, float>(a, s);
        return bf ? launch_t<128, false, __nv_bfloat16, __nv_bfloat16>(a, s) : launch_t<128, false, float, float>(a, s);
    }
    if (d == 64) {
        if (kda) return bf ? launch_t<64, true, __nv_bfloat16, float>(a, s) : launch_t<64, true, float, float>(a, s);
        return bf ? launch_t<64, false, __nv_bfloat16, __nv_bfloat16>(a, s) : launch_t<64, false, float, float>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lq
