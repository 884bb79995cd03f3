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
// where S~ = sigma Q s + C is the window-start state and kappa_j = k_j/gamma_j
// (for the scalar gate kappa_j . x^k is evaluated as exp(G_t - G_j)(k_j . k_t)
// so that raw keys can be buffered).  The step reads the INT8 tile once,
// forms both products S~ x^q and S~ x^k in that pass, adds the
// O((n_c + n_buf) d) corrections and appends (delta_t, key_t, G_t) to the
// buffer.  It writes no state.
//
// Persistent and warp-specialized: a grid of two CTAs per SM walks the
// (sequence, head) units.  In each CTA one producer thread streams every
// unit's data with 1-D bulk async copies through a ring of three 32 KB
// shared-memory slots -- first a header segment (INT8 tile, row scales,
// smoothing factors, q/k/v, compensators), then the buffered entries in
// chunks -- each slot guarded by a full/empty mbarrier pair, so the next
// unit's bytes are in flight while eight consumer warps compute on the
// current one.  The INT8 tile is widened with an exact exponent-bias trick
// and accumulated with packed FP32 FMAs.  Every wait is bounded; an expired
// wait records LQ_DEVERR_TIMEOUT and all consumer warps leave together.
#include "lq_kernels.h"

namespace lq {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kConsumers + 32;     // + one producer warp
constexpr int kSlotBytes = 32768;
constexpr int kSlots = 3;
constexpr int kCtasPerSm = 2;
constexpr int kConsumerBarrier = 1;           // named barrier of the consumer warps
constexpr float kMaxAbsGateSum = 80.0f;

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

template <int D, bool KDA, typename InT, typename KeyT>
struct Shape {
    static constexpr int KB = (int)sizeof(KeyT);
    static constexpr int ENTRY = 4 * D + KB * D + (KDA ? 0 : 8);   // bytes per buffered entry
    static constexpr int E0 = (kSlotBytes / ENTRY) & ~7;
    static constexpr int E = E0 < 32 ? E0 : 32;                   // entries per chunk segment
    static constexpr int C_KEY = 4 * D * E;                        // chunk: deltas, keys, G_j
    static constexpr int C_GATE = C_KEY + KB * D * E;
    static constexpr int LPR = D / 16;                             // lanes per INT8 row
    static constexpr int RPW = 32 / LPR;                           // rows per warp per round
    static constexpr int ROUNDS = D / (kConsumerWarps * RPW);
    static constexpr int VPL = D / 32;                             // key elements per lane
    static constexpr int NH = kConsumers / D;                      // threads per state row
    // consumer scratch after the ring (floats)
    static constexpr int S_XQ = 0, S_XK = D, S_YQ = 2 * D, S_YK = 3 * D, S_QR = 4 * D, S_KR = 5 * D,
                         S_V = 6 * D, S_A = 7 * D, S_B = 8 * D, S_EX = 9 * D, S_CK = 9 * D + 2 * (NH - 1) * D,
                         S_CQ = S_CK + 32, S_RCK = S_CQ + 32, S_RCQ = S_RCK + 8, S_RED = S_RCQ + 8,
                         S_FLOATS = S_RED + 8;
    static constexpr int SMEM = 128 + kSlots * kSlotBytes + 4 * S_FLOATS;
    static_assert(E >= 8, "chunk too small");
    static_assert(ROUNDS >= 1, "row rounds");
};

// Offsets inside a header segment.
struct Header {
    int q, sig, s, qin, kin, vin, gin, gsum, cidx, crow, ccol, bytes;
};

template <int D, bool KDA, typename InT>
__host__ __device__ Header header_layout(int ncr, int ncc, int cis) {
    Header h{};
    int o = 0;
    h.q = o;    o += D * D;
    h.sig = o;  o += 4 * D;
    h.s = o;    o += 4 * D;
    h.qin = o;  o += (int)sizeof(InT) * D;
    h.kin = o;  o += (int)sizeof(InT) * D;
    h.vin = o;  o += (int)sizeof(InT) * D;
    h.gin = o;  o += KDA ? 4 * D : 0;
    h.gsum = o; o += KDA ? 8 * D : 0;
    h.cidx = o; o += (ncr + ncc) > 0 ? 4 * cis : 0;
    h.crow = o; o += 4 * D * ncr;
    h.ccol = o; o += 4 * D * ncc;
    h.bytes = o;
    return h;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x) { return static_cast<float>(x); }
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }

template <typename KeyT, int VPL>
__device__ __forceinline__ void load_key(const KeyT *p, float (&out)[VPL]) {
    if constexpr (sizeof(KeyT) == 2) {
        if constexpr (VPL == 4) {
            uint2 w = *reinterpret_cast<const uint2 *>(p);
            out[0] = bf16_bits_to_f32(w.x & 0xffffu); out[1] = bf16_bits_to_f32(w.x >> 16);
            out[2] = bf16_bits_to_f32(w.y & 0xffffu); out[3] = bf16_bits_to_f32(w.y >> 16);
        } else {
            uint32_t w = *reinterpret_cast<const uint32_t *>(p);
            out[0] = bf16_bits_to_f32(w & 0xffffu); out[1] = bf16_bits_to_f32(w >> 16);
        }
    } else {
        if constexpr (VPL == 4) {
            float4 w = *reinterpret_cast<const float4 *>(p);
            out[0] = w.x; out[1] = w.y; out[2] = w.z; out[3] = w.w;
        } else {
            float2 w = *reinterpret_cast<const float2 *>(p);
            out[0] = w.x; out[1] = w.y;
        }
    }
}

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync %0, %1;" ::"r"(kConsumerBarrier), "r"(kConsumers) : "memory");
}

// Consumer barrier that also ORs a predicate over the consumer threads.
__device__ __forceinline__ bool consumer_sync_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(kConsumerBarrier), "r"(kConsumers)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Two int8 codes (bytes b, b+1 of word u, already offset by 128) as exact floats.
__device__ __forceinline__ float2 i8pair(uint32_t u, uint32_t sel_lo, uint32_t sel_hi) {
    const float2 biased = make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, sel_lo)),
                                      __uint_as_float(__byte_perm(u, 0x4B000000u, sel_hi)));
    return __fadd2_rn(biased, make_float2(-8388736.0f, -8388736.0f));   // minus (2^23 + 128)
}

template <int D, bool KDA, typename InT, typename KeyT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_window_kernel(DecodeArgs a) {
    using Sh = Shape<D, KDA, InT, KeyT>;
    constexpr int E = Sh::E, LPR = Sh::LPR, RPW = Sh::RPW, ROUNDS = Sh::ROUNDS, VPL = Sh::VPL, NH = Sh::NH;
    const Views &w = a.w;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ncr = w.n_comp_rows, ncc = w.n_comp_cols, cis = w.comp_index_stride, ncomp = ncr + ncc;
    const int n_buf = a.n_buf, nchunks = (n_buf + E - 1) / E, units = w.units;
    const Header H = header_layout<D, KDA, InT>(ncr, ncc, cis);

    extern __shared__ __align__(128) unsigned char sm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(sm);
    uint64_t *empty = full + kSlots;
    unsigned char *ring = sm + 128;
    float *scr = reinterpret_cast<float *>(ring + kSlots * kSlotBytes);

    if (tid == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // ================================================================ producer
    if (warp == kConsumerWarps) {
        if (lane != 0) return;
        const uint64_t stream_once = l2_policy_evict_first();
        const uint32_t in_b = (uint32_t)sizeof(InT) * D;
        int slot = 0;
        uint32_t ph = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            if (!mbar_wait(&empty[slot], ph ^ 1u, kWaitBudgetCycles)) {
                report_error(w.err, LQ_DEVERR_TIMEOUT, u, -1);
                return;
            }
            unsigned char *dst = ring + slot * kSlotBytes;
            uint64_t *bar = &full[slot];
            mbar_arrive_expect_tx(bar, (uint32_t)H.bytes);
            bulk_g2s_stream(dst + H.q, w.codes + (size_t)u * D * D, D * D, bar, stream_once);
            bulk_g2s(dst + H.sig, w.row_scale + (size_t)u * D, 4 * D, bar);
            bulk_g2s(dst + H.s, w.col_smooth + (size_t)u * D, 4 * D, bar);
            bulk_g2s(dst + H.qin, reinterpret_cast<const InT *>(a.q) + (size_t)u * D, in_b, bar);
            bulk_g2s(dst + H.kin, reinterpret_cast<const InT *>(a.k) + (size_t)u * D, in_b, bar);
            bulk_g2s(dst + H.vin, reinterpret_cast<const InT *>(a.v) + (size_t)u * D, in_b, bar);
            if (KDA) {
                bulk_g2s(dst + H.gin, a.g + (size_t)u * D, 4 * D, bar);
                bulk_g2s(dst + H.gsum, w.gate_sum + (size_t)u * D, 8 * D, bar);
            }
            if (ncomp > 0) {
                bulk_g2s(dst + H.cidx, w.comp_index + (size_t)u * cis, 4 * cis, bar);
                if (ncr > 0) bulk_g2s(dst + H.crow, w.comp_row_vec + (size_t)u * ncr * D, 4 * D * ncr, bar);
                if (ncc > 0) bulk_g2s(dst + H.ccol, w.comp_col_vec + (size_t)u * ncc * D, 4 * D * ncc, bar);
            }
            if (++slot == kSlots) { slot = 0; ph ^= 1u; }
            for (int c = 0; c < nchunks; ++c) {
                if (!mbar_wait(&empty[slot], ph ^ 1u, kWaitBudgetCycles)) {
                    report_error(w.err, LQ_DEVERR_TIMEOUT, u, -2 - c);
                    return;
                }
                const int e0 = c * E, ne = min(E, n_buf - e0);
                const size_t first = (size_t)u * w.window + e0;
                const uint32_t bd = 4u * ne * D, bk = (uint32_t)sizeof(KeyT) * ne * D;
                const uint32_t bg = KDA ? 0u : 8u * (uint32_t)align_up(ne, 2);
                dst = ring + slot * kSlotBytes;
                bar = &full[slot];
                mbar_arrive_expect_tx(bar, bd + bk + bg);
                bulk_g2s(dst, w.buf_delta + first * D, bd, bar);
                bulk_g2s(dst + Sh::C_KEY, reinterpret_cast<const KeyT *>(w.buf_key) + first * D, bk, bar);
                if (!KDA) bulk_g2s(dst + Sh::C_GATE, w.buf_gate + (size_t)u * w.window_pad + e0, bg, bar);
                if (++slot == kSlots) { slot = 0; ph ^= 1u; }
            }
        }
        return;
    }

    // =============================================================== consumers
    float *sXq = scr + Sh::S_XQ, *sXk = scr + Sh::S_XK, *sYq = scr + Sh::S_YQ, *sYk = scr + Sh::S_YK;
    float *sQr = scr + Sh::S_QR, *sKr = scr + Sh::S_KR, *sV = scr + Sh::S_V;
    float *sA = scr + Sh::S_A, *sB = scr + Sh::S_B, *sEx = scr + Sh::S_EX;
    float *sCk = scr + Sh::S_CK, *sCq = scr + Sh::S_CQ, *sRck = scr + Sh::S_RCK, *sRcq = scr + Sh::S_RCQ;
    float *sRed = scr + Sh::S_RED;
    const int row = tid % D, part = tid / D;      // state row this thread accumulates, and which share

    int slot = 0;
    uint32_t ph = 0;
    int u = blockIdx.x;
    float beta_n = 0.0f, g_n = 0.0f;
    double G_n = 0.0;
    if (u < units) {
        beta_n = a.beta[u];
        if (!KDA) { g_n = a.g[u]; G_n = w.gate_sum[u]; }
    }
    for (; u < units; u += gridDim.x) {
        const float beta = beta_n;
        const double Gt_s = KDA ? 0.0 : G_n + (double)g_n;
        const int un = u + gridDim.x;
        if (un < units) {                          // next unit's scalars, in flight meanwhile
            beta_n = a.beta[un];
            if (!KDA) { g_n = a.g[un]; G_n = w.gate_sum[un]; }
        }

        // ---------------------------------------------------- header segment
        bool ok = mbar_wait(&full[slot], ph, kWaitBudgetCycles);
        const unsigned char *hp = ring + slot * kSlotBytes;
        double Gt_j = 0.0;
        float kappa_j = 0.0f, kq = 0.0f;
        if (ok && tid < D) {                       // A1: gate and operand prep, one key channel each
            const int j = tid;
            float gam;
            if (KDA) {
                Gt_j = reinterpret_cast<const double *>(hp + H.gsum)[j] + (double)reinterpret_cast<const float *>(hp + H.gin)[j];
                gam = (float)exp(Gt_j);
                if (fabs(Gt_j) > (double)kMaxAbsGateSum) report_error(w.err, LQ_DEVERR_RANGE, u, j);
            } else {
                gam = (float)exp(Gt_s);
            }
            const float qj = to_f32(reinterpret_cast<const InT *>(hp + H.qin)[j]);
            const float kj = to_f32(reinterpret_cast<const InT *>(hp + H.kin)[j]);
            const float sj = reinterpret_cast<const float *>(hp + H.s)[j];
            const float xq = gam * qj, xk = gam * kj;
            sXq[j] = xq;
            sXk[j] = xk;
            sYq[j] = sj * xq;
            sYk[j] = sj * xk;
            sQr[j] = qj;
            sKr[j] = kj;
            sV[j] = to_f32(reinterpret_cast<const InT *>(hp + H.vin)[j]);
            kq = kj * qj;
            if (KDA) kappa_j = kj * (float)exp(-Gt_j);
        }
        kq = group_sum<32>(kq);
        if (lane == 0) sRed[warp] = kq;
        if (consumer_sync_or(!ok)) {
            if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 0);
            return;
        }

        // A2: one pass over the INT8 tile: a = sigma (Q (s x^q)), b = sigma (Q (s x^k))
        {
            const int8_t *sQ = reinterpret_cast<const int8_t *>(hp + H.q);
            const float *sSig = reinterpret_cast<const float *>(hp + H.sig);
            const int cb = lane % LPR, rsub = lane / LPR;
            float2 yq[8], yk[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                yq[m] = *reinterpret_cast<const float2 *>(sYq + cb * 16 + 2 * m);
                yk[m] = *reinterpret_cast<const float2 *>(sYk + cb * 16 + 2 * m);
            }
            uint4 qw[ROUNDS];
#pragma unroll
            for (int r = 0; r < ROUNDS; ++r) {
                const int i = r * (kConsumerWarps * RPW) + warp * RPW + rsub;
                qw[r] = *reinterpret_cast<const uint4 *>(sQ + i * D + cb * 16);
            }
#pragma unroll
            for (int r = 0; r < ROUNDS; ++r) {
                const int i = r * (kConsumerWarps * RPW) + warp * RPW + rsub;
                const uint32_t words[4] = {qw[r].x ^ 0x80808080u, qw[r].y ^ 0x80808080u, qw[r].z ^ 0x80808080u,
                                           qw[r].w ^ 0x80808080u};
                float2 pa = make_float2(0.0f, 0.0f), pb = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 f01 = i8pair(words[h], 0x7540, 0x7541);
                    const float2 f23 = i8pair(words[h], 0x7542, 0x7543);
                    pa = __ffma2_rn(f01, yq[2 * h], pa);
                    pb = __ffma2_rn(f01, yk[2 * h], pb);
                    pa = __ffma2_rn(f23, yq[2 * h + 1], pa);
                    pb = __ffma2_rn(f23, yk[2 * h + 1], pb);
                }
                float sa = group_sum<LPR>(pa.x + pa.y);
                float sb = group_sum<LPR>(pb.x + pb.y);
                if (cb == 0) {
                    sA[i] = sSig[i] * sa;
                    sB[i] = sSig[i] * sb;
                }
            }
        }
        // row compensators: k_c . x, one warp each
        for (int c = warp; c < ncr; c += kConsumerWarps) {
            const float *kc = reinterpret_cast<const float *>(hp + H.crow) + c * D;
            float dk = 0.0f, dq = 0.0f;
            for (int j = lane; j < D; j += 32) {
                dk = fmaf(kc[j], sXk[j], dk);
                dq = fmaf(kc[j], sXq[j], dq);
            }
            dk = group_sum<32>(dk);
            dq = group_sum<32>(dq);
            if (lane == 0) { sRck[c] = dk; sRcq[c] = dq; }
        }
        consumer_sync();

        // A3 (start): the dequantized products and the compensators of this row
        float acc_k = 0.0f, acc_q = 0.0f;
        if (part == 0) {
            acc_k = sB[row];
            acc_q = sA[row];
            if (ncomp > 0) {
                const int32_t *cidx = reinterpret_cast<const int32_t *>(hp + H.cidx);
                const float *ccol = reinterpret_cast<const float *>(hp + H.ccol);
                for (int c = 0; c < ncr; ++c)
                    if (cidx[c] == row) { acc_k += sRck[c]; acc_q += sRcq[c]; }
                for (int c = 0; c < ncc; ++c) {
                    const int j = cidx[ncr + c];
                    const float vc = ccol[c * D + row];
                    acc_k = fmaf(vc, sXk[j], acc_k);
                    acc_q = fmaf(vc, sXq[j], acc_q);
                }
            }
        }
        float xs_k[VPL], xs_q[VPL];
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            xs_k[v] = KDA ? sXk[lane * VPL + v] : sKr[lane * VPL + v];
            xs_q[v] = KDA ? sXq[lane * VPL + v] : sQr[lane * VPL + v];
        }
        kq = 0.0f;
#pragma unroll
        for (int i = 0; i < kConsumerWarps; ++i) kq += sRed[i];
        const float v_row = sV[row];
        float k_keep = 0.0f;
        if (!KDA && tid < D) k_keep = sKr[tid];
        consumer_sync();                           // header fully read
        if (tid == 0) mbar_arrive(&empty[slot]);
        if (++slot == kSlots) { slot = 0; ph ^= 1u; }

        // ------------------------------------------------ A3: buffered entries
        for (int c = 0; c < nchunks; ++c) {
            ok = mbar_wait(&full[slot], ph, kWaitBudgetCycles);
            const unsigned char *cp = ring + slot * kSlotBytes;
            const float *sDelta = reinterpret_cast<const float *>(cp);
            const KeyT *sKey = reinterpret_cast<const KeyT *>(cp + Sh::C_KEY);
            const double *sGate = reinterpret_cast<const double *>(cp + Sh::C_GATE);
            const int ne = min(E, n_buf - c * E);
            if (ok) {
                constexpr int PER = (E + kConsumerWarps - 1) / kConsumerWarps;
                float dk[PER], dq[PER];
#pragma unroll
                for (int r = 0; r < PER; ++r) {
                    const int el = warp + r * kConsumerWarps;
                    dk[r] = 0.0f;
                    dq[r] = 0.0f;
                    if (el < ne) {
                        float kv[VPL];
                        load_key<KeyT, VPL>(sKey + el * D + lane * VPL, kv);
#pragma unroll
                        for (int v = 0; v < VPL; ++v) {
                            dk[r] = fmaf(kv[v], xs_k[v], dk[r]);
                            dq[r] = fmaf(kv[v], xs_q[v], dq[r]);
                        }
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                    for (int r = 0; r < PER; ++r) {
                        dk[r] += __shfl_xor_sync(0xffffffffu, dk[r], o);
                        dq[r] += __shfl_xor_sync(0xffffffffu, dq[r], o);
                    }
                }
#pragma unroll
                for (int r = 0; r < PER; ++r) {
                    const int el = warp + r * kConsumerWarps;
                    if (lane == r && el < ne) {
                        const float f = KDA ? 1.0f : (float)exp(Gt_s - sGate[el]);
                        sCk[el] = f * dk[r];
                        sCq[el] = f * dq[r];
                    }
                }
            }
            if (consumer_sync_or(!ok)) {
                if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 1 + c);
                return;
            }
            float ak2 = 0.0f, aq2 = 0.0f;
            int el = part;
            for (; el + NH < ne; el += 2 * NH) {
                const float d0 = sDelta[el * D + row], d1 = sDelta[(el + NH) * D + row];
                acc_k = fmaf(sCk[el], d0, acc_k);
                acc_q = fmaf(sCq[el], d0, acc_q);
                ak2 = fmaf(sCk[el + NH], d1, ak2);
                aq2 = fmaf(sCq[el + NH], d1, aq2);
            }
            if (el < ne) {
                const float d0 = sDelta[el * D + row];
                acc_k = fmaf(sCk[el], d0, acc_k);
                acc_q = fmaf(sCq[el], d0, acc_q);
            }
            acc_k += ak2;
            acc_q += aq2;
            consumer_sync();                       // chunk fully read
            if (tid == 0) mbar_arrive(&empty[slot]);
            if (++slot == kSlots) { slot = 0; ph ^= 1u; }
        }

        // ------------------------------------------------- A4: emit and append
        if (part > 0) {
            sEx[(part - 1) * 2 * D + row] = acc_k;
            sEx[(part - 1) * 2 * D + D + row] = acc_q;
        }
        consumer_sync();
        const size_t slot_g = (size_t)u * w.window + n_buf;
        if (part == 0) {
#pragma unroll
            for (int p = 1; p < NH; ++p) {
                acc_k += sEx[(p - 1) * 2 * D + row];
                acc_q += sEx[(p - 1) * 2 * D + D + row];
            }
            const float delta = beta * (v_row - acc_k);
            a.o[(size_t)u * D + row] = fmaf(delta, kq, acc_q);
            w.buf_delta[slot_g * D + row] = delta;
        }
        if (tid < D) {
            if (KDA) {
                reinterpret_cast<float *>(w.buf_key)[slot_g * D + tid] = kappa_j;
                w.gate_sum[(size_t)u * D + tid] = Gt_j;
            } else {
                reinterpret_cast<KeyT *>(w.buf_key)[slot_g * D + tid] = static_cast<KeyT>(k_keep);
            }
        }
        if (!KDA && tid == 0) {
            w.buf_gate[(size_t)u * w.window_pad + n_buf] = Gt_s;
            w.gate_sum[u] = Gt_s;
        }
    }
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

template <int D, bool KDA, typename InT, typename KeyT>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    using Sh = Shape<D, KDA, InT, KeyT>;
    const Header H = header_layout<D, KDA, InT>(a.w.n_comp_rows, a.w.n_comp_cols, a.w.comp_index_stride);
    if (H.bytes > kSlotBytes) return cudaErrorInvalidValue;
    auto kern = decode_window_kernel<D, KDA, InT, KeyT>;
    // The opt-in shared-memory size is set once per device, so that launches
    // inside a stream capture make no attribute calls.
    static bool opted_in[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !opted_in[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::SMEM);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) opted_in[dev] = true;
    }
    const int grid = min(a.w.units, kCtasPerSm * sm_count());
    kern<<<grid, kThreads, Sh::SMEM, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

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
