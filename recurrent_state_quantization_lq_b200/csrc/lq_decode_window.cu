// Windowed INT8 decode step (the hot path).
//
// LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent
// State Quantization", section "Abstract (arXiv)"): within a window, outputs
// are computed from the fixed low-bit state together with high-precision
// buffered updates, and Compensator Tokens share the update path of real
// tokens.  With G_t the log-gate summed since the window start,
// gamma_t = exp(G_t), x^q = gamma_t * q_t and x^k = gamma_t * k_t:
//   S_{t-1}(alpha_t * k_t) = S~ x^k + sum_{j<t} delta_j (kappa_j . x^k)
//   delta_t = beta_t (v_t - S_{t-1}(alpha_t * k_t))
//   o_t     = S~ x^q + sum_{j<t} delta_j (kappa_j . x^q) + delta_t (k_t . q_t)
// where S~ = sigma Q s + C is the window-start state and kappa_j = k_j/gamma_j
// (for the scalar gate kappa_j . x = exp(G_t - G_j)(k_j . x / gamma_t) is
// evaluated as exp(G_t - G_j)(k_j . k_t) so raw keys can be buffered).  The
// step reads the INT8 tile once, computes both products S~ x^q and S~ x^k in
// that one pass, adds the O((n_c + n_buf) d) corrections and appends
// (delta_t, key_t, G_t) to the buffer.  It writes no state.
//
// One CTA per (sequence, head).  Thread 0 streams the unit's data into
// shared memory with 1-D bulk async copies: a header (INT8 tile, scales,
// smoothing factors, q/k/v, compensators) on one mbarrier and the buffered
// entries in chunks of 16 through a ring of slots, each on its own mbarrier.
// All waits are bounded; an expired wait records LQ_DEVERR_TIMEOUT and the
// CTA returns.
#include "lq_kernels.h"

namespace lq {
namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 16;      // buffered entries per ring slot
constexpr float kMaxAbsGateSum = 80.0f;

struct DecLayout {
    int bars, q, sig, s, qin, kin, vin, gin, gsum, cidx, crow, ccol;
    int ring, slot_bytes, slot_delta, slot_key, slot_gate;
    int xq, xk, yq, yk, qk_raw, a, b, coef_k, coef_q, fac, rc_k, rc_q, red;
    int total;
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

template <int D, bool KDA, typename InT, typename KeyT>
struct DecShape {
    static constexpr int NS = KDA ? 2 : 3;     // ring slots
    static constexpr int LPR = D / 16;         // lanes per INT8 row (16 codes per lane)
    static constexpr int RPW = 32 / LPR;       // rows per warp per step
    static constexpr int VPL = D / 32;         // key elements per lane in the entry dots

    __host__ __device__ static DecLayout layout(int ncr, int ncc, int cis) {
        DecLayout L{};
        int o = 0;
        L.bars = o;   o += 8 * (1 + NS);
        o = align_up(o, 128);
        L.q = o;      o += D * D;
        L.sig = o;    o += 4 * D;
        L.s = o;      o += 4 * D;
        L.qin = o;    o += (int)sizeof(InT) * D;
        L.kin = o;    o += (int)sizeof(InT) * D;
        L.vin = o;    o += (int)sizeof(InT) * D;
        L.gin = o;    o += KDA ? 4 * D : 0;
        L.gsum = o;   o += KDA ? 8 * D : 0;
        L.cidx = o;   o += align_up(4 * cis, 16);
        L.crow = o;   o += 4 * D * ncr;
        L.ccol = o;   o += 4 * D * ncc;
        o = align_up(o, 128);
        L.slot_delta = 0;
        L.slot_key = 4 * kChunk * D;
        L.slot_gate = L.slot_key + (int)sizeof(KeyT) * kChunk * D;
        L.slot_bytes = align_up(L.slot_gate + (KDA ? 0 : 8 * kChunk), 128);
        L.ring = o;   o += NS * L.slot_bytes;
        L.xq = o;     o += 4 * D;
        L.xk = o;     o += 4 * D;
        L.yq = o;     o += 4 * D;
        L.yk = o;     o += 4 * D;
        L.qk_raw = o; o += 4 * 2 * D;   // raw q, k as FP32 (scalar-gate entry dots)
        L.a = o;      o += 4 * D;
        L.b = o;      o += 4 * D;
        L.coef_k = o; o += 4 * kChunk;
        L.coef_q = o; o += 4 * kChunk;
        L.fac = o;    o += 4 * kChunk;
        L.rc_k = o;   o += 4 * 16;
        L.rc_q = o;   o += 4 * 16;
        L.red = o;    o += 4 * 8;
        L.total = align_up(o, 128);
        return L;
    }
};

template <typename T>
__device__ __forceinline__ float to_f32(T x) { return static_cast<float>(x); }
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }

// VPL consecutive key elements starting at p, widened to FP32.
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

template <int D, bool KDA, typename InT, typename KeyT>
__global__ void __launch_bounds__(kThreads) decode_window_kernel(DecodeArgs a) {
    using Sh = DecShape<D, KDA, InT, KeyT>;
    constexpr int NS = Sh::NS, LPR = Sh::LPR, RPW = Sh::RPW, VPL = Sh::VPL;
    const Views &w = a.w;
    const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ncr = w.n_comp_rows, ncc = w.n_comp_cols, cis = w.comp_index_stride;
    const int n_buf = a.n_buf;
    const int nchunks = (n_buf + kChunk - 1) / kChunk;
    const DecLayout L = Sh::layout(ncr, ncc, cis);

    extern __shared__ __align__(128) unsigned char sm[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bars);
    const int8_t *sQ = reinterpret_cast<const int8_t *>(sm + L.q);
    const float *sSig = reinterpret_cast<const float *>(sm + L.sig);
    const float *sS = reinterpret_cast<const float *>(sm + L.s);
    const InT *sQin = reinterpret_cast<const InT *>(sm + L.qin);
    const InT *sKin = reinterpret_cast<const InT *>(sm + L.kin);
    const InT *sVin = reinterpret_cast<const InT *>(sm + L.vin);
    const float *sGin = reinterpret_cast<const float *>(sm + L.gin);
    const double *sGsum = reinterpret_cast<const double *>(sm + L.gsum);
    const int32_t *sCidx = reinterpret_cast<const int32_t *>(sm + L.cidx);
    const float *sCrow = reinterpret_cast<const float *>(sm + L.crow);
    const float *sCcol = reinterpret_cast<const float *>(sm + L.ccol);
    float *sXq = reinterpret_cast<float *>(sm + L.xq);
    float *sXk = reinterpret_cast<float *>(sm + L.xk);
    float *sYq = reinterpret_cast<float *>(sm + L.yq);
    float *sYk = reinterpret_cast<float *>(sm + L.yk);
    float *sQraw = reinterpret_cast<float *>(sm + L.qk_raw);
    float *sKraw = sQraw + D;
    float *sA = reinterpret_cast<float *>(sm + L.a);
    float *sB = reinterpret_cast<float *>(sm + L.b);
    float *sCk = reinterpret_cast<float *>(sm + L.coef_k);
    float *sCq = reinterpret_cast<float *>(sm + L.coef_q);
    float *sFac = reinterpret_cast<float *>(sm + L.fac);
    float *sRck = reinterpret_cast<float *>(sm + L.rc_k);
    float *sRcq = reinterpret_cast<float *>(sm + L.rc_q);
    float *sRed = reinterpret_cast<float *>(sm + L.red);

    auto slot_ptr = [&](int slot) { return sm + L.ring + slot * L.slot_bytes; };
    auto issue_chunk = [&](int c) {
        const int slot = c % NS, e0 = c * kChunk, ne = min(kChunk, n_buf - e0);
        unsigned char *dst = slot_ptr(slot);
        const size_t first = (size_t)u * w.window + e0;
        const uint32_t bd = 4u * ne * D, bk = (uint32_t)sizeof(KeyT) * ne * D;
        const uint32_t bg = KDA ? 0u : 8u * (uint32_t)align_up(ne, 2);
        mbar_arrive_expect_tx(&bars[1 + slot], bd + bk + bg);
        bulk_g2s(dst + L.slot_delta, w.buf_delta + first * D, bd, &bars[1 + slot]);
        bulk_g2s(dst + L.slot_key, reinterpret_cast<const KeyT *>(w.buf_key) + first * D, bk, &bars[1 + slot]);
        if (!KDA)
            bulk_g2s(dst + L.slot_gate, w.buf_gate + (size_t)u * w.window_pad + e0, bg, &bars[1 + slot]);
    };

    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < 1 + NS; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (tid == 0) {
        const uint64_t stream_once = l2_policy_evict_first();
        const uint32_t in_b = (uint32_t)sizeof(InT) * D;
        uint32_t hb = D * D + 8 * D + 3 * in_b;
        if (KDA) hb += 12 * D;
        if (ncr + ncc > 0) hb += 4 * cis + 4 * D * (ncr + ncc);
        mbar_arrive_expect_tx(&bars[0], hb);
        bulk_g2s_stream(sm + L.q, w.codes + (size_t)u * D * D, D * D, &bars[0], stream_once);
        bulk_g2s(sm + L.sig, w.row_scale + (size_t)u * D, 4 * D, &bars[0]);
        bulk_g2s(sm + L.s, w.col_smooth + (size_t)u * D, 4 * D, &bars[0]);
        bulk_g2s(sm + L.qin, reinterpret_cast<const InT *>(a.q) + (size_t)u * D, in_b, &bars[0]);
        bulk_g2s(sm + L.kin, reinterpret_cast<const InT *>(a.k) + (size_t)u * D, in_b, &bars[0]);
        bulk_g2s(sm + L.vin, reinterpret_cast<const InT *>(a.v) + (size_t)u * D, in_b, &bars[0]);
        if (KDA) {
            bulk_g2s(sm + L.gin, a.g + (size_t)u * D, 4 * D, &bars[0]);
            bulk_g2s(sm + L.gsum, w.gate_sum + (size_t)u * D, 8 * D, &bars[0]);
        }
        if (ncr + ncc > 0) {
            bulk_g2s(sm + L.cidx, w.comp_index + (size_t)u * cis, 4 * cis, &bars[0]);
            if (ncr > 0) bulk_g2s(sm + L.crow, w.comp_row_vec + (size_t)u * ncr * D, 4 * D * ncr, &bars[0]);
            if (ncc > 0) bulk_g2s(sm + L.ccol, w.comp_col_vec + (size_t)u * ncc * D, 4 * D * ncc, &bars[0]);
        }
        for (int c = 0; c < min(NS, nchunks); ++c) issue_chunk(c);
    }

    // per-unit scalars (plain loads, overlapping the copies)
    const float beta = a.beta[u];
    double Gt_s = 0.0;
    if (!KDA) Gt_s = w.gate_sum[u] + (double)a.g[u];

    int bad = !mbar_wait(&bars[0], 0, kWaitBudgetCycles);
    if (__syncthreads_or(bad)) {
        if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 0);
        return;
    }

    // ---------------------------------------------------------- A1: prologue
    double Gt_j = 0.0;
    float kappa_j = 0.0f, kq = 0.0f;
    if (tid < D) {
        const int j = tid;
        float gam;
        if (KDA) {
            Gt_j = sGsum[j] + (double)sGin[j];
            gam = (float)exp(Gt_j);
            if (fabs(Gt_j) > (double)kMaxAbsGateSum) report_error(w.err, LQ_DEVERR_RANGE, u, j);
        } else {
            gam = (float)exp(Gt_s);
        }
        const float qj = to_f32(sQin[j]), kj = to_f32(sKin[j]);
        const float xq = gam * qj, xk = gam * kj;
        sXq[j] = xq;
        sXk[j] = xk;
        sYq[j] = sS[j] * xq;
        sYk[j] = sS[j] * xk;
        sQraw[j] = qj;
        sKraw[j] = kj;
        kq = kj * qj;
        if (KDA) kappa_j = kj * (float)exp(-Gt_j);
    }
    kq = group_sum<32>(kq);
    if (lane == 0) sRed[warp] = kq;
    __syncthreads();
    kq = 0.0f;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) kq += sRed[i];

    // ------------------------------------- A2: one pass over the INT8 tile
    {
        const int cb = lane % LPR, rsub = lane / LPR;
        float yq[16], yk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            yq[i] = sYq[cb * 16 + i];
            yk[i] = sYk[cb * 16 + i];
        }
#pragma unroll 2
        for (int r0 = 0; r0 < D; r0 += 4 * RPW) {
            const int r = r0 + warp * RPW + rsub;
            const uint4 qw = *reinterpret_cast<const uint4 *>(sQ + r * D + cb * 16);
            const uint32_t words[4] = {qw.x, qw.y, qw.z, qw.w};
            float pa = 0.0f, pb = 0.0f;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float f0, f1, f2, f3;
                i8x4_to_f32(words[h], f0, f1, f2, f3);
                pa = fmaf(f0, yq[4 * h + 0], pa); pb = fmaf(f0, yk[4 * h + 0], pb);
                pa = fmaf(f1, yq[4 * h + 1], pa); pb = fmaf(f1, yk[4 * h + 1], pb);
                pa = fmaf(f2, yq[4 * h + 2], pa); pb = fmaf(f2, yk[4 * h + 2], pb);
                pa = fmaf(f3, yq[4 * h + 3], pa); pb = fmaf(f3, yk[4 * h + 3], pb);
            }
            pa = group_sum<LPR>(pa);
            pb = group_sum<LPR>(pb);
            if (cb == 0) {
                sA[r] = sSig[r] * pa;
                sB[r] = sSig[r] * pb;
            }
        }
    }
    // row compensators: k_c . x (one warp per compensator)
    for (int c = warp; c < ncr; c += kThreads / 32) {
        float dk = 0.0f, dq = 0.0f;
        for (int j = lane; j < D; j += 32) {
            const float kc = sCrow[c * D + j];
            dk = fmaf(kc, sXk[j], dk);
            dq = fmaf(kc, sXq[j], dq);
        }
        dk = group_sum<32>(dk);
        dq = group_sum<32>(dq);
        if (lane == 0) { sRck[c] = dk; sRcq[c] = dq; }
    }
    __syncthreads();

    // -------------------------------- A3: compensators + buffered corrections
    float acc_k = 0.0f, acc_q = 0.0f;
    if (tid < D) {
        const int i = tid;
        acc_k = sB[i];
        acc_q = sA[i];
        for (int c = 0; c < ncr; ++c)
            if (sCidx[c] == i) { acc_k += sRck[c]; acc_q += sRcq[c]; }
        for (int c = 0; c < ncc; ++c) {
            const int j = sCidx[ncr + c];
            const float vci = sCcol[c * D + i];
            acc_k = fmaf(vci, sXk[j], acc_k);
            acc_q = fmaf(vci, sXq[j], acc_q);
        }
    }
    // this lane's slice of the vectors the buffered keys are dotted with
    float xs_k[VPL], xs_q[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
        xs_k[v] = KDA ? sXk[lane * VPL + v] : sKraw[lane * VPL + v];
        xs_q[v] = KDA ? sXq[lane * VPL + v] : sQraw[lane * VPL + v];
    }

    for (int c = 0; c < nchunks; ++c) {
        const int slot = c % NS, e0 = c * kChunk, ne = min(kChunk, n_buf - e0);
        const unsigned char *sp = slot_ptr(slot);
        const float *sDelta = reinterpret_cast<const float *>(sp + L.slot_delta);
        const KeyT *sKey = reinterpret_cast<const KeyT *>(sp + L.slot_key);
        const double *sGate = reinterpret_cast<const double *>(sp + L.slot_gate);
        bad = !mbar_wait(&bars[1 + slot], (uint32_t)((c / NS) & 1), kWaitBudgetCycles);
        if (!KDA && !bad && tid < ne) sFac[tid] = (float)exp(Gt_s - sGate[tid]);
        if (__syncthreads_or(bad)) {
            if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 1 + c);
            return;
        }
        for (int el = warp; el < ne; el += kThreads / 32) {
            float kv[VPL];
            load_key<KeyT, VPL>(sKey + el * D + lane * VPL, kv);
            float dk = 0.0f, dq = 0.0f;
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                dk = fmaf(kv[v], xs_k[v], dk);
                dq = fmaf(kv[v], xs_q[v], dq);
            }
            dk = group_sum<32>(dk);
            dq = group_sum<32>(dq);
            if (lane == 0) {
                const float f = KDA ? 1.0f : sFac[el];
                sCk[el] = f * dk;
                sCq[el] = f * dq;
            }
        }
        __syncthreads();
        if (tid < D) {
            for (int el = 0; el < ne; ++el) {
                const float d = sDelta[el * D + tid];
                acc_k = fmaf(sCk[el], d, acc_k);
                acc_q = fmaf(sCq[el], d, acc_q);
            }
        }
        __syncthreads();
        if (tid == 0 && c + NS < nchunks) {
            fence_proxy_async_smem();
            issue_chunk(c + NS);
        }
    }

    // ------------------------------------------------- A4: emit and append
    if (tid < D) {
        const int i = tid;
        const float delta = beta * (to_f32(sVin[i]) - acc_k);
        a.o[(size_t)u * D + i] = fmaf(delta, kq, acc_q);
        const size_t slot = (size_t)u * w.window + n_buf;
        w.buf_delta[slot * D + i] = delta;
        if (KDA) {
            reinterpret_cast<float *>(w.buf_key)[slot * D + i] = kappa_j;
            w.gate_sum[(size_t)u * D + i] = Gt_j;
        } else {
            reinterpret_cast<KeyT *>(w.buf_key)[slot * D + i] = static_cast<KeyT>(sKin[i]);
        }
    }
    if (!KDA && tid == 0) {
        w.buf_gate[(size_t)u * w.window_pad + n_buf] = Gt_s;
        w.gate_sum[u] = Gt_s;
    }
}

template <int D, bool KDA, typename InT, typename KeyT>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    using Sh = DecShape<D, KDA, InT, KeyT>;
    const DecLayout L = Sh::layout(a.w.n_comp_rows, a.w.n_comp_cols, a.w.comp_index_stride);
    auto kern = decode_window_kernel<D, KDA, InT, KeyT>;
    // The opt-in shared-memory size is set once per device and size, so that
    // launches inside a stream capture make no attribute calls.
    static int opted_in[64] = {0};
    if (L.total > 48 * 1024) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 64 || opted_in[dev] < L.total) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) opted_in[dev] = L.total;
        }
    }
    kern<<<a.w.units, kThreads, L.total, s>>>(a);
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
