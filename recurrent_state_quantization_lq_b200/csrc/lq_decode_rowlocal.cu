// Comparator decode kernels: FP32 state and naive per-token INT8 state.
//
// Both are the baselines LeapQuant is measured against (bedrocknews.com
// article on arXiv 2609.38166v1, mechanism paragraph: FP32 inference is the
// baseline, and naive per-token quantization collapses quality).  Each state
// row is independent given the token, so every row takes one pass:
//   sk_i    = sum_j S_ij alpha_j k_j            (scalar gate: alpha sum_j S_ij k_j)
//   delta_i = beta (v_i - sk_i)
//   S'_ij   = alpha_j S_ij + delta_i k_j
//   o_i     = sum_j S'_ij q_j
// The FP32 kernel reads and writes the FP32 row.  The naive kernel
// dequantizes the row (sigma_i Q_ij), applies the same update, emits o from
// the updated FP32 row, then requantizes it with a fresh per-row scale
// (M_i = max_j |S'_ij|, sigma'_i = M_i / 127, Q'_ij = rint(S'_ij * (127 / M_i)))
// and no compensators or smoothing.  The FP32 kernel takes one CTA per
// (sequence, head), rows spread over lane groups with 16-byte vector loads;
// the naive kernel is described at its definition.
#include "lq_decode_parts.cuh"
#include "lq_kernels.h"

namespace lq {
namespace {

using dec::mbar_arrive;
using dec::to_f32;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename T>
__device__ __forceinline__ float ld_f32(const T *p) { return static_cast<float>(*p); }
template <>
__device__ __forceinline__ float ld_f32<float>(const float *p) { return __ldg(p); }

// N consecutive input elements at p (16-byte aligned for N * sizeof(T) >= 16).
template <typename T, int N>
__device__ __forceinline__ void ld_vec(const T *p, float (&out)[N]) {
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            float4 x = __ldg(reinterpret_cast<const float4 *>(p + i));
            out[i] = x.x; out[i + 1] = x.y; out[i + 2] = x.z; out[i + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            uint2 x = __ldg(reinterpret_cast<const uint2 *>(p + i));
            out[i] = bf16_bits_to_f32(x.x & 0xffffu); out[i + 1] = bf16_bits_to_f32(x.x >> 16);
            out[i + 2] = bf16_bits_to_f32(x.y & 0xffffu); out[i + 3] = bf16_bits_to_f32(x.y >> 16);
        }
    }
}

// ------------------------------------------------------------- FP32 state

template <int D, bool KDA, typename InT>
__global__ void __launch_bounds__(kThreads) decode_fp32_kernel(DecodeArgs a) {
    constexpr int LPR = D / 4;            // lanes per row, 4 columns each
    constexpr int RPW = 32 / LPR;         // rows per warp per step
    constexpr int RPS = kWarps * RPW;     // rows per CTA per step
    constexpr int STEPS = D / RPS;
    constexpr int U = 4;                  // rows in flight per lane
    static_assert(STEPS % U == 0, "row steps must divide");
    const int u = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = (lane % LPR) * 4, rsub = lane / LPR;
    const InT *q = reinterpret_cast<const InT *>(a.q) + (size_t)u * D;
    const InT *k = reinterpret_cast<const InT *>(a.k) + (size_t)u * D;
    const InT *v = reinterpret_cast<const InT *>(a.v) + (size_t)u * D;
    float k4[4], q4[4], al[4];
    ld_vec<InT, 4>(k + c0, k4);
    ld_vec<InT, 4>(q + c0, q4);
    if (KDA) {
        float g4[4];
        ld_vec<float, 4>(a.g + (size_t)u * D + c0, g4);
#pragma unroll
        for (int i = 0; i < 4; ++i) al[i] = expf(g4[i]);
    } else {
        const float alpha = expf(__ldg(a.g + u));
#pragma unroll
        for (int i = 0; i < 4; ++i) al[i] = alpha;
    }
    float ak[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) ak[i] = al[i] * k4[i];
    const float beta = __ldg(a.beta + u);
    float *S = a.w.state_f32 + (size_t)u * D * D;

    for (int s0 = 0; s0 < STEPS; s0 += U) {
        float4 x[U];
        float vr[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int r = (s0 + i) * RPS + warp * RPW + rsub;
            x[i] = __ldcs(reinterpret_cast<const float4 *>(S + (size_t)r * D + c0));
            vr[i] = ld_f32(v + r);
        }
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int r = (s0 + i) * RPS + warp * RPW + rsub;
            float sk = x[i].x * ak[0];
            sk = fmaf(x[i].y, ak[1], sk);
            sk = fmaf(x[i].z, ak[2], sk);
            sk = fmaf(x[i].w, ak[3], sk);
            sk = group_sum<LPR>(sk);
            const float delta = beta * (vr[i] - sk);
            float4 y;
            y.x = fmaf(al[0], x[i].x, delta * k4[0]);
            y.y = fmaf(al[1], x[i].y, delta * k4[1]);
            y.z = fmaf(al[2], x[i].z, delta * k4[2]);
            y.w = fmaf(al[3], x[i].w, delta * k4[3]);
            __stcs(reinterpret_cast<float4 *>(S + (size_t)r * D + c0), y);
            float po = y.x * q4[0];
            po = fmaf(y.y, q4[1], po);
            po = fmaf(y.z, q4[2], po);
            po = fmaf(y.w, q4[3], po);
            po = group_sum<LPR>(po);
            if (lane % LPR == 0) a.o[(size_t)u * D + r] = po;
        }
    }
}

// ------------------------------------------------- naive per-token INT8
//
// Persistent and warp-specialized, like the windowed decode: several CTAs per
// SM walk the units; in each, one producer thread bulk-copies every unit's
// codes, row scales and q/k/v (and the per-channel gate) into a ring of
// shared-memory slots, and four consumer warps take the unit's rows from
// there.  A row is handled by D/16 lanes (16 codes each) of one warp, so no
// warp waits for another: the only synchronization is the slot ring.  The
// copies of up to NS units per CTA are in flight at once, which is what keeps
// HBM busy; the per-row chain (two dots, the update, the maximum, the codes)
// runs on packed FP32 pairs.

namespace naive {
constexpr int kConsWarps = 4;
constexpr int kCons = 32 * kConsWarps;
constexpr int kThreadsN = kCons + 32;            // + one producer warp
// four CTAs per SM for the scalar gate; three for the per-channel gate, whose
// gate vectors need the registers
template <bool KDA>
constexpr int ctas_per_sm() { return KDA ? 3 : 4; }

template <int D, bool KDA, typename InT>
struct Slot {
    static constexpr int CODES = 0;
    static constexpr int SIG = D * D;
    static constexpr int QIN = SIG + 4 * D;
    static constexpr int KIN = QIN + (int)sizeof(InT) * D;
    static constexpr int VIN = KIN + (int)sizeof(InT) * D;
    static constexpr int GIN = VIN + (int)sizeof(InT) * D;  // per-channel log-gate
    static constexpr int COPY = GIN + (KDA ? 4 * D : 0);     // bytes copied per unit
    static constexpr int BYTES = (COPY + 127) / 128 * 128;
    static constexpr int NS = (KDA && BYTES <= 18432) ? 4 : 3;   // ring slots that fit the CTAs of an SM
    static constexpr int SMEM = 1024 + NS * BYTES;           // barriers, then the ring
};
}  // namespace naive

// N consecutive inputs from shared memory as floats (16-byte aligned).
template <typename InT, int N>
__device__ __forceinline__ void ld_smem(const InT *p, float (&out)[N]) {
    if constexpr (sizeof(InT) == 4) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(p + i);
            out[i] = x.x; out[i + 1] = x.y; out[i + 2] = x.z; out[i + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 8) {
            const uint4 x = *reinterpret_cast<const uint4 *>(p + i);
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                out[i + 2 * h] = bf16_bits_to_f32(w[h] & 0xffffu);
                out[i + 2 * h + 1] = bf16_bits_to_f32(w[h] >> 16);
            }
        }
    }
}

// max(|a|, |b|, |c|) in one instruction (the three-input form of max with
// .abs, which takes the absolute values of its inputs).
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
    float r;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Sixteen int8 codes (one 16-byte word) as eight float pairs, exactly: the
// byte permutes of i8x4_to_f32, with the bias taken off two values at a time.
__device__ __forceinline__ void codes_to_f32x2(uint4 cw, float2 (&f)[8]) {
    const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
    const float2 bias = make_float2(-8388736.0f, -8388736.0f);   // -(2^23 + 128)
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const uint32_t u = w[h] ^ 0x80808080u;
        f[2 * h] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)),
                                          __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541))), bias);
        f[2 * h + 1] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)),
                                              __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543))), bias);
    }
}

// Low bytes of rint(x * rho) for 16 values (8 pairs), packed as codes.  The
// caller guarantees |x * rho| <= 127 before rounding (rho = RN(127 / max|x|)
// makes the product at most 127.00002), so rint lands in [-127, 127]: adding
// 1.5 * 2^23 rounds to the nearest integer (ties to even, as rintf) and leaves
// it, in two's complement, in the low byte.
__device__ __forceinline__ uint4 requantize16(const float2 *x, float rho) {
    const float2 r2 = make_float2(rho, rho), magic = make_float2(12582912.0f, 12582912.0f);
    uint32_t b[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 tq = __fadd2_rn(__fmul2_rn(x[i], r2), magic);
        b[2 * i] = __float_as_uint(tq.x);
        b[2 * i + 1] = __float_as_uint(tq.y);
    }
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const uint32_t lo = __byte_perm(b[4 * h], b[4 * h + 1], 0x0040u);       // bytes b0, b1
        const uint32_t hi = __byte_perm(b[4 * h + 2], b[4 * h + 3], 0x0040u);   // bytes b2, b3
        w[h] = __byte_perm(lo, hi, 0x5410u);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int D, bool KDA, typename InT>
__global__ void __launch_bounds__(naive::kThreadsN, naive::ctas_per_sm<KDA>()) decode_naive_kernel(DecodeArgs a) {
    using Sl = naive::Slot<D, KDA, InT>;
    constexpr int NS = Sl::NS;
    constexpr int EPL = 16;                      // codes per lane (one 16-byte word)
    constexpr int NP = EPL / 2;                  // value pairs per lane
    constexpr int LPR = D / EPL;                 // lanes per row
    constexpr int RPW = 32 / LPR;                // rows per warp per step
    constexpr int RPS = naive::kConsWarps * RPW; // rows per CTA per step
    constexpr int STEPS = D / RPS;
    constexpr int RPI = 1;                       // rows per thread per iteration
    const Views &w = a.w;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int units = w.units;

    extern __shared__ __align__(128) unsigned char sm_raw[];
    uint64_t *full = reinterpret_cast<uint64_t *>(sm_raw);
    uint64_t *empty = full + NS;
    unsigned char *ring = sm_raw + 1024;
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], naive::kCons);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // ---------------------------------------------------------------- producer
    if (warp == naive::kConsWarps) {
        if (lane != 0) return;
        constexpr uint32_t in_b = (uint32_t)sizeof(InT) * D;
        int slot = 0;
        uint32_t ph = 0, armed = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            if (!mbar_wait(&empty[slot], ph ^ 1u, kWaitBudgetCycles)) {
                report_error(w.err, LQ_DEVERR_TIMEOUT, u, -1);
                // the consumers have stopped: let this thread's copies land first
                for (int i = 0; i < NS; ++i)
                    if (armed & (1u << i)) mbar_wait(&full[i], i < slot ? ph : (ph ^ 1u), kWaitBudgetCycles);
                return;
            }
            armed |= 1u << slot;
            unsigned char *dst = ring + slot * Sl::BYTES;
            uint64_t *bar = &full[slot];
            mbar_arrive_expect_tx(bar, (uint32_t)Sl::COPY);
            bulk_g2s(dst + Sl::CODES, w.codes + (size_t)u * D * D, D * D, bar);
            bulk_g2s(dst + Sl::SIG, w.row_scale + (size_t)u * D, 4 * D, bar);
            bulk_g2s(dst + Sl::QIN, reinterpret_cast<const InT *>(a.q) + (size_t)u * D, in_b, bar);
            bulk_g2s(dst + Sl::KIN, reinterpret_cast<const InT *>(a.k) + (size_t)u * D, in_b, bar);
            bulk_g2s(dst + Sl::VIN, reinterpret_cast<const InT *>(a.v) + (size_t)u * D, in_b, bar);
            if (KDA) bulk_g2s(dst + Sl::GIN, a.g + (size_t)u * D, 4 * D, bar);
            if (++slot == NS) { slot = 0; ph ^= 1u; }
        }
        return;
    }

    // --------------------------------------------------------------- consumers
    const int c0 = (lane % LPR) * EPL, rsub = lane / LPR;
    int slot = 0;
    uint32_t ph = 0;
    int u = blockIdx.x;
    float beta_n = 0.0f, g_n = 0.0f;
    if (u < units) {
        beta_n = __ldg(a.beta + u);
        if (!KDA) g_n = __ldg(a.g + u);
    }
    for (; u < units; u += gridDim.x) {
        const float beta = beta_n, g_s = g_n;
        if (u + (int)gridDim.x < units) {      // next unit's scalars, in flight meanwhile
            beta_n = __ldg(a.beta + u + gridDim.x);
            if (!KDA) g_n = __ldg(a.g + u + gridDim.x);
        }
        if (!mbar_wait(&full[slot], ph, kWaitBudgetCycles)) {
            report_error(w.err, LQ_DEVERR_TIMEOUT, u, 0);
            return;                            // no further arrival: the producer gives up too
        }
        const unsigned char *sp = ring + slot * Sl::BYTES;
        const float *sig_s = reinterpret_cast<const float *>(sp + Sl::SIG);
        const InT *v_s = reinterpret_cast<const InT *>(sp + Sl::VIN);
        // this lane's EPL columns of k and q (and of alpha for the per-channel gate)
        float2 kk[NP], qq[NP], al[KDA ? NP : 1], ak[KDA ? NP : 1];
        float kq = 0.0f;                       // k . q over the row (once per unit)
        {
#pragma unroll
            for (int i = 0; i < NP; i += 4) {  // 8 values of k and of q at a time
                float kv[8], qv[8];
                ld_smem<InT, 8>(reinterpret_cast<const InT *>(sp + Sl::KIN) + c0 + 2 * i, kv);
                ld_smem<InT, 8>(reinterpret_cast<const InT *>(sp + Sl::QIN) + c0 + 2 * i, qv);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kk[i + e] = make_float2(kv[2 * e], kv[2 * e + 1]);
                    qq[i + e] = make_float2(qv[2 * e], qv[2 * e + 1]);
                    kq = fmaf(kv[2 * e], qv[2 * e], fmaf(kv[2 * e + 1], qv[2 * e + 1], kq));
                }
            }
            if constexpr (KDA) {
                float gv[EPL];
                ld_smem<float, EPL>(reinterpret_cast<const float *>(sp + Sl::GIN) + c0, gv);
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    al[i] = make_float2(expf(gv[2 * i]), expf(gv[2 * i + 1]));
                    ak[i] = __fmul2_rn(al[i], kk[i]);
                }
            }
        }
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
        const float alpha = KDA ? 1.0f : expf(g_s);
#pragma unroll 1
        for (int s = 0; s < STEPS; s += RPI) {
            int r[RPI];
            uint4 cw[RPI][EPL / 16];
            float sig[RPI], vr[RPI];
#pragma unroll
            for (int h = 0; h < RPI; ++h) {
                r[h] = (s + h) * RPS + warp * RPW + rsub;
#pragma unroll
                for (int c = 0; c < EPL / 16; ++c)
                    cw[h][c] = *reinterpret_cast<const uint4 *>(sp + Sl::CODES + r[h] * D + c0 + 16 * c);
                sig[h] = sig_s[r[h]];
                vr[h] = to_f32(v_s[r[h]]);
            }
            // Scalar gate: with a_i = alpha sigma_i the key and output sums come from
            // the codes,
            //   sk_i = a_i sum_j Q_ij k_j,   o_i = a_i sum_j Q_ij q_j + delta_i (k . q),
            // in one shared reduction, and S'_ij = a_i Q_ij + delta_i k_j.
            // Per-channel gate: S'_ij = alpha_j sigma_i Q_ij + delta_i k_j, and the
            // output sum is taken from the updated row.
            float2 x[RPI][NP];
            float sk[RPI], qs[RPI];
#pragma unroll
            for (int h = 0; h < RPI; ++h) {
#pragma unroll
                for (int c = 0; c < EPL / 16; ++c) codes_to_f32x2(cw[h][c], *reinterpret_cast<float2(*)[8]>(&x[h][8 * c]));
                float2 p0 = make_float2(0.0f, 0.0f), p1 = p0, r0 = p0, r1 = p0;
#pragma unroll
                for (int i = 0; i < NP; i += 2) {
                    p0 = __ffma2_rn(x[h][i], KDA ? ak[i] : kk[i], p0);
                    p1 = __ffma2_rn(x[h][i + 1], KDA ? ak[i + 1] : kk[i + 1], p1);
                    if constexpr (!KDA) {
                        r0 = __ffma2_rn(x[h][i], qq[i], r0);
                        r1 = __ffma2_rn(x[h][i + 1], qq[i + 1], r1);
                    }
                }
                sk[h] = (p0.x + p0.y) + (p1.x + p1.y);
                qs[h] = (r0.x + r0.y) + (r1.x + r1.y);
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1)
#pragma unroll
                for (int h = 0; h < RPI; ++h) {
                    sk[h] += __shfl_xor_sync(0xffffffffu, sk[h], o);
                    if constexpr (!KDA) qs[h] += __shfl_xor_sync(0xffffffffu, qs[h], o);
                }
            float po[RPI], m[RPI];
#pragma unroll
            for (int h = 0; h < RPI; ++h) {
                const float as = alpha * sig[h];
                const float delta = beta * (vr[h] - sk[h] * as);
                float m0 = 0.0f, m1 = 0.0f;
                if constexpr (KDA) {
                    const float2 dd = make_float2(delta, delta), sg = make_float2(sig[h], sig[h]);
                    float2 p0 = make_float2(0.0f, 0.0f), p1 = p0;
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
                        x[h][i] = __ffma2_rn(__fmul2_rn(al[i], sg), x[h][i], __fmul2_rn(dd, kk[i]));
                        if (i & 1) p1 = __ffma2_rn(x[h][i], qq[i], p1);
                        else p0 = __ffma2_rn(x[h][i], qq[i], p0);
                        if (i & 1) m1 = max3_abs(x[h][i].x, x[h][i].y, m1);
                        else m0 = max3_abs(x[h][i].x, x[h][i].y, m0);
                    }
                    po[h] = (p0.x + p0.y) + (p1.x + p1.y);
                } else {
                    const float2 dd = make_float2(delta, delta), sc = make_float2(as, as);
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
                        x[h][i] = __ffma2_rn(sc, x[h][i], __fmul2_rn(dd, kk[i]));
                        if (i & 1) m1 = max3_abs(x[h][i].x, x[h][i].y, m1);
                        else m0 = max3_abs(x[h][i].x, x[h][i].y, m0);
                    }
                    po[h] = fmaf(delta, kq, as * qs[h]);
                }
                m[h] = fmaxf(m0, m1);
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1)
#pragma unroll
                for (int h = 0; h < RPI; ++h) {
                    if constexpr (KDA) po[h] += __shfl_xor_sync(0xffffffffu, po[h], o);
                    m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], o));
                }
#pragma unroll
            for (int h = 0; h < RPI; ++h) {
                // sigma' = M / 127 and codes rint(S' * (127 / M)), M = max_j |S'_ij|,
                // with 1 / M as an IEEE reciprocal (one rounding more than a division:
                // a code on a rounding boundary may move by one); a row whose largest
                // magnitude is below 2^-100 (where 127 / M could overflow) keeps zero
                // codes
                const float sigma = m[h] * (1.0f / 127.0f);
                const float rho = (m[h] >= 0x1p-100f) ? 127.0f * __frcp_rn(m[h]) : 0.0f;
#pragma unroll
                for (int c = 0; c < EPL / 16; ++c) {
                    const uint4 out = requantize16(&x[h][8 * c], rho);
                    __stcs(reinterpret_cast<uint4 *>(w.codes + (size_t)u * D * D + (size_t)r[h] * D + c0 + 16 * c), out);
                }
                if (lane % LPR == 0) {
                    w.row_scale[(size_t)u * D + r[h]] = sigma;
                    a.o[(size_t)u * D + r[h]] = po[h];
                }
            }
        }
        mbar_arrive(&empty[slot]);             // this thread's last read of the slot
        if (++slot == NS) { slot = 0; ph ^= 1u; }
    }
}

template <int D, bool KDA, typename InT>
cudaError_t launch_fp32_t(const DecodeArgs &a, cudaStream_t s) {
    decode_fp32_kernel<D, KDA, InT><<<a.w.units, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <int D, bool KDA, typename InT>
cudaError_t launch_naive_t(const DecodeArgs &a, cudaStream_t s) {
    using Sl = naive::Slot<D, KDA, InT>;
    const cudaError_t e = opt_in_smem<decode_naive_kernel<D, KDA, InT>>(Sl::SMEM);
    if (e != cudaSuccess) return e;
    const int grid = min(a.w.units, naive::ctas_per_sm<KDA>() * sm_count());
    decode_naive_kernel<D, KDA, InT><<<grid, naive::kThreadsN, Sl::SMEM, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

#define LQ_DISPATCH(FN)                                                                             \
    const bool kda = (gate == LQ_GATE_CHANNEL), bf = (in_dtype == LQ_DTYPE_BF16);                   \
    if (d == 128) {                                                                                 \
        if (kda) return bf ? FN<128, true, __nv_bfloat16>(a, s) : FN<128, true, float>(a, s);       \
        return bf ? FN<128, false, __nv_bfloat16>(a, s) : FN<128, false, float>(a, s);              \
    }                                                                                               \
    if (d == 64) {                                                                                  \
        if (kda) return bf ? FN<64, true, __nv_bfloat16>(a, s) : FN<64, true, float>(a, s);         \
        return bf ? FN<64, false, __nv_bfloat16>(a, s) : FN<64, false, float>(a, s);                \
    }                                                                                               \
    return cudaErrorInvalidValue;

cudaError_t launch_decode_fp32(const DecodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s) {
    LQ_DISPATCH(launch_fp32_t)
}

cudaError_t launch_decode_naive(const DecodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s) {
    LQ_DISPATCH(launch_naive_t)
}

#undef LQ_DISPATCH

}  // namespace lq
