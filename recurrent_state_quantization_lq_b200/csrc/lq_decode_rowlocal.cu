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
// and no compensators or smoothing.  One CTA per (sequence, head), rows spread over
// lanes groups with 16-byte vector loads.
#include "lq_kernels.h"

namespace lq {
namespace {

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

template <int D, bool KDA, typename InT>
__global__ void __launch_bounds__(kThreads) decode_naive_kernel(DecodeArgs a) {
    constexpr int LPR = D / 16;           // lanes per row, 16 codes each
    constexpr int RPW = 32 / LPR;
    constexpr int RPS = kWarps * RPW;
    constexpr int STEPS = D / RPS;        // rows per lane
    const int u = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = (lane % LPR) * 16, rsub = lane / LPR;
    const InT *q = reinterpret_cast<const InT *>(a.q) + (size_t)u * D;
    const InT *k = reinterpret_cast<const InT *>(a.k) + (size_t)u * D;
    const InT *v = reinterpret_cast<const InT *>(a.v) + (size_t)u * D;
    int8_t *Qu = a.w.codes + (size_t)u * D * D;
    float *sig = a.w.row_scale + (size_t)u * D;

    uint4 cw[STEPS];
    float sg[STEPS], vr[STEPS];
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
        const int r = s * RPS + warp * RPW + rsub;
        cw[s] = __ldcs(reinterpret_cast<const uint4 *>(Qu + (size_t)r * D + c0));
        sg[s] = __ldcs(sig + r);
        vr[s] = ld_f32(v + r);
    }
    float k16[16], q16[16], al[16];
    ld_vec<InT, 16>(k + c0, k16);
    ld_vec<InT, 16>(q + c0, q16);
    if (KDA) {
        float g16[16];
        ld_vec<float, 16>(a.g + (size_t)u * D + c0, g16);
#pragma unroll
        for (int i = 0; i < 16; ++i) al[i] = expf(g16[i]);
    } else {
        const float alpha = expf(__ldg(a.g + u));
#pragma unroll
        for (int i = 0; i < 16; ++i) al[i] = alpha;
    }
    const float beta = __ldg(a.beta + u);

#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
        const int r = s * RPS + warp * RPW + rsub;
        float R[16];
        const uint32_t words[4] = {cw[s].x, cw[s].y, cw[s].z, cw[s].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            float f0, f1, f2, f3;
            i8x4_to_f32(words[h], f0, f1, f2, f3);
            R[4 * h] = sg[s] * f0; R[4 * h + 1] = sg[s] * f1;
            R[4 * h + 2] = sg[s] * f2; R[4 * h + 3] = sg[s] * f3;
        }
        float sk = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) sk = fmaf(R[i], al[i] * k16[i], sk);
        sk = group_sum<LPR>(sk);
        const float delta = beta * (vr[s] - sk);
        float po = 0.0f, m = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            R[i] = fmaf(al[i], R[i], delta * k16[i]);
            po = fmaf(R[i], q16[i], po);
            m = fmaxf(m, fabsf(R[i]));
        }
        po = group_sum<LPR>(po);
        m = group_max<LPR>(m);
        const float sigma = __fdiv_rn(m, 127.0f);
        const float rho = (m > 0.0f) ? __fdiv_rn(127.0f, m) : 0.0f;
        uint32_t out[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            uint32_t word = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float code = fminf(fmaxf(rintf(__fmul_rn(R[4 * h + c], rho)), -127.0f), 127.0f);
                word |= (uint32_t)((int)code & 0xff) << (8 * c);
            }
            out[h] = word;
        }
        __stcs(reinterpret_cast<uint4 *>(Qu + (size_t)r * D + c0), make_uint4(out[0], out[1], out[2], out[3]));
        if (lane % LPR == 0) {
            sig[r] = sigma;
            a.o[(size_t)u * D + r] = po;
        }
    }
}

template <int D, bool KDA, typename InT>
cudaError_t launch_fp32_t(const DecodeArgs &a, cudaStream_t s) {
    decode_fp32_kernel<D, KDA, InT><<<a.w.units, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <int D, bool KDA, typename InT>
cudaError_t launch_naive_t(const DecodeArgs &a, cudaStream_t s) {
    decode_naive_kernel<D, KDA, InT><<<a.w.units, kThreads, 0, s>>>(a);
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
