// Prefill from prompt tokens: the FP32 recurrence over the prompt with the
// state held in registers, then the state codec, so the INT8 window-start
// state is emitted directly.
//
// LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent
// State Quantization", section "Abstract (arXiv)") quantizes the recurrent
// state at window ends during decoding.  The prompt itself runs at full
// precision here: its final FP32 state is what an ingested state would be, and
// it is encoded once, as by the prefill ingestion.  Per (sequence, head) unit
// and prompt token t (the gated delta rule of Gated DeltaNet and Kimi Delta
// Attention):
//   GDN: S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
//   KDA: S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
//   o_t = S_t q_t,  alpha_t = exp(g_t).
// With u_t = beta_t (v_t - S_{t-1} diag(alpha_t) k_t) this is
// S_t = S_{t-1} diag(alpha_t) + u_t k_t^T.  Inside a chunk of tokens the kernel
// keeps S' with S_t = S'_t diag(c_t), c_t the product of the chunk's gates up
// to t (one value for GDN, one per key channel for KDA), so that
//   u_t = beta_t (v_t - S'_{t-1} (c_t . k_t)),
//   S'_t = S'_{t-1} + u_t (k_t / c_t)^T,   o_t = S'_t (c_t . q_t),
// one fused multiply-add per state element per product, and multiplies S' by
// c at each chunk's end.  A chunk whose summed log-gate exceeds 80 in
// magnitude in some channel is reported as a range error, as in the decode.
//
// One CTA of 256 threads per unit; the state stays in registers for the whole
// prompt.  A thread owns a 4-row x CW-column block (CW = D^2 / 1024), so every
// value read from shared memory feeds four FMAs: with one row per thread the
// broadcast vectors c.k, k/c and c.q would cost D times their size in
// shared-memory bandwidth per token, well above the FMA time.  The LPR = D / CW
// threads of a row block are adjacent lanes; they own interleaved 4-column
// pieces so that their 16-byte reads are contiguous.  A row's dot products are
// reduced over its LPR lanes by a butterfly that halves the four row partials
// at each of the first two levels, and the rows' u_t come back with four
// indexed shuffles.  Tokens
// pass through shared memory in chunks of 16: the next chunk's raw inputs
// arrive by asynchronous copies while the current one is applied, then are
// turned into c . k, k / c, c . q and v in FP32 once per chunk; the chunk's
// outputs leave as whole rows.  After the last token the state goes through
// shared memory into the codec's tile layout (lq_codec.cuh) and is encoded by
// the same threads, or (FP32-state mode) stored.
#include "lq_codec.cuh"
#include "lq_kernels.h"

namespace lq {
namespace {

constexpr int kTokChunk = 16;      // prompt tokens staged per pass
constexpr float kMaxChunkLogGate = 80.0f;

template <int D, bool KDA, int IB>
struct TokShape {
    static constexpr int NT = kTile;               // threads
    static constexpr int CW = D * D / (4 * NT);    // columns of a thread's 4-row block
    static constexpr int LPR = D / CW;             // lanes sharing a row block
    static constexpr int MG = CW / 4;              // 4-column pieces a thread owns
    static_assert(LPR >= 8 && LPR <= 32 && MG >= 1, "row blocks within a warp");
    // the FP32 stage (words): c.k, k/c, c.q, v, outputs [kTokChunk][D]; beta [kTokChunk];
    // c and 1/c [kTokChunk][D or 1]; c at the chunk's end [D or 1]
    static constexpr int GD = KDA ? D : 1;
    static constexpr int SKC = 0, SKD = kTokChunk * D, SQC = 2 * kTokChunk * D, SV = 3 * kTokChunk * D;
    static constexpr int SO = 4 * kTokChunk * D, SB = 5 * kTokChunk * D, SC = SB + kTokChunk;
    static constexpr int SCI = SC + kTokChunk * GD;
    static constexpr int STAGE = SCI + kTokChunk * GD;
    // the raw copy of the next chunk (words): k, q, v in the input type, g, beta
    static constexpr int RK = (STAGE + 3) / 4 * 4, RQ = RK + kTokChunk * D * IB / 4, RV = RQ + kTokChunk * D * IB / 4;
    static constexpr int RG = RV + kTokChunk * D * IB / 4;
    static constexpr int RB = RG + kTokChunk * GD;
    static constexpr int WORDS_STAGES = RB + kTokChunk;
    static constexpr int WORDS_CODEC = D * D;      // the final state, row-major (the codec scratch reuses it)
    static constexpr int WORDS = WORDS_STAGES > WORDS_CODEC ? WORDS_STAGES : WORDS_CODEC;
    static_assert(CodecScratch<D>::FLOATS <= WORDS_CODEC, "codec scratch fits");
    static_assert(2 * kTokChunk <= NT && kTokChunk <= NT, "gate and beta copies");
    static_assert(RQ % 4 == 0 && RV % 4 == 0 && RG % 4 == 0 && RB % 4 == 0, "16-byte aligned");
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// eight input values of a 16-byte piece (bf16) or four (f32), widened
template <typename T>
__device__ __forceinline__ void widen(const uint4 raw, float *f) {
    if constexpr (sizeof(T) == 2) {
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            f[2 * h] = bf16_bits_to_f32(wd[h] & 0xffffu);
            f[2 * h + 1] = bf16_bits_to_f32(wd[h] >> 16);
        }
    } else {
        f[0] = __uint_as_float(raw.x); f[1] = __uint_as_float(raw.y);
        f[2] = __uint_as_float(raw.z); f[3] = __uint_as_float(raw.w);
    }
}

template <int D, bool KDA, typename InT>
__global__ void __launch_bounds__(kTile, 2) prefill_tokens_kernel(TokenPrefillArgs a) {
    constexpr int IB = (int)sizeof(InT);
    using Sh = TokShape<D, KDA, IB>;
    constexpr int NT = Sh::NT, MG = Sh::MG, GD = Sh::GD, LPR = Sh::LPR;
    constexpr int VALS = 16 / IB;                                  // input values per 16-byte piece
    constexpr int TOTAL = kTokChunk * D / VALS;                    // 16-byte pieces of k (or q, v) per chunk
    constexpr int PIECES = (TOTAL + NT - 1) / NT;                  // per thread
    constexpr int GPIECES = KDA ? kTokChunk * D / 4 / NT : 0;      // float4 pieces of g (KDA) per thread
    static_assert(!KDA || GPIECES * 4 * NT == kTokChunk * D, "gate pieces");

    extern __shared__ __align__(16) float ps[];
    const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const int cg = lane % LPR;                                       // column piece index in the row block
    const int r0 = (tid / LPR) * 4;                                  // the block's first row
    const int lane0 = lane - cg;                                     // the row block's first lane
    const int units = a.w.units, b = u / a.heads;
    if (a.seq_mask != nullptr && a.seq_mask[b] == 0) return;       // sequence not restarted
    if (a.lengths != nullptr && threadIdx.x == 0)   // checked build: report a length outside 0..n_tokens
        in_bounds(a.w.err, a.lengths[b], 0, (long long)a.n_tokens + 1, u, -40);
    const int T = a.lengths != nullptr ? min(max(a.lengths[b], 0), a.n_tokens) : a.n_tokens;
    auto col = [&](int m) { return m * 4 * LPR + cg * 4; };          // first of 4 owned columns in piece m
    // after the butterfly this lane holds the sum of row r0 + mine
    const bool hb = (cg & (LPR / 2)) != 0, lb = (cg & (LPR / 4)) != 0;
    const int mine = (hb ? 2 : 0) + (lb ? 1 : 0);
    auto rows_reduce = [&](const float *v) -> float {
        float a0 = hb ? v[2] : v[0], a1 = hb ? v[3] : v[1];
        const float s0 = hb ? v[0] : v[2], s1 = hb ? v[1] : v[3];
        a0 += __shfl_xor_sync(0xffffffffu, s0, LPR / 2);
        a1 += __shfl_xor_sync(0xffffffffu, s1, LPR / 2);
        float c = lb ? a1 : a0;
        c += __shfl_xor_sync(0xffffffffu, lb ? a0 : a1, LPR / 4);
#pragma unroll
        for (int o = LPR / 8; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        return c;
    };

    // ---------------------------------------------------------------- state
    float2 S[4][MG][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MG; ++m) {
            float4 x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (a.S0 != nullptr) x = *reinterpret_cast<const float4 *>(a.S0 + ((size_t)u * D + r0 + i) * D + col(m));
            S[i][m][0] = make_float2(x.x, x.y);
            S[i][m][1] = make_float2(x.z, x.w);
        }

    // -------------------------------------------------------------- staging
    auto copy_chunk = [&](int t0) {               // raw copies; tokens past the prompt are not copied
        const int ne = min(kTokChunk, T - t0);
        unsigned char *rk = reinterpret_cast<unsigned char *>(ps + Sh::RK);
        unsigned char *rq = reinterpret_cast<unsigned char *>(ps + Sh::RQ);
        unsigned char *rv = reinterpret_cast<unsigned char *>(ps + Sh::RV);
#pragma unroll
        for (int p = 0; p < PIECES; ++p) {
            const int idx = p * NT + tid, e = idx / (D / VALS), j = (idx % (D / VALS)) * VALS;
            if (idx < TOTAL && e < ne) {
                const size_t off = ((size_t)(t0 + e) * units + u) * D + j;
                cp_async16(rk + 16 * idx, reinterpret_cast<const InT *>(a.k) + off);
                cp_async16(rq + 16 * idx, reinterpret_cast<const InT *>(a.q) + off);
                cp_async16(rv + 16 * idx, reinterpret_cast<const InT *>(a.v) + off);
            }
        }
        if constexpr (KDA) {
#pragma unroll
            for (int p = 0; p < GPIECES; ++p) {
                const int idx = p * NT + tid, e = idx / (D / 4), j = (idx % (D / 4)) * 4;
                if (e < ne) cp_async16(ps + Sh::RG + 4 * idx, a.g + ((size_t)(t0 + e) * units + u) * D + j);
            }
            if (tid < ne) cp_async4(ps + Sh::RB + tid, a.beta + (size_t)(t0 + tid) * units + u);
        } else {
            const int e = tid % kTokChunk;
            if (tid < 2 * kTokChunk && e < ne)
                cp_async4(ps + (tid < kTokChunk ? Sh::RG : Sh::RB) + e,
                          (tid < kTokChunk ? a.g : a.beta) + (size_t)(t0 + e) * units + u);
        }
    };
    // pass 1: the gate products c_t and 1/c_t of every channel (serial over the chunk)
    auto scan_chunk = [&](int t0) {
        const int ne = min(kTokChunk, T - t0);
        if (tid < GD) {
            float G = 0.0f;
            for (int e = 0; e < kTokChunk; ++e) {
                if (e < ne) G += ps[Sh::RG + e * GD + tid];
                ps[Sh::SC + e * GD + tid] = expf(G);
                ps[Sh::SCI + e * GD + tid] = expf(-G);
            }
            if (fabsf(G) > kMaxChunkLogGate) report_error(a.w.err, LQ_DEVERR_RANGE, u, t0);
        }
        if (tid < kTokChunk) ps[Sh::SB + tid] = ps[Sh::RB + tid];
    };
    // pass 2: c.k, k/c, c.q, v in FP32
    auto stage_chunk = [&]() {
#pragma unroll
        for (int p = 0; p < PIECES; ++p) {
            const int idx = p * NT + tid, e = idx / (D / VALS), j = (idx % (D / VALS)) * VALS;
            if (idx >= TOTAL) break;
            float kf[VALS], qf[VALS], vf[VALS];
            widen<InT>(reinterpret_cast<const uint4 *>(ps + Sh::RK)[idx], kf);
            widen<InT>(reinterpret_cast<const uint4 *>(ps + Sh::RQ)[idx], qf);
            widen<InT>(reinterpret_cast<const uint4 *>(ps + Sh::RV)[idx], vf);
#pragma unroll
            for (int x = 0; x < VALS; x += 4) {
                float c[4], ci[4];
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    c[y] = ps[Sh::SC + e * GD + (KDA ? j + x + y : 0)];
                    ci[y] = ps[Sh::SCI + e * GD + (KDA ? j + x + y : 0)];
                }
                const int o = e * D + j + x;
                *reinterpret_cast<float4 *>(ps + Sh::SKC + o) =
                    make_float4(c[0] * kf[x], c[1] * kf[x + 1], c[2] * kf[x + 2], c[3] * kf[x + 3]);
                *reinterpret_cast<float4 *>(ps + Sh::SKD + o) =
                    make_float4(ci[0] * kf[x], ci[1] * kf[x + 1], ci[2] * kf[x + 2], ci[3] * kf[x + 3]);
                *reinterpret_cast<float4 *>(ps + Sh::SQC + o) =
                    make_float4(c[0] * qf[x], c[1] * qf[x + 1], c[2] * qf[x + 2], c[3] * qf[x + 3]);
                *reinterpret_cast<float4 *>(ps + Sh::SV + o) = make_float4(vf[x], vf[x + 1], vf[x + 2], vf[x + 3]);
            }
        }
    };
    auto prepare = [&](int t0) {                  // the raw copy of chunk t0 has arrived for every thread
        scan_chunk(t0);
        __syncthreads();
        stage_chunk();
        __syncthreads();
    };

    // ----------------------------------------------------------- recurrence
    const int nch = (T + kTokChunk - 1) / kTokChunk;
    if (nch > 0) {
        copy_chunk(0);
        cp_async_wait_all();
        __syncthreads();
        prepare(0);
    }
    for (int ch = 0; ch < nch; ++ch) {
        const int t0 = ch * kTokChunk, ne = min(kTokChunk, T - t0);
        if (ch + 1 < nch) copy_chunk(t0 + kTokChunk);     // the raw area is free: its last copy is staged
        for (int e = 0; e < ne; ++e) {
            const float *kc = ps + Sh::SKC + e * D, *kd = ps + Sh::SKD + e * D, *qc = ps + Sh::SQC + e * D;
            // (S'_{t-1} (c_t . k_t)) of the block's rows
            float2 acc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int m = 0; m < MG; ++m) {
                const float4 x = *reinterpret_cast<const float4 *>(kc + col(m));
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[i] = __ffma2_rn(S[i][m][0], make_float2(x.x, x.y), acc[i]);
                    acc[i] = __ffma2_rn(S[i][m][1], make_float2(x.z, x.w), acc[i]);
                }
            }
            float part[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) part[i] = acc[i].x + acc[i].y;
            const float dot = rows_reduce(part);
            const float um = ps[Sh::SB + e] * (ps[Sh::SV + e * D + r0 + mine] - dot);
            float uu[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) uu[i] = __shfl_sync(0xffffffffu, um, lane0 + (i >> 1) * (LPR / 2) + (i & 1) * (LPR / 4));
            // S'_t = S'_{t-1} + u_t (k_t / c_t)^T, then (S'_t (c_t . q_t)) of the block's rows
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int m = 0; m < MG; ++m) {
                const float4 y = *reinterpret_cast<const float4 *>(kd + col(m));
                const float4 z = *reinterpret_cast<const float4 *>(qc + col(m));
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 u2 = make_float2(uu[i], uu[i]);
                    S[i][m][0] = __ffma2_rn(u2, make_float2(y.x, y.y), S[i][m][0]);
                    S[i][m][1] = __ffma2_rn(u2, make_float2(y.z, y.w), S[i][m][1]);
                    acc[i] = __ffma2_rn(S[i][m][0], make_float2(z.x, z.y), acc[i]);
                    acc[i] = __ffma2_rn(S[i][m][1], make_float2(z.z, z.w), acc[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) part[i] = acc[i].x + acc[i].y;
            const float o = rows_reduce(part);
            if ((cg & (LPR / 4 - 1)) == 0) ps[Sh::SO + e * D + r0 + mine] = o;
        }
        // back to the true state: S = S' diag(c at the chunk's last token)
        {
            const float *ce = ps + Sh::SC + (ne - 1) * GD;
#pragma unroll
            for (int m = 0; m < MG; ++m) {
                const float4 c = KDA ? *reinterpret_cast<const float4 *>(ce + col(m)) : make_float4(ce[0], ce[0], ce[0], ce[0]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    S[i][m][0] = __fmul2_rn(S[i][m][0], make_float2(c.x, c.y));
                    S[i][m][1] = __fmul2_rn(S[i][m][1], make_float2(c.z, c.w));
                }
            }
        }
        __syncthreads();                          // the chunk's outputs are complete
        if (a.o != nullptr) {
            for (int idx = tid; idx < ne * D / 4; idx += NT) {
                const int e = idx / (D / 4), j = (idx % (D / 4)) * 4;
                *reinterpret_cast<float4 *>(a.o + ((size_t)(t0 + e) * units + u) * D + j) =
                    *reinterpret_cast<const float4 *>(ps + Sh::SO + e * D + j);
            }
        }
        if (ch + 1 < nch) {
            cp_async_wait_all();
            __syncthreads();                      // chunk ch is applied and written; chunk ch + 1 has arrived
            prepare(t0 + kTokChunk);
        }
    }

    // ------------------------------------------------------- store or encode
    if (a.fp32_state) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < MG; ++m)
                *reinterpret_cast<float4 *>(a.w.state_f32 + ((size_t)u * D + r0 + i) * D + col(m)) =
                    make_float4(S[i][m][0].x, S[i][m][0].y, S[i][m][1].x, S[i][m][1].y);
        return;
    }
    __syncthreads();                              // the stages are no longer read
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int m = 0; m < MG; ++m)
            *reinterpret_cast<float4 *>(ps + (r0 + i) * D + col(m)) =
                make_float4(S[i][m][0].x, S[i][m][0].y, S[i][m][1].x, S[i][m][1].y);
    __syncthreads();
    if (a.fill != nullptr && tid == 0) a.fill[u] = 0;                // the unit's window starts empty
    constexpr int G = Tile<D>::G, NR = Tile<D>::NR;
    Tile<D> Tl;
    Tl.tid = tid;
    Tl.tx = tid & 15;
    Tl.ty = tid >> 4;
#pragma unroll
    for (int i = 0; i < NR; ++i)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float4 x = *reinterpret_cast<const float4 *>(ps + Tl.row(i) * D + g * 64 + Tl.tx * 4);
            Tl.acc[i][g * 2] = make_float2(x.x, x.y);
            Tl.acc[i][g * 2 + 1] = make_float2(x.z, x.w);
        }
    codec_store<D, KDA>(Tl, u, a.w, a.n_rows, a.n_cols, a.smooth, a.select, ps);   // begins with a barrier
}

template <int D, bool KDA, typename InT>
cudaError_t launch_t(const TokenPrefillArgs &a, cudaStream_t s) {
    using Sh = TokShape<D, KDA, (int)sizeof(InT)>;
    auto kern = prefill_tokens_kernel<D, KDA, InT>;
    const int smem = 4 * Sh::WORDS;
    const cudaError_t e = opt_in_smem<prefill_tokens_kernel<D, KDA, InT>>(smem);
    if (e != cudaSuccess) return e;
    kern<<<a.w.units, Sh::NT, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tokens(const TokenPrefillArgs &a, int d, int gate, int in_dtype, cudaStream_t s) {
    if (a.n_tokens < 0 || a.w.units <= 0) return cudaErrorInvalidValue;
    const bool kda = (gate == LQ_GATE_CHANNEL);
    const bool bf = (in_dtype == LQ_DTYPE_BF16);
    if (d == 128) {
        if (kda) return bf ? launch_t<128, true, __nv_bfloat16>(a, s) : launch_t<128, true, float>(a, s);
        return bf ? launch_t<128, false, __nv_bfloat16>(a, s) : launch_t<128, false, float>(a, s);
    }
    if (d == 64) {
        if (kda) return bf ? launch_t<64, true, __nv_bfloat16>(a, s) : launch_t<64, true, float>(a, s);
        return bf ? launch_t<64, false, __nv_bfloat16>(a, s) : launch_t<64, false, float>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lq
