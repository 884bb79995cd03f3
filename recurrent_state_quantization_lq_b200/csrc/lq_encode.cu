// State codec kernel: prefill ingestion and window flush.
//
// LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent
// State Quantization", section "Abstract (arXiv)") quantizes the state only
// once, at the end of each window; before that it keeps the state's largest
// outliers as high-precision Compensator Tokens and smooths the remaining
// residual.  One CTA per (sequence, head):
//   1. rebuild the end-of-window state in FP32 registers,
//        R = (R^ + C) diag(gamma_W) + sum_j delta_j (kappa_j * gamma_W)^T,
//      a rank-(n_c + n_buf) update of the dequantized window-start state
//      (compensators enter as buffered pairs with G = 0), or take the
//      prefilled state as given;
//   2. compensator rows (largest L2 norm, or max-abs), then columns of the
//      row-zeroed residual, stored as FP32 pairs and zeroed;
//   3. s_j = sqrt(max_i |R_ij|) (1 for an empty column);
//   4. R'_ij = R_ij * (1/s_j), M_i = max_j |R'_ij|, sigma_i = M_i / 127,
//      Q_ij = rint(R'_ij * (127 / M_i)).
// Every value that decides a code is computed with IEEE round-to-nearest FP32
// operations (square root, one division per column and per row, products
// without fused adds), so a given FP32 state always encodes to the same codes,
// scales and smoothing factors.
#include "lq_kernels.h"

namespace lq {
namespace {

constexpr int kEncThreads = 256;  // 16 x 16 thread grid over the d x d tile
constexpr int kEncChunk = 16;     // buffered entries staged in shared memory per step

template <int D>
struct EncShape {
    static constexpr int G = D / 64;   // 64-wide groups of rows / columns per thread
    static constexpr int NR = 4 * G;   // rows (and columns) a thread owns
    // thread (ty, tx) owns rows  g*64 + ty*4 + r  and columns  g*64 + tx*4 + c
    static constexpr size_t smem_bytes =
        sizeof(float) * (2 * kEncChunk * D + 16 * D + 3 * D + kEncChunk) + sizeof(int) * 32;
};

// Warp-wide argmax over `n` scores with ties to the lower index; entries with
// score < 0 are excluded.  Every lane returns the winner.
__device__ int warp_argmax(const float *score, int n) {
    const int lane = threadIdx.x & 31;
    float best = -1.0f;
    int bi = 0x7fffffff;
    for (int i = lane; i < n; i += 32) {
        float s = score[i];
        if (s > best) { best = s; bi = i; }   // i increases: strict '>' keeps the lower index
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float ob = __shfl_xor_sync(0xffffffffu, best, o);
        int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    return bi;
}

template <int D, bool KDA, typename KeyT>
__global__ void __launch_bounds__(kEncThreads, 2) encode_kernel(EncodeArgs a) {
    using Sh = EncShape<D>;
    constexpr int G = Sh::G, NR = Sh::NR;
    const int u = blockIdx.x;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const Views &w = a.w;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *sh_delta = reinterpret_cast<float *>(smem_raw);    // [chunk][D]
    float *sh_kap = sh_delta + kEncChunk * D;                   // [chunk][D]
    float *sh_part = sh_kap + kEncChunk * D;                    // [16][D]
    float *sh_gam = sh_part + 16 * D;                           // [D] gamma_W per key channel
    float *sh_score = sh_gam + D;                               // [D]
    float *sh_s = sh_score + D;                                 // [D] 1 / smoothing factor
    float *sh_fac = sh_s + D;                                   // [chunk]
    int *sh_sel = reinterpret_cast<int *>(sh_fac + kEncChunk);  // [32]: rows then columns

    auto row_of = [&](int r) { return (r >> 2) * 64 + ty * 4 + (r & 3); };
    auto col_of = [&](int c) { return (c >> 2) * 64 + tx * 4 + (c & 3); };

    // The tile lives in registers as column pairs so the rank update can use
    // packed FP32 FMAs; ACC(r, c) names one element.
    float2 acc2[NR][NR / 2];
#define ACC(r, c) ((((c) & 1) != 0) ? acc2[r][(c) >> 1].y : acc2[r][(c) >> 1].x)

    // ------------------------------------------------------------ 1. rebuild
    if (!a.from_buffer) {
        if (a.S0 != nullptr) {
            const float *S0 = a.S0 + (size_t)u * D * D;
#pragma unroll
            for (int r = 0; r < NR; ++r)
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float4 x = *reinterpret_cast<const float4 *>(S0 + (size_t)row_of(r) * D + g * 64 + tx * 4);
                    ACC(r, g * 4 + 0) = x.x; ACC(r, g * 4 + 1) = x.y;
                    ACC(r, g * 4 + 2) = x.z; ACC(r, g * 4 + 3) = x.w;
                }
        } else {
#pragma unroll
            for (int r = 0; r < NR; ++r)
#pragma unroll
                for (int c = 0; c < NR; ++c) ACC(r, c) = 0.0f;
        }
    } else {
        // gamma_W per key channel (scalar gate: one value for all)
        double GW_scalar = 0.0;
        if (KDA) {
            for (int j = tid; j < D; j += kEncThreads) sh_gam[j] = (float)exp(w.gate_sum[(size_t)u * D + j]);
        } else {
            GW_scalar = w.gate_sum[u];
            for (int j = tid; j < D; j += kEncThreads) sh_gam[j] = (float)exp(GW_scalar);
        }
        __syncthreads();
        // dequantized window-start state, decayed: sigma_i Q_ij (s_j gamma_j)
        const int8_t *Qu = w.codes + (size_t)u * D * D;
        const float *sig = w.row_scale + (size_t)u * D;
        const float *sm = w.col_smooth + (size_t)u * D;
        float sg[NR];
#pragma unroll
        for (int c = 0; c < NR; ++c) sg[c] = sm[col_of(c)] * sh_gam[col_of(c)];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const float si = sig[row_of(r)];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                uint32_t word = *reinterpret_cast<const uint32_t *>(Qu + (size_t)row_of(r) * D + g * 64 + tx * 4);
                float f0, f1, f2, f3;
                i8x4_to_f32(word, f0, f1, f2, f3);
                ACC(r, g * 4 + 0) = (si * f0) * sg[g * 4 + 0];
                ACC(r, g * 4 + 1) = (si * f1) * sg[g * 4 + 1];
                ACC(r, g * 4 + 2) = (si * f2) * sg[g * 4 + 2];
                ACC(r, g * 4 + 3) = (si * f3) * sg[g * 4 + 3];
            }
        }
        // compensators (entries with G = 0), then the buffered tokens
        const int ncomp = w.n_comp_rows + w.n_comp_cols;
        const int total = ncomp + a.n_buf;
        const int32_t *cidx = w.comp_index + (size_t)u * w.comp_index_stride;
        for (int e0 = 0; e0 < total; e0 += kEncChunk) {
            const int ne = min(kEncChunk, total - e0);
            if (!KDA && tid < ne) {
                const int e = e0 + tid;
                // buffered tokens carry omega_j = exp(-G_j): factor exp(G_W - G_j) = gamma_W omega_j
                const float gW = (float)exp(GW_scalar);
                sh_fac[tid] = (e < ncomp) ? gW : gW * w.buf_gate[(size_t)u * w.window_pad + (e - ncomp)];
            }
            __syncthreads();
            for (int idx = tid; idx < ne * D; idx += kEncThreads) {
                const int el = idx / D, j = idx - el * D, e = e0 + el;
                float dv, kv;
                if (e < w.n_comp_rows) {                       // row compensator (e_i, k_c)
                    dv = (j == cidx[e]) ? 1.0f : 0.0f;
                    kv = w.comp_row_vec[((size_t)u * w.n_comp_rows + e) * D + j] * sh_gam[j];
                } else if (e < ncomp) {                        // column compensator (v_c, e_j)
                    const int c = e - w.n_comp_rows;
                    dv = w.comp_col_vec[((size_t)u * w.n_comp_cols + c) * D + j];
                    kv = (j == cidx[w.n_comp_rows + c]) ? sh_gam[j] : 0.0f;
                } else {                                       // buffered token
                    const size_t slot = (size_t)u * w.window + (e - ncomp);
                    dv = w.buf_delta[slot * D + j];
                    if (KDA) {
                        kv = reinterpret_cast<const float *>(w.buf_key)[slot * D + j] * sh_gam[j];
                    } else {
                        const KeyT *kp = reinterpret_cast<const KeyT *>(w.buf_key) + slot * D + j;
                        kv = static_cast<float>(*kp) * sh_fac[el];
                    }
                }
                sh_delta[el * D + j] = dv;
                sh_kap[el * D + j] = kv;
            }
            __syncthreads();
            for (int el = 0; el < ne; ++el) {
                float dr[NR];
                float2 kc[NR / 2];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float4 x = *reinterpret_cast<const float4 *>(sh_delta + el * D + g * 64 + ty * 4);
                    float4 y = *reinterpret_cast<const float4 *>(sh_kap + el * D + g * 64 + tx * 4);
                    dr[g * 4 + 0] = x.x; dr[g * 4 + 1] = x.y; dr[g * 4 + 2] = x.z; dr[g * 4 + 3] = x.w;
                    kc[g * 2 + 0] = make_float2(y.x, y.y);
                    kc[g * 2 + 1] = make_float2(y.z, y.w);
                }
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float2 dd = make_float2(dr[r], dr[r]);
#pragma unroll
                    for (int m = 0; m < NR / 2; ++m) acc2[r][m] = __ffma2_rn(dd, kc[m], acc2[r][m]);
                }
            }
            __syncthreads();
        }
    }

    // ------------------------------------------------- 2a. compensator rows
    if (a.n_rows > 0) {
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            float p = 0.0f;
#pragma unroll
            for (int c = 0; c < NR; ++c) {
                const float x = fabsf(ACC(r, c));
                p = (a.select == LQ_SELECT_L2) ? p + x * x : fmaxf(p, x);
            }
            p = (a.select == LQ_SELECT_L2) ? group_sum<16>(p) : group_max<16>(p);
            if (tx == 0) sh_score[row_of(r)] = p;
        }
        __syncthreads();
        if (tid < 32) {
            for (int c = 0; c < a.n_rows; ++c) {
                const int i = warp_argmax(sh_score, D);
                if (tid == 0) {
                    sh_sel[c] = i;
                    sh_score[i] = -1.0f;
                    w.comp_index[(size_t)u * w.comp_index_stride + c] = i;
                }
                __syncwarp();
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            for (int c = 0; c < a.n_rows; ++c) {
                if (sh_sel[c] == row_of(r)) {
                    float *dst = w.comp_row_vec + ((size_t)u * a.n_rows + c) * D;
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        *reinterpret_cast<float4 *>(dst + g * 64 + tx * 4) =
                            make_float4(ACC(r, g * 4), ACC(r, g * 4 + 1), ACC(r, g * 4 + 2), ACC(r, g * 4 + 3));
#pragma unroll
                    for (int cc = 0; cc < NR; ++cc) ACC(r, cc) = 0.0f;
                }
            }
        }
    }

    // ---------------------------------------------- 2b. compensator columns
    if (a.n_cols > 0) {
#pragma unroll
        for (int c = 0; c < NR; ++c) {
            float p = 0.0f;
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const float x = fabsf(ACC(r, c));
                p = (a.select == LQ_SELECT_L2) ? p + x * x : fmaxf(p, x);
            }
            sh_part[ty * D + col_of(c)] = p;
        }
        __syncthreads();
        for (int j = tid; j < D; j += kEncThreads) {
            float p = 0.0f;
            for (int y = 0; y < 16; ++y) {
                const float x = sh_part[y * D + j];
                p = (a.select == LQ_SELECT_L2) ? p + x : fmaxf(p, x);
            }
            sh_score[j] = p;
        }
        __syncthreads();
        if (tid < 32) {
            for (int c = 0; c < a.n_cols; ++c) {
                const int j = warp_argmax(sh_score, D);
                if (tid == 0) {
                    sh_sel[16 + c] = j;
                    sh_score[j] = -1.0f;
                    w.comp_index[(size_t)u * w.comp_index_stride + a.n_rows + c] = j;
                }
                __syncwarp();
            }
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < NR; ++c) {
            for (int cc = 0; cc < a.n_cols; ++cc) {
                if (sh_sel[16 + cc] == col_of(c)) {
                    float *dst = w.comp_col_vec + ((size_t)u * a.n_cols + cc) * D;
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        *reinterpret_cast<float4 *>(dst + g * 64 + ty * 4) =
                            make_float4(ACC(g * 4, c), ACC(g * 4 + 1, c), ACC(g * 4 + 2, c), ACC(g * 4 + 3, c));
#pragma unroll
                    for (int r = 0; r < NR; ++r) ACC(r, c) = 0.0f;
                }
            }
        }
    }

    // ------------------------------------------------------- 3. smoothing
#pragma unroll
    for (int c = 0; c < NR; ++c) {
        float m = 0.0f;
#pragma unroll
        for (int r = 0; r < NR; ++r) m = fmaxf(m, fabsf(ACC(r, c)));
        sh_part[ty * D + col_of(c)] = m;
    }
    __syncthreads();
    for (int j = tid; j < D; j += kEncThreads) {
        float m = 0.0f;
        for (int y = 0; y < 16; ++y) m = fmaxf(m, sh_part[y * D + j]);
        const float s = (a.smooth && m > 0.0f) ? __fsqrt_rn(m) : 1.0f;
        sh_s[j] = __fdiv_rn(1.0f, s);          // applied as a multiplication
        if (w.col_smooth != nullptr) w.col_smooth[(size_t)u * D + j] = s;
    }
    __syncthreads();

    // ------------------------------------------ 4. row scales and the codes
    // R'_ij = R_ij * (1/s_j); M_i = max_j |R'_ij|; sigma_i = M_i / 127;
    // Q_ij = rint(R'_ij * (127 / M_i)).
    float rs[NR];
#pragma unroll
    for (int c = 0; c < NR; ++c) rs[c] = sh_s[col_of(c)];
    int8_t *Qu = w.codes + (size_t)u * D * D;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        float m = 0.0f;
#pragma unroll
        for (int c = 0; c < NR; ++c) {
            ACC(r, c) = __fmul_rn(ACC(r, c), rs[c]);
            m = fmaxf(m, fabsf(ACC(r, c)));
        }
        m = group_max<16>(m);
        const float sigma = __fdiv_rn(m, 127.0f);
        const float rho = (m > 0.0f) ? __fdiv_rn(127.0f, m) : 0.0f;
        if (tx == 0) w.row_scale[(size_t)u * D + row_of(r)] = sigma;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            uint32_t word = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float code = fminf(fmaxf(rintf(__fmul_rn(ACC(r, g * 4 + c), rho)), -127.0f), 127.0f);
                word |= (uint32_t)((int)code & 0xff) << (8 * c);
            }
            *reinterpret_cast<uint32_t *>(Qu + (size_t)row_of(r) * D + g * 64 + tx * 4) = word;
        }
    }

    // -------------------------------------------- 5. start the next window
    if (w.gate_sum != nullptr) {
        const int gd = KDA ? D : 1;
        for (int j = tid; j < gd; j += kEncThreads) w.gate_sum[(size_t)u * gd + j] = 0.0;
    }
#undef ACC
}

template <int D, bool KDA, typename KeyT>
cudaError_t launch_encode_t(const EncodeArgs &a, cudaStream_t s) {
    const size_t smem = EncShape<D>::smem_bytes;
    encode_kernel<D, KDA, KeyT><<<a.w.units, kEncThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode(const EncodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s) {
    const bool kda = (gate == LQ_GATE_CHANNEL);
    const bool bf = (in_dtype == LQ_DTYPE_BF16);
    if (d == 128) {
        if (kda) return launch_encode_t<128, true, float>(a, s);
        return bf ? launch_encode_t<128, false, __nv_bfloat16>(a, s) : launch_encode_t<128, false, float>(a, s);
    }
    if (d == 64) {
        if (kda) return launch_encode_t<64, true, float>(a, s);
        return bf ? launch_encode_t<64, false, __nv_bfloat16>(a, s) : launch_encode_t<64, false, float>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lq
