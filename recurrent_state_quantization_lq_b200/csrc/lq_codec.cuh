// The state codec on a tile held in registers (sm_100a), shared by the
// prefill, token-prefill and window-flush kernels.
//
// LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent
// State Quantization", section "Abstract (arXiv)") keeps the state's largest
// outliers as high-precision Compensator Tokens and smooths the remaining
// residual before quantizing it.  Per (sequence, head) unit, on the FP32 state:
//   2. compensator rows (largest L2 norm, or max-abs), then columns of the
//      row-zeroed residual, stored as FP32 pairs and zeroed;
//   3. s_j = sqrt(max_i |R_ij|) (1 for an empty column);
//   4. R'_ij = R_ij * (1/s_j), M_i = max_j |R'_ij|, sigma_i = M_i / 127,
//      Q_ij = rint(R'_ij * (127 / M_i)).
// Every value that decides a code is computed with IEEE round-to-nearest FP32
// operations (square root, one division per column and per row, products
// without fused adds), so a given FP32 state always encodes to the same codes,
// scales and smoothing factors.
//
// The tile lives in registers: kTile = 256 threads in a 16 x 16 grid, thread
// (ty, tx) owning rows g*64 + ty*4 + r and columns g*64 + tx*4 + c (g < d/64,
// r, c < 4), as column pairs so a rank update runs on packed FP32 FMAs.
#pragma once

#include "lq_common.cuh"
#include "lq_select.cuh"

namespace lq {

constexpr int kTile = 256;                // threads holding the tile
constexpr int kTileBarrier = 1;           // named barrier of those threads

__device__ __forceinline__ void tile_sync() {
    asm volatile("bar.sync %0, %1;" ::"r"(kTileBarrier), "r"(kTile) : "memory");
}

// Codec scratch in shared memory (floats): per-warp column partial sums and
// maxima (8 x D each), column scores, column maxima, reciprocal smoothing factors.
template <int D>
struct CodecScratch {
    static constexpr int PSUM = 0, PMAX = 8 * D, SCORE = 16 * D, CMAX = 17 * D, RS = 18 * D, FLOATS = 19 * D;
};

template <int D>
struct Tile {
    static constexpr int G = D / 64;
    static constexpr int NR = 4 * G;      // rows (and columns) a thread owns
    float2 acc[NR][NR / 2];
    int tx, ty, tid;
    __device__ __forceinline__ int row(int r) const { return (r >> 2) * 64 + ty * 4 + (r & 3); }
    __device__ __forceinline__ int col(int c) const { return (c >> 2) * 64 + tx * 4 + (c & 3); }
    __device__ __forceinline__ float &at(int r, int c) { return (c & 1) ? acc[r][c >> 1].y : acc[r][c >> 1].x; }
};

// Steps 2-4 of the codec on the tile in registers, plus the stores.  Called by
// exactly the kTile tile threads (tid < kTile).
template <int D, bool KDA>
__device__ __forceinline__ void codec_store(Tile<D> &T, int u, const Views &w, int n_rows, int n_cols, int smooth,
                                            int select, float *scratch) {
    using CS = CodecScratch<D>;
    constexpr int G = Tile<D>::G, NR = Tile<D>::NR;
    float *sh_psum = scratch + CS::PSUM, *sh_pmax = scratch + CS::PMAX, *sh_score = scratch + CS::SCORE;
    float *sh_cmax = scratch + CS::CMAX, *sh_rs = scratch + CS::RS;
    const int tid = T.tid, tx = T.tx, ty = T.ty, lane = tid & 31;
    const bool l2 = (select == LQ_SELECT_L2);
    int32_t *cidx = w.comp_index + (size_t)u * w.comp_index_stride;
    tile_sync();   // the scratch of the previous unit is free

    // ------------------------------------------------- 2a. compensator rows
    if (n_rows > 0) {
        if (l2) {                                 // one branch per ranking, taken by every thread alike
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                float p = 0.0f;
#pragma unroll
                for (int c = 0; c < NR; ++c) {
                    const float x = fabsf(T.at(r, c));
                    p = p + x * x;
                }
                p = group_sum<16>(p);
                if (tx == 0) sh_score[T.row(r)] = p;
            }
        } else {
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                float p = 0.0f;
#pragma unroll
                for (int c = 0; c < NR; ++c) p = fmaxf(p, fabsf(T.at(r, c)));
                p = group_max<16>(p);
                if (tx == 0) sh_score[T.row(r)] = p;
            }
        }
        tile_sync();
        const uint2 sel = select_top<D>(sh_score, n_rows);
        if (tid == 0) {
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c < n_rows) cidx[c] = sel_at(sel, c);
        }
        // row i is held by the threads with ty = (i / 4) mod 16, as their row
        // (i / 64) * 4 + i mod 4; only they store and clear it
        for (int c = 0; c < n_rows; ++c) {
            const int i = sel_at(sel, c);
            if (((i >> 2) & 15) != ty) continue;
            const int ri = ((i >> 6) << 2) | (i & 3);
            float *dst = w.comp_row_vec + ((size_t)u * n_rows + c) * D;
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                if (r != ri) continue;
#pragma unroll
                for (int g = 0; g < G; ++g)
                    *reinterpret_cast<float4 *>(dst + g * 64 + tx * 4) =
                        make_float4(T.at(r, g * 4), T.at(r, g * 4 + 1), T.at(r, g * 4 + 2), T.at(r, g * 4 + 3));
#pragma unroll
                for (int m = 0; m < NR / 2; ++m) T.acc[r][m] = make_float2(0.0f, 0.0f);
            }
        }
    }

    // ------------------- 2b, 3. column statistics of the row-zeroed residual
    // One pass gives each column's score (sum of squares, or max) and its max.
    // Zeroing the chosen columns leaves the other columns' maxima unchanged
    // and makes their own zero, so the smoothing factors follow from the same pass.
#pragma unroll
    for (int c = 0; c < NR; ++c) {
        float sq = 0.0f, mx = 0.0f;
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const float x = fabsf(T.at(r, c));
            sq = sq + x * x;
            mx = fmaxf(mx, x);
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 16);          // the warp's two rows of tx groups
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (lane < 16) {
            sh_psum[(ty >> 1) * D + T.col(c)] = sq;
            sh_pmax[(ty >> 1) * D + T.col(c)] = mx;
        }
    }
    tile_sync();
    for (int j = tid; j < D; j += kTile) {
        float sq = 0.0f, mx = 0.0f;
#pragma unroll
        for (int y = 0; y < 8; ++y) {
            sq += sh_psum[y * D + j];
            mx = fmaxf(mx, sh_pmax[y * D + j]);
        }
        sh_score[j] = l2 ? sq : mx;
        sh_cmax[j] = mx;
    }
    tile_sync();
    const uint2 csel = select_top<D>(sh_score, n_cols);
    if (tid == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if (c < n_cols) cidx[n_rows + c] = sel_at(csel, c);
    }
    for (int j = tid; j < D; j += kTile) {
        bool chosen = false;
#pragma unroll
        for (int c = 0; c < 8; ++c) chosen |= (c < n_cols && sel_at(csel, c) == j);
        const float m = chosen ? 0.0f : sh_cmax[j];
        const float s = (smooth && m > 0.0f) ? __fsqrt_rn(m) : 1.0f;
        sh_rs[j] = __fdiv_rn(1.0f, s);          // applied as a multiplication
        if (w.col_smooth != nullptr) w.col_smooth[(size_t)u * D + j] = s;
    }
    // column j is held by the threads with tx = (j / 4) mod 16, as their
    // column (j / 64) * 4 + j mod 4; only they store and clear it
    for (int cc = 0; cc < n_cols; ++cc) {
        const int j = sel_at(csel, cc);
        if (((j >> 2) & 15) != tx) continue;
        const int cj = ((j >> 6) << 2) | (j & 3);
        float *dst = w.comp_col_vec + ((size_t)u * n_cols + cc) * D;
#pragma unroll
        for (int c = 0; c < NR; ++c) {
            if (c != cj) continue;
#pragma unroll
            for (int g = 0; g < G; ++g)
                *reinterpret_cast<float4 *>(dst + g * 64 + ty * 4) =
                    make_float4(T.at(g * 4, c), T.at(g * 4 + 1, c), T.at(g * 4 + 2, c), T.at(g * 4 + 3, c));
#pragma unroll
            for (int r = 0; r < NR; ++r) T.at(r, c) = 0.0f;
        }
    }
    tile_sync();

    // ------------------------------------------ 4. row scales and the codes
    float rs[NR];
#pragma unroll
    for (int c = 0; c < NR; ++c) rs[c] = sh_rs[T.col(c)];
    float m[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        float mm = 0.0f;
#pragma unroll
        for (int c = 0; c < NR; ++c) {
            T.at(r, c) = __fmul_rn(T.at(r, c), rs[c]);
            mm = fmaxf(mm, fabsf(T.at(r, c)));
        }
        m[r] = group_max<16>(mm);
    }
    // lane tx divides for row tx mod NR of its group; the rest take rho by shuffle
    float mine = m[0];
#pragma unroll
    for (int r = 1; r < NR; ++r) mine = ((tx & (NR - 1)) == r) ? m[r] : mine;
    const float rho_mine = (mine > 0.0f) ? __fdiv_rn(127.0f, mine) : 0.0f;
    if (tx < NR) w.row_scale[(size_t)u * D + T.row(tx)] = __fdiv_rn(mine, 127.0f);
    int8_t *Qu = w.codes + (size_t)u * D * D;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        const float rho = __shfl_sync(0xffffffffu, rho_mine, (lane & 16) + r);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            // rint by adding 1.5 * 2^23 (|x| <= 127.5 here, so the sum is exact
            // up to the one rounding to an integer, to nearest, ties to even);
            // the code is then the low byte of the sum's bit pattern.  |x rho|
            // never exceeds 127 (rho = 127 / max of the row), so no clamp is needed.
            uint32_t b[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                b[c] = __float_as_uint(__fadd_rn(__fmul_rn(T.at(r, g * 4 + c), rho), 12582912.0f));
            const uint32_t word = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
            *reinterpret_cast<uint32_t *>(Qu + (size_t)T.row(r) * D + g * 64 + tx * 4) = word;
        }
    }

    // -------------------------------------------- 5. start the next window
    if (w.gate_sum != nullptr) {
        const int gd = KDA ? D : 1;
        for (int j = tid; j < gd; j += kTile) w.gate_sum[(size_t)u * gd + j] = 0.0;
    }
}

}  // namespace lq
