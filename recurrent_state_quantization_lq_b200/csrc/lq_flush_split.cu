// Window flush for ragged window phases: one thread-block cluster per unit.
//
// LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent
// State Quantization", section "Abstract (arXiv)") re-quantizes a state once
// per window.  When every sequence keeps its own window phase, only the units
// whose window is due are flushed at a step: with B sequences and windows of W
// tokens, about B / W sequences' heads.  One CTA per unit would leave most SMs
// idle and put a whole unit's rebuild and codec on one SM's critical path.
//
// Here a cluster of C = D / 16 CTAs shares a unit.  CTA r owns state rows
// 16 r .. 16 r + 15 (all columns): it dequantizes them, adds the compensators,
// applies the rank-n update and the window's decay, and encodes them.  The
// codec's statistics across rows travel through distributed shared memory:
//   * the row scores that choose compensator rows (each CTA sends its 16),
//   * per-column sums of squares and maxima of the row-zeroed residual, which
//     choose compensator columns and give the smoothing factors (each CTA
//     sends its partials over its 16 rows).
// Every CTA reduces the exchanged values in the same fixed order, so all CTAs
// of a cluster take the same decisions.  The arithmetic of each element is
// the one-CTA flush's (same dequantization, same entry order of FP32 fused
// multiply-adds, same decay); only the order of the cross-row sums differs.
//
// Clusters are persistent.  Cluster k takes units k, k + K, k + 2K, ... (K
// clusters) and reads the buffered counts of up to 128 of them in one parallel
// load, so the units that are due (often a contiguous run of one sequence's
// heads) spread over the clusters and the scan costs one memory round trip.
// Nothing waits on a flag: the only waits are the cluster barriers, which all
// CTAs of a cluster reach the same number of times.
#include <cooperative_groups.h>

#include "lq_kernels.h"
#include "lq_select.cuh"

namespace lq {
namespace {

namespace cg = cooperative_groups;

constexpr int kRows = 16;         // state rows per CTA
constexpr int kThreads = 128;     // 4 warps x 4 rows; lane l owns columns l*CL .. l*CL + CL - 1
// 16-byte pieces of a unit's compensator data per thread: 16 indices, 8 rows
// of D, 8 column slices of kRows
constexpr int kMetaPieces = (4 + 8 * 128 / 4 + 8 * kRows / 4 + kThreads - 1) / kThreads;

template <int D, int KB>
struct SplitShape {
    static constexpr int C = D / kRows;                 // CTAs per cluster
    static constexpr int CL = D / 32;                   // columns per lane
    // buffered entries staged per pass (a second pass loads while the first
    // computes; staging a whole 64-entry window at once measured no faster and
    // fits fewer CTAs on an SM)
    static constexpr int CH = 32;
    static constexpr int DP = CH * 4 / kThreads;        // 16-byte delta pieces per thread
    // shared memory, in 4-byte words
    static constexpr int KAP = 0;                       // [CH][D] omega_j k_j (KDA: kappa_j)
    static constexpr int WSQ = 0;                       // [4][D] per-warp column partials (after the
    static constexpr int WMX = WSQ + 4 * D;             //   rank update, in the staging area)
    static constexpr int DEL = KAP + CH * D;            // [CH][kRows] this CTA's rows of delta_j
    static constexpr int META = DEL + CH * kRows;       // comp_index [cis], rows [n_r][D], columns [n_c][kRows]
    static constexpr int RSCORE = META + 16 + 8 * D + 8 * kRows;   // [2][D] row scores (exchanged)
    static constexpr int CSQ = RSCORE + 2 * D;          // [2][C][D] column sums of squares (exchanged)
    static constexpr int CMX = CSQ + 2 * C * D;         // [2][C][D] column maxima (exchanged)
    static constexpr int SCORE = CMX + 2 * C * D;       // [D] column scores
    static constexpr int CMAX = SCORE + D;              // [D] column maxima
    static constexpr int RS = CMAX + D;                 // [D] 1 / s_j
    static constexpr int LIST = RS + D;                 // [kThreads] buffered counts of candidate units
    static constexpr int BALLOT = LIST + kThreads;      // [4] due-unit masks
    static constexpr int WORDS = BALLOT + 4;
    static_assert(DP * kThreads == CH * 4, "16-byte delta pieces");
    static_assert(8 * D <= CH * D, "column partials fit the staging area");
};

template <int D, bool KDA, typename KeyT>
__global__ void __launch_bounds__(kThreads) flush_split_kernel(EncodeArgs a) {
    constexpr int KB = (int)sizeof(KeyT);
    using Sh = SplitShape<D, KB>;
    constexpr int C = Sh::C, CL = Sh::CL, CH = Sh::CH, DP = Sh::DP;
    constexpr int PER_ENTRY = D * KB / 16;                       // 16-byte pieces of one key
    constexpr int PIECES = CH * PER_ENTRY / kThreads;            // key pieces per thread and pass
    constexpr int VALS = 16 / KB;                                // key values per piece
    static_assert(PIECES * kThreads == CH * PER_ENTRY, "key pieces");

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int cid = (int)blockIdx.x / C, ncl = (int)gridDim.x / C;
    const Views &w = a.w;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ncr = w.n_comp_rows, ncc = w.n_comp_cols, cis = w.comp_index_stride;
    const int W = w.window;
    const bool l2 = (a.select == LQ_SELECT_L2);
    const int row0 = rank * kRows + warp * 4;    // this thread's rows row0 .. row0 + 3
    const int col0 = lane * CL;                  // and columns col0 .. col0 + CL - 1

    extern __shared__ __align__(16) float fs[];
    float *kap = fs + Sh::KAP, *dl = fs + Sh::DEL, *meta = fs + Sh::META;
    float *wsq = fs + Sh::WSQ, *wmx = fs + Sh::WMX;
    float *sh_score = fs + Sh::SCORE, *sh_cmax = fs + Sh::CMAX, *sh_rs = fs + Sh::RS;
    int *nlist = reinterpret_cast<int *>(fs + Sh::LIST);
    uint32_t *ballots = reinterpret_cast<uint32_t *>(fs + Sh::BALLOT);
    int parity = 0;                              // exchange buffers of the current unit

    const int per = (w.units - cid + ncl - 1) / ncl;     // this cluster's candidate units (cid < units)
    for (int p0 = 0; p0 < per; p0 += kThreads) {
        // ------------------------------------ which candidates are due
        const int k = p0 + tid;
        const int n = (k < per) ? a.fill[cid + k * ncl] : 0;
        if (k < per) in_bounds(w.err, n, 0, (long long)w.window + 1, cid + k * ncl, -30);   // checked build: report
        const bool due = (k < per) && n >= a.flush_min;
        const uint32_t mask = __ballot_sync(0xffffffffu, due);
        if (lane == 0) ballots[warp] = mask;
        nlist[tid] = n;
        __syncthreads();
        for (int wq = 0; wq < kThreads / 32; ++wq) {
            uint32_t bits = ballots[wq];
            while (bits != 0u) {
                const int kk = wq * 32 + __ffs(bits) - 1;
                bits &= bits - 1u;
                const int u = cid + (p0 + kk) * ncl;
                const int n_buf = min(nlist[kk], W);
                const int nch = (n_buf + CH - 1) / CH;
                const KeyT *keys = reinterpret_cast<const KeyT *>(w.buf_key) + (size_t)u * W * D;

                // ---------------- one round of loads: compensators and their
                // indices, this CTA's rows, its scales, the gate sum, chunk 0
                const int n_meta = cis / 4 + ncr * (D / 4) + ncc * (kRows / 4);   // 16-byte pieces
                float4 mv[kMetaPieces];
#pragma unroll
                for (int j = 0; j < kMetaPieces; ++j) {
                    const int idx = tid + j * kThreads;
                    mv[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (idx < n_meta) {
                        const float *src;
                        const int r1 = idx - cis / 4, r2 = r1 - ncr * (D / 4);
                        if (r1 < 0) src = reinterpret_cast<const float *>(w.comp_index + (size_t)u * cis) + 4 * idx;
                        else if (r2 < 0) src = w.comp_row_vec + (size_t)u * ncr * D + 4 * r1;
                        else src = w.comp_col_vec + ((size_t)u * ncc + (r2 >> 2)) * D + rank * kRows + 4 * (r2 & 3);
                        mv[j] = *reinterpret_cast<const float4 *>(src);
                    }
                }
                float sc[CL], si[4];
                uint32_t word[4];
#pragma unroll
                for (int c = 0; c < CL; ++c) sc[c] = w.col_smooth[(size_t)u * D + col0 + c];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    si[i] = w.row_scale[(size_t)u * D + row0 + i];
                    const int8_t *q = w.codes + (size_t)u * D * D + (size_t)(row0 + i) * D + col0;
                    if constexpr (CL == 4) word[i] = *reinterpret_cast<const uint32_t *>(q);
                    else word[i] = *reinterpret_cast<const uint16_t *>(q);
                }
                double gsum[KDA ? CL : 1];
                if (KDA) {
#pragma unroll
                    for (int c = 0; c < (KDA ? CL : 1); ++c) gsum[c] = w.gate_sum[(size_t)u * D + col0 + c];
                } else {
                    gsum[0] = w.gate_sum[u];
                }
                uint4 raw[PIECES];
                float om[PIECES];
                float4 dv[DP];
                auto load_chunk = [&](int e0) {
                    const int ne = min(CH, n_buf - e0);
#pragma unroll
                    for (int p = 0; p < PIECES; ++p) {
                        const int idx = p * kThreads + tid, el = idx / PER_ENTRY;
                        raw[p] = make_uint4(0u, 0u, 0u, 0u);
                        om[p] = 1.0f;
                        if (el < ne) {
                            raw[p] = reinterpret_cast<const uint4 *>(keys + (size_t)e0 * D)[idx];
                            if (!KDA) om[p] = w.buf_gate[(size_t)u * w.window_pad + e0 + el];
                        }
                    }
#pragma unroll
                    for (int p = 0; p < DP; ++p) {
                        const int idx = p * kThreads + tid, del_el = idx >> 2, del_q = idx & 3;
                        dv[p] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        if (del_el < ne)
                            dv[p] = *reinterpret_cast<const float4 *>(w.buf_delta + ((size_t)u * W + e0 + del_el) * D +
                                                                      rank * kRows + del_q * 4);
                    }
                };
                // omega_j k_j (or kappa_j) as FP32, each key value converted once
                auto stage_chunk = [&]() {
#pragma unroll
                    for (int p = 0; p < PIECES; ++p) {
                        const int idx = p * kThreads + tid, el = idx / PER_ENTRY, j0 = (idx % PER_ENTRY) * VALS;
                        float *dst = kap + el * D + j0;
                        if constexpr (KB == 2) {
                            const uint32_t wd[4] = {raw[p].x, raw[p].y, raw[p].z, raw[p].w};
                            float kv[8];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                kv[2 * h] = om[p] * bf16_bits_to_f32(wd[h] & 0xffffu);
                                kv[2 * h + 1] = om[p] * bf16_bits_to_f32(wd[h] >> 16);
                            }
                            *reinterpret_cast<float4 *>(dst) = make_float4(kv[0], kv[1], kv[2], kv[3]);
                            *reinterpret_cast<float4 *>(dst + 4) = make_float4(kv[4], kv[5], kv[6], kv[7]);
                        } else {
                            float4 x = make_float4(__uint_as_float(raw[p].x), __uint_as_float(raw[p].y),
                                                   __uint_as_float(raw[p].z), __uint_as_float(raw[p].w));
                            if (!KDA) x = make_float4(om[p] * x.x, om[p] * x.y, om[p] * x.z, om[p] * x.w);
                            *reinterpret_cast<float4 *>(dst) = x;
                        }
                    }
#pragma unroll
                    for (int p = 0; p < DP; ++p) {
                        const int idx = p * kThreads + tid;
                        *reinterpret_cast<float4 *>(dl + (idx >> 2) * kRows + (idx & 3) * 4) = dv[p];
                    }
                };
                load_chunk(0);
                __syncthreads();          // the previous unit's codec is done with the shared arrays
#pragma unroll
                for (int j = 0; j < kMetaPieces; ++j)
                    if (tid + j * kThreads < n_meta) *reinterpret_cast<float4 *>(meta + 4 * (tid + j * kThreads)) = mv[j];
                stage_chunk();
                __syncthreads();

                // ---------------- dequantized rows plus compensators (undecayed)
                float2 acc[4][CL / 2];
                {
                    const int32_t *mci = reinterpret_cast<const int32_t *>(meta);
                    const float *mcr = meta + cis, *mcc = meta + cis + ncr * D;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float f[4];
                        i8x4_to_f32(word[i], f[0], f[1], f[2], f[3]);
#pragma unroll
                        for (int m = 0; m < CL / 2; ++m)
                            acc[i][m] = make_float2((si[i] * f[2 * m]) * sc[2 * m], (si[i] * f[2 * m + 1]) * sc[2 * m + 1]);
                    }
                    for (int c = 0; c < ncr; ++c) {
                        const int i0 = mci[c];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (row0 + i == i0) {
#pragma unroll
                                for (int m = 0; m < CL / 2; ++m) {
                                    acc[i][m].x += mcr[c * D + col0 + 2 * m];
                                    acc[i][m].y += mcr[c * D + col0 + 2 * m + 1];
                                }
                            }
                        }
                    }
                    for (int c = 0; c < ncc; ++c) {
                        const int j0 = mci[ncr + c];
#pragma unroll
                        for (int cc = 0; cc < CL; ++cc) {
                            if (col0 + cc == j0) {
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const float x = mcc[c * kRows + warp * 4 + i];
                                    if (cc & 1) acc[i][cc >> 1].y += x;
                                    else acc[i][cc >> 1].x += x;
                                }
                            }
                        }
                    }
                }

                // ---------------- rank-n_buf update; chunk c + 1 loads while chunk c computes
                for (int ch = 0; ch < nch; ++ch) {
                    const int e0 = ch * CH, ne = min(CH, n_buf - e0);
                    if (ch > 0) {
                        __syncthreads();              // chunk ch - 1 is consumed
                        stage_chunk();
                        __syncthreads();
                    }
                    if (ch + 1 < nch) load_chunk(e0 + CH);
#pragma unroll 4
                    for (int e = 0; e < ne; ++e) {
                        const float4 d4 = *reinterpret_cast<const float4 *>(dl + e * kRows + warp * 4);
                        float2 kc[CL / 2];
                        if constexpr (CL == 4) {
                            const float4 k4 = *reinterpret_cast<const float4 *>(kap + e * D + col0);
                            kc[0] = make_float2(k4.x, k4.y);
                            kc[1] = make_float2(k4.z, k4.w);
                        } else {
                            kc[0] = *reinterpret_cast<const float2 *>(kap + e * D + col0);
                        }
                        const float dr[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 dd = make_float2(dr[i], dr[i]);
#pragma unroll
                            for (int m = 0; m < CL / 2; ++m) acc[i][m] = __ffma2_rn(dd, kc[m], acc[i][m]);
                        }
                    }
                }
                // decay of the window: gamma_W = exp(G_W) per key channel (scalar gate: one value)
                {
                    float2 gam[CL / 2];
#pragma unroll
                    for (int m = 0; m < CL / 2; ++m)
                        gam[m] = KDA ? make_float2(exp_of_double(gsum[KDA ? 2 * m : 0]), exp_of_double(gsum[KDA ? 2 * m + 1 : 0]))
                                     : make_float2(exp_of_double(gsum[0]), exp_of_double(gsum[0]));
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int m = 0; m < CL / 2; ++m) acc[i][m] = __fmul2_rn(acc[i][m], gam[m]);
                }
                __syncthreads();                      // the column partials below reuse the staging area

                // ---------------- codec (steps 2-4) across the cluster
                auto at = [&](int i, int c) -> float & { return (c & 1) ? acc[i][c >> 1].y : acc[i][c >> 1].x; };
                float *rsc = fs + Sh::RSCORE + parity * D;
                float *csq = fs + Sh::CSQ + parity * C * D, *cmx = fs + Sh::CMX + parity * C * D;
                int32_t *cidx = w.comp_index + (size_t)u * cis;

                // Every global store of the unit waits until after the last cluster
                // barrier: a barrier's release would otherwise wait for them to drain.
                // 2a. compensator rows: every CTA sends its 16 row scores to every CTA
                uint2 sel = make_uint2(0xffffffffu, 0xffffffffu);
                int rslot[4] = {-1, -1, -1, -1};          // compensator slot of each of this thread's rows
                if (ncr > 0) {
                    float pr[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float p = 0.0f;
#pragma unroll
                        for (int c = 0; c < CL; ++c) {
                            const float x = fabsf(at(i, c));
                            p = l2 ? p + x * x : fmaxf(p, x);
                        }
                        pr[i] = l2 ? group_sum<32>(p) : group_max<32>(p);
                    }
                    if (lane < 4 * C) {
                        const int i = lane & 3;
                        const float v = i == 0 ? pr[0] : i == 1 ? pr[1] : i == 2 ? pr[2] : pr[3];
                        cluster.map_shared_rank(rsc, (unsigned)(lane >> 2))[row0 + i] = v;
                    }
                    cluster.sync();
                    sel = select_top<D>(rsc, ncr);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (c < ncr && sel_at(sel, c) == row0 + i) rslot[i] = c;
                }

                // 2b, 3. column statistics of the row-zeroed residual (the chosen rows
                // count as zero): partials over this CTA's rows, sent to every CTA,
                // reduced in rank order
#pragma unroll
                for (int c = 0; c < CL; ++c) {
                    float sq = 0.0f, mx = 0.0f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float x = rslot[i] >= 0 ? 0.0f : fabsf(at(i, c));
                        sq = sq + x * x;
                        mx = fmaxf(mx, x);
                    }
                    wsq[warp * D + col0 + c] = sq;
                    wmx[warp * D + col0 + c] = mx;
                }
                __syncthreads();
                if (tid < D) {
                    float sq = 0.0f, mx = 0.0f;
#pragma unroll
                    for (int wq = 0; wq < 4; ++wq) {
                        sq += wsq[wq * D + tid];
                        mx = fmaxf(mx, wmx[wq * D + tid]);
                    }
#pragma unroll
                    for (int r = 0; r < C; ++r) {
                        cluster.map_shared_rank(csq, (unsigned)r)[rank * D + tid] = sq;
                        cluster.map_shared_rank(cmx, (unsigned)r)[rank * D + tid] = mx;
                    }
                }
                cluster.sync();
                if (tid < D) {
                    float sq = 0.0f, mx = 0.0f;
#pragma unroll
                    for (int r = 0; r < C; ++r) {
                        sq += csq[r * D + tid];
                        mx = fmaxf(mx, cmx[r * D + tid]);
                    }
                    sh_score[tid] = l2 ? sq : mx;
                    sh_cmax[tid] = mx;
                }
                __syncthreads();
                const uint2 csel = select_top<D>(sh_score, ncc);
                if (rank == 0 && tid == 0) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        if (c < ncr) cidx[c] = sel_at(sel, c);
                        if (c < ncc) cidx[ncr + c] = sel_at(csel, c);
                    }
                }
                // the chosen rows: stored, then zeroed
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (rslot[i] >= 0) {
                        float *dst = w.comp_row_vec + ((size_t)u * ncr + rslot[i]) * D + col0;
                        if constexpr (CL == 4)
                            *reinterpret_cast<float4 *>(dst) = make_float4(acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y);
                        else
                            *reinterpret_cast<float2 *>(dst) = acc[i][0];
#pragma unroll
                        for (int m = 0; m < CL / 2; ++m) acc[i][m] = make_float2(0.0f, 0.0f);
                    }
                }
                if (tid < D) {
                    bool chosen = false;
#pragma unroll
                    for (int c = 0; c < 8; ++c) chosen |= (c < ncc && sel_at(csel, c) == tid);
                    const float m = chosen ? 0.0f : sh_cmax[tid];
                    const float s = (a.smooth && m > 0.0f) ? __fsqrt_rn(m) : 1.0f;
                    sh_rs[tid] = __fdiv_rn(1.0f, s);          // applied as a multiplication
                    if (rank == 0) w.col_smooth[(size_t)u * D + tid] = s;
                }
                if (ncc > 0) {
#pragma unroll
                    for (int c = 0; c < CL; ++c) {
                        int slot = -1;
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc)
                            if (cc < ncc && sel_at(csel, cc) == col0 + c) slot = cc;
                        if (slot >= 0) {
                            float *dst = w.comp_col_vec + ((size_t)u * ncc + slot) * D + row0;
                            *reinterpret_cast<float4 *>(dst) = make_float4(at(0, c), at(1, c), at(2, c), at(3, c));
#pragma unroll
                            for (int i = 0; i < 4; ++i) at(i, c) = 0.0f;
                        }
                    }
                }
                __syncthreads();

                // 4. row scales and the codes
                float rsv[CL];
#pragma unroll
                for (int c = 0; c < CL; ++c) rsv[c] = sh_rs[col0 + c];
                int8_t *Qu = w.codes + (size_t)u * D * D;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float mm = 0.0f;
#pragma unroll
                    for (int c = 0; c < CL; ++c) {
                        at(i, c) = __fmul_rn(at(i, c), rsv[c]);
                        mm = fmaxf(mm, fabsf(at(i, c)));
                    }
                    const float mrow = group_max<32>(mm);
                    const float rho = (mrow > 0.0f) ? __fdiv_rn(127.0f, mrow) : 0.0f;
                    if (lane == i) w.row_scale[(size_t)u * D + row0 + i] = __fdiv_rn(mrow, 127.0f);
                    // rint by adding 1.5 * 2^23 (|x rho| <= 127 here, so the sum is exact
                    // up to the one rounding to an integer, to nearest, ties to even); the
                    // code is the low byte of the sum's bit pattern
                    uint32_t b[CL];
#pragma unroll
                    for (int c = 0; c < CL; ++c)
                        b[c] = __float_as_uint(__fadd_rn(__fmul_rn(at(i, c), rho), 12582912.0f));
                    int8_t *dstq = Qu + (size_t)(row0 + i) * D + col0;
                    if constexpr (CL == 4)
                        *reinterpret_cast<uint32_t *>(dstq) =
                            __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
                    else
                        *reinterpret_cast<uint16_t *>(dstq) = (uint16_t)(__byte_perm(b[0], b[1], 0x0040) & 0xffffu);
                }

                // 5. start the unit's next window
                if (rank == 0) {
                    if (KDA) {
                        if (tid < D) w.gate_sum[(size_t)u * D + tid] = 0.0;
                    } else if (tid == 0) {
                        w.gate_sum[u] = 0.0;
                    }
                    if (tid == 0) a.fill[u] = 0;
                }
                parity ^= 1;
            }
        }
        __syncthreads();                                 // before the counts are read again
    }
    // No CTA leaves while another may still write its shared memory; nothing is
    // exchanged here, so the arrival orders no memory.
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

template <int D, bool KDA, typename KeyT>
cudaError_t launch_t(const EncodeArgs &a, cudaStream_t s) {
    using Sh = SplitShape<D, (int)sizeof(KeyT)>;
    auto kern = flush_split_kernel<D, KDA, KeyT>;
    const size_t smem = 4 * (size_t)Sh::WORDS;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Sh::C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Clusters that fit on the GPU at once, found once per device (outside any
    // stream capture: the first flush of a handle runs before graphs are made).
    static DeviceCache clusters;
    int dev = 0, n_clusters = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = clusters.get(dev, &n_clusters, [&](int *v) {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (r != cudaSuccess) return r;
        cudaLaunchConfig_t probe = cfg;
        probe.gridDim = dim3(Sh::C, 1, 1);
        return cudaOccupancyMaxActiveClusters(v, kern, &probe);
    });
    if (e != cudaSuccess) return e;
    const int ncl = min(n_clusters, a.w.units);
    cfg.gridDim = dim3((unsigned)(ncl * Sh::C), 1, 1);
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

cudaError_t launch_flush_split(const EncodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s) {
    if (a.fill == nullptr || a.flush_min < 1 || a.w.units <= 0) return cudaErrorInvalidValue;
    if (a.w.n_comp_rows > 8 || a.w.n_comp_cols > 8) return cudaErrorInvalidValue;
    const bool kda = (gate == LQ_GATE_CHANNEL);
    const bool bf = (in_dtype == LQ_DTYPE_BF16);
    if (d == 128) {
        if (kda) return launch_t<128, true, float>(a, s);
        return bf ? launch_t<128, false, __nv_bfloat16>(a, s) : launch_t<128, false, float>(a, s);
    }
    if (d == 64) {
        if (kda) return launch_t<64, true, float>(a, s);
        return bf ? launch_t<64, false, __nv_bfloat16>(a, s) : launch_t<64, false, float>(a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lq
