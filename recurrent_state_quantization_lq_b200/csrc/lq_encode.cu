// State codec kernels: prefill ingestion and window flush.
//
// LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent
// State Quantization", section "Abstract (arXiv)") quantizes the state only
// once, at the end of each window.  Per (sequence, head) unit the kernels here
// take the end-of-window state in FP32 registers: the prefilled state as
// given, or (flush) the rebuild
//     R = (R^ + C + sum_j delta_j kappa_j^T) diag(gamma_W),
// a rank-n_buf update of the dequantized window-start state; they then encode
// it with the codec steps 2-4 of lq_codec.cuh.
//
// The flush kernel is persistent and warp-specialized like the decode kernel:
// a producer thread streams each unit's meta segment (scales, gate sums,
// compensators), INT8 tile and buffered-entry chunks through a ring of 16 KB
// shared-memory slots with 1-D bulk async copies and bounded mbarrier waits;
// eight consumer warps rebuild, encode and store.
#include "lq_codec.cuh"
#include "lq_kernels.h"

namespace lq {
namespace {

constexpr int kSlotBytes = 16384;
constexpr int kSlots = 4;
constexpr int kFlushThreads = kTile + 32; // + one producer warp
constexpr int kMaxChunk = 16;

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

__device__ __forceinline__ bool tile_sync_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(kTileBarrier), "r"(kTile)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ================================================================== prefill

template <int D, bool KDA>
__global__ void __launch_bounds__(kTile, 2) prefill_kernel(EncodeArgs a) {
    constexpr int G = Tile<D>::G, NR = Tile<D>::NR;
    extern __shared__ __align__(16) float pf_scratch[];
    Tile<D> T;
    T.tid = threadIdx.x;
    T.tx = T.tid & 15;
    T.ty = T.tid >> 4;
    const int u = blockIdx.x;
    if (a.seq_mask != nullptr && a.seq_mask[u / a.heads] == 0) return;   // sequence not restarted
    if (a.S0 != nullptr) {
        const float *S0 = a.S0 + (size_t)u * D * D;
#pragma unroll
        for (int r = 0; r < NR; ++r)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float4 x = *reinterpret_cast<const float4 *>(S0 + (size_t)T.row(r) * D + g * 64 + T.tx * 4);
                T.acc[r][g * 2] = make_float2(x.x, x.y);
                T.acc[r][g * 2 + 1] = make_float2(x.z, x.w);
            }
    } else {
#pragma unroll
        for (int r = 0; r < NR; ++r)
#pragma unroll
            for (int m = 0; m < NR / 2; ++m) T.acc[r][m] = make_float2(0.0f, 0.0f);
    }
    codec_store<D, KDA>(T, u, a.w, a.n_rows, a.n_cols, a.smooth, a.select, pf_scratch);
    if (a.fill != nullptr && T.tid == 0) a.fill[u] = 0;
}

// ==================================================================== flush

template <int D, bool KDA, typename KeyT>
struct FlushShape {
    static constexpr int KB = (int)sizeof(KeyT);
    static constexpr int ENTRY = 4 * D + KB * D + (KDA ? 0 : 4);
    static constexpr int E0 = (kSlotBytes / ENTRY) & ~3;
    static constexpr int E = E0 < kMaxChunk ? E0 : kMaxChunk;      // entries per chunk segment
    static constexpr int C_KEY = 4 * D * E;                         // chunk: deltas, keys, omega_j
    static constexpr int C_GATE = C_KEY + KB * D * E;
    // shared memory: barriers, ring, staged keys (two buffers), codec scratch
    static constexpr int OFF_RING = 128;        // barriers (64 bytes), unit records (64 bytes)
    static constexpr int OFF_STAGE = OFF_RING + kSlots * kSlotBytes;
    static constexpr int OFF_GAMMA = OFF_STAGE + (KDA ? 0 : 2 * kMaxChunk * D * 4);
    static constexpr int OFF_CODEC = OFF_GAMMA + 4 * D;
    static constexpr int SMEM = OFF_CODEC + 4 * CodecScratch<D>::FLOATS;
    static_assert(E >= 4, "chunk size");
};

struct FlushMeta {
    int sig, s, gsum, cidx, crow, ccol, bytes;
};

// What the producer tells the tile threads about the unit whose meta segment
// fills a slot (u < 0: no unit is left).
struct FlushRec {
    double gw;     // scalar gate: G at the window end
    int u;
    int pad;
};

// The flush's unit-ticket counter: a 64-bit word in the error region (int32 index).
constexpr int kFlushTicketWord = 34;

template <int D, bool KDA>
__host__ __device__ FlushMeta flush_meta_layout(int ncr, int ncc, int cis) {
    FlushMeta m{};
    int o = 0;
    m.sig = o;  o += 4 * D;
    m.s = o;    o += 4 * D;
    m.gsum = o; o += KDA ? 8 * D : 0;
    m.cidx = o; o += (ncr + ncc) > 0 ? 4 * cis : 0;
    m.crow = o; o += 4 * D * ncr;
    m.ccol = o; o += 4 * D * ncc;
    m.bytes = o;
    return m;
}

template <int D, bool KDA, typename KeyT>
__global__ void __launch_bounds__(kFlushThreads, 2) flush_kernel(EncodeArgs a) {
    using Sh = FlushShape<D, KDA, KeyT>;
    constexpr int G = Tile<D>::G, NR = Tile<D>::NR, E = Sh::E;
    const Views &w = a.w;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ncr = w.n_comp_rows, ncc = w.n_comp_cols, cis = w.comp_index_stride, ncomp = ncr + ncc;
    const int units = w.units, n_buf = a.n_buf;      // one window phase for every unit
    const int nchunks = (n_buf + E - 1) / E;
    const FlushMeta M = flush_meta_layout<D, KDA>(ncr, ncc, cis);
    if (!in_bounds(w.err, n_buf, 0, w.window + 1, -1, -20)) return;   // checked build; every thread alike

    extern __shared__ __align__(128) unsigned char sm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(sm);
    uint64_t *empty = full + kSlots;
    FlushRec *rec = reinterpret_cast<FlushRec *>(empty + kSlots);   // one per ring slot
    unsigned char *ring = sm + Sh::OFF_RING;
    float *stage = reinterpret_cast<float *>(sm + Sh::OFF_STAGE);
    float *sgam = reinterpret_cast<float *>(sm + Sh::OFF_GAMMA);     // gamma_W per key channel
    float *scratch = reinterpret_cast<float *>(sm + Sh::OFF_CODEC);

    if (tid == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kTile);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // ---------------------------------------------------------------- producer
    if (warp == kTile / 32) {
        if (lane != 0) return;
        const uint64_t stream_once = l2_policy_evict_first();
        // Units: a CTA's first is its own index, the others are handed out by
        // ticket (see ticket_unit), so that a CTA that runs faster than the
        // other one on its SM takes more of them.  The kernel before a flush
        // has completed when it starts, so no two launches draw at the same time.
        const int grid = (int)gridDim.x, n_dyn = units - grid;
        unsigned long long *tickets = reinterpret_cast<unsigned long long *>(w.err + kFlushTicketWord);
        int slot = 0;
        uint32_t ph = 0;
        uint32_t armed = 0;                        // slots filled at least once
        auto acquire = [&](int u, int detail) -> unsigned char * {
            if (!mbar_wait(&empty[slot], ph ^ 1u, kWaitBudgetCycles)) {
                report_error(w.err, LQ_DEVERR_TIMEOUT, u, detail);
                return nullptr;
            }
            armed |= 1u << slot;
            return ring + slot * kSlotBytes;
        };
        auto advance = [&]() {
            if (++slot == kSlots) { slot = 0; ph ^= 1u; }
        };
        // After a timed-out acquire: a meta slot still owed its record gets the
        // end one, then wait (bounded) until every copy this thread started has
        // landed, so that none writes into the shared memory of an exited CTA.
        // Slot i was last filled in the round of parity ph (i < slot) or ph ^ 1.
        auto fail = [&](int pend) {
            if (pend >= 0) {
                rec[pend].u = -1;
                mbar_arrive(&full[pend]);
            }
            for (int i = 0; i < kSlots; ++i)
                if (armed & (1u << i)) mbar_wait(&full[i], i < slot ? ph : (ph ^ 1u), kWaitBudgetCycles);
        };
        int u = (int)blockIdx.x;
        unsigned long long tk = 0;
        bool draw = n_dyn > 0;
        if (draw) tk = atomicAdd(tickets, 1ull);   // the second unit's ticket
        while (u >= 0) {
            const double gw = KDA ? 0.0 : w.gate_sum[u];   // scalar gate: G at the window end
            unsigned char *dst = acquire(u, -1);
            if (dst == nullptr) { fail(-1); return; }
            const int meta_slot = slot;
            uint64_t *bar = &full[slot];
            mbar_expect_tx(bar, (uint32_t)M.bytes);       // the arrival comes with the record
            bulk_g2s(dst + M.sig, w.row_scale + (size_t)u * D, 4 * D, bar);
            bulk_g2s(dst + M.s, w.col_smooth + (size_t)u * D, 4 * D, bar);
            if (KDA) bulk_g2s(dst + M.gsum, w.gate_sum + (size_t)u * D, 8 * D, bar);
            if (ncomp > 0) {
                bulk_g2s(dst + M.cidx, w.comp_index + (size_t)u * cis, 4 * cis, bar);
                if (ncr > 0) bulk_g2s(dst + M.crow, w.comp_row_vec + (size_t)u * ncr * D, 4 * D * ncr, bar);
                if (ncc > 0) bulk_g2s(dst + M.ccol, w.comp_col_vec + (size_t)u * ncc * D, 4 * D * ncc, bar);
            }
            advance();
            dst = acquire(u, -2);
            if (dst == nullptr) { fail(meta_slot); return; }
            bar = &full[slot];
            mbar_arrive_expect_tx(bar, D * D);
            bulk_g2s_stream(dst, w.codes + (size_t)u * D * D, D * D, bar, stream_once);
            advance();
            rec[meta_slot].gw = gw;
            rec[meta_slot].u = u;
            mbar_arrive(&full[meta_slot]);        // releases the record; the phase ends when the bytes land
            for (int c = 0; c < nchunks; ++c) {
                dst = acquire(u, -3 - c);
                if (dst == nullptr) { fail(-1); return; }
                const int e0 = c * E, ne = min(E, n_buf - e0);
                const size_t first = (size_t)u * w.window + e0;
                const uint32_t bd = 4u * ne * D, bk = (uint32_t)sizeof(KeyT) * ne * D;
                const uint32_t bg = KDA ? 0u : 4u * (uint32_t)align_up(ne, 4);
                bar = &full[slot];
                mbar_arrive_expect_tx(bar, bd + bk + bg);
                bulk_g2s_stream(dst, w.buf_delta + first * D, bd, bar, stream_once);
                bulk_g2s_stream(dst + Sh::C_KEY, reinterpret_cast<const KeyT *>(w.buf_key) + first * D, bk, bar,
                                stream_once);
                if (!KDA) bulk_g2s(dst + Sh::C_GATE, w.buf_gate + (size_t)u * w.window_pad + e0, bg, bar);
                advance();
            }
            // the next unit: its ticket was drawn a unit ago
            u = -1;
            if (draw) {
                const int r = ticket_unit(tk, n_dyn, grid, tickets, w.err);
                if (r >= 0) {
                    u = grid + r;
                    tk = atomicAdd(tickets, 1ull);
                } else {
                    draw = false;
                }
            }
        }
        // no unit left: a record that says so
        if (acquire(-1, -5) == nullptr) { fail(-1); return; }
        rec[slot].u = -1;
        mbar_arrive(&full[slot]);
        return;
    }

    // ------------------------------------------------------------ tile threads
    Tile<D> T;
    T.tid = tid;
    T.tx = tid & 15;
    T.ty = tid >> 4;
    int slot = 0;
    uint32_t ph = 0;
    auto advance = [&]() {
        if (++slot == kSlots) { slot = 0; ph ^= 1u; }
    };
    for (;;) {
        bool bad = !mbar_wait(&full[slot], ph, kWaitBudgetCycles);
        const int u = rec[slot].u;
        const double GW = rec[slot].gw;              // scalar gate: G at the window end
        if (tile_sync_or(bad || u < 0)) {           // a timeout, or no unit left
            if (bad) report_error(w.err, LQ_DEVERR_TIMEOUT, -1, 0);
            return;
        }
        // -------- dequantized window-start state plus compensators (undecayed)
        const unsigned char *mp = ring + slot * kSlotBytes;
        const int meta_slot = slot;
        advance();
        bad = !mbar_wait(&full[slot], ph, kWaitBudgetCycles);
        const int8_t *sQ = reinterpret_cast<const int8_t *>(ring + slot * kSlotBytes);
        const int q_slot = slot;
        advance();
        if (tile_sync_or(bad)) {
            if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 0);
            return;
        }
        {
            const float *sig = reinterpret_cast<const float *>(mp + M.sig);
            const float *sm_s = reinterpret_cast<const float *>(mp + M.s);
            float sc[NR];
#pragma unroll
            for (int c = 0; c < NR; ++c) sc[c] = sm_s[T.col(c)];
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const float si = sig[T.row(r)];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const uint32_t word = *reinterpret_cast<const uint32_t *>(sQ + T.row(r) * D + g * 64 + T.tx * 4);
                    float f0, f1, f2, f3;
                    i8x4_to_f32(word, f0, f1, f2, f3);
                    T.acc[r][g * 2] = make_float2((si * f0) * sc[g * 4 + 0], (si * f1) * sc[g * 4 + 1]);
                    T.acc[r][g * 2 + 1] = make_float2((si * f2) * sc[g * 4 + 2], (si * f3) * sc[g * 4 + 3]);
                }
            }
            // The compensators as rank-1 terms on the packed FMAs, rows first,
            // then columns: e_i k_c^T and v_c e_j^T.  fma(1, x, acc) = acc + x
            // and fma(0, x, acc) = acc, so each element gets exactly the adds
            // of its own compensators, in that order.
            if (ncomp > 0) {
                const int32_t *cidx = reinterpret_cast<const int32_t *>(mp + M.cidx);
                const float *crow = reinterpret_cast<const float *>(mp + M.crow);
                const float *ccol = reinterpret_cast<const float *>(mp + M.ccol);
                for (int c = 0; c < ncr; ++c) {
                    const int i = cidx[c];
                    float2 kc[NR / 2];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float4 y = *reinterpret_cast<const float4 *>(crow + c * D + g * 64 + T.tx * 4);
                        kc[g * 2 + 0] = make_float2(y.x, y.y);
                        kc[g * 2 + 1] = make_float2(y.z, y.w);
                    }
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        const float e = T.row(r) == i ? 1.0f : 0.0f;
#pragma unroll
                        for (int m = 0; m < NR / 2; ++m) T.acc[r][m] = __ffma2_rn(make_float2(e, e), kc[m], T.acc[r][m]);
                    }
                }
                for (int c = 0; c < ncc; ++c) {
                    const int j = cidx[ncr + c];
                    float2 ec[NR / 2];
#pragma unroll
                    for (int m = 0; m < NR / 2; ++m)
                        ec[m] = make_float2(T.col(2 * m) == j ? 1.0f : 0.0f, T.col(2 * m + 1) == j ? 1.0f : 0.0f);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float4 x = *reinterpret_cast<const float4 *>(ccol + c * D + g * 64 + T.ty * 4);
                        const float xr[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int rr = 0; rr < 4; ++rr) {
#pragma unroll
                            for (int m = 0; m < NR / 2; ++m)
                                T.acc[g * 4 + rr][m] =
                                    __ffma2_rn(make_float2(xr[rr], xr[rr]), ec[m], T.acc[g * 4 + rr][m]);
                        }
                    }
                }
            }
        }
        // decay of the window: gamma_W per key channel (scalar gate: one value)
        if (tid < D) {
            sgam[tid] = KDA ? exp_of_double(reinterpret_cast<const double *>(mp + M.gsum)[tid]) : exp_of_double(GW);
        }
        mbar_arrive(&empty[meta_slot]);
        mbar_arrive(&empty[q_slot]);

        // -------- rank-n_buf update with the buffered entries
        for (int c = 0; c < nchunks; ++c) {
            bad = !mbar_wait(&full[slot], ph, kWaitBudgetCycles);
            const unsigned char *cp = ring + slot * kSlotBytes;
            const float *sDelta = reinterpret_cast<const float *>(cp);
            const int ne = min(E, n_buf - c * E);
            const float *kap;
            if (KDA) {
                kap = reinterpret_cast<const float *>(cp + Sh::C_KEY);
            } else {
                // stage omega_j k_j as FP32 (each key element converted once)
                float *sb = stage + (c & 1) * kMaxChunk * D;
                const KeyT *keys = reinterpret_cast<const KeyT *>(cp + Sh::C_KEY);
                const float *omega = reinterpret_cast<const float *>(cp + Sh::C_GATE);
                for (int idx = tid; idx < ne * (D / 8); idx += kTile) {
                    const int el = idx / (D / 8), j0 = (idx % (D / 8)) * 8;
                    const float om = omega[el];
                    float kv[8];
                    if constexpr (sizeof(KeyT) == 2) {
                        const uint4 raw = *reinterpret_cast<const uint4 *>(keys + el * D + j0);
                        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            kv[2 * h] = bf16_bits_to_f32(wd[h] & 0xffffu);
                            kv[2 * h + 1] = bf16_bits_to_f32(wd[h] >> 16);
                        }
                    } else {
                        const float4 x0 = *reinterpret_cast<const float4 *>(keys + el * D + j0);
                        const float4 x1 = *reinterpret_cast<const float4 *>(keys + el * D + j0 + 4);
                        kv[0] = x0.x; kv[1] = x0.y; kv[2] = x0.z; kv[3] = x0.w;
                        kv[4] = x1.x; kv[5] = x1.y; kv[6] = x1.z; kv[7] = x1.w;
                    }
                    *reinterpret_cast<float4 *>(sb + el * D + j0) =
                        make_float4(om * kv[0], om * kv[1], om * kv[2], om * kv[3]);
                    *reinterpret_cast<float4 *>(sb + el * D + j0 + 4) =
                        make_float4(om * kv[4], om * kv[5], om * kv[6], om * kv[7]);
                }
                kap = sb;
            }
            if (tile_sync_or(bad)) {
                if (tid == 0) report_error(w.err, LQ_DEVERR_TIMEOUT, u, 1 + c);
                return;
            }
            for (int el = 0; el < ne; ++el) {
                float dr[NR];
                float2 kc[NR / 2];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float4 x = *reinterpret_cast<const float4 *>(sDelta + el * D + g * 64 + T.ty * 4);
                    const float4 y = *reinterpret_cast<const float4 *>(kap + el * D + g * 64 + T.tx * 4);
                    dr[g * 4 + 0] = x.x; dr[g * 4 + 1] = x.y; dr[g * 4 + 2] = x.z; dr[g * 4 + 3] = x.w;
                    kc[g * 2 + 0] = make_float2(y.x, y.y);
                    kc[g * 2 + 1] = make_float2(y.z, y.w);
                }
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float2 dd = make_float2(dr[r], dr[r]);
#pragma unroll
                    for (int m = 0; m < NR / 2; ++m) T.acc[r][m] = __ffma2_rn(dd, kc[m], T.acc[r][m]);
                }
            }
            mbar_arrive(&empty[slot]);
            advance();
        }

        // -------- apply the window's decay
        tile_sync();
        {
            float2 gg[NR / 2];
#pragma unroll
            for (int m = 0; m < NR / 2; ++m) gg[m] = make_float2(sgam[T.col(2 * m)], sgam[T.col(2 * m + 1)]);
#pragma unroll
            for (int r = 0; r < NR; ++r)
#pragma unroll
                for (int m = 0; m < NR / 2; ++m) T.acc[r][m] = __fmul2_rn(T.acc[r][m], gg[m]);
        }
        codec_store<D, KDA>(T, u, w, ncr, ncc, a.smooth, a.select, scratch);
    }
}

template <int D, bool KDA, typename KeyT>
cudaError_t launch_flush_t(const EncodeArgs &a, cudaStream_t s) {
    using Sh = FlushShape<D, KDA, KeyT>;
    const FlushMeta M = flush_meta_layout<D, KDA>(a.w.n_comp_rows, a.w.n_comp_cols, a.w.comp_index_stride);
    if (M.bytes > kSlotBytes || D * D > kSlotBytes) return cudaErrorInvalidValue;
    auto kern = flush_kernel<D, KDA, KeyT>;
    const cudaError_t e = opt_in_smem<flush_kernel<D, KDA, KeyT>>(Sh::SMEM);
    if (e != cudaSuccess) return e;
    const int grid = min(a.w.units, 2 * sm_count());
    kern<<<grid, kFlushThreads, Sh::SMEM, s>>>(a);
    return cudaGetLastError();
}

template <int D, bool KDA, typename KeyT>
cudaError_t launch_encode_t(const EncodeArgs &a, cudaStream_t s) {
    if (!a.from_buffer) {
        prefill_kernel<D, KDA><<<a.w.units, kTile, 4 * CodecScratch<D>::FLOATS, s>>>(a);
        return cudaGetLastError();
    }
    return launch_flush_t<D, KDA, KeyT>(a, s);
}

}  // namespace

cudaError_t launch_encode(const EncodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s) {
    // Shared window phases flush every unit here; ragged phases flush the
    // units that are due, one thread-block cluster per unit.
    if (a.from_buffer && a.fill != nullptr) return launch_flush_split(a, d, gate, in_dtype, s);
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
