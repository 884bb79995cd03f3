// liblq C ABI: config validation, workspace layout, handles and launches.
// The declarations and the contract of every entry point are in include/lq.h.
#include <cuda.h>

#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "lq.h"
#include <nvtx3/nvToolsExt.h>

#include "lq_kernels.h"

namespace {

thread_local std::string g_last_error;

lq_status fail(lq_status code, const std::string &why) {
    g_last_error = why;
    return code;
}

constexpr uint32_t kMagic = 0x4c515354u;  // "LQST"
constexpr int kMaxComp = 8;
constexpr int kMaxWindow = 4096;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool validate(const lq_config *c, std::string *why) {
    if (c == nullptr) { *why = "config is NULL"; return false; }
    if (c->batch < 1 || c->heads < 1) { *why = "batch and heads must be >= 1"; return false; }
    if ((long long)c->batch * c->heads > (1LL << 24)) { *why = "batch * heads must be <= 2^24"; return false; }
    if (c->d_k != c->d_v) { *why = "d_k must equal d_v"; return false; }
    if (c->d_k != 64 && c->d_k != 128) { *why = "d_k must be 64 or 128"; return false; }
    if (c->gate != LQ_GATE_SCALAR && c->gate != LQ_GATE_CHANNEL) { *why = "gate must be LQ_GATE_SCALAR or LQ_GATE_CHANNEL"; return false; }
    if (c->mode != LQ_MODE_WINDOW && c->mode != LQ_MODE_NAIVE && c->mode != LQ_MODE_FP32) { *why = "mode must be one of LQ_MODE_*"; return false; }
    if (c->in_dtype != LQ_DTYPE_F32 && c->in_dtype != LQ_DTYPE_BF16) { *why = "in_dtype must be LQ_DTYPE_F32 or LQ_DTYPE_BF16"; return false; }
    if (c->mode == LQ_MODE_WINDOW) {
        if (c->window < 1 || c->window > kMaxWindow) { *why = "window must be in 1..4096"; return false; }
        if (c->n_comp_rows < 0 || c->n_comp_rows > kMaxComp || c->n_comp_cols < 0 || c->n_comp_cols > kMaxComp) {
            *why = "n_comp_rows and n_comp_cols must be in 0..8"; return false;
        }
        if (c->smooth != 0 && c->smooth != 1) { *why = "smooth must be 0 or 1"; return false; }
        if (c->select != LQ_SELECT_L2 && c->select != LQ_SELECT_MAXABS) { *why = "select must be LQ_SELECT_L2 or LQ_SELECT_MAXABS"; return false; }
    }
    if (c->ragged != 0 && c->ragged != 1) { *why = "ragged must be 0 or 1"; return false; }
    if (c->ragged && c->mode != LQ_MODE_WINDOW) { *why = "ragged window phases need the windowed mode"; return false; }
    return true;
}

void compute_layout(const lq_config *c, lq_layout *L) {
    const size_t N = (size_t)c->batch * c->heads, d = (size_t)c->d_k;
    size_t off = 0;
    auto take = [&](size_t bytes) -> size_t {
        if (bytes == 0) return LQ_ABSENT;
        off = align256(off);
        const size_t r = off;
        off += bytes;
        return r;
    };
    lq_layout z;
    z.total_bytes = 0;
    z.err = z.codes = z.row_scale = z.col_smooth = z.comp_index = z.comp_row_vec = z.comp_col_vec = LQ_ABSENT;
    z.gate_sum = z.buf_delta = z.buf_key = z.buf_gate = z.state_f32 = z.fill = LQ_ABSENT;
    z.comp_index_stride = 0;
    z.window_pad = 0;
    *L = z;
    L->err = take(256);
    if (c->mode == LQ_MODE_FP32) {
        L->state_f32 = take(N * d * d * 4);
    } else if (c->mode == LQ_MODE_NAIVE) {
        L->codes = take(N * d * d);
        L->row_scale = take(N * d * 4);
    } else {
        const int ncomp = c->n_comp_rows + c->n_comp_cols;
        L->comp_index_stride = ((ncomp + 3) / 4) * 4;
        L->window_pad = ((c->window + 3) / 4) * 4;
        const size_t gd = (c->gate == LQ_GATE_CHANNEL) ? d : 1;
        const size_t key_b = (c->gate == LQ_GATE_CHANNEL || c->in_dtype == LQ_DTYPE_F32) ? 4 : 2;
        L->codes = take(N * d * d);
        L->row_scale = take(N * d * 4);
        L->col_smooth = take(N * d * 4);
        L->comp_index = take(N * (size_t)L->comp_index_stride * 4);
        L->comp_row_vec = take(N * (size_t)c->n_comp_rows * d * 4);
        L->comp_col_vec = take(N * (size_t)c->n_comp_cols * d * 4);
        L->gate_sum = take(N * gd * 8);
        L->buf_delta = take(N * (size_t)c->window * d * 4);
        L->buf_key = take(N * (size_t)c->window * d * key_b);
        if (c->gate == LQ_GATE_SCALAR) L->buf_gate = take(N * (size_t)L->window_pad * 4);
        if (c->ragged) L->fill = take(N * 4);
    }
    L->total_bytes = align256(off);
}

template <typename T>
T *region(unsigned char *base, size_t off) {
    return off == LQ_ABSENT ? nullptr : reinterpret_cast<T *>(base + off);
}

lq_status cuda_fail(cudaError_t e, const char *what) {
    return fail(LQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

}  // namespace

struct lq_state_s {
    CUtensorMap codes_map;   // INT8 tiles for the windowed decode (made at its first call)
    uint32_t magic;
    lq_config cfg;
    lq_layout lay;
    unsigned char *ws;
    int32_t n_buf;
    int prefilled;
    int codes_map_ready;
    // No call but a decode was made since the codes were last written: the
    // previous kernel in any stream order can no longer be their writer.
    int codes_settled;
    // ragged handles: every unit is known to be in the same window phase
    // (n_buf tokens) until an active mask or a sequence restart is used
    int aligned;
};

namespace {

bool check_handle(lq_handle h) { return h != nullptr && h->magic == kMagic; }

// An NVTX range around a stream-ordered call, for timeline tools (nsys, ncu);
// nearly free when no tool is attached.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};

lq::Views views(lq_handle h) {
    lq::Views v;
    unsigned char *b = h->ws;
    const lq_layout &L = h->lay;
    v.err = region<int32_t>(b, L.err);
    v.codes = region<int8_t>(b, L.codes);
    v.row_scale = region<float>(b, L.row_scale);
    v.col_smooth = region<float>(b, L.col_smooth);
    v.comp_index = region<int32_t>(b, L.comp_index);
    v.comp_row_vec = region<float>(b, L.comp_row_vec);
    v.comp_col_vec = region<float>(b, L.comp_col_vec);
    v.gate_sum = region<double>(b, L.gate_sum);
    v.buf_delta = region<float>(b, L.buf_delta);
    v.buf_key = region<void>(b, L.buf_key);
    v.buf_gate = region<float>(b, L.buf_gate);
    v.state_f32 = region<float>(b, L.state_f32);
    v.comp_index_stride = L.comp_index_stride;
    v.window = h->cfg.window;
    v.window_pad = L.window_pad;
    v.n_comp_rows = h->cfg.mode == LQ_MODE_WINDOW ? h->cfg.n_comp_rows : 0;
    v.n_comp_cols = h->cfg.mode == LQ_MODE_WINDOW ? h->cfg.n_comp_cols : 0;
    v.units = h->cfg.batch * h->cfg.heads;
    return v;
}

}  // namespace

extern "C" {

size_t lq_workspace_bytes(const lq_config *cfg) {
    std::string why;
    if (!validate(cfg, &why)) {
        g_last_error = why;
        return 0;
    }
    lq_layout L;
    compute_layout(cfg, &L);
    return L.total_bytes;
}

lq_status lq_workspace_layout(const lq_config *cfg, lq_layout *out) {
    std::string why;
    if (out == nullptr) return fail(LQ_ERR_INVALID_ARG, "layout output is NULL");
    if (!validate(cfg, &why)) return fail(LQ_ERR_INVALID_ARG, why);
    compute_layout(cfg, out);
    return LQ_OK;
}

lq_status lq_state_create(const lq_config *cfg, void *d_workspace, size_t bytes, lq_handle *out) {
    std::string why;
    if (out == nullptr) return fail(LQ_ERR_INVALID_ARG, "handle output is NULL");
    *out = nullptr;
    if (!validate(cfg, &why)) return fail(LQ_ERR_INVALID_ARG, why);
    if (d_workspace == nullptr) return fail(LQ_ERR_WORKSPACE, "workspace is NULL");
    if (!aligned(d_workspace, 256)) return fail(LQ_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    lq_layout L;
    compute_layout(cfg, &L);
    if (bytes < L.total_bytes)
        return fail(LQ_ERR_WORKSPACE, "workspace has " + std::to_string(bytes) + " bytes, needs " +
                                          std::to_string(L.total_bytes));
    lq_state_s *h = new (std::nothrow) lq_state_s;
    if (h == nullptr) return fail(LQ_ERR_INVALID_ARG, "out of host memory");
    h->magic = kMagic;
    h->cfg = *cfg;
    h->lay = L;
    h->ws = static_cast<unsigned char *>(d_workspace);
    h->n_buf = 0;
    h->prefilled = 0;
    h->aligned = 0;
    h->codes_map_ready = 0;
    h->codes_settled = 0;
    *out = h;
    return LQ_OK;
}

lq_status lq_state_destroy(lq_handle h) {
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    h->magic = 0;
    delete h;
    return LQ_OK;
}

lq_status lq_state_resume(lq_handle h, int32_t n_buf) {
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    h->codes_settled = 0;
    const lq_config &c = h->cfg;
    const int32_t max_buf = (c.mode == LQ_MODE_WINDOW && !c.ragged) ? c.window : 0;
    if (n_buf < 0 || n_buf > max_buf) return fail(LQ_ERR_INVALID_ARG, "n_buf out of range for this handle");
    h->n_buf = n_buf;
    h->prefilled = 1;
    h->aligned = 0;                      // ragged: the phases are whatever the counts say
    return LQ_OK;
}

int32_t lq_window_fill(lq_handle h) {
    if (!check_handle(h) || h->cfg.ragged) return -1;   // ragged counts live on the device
    return h->n_buf;
}

lq_status lq_prefill_state(lq_handle h, const float *d_S0, void *stream) {
    Range nvtx_range("lq_prefill_state");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    h->codes_settled = 0;
    if (d_S0 != nullptr && !aligned(d_S0, 16)) return fail(LQ_ERR_INVALID_ARG, "S0 must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const lq_config &c = h->cfg;
    const size_t N = (size_t)c.batch * c.heads, d = (size_t)c.d_k;
    lq::Views v = views(h);
    cudaError_t e = cudaMemsetAsync(v.err, 0, 256, s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
    if (c.mode == LQ_MODE_FP32) {
        e = d_S0 ? cudaMemcpyAsync(v.state_f32, d_S0, N * d * d * 4, cudaMemcpyDeviceToDevice, s)
                 : cudaMemsetAsync(v.state_f32, 0, N * d * d * 4, s);
        if (e != cudaSuccess) return cuda_fail(e, "loading the FP32 state");
    } else {
        lq::EncodeArgs a;
        a.w = v;
        a.S0 = d_S0;
        a.from_buffer = 0;
        a.n_buf = 0;
        const bool win = (c.mode == LQ_MODE_WINDOW);
        a.n_rows = win ? c.n_comp_rows : 0;
        a.n_cols = win ? c.n_comp_cols : 0;
        a.smooth = win ? c.smooth : 0;
        a.select = win ? c.select : LQ_SELECT_L2;
        a.fill = nullptr;                  // every unit; the counts are cleared below
        a.flush_min = 0;
        a.seq_mask = nullptr;
        a.heads = c.heads;
        e = lq::launch_encode(a, c.d_k, c.gate, c.in_dtype, s);
        if (e != cudaSuccess) return cuda_fail(e, "launching the encode kernel");
        if (c.ragged) {
            e = cudaMemsetAsync(h->ws + h->lay.fill, 0, N * 4, s);
            if (e != cudaSuccess) return cuda_fail(e, "clearing the window counts");
        }
    }
    h->n_buf = 0;
    h->prefilled = 1;
    h->aligned = 1;
    return LQ_OK;
}

lq_status lq_prefill_tokens(lq_handle h, const float *d_S0, const void *d_q, const void *d_k, const void *d_v,
                            const float *d_g, const float *d_beta, int32_t n_tokens, float *d_o, void *stream) {
    Range nvtx_range("lq_prefill_tokens");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    h->codes_settled = 0;
    if (n_tokens < 0) return fail(LQ_ERR_INVALID_ARG, "negative n_tokens");
    if (n_tokens == 0) return lq_prefill_state(h, d_S0, stream);
    const lq_config &c = h->cfg;
    if (!d_q || !d_k || !d_v || !d_g || !d_beta) return fail(LQ_ERR_INVALID_ARG, "NULL prompt input");
    if (!aligned(d_q, 16) || !aligned(d_k, 16) || !aligned(d_v, 16))
        return fail(LQ_ERR_INVALID_ARG, "q, k, v must be 16-byte aligned");
    if (!aligned(d_g, c.gate == LQ_GATE_CHANNEL ? 16 : 4) || !aligned(d_beta, 4) || (d_o && !aligned(d_o, 4)))
        return fail(LQ_ERR_INVALID_ARG, "g, beta, o misaligned (g per-channel: 16 bytes; others: 4)");
    if (d_S0 != nullptr && !aligned(d_S0, 16)) return fail(LQ_ERR_INVALID_ARG, "S0 must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    lq::Views v = views(h);
    cudaError_t e = cudaMemsetAsync(v.err, 0, 256, s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
    lq::TokenPrefillArgs a;
    a.w = v;
    a.S0 = d_S0;
    a.q = d_q; a.k = d_k; a.v = d_v; a.g = d_g; a.beta = d_beta; a.o = d_o;
    a.n_tokens = n_tokens;
    const bool win = (c.mode == LQ_MODE_WINDOW);
    a.n_rows = win ? c.n_comp_rows : 0;
    a.n_cols = win ? c.n_comp_cols : 0;
    a.smooth = win ? c.smooth : 0;
    a.select = win ? c.select : LQ_SELECT_L2;
    a.fp32_state = (c.mode == LQ_MODE_FP32);
    a.seq_mask = nullptr;
    a.lengths = nullptr;
    a.heads = c.heads;
    a.fill = nullptr;                     // every count is cleared below
    e = lq::launch_prefill_tokens(a, c.d_k, c.gate, c.in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "launching the token prefill kernel");
    if (c.ragged) {
        e = cudaMemsetAsync(h->ws + h->lay.fill, 0, (size_t)c.batch * c.heads * 4, s);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the window counts");
    }
    h->n_buf = 0;
    h->prefilled = 1;
    h->aligned = 1;
    return LQ_OK;
}

lq_status lq_prefill_sequences_tokens(lq_handle h, const float *d_S0, const void *d_q, const void *d_k,
                                      const void *d_v, const float *d_g, const float *d_beta, int32_t max_tokens,
                                      const int32_t *d_lengths, const uint8_t *d_mask, float *d_o, void *stream) {
    Range nvtx_range("lq_prefill_sequences_tokens");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    h->codes_settled = 0;
    const lq_config &c = h->cfg;
    if (!c.ragged) return fail(LQ_ERR_STATE, "lq_prefill_sequences_tokens needs a ragged handle");
    if (!h->prefilled) return fail(LQ_ERR_STATE, "lq_prefill_sequences_tokens before lq_prefill_state");
    if (d_mask == nullptr) return fail(LQ_ERR_INVALID_ARG, "NULL sequence mask");
    if (max_tokens < 0) return fail(LQ_ERR_INVALID_ARG, "negative max_tokens");
    if (max_tokens > 0) {
        if (!d_q || !d_k || !d_v || !d_g || !d_beta) return fail(LQ_ERR_INVALID_ARG, "NULL prompt input");
        if (!aligned(d_q, 16) || !aligned(d_k, 16) || !aligned(d_v, 16))
            return fail(LQ_ERR_INVALID_ARG, "q, k, v must be 16-byte aligned");
        if (!aligned(d_g, c.gate == LQ_GATE_CHANNEL ? 16 : 4) || !aligned(d_beta, 4) || (d_o && !aligned(d_o, 4)))
            return fail(LQ_ERR_INVALID_ARG, "g, beta, o misaligned (g per-channel: 16 bytes; others: 4)");
    }
    if (d_lengths != nullptr && !aligned(d_lengths, 4)) return fail(LQ_ERR_INVALID_ARG, "lengths misaligned");
    if (d_S0 != nullptr && !aligned(d_S0, 16)) return fail(LQ_ERR_INVALID_ARG, "S0 must be 16-byte aligned");
    lq::TokenPrefillArgs a;
    a.w = views(h);
    a.S0 = d_S0;
    a.q = d_q; a.k = d_k; a.v = d_v; a.g = d_g; a.beta = d_beta; a.o = d_o;
    a.n_tokens = max_tokens;
    a.n_rows = c.n_comp_rows;
    a.n_cols = c.n_comp_cols;
    a.smooth = c.smooth;
    a.select = c.select;
    a.fp32_state = 0;
    a.seq_mask = d_mask;
    a.lengths = d_lengths;
    a.heads = c.heads;
    a.fill = reinterpret_cast<int32_t *>(h->ws + h->lay.fill);
    cudaError_t e = lq::launch_prefill_tokens(a, c.d_k, c.gate, c.in_dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "launching the token prefill kernel");
    h->aligned = 0;                       // the restarted sequences start a new phase
    return LQ_OK;
}

namespace {

lq_status decode_impl(lq_handle h, const void *d_q, const void *d_k, const void *d_v, const float *d_g,
                      const float *d_beta, const uint8_t *d_active, float *d_o, void *stream) {
    if (!d_q || !d_k || !d_v || !d_g || !d_beta || !d_o) return fail(LQ_ERR_INVALID_ARG, "NULL input or output");
    if (!aligned(d_q, 16) || !aligned(d_k, 16) || !aligned(d_v, 16))
        return fail(LQ_ERR_INVALID_ARG, "q, k, v must be 16-byte aligned");
    const lq_config &c = h->cfg;
    if (!aligned(d_g, c.gate == LQ_GATE_CHANNEL ? 16 : 4) || !aligned(d_beta, 4) || !aligned(d_o, 4))
        return fail(LQ_ERR_INVALID_ARG, "g, beta, o misaligned (g per-channel: 16 bytes; others: 4)");
    if (!h->prefilled) return fail(LQ_ERR_STATE, "decode before lq_prefill_state");
    if (c.mode == LQ_MODE_WINDOW && !c.ragged && h->n_buf >= c.window)
        return fail(LQ_ERR_WINDOW_FULL, "window holds W tokens: call lq_window_flush first");
    if (c.mode == LQ_MODE_WINDOW && !h->codes_map_ready) {
        cudaError_t e = lq::make_codes_map(&h->codes_map, reinterpret_cast<const int8_t *>(h->ws + h->lay.codes),
                                           c.d_k, c.batch * c.heads);
        if (e != cudaSuccess) return cuda_fail(e, "encoding the tensor map of the codes");
        h->codes_map_ready = 1;
    }
    lq::DecodeArgs a;
    a.w = views(h);
    a.q = d_q; a.k = d_k; a.v = d_v; a.g = d_g; a.beta = d_beta; a.o = d_o;
    a.n_buf = h->n_buf;
    a.codes_map = &h->codes_map;
    a.fill = c.ragged ? reinterpret_cast<int32_t *>(h->ws + h->lay.fill) : nullptr;
    a.active = c.ragged ? d_active : nullptr;
    a.heads = c.heads;
    a.codes_settled = h->codes_settled;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (c.mode == LQ_MODE_WINDOW) e = lq::launch_decode_window(a, c.d_k, c.gate, c.in_dtype, s);
    else if (c.mode == LQ_MODE_NAIVE) e = lq::launch_decode_naive(a, c.d_k, c.gate, c.in_dtype, s);
    else e = lq::launch_decode_fp32(a, c.d_k, c.gate, c.in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "launching the decode kernel");
    h->codes_settled = 1;
    if (c.mode == LQ_MODE_WINDOW && !c.ragged) h->n_buf += 1;
    if (c.ragged) {
        if (d_active != nullptr) h->aligned = 0;
        else if (h->n_buf < c.window) h->n_buf += 1;   // a full window refuses the token on the device
    }
    return LQ_OK;
}

// Flush the windowed state: every unit (shared phase), or the units holding at
// least flush_min buffered tokens (ragged phases).
lq_status flush_impl(lq_handle h, int flush_min, void *stream) {
    const lq_config &c = h->cfg;
    h->codes_settled = 0;
    if (c.mode != LQ_MODE_WINDOW) return LQ_OK;
    if (!h->prefilled) return fail(LQ_ERR_STATE, "flush before lq_prefill_state");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // A ragged handle whose units share one phase flushes like a shared-phase
    // handle (every unit, or none when none is due) and clears the counts.
    const bool per_unit = c.ragged && !h->aligned;
    if (c.ragged && h->aligned && h->n_buf < flush_min) return LQ_OK;
    lq::EncodeArgs a;
    a.w = views(h);
    a.S0 = nullptr;
    a.from_buffer = 1;
    a.n_buf = h->n_buf;
    a.n_rows = c.n_comp_rows;
    a.n_cols = c.n_comp_cols;
    a.smooth = c.smooth;
    a.select = c.select;
    a.fill = per_unit ? reinterpret_cast<int32_t *>(h->ws + h->lay.fill) : nullptr;
    a.flush_min = flush_min;
    a.seq_mask = nullptr;
    a.heads = c.heads;
    cudaError_t e = lq::launch_encode(a, c.d_k, c.gate, c.in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "launching the flush kernel");
    if (c.ragged && h->aligned) {
        e = cudaMemsetAsync(h->ws + h->lay.fill, 0, (size_t)c.batch * c.heads * 4, s);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the window counts");
    }
    if (c.ragged && flush_min <= 1) h->aligned = 1;     // every unit's window is empty again
    h->n_buf = 0;
    return LQ_OK;
}

}  // namespace

lq_status lq_decode_step(lq_handle h, const void *d_q, const void *d_k, const void *d_v, const float *d_g,
                         const float *d_beta, float *d_o, void *stream) {
    Range nvtx_range("lq_decode_step");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    return decode_impl(h, d_q, d_k, d_v, d_g, d_beta, nullptr, d_o, stream);
}

lq_status lq_decode_step_active(lq_handle h, const void *d_q, const void *d_k, const void *d_v, const float *d_g,
                                const float *d_beta, const uint8_t *d_active, float *d_o, void *stream) {
    Range nvtx_range("lq_decode_step_active");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    if (!h->cfg.ragged) return fail(LQ_ERR_STATE, "lq_decode_step_active needs a ragged handle");
    return decode_impl(h, d_q, d_k, d_v, d_g, d_beta, d_active, d_o, stream);
}

lq_status lq_window_flush(lq_handle h, void *stream) {
    Range nvtx_range("lq_window_flush");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    return flush_impl(h, h->cfg.window, stream);
}

lq_status lq_window_flush_pending(lq_handle h, void *stream) {
    Range nvtx_range("lq_window_flush_pending");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    return flush_impl(h, 1, stream);
}

lq_status lq_prefill_sequences(lq_handle h, const float *d_S0, const uint8_t *d_mask, void *stream) {
    Range nvtx_range("lq_prefill_sequences");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    h->codes_settled = 0;
    const lq_config &c = h->cfg;
    if (!c.ragged) return fail(LQ_ERR_STATE, "lq_prefill_sequences needs a ragged handle");
    if (!h->prefilled) return fail(LQ_ERR_STATE, "lq_prefill_sequences before lq_prefill_state");
    if (d_mask == nullptr) return fail(LQ_ERR_INVALID_ARG, "NULL sequence mask");
    if (d_S0 != nullptr && !aligned(d_S0, 16)) return fail(LQ_ERR_INVALID_ARG, "S0 must be 16-byte aligned");
    lq::EncodeArgs a;
    a.w = views(h);
    a.S0 = d_S0;
    a.from_buffer = 0;
    a.n_buf = 0;
    a.n_rows = c.n_comp_rows;
    a.n_cols = c.n_comp_cols;
    a.smooth = c.smooth;
    a.select = c.select;
    a.fill = reinterpret_cast<int32_t *>(h->ws + h->lay.fill);
    a.flush_min = 0;
    a.seq_mask = d_mask;
    a.heads = c.heads;
    cudaError_t e = lq::launch_encode(a, c.d_k, c.gate, c.in_dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "launching the encode kernel");
    h->aligned = 0;                       // the restarted sequences start a new phase
    return LQ_OK;
}

lq_status lq_state_export(lq_handle h, const lq_export *dst, void *stream) {
    Range nvtx_range("lq_state_export");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    if (dst == nullptr) return fail(LQ_ERR_INVALID_ARG, "export destinations are NULL");
    const lq_config &c = h->cfg;
    const lq_layout &L = h->lay;
    const size_t N = (size_t)c.batch * c.heads, d = (size_t)c.d_k, W = (size_t)c.window;
    const size_t gd = (c.gate == LQ_GATE_CHANNEL) ? d : 1;
    const size_t key_b = (c.gate == LQ_GATE_CHANNEL || c.in_dtype == LQ_DTYPE_F32) ? 4 : 2;
    const size_t ncomp = (size_t)(c.n_comp_rows + c.n_comp_cols);
    // (destination, workspace offset, rows, packed row bytes, workspace row pitch)
    struct Region {
        void *dst;
        size_t off, rows, row_bytes, pitch;
        const char *name;
    };
    const Region regions[] = {
        {dst->codes, L.codes, N, d * d, d * d, "codes"},
        {dst->row_scale, L.row_scale, N, d * 4, d * 4, "row_scale"},
        {dst->col_smooth, L.col_smooth, N, d * 4, d * 4, "col_smooth"},
        {dst->comp_index, L.comp_index, N, ncomp * 4, (size_t)L.comp_index_stride * 4, "comp_index"},
        {dst->comp_row_vec, L.comp_row_vec, N, (size_t)c.n_comp_rows * d * 4, (size_t)c.n_comp_rows * d * 4,
         "comp_row_vec"},
        {dst->comp_col_vec, L.comp_col_vec, N, (size_t)c.n_comp_cols * d * 4, (size_t)c.n_comp_cols * d * 4,
         "comp_col_vec"},
        {dst->buf_delta, L.buf_delta, N, W * d * 4, W * d * 4, "buf_delta"},
        {dst->buf_key, L.buf_key, N, W * d * key_b, W * d * key_b, "buf_key"},
        {dst->buf_gate, L.buf_gate, N, W * 4, (size_t)L.window_pad * 4, "buf_gate"},
        {dst->gate_sum, L.gate_sum, N, gd * 8, gd * 8, "gate_sum"},
        {dst->state_f32, L.state_f32, N, d * d * 4, d * d * 4, "state_f32"},
    };
    // every requested region must exist before anything is copied
    for (const Region &r : regions)
        if (r.dst != nullptr && r.off == LQ_ABSENT)
            return fail(LQ_ERR_INVALID_ARG, std::string("this handle's mode keeps no ") + r.name);
    if (dst->fill != nullptr && c.mode != LQ_MODE_WINDOW)
        return fail(LQ_ERR_INVALID_ARG, "this handle's mode keeps no window counts");
    if (!h->prefilled) return fail(LQ_ERR_STATE, "export before lq_prefill_state");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    for (const Region &r : regions) {
        if (r.dst == nullptr || r.row_bytes == 0) continue;
        if (r.row_bytes == r.pitch)
            e = cudaMemcpyAsync(r.dst, h->ws + r.off, r.rows * r.row_bytes, cudaMemcpyDefault, s);
        else
            e = cudaMemcpy2DAsync(r.dst, r.row_bytes, h->ws + r.off, r.pitch, r.row_bytes, r.rows, cudaMemcpyDefault,
                                  s);
        if (e != cudaSuccess) return cuda_fail(e, (std::string("exporting ") + r.name).c_str());
    }
    // window counts: on the device for ragged handles, else the handle's shared count
    std::vector<int32_t> shared_fill;
    if (dst->fill != nullptr) {
        if (c.ragged) {
            e = cudaMemcpyAsync(dst->fill, h->ws + L.fill, N * 4, cudaMemcpyDefault, s);
        } else {
            shared_fill.assign(N, h->n_buf);
            e = cudaMemcpyAsync(dst->fill, shared_fill.data(), N * 4, cudaMemcpyDefault, s);
        }
        if (e != cudaSuccess) return cuda_fail(e, "exporting the window counts");
    }
    // drains the stream (the host count buffer stays alive until then) and
    // reports the error word
    return lq_device_status(h, stream);
}

lq_status lq_device_status(lq_handle h, void *stream) {
    Range nvtx_range("lq_device_status");
    if (!check_handle(h)) return fail(LQ_ERR_INVALID_ARG, "invalid handle");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "synchronizing the stream");
    int32_t word[3] = {0, 0, 0};
    e = cudaMemcpy(word, h->ws + h->lay.err, sizeof(word), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
    if (word[0] == LQ_DEVERR_NONE) return LQ_OK;
    char buf[160];
    if (word[0] == LQ_DEVERR_WINDOW_FULL) {
        snprintf(buf, sizeof buf, "decode into a full window at unit %d (%d tokens buffered): flush after every step",
                 word[1], word[2]);
        return fail(LQ_ERR_WINDOW_FULL, buf);
    }
    if (word[0] == LQ_DEVERR_RANGE) {
        snprintf(buf, sizeof buf, "gate sum outside +-80 at unit %d, key channel %d: flush more often", word[1], word[2]);
        return fail(LQ_ERR_RANGE, buf);
    }
    if (word[0] == LQ_DEVERR_BOUNDS && word[2] == -50) {
        snprintf(buf, sizeof buf, "unit ticket out of range: a ticket counter was left set (after a device error); "
                 "prefill the state again");
        return fail(LQ_ERR_DEVICE, buf);
    }
    if (word[0] == LQ_DEVERR_BOUNDS) {
        snprintf(buf, sizeof buf, "index out of range at unit %d (check site %d; bounds-checked build): the "
                 "workspace holds an inconsistent state", word[1], word[2]);
        return fail(LQ_ERR_DEVICE, buf);
    }
    snprintf(buf, sizeof buf, "device error %d at unit %d (detail %d)", word[0], word[1], word[2]);
    return fail(LQ_ERR_DEVICE, buf);
}

const char *lq_last_error_string(void) { return g_last_error.c_str(); }

}  // extern "C"
