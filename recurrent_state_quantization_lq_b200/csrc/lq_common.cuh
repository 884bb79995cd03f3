// Device helpers shared by the liblq kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lq.h"

namespace lq {

// ---------------------------------------------------------------- launch params

// Pointers into one workspace plus the per-call inputs; every kernel reads the
// fields it needs.  Unit u = sequence * heads + head.
struct Views {
    int32_t *err;
    int8_t *codes;
    float *row_scale;
    float *col_smooth;
    int32_t *comp_index;
    float *comp_row_vec;
    float *comp_col_vec;
    double *gate_sum;
    float *buf_delta;
    void *buf_key;
    float *buf_gate;
    float *state_f32;
    int comp_index_stride;
    int window;
    int window_pad;
    int n_comp_rows;
    int n_comp_cols;
    int units;
};

// ------------------------------------------------------------------ conversions

// Exact int8 -> float for the four bytes of a word.  With u = b + 128 in
// [0, 255] (the byte with its sign bit flipped), the IEEE-754 binary32 word
// 0x4B000000 | u is the number 2^23 + u exactly, because at 2^23 the 23-bit
// fraction counts in units of 1; subtracting 2^23 + 128 leaves b exactly.  One
// byte permute and one add per value, both on full-rate pipes.
__device__ __forceinline__ void i8x4_to_f32(uint32_t w, float &f0, float &f1, float &f2, float &f3) {
    const uint32_t u = w ^ 0x80808080u;
    const float bias = 8388736.0f;  // 2^23 + 128
    f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)) - bias;
    f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541)) - bias;
    f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)) - bias;
    f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543)) - bias;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// ------------------------------------------------------------------- reductions

template <int WIDTH>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <int WIDTH>
__device__ __forceinline__ float group_max(float x) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// exp(x) for a double x with |x| <= 80, to about two float ulps: expf of the
// float-rounded argument, corrected to first order by the rounding remainder
// (exp(xf + r) = exp(xf)(1 + r + O(r^2)) with |r| <= 2^-24 |x|).
__device__ __forceinline__ float exp_of_double(double x) {
    const float xf = (float)x;
    const float r = (float)(x - (double)xf);
    const float e = expf(xf);
    return fmaf(e, r, e);
}

// ------------------------------------------------------------- error reporting

__device__ __forceinline__ void report_error(int32_t *err, int code, int unit, int detail) {
    if (err == nullptr) return;
    if (atomicCAS(err, 0, code) == 0) {
        err[1] = unit;
        err[2] = detail;
    }
}

// ------------------------------------------------------ bounds-checked build
//
// Built with -DLQ_BOUNDS_CHECK (liblq_checked.so), the kernels test the
// indices they compute from workspace contents or launch arguments before
// they use them; an index outside its region is recorded as LQ_DEVERR_BOUNDS
// (unit, detail) and the access is skipped.  The normal build compiles every
// check away.
#ifdef LQ_BOUNDS_CHECK
constexpr bool kBoundsChecked = true;
#else
constexpr bool kBoundsChecked = false;
#endif

// True when lo <= idx < hi; in the checked build a violation is also reported.
__device__ __forceinline__ bool in_bounds(int32_t *err, long long idx, long long lo, long long hi, int unit,
                                          int detail) {
    if (!kBoundsChecked) return true;
    if (idx >= lo && idx < hi) return true;
    report_error(err, LQ_DEVERR_BOUNDS, unit, detail);
    return false;
}

// --------------------------------------------------------------- unit tickets
//
// A launch that hands out n_dyn of its units by ticket draws from a 64-bit
// counter in the workspace that is zero when it starts: ticket t < n_dyn names
// the launch's dynamic unit t, any other names none.  Each of the grid CTAs
// draws until it gets one that names none, so a launch draws exactly
// n_dyn + grid tickets, and the CTA that draws the last one sets the counter
// back to zero: no draw of this launch follows it, and the next launch draws
// only after this one has completed.  A ticket past the last one means the
// counter was not zero at the start (left by a launch that ended on a device
// error); it is reported as LQ_DEVERR_BOUNDS.  Returns the unit number or -1.
__device__ __forceinline__ int ticket_unit(unsigned long long t, int n_dyn, int grid, unsigned long long *counter,
                                           int32_t *err) {
    const unsigned long long last = (unsigned long long)n_dyn + (unsigned long long)grid - 1ull;
    // a plain store: every draw of this launch came before this thread's last
    // one, and an atomic exchange would hold the thread for its reply
    if (t == last) *reinterpret_cast<volatile unsigned long long *>(counter) = 0ull;
    else if (t > last) report_error(err, LQ_DEVERR_BOUNDS, -1, -50);
    return t < (unsigned long long)n_dyn ? (int)t : -1;
}

// ------------------------------------------------- mbarrier + bulk async copies

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Add `bytes` to the transaction count of the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, giving up after
// `budget_cycles` SM clocks.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long budget_cycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > budget_cycles) return false;
    }
}

// 1-D bulk copy global -> shared, completing `bytes` transaction bytes on
// `bar`.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Same, with an L2 eviction hint for data read once per call.
__device__ __forceinline__ void bulk_g2s_stream(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                                uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// --------------------------------------------- programmatic dependent launch
//
// A kernel launched with programmatic stream serialization may start while the
// kernel before it in the stream is still running.  It must not read anything
// that kernel may write, nor write anything it may read, before
// grid_dependency_wait() returns in the thread that makes the access; the
// wait returns once the earlier kernel has completed and its writes are
// visible (immediately, when the launch had no such attribute).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Let the next kernel in the stream start once every CTA of this grid has
// signalled (or exited).  Signalled only after this CTA's own wait, so that a
// kernel which starts early finds everything before its predecessor completed.
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// About one second at the B200's clocks: a bulk copy that has not landed by
// then never will.
constexpr long long kWaitBudgetCycles = 2000000000LL;

}  // namespace lq
