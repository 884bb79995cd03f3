// Host-side launchers of the liblq kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "lq_common.cuh"

namespace lq {

constexpr int kMaxDevices = 64;

// A positive per-device value that a launcher computes on its first call on a
// device (an occupancy figure, or 1 once a function attribute is set) and then
// reuses, so that launches inside a stream capture make no runtime queries.
// Different handles may be driven from different host threads: the first
// calls on a device are serialized and `make` runs once per device until it
// succeeds; later calls read the value without taking the lock.
class DeviceCache {
  public:
    template <typename F>
    cudaError_t get(int dev, int *out, F &&make) {
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        int v = value_[dev].load(std::memory_order_acquire);
        if (v <= 0) {
            std::lock_guard<std::mutex> lock(mutex_);
            v = value_[dev].load(std::memory_order_relaxed);
            if (v <= 0) {
                const cudaError_t e = make(&v);
                if (e != cudaSuccess) return e;
                if (v <= 0) return cudaErrorInvalidConfiguration;
                value_[dev].store(v, std::memory_order_release);
            }
        }
        *out = v;
        return cudaSuccess;
    }

  private:
    std::atomic<int> value_[kMaxDevices] = {};
    std::mutex mutex_;
};

// Streaming multiprocessors of the current device (148 on a B200 if the query
// fails).
inline int sm_count() {
    static DeviceCache cache;
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    const cudaError_t e = cache.get(dev, &n, [dev](int *v) {
        if (cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || *v <= 0) *v = 148;
        return cudaSuccess;
    });
    return e == cudaSuccess ? n : 148;
}

// Set a kernel's dynamic shared-memory limit once per device (one cache per
// kernel: the template is keyed on the kernel's address, not on its type).
template <auto kern>
cudaError_t opt_in_smem(int bytes) {
    static DeviceCache cache;
    int dev = 0, done = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    return cache.get(dev, &done, [&](int *v) {
        const cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        *v = 1;
        return r;
    });
}

struct EncodeArgs {
    Views w;
    const float *S0;   // prefill source [N][d][d], or nullptr for zeros (prefill only)
    int from_buffer;   // 1: window flush (stored state + buffer); 0: prefill
    int n_buf;         // buffered tokens (flush)
    int n_rows;        // compensator rows to extract
    int n_cols;        // compensator columns to extract
    int smooth;        // column smoothing on/off
    int select;        // LQ_SELECT_*
    // ragged window phases: per-unit buffered counts (null: n_buf for every unit)
    int32_t *fill;
    int flush_min;     // ragged flush: units holding at least this many tokens
    const uint8_t *seq_mask;   // prefill: sequences to encode (null: all)
    int heads;         // units per sequence (for seq_mask)
};

struct DecodeArgs {
    Views w;
    const void *q;
    const void *k;
    const void *v;
    const float *g;
    const float *beta;
    float *o;
    int n_buf;         // tokens buffered before this one (windowed mode)
    const void *codes_map;   // host copy of the tensor map of the INT8 codes (windowed mode)
    // ragged window phases: per-unit buffered counts (null: n_buf for every
    // unit) and per-sequence activity (null: all active)
    int32_t *fill;
    const uint8_t *active;
    int heads;         // units per sequence
    // The INT8 codes were last written before the kernel that precedes this
    // launch in its stream: the first code tile may be fetched before that
    // kernel completes (shared window phases only).
    int codes_settled;
};

struct TokenPrefillArgs {
    Views w;
    const float *S0;   // starting state [N][d][d], or nullptr for zeros
    const void *q;     // prompt inputs [T][N][d] (in_dtype)
    const void *k;
    const void *v;
    const float *g;    // log alpha [T][N] (GDN) or [T][N][d] (KDA)
    const float *beta; // [T][N]
    float *o;          // outputs [T][N][d], or nullptr
    int n_tokens;      // T
    int n_rows;        // compensator rows to extract
    int n_cols;        // compensator columns to extract
    int smooth;        // column smoothing on/off
    int select;        // LQ_SELECT_*
    int fp32_state;    // 1: store the FP32 state (FP32 mode) instead of encoding it
    // ragged restarts: sequences to prefill (null: all), per-sequence prompt
    // lengths <= n_tokens (null: n_tokens), units per sequence, counts to clear
    const uint8_t *seq_mask;
    const int32_t *lengths;
    int heads;
    int32_t *fill;
};

// Encode the tensor map the windowed decode uses to load one unit's INT8 tile
// (d x d, 128- or 64-byte swizzle) from `codes` ([units][d][d]).  Host only.
cudaError_t make_codes_map(void *map_out, const int8_t *codes, int d, int units);

// d = d_k = d_v in {64, 128}; gate: LQ_GATE_*; in_dtype: LQ_DTYPE_*.
cudaError_t launch_encode(const EncodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s);
cudaError_t launch_flush_split(const EncodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s);
cudaError_t launch_prefill_tokens(const TokenPrefillArgs &a, int d, int gate, int in_dtype, cudaStream_t s);
cudaError_t launch_decode_window(const DecodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s);
cudaError_t launch_decode_fp32(const DecodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s);
cudaError_t launch_decode_naive(const DecodeArgs &a, int d, int gate, int in_dtype, cudaStream_t s);

}  // namespace lq
