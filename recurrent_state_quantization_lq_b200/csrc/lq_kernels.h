// Host-side launchers of the liblq kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "lq_common.cuh"

namespace lq {

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
