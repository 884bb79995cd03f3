// Device pieces shared by the windowed decode kernels (internal to liblq):
// the meta segment layout, key loads, named barriers, the tile swizzle, the
// exact int8 digit split of the INT8 pass and the tcgen05 / mma.sync pieces
// that consume it.  See lq_decode_window.cu for the method.
#pragma once

#include <cuda.h>

#include "lq_common.cuh"

namespace lq {
namespace dec {

constexpr double kMaxAbsGateSum = 80.0;

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Offsets inside a meta segment.
struct Meta {
    int sig, s, qin, kin, vin, gin, gsum, cidx, crow, ccol, bytes;
};

template <int D, bool KDA, typename InT>
__host__ __device__ Meta meta_layout(int ncr, int ncc, int cis) {
    Meta m{};
    int o = 0;
    m.sig = o;  o += 4 * D;
    m.s = o;    o += 4 * D;
    m.qin = o;  o += (int)sizeof(InT) * D;
    m.kin = o;  o += (int)sizeof(InT) * D;
    m.vin = o;  o += (int)sizeof(InT) * D;
    m.gin = o;  o += KDA ? 4 * D : 0;
    m.gsum = o; o += KDA ? 8 * D : 0;
    m.cidx = o; o += (ncr + ncc) > 0 ? 4 * cis : 0;
    m.crow = o; o += 4 * D * ncr;
    m.ccol = o; o += 4 * D * ncc;
    m.bytes = o;
    return m;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x) { return static_cast<float>(x); }
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }

template <typename KeyT, int VPL>
__device__ __forceinline__ void load_key(const KeyT *p, float (&out)[VPL]) {
    if constexpr (sizeof(KeyT) == 2) {
        if constexpr (VPL == 4) {
            uint2 w = *reinterpret_cast<const uint2 *>(p);
            out[0] = bf16_bits_to_f32(w.x & 0xffffu); out[1] = bf16_bits_to_f32(w.x >> 16);
            out[2] = bf16_bits_to_f32(w.y & 0xffffu); out[3] = bf16_bits_to_f32(w.y >> 16);
        } else {
            uint32_t w = *reinterpret_cast<const uint32_t *>(p);
            out[0] = bf16_bits_to_f32(w & 0xffffu); out[1] = bf16_bits_to_f32(w >> 16);
        }
    } else {
        if constexpr (VPL == 4) {
            float4 w = *reinterpret_cast<const float4 *>(p);
            out[0] = w.x; out[1] = w.y; out[2] = w.z; out[3] = w.w;
        } else {
            float2 w = *reinterpret_cast<const float2 *>(p);
            out[0] = w.x; out[1] = w.y;
        }
    }
}

// Named barrier `id` over `count` threads that also ORs a predicate over them.
__device__ __forceinline__ bool named_sync_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void named_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// `count` arrivals at once (for a barrier that waits on a whole thread group
// that one thread speaks for).
__device__ __forceinline__ void mbar_arrive_n(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Byte offset of the 16-byte chunk `chunk` of row `row` in a D x D int8 tile
// written by the tensor copy with the 128-byte (D = 128) or 64-byte (D = 64)
// swizzle: the chunk index is XORed with address bits 7-9 (resp. 7-8).
template <int D>
__device__ __forceinline__ int swz(int row, int chunk) {
    if constexpr (D == 128) return row * 128 + ((chunk ^ (row & 7)) << 4);
    else return row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4);
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D (16x8 s32) += A (16x32 s8, row) * B (32x8 s8, col)
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2-D tensor copy of the (x, y) box of `map` into shared memory.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// tcgen05 pieces of the d = 128 INT8 pass.  Both operands are K-major with
// 128-byte swizzle: rows of 128 int8 (one row of the state tile, or one digit
// column), 8-row groups 1024 B apart, 16-byte pieces permuted by the row's
// index mod 8 -- the layout the tile's 2-D tensor copy writes.
constexpr int kTmemCols = 64;                 // 4 blocks x 16 accumulator columns
// s32 accumulator, s8 A and B, both K-major, N = 16, M = 128
constexpr uint32_t kI8Idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fff);   // start address
    d |= (uint64_t)(16 >> 4) << 16;           // leading byte offset (unused with this swizzle)
    d |= (uint64_t)(1024 >> 4) << 32;         // stride byte offset: 8-row groups
    d |= (uint64_t)1 << 46;                   // descriptor version
    d |= (uint64_t)2 << 61;                   // 128-byte swizzle
    return d;
}
__device__ __forceinline__ int sw128_off(int row, int kbyte) {
    return (row >> 3) * 1024 + (row & 7) * 128 + ((((kbyte >> 4) ^ (row & 7))) << 4) + (kbyte & 15);
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Exact int -> float for |x| < 2^22 without the conversion unit: at 1.5 * 2^23
// the float spacing is 1, so the word 0x4B400000 + x is the number 1.5 * 2^23 + x.
__device__ __forceinline__ float i2f_exact(int x) { return __int_as_float(0x4B400000 + x) - 12582912.0f; }

// 2^k as a float, for |k| <= 126.
__device__ __forceinline__ float pow2i(int k) { return __int_as_float((127 + k) << 23); }

// Block exponent of a block with maximum |y| = m: 2^E with m 2^-E in [32, 64),
// returned as (2^-E, 2^E); (0, 0) for a block too small to matter.
__device__ __forceinline__ float2 block_scale(float m) {
    const int biased = (__float_as_int(m) >> 23) & 0xff;     // m = 1.f x 2^(biased - 127)
    if (biased < 20) return make_float2(0.0f, 0.0f);          // |y| < 2^-107 (or zero)
    const int E = biased - 127 + 1 - 6;
    return make_float2(pow2i(-E), pow2i(E));
}

// The four base-2^7 int8 digits of y * 2^-E (|y 2^-E| < 64), packed low to high.
// Every |r| here is at most 64, so adding 1.5 * 2^23 rounds r to an integer
// (to nearest, ties to even, as rintf) with no conversion instruction: the
// sum minus 1.5 * 2^23 is the digit as a float, and the sum's low byte is its
// two's-complement byte.
__device__ __forceinline__ uint32_t digits4(float y, float down) {
    float r = y * down;
    uint32_t out = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float t = __fadd_rn(r, 12582912.0f);
        const float d = __fsub_rn(t, 12582912.0f);
        out |= (__float_as_uint(t) & 0xffu) << (8 * p);
        r = (r - d) * 128.0f;
    }
    return out;
}

}  // namespace dec
}  // namespace lq
