// smla_device.cuh -- cache layout constants, index translation and FP8/UE8M0
// dequantisation shared by the decode kernel and the gather debug kernel.
//
// Layout ("The Validation Gate: Writing a Standalone Correctness Test for a
// Custom MMA Sparse-Decode Kernel", section "The Test Design"): a page holds 256
// token rows of 576 bytes (448 e4m3 nope bytes, 64 little-endian bf16 rope
// values) followed by 256 scale rows of 8 bytes (UE8M0, one per 64 nope dims).
// Page indexing ("The Validation Moment"): page = block_table[b][idx / 256],
// slot = idx % 256.
#pragma once

#include <cstdint>

#include "../../include/smla.h"
#include "sm100_ptx.cuh"

namespace smla {

constexpr int kHeads = 64;
constexpr int kDim = 512;
constexpr int kNope = 448;
constexpr int kPageTokens = 256;
constexpr int kRowBytes = 576;
constexpr int kScaleRowBytes = 8;
constexpr long long kPageBytes = 149504;
constexpr long long kScaleBlockOffset = 147456;
constexpr int kRowChunks = kRowBytes / 16;  // 36 sixteen-byte chunks per token row
constexpr int kNopeChunks = kNope / 16;     // 28 of them are nope (16 dims each)

static_assert(kRowBytes % 16 == 0, "token rows must stay 16-byte aligned");
static_assert(kPageBytes % 128 == 0, "pages must stay 128-byte aligned");
static_assert(kPageBytes == kPageTokens * (kRowBytes + kScaleRowBytes), "page size");
static_assert(kScaleBlockOffset == kPageTokens * kRowBytes, "scale block follows the rows");

// Index translation in two steps, so a caller can put the block-table load between
// them (the decode kernel keeps that load in flight while it computes).
//   1. slot_in_range: 0 <= idx < seq_len and idx / 256 < max_blocks; only then is
//      block_table[b][idx / 256] read.
//   2. slot_code: token code = page * 256 + idx % 256, or -1 (and the error bit)
//      for a block-table entry outside [0, num_pages).
__device__ __forceinline__ bool slot_in_range(int idx, int seq_len, int max_blocks) {
    return idx >= 0 && idx < seq_len && (idx >> 8) < max_blocks;
}
__device__ __forceinline__ int slot_code(int idx, int page, long long num_pages, uint32_t *err) {
    if (page < 0 || static_cast<long long>(page) >= num_pages) {
        atomicOr(err, SMLA_FLAG_BAD_PAGE);
        return -1;
    }
    return page * kPageTokens + (idx & (kPageTokens - 1));
}

// Token code = page * 256 + slot for a valid topk slot, else -1.  A block-table
// entry outside [0, num_pages) is masked and reported in the error word.
__device__ __forceinline__ int translate_slot(const int32_t *bt_row, int max_blocks, int seq_len,
                                              long long num_pages, int idx, uint32_t *err) {
    if (!slot_in_range(idx, seq_len, max_blocks)) return -1;
    return slot_code(idx, __ldg(bt_row + (idx >> 8)), num_pages, err);
}

__device__ __forceinline__ const uint8_t *token_row(const uint8_t *cache, int code) {
    return cache + static_cast<size_t>(code >> 8) * kPageBytes + static_cast<size_t>(code & 255) * kRowBytes;
}

__device__ __forceinline__ const uint8_t *token_scales(const uint8_t *cache, int code) {
    return cache + static_cast<size_t>(code >> 8) * kPageBytes + kScaleBlockOffset +
           static_cast<size_t>(code & 255) * kScaleRowBytes;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Two e4m3 bytes (low byte -> low half) -> bf16x2 holding value * 2^-112.
// The hardware conversion gives f16, where every e4m3 value is a normal number
// with at most 3 mantissa bits; moving its 5-bit exponent and top mantissa bits
// into bf16 position reads the same bits with bias 127 instead of 15, i.e. scales
// by 2^-112, exactly (zero stays zero).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2_shifted(uint32_t two_bytes) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<unsigned short>(two_bytes)));
    return ((h2 >> 3) & 0x0FFF0FFFu) | (h2 & 0x80008000u);
}

// Scale bytes above 142: 2^(s-15) is not a bf16 normal, so multiply by 2^127 and then by
// 2^(s-142); 0xFF gives NaN.  Inline like the common path: an out-of-line call would take
// the address of o, which then lives in local memory on every dequantisation.
__device__ __forceinline__ void scale_big(uint32_t (&o)[8], uint32_t s) {
    const uint32_t big = 0x7F007F00u;                              // 2^127 in both halves
    const uint32_t m = (s == 255u) ? 0x7FC0u : ((s - 15u) << 7);  // 2^(s-142) or NaN
    const uint32_t m2 = m | (m << 16);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = bf16x2_mul(bf16x2_mul(o[i], big), m2);
}

// 16 e4m3 bytes with UE8M0 scale byte s -> 16 bf16 values e4m3 * 2^(s-127),
// returned as two 16-byte chunks (dims 0-7, dims 8-15).  One bf16 multiply by
// 2^(s-15) (two for s > 142, whose factor is not a bf16 normal); 0xFF gives NaN.
__device__ __forceinline__ void dequant16(const uint4 raw, const uint32_t s, uint4 &lo, uint4 &hi) {
    uint32_t o[8];
    o[0] = e4m3x2_to_bf16x2_shifted(raw.x & 0xFFFFu);
    o[1] = e4m3x2_to_bf16x2_shifted(raw.x >> 16);
    o[2] = e4m3x2_to_bf16x2_shifted(raw.y & 0xFFFFu);
    o[3] = e4m3x2_to_bf16x2_shifted(raw.y >> 16);
    o[4] = e4m3x2_to_bf16x2_shifted(raw.z & 0xFFFFu);
    o[5] = e4m3x2_to_bf16x2_shifted(raw.z >> 16);
    o[6] = e4m3x2_to_bf16x2_shifted(raw.w & 0xFFFFu);
    o[7] = e4m3x2_to_bf16x2_shifted(raw.w >> 16);
    if (s <= 142u) {
        const uint32_t m = (s + 112u) << 7;  // bf16 bits of 2^(s-15)
        const uint32_t m2 = m | (m << 16);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = bf16x2_mul(o[i], m2);
    } else {
        scale_big(o, s);
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ uint32_t scale_byte(const uint2 sc, int g) {
    const uint32_t w = (g < 4) ? sc.x : sc.y;
    return (w >> ((g & 3) * 8)) & 0xFFu;
}

}  // namespace smla
