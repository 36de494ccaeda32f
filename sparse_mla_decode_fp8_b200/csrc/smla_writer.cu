// smla_writer.cu -- the KV-cache writer: new 512-d latents quantised into the FP8 paged
// cache format the decode kernel reads, and scattered to their (page, slot).
//
// Byte layout: "The Validation Gate: Writing a Standalone Correctness Test for a Custom
// MMA Sparse-Decode Kernel", section "The Test Design" (256-token pages: 256 rows of 448
// e4m3 nope bytes + 64 little-endian bf16 rope values, then 256 scale rows of 8 bytes);
// the page indexing of "The Validation Moment" (page = block_table[b][pos / 256],
// slot = pos % 256).  The pages do not state how the scales are chosen; the writer takes
// the rule of the synthetic caches: per 64-dim nope group, the smallest exponent e with
// max|x| <= 448 * 2^e (clamped to [-127, 127], -127 for an all-zero group), scale byte
// e + 127, nope byte = e4m3 of x / 2^e rounded to nearest even, rope = bf16 of x rounded
// to nearest even.
//
// One warp per token: lane l < 28 quantises nope dims [16l, 16l+16) (a 64-dim group is
// four lanes, whose max is two shuffles away), lanes 28..31 convert the 64 rope values;
// the 576-byte row is written with coalesced 16-byte stores and lane 0 writes the
// 8-byte scale row.  HBM-bound: 2 KB (fp32) or 1 KB (bf16) read and 584 bytes written
// per token.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/smla.h"
#include "smla_device.cuh"

namespace smla {

constexpr int kWriterWarps = 8;  // tokens per 256-thread block

// Two fp32 values -> two e4m3 bytes (lo in the low byte), round to nearest even,
// saturating at +-448 (infinities too).
__device__ __forceinline__ uint32_t e4m3x2_rn_satfinite(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Smallest e with amax <= 448 * 2^e = 1.75 * 2^(e+8), from amax's binary32 fields:
// amax = (1 + m / 2^23) * 2^(E-127) needs e = E-127-8, one more if its significand
// exceeds 1.75.  Subnormal or zero amax (below 448 * 2^-127) gives the clamp, -127.
__device__ __forceinline__ int scale_exponent(float amax) {
    const uint32_t bits = __float_as_uint(amax);
    const int E = static_cast<int>((bits >> 23) & 0xFFu);
    if (E == 0) return -127;
    const int e = (E - 127) - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return e < -127 ? -127 : e;  // finite amax: e <= 119
}

__device__ __forceinline__ uint32_t bf16_rn(float x) {
    if (isnan(x)) return 0x7FC0u;
    uint32_t r;
    asm("{\n\t.reg .b16 h;\n\tcvt.rn.bf16.f32 h, %1;\n\tmov.b32 %0, {h, 0};\n\t}" : "=r"(r) : "f"(x));
    return r & 0xFFFFu;
}

__device__ __forceinline__ void load16_latent(const void *latents, int bf16, size_t token, int lane, float (&x)[16]) {
    if (bf16) {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(latents) + token * kDim) +
                           2 * lane;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint4 v = __ldg(src + k);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[8 * k + 2 * j] = __uint_as_float(w[j] << 16);
                x[8 * k + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        }
    } else {
        const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(latents) + token * kDim) +
                            4 * lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 v = __ldg(src + k);
            x[4 * k] = v.x;
            x[4 * k + 1] = v.y;
            x[4 * k + 2] = v.z;
            x[4 * k + 3] = v.w;
        }
    }
}

__global__ void __launch_bounds__(32 * kWriterWarps) write_kv_kernel(
    const void *__restrict__ latents, int bf16, int n, const int32_t *__restrict__ req,
    const int32_t *__restrict__ pos, const int32_t *__restrict__ block_table, int B, int max_blocks,
    long long num_pages, uint8_t *__restrict__ cache, uint32_t *err) {
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * kWriterWarps + (threadIdx.x >> 5);
    if (i >= n) return;  // warp-uniform
    const int b = __ldg(req + i), p = __ldg(pos + i);
    int page = -1;
    if (b >= 0 && b < B && p >= 0 && (p >> 8) < max_blocks)
        page = __ldg(block_table + static_cast<size_t>(b) * max_blocks + (p >> 8));
    if (page < 0 || static_cast<long long>(page) >= num_pages) {
        if (lane == 0 && err) atomicOr(err, SMLA_FLAG_BAD_PAGE);
        return;
    }
    const int code = page * kPageTokens + (p & (kPageTokens - 1));
    uint8_t *row = const_cast<uint8_t *>(token_row(cache, code));

    float x[16];
    load16_latent(latents, bf16, static_cast<size_t>(i), lane, x);
    // the group's max |x| and whether it holds a non-finite value (lanes 4g..4g+3)
    float amax = 0.0f;
    uint32_t bad = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        amax = fmaxf(amax, fabsf(x[k]));
        bad |= isfinite(x[k]) ? 0u : 1u;
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        bad |= __shfl_xor_sync(0xffffffffu, bad, o);
    }
    const int e = bad ? 127 : scale_exponent(amax);
    if (lane < 28) {
        // 2^-e (a normal binary32 for e <= 126, the subnormal 2^-127 for e = 127): x / 2^e is
        // exact, or below 2^-126 where e4m3 rounds it to zero anyway
        const float inv = __uint_as_float(e <= 126 ? static_cast<uint32_t>(127 - e) << 23 : 0x00400000u);
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t v = e4m3x2_rn_satfinite(x[4 * k] * inv, x[4 * k + 1] * inv) |
                         (e4m3x2_rn_satfinite(x[4 * k + 2] * inv, x[4 * k + 3] * inv) << 16);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (isnan(x[4 * k + j])) v = (v & ~(0xFFu << (8 * j))) | (0x7Fu << (8 * j));
            w[k] = v;
        }
        *reinterpret_cast<uint4 *>(row + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = bf16_rn(x[2 * k]) | (bf16_rn(x[2 * k + 1]) << 16);
        uint4 *dst = reinterpret_cast<uint4 *>(row + kNope + 32 * (lane - 28));
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
    // scale row: byte g from lane 4g, byte 7 zero
    const uint32_t sbyte = static_cast<uint32_t>(e + 127);
    uint32_t s[7];
#pragma unroll
    for (int g = 0; g < 7; ++g) s[g] = __shfl_sync(0xffffffffu, sbyte, 4 * g);
    if (lane == 0) {
        uint8_t *srow = const_cast<uint8_t *>(token_scales(cache, code));
        *reinterpret_cast<uint2 *>(srow) =
            make_uint2(s[0] | (s[1] << 8) | (s[2] << 16) | (s[3] << 24), s[4] | (s[5] << 8) | (s[6] << 16));
    }
}

}  // namespace smla

namespace {

constexpr int kWriterMaxDevices = 64;
std::mutex g_writer_mutex;
int g_writer_supported[kWriterMaxDevices] = {};  // 0 unknown, 1 sm_100, -1 other

int writer_device_ok() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kWriterMaxDevices) return SMLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_writer_mutex);
    if (g_writer_supported[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return SMLA_ERR_CUDA;
        g_writer_supported[dev] = (major == 10 && minor == 0) ? 1 : -1;
    }
    return g_writer_supported[dev] > 0 ? SMLA_OK : SMLA_ERR_DEVICE;
}

bool aligned_to(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int smla_write_kv(const void *latents, int latents_bf16, int n, const int32_t *req, const int32_t *pos,
                             const int32_t *block_table, int B, int max_blocks, int num_pages, uint8_t *kv_cache,
                             uint32_t *err, void *stream) {
    if (n < 0 || B < 1 || max_blocks < 1 || num_pages < 1 || num_pages >= (1 << 23)) return SMLA_ERR_INVALID;
    if (n == 0) return SMLA_OK;
    if (!latents || !req || !pos || !block_table || !kv_cache) return SMLA_ERR_INVALID;
    if (!aligned_to(latents, 16) || !aligned_to(kv_cache, 16) || !aligned_to(req, 4) || !aligned_to(pos, 4) ||
        !aligned_to(block_table, 4) || (err && !aligned_to(err, 4)))
        return SMLA_ERR_INVALID;
    const int rc = writer_device_ok();
    if (rc != SMLA_OK) return rc;
    (void)cudaGetLastError();
    const unsigned blocks = static_cast<unsigned>((n + smla::kWriterWarps - 1) / smla::kWriterWarps);
    smla::write_kv_kernel<<<blocks, 32 * smla::kWriterWarps, 0, static_cast<cudaStream_t>(stream)>>>(
        latents, latents_bf16 ? 1 : 0, n, req, pos, block_table, B, max_blocks, num_pages, kv_cache, err);
    return cudaGetLastError() == cudaSuccess ? SMLA_OK : SMLA_ERR_LAUNCH;
}
