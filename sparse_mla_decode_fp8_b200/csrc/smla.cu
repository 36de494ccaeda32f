// smla.cu -- sparse MLA decode over an FP8 paged latent cache on B200 (sm_100a):
// the decode kernel (gather -> dequant -> tcgen05 QK^T -> fp32 online softmax ->
// tcgen05 PV), the split-K LSE-merge kernel, the gather debug kernel and the
// C ABI declared in include/smla.h.
//
// Method ("The Turning Point: Architecting a Custom MMA Sparse-MLA Decode
// Kernel"): one program per (request, topk split) handles all 64 heads, so each
// gathered KV tile is read once for every head (Step 3), the two contractions
// run on tensor cores with fp32 accumulation, and split partials are merged by
// their log-sum-exp (Step 5).
//
// B200 mapping, per CTA (one per SM, 256 threads):
//   * Q[b] (64 heads x 512, bf16) stays in shared memory for the whole CTA.
//   * A tile of 128 topk slots is translated through the block table, its FP8
//     rows are loaded with 16-byte loads and dequantised in registers into a
//     bf16 [128 x 512] tile in the 128-byte-swizzled layout the tensor core reads.
//   * S^T[128 tokens x 64 heads] = K_tile . Q^T: tcgen05.mma M=128 N=64, fp32 in
//     tensor memory.  Tokens fill the 128-row M dimension, not the 64 heads.
//   * Softmax warps (one thread per token lane) read S^T from tensor memory,
//     keep the running max / sum per head, rescale O^T in tensor memory when the
//     max grows, and write P^T as two bf16 terms (P = P_hi + P_lo).
//   * O^T[512 x 64] += V^T . P^T with V = the same bf16 tile read MN-major:
//     4 MMAs of M=128 per 16-token step, once with P_hi and once with P_lo, so P
//     carries ~16 significant bits (a single bf16 P is not accurate enough when
//     a few large latents dominate).
//   * The epilogue reads O^T from tensor memory and writes O/l (or a normalised
//     split partial) and LSE = (m + log2 l) ln 2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/smla.h"
#include "sm100_ptx.cuh"
#include "smla_device.cuh"

namespace smla {

constexpr int kThreads = 256;
constexpr int kTile = 128;

// Dynamic shared memory map (bytes from a 1024-aligned base).
constexpr int kSmemQ = 0;                           // 64 KB: 8 K-blocks x [64 heads x 128 B]
constexpr int kSmemKV = kSmemQ + 65536;             // 128 KB: 8 K-blocks x [128 tokens x 128 B]
constexpr int kSmemPhi = kSmemKV + 131072;          // 16 KB: [128 tokens x 64 heads] bf16
constexpr int kSmemPlo = kSmemPhi + 16384;          // 16 KB
constexpr int kSmemCodes = kSmemPlo + 16384;        // 128 int32 token codes
constexpr int kSmemScales = kSmemCodes + 512;       // 128 x 8 B scale rows; reused as [4][64] f32
constexpr int kSmemHeadM = kSmemScales + 1024;      // per-head running max (log2 units)
constexpr int kSmemHeadL = kSmemHeadM + 256;        // per-head running sum
constexpr int kSmemHeadAlpha = kSmemHeadL + 256;    // per-head rescale factor of this tile
constexpr int kSmemHeadMnew = kSmemHeadAlpha + 256;  // per-head max after this tile
constexpr int kSmemBar = kSmemHeadMnew + 256;       // mbarrier: MMA completion
constexpr int kSmemBarSpare = kSmemBar + 8;         // mbarrier: test hook
constexpr int kSmemTmemSlot = kSmemBarSpare + 8;
constexpr int kSmemBytes = kSmemTmemSlot + 16;
static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-block shared memory limit");

constexpr uint32_t kTmemCols = 512;  // O^T: columns [0,256), S^T: [256,320)
constexpr uint32_t kTmemS = 256;
constexpr uint32_t kIdescQK = idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16(128, 64, true, true);

struct DecodeParams {
    const uint16_t *q;
    const uint8_t *cache;
    const int32_t *block_table;
    const int32_t *topk_idx;
    const int32_t *seq_lens;
    float *out;
    float *lse;
    float *part_o;
    float *part_lse;
    uint32_t *err;
    long long num_pages;
    unsigned long long timeout_ns;
    int topk;
    int max_blocks;
    int nsplit;
    int tiles_per_split;
    float scale_log2;  // sm_scale * log2(e)
    uint32_t debug_flags;
};

struct MaxOp {
    __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct AddOp {
    __device__ __forceinline__ float operator()(float a, float b) const { return a + b; }
};

// Reduces 64 per-thread values across the 32 lanes of a warp, value i with value
// i of every other lane.  Afterwards lane L holds the results for entries 2L and
// 2L+1 in v[0], v[1].  Each round halves the live entries: a lane keeps the half
// selected by its lane bit and sends the other half to its partner.
template <class Op>
__device__ __forceinline__ void warp_transpose_reduce64(float (&v)[64], int lane, Op op) {
#pragma unroll
    for (int w = 32, off = 16; off >= 1; w >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float send = upper ? v[i] : v[i + w];
            const float keep = upper ? v[i + w] : v[i];
            v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, off));
        }
    }
}

// Stores one 16-byte chunk of a token row, dequantised, into the swizzled tile.
// c < 28: nope dims [16c, 16c+16) -> K-block c/4, chunks 2(c%4), 2(c%4)+1.
// c >= 28: rope dims [448 + 8(c-28), +8) -> K-block 7, chunk c-28, copied as is.
__device__ __forceinline__ void store_chunk(uint8_t *kv, int r, int c, const uint4 raw, const uint2 sc) {
    const int sw = r & 7;
    if (c < kNopeChunks) {
        uint4 lo, hi;
        dequant16(raw, scale_byte(sc, c >> 2), lo, hi);
        uint8_t *row = kv + (c >> 2) * (kTile * 128) + r * 128;
        const int oc = (c & 3) * 2;
        *reinterpret_cast<uint4 *>(row + ((oc ^ sw) << 4)) = lo;
        *reinterpret_cast<uint4 *>(row + (((oc + 1) ^ sw) << 4)) = hi;
    } else {
        uint8_t *row = kv + 7 * (kTile * 128) + r * 128;
        *reinterpret_cast<uint4 *>(row + (((c - kNopeChunks) ^ sw) << 4)) = raw;
    }
}

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int split = blockIdx.x;
    const int b = blockIdx.y;

    if (smem_addr(smem) & 1023u) {
        if (tid == 0) atomicOr(p.err, SMLA_FLAG_SMEM);
        return;
    }
    uint8_t *sQ = smem + kSmemQ;
    uint8_t *sKV = smem + kSmemKV;
    uint8_t *sPhi = smem + kSmemPhi;
    uint8_t *sPlo = smem + kSmemPlo;
    int *codes = reinterpret_cast<int *>(smem + kSmemCodes);
    uint2 *scales = reinterpret_cast<uint2 *>(smem + kSmemScales);
    float *red = reinterpret_cast<float *>(smem + kSmemScales);
    float *head_m = reinterpret_cast<float *>(smem + kSmemHeadM);
    float *head_l = reinterpret_cast<float *>(smem + kSmemHeadL);
    float *head_alpha = reinterpret_cast<float *>(smem + kSmemHeadAlpha);
    float *head_mnew = reinterpret_cast<float *>(smem + kSmemHeadMnew);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kSmemBar);
    uint64_t *bar_spare = reinterpret_cast<uint64_t *>(smem + kSmemBarSpare);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmemTmemSlot);

    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar_spare, 1);
        fence_barrier_init();
    }
    if (tid < kHeads) {
        head_m[tid] = -INFINITY;
        head_l[tid] = 0.0f;
    }
    // Q[b] -> shared memory, K-major 128-byte swizzle: K-block kb = dims [64kb, 64kb+64).
    {
        const uint4 *qg = reinterpret_cast<const uint4 *>(p.q + static_cast<size_t>(b) * kHeads * kDim);
#pragma unroll 4
        for (int c = tid; c < kHeads * kDim / 8; c += kThreads) {
            const int head = c >> 6, kc = c & 63;
            const uint4 v = ld_stream_v4(qg + c);
            *reinterpret_cast<uint4 *>(sQ + (kc >> 3) * 8192 + head * 128 + (((kc & 7) ^ (head & 7)) << 4)) = v;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sQ_a = smem_addr(sQ), sKV_a = smem_addr(sKV), sPhi_a = smem_addr(sPhi), sPlo_a = smem_addr(sPlo);

    const int num_tiles = (p.topk + kTile - 1) / kTile;
    const int t_begin = split * p.tiles_per_split;
    const int t_end = min(num_tiles, t_begin + p.tiles_per_split);
    const int seq_len = __ldg(p.seq_lens + b);
    const int32_t *bt_row = p.block_table + static_cast<size_t>(b) * p.max_blocks;
    const int32_t *idx_row = p.topk_idx + static_cast<size_t>(b) * p.topk;
    const uint32_t lane_base = static_cast<uint32_t>(warp & 3) * 32u << 16;

    uint32_t phase = 0;
    bool have_o = false, failed = false, first = true, spare_armed = false;

    for (int t = t_begin; t < t_end; ++t) {
        // ---- translate 128 slots, fetch their scale rows
        int code = -1;
        if (tid < kTile) {
            const int i = t * kTile + tid;
            if (i < p.topk) code = translate_slot(bt_row, p.max_blocks, seq_len, p.num_pages, __ldg(idx_row + i), p.err);
            codes[tid] = code;
            scales[tid] = (code >= 0) ? ld_stream_v2(token_scales(p.cache, code)) : make_uint2(0u, 0u);
        }
        if (__syncthreads_count(code >= 0) == 0) continue;  // whole tile masked: nothing to add

        // ---- gather + dequantise 128 x 36 chunks into the bf16 tile
#pragma unroll
        for (int it = 0; it < kTile * kRowChunks / kThreads; it += 6) {
            uint4 raw[6];
            int rr[6], cc[6];
#pragma unroll
            for (int u = 0; u < 6; ++u) {
                const int i = tid + (it + u) * kThreads;
                rr[u] = i / kRowChunks;
                cc[u] = i - rr[u] * kRowChunks;
                const int cd = codes[rr[u]];
                raw[u] = (cd >= 0) ? ld_stream_v4(token_row(p.cache, cd) + cc[u] * 16) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 6; ++u) store_chunk(sKV, rr[u], cc[u], raw[u], scales[rr[u]]);
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- S^T = K_tile . Q^T  (M=128 tokens, N=64 heads, K=512)
        const bool skip_commit = first && (p.debug_flags & SMLA_DEBUG_SKIP_FIRST_COMMIT);
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int kb = 0; kb < 8; ++kb) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = sw128_desc(sKV_a + kb * (kTile * 128) + kk * 32, 16, 1024);
                    const uint64_t bq = sw128_desc(sQ_a + kb * 8192 + kk * 32, 16, 1024);
                    mma_bf16_ss(tmem + kTmemS, a, bq, kIdescQK, (kb | kk) != 0);
                }
            }
            mma_commit(skip_commit ? bar_spare : bar);
        }
        if (skip_commit) spare_armed = true;
        first = false;
        bool ok = mbar_wait(bar, phase, p.timeout_ns);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        phase ^= 1u;
        tc_fence_after_sync();

        // ---- online softmax (warps 0-3: thread = token lane of S^T)
        if (warp < 4) {
            const int r = tid;
            const bool valid = codes[r] >= 0;
            float v[64];
            tmem_ld64(tmem + lane_base + kTmemS, v);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 64; ++h) v[h] = valid ? v[h] * p.scale_log2 : -INFINITY;
            warp_transpose_reduce64(v, lane, MaxOp());
            red[warp * 64 + 2 * lane] = v[0];
            red[warp * 64 + 2 * lane + 1] = v[1];
            named_barrier_sync(1, 128);
            if (r < kHeads) {
                const float tm = fmaxf(fmaxf(red[r], red[64 + r]), fmaxf(red[128 + r], red[192 + r]));
                const float mo = head_m[r];
                const float mn = fmaxf(mo, tm);
                head_alpha[r] = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
                head_mnew[r] = mn;
            }
            named_barrier_sync(1, 128);
            tmem_ld64(tmem + lane_base + kTmemS, v);
            tmem_wait_ld();
#pragma unroll
            for (int h4 = 0; h4 < 16; ++h4) {
                const float4 mn = reinterpret_cast<const float4 *>(head_mnew)[h4];
                const float m4[4] = {mn.x, mn.y, mn.z, mn.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int h = 4 * h4 + j;
                    v[h] = (valid && m4[j] != -INFINITY) ? exp2f(v[h] * p.scale_log2 - m4[j]) : 0.0f;
                }
            }
            // P^T rows (token r, 64 heads) as bf16 hi and lo terms, MN-major swizzled.
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float a0 = v[8 * c + 2 * j], a1 = v[8 * c + 2 * j + 1];
                    const __nv_bfloat162 hb = __floats2bfloat162_rn(a0, a1);
                    const float2 hf = __bfloat1622float2(hb);
                    const __nv_bfloat162 lb = __floats2bfloat162_rn(a0 - hf.x, a1 - hf.y);
                    hw[j] = *reinterpret_cast<const uint32_t *>(&hb);
                    lw[j] = *reinterpret_cast<const uint32_t *>(&lb);
                }
                const int off = r * 128 + ((c ^ (r & 7)) << 4);
                *reinterpret_cast<uint4 *>(sPhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(sPlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            warp_transpose_reduce64(v, lane, AddOp());
            red[warp * 64 + 2 * lane] = v[0];
            red[warp * 64 + 2 * lane + 1] = v[1];
            named_barrier_sync(1, 128);
            if (r < kHeads) {
                const float s = (red[r] + red[64 + r]) + (red[128 + r] + red[192 + r]);
                head_l[r] = head_l[r] * head_alpha[r] + s;
                head_m[r] = head_mnew[r];
            }
            if (have_o) {
                float alpha[64];
                bool any = false;
#pragma unroll
                for (int h4 = 0; h4 < 16; ++h4) {
                    const float4 a4 = reinterpret_cast<const float4 *>(head_alpha)[h4];
                    alpha[4 * h4] = a4.x;
                    alpha[4 * h4 + 1] = a4.y;
                    alpha[4 * h4 + 2] = a4.z;
                    alpha[4 * h4 + 3] = a4.w;
                    any |= (a4.x != 1.0f) | (a4.y != 1.0f) | (a4.z != 1.0f) | (a4.w != 1.0f);
                }
                if (any) {
#pragma unroll 1
                    for (int mc = 0; mc < 4; ++mc) {
                        float o[64];
                        tmem_ld64(tmem + lane_base + 64 * mc, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < 64; ++h) o[h] *= alpha[h];
                        tmem_st64(tmem + lane_base + 64 * mc, o);
                    }
                    tmem_wait_st();
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
        }
        __syncthreads();

        // ---- O^T += V^T . P^T  (4 x M=128 dims, N=64 heads, K=128 tokens; P = hi + lo)
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int mc = 0; mc < 4; ++mc) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t a = sw128_desc(sKV_a + 2 * mc * (kTile * 128) + ks * 2048, kTile * 128, 1024);
                    const uint64_t bh = sw128_desc(sPhi_a + ks * 2048, 8192, 1024);
                    const uint64_t bl = sw128_desc(sPlo_a + ks * 2048, 8192, 1024);
                    mma_bf16_ss(tmem + 64 * mc, a, bh, kIdescPV, (have_o || ks > 0) ? 1u : 0u);
                    mma_bf16_ss(tmem + 64 * mc, a, bl, kIdescPV, 1u);
                }
            }
            mma_commit(bar);
        }
        ok = mbar_wait(bar, phase, p.timeout_ns);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        phase ^= 1u;
        tc_fence_after_sync();
        have_o = true;
    }

    if (failed) {
        if (tid == 0) {
            atomicOr(p.err, SMLA_FLAG_TIMEOUT);
            // MMAs committed to the spare barrier must finish before tensor memory is released.
            if (spare_armed) (void)mbar_wait(bar_spare, 0, p.timeout_ns);
        }
    } else if (warp < 4) {
        // ---- epilogue: O^T lane = output dim within a 128-row block, column = head
        float inv_l[64];
#pragma unroll
        for (int h = 0; h < 64; ++h) {
            const float l = head_l[h];
            inv_l[h] = (have_o && l > 0.0f) ? 1.0f / l : 0.0f;
        }
#pragma unroll 1
        for (int mc = 0; mc < 4; ++mc) {
            float o[64];
            tmem_ld64(tmem + lane_base + 64 * mc, o);
            tmem_wait_ld();
            const int d = 128 * mc + 32 * warp + lane;
            if (p.nsplit == 1) {
                float *dst = p.out + static_cast<size_t>(b) * kHeads * kDim + d;
#pragma unroll
                for (int h = 0; h < 64; ++h) dst[h * kDim] = o[h] * inv_l[h];
            } else {
                float *dst = p.part_o + (static_cast<size_t>(b) * kHeads * p.nsplit + split) * kDim + d;
#pragma unroll
                for (int h = 0; h < 64; ++h) dst[static_cast<size_t>(h) * p.nsplit * kDim] = o[h] * inv_l[h];
            }
        }
        if (tid < kHeads) {
            const float l = head_l[tid];
            const float val = (have_o && l > 0.0f) ? (head_m[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
            if (p.nsplit == 1)
                p.lse[static_cast<size_t>(b) * kHeads + tid] = val;
            else
                p.part_lse[(static_cast<size_t>(b) * kHeads + tid) * p.nsplit + split] = val;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Split-K merge: one CTA of 128 threads per (b, h), 4 output dims per thread.
__global__ void __launch_bounds__(128) combine_kernel(const float *__restrict__ part_o,
                                                      const float *__restrict__ part_lse, float *__restrict__ out,
                                                      float *__restrict__ lse, int nsplit) {
    const size_t bh = blockIdx.x;
    const int tid = threadIdx.x;
    const float *L = part_lse + bh * nsplit;
    float lmax = -INFINITY;
    for (int s = 0; s < nsplit; ++s) lmax = fmaxf(lmax, __ldg(L + s));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lmax == -INFINITY) {
        reinterpret_cast<float4 *>(out + bh * kDim)[tid] = acc;
        if (tid == 0) lse[bh] = -INFINITY;
        return;
    }
    float wsum = 0.0f;
    for (int s = 0; s < nsplit; ++s) {
        const float ls = __ldg(L + s);
        if (ls == -INFINITY) continue;
        const float w = expf(ls - lmax);
        wsum += w;
        const float4 o = __ldg(reinterpret_cast<const float4 *>(part_o + (bh * nsplit + s) * kDim) + tid);
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
    }
    const float inv = 1.0f / wsum;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    reinterpret_cast<float4 *>(out + bh * kDim)[tid] = acc;
    if (tid == 0) lse[bh] = lmax + logf(wsum);
}

// Gather debug kernel: the translation and dequantisation of decode_kernel,
// written out as fp32 latents and (page, slot) pairs.  Grid (tiles, B).
__global__ void __launch_bounds__(kThreads) gather_kernel(const uint8_t *cache, const int32_t *block_table,
                                                          const int32_t *topk_idx, const int32_t *seq_lens,
                                                          long long num_pages, int topk, int max_blocks,
                                                          float *latents, int32_t *page_slot, uint32_t *err) {
    __shared__ int codes[kTile];
    __shared__ uint2 scales[kTile];
    __shared__ __align__(16) uint8_t tile_row[kThreads][32];
    const int tid = threadIdx.x, t = blockIdx.x, b = blockIdx.y;
    if (tid < kTile) {
        const int i = t * kTile + tid;
        int code = -1;
        if (i < topk)
            code = translate_slot(block_table + static_cast<size_t>(b) * max_blocks, max_blocks, __ldg(seq_lens + b),
                                  num_pages, __ldg(topk_idx + static_cast<size_t>(b) * topk + i), err);
        codes[tid] = code;
        scales[tid] = (code >= 0) ? ld_stream_v2(token_scales(cache, code)) : make_uint2(0u, 0u);
        if (i < topk) {
            page_slot[(static_cast<size_t>(b) * topk + i) * 2] = code >= 0 ? (code >> 8) : -1;
            page_slot[(static_cast<size_t>(b) * topk + i) * 2 + 1] = code >= 0 ? (code & 255) : -1;
        }
    }
    __syncthreads();
    for (int i = tid; i < kTile * kRowChunks; i += kThreads) {
        const int r = i / kRowChunks, c = i - r * kRowChunks;
        const int slot = t * kTile + r;
        if (slot >= topk) continue;
        const int cd = codes[r];
        const uint4 raw = (cd >= 0) ? ld_stream_v4(token_row(cache, cd) + c * 16) : make_uint4(0u, 0u, 0u, 0u);
        float *dst = latents + (static_cast<size_t>(b) * topk + slot) * kDim;
        const uint16_t *h;
        int n, d0;
        uint4 lo, hi;
        if (c < kNopeChunks) {
            dequant16(raw, scale_byte(scales[r], c >> 2), lo, hi);
            *reinterpret_cast<uint4 *>(&tile_row[tid][0]) = lo;
            *reinterpret_cast<uint4 *>(&tile_row[tid][16]) = hi;
            n = 16;
            d0 = 16 * c;
        } else {
            *reinterpret_cast<uint4 *>(&tile_row[tid][0]) = raw;
            n = 8;
            d0 = kNope + 8 * (c - kNopeChunks);
        }
        h = reinterpret_cast<const uint16_t *>(&tile_row[tid][0]);
        for (int j = 0; j < n; ++j) dst[d0 + j] = __uint_as_float(static_cast<uint32_t>(h[j]) << 16);
    }
}

}  // namespace smla

// ======================================================================== host
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    bool supported = false;
    int sms = 0;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

int device_info(DeviceInfo *&info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SMLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &d = g_devices[dev];
    if (!d.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return SMLA_ERR_CUDA;
        d.supported = (major == 10 && minor == 0);
        d.sms = sms;
        if (d.supported &&
            cudaFuncSetAttribute(smla::decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smla::kSmemBytes) != cudaSuccess)
            return SMLA_ERR_CUDA;
        d.ready = true;
    }
    info = &d;
    return d.supported ? SMLA_OK : SMLA_ERR_DEVICE;
}

int num_tiles(int topk) { return (topk + smla::kTile - 1) / smla::kTile; }

// Effective split count: every split gets ceil(tiles / nsplit) tiles, none is empty.
int effective_splits(int topk, int nsplit) {
    const int tiles = num_tiles(topk);
    if (nsplit < 1) nsplit = 1;
    if (nsplit > tiles) nsplit = tiles;
    const int per = (tiles + nsplit - 1) / nsplit;
    return (tiles + per - 1) / per;
}

int heuristic_splits(int B, int topk, int sms) {
    int ns = (B > 0 && sms > B) ? sms / B : 1;
    return effective_splits(topk, ns);
}

bool sizes_ok(int B, int H, int topk) {
    return B >= 1 && B <= 65535 && H == SMLA_HEADS && topk >= 1 && topk <= SMLA_MAX_TOPK;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t workspace_for(int B, int topk, int nsplit) {
    size_t bytes = SMLA_WORKSPACE_HEADER;
    if (nsplit > 1) {
        const size_t rows = static_cast<size_t>(B) * SMLA_HEADS * nsplit;
        bytes += round256(rows * sizeof(float)) + rows * SMLA_DIM * sizeof(float);
    }
    (void)topk;
    return bytes;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" {

const char *smla_version(void) { return "smla 0.1 (sm_100a tcgen05 sparse MLA decode)"; }

int smla_num_splits(int B, int H, int topk) {
    if (!sizes_ok(B, H, topk)) return SMLA_ERR_INVALID;
    DeviceInfo *info = nullptr;
    const int rc = device_info(info);
    if (rc != SMLA_OK) return rc;
    return heuristic_splits(B, topk, info->sms);
}

size_t smla_workspace_bytes_ex(int B, int H, int topk, int nsplit) {
    if (!sizes_ok(B, H, topk) || nsplit < 1 || nsplit > num_tiles(topk)) return 0;
    return workspace_for(B, topk, effective_splits(topk, nsplit));
}

size_t smla_workspace_bytes(int B, int H, int topk) {
    const int ns = smla_num_splits(B, H, topk);
    if (ns < 1) return 0;
    return workspace_for(B, topk, ns);
}

int smla_combine(const float *part_o, const float *part_lse, int nsplit, float *out, float *lse, int B, int H,
                 void *stream) {
    if (!part_o || !part_lse || !out || !lse || nsplit < 1 || nsplit > 1024 || B < 1 || H < 1) return SMLA_ERR_INVALID;
    if (!aligned(part_o, 16) || !aligned(out, 16)) return SMLA_ERR_INVALID;
    DeviceInfo *info = nullptr;
    const int rc = device_info(info);
    if (rc != SMLA_OK) return rc;
    (void)cudaGetLastError();
    smla::combine_kernel<<<static_cast<unsigned>(B) * static_cast<unsigned>(H), 128, 0,
                           static_cast<cudaStream_t>(stream)>>>(part_o, part_lse, out, lse, nsplit);
    return cudaGetLastError() == cudaSuccess ? SMLA_OK : SMLA_ERR_LAUNCH;
}

int smla_decode_ex(const void *q, const uint8_t *kv_cache, const int32_t *block_table, const int32_t *topk_idx,
                   const int32_t *seq_lens, float sm_scale, float *out, float *lse, int B, int H, int topk,
                   int max_blocks, int num_pages, void *workspace, size_t workspace_bytes,
                   const smla_options *opts, void *stream) {
    if (!q || !kv_cache || !block_table || !topk_idx || !seq_lens || !out || !lse || !workspace)
        return SMLA_ERR_INVALID;
    if (!sizes_ok(B, H, topk) || max_blocks < 1 || num_pages < 1 || num_pages >= (1 << 23)) return SMLA_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(kv_cache, 16) || !aligned(out, 16) || !aligned(workspace, 256) ||
        !aligned(block_table, 4) || !aligned(topk_idx, 4) || !aligned(seq_lens, 4) || !aligned(lse, 4))
        return SMLA_ERR_INVALID;
    if (!std::isfinite(sm_scale)) return SMLA_ERR_INVALID;
    DeviceInfo *info = nullptr;
    int rc = device_info(info);
    if (rc != SMLA_OK) return rc;
    int nsplit = (opts && opts->nsplit > 0) ? effective_splits(topk, opts->nsplit) : heuristic_splits(B, topk, info->sms);
    if (workspace_bytes < workspace_for(B, topk, nsplit)) return SMLA_ERR_INVALID;
    const int tiles = num_tiles(topk);
    const int per = (tiles + nsplit - 1) / nsplit;

    smla::DecodeParams p{};
    p.q = static_cast<const uint16_t *>(q);
    p.cache = kv_cache;
    p.block_table = block_table;
    p.topk_idx = topk_idx;
    p.seq_lens = seq_lens;
    p.out = out;
    p.lse = lse;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    p.err = reinterpret_cast<uint32_t *>(ws);
    const size_t rows = static_cast<size_t>(B) * SMLA_HEADS * nsplit;
    p.part_lse = reinterpret_cast<float *>(ws + SMLA_WORKSPACE_HEADER);
    p.part_o = reinterpret_cast<float *>(ws + SMLA_WORKSPACE_HEADER + round256(rows * sizeof(float)));
    p.num_pages = num_pages;
    p.timeout_ns = (opts && opts->wait_timeout_ns) ? opts->wait_timeout_ns : 1000000000ull;
    p.topk = topk;
    p.max_blocks = max_blocks;
    p.nsplit = nsplit;
    p.tiles_per_split = per;
    p.scale_log2 = sm_scale * 1.4426950408889634f;
    p.debug_flags = opts ? opts->debug_flags : 0u;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    (void)cudaGetLastError();
    smla::decode_kernel<<<dim3(nsplit, B), smla::kThreads, smla::kSmemBytes, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SMLA_ERR_LAUNCH;
    if (nsplit > 1) {
        smla::combine_kernel<<<static_cast<unsigned>(B) * SMLA_HEADS, 128, 0, st>>>(p.part_o, p.part_lse, out, lse,
                                                                                   nsplit);
        if (cudaGetLastError() != cudaSuccess) return SMLA_ERR_LAUNCH;
    }
    return SMLA_OK;
}

int smla_decode(const void *q, const uint8_t *kv_cache, const int32_t *block_table, const int32_t *topk_idx,
                const int32_t *seq_lens, float sm_scale, float *out, float *lse, int B, int H, int topk,
                int max_blocks, int num_pages, void *workspace, size_t workspace_bytes, void *stream) {
    return smla_decode_ex(q, kv_cache, block_table, topk_idx, seq_lens, sm_scale, out, lse, B, H, topk, max_blocks,
                          num_pages, workspace, workspace_bytes, nullptr, stream);
}

int smla_read_error(void *workspace, void *stream, uint32_t *flags) {
    if (!workspace || !flags) return SMLA_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SMLA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(v), st) != cudaSuccess) return SMLA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SMLA_ERR_CUDA;
    *flags = v;
    return SMLA_OK;
}

int smla_debug_gather(const uint8_t *kv_cache, const int32_t *block_table, const int32_t *topk_idx,
                      const int32_t *seq_lens, int B, int topk, int max_blocks, int num_pages, float *latents,
                      int32_t *page_slot, void *workspace, size_t workspace_bytes, void *stream) {
    if (!kv_cache || !block_table || !topk_idx || !seq_lens || !latents || !page_slot || !workspace)
        return SMLA_ERR_INVALID;
    if (B < 1 || B > 65535 || topk < 1 || topk > SMLA_MAX_TOPK || max_blocks < 1 || num_pages < 1 ||
        num_pages >= (1 << 23) || workspace_bytes < SMLA_WORKSPACE_HEADER)
        return SMLA_ERR_INVALID;
    if (!aligned(kv_cache, 16) || !aligned(workspace, 256)) return SMLA_ERR_INVALID;
    DeviceInfo *info = nullptr;
    const int rc = device_info(info);
    if (rc != SMLA_OK) return rc;
    (void)cudaGetLastError();
    smla::gather_kernel<<<dim3(num_tiles(topk), B), smla::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        kv_cache, block_table, topk_idx, seq_lens, num_pages, topk, max_blocks, latents, page_slot,
        static_cast<uint32_t *>(workspace));
    return cudaGetLastError() == cudaSuccess ? SMLA_OK : SMLA_ERR_LAUNCH;
}

}  // extern "C"

// ======================================================================== no-allocation entry point
// Some callers cannot hand the library a workspace: a serving engine that has
// frozen its device memory pool after capturing its decode step into CUDA
// graphs, or a plugin host that owns every device allocation and forbids its
// plugins to call the allocator.  smla_decode_noalloc serves them from a
// fixed scratch array that is part of this library's device image.
namespace {

constexpr size_t kStaticScratchBytes = SMLA_STATIC_SCRATCH_BYTES;
void *g_static_scratch[kMaxDevices] = {};

}  // namespace

// Split-K partials and the error word of smla_decode_noalloc.  Every device that
// loads this library holds these bytes until the process exits.  In host code
// this name is only a stand-in: the device address comes from
// cudaGetSymbolAddress, taken once per device below.
static __device__ __align__(256) uint8_t g_smla_static_scratch[kStaticScratchBytes];

extern "C" int smla_decode_noalloc(const void *q, const uint8_t *kv_cache, const int32_t *block_table,
                                   const int32_t *topk_idx, const int32_t *seq_lens, float sm_scale, float *out,
                                   float *lse, int B, int H, int topk, int max_blocks, int num_pages, void *stream) {
    if (!sizes_ok(B, H, topk)) return SMLA_ERR_INVALID;
    DeviceInfo *info = nullptr;
    const int rc = device_info(info);
    if (rc != SMLA_OK) return rc;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SMLA_ERR_CUDA;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_static_scratch[dev] == nullptr) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_smla_static_scratch) != cudaSuccess || p == nullptr) return SMLA_ERR_CUDA;
            g_static_scratch[dev] = p;
        }
        scratch = g_static_scratch[dev];
    }
    if (workspace_for(B, topk, heuristic_splits(B, topk, info->sms)) > kStaticScratchBytes) return SMLA_ERR_SCRATCH;
    return smla_decode_ex(q, kv_cache, block_table, topk_idx, seq_lens, sm_scale, out, lse, B, H, topk, max_blocks,
                          num_pages, scratch, kStaticScratchBytes, nullptr, stream);
}

