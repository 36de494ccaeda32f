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
// B200 mapping, per CTA (one per SM, 512 threads):
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
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/smla.h"
#include "sm100_ptx.cuh"
#include "smla_device.cuh"

namespace smla {

constexpr int kTile = 128;           // topk slots per MMA tile (the M of S^T)
constexpr int kThreads = 512;        // 16 warps, one CTA per SM; every warp takes part in every phase
constexpr int kGatherThreads = 256;  // threads of the gather debug kernel

// Dynamic shared memory map (bytes from a 1024-aligned base).
constexpr int kSmemQ = 0;                          // 64 KB: 8 K-blocks x [64 heads x 128 B], TMA-written
constexpr int kSmemKV = kSmemQ + 65536;            // 128 KB: 8 K-blocks x [128 tokens x 128 B]
constexpr int kSmemPhi = kSmemKV + 131072;         // 16 KB: P_hi^T [128 tokens x 64 heads] bf16
constexpr int kSmemPlo = kSmemPhi + 16384;         // 16 KB: P_lo^T
constexpr int kSmemCodes = kSmemPlo + 16384;       // [2][128] int32 token codes (double-buffered)
constexpr int kSmemHeadM = kSmemCodes + 1024;      // [64] running max per head (log2 units)
constexpr int kSmemHeadAlpha = kSmemHeadM + 256;   // [64] rescale factor of the last max update
constexpr int kSmemRed = kSmemHeadAlpha + 256;     // [4][64] f32 cross-quadrant reduction scratch
constexpr int kSmemBars = kSmemRed + 1024;         // mbarriers (8 B each)
constexpr int kNumBars = 8;
constexpr int kSmemTmemSlot = kSmemBars + kNumBars * 8;
constexpr int kSmemAbort = kSmemTmemSlot + 4;
constexpr int kSmemBytes = kSmemAbort + 12;
constexpr int kSmemMl = kSmemCodes - 2048;         // cluster merge: [4][m(64) | l(64)] f32, inside P_lo (dead by then)
static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-block shared memory limit");

enum Bar : int {
    kBarQ = 0,       // Q landed (TMA transaction bytes)
    kBarKvFull = 1,  // bf16 tile written (16 warp arrivals after a proxy fence)
    kBarSFull = 2,   // S^T complete (MMA commit)
    kBarPFull = 3,   // P^T written (16 warp arrivals after a proxy fence)
    kBarPvDone = 4,  // PV complete (MMA commit): tile buffers and O^T free
    kBarDrain = 5,   // final commit before tensor memory is released
    kBarSpare = 6,   // test hook target
    kBarRecv = 7,    // cluster merge: partials received from the other CTAs (bulk-copy bytes)
};

constexpr uint32_t kTmemCols = 512;  // O^T [0,256), S^T [256,320), per-lane running sums [320,384)
constexpr uint32_t kTmemS = 256;
constexpr uint32_t kTmemL = 320;
constexpr uint32_t kIdescQK = idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16(128, 64, true, true);
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p = 2^(s - m) stays below 256 without a rescale

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
    int cluster_merge;  // 1: the nsplit CTAs of a request form a cluster and merge through DSMEM
};

// Reduces 16 per-thread values across the 32 lanes of a warp, value i with value i
// of every other lane.  Afterwards lanes 2j and 2j+1 both hold the result for entry
// j.  Each round halves the live entries: a lane keeps the half selected by its
// lane bit and sends the other half to its partner; the last round combines pairs.
template <bool kMax>
__device__ __forceinline__ float warp_transpose_reduce16(float (&v)[16], int lane) {
#pragma unroll
    for (int w = 8, off = 16; off >= 2; w >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float send = upper ? v[i] : v[i + w];
            const float keep = upper ? v[i + w] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, off);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    const float got = __shfl_xor_sync(0xffffffffu, v[0], 1);
    return kMax ? fmaxf(v[0], got) : v[0] + got;
}

// Bounded wait on an mbarrier phase.  Gives up when another thread has aborted the
// CTA or when `timeout_ns` passes (then it aborts the CTA and flags the error).
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                           const DecodeParams &p) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 50000u)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > p.timeout_ns) {
            *abort_flag = 1;
            atomicOr(p.err, SMLA_FLAG_TIMEOUT);
            return false;
        }
    }
}

// Warp-uniform version: lane 0 waits, the verdict is broadcast, and every lane then
// observes the completed phase itself (acquire) before touching the guarded data.
__device__ __forceinline__ bool warp_wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                const DecodeParams &p, int lane) {
    int ok = 1;
    if (lane == 0) ok = wait_phase(bar, parity, abort_flag, p) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) (void)mbar_try_wait(bar, parity);
    return ok != 0;
}

// ------------------------------------------------------------------ gather + dequant
// The 128 x 36 sixteen-byte chunks of a tile are dealt out in four groups, one per
// K-block pair c (dims [128c, 128c+128)):
//   pairs 0..2: 128 tokens x 8 nope chunks (16 dims)          -> 2 items per thread
//   pair 3:     128 tokens x (4 nope + 8 rope chunks)          -> 3 items per thread
// Consecutive threads take consecutive chunks of a token row (coalesced loads).
template <int C>
struct PairShape {
    static constexpr int kItems = (C < 3) ? 2 : 3;
};

template <int C>
__device__ __forceinline__ void pair_item(int t, int u, int &r, int &chunk, int &kb, int &oc, bool &nope) {
    const int j = t + kThreads * u;
    if constexpr (C < 3) {
        r = j >> 3;
        const int k = j & 7;
        chunk = 8 * C + k;
        kb = 2 * C + (k >> 2);
        oc = 2 * (k & 3);
        nope = true;
    } else {
        r = j / 12;
        const int k = j - 12 * r;
        if (k < 4) {
            chunk = 24 + k;
            kb = 6;
            oc = 2 * k;
            nope = true;
        } else {
            chunk = 28 + (k - 4);
            kb = 7;
            oc = k - 4;
            nope = false;
        }
    }
}

// The FP8 bytes (and the scale byte) of one tile, held in registers between the
// load and the dequantisation.
struct TileRegs {
    uint4 raw0[2], raw1[2], raw2[2], raw3[3];
    uint32_t sc0[2], sc1[2], sc2[2], sc3[3];
};

template <int C>
__device__ __forceinline__ void load_pair(int t, const int *codes, const uint8_t *cache,
                                          uint4 (&raw)[PairShape<C>::kItems], uint32_t (&sc)[PairShape<C>::kItems]) {
#pragma unroll
    for (int u = 0; u < PairShape<C>::kItems; ++u) {
        int r, chunk, kb, oc;
        bool nope;
        pair_item<C>(t, u, r, chunk, kb, oc, nope);
        const int code = codes[r];
        raw[u] = make_uint4(0u, 0u, 0u, 0u);
        sc[u] = 0u;
        if (code >= 0) {
            raw[u] = ld_stream_v4(token_row(cache, code) + chunk * 16);
            if (nope) sc[u] = ld_stream_u8(token_scales(cache, code) + (chunk >> 2));
        }
    }
}

__device__ __forceinline__ void load_tile(int t, const int *codes, const uint8_t *cache, TileRegs &tr) {
    load_pair<0>(t, codes, cache, tr.raw0, tr.sc0);
    load_pair<1>(t, codes, cache, tr.raw1, tr.sc1);
    load_pair<2>(t, codes, cache, tr.raw2, tr.sc2);
    load_pair<3>(t, codes, cache, tr.raw3, tr.sc3);
}

// Dequantises this thread's items of pair C into the swizzled bf16 tile (plain shared
// stores; `kv` is the tile's shared-window address).
template <int C>
__device__ __forceinline__ void store_pair(int t, uint32_t kv, const uint4 (&raw)[PairShape<C>::kItems],
                                           const uint32_t (&sc)[PairShape<C>::kItems]) {
#pragma unroll
    for (int u = 0; u < PairShape<C>::kItems; ++u) {
        int r, chunk, kb, oc;
        bool nope;
        pair_item<C>(t, u, r, chunk, kb, oc, nope);
        const uint32_t row = kv + kb * (kTile * 128) + r * 128;
        const int sw = r & 7;
        if (nope) {
            uint4 lo, hi;
            dequant16(raw[u], sc[u], lo, hi);
            // odd K-blocks store their high half first so the 8 lanes of a store phase hit 8 bank groups
            if ((kb & 1) == 0) {
                sts_v4(row + ((oc ^ sw) << 4), lo);
                sts_v4(row + (((oc + 1) ^ sw) << 4), hi);
            } else {
                sts_v4(row + (((oc + 1) ^ sw) << 4), hi);
                sts_v4(row + ((oc ^ sw) << 4), lo);
            }
        } else {
            sts_v4(row + ((oc ^ sw) << 4), raw[u]);
        }
    }
}

// ------------------------------------------------------------------ split merge in a cluster
// The nsplit CTAs of one request form a thread-block cluster.  After the last PV,
// CTA s holds un-normalised O^T_s (tensor memory), its per-head running max m_s (log2
// units) and sum l_s.  With L = log2 sum_s 2^(m_s) l_s, the merged output is
// O = sum_s 2^(m_s - L) O^T_s and LSE = L ln 2 (the split-K log-sum-exp merge).
// Output dims are dealt out by 128-dim chunk: chunk mc belongs to CTA mc % nsplit.
// Once every CTA's MMAs are done (its Q, KV and P buffers are dead), each CTA stages
// its (m_s, l_s) row and the O^T_s chunks it does not own in its own shared memory
// and sends them with bulk shared-to-shared copies into the owners' receive areas,
// where they are counted in bytes on kBarRecv.  Receive area of a CTA: blocks
// [owned chunk lci][sender slot] from offset 0, the (m, l) rows at kSmemMl; its send
// staging follows its receive blocks.
constexpr int kRecvRow = 272;               // 64 heads x fp32 + 16 B pad: conflict-free row stores
constexpr int kRecvBlock = 128 * kRecvRow;  // one 128-dim chunk of O^T
constexpr int kMlRow = 512;                 // m[64] | l[64], f32

__host__ __device__ constexpr int owned_chunks(int me, int ns) { return (4 - me + ns - 1) / ns; }
static_assert(4 * kRecvBlock + 2 * kRecvBlock <= kSmemMl, "receive + send areas overlap the (m, l) rows");
static_assert(3 * kRecvBlock + 3 * kRecvBlock <= kSmemMl, "receive + send areas overlap the (m, l) rows");

__device__ __noinline__ void cluster_epilogue(const DecodeParams &p, int b, bool ok, int n, int tid, int q, int g,
                                              int lane, uint32_t tmem, uint32_t lane_base, uint8_t *smem,
                                              uint64_t *bar_recv, const float *head_m, const float *l_head,
                                              float *weights) {
    const int ns = p.nsplit;
    const int me = static_cast<int>(cluster_ctarank());
    const int n_own = owned_chunks(me, ns);
    const uint32_t base = smem_addr(smem);
    const uint32_t send = base + n_own * (ns - 1) * kRecvBlock;
    float *ml = reinterpret_cast<float *>(smem + kSmemMl);  // [s][m(64) | l(64)]
    const int d = 32 * q + lane;                            // row of O^T within a chunk
    const bool live = ok && n > 0;

    // barrier 1: every CTA's MMAs are done, so its operand buffers may be overwritten
    cluster_sync();
    if (tid < kHeads) {
        ml[me * 128 + tid] = live ? head_m[tid] : -INFINITY;
        ml[me * 128 + 64 + tid] = live ? l_head[tid] : 0.0f;
    }
    {
        int js = 0;
#pragma unroll 1
        for (int mc = 0; mc < 4; ++mc) {
            if (mc % ns == me) continue;
            float o[16];
            if (live) {
                tmem_ld16(tmem + lane_base + 64 * mc + 16 * g, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int h = 0; h < 16; ++h) o[h] = 0.0f;
            }
            const uint32_t row = send + js * kRecvBlock + d * kRecvRow + 64 * g;
#pragma unroll
            for (int j = 0; j < 4; ++j) sts_v4f(row + 16 * j, o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
            ++js;
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid < ns && tid != me) {
        const int peer = tid;
        const uint32_t bar_c = map_to_rank(bar_recv, peer);
        bulk_copy_to_cluster(map_to_rank(ml + me * 128, peer), smem_addr(ml + me * 128), kMlRow, bar_c);
        int js = 0;
        for (int mc = 0; mc < 4; ++mc) {
            const int owner = mc % ns;
            if (owner == me) continue;
            if (owner == peer) {
                const int slot = (me < peer) ? me : me - 1;
                const int blk = (mc / ns) * (ns - 1) + slot;
                bulk_copy_to_cluster(map_to_rank(smem + blk * kRecvBlock, peer), send + js * kRecvBlock, kRecvBlock,
                                     bar_c);
            }
            ++js;
        }
    }
    // the other CTAs' rows and chunks have landed (bounded wait; the copies are in flight
    // whatever happened elsewhere, so the abort flag does not cut it short)
    int got = 1;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_recv, (ns - 1) * (kMlRow + n_own * kRecvBlock));
        got = mbar_wait(bar_recv, 0, p.timeout_ns) ? 1 : 0;
        if (!got) atomicOr(p.err, SMLA_FLAG_TIMEOUT);
    }
    got = __syncthreads_and(got);
    if (got) (void)mbar_try_wait(bar_recv, 0);  // every thread observes the completed phase
    const bool write = got && ok;
    if (tid < kHeads) {
        float mx = -INFINITY;
        for (int s = 0; s < ns; ++s)
            if (ml[s * 128 + 64 + tid] > 0.0f) mx = fmaxf(mx, ml[s * 128 + tid]);
        float sum = 0.0f;
        for (int s = 0; s < ns; ++s) {
            const float l = ml[s * 128 + 64 + tid];
            if (l > 0.0f) sum += exp2f(ml[s * 128 + tid] - mx) * l;
        }
        const float L = (sum > 0.0f) ? mx + log2f(sum) : -INFINITY;
        for (int s = 0; s < ns; ++s)
            weights[s * kHeads + tid] = (sum > 0.0f && ml[s * 128 + 64 + tid] > 0.0f) ? exp2f(ml[s * 128 + tid] - L)
                                                                                      : 0.0f;
        if (me == 0 && write)
            p.lse[static_cast<size_t>(b) * kHeads + tid] = (sum > 0.0f) ? L * 0.69314718055994531f : -INFINITY;
    }
    __syncthreads();
    if (write) {
#pragma unroll 1
        for (int mc = me; mc < 4; mc += ns) {
            const int lci = mc / ns;
            float acc[16];
            if (live) {
                tmem_ld16(tmem + lane_base + 64 * mc + 16 * g, acc);
                tmem_wait_ld();
            }
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                const float w = weights[me * kHeads + 16 * g + h];
                acc[h] = (live && w != 0.0f) ? acc[h] * w : 0.0f;
            }
            for (int s = 0; s < ns; ++s) {
                if (s == me) continue;
                const int slot = (s < me) ? s : s - 1;
                const float4 *src = reinterpret_cast<const float4 *>(smem + (lci * (ns - 1) + slot) * kRecvBlock +
                                                                     d * kRecvRow + 64 * g);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 v = src[j];
                    const float *w = weights + s * kHeads + 16 * g + 4 * j;
                    if (w[0] != 0.0f) acc[4 * j] += v.x * w[0];
                    if (w[1] != 0.0f) acc[4 * j + 1] += v.y * w[1];
                    if (w[2] != 0.0f) acc[4 * j + 2] += v.z * w[2];
                    if (w[3] != 0.0f) acc[4 * j + 3] += v.w * w[3];
                }
            }
            float *dst = p.out + (static_cast<size_t>(b) * kHeads + 16 * g) * kDim + 128 * mc + d;
#pragma unroll
            for (int h = 0; h < 16; ++h) dst[h * kDim] = acc[h];
        }
    }
    // barrier 2: no CTA leaves while a bulk copy may still be reading its staging area
    cluster_sync();
}

// ------------------------------------------------------------------ the decode kernel
// One CTA per (topk split, request), 16 warps, one 128-slot tile at a time:
//   1. every thread dequantises its 9 prefetched chunks of the tile into the bf16
//      tile (plain shared stores, a proxy fence, one mbarrier arrival per warp);
//   2. every thread issues the loads of the next tile (they stay in flight through
//      the MMA and softmax phases), and threads 0..127 run the index translation of
//      the tile after next, spread over the phases so its latency is hidden;
//   3. thread 0 issues S^T = K.Q^T (32 tcgen05.mma, M=128 tokens, N=64 heads);
//   4. softmax on all 16 warps: warp w reads TMEM lanes 32(w%4).. (tokens) and
//      columns 16(w/4).. (heads); p = 2^(s*c - m) against the running max m, which
//      is raised (with a rescale of O^T and of the per-lane running sums) only when a
//      score exceeds it by more than 2^8; P^T is written as bf16 hi + lo terms;
//   5. thread 0 issues O^T += V^T.P_hi^T + V^T.P_lo^T (64 tcgen05.mma).
// The epilogue reduces the per-lane sums and writes O/l and LSE, merging the splits of
// a request inside its thread-block cluster when there are several.
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_q) {
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
    float *head_m = reinterpret_cast<float *>(smem + kSmemHeadM);
    float *head_alpha = reinterpret_cast<float *>(smem + kSmemHeadAlpha);
    float *red = reinterpret_cast<float *>(smem + kSmemRed);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kSmemBars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmemTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kSmemAbort);

    const int num_tiles = (p.topk + kTile - 1) / kTile;
    const int t_begin = split * p.tiles_per_split;
    const int n = max(0, min(num_tiles, t_begin + p.tiles_per_split) - t_begin);
    const int seq_len = __ldg(p.seq_lens + b);
    const int32_t *bt_row = p.block_table + static_cast<size_t>(b) * p.max_blocks;
    const int32_t *idx_row = p.topk_idx + static_cast<size_t>(b) * p.topk;

    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        mbar_init(&bars[kBarQ], 1);
        mbar_init(&bars[kBarKvFull], 16);
        mbar_init(&bars[kBarSFull], 1);
        mbar_init(&bars[kBarPFull], 16);
        mbar_init(&bars[kBarPvDone], 1);
        mbar_init(&bars[kBarDrain], 1);
        mbar_init(&bars[kBarSpare], 1);
        mbar_init(&bars[kBarRecv], 1);
        fence_barrier_init();
        *abort_flag = 0;
        mbar_arrive_expect_tx(&bars[kBarQ], kHeads * kDim * 2);
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) tma_load_2d(sQ + kb * 8192, &tmap_q, 64 * kb, kHeads * b, &bars[kBarQ]);
    }
    if (tid < kHeads) head_m[tid] = -INFINITY;
    // index translation of tiles 0 and 1 (threads 0..255: tile tid/128, slot tid%128)
    if (tid < 2 * kTile) {
        const int ti = tid >> 7;
        const int slot = (t_begin + ti) * kTile + (tid & (kTile - 1));
        int code = -1;
        if (ti < n && slot < p.topk)
            code = translate_slot(bt_row, p.max_blocks, seq_len, p.num_pages, __ldg(idx_row + slot), p.err);
        codes[tid] = code;
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t kv_s = smem_addr(sKV);
    const uint32_t phi_s = smem_addr(sPhi);
    const uint32_t plo_s = smem_addr(sPlo);

    // thread roles inside the softmax / epilogue: TMEM lane quadrant q, head group g
    const int q = warp & 3;
    const int g = warp >> 2;
    const int r = 32 * q + lane;  // token lane of S^T, output-dim lane of O^T
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const float c = p.scale_log2;

    // MMA descriptors of the operand bases; every MMA adds a compile-time offset (bytes >> 4)
    const uint64_t dQK_a = sw128_desc(smem_addr(sKV), 16, 1024);
    const uint64_t dQK_b = sw128_desc(smem_addr(sQ), 16, 1024);
    const uint64_t dPV_a = sw128_desc(smem_addr(sKV), kTile * 128, 1024);
    const uint64_t dPV_bh = sw128_desc(smem_addr(sPhi), 8192, 1024);
    const uint64_t dPV_bl = sw128_desc(smem_addr(sPlo), 8192, 1024);

    TileRegs tr;
    if (n > 0) load_tile(tid, codes, p.cache, tr);
    bool failed = false, spare_used = false;
    int idx_next = -1, page_next = -1;

    for (int i = 0; i < n; ++i) {
        const int buf = i & 1;
        const bool valid = codes[buf * kTile + r] >= 0;
        // ---- 1. dequantise the tile
        store_pair<0>(tid, kv_s, tr.raw0, tr.sc0);
        store_pair<1>(tid, kv_s, tr.raw1, tr.sc1);
        store_pair<2>(tid, kv_s, tr.raw2, tr.sc2);
        store_pair<3>(tid, kv_s, tr.raw3, tr.sc3);
        fence_proxy_async_smem();  // this thread's tile stores -> visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarKvFull]);
        // ---- 2. prefetch the next tile, start translating the tile after it
        if (i + 1 < n) load_tile(tid, codes + (buf ^ 1) * kTile, p.cache, tr);
        const int slot2 = (t_begin + i + 2) * kTile + tid;
        if (tid < kTile && i + 2 < n && slot2 < p.topk) idx_next = __ldg(idx_row + slot2);
        // ---- 3. S^T = K.Q^T
        if (tid == 0) {
            bool ok = (i > 0 || wait_phase(&bars[kBarQ], 0, abort_flag, p)) &&
                      wait_phase(&bars[kBarKvFull], i & 1, abort_flag, p);
            if (ok) {
                tc_fence_after_sync();
#pragma unroll
                for (int kb = 0; kb < 8; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tmem + kTmemS, dQK_a + (kb * (kTile * 128) + kk * 32) / 16,
                                    dQK_b + (kb * 8192 + kk * 32) / 16, kIdescQK, (kb | kk) != 0);
                const bool hook = (i == 0) && (p.debug_flags & SMLA_DEBUG_SKIP_FIRST_COMMIT);
                mma_commit(hook ? &bars[kBarSpare] : &bars[kBarSFull]);
                spare_used = hook;
            }
        }
        bool ok = warp_wait_phase(&bars[kBarSFull], i & 1, abort_flag, p, lane);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        tc_fence_after_sync();
        if (tid < kTile && i + 2 < n && idx_next >= 0 && idx_next < seq_len && (idx_next >> 8) < p.max_blocks)
            page_next = __ldg(bt_row + (idx_next >> 8));
        // ---- 4. online softmax over 16 warps
        float x[16];
        tmem_ld16(tmem + lane_base + kTmemS + 16 * g, x);
        tmem_wait_ld();
        bool over = false;
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            x[h] = valid ? fmaf(x[h], c, -head_m[16 * g + h]) : -INFINITY;
            over |= x[h] > kRescaleThreshold;
        }
        if (__syncthreads_or(over)) {
            // raise each head's running max to max(m, tile max); rescale what was accumulated
            tmem_ld16(tmem + lane_base + kTmemS + 16 * g, x);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 16; ++h) x[h] = valid ? x[h] * c : -INFINITY;
            const float tmax = warp_transpose_reduce16<true>(x, lane);
            if ((lane & 1) == 0) red[q * 64 + 16 * g + (lane >> 1)] = tmax;
            __syncthreads();
            if (tid < kHeads) {
                const float tm = fmaxf(fmaxf(red[tid], red[64 + tid]), fmaxf(red[128 + tid], red[192 + tid]));
                const float mo = head_m[tid];
                const float mn = fmaxf(mo, tm);
                head_alpha[tid] = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
                head_m[tid] = mn;
            }
            __syncthreads();
            if (i > 0) {
                float al[16], o[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) al[h] = head_alpha[16 * g + h];
#pragma unroll 1
                for (int cc = 0; cc < 5; ++cc) {  // 4 O^T chunks + the running sums
                    const uint32_t col = (cc < 4 ? 64u * cc : kTmemL) + 16u * g;
                    tmem_ld16(tmem + lane_base + col, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 16; ++h) o[h] *= al[h];
                    tmem_st16(tmem + lane_base + col, o);
                }
            }
            tmem_ld16(tmem + lane_base + kTmemS + 16 * g, x);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 16; ++h) x[h] = valid ? fmaf(x[h], c, -head_m[16 * g + h]) : -INFINITY;
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) x[h] = fast_exp2(x[h]);
        {
            float l[16];
            if (i == 0) {
#pragma unroll
                for (int h = 0; h < 16; ++h) l[h] = x[h];
            } else {
                tmem_ld16(tmem + lane_base + kTmemL + 16 * g, l);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < 16; ++h) l[h] += x[h];
            }
            tmem_st16(tmem + lane_base + kTmemL + 16 * g, l);
        }
        // P^T row r, heads 16g..16g+15: two 16-byte chunks of hi and two of lo
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float a0 = x[8 * half + 2 * j], a1 = x[8 * half + 2 * j + 1];
                hw[j] = pack_bf16x2(a0, a1);
                lw[j] = pack_bf16x2(a0 - __uint_as_float(hw[j] << 16), a1 - __uint_as_float(hw[j] & 0xFFFF0000u));
            }
            const uint32_t off = r * 128 + (((2 * g + half) ^ (r & 7)) << 4);
            sts_v4(phi_s + off, make_uint4(hw[0], hw[1], hw[2], hw[3]));
            sts_v4(plo_s + off, make_uint4(lw[0], lw[1], lw[2], lw[3]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarPFull]);
        tmem_wait_st();
        tc_fence_before_sync();
        __syncthreads();
        // ---- 5. O^T += V^T.P^T
        if (tid == 0) {
            if (wait_phase(&bars[kBarPFull], i & 1, abort_flag, p)) {
                tc_fence_after_sync();
                const uint32_t acc0 = (i > 0) ? 1u : 0u;
#pragma unroll
                for (int mc = 0; mc < 4; ++mc) {
                    const uint64_t a0 = dPV_a + static_cast<uint64_t>(mc * 2 * (kTile * 128 / 16));
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        mma_bf16_ss(tmem + 64 * mc, a0 + ks * (2048 / 16), dPV_bh + ks * (2048 / 16), kIdescPV,
                                    ks > 0 ? 1u : acc0);
                        mma_bf16_ss(tmem + 64 * mc, a0 + ks * (2048 / 16), dPV_bl + ks * (2048 / 16), kIdescPV, 1u);
                    }
                }
                mma_commit(&bars[kBarPvDone]);
            }
        }
        ok = warp_wait_phase(&bars[kBarPvDone], i & 1, abort_flag, p, lane);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        tc_fence_after_sync();
        // translation of tile i+2 completes into the buffer tile i used
        if (tid < kTile && i + 2 < n) {
            int code = -1;
            if (idx_next >= 0 && idx_next < seq_len && (idx_next >> 8) < p.max_blocks) {
                if (page_next < 0 || static_cast<long long>(page_next) >= p.num_pages)
                    atomicOr(p.err, SMLA_FLAG_BAD_PAGE);
                else
                    code = page_next * kPageTokens + (idx_next & (kPageTokens - 1));
            }
            codes[buf * kTile + tid] = code;
            idx_next = -1;
            page_next = -1;
        }
        __syncthreads();
    }

    // every MMA issued above must be complete before tensor memory is released
    if (tid == 0) {
        if (spare_used) (void)mbar_wait(&bars[kBarSpare], 0, p.timeout_ns);
        mma_commit(&bars[kBarDrain]);
        (void)mbar_wait(&bars[kBarDrain], 0, p.timeout_ns);
    }
    __syncthreads();
    const bool ok = !failed && !*abort_flag;

    // ---- epilogue: per-head sums over the 128 token lanes, then O/l (or the cluster merge)
    float l_part = 0.0f;
    if (ok && n > 0) {
        tc_fence_after_sync();
        float v[16];
        tmem_ld16(tmem + lane_base + kTmemL + 16 * g, v);
        tmem_wait_ld();
        l_part = warp_transpose_reduce16<false>(v, lane);
    }
    if ((lane & 1) == 0) red[q * 64 + 16 * g + (lane >> 1)] = l_part;
    __syncthreads();
    float *l_head = head_alpha;  // per-head sums for the epilogue
    if (tid < kHeads) l_head[tid] = (red[tid] + red[64 + tid]) + (red[128 + tid] + red[192 + tid]);
    __syncthreads();
    if (p.cluster_merge) {
        cluster_epilogue(p, b, ok, n, tid, q, g, lane, tmem, lane_base, smem, &bars[kBarRecv], head_m, l_head, red);
    } else if (ok) {
        if (tid < kHeads) {
            const float l = l_head[tid];
            const float val = (l > 0.0f) ? (head_m[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
            if (p.nsplit == 1)
                p.lse[static_cast<size_t>(b) * kHeads + tid] = val;
            else
                p.part_lse[(static_cast<size_t>(b) * kHeads + tid) * p.nsplit + split] = val;
        }
        float inv[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            const float l = l_head[16 * g + h];
            inv[h] = (l > 0.0f) ? 1.0f / l : 0.0f;
        }
#pragma unroll 1
        for (int mc = 0; mc < 4; ++mc) {
            float o[16];
            if (n > 0) {
                tmem_ld16(tmem + lane_base + 64 * mc + 16 * g, o);
                tmem_wait_ld();
            }
            const int d = 128 * mc + r;
            if (p.nsplit == 1) {
                float *dst = p.out + (static_cast<size_t>(b) * kHeads + 16 * g) * kDim + d;
#pragma unroll
                for (int h = 0; h < 16; ++h) dst[h * kDim] = (n > 0) ? o[h] * inv[h] : 0.0f;
            } else {
                float *dst = p.part_o + ((static_cast<size_t>(b) * kHeads + 16 * g) * p.nsplit + split) * kDim + d;
#pragma unroll
                for (int h = 0; h < 16; ++h)
                    dst[static_cast<size_t>(h) * p.nsplit * kDim] = (n > 0) ? o[h] * inv[h] : 0.0f;
            }
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
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const uint8_t *cache, const int32_t *block_table,
                                                          const int32_t *topk_idx, const int32_t *seq_lens,
                                                          long long num_pages, int topk, int max_blocks,
                                                          float *latents, int32_t *page_slot, uint32_t *err) {
    __shared__ int codes[kTile];
    __shared__ uint2 scales[kTile];
    __shared__ __align__(16) uint8_t tile_row[kGatherThreads][32];
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
    for (int i = tid; i < kTile * kRowChunks; i += kGatherThreads) {
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
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
int tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000 &fn) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_encode_tiled == nullptr) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || f == nullptr)
            return SMLA_ERR_CUDA;
        g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    fn = g_encode_tiled;
    return SMLA_OK;
}

// Q [B*64 rows, 512 bf16] as a 2-D tensor; a box of 64 dims x 64 heads with the
// 128-byte swizzle lands as one K-block of the shared-memory Q operand.
int encode_q_map(CUtensorMap *map, const void *q, int B) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    const int rc = tensor_map_encoder(fn);
    if (rc != SMLA_OK) return rc;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(SMLA_DIM), static_cast<cuuint64_t>(B) * SMLA_HEADS};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(SMLA_DIM) * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(q), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? SMLA_OK : SMLA_ERR_INVALID;
}

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

// Up to this many splits of a request merge inside a thread-block cluster (through
// distributed shared memory); beyond it they go through global partials and the
// merge kernel.
constexpr int kMaxClusterSplits = 4;

size_t workspace_for(int B, int topk, int nsplit) {
    size_t bytes = SMLA_WORKSPACE_HEADER;
    if (nsplit > kMaxClusterSplits) {
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

    alignas(64) CUtensorMap tmap_q;
    rc = encode_q_map(&tmap_q, q, B);
    if (rc != SMLA_OK) return rc;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    (void)cudaGetLastError();
    p.cluster_merge = (nsplit > 1 && nsplit <= kMaxClusterSplits) ? 1 : 0;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(nsplit, B);
    cfg.blockDim = dim3(smla::kThreads);
    cfg.dynamicSmemBytes = smla::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.cluster_merge ? nsplit : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, smla::decode_kernel, p, tmap_q) != cudaSuccess) return SMLA_ERR_LAUNCH;
    if (cudaGetLastError() != cudaSuccess) return SMLA_ERR_LAUNCH;
    if (nsplit > 1 && !p.cluster_merge) {
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
    smla::gather_kernel<<<dim3(num_tiles(topk), B), smla::kGatherThreads, 0, static_cast<cudaStream_t>(stream)>>>(
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

