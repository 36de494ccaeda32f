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
// B200 mapping, per CTA (one per SM, 512 threads in two warp roles):
//   * Q[b] (64 heads x 512, bf16) stays in shared memory for the whole CTA (TMA).
//   * Producer warps translate a tile of 128 topk slots through the block table,
//     keep its FP8 rows in flight in registers (16-byte loads) while the previous
//     tile is computed, and dequantise them into a bf16 [128 x 512] tile in the
//     128-byte-swizzled layout the tensor core reads, one 128-dim K-block pair at
//     a time as the previous tile's PV releases it.
//   * S^T[128 tokens x 64 heads] = K_tile . Q^T: tcgen05.mma M=128 N=64, fp32 in
//     tensor memory (two S^T buffers).  Tokens fill the 128-row M dimension, not
//     the 64 heads.
//   * Softmax warps (one thread per token lane and 32 heads) read S^T from tensor
//     memory, keep the running max per head and the sums in registers, rescale
//     O^T in tensor memory when the max grows, and write P^T as two bf16 terms
//     (P = P_hi + P_lo).  One of their threads issues the MMAs.
//   * O^T[512 x 64] += V^T . P^T with V = the same bf16 tile read MN-major:
//     4 MMAs of M=128 per 16-token step, once with P_hi and once with P_lo, so P
//     carries ~16 significant bits (a single bf16 P is not accurate enough when
//     a few large latents dominate).
//   * The epilogue reads O^T from tensor memory and writes O/l (or merges the
//     splits of a request inside its cluster) and LSE = (m + log2 l) ln 2.
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

constexpr int kTile = 128;                                  // topk slots per MMA tile (the M of S^T)
constexpr int kSoftmaxWarps = 8;                            // warps 0..7: softmax and epilogue; warp 0 also
                                                            // owns tensor memory and issues TMA and MMAs
constexpr int kProducerWarps = 8;                           // warps 8..15: translation, gather, dequantisation
constexpr int kThreads = 32 * (kSoftmaxWarps + kProducerWarps);  // 512: 128 registers per thread
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;         // 256
constexpr int kProducerThreads = 32 * kProducerWarps;       // 256
constexpr int kGatherThreads = 256;                         // threads of the gather debug kernel
constexpr uint32_t kBarIdSoftmax = 1;                       // named barrier of the softmax warps
constexpr uint32_t kBarIdProducer = 2;                      // named barrier of the producer warps

// Dynamic shared memory map (bytes from a 1024-aligned base).
constexpr int kSmemQ = 0;                         // 64 KB: 8 K-blocks x [64 heads x 128 B], TMA-written
constexpr int kSmemKV = kSmemQ + 65536;           // 128 KB: 8 K-blocks x [128 tokens x 128 B]
constexpr int kSmemPhi = kSmemKV + 131072;        // 16 KB: P_hi^T [128 tokens x 64 heads] bf16
constexpr int kSmemPlo = kSmemPhi + 16384;        // 16 KB: P_lo^T
constexpr int kSmemCodes = kSmemPlo + 16384;      // [2][128] int32 token codes (producers only)
constexpr int kSmemMask = kSmemCodes + 1024;      // [4][4] u32: valid-token bits of a tile, ring of 4 tiles
constexpr int kSmemHeadM = kSmemMask + 64;        // [64] running max per head (log2 units)
constexpr int kSmemHeadAlpha = kSmemHeadM + 256;  // [64] rescale factor of the last max update; then the sums
constexpr int kSmemRed = kSmemHeadAlpha + 256;    // [4][64] f32 cross-quadrant scratch
constexpr int kSmemBars = kSmemRed + 1024;        // mbarriers (8 B each)

enum Bar : int {
    kBarQ = 0,        // Q landed (TMA transaction bytes)
    kBarKvFull = 1,   // + c (c = 0..3): K-block pair c of the tile written (8 producer-warp arrivals)
    kBarKvFree = 5,   // + c: PV chunk c of the tile done (MMA commit): pair c may be overwritten
    kBarSFull = 9,    // + s (s = 0..1): S^T buffer s complete (MMA commit)
    kBarPFull = 11,   // P^T written (8 softmax-warp arrivals)
    kBarDrain = 12,   // final commit before tensor memory is released
    kBarSpare = 13,   // test hook target
    kBarXch = 14,     // cluster merge: the other CTAs' rows and chunks landed (bulk-copy bytes)
    kNumBars = 15,
};
constexpr int kSmemTmemSlot = kSmemBars + kNumBars * 8;
constexpr int kSmemAbort = kSmemTmemSlot + 4;
constexpr int kSmemBytes = kSmemAbort + 4;
static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-block shared memory limit");
static_assert(kSmemBars % 8 == 0, "mbarriers need 8-byte alignment");

// Tensor memory: O^T [0,256) (4 chunks of 128 dims x 64 heads), S^T buffers at 256 and 320,
// per-lane running sums L at 384 (lane = token of the tile, column = head).
constexpr int kMlBytes = 128 * 4;  // one (m, l) row of the cluster merge
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 256;
constexpr uint32_t kTmemL = 384;
constexpr uint32_t kIdescQK = idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16(128, 64, true, true);
// log2 units: the running max m of a head is raised (and O^T, the sums rescaled) only when a
// score exceeds it by more than this, so p = 2^(s - m) stays below 2^24: P_hi + P_lo keep their
// relative precision at any magnitude, and fp32 O^T sums of 2^24 x |v| stay far from overflow.
constexpr float kRescaleThreshold = 24.0f;

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
    int cluster_merge;  // 1: the nsplit CTAs of a request form a cluster and merge in the kernel
};

// Reduces N (16 or 32) per-thread values across the 32 lanes of a warp, value i with
// value i of every other lane.  Each round halves the live entries: a lane keeps the
// half selected by its lane bit and sends the other half to its partner.  With N = 32
// lane j ends with entry j; with N = 16 lanes 2j and 2j+1 end with entry j.
template <bool kMax, int N>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[N], int lane) {
    static_assert(N == 16 || N == 32, "16 or 32 entries");
#pragma unroll
    for (int w = N / 2, off = 16; w >= 1; w >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float send = upper ? v[i] : v[i + w];
            const float keep = upper ? v[i + w] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, off);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    if constexpr (N == 16) {
        const float got = __shfl_xor_sync(0xffffffffu, v[0], 1);
        return kMax ? fmaxf(v[0], got) : v[0] + got;
    }
    return v[0];
}

// 16 consecutive floats of shared memory (16-byte aligned) into registers.
__device__ __forceinline__ void load16(const float *src, float (&v)[16]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 t = reinterpret_cast<const float4 *>(src)[j];
        v[4 * j] = t.x;
        v[4 * j + 1] = t.y;
        v[4 * j + 2] = t.z;
        v[4 * j + 3] = t.w;
    }
}

// Bounded wait on an mbarrier phase.  Gives up when another thread has aborted the
// CTA or when `timeout_ns` passes (then it aborts the CTA and flags the error).
__device__ __noinline__ bool wait_phase_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             const DecodeParams &p) {
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
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                           const DecodeParams &p) {
    return mbar_try_wait(bar, parity) || wait_phase_slow(bar, parity, abort_flag, p);
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
// The 128 x 36 sixteen-byte chunks of a tile are dealt out to the 256 producer threads
// (pt) in four groups, one per K-block pair c (dims [128c, 128c+128)):
//   pairs 0..2: chunk 8c + (pt & 7) of the tokens (pt >> 3) + 32u, u < 4     (nope)
//   pair 3:     chunk 24 + (pt & 3) of the tokens (pt >> 2) + 64u, u < 2     (nope)
//               chunk 28 + (pt & 7) of the tokens (pt >> 3) + 32u, u < 4     (rope)
// Consecutive threads take consecutive chunks of a token row (coalesced loads).

// The FP8 bytes of one tile and their scales, held in registers between the load and
// the dequantisation.  For pairs 0..2 each token's 8-byte scale row is loaded once.
struct TileRegs {
    uint4 raw0[4], raw1[4], raw2[4], nope3[2], rope[4];
    uint2 srow[4];
    uint32_t sc3[2];
};

__device__ __forceinline__ void load_tile(int t, const int *codes, const uint8_t *cache, TileRegs &tr) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int code = codes[(t >> 3) + 32 * u];
        const int chunk = t & 7;
        tr.raw0[u] = tr.raw1[u] = tr.raw2[u] = tr.rope[u] = make_uint4(0u, 0u, 0u, 0u);
        tr.srow[u] = make_uint2(0u, 0u);
        if (code >= 0) {
            const uint8_t *row = token_row(cache, code);
            tr.raw0[u] = ld_stream_v4(row + chunk * 16);
            tr.raw1[u] = ld_stream_v4(row + (8 + chunk) * 16);
            tr.raw2[u] = ld_stream_v4(row + (16 + chunk) * 16);
            tr.srow[u] = ld_stream_v2(token_scales(cache, code));
            tr.rope[u] = ld_stream_v4(row + (28 + chunk) * 16);
        }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int code = codes[(t >> 2) + 64 * u];
        tr.nope3[u] = make_uint4(0u, 0u, 0u, 0u);
        tr.sc3[u] = 0u;
        if (code >= 0) {
            tr.nope3[u] = ld_stream_v4(token_row(cache, code) + (24 + (t & 3)) * 16);
            tr.sc3[u] = ld_stream_u8(token_scales(cache, code) + 6);
        }
    }
}

// Dequantises 16 e4m3 bytes (or copies 16 rope bytes) into row r of K-block kb of the
// swizzled bf16 tile at 16-byte unit oc (two units for nope).
__device__ __forceinline__ void store_item(uint32_t kv, int r, int kb, int oc, bool nope, const uint4 raw,
                                           uint32_t sc) {
    const uint32_t row = kv + kb * (kTile * 128) + r * 128;
    const int sw = r & 7;
    if (nope) {
        uint4 lo, hi;
        dequant16(raw, sc, lo, hi);
        // odd K-blocks store their high half first so the 8 lanes of a store phase hit 8 bank groups
        const bool odd = (kb & 1) != 0;
        sts_v4(row + (((oc + (odd ? 1 : 0)) ^ sw) << 4), odd ? hi : lo);
        sts_v4(row + (((oc + (odd ? 0 : 1)) ^ sw) << 4), odd ? lo : hi);
    } else {
        sts_v4(row + ((oc ^ sw) << 4), raw);
    }
}

// Publishes K-block pair c of the tile to the tensor core once this warp's stores are
// visible to the async proxy.
__device__ __forceinline__ void publish_pair(int c, int lane, uint64_t *bars) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kBarKvFull + c]);
}

// Producer steps for one tile: each K-block pair is dequantised as soon as the PV of the
// previous tile has released it.  Pairs 0..2 share one rolled loop (in them a thread
// takes chunk (pt & 7) of the tokens (pt >> 3) + 32u); pair 3 holds the last nope chunk
// group and the rope.
__device__ __forceinline__ bool produce_tile(int i, int pt, int lane, uint32_t kv_s, uint64_t *bars,
                                             volatile int *abort_flag, const DecodeParams &p, const TileRegs &tr) {
    const int k = pt & 7;
#pragma unroll 1
    for (int c = 0; c < 3; ++c) {
        if (i > 0 && !warp_wait_phase(&bars[kBarKvFree + c], (i - 1) & 1, abort_flag, p, lane)) return false;
        const int byte = 2 * c + (k >> 2);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint4 raw = (c == 0) ? tr.raw0[u] : (c == 1) ? tr.raw1[u] : tr.raw2[u];
            const uint32_t w = (byte < 4) ? tr.srow[u].x : tr.srow[u].y;
            store_item(kv_s, (pt >> 3) + 32 * u, 2 * c + (k >> 2), 2 * (k & 3), true, raw,
                       (w >> (8 * (byte & 3))) & 0xFFu);
        }
        publish_pair(c, lane, bars);
    }
    if (i > 0 && !warp_wait_phase(&bars[kBarKvFree + 3], (i - 1) & 1, abort_flag, p, lane)) return false;
#pragma unroll
    for (int u = 0; u < 2; ++u) store_item(kv_s, (pt >> 2) + 64 * u, 6, 2 * (pt & 3), true, tr.nope3[u], tr.sc3[u]);
#pragma unroll
    for (int u = 0; u < 4; ++u) store_item(kv_s, (pt >> 3) + 32 * u, 7, k, false, tr.rope[u], 0u);
    publish_pair(3, lane, bars);
    return true;
}

// ------------------------------------------------------------------ split merge in a cluster
// The nsplit (2..4) CTAs of one request form a thread-block cluster, which makes them
// co-resident.  After the last PV, CTA s holds un-normalised O^T_s (tensor memory), its
// per-head running max m_s (log2 units) and sum l_s.  With L = log2 sum_s 2^(m_s) l_s,
// the merged output is O = sum_s 2^(m_s - L) O^T_s and LSE = L ln 2 (the split-K
// log-sum-exp merge).  Output dims are dealt out by 128-dim chunk: chunk mc belongs to
// CTA mc % nsplit.  Each CTA publishes its (m_s, l_s) row and the O^T_s chunks it does
// not own to the workspace (coalesced stores that stay in L2); after one cluster barrier
// (release / acquire) each owner pulls what it needs into its own shared memory with
// bulk copies counted on one mbarrier (a single L2 round trip), then merges.
// Distributed shared memory is not used for the exchange: its per-SM bandwidth is a
// fraction of what L2 gives one SM.
//   ml   [B][nsplit][m(64) | l(64)] f32
//   xch  [B][4 chunks][nsplit - 1 sender slots][64 heads][128 dims] f32 (a warp's
//        32 consecutive dims are one 128-byte line); the sender slot of CTA s in
//        chunk mc is s, minus one when s is above the owner.
// Shared memory (the operand buffers are dead by then): the rows at the Q buffer
// [nsplit][128] f32, the received chunks at the KV buffer [owned chunk][sender slot]
// [64][128] f32.
// Called by every thread of the CTA (the cluster barrier needs them all); the softmax
// warps (quadrant q, head half hh) do the work.
constexpr int kXchBlock = kHeads * 128 * 4;  // one 128-dim chunk of O^T, bytes

__device__ __noinline__ void cluster_epilogue(const DecodeParams &p, int b, bool ok, int n, int tid, int warp,
                                              int lane, uint32_t tmem, uint8_t *smem, uint64_t *bar_xch,
                                              const float *head_m, const float *l_head, float *weights) {
    const int ns = p.nsplit;
    const int me = static_cast<int>(cluster_ctarank());
    const int n_own = (4 - me + ns - 1) / ns;  // chunks me, me + ns, ... below 4
    const bool worker = warp < kSoftmaxWarps;
    const int q = warp & 3, hh = (warp >> 2) & 1;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const int d = 32 * q + lane;  // row of O^T within a chunk
    const bool live = ok && n > 0;
    float *ml = p.part_lse + static_cast<size_t>(b) * ns * 128;
    float *xch = p.part_o + static_cast<size_t>(b) * 4 * (ns - 1) * (kHeads * 128);
    float *ml_s = reinterpret_cast<float *>(smem + kSmemQ);
    const float *recv = reinterpret_cast<const float *>(smem + kSmemKV);

    if (tid < kHeads) {
        const float mv = live ? head_m[tid] : -INFINITY;
        const float lv = live ? l_head[tid] : 0.0f;
        ml[me * 128 + tid] = mv;
        ml[me * 128 + 64 + tid] = lv;
        ml_s[me * 128 + tid] = mv;
        ml_s[me * 128 + 64 + tid] = lv;
    }
    if (worker) {
#pragma unroll 1
        for (int part = 0; part < 8; ++part) {  // 4 chunks x 2 halves of 16 heads
            const int mc = part >> 1, h0 = 32 * hh + 16 * (part & 1);
            const int owner = mc % ns;
            if (owner == me) continue;
            float o[16];
            if (live) {
                tmem_ld16(tmem + lane_base + 64 * mc + h0, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int h = 0; h < 16; ++h) o[h] = 0.0f;
            }
            const int slot = (me < owner) ? me : me - 1;
            float *dst = xch + ((mc * (ns - 1) + slot) * kHeads + h0) * 128 + d;
#pragma unroll
            for (int h = 0; h < 16; ++h) __stcg(dst + h * 128, o[h]);
        }
    }
    fence_proxy_async_all();  // the peers read these rows and chunks with bulk copies
    // every CTA's row and chunks are written before any owner fetches them
    cluster_sync();
    int got = 1;
    if (tid == 0) {
        fence_proxy_async_all();
        mbar_arrive_expect_tx(bar_xch, (ns - 1) * (kMlBytes + n_own * kXchBlock));
        for (int s = 0; s < ns; ++s) {
            if (s == me) continue;
            bulk_load(ml_s + s * 128, ml + s * 128, kMlBytes, bar_xch);
            const int slot = (s < me) ? s : s - 1;
            for (int lci = 0; lci < n_own; ++lci) {
                const int mc = me + lci * ns;
                bulk_load(smem + kSmemKV + (lci * (ns - 1) + slot) * kXchBlock,
                          xch + (mc * (ns - 1) + slot) * (kHeads * 128), kXchBlock, bar_xch);
            }
        }
        got = mbar_wait(bar_xch, 0, p.timeout_ns) ? 1 : 0;
        if (!got) atomicOr(p.err, SMLA_FLAG_TIMEOUT);
    }
    got = __syncthreads_and(got);
    if (got) (void)mbar_try_wait(bar_xch, 0);  // every thread observes the completed phase
    const bool write = ok && got;
    if (tid < kHeads) {
        float mx = -INFINITY;
        for (int s = 0; s < ns; ++s)
            if (ml_s[s * 128 + 64 + tid] > 0.0f) mx = fmaxf(mx, ml_s[s * 128 + tid]);
        float sum = 0.0f;
        for (int s = 0; s < ns; ++s) {
            const float lv = ml_s[s * 128 + 64 + tid];
            if (lv > 0.0f) sum += exp2f(ml_s[s * 128 + tid] - mx) * lv;
        }
        const float L = (sum > 0.0f) ? mx + log2f(sum) : -INFINITY;
        for (int s = 0; s < ns; ++s) {
            const float lv = ml_s[s * 128 + 64 + tid];
            weights[s * kHeads + tid] = (sum > 0.0f && lv > 0.0f) ? exp2f(ml_s[s * 128 + tid] - L) : 0.0f;
        }
        if (me == 0 && write)
            p.lse[static_cast<size_t>(b) * kHeads + tid] = (sum > 0.0f) ? L * 0.69314718055994531f : -INFINITY;
    }
    __syncthreads();
    if (!write || !worker) return;
#pragma unroll 1
    for (int part = 0; part < 2 * n_own; ++part) {  // owned chunks x 2 halves of 16 heads
        const int lci = part >> 1, mc = me + lci * ns, h0 = 32 * hh + 16 * (part & 1);
        float acc[16];
        if (live) {
            tmem_ld16(tmem + lane_base + 64 * mc + h0, acc);
            tmem_wait_ld();
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            const float w = weights[me * kHeads + h0 + h];
            acc[h] = (live && w != 0.0f) ? acc[h] * w : 0.0f;
        }
        for (int s = 0; s < ns; ++s) {
            if (s == me) continue;
            const int slot = (s < me) ? s : s - 1;
            const float *src = recv + ((lci * (ns - 1) + slot) * kHeads + h0) * 128 + d;
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                const float w = weights[s * kHeads + h0 + h];
                if (w != 0.0f) acc[h] += src[h * 128] * w;
            }
        }
        float *dst = p.out + (static_cast<size_t>(b) * kHeads + h0) * kDim + 128 * mc + d;
#pragma unroll
        for (int h = 0; h < 16; ++h) dst[h * kDim] = acc[h];
    }
}

// ------------------------------------------------------------------ MMA issue
// The tensor-core side of the pipeline, run by one thread.  Every wait is bounded; a
// failed wait leaves `ok` false and issues nothing more.
struct MmaIssuer {
    uint64_t dQK_a, dQK_b, dPV_a, dPV_bh, dPV_bl;
    uint32_t tmem;
    const DecodeParams &p;
    uint64_t *bars;
    volatile int *abort_flag;
    bool ok = true;
    bool spare_used = false;

    __device__ MmaIssuer(uint8_t *smem, uint32_t tmem_, const DecodeParams &p_, uint64_t *bars_,
                         volatile int *abort_)
        : tmem(tmem_), p(p_), bars(bars_), abort_flag(abort_) {
        dQK_a = sw128_desc(smem_addr(smem + kSmemKV), 16, 1024);
        dQK_b = sw128_desc(smem_addr(smem + kSmemQ), 16, 1024);
        dPV_a = sw128_desc(smem_addr(smem + kSmemKV), kTile * 128, 1024);
        dPV_bh = sw128_desc(smem_addr(smem + kSmemPhi), 8192, 1024);
        dPV_bl = sw128_desc(smem_addr(smem + kSmemPlo), 8192, 1024);
    }

    // S^T[tile i] = K.Q^T into buffer i&1, one K-block pair as soon as it is published.
    __device__ void qk(int i) {
        if (!ok) return;
        const uint32_t s_col = tmem + kTmemS + 64 * (i & 1);
        uint64_t a = dQK_a, bq = dQK_b;
        uint32_t acc = 0u;
#pragma unroll 1
        for (int cp = 0; cp < 4; ++cp) {
            ok = ok && (i > 0 || cp > 0 || wait_phase(&bars[kBarQ], 0, abort_flag, p)) &&
                 wait_phase(&bars[kBarKvFull + cp], i & 1, abort_flag, p);
            if (!ok) return;
            tc_fence_after_sync();
#pragma unroll 1
            for (int kb = 0; kb < 2; ++kb) {
                // K-block: 4 MMAs of K=16 (32 bytes apart), the next K-block 16 KB (K) / 8 KB (Q) on
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    mma_bf16_ss(s_col, a + kk * 2, bq + kk * 2, kIdescQK, acc);
                    acc = 1u;
                }
                a += (kTile * 128) / 16;
                bq += 8192 / 16;
            }
        }
        const bool hook = (i == 0) && (p.debug_flags & SMLA_DEBUG_SKIP_FIRST_COMMIT);
        mma_commit(hook ? &bars[kBarSpare] : &bars[kBarSFull + (i & 1)]);
        spare_used = spare_used || hook;
    }

    // O^T += V^T.P_hi^T + V^T.P_lo^T of tile i once every softmax warp has written P^T;
    // each 128-dim chunk is committed to the producers as it completes.
    __device__ bool pv(int i) {
        if (!ok) return false;
        ok = wait_phase(&bars[kBarPFull], i & 1, abort_flag, p);
        if (!ok) return false;
        tc_fence_after_sync();
        const uint32_t acc0 = (i > 0) ? 1u : 0u;
#pragma unroll 1
        for (int mc = 0; mc < 4; ++mc) {
            uint64_t a = dPV_a + static_cast<uint64_t>(mc * 2 * (kTile * 128 / 16));
            uint64_t bh = dPV_bh, bl = dPV_bl;
            uint32_t acc = acc0;
#pragma unroll 2
            for (int ks = 0; ks < 8; ++ks) {  // 16 tokens per step: 2 KB on in V^T and in P^T
                mma_bf16_ss(tmem + 64 * mc, a, bh, kIdescPV, acc);
                mma_bf16_ss(tmem + 64 * mc, a, bl, kIdescPV, 1u);
                acc = 1u;
                a += 2048 / 16;
                bh += 2048 / 16;
                bl += 2048 / 16;
            }
            mma_commit(&bars[kBarKvFree + mc]);
        }
        return true;
    }

    __device__ void drain() {
        if (spare_used) (void)mbar_wait(&bars[kBarSpare], 0, p.timeout_ns);
        mma_commit(&bars[kBarDrain]);
        (void)mbar_wait(&bars[kBarDrain], 0, p.timeout_ns);
    }
};

// ------------------------------------------------------------------ the decode kernel
// One CTA per (topk split, request), one 128-slot tile at a time, three warp roles
// that hand work to each other through mbarriers:
//   producers (8 warps): translate the slots of tile i+2 through the block table,
//     keep the FP8 rows of tile i+1 in flight in registers, and dequantise tile i
//     into the bf16 tile one K-block pair at a time, each pair as soon as the PV of
//     tile i-1 has released it (so dequantisation overlaps the previous PV);
//   MMA issue (lane 0 of softmax warp 0, between its softmax steps): once P^T of tile
//     i is written, O^T += V^T.P_hi^T + V^T.P_lo^T (64 MMAs), committing each 128-dim
//     chunk to the producers; then S^T = K.Q^T of tile i+1 (M=128 tokens, N=64
//     heads) pair by pair as the producers publish them, into the other of two S^T
//     buffers in tensor memory;
//   softmax (8 warps; warp w reads TMEM lanes 32(w%4).. = tokens, columns for heads
//     32(w/4)..): p = 2^(s*c - m) against the running max m, which is raised (with a
//     rescale of O^T and of the per-thread sums) only when a score exceeds it by more
//     than 2^8; P^T is written as bf16 hi + lo terms.
// The epilogue reduces the per-thread sums and writes O/l and LSE, merging the splits of
// a request inside its thread-block cluster when there are 2..4 of them.
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
    int *codes = reinterpret_cast<int *>(smem + kSmemCodes);
    uint32_t *mask = reinterpret_cast<uint32_t *>(smem + kSmemMask);
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

    // ---- setup
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
        if (lane == 0) {
            mbar_init(&bars[kBarQ], 1);
            for (int c = 0; c < 4; ++c) {
                mbar_init(&bars[kBarKvFull + c], kProducerWarps);
                mbar_init(&bars[kBarKvFree + c], 1);
            }
            mbar_init(&bars[kBarSFull], 1);
            mbar_init(&bars[kBarSFull + 1], 1);
            mbar_init(&bars[kBarPFull], kSoftmaxWarps);
            mbar_init(&bars[kBarDrain], 1);
            mbar_init(&bars[kBarSpare], 1);
            mbar_init(&bars[kBarXch], 1);
            fence_barrier_init();
            *abort_flag = 0;
            mbar_arrive_expect_tx(&bars[kBarQ], kHeads * kDim * 2);
#pragma unroll
            for (int kb = 0; kb < 8; ++kb) tma_load_2d(sQ + kb * 8192, &tmap_q, 64 * kb, kHeads * b, &bars[kBarQ]);
        }
    } else if (warp >= kSoftmaxWarps) {
        // index translation of tiles 0 and 1 (producer thread pt: tile pt/128, slot pt%128)
        const int pt = tid - kSoftmaxThreads;
        const int ti = pt >> 7;
        const int slot = (t_begin + ti) * kTile + (pt & (kTile - 1));
        int code = -1;
        if (ti < n && slot < p.topk)
            code = translate_slot(bt_row, p.max_blocks, seq_len, p.num_pages, __ldg(idx_row + slot), p.err);
        codes[pt] = code;
        const uint32_t bits = __ballot_sync(0xffffffffu, code >= 0);
        if (lane == 0) mask[ti * 4 + ((pt >> 5) & 3)] = bits;
    }
    if (tid < kHeads) head_m[tid] = -INFINITY;
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const float c = p.scale_log2;

    if (warp < kSoftmaxWarps) {
        // ================================================================ softmax (+ MMA issue)
        const int q = warp & 3;
        const int hh = warp >> 2;
        const int r = 32 * q + lane;  // token lane of S^T
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        const uint32_t phi_s = smem_addr(smem + kSmemPhi);
        const uint32_t plo_s = smem_addr(smem + kSmemPlo);
        const bool issuer = (tid == 0);
        MmaIssuer mma(smem, tmem, p, bars, abort_flag);
        if (issuer && n > 0) mma.qk(0);
        __syncwarp();
        bool failed = false;
        for (int i = 0; i < n; ++i) {
            const int sb = i & 1;
            const uint32_t s_cols = tmem + lane_base + kTmemS + 64 * sb + 32 * hh;
            const uint32_t l_cols = tmem + lane_base + kTmemL + 32 * hh;
            const bool ok = warp_wait_phase(&bars[kBarSFull + sb], (i >> 1) & 1, abort_flag, p, lane);
            if (barrier_or(kBarIdSoftmax, kSoftmaxThreads, !ok)) {
                failed = true;
                break;
            }
            tc_fence_after_sync();
            const bool valid = (mask[(i & 3) * 4 + q] >> lane) & 1u;
            // does any score exceed its head's running max by more than the threshold?
            bool over = false;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float x[16];
                tmem_ld16(s_cols + 16 * half, x);
                tmem_wait_ld();
                float m[16];
                load16(head_m + 32 * hh + 16 * half, m);
#pragma unroll
                for (int h = 0; h < 16; ++h) over |= valid && (x[h] * c - m[h]) > kRescaleThreshold;
            }
            if (barrier_or(kBarIdSoftmax, kSoftmaxThreads, over)) {
                // raise each head's running max to max(m, tile max); rescale what was accumulated
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float x[16];
                    tmem_ld16(s_cols + 16 * half, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 16; ++h) x[h] = valid ? x[h] * c : -INFINITY;
                    const float tmax = warp_transpose_reduce<true, 16>(x, lane);
                    if ((lane & 1) == 0) red[q * 64 + 32 * hh + 16 * half + (lane >> 1)] = tmax;
                }
                named_barrier_sync(kBarIdSoftmax, kSoftmaxThreads);
                if (tid < kHeads) {
                    const float tm = fmaxf(fmaxf(red[tid], red[64 + tid]), fmaxf(red[128 + tid], red[192 + tid]));
                    const float mo = head_m[tid];
                    const float mn = fmaxf(mo, tm);
                    head_alpha[tid] = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
                    head_m[tid] = mn;
                }
                named_barrier_sync(kBarIdSoftmax, kSoftmaxThreads);
                if (i > 0) {
                    // the PV of tile i-1 is complete (the S^T commit of tile i covers it): rescale
                    // the 4 O^T chunks and the sums, 16 heads at a time
#pragma unroll 1
                    for (int part = 0; part < 10; ++part) {
                        const int h0 = 16 * (part & 1);
                        const uint32_t col = (part < 8 ? tmem + lane_base + 64 * (part >> 1) + 32 * hh : l_cols) + h0;
                        float o[16], al[16];
                        tmem_ld16(col, o);
                        load16(head_alpha + 32 * hh + h0, al);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < 16; ++h) o[h] *= al[h];
                        tmem_st16(col, o);
                    }
                }
            }
            // p = 2^(s c - m): add to the sums, write P^T row r as bf16 hi + lo
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float x[16], l[16];
                tmem_ld16(s_cols + 16 * half, x);
                if (i > 0) tmem_ld16(l_cols + 16 * half, l);
                tmem_wait_ld();
                float m[16];
                load16(head_m + 32 * hh + 16 * half, m);
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    x[h] = valid ? fast_exp2(x[h] * c - m[h]) : 0.0f;
                    l[h] = (i > 0) ? l[h] + x[h] : x[h];
                }
                tmem_st16(l_cols + 16 * half, l);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a0 = x[8 * j + 2 * e], a1 = x[8 * j + 2 * e + 1];
                        hw[e] = pack_bf16x2(a0, a1);
                        lw[e] = pack_bf16x2(a0 - __uint_as_float(hw[e] << 16), a1 - __uint_as_float(hw[e] & 0xFFFF0000u));
                    }
                    const uint32_t off = r * 128 + (((4 * hh + 2 * half + j) ^ (r & 7)) << 4);
                    sts_v4(phi_s + off, make_uint4(hw[0], hw[1], hw[2], hw[3]));
                    sts_v4(plo_s + off, make_uint4(lw[0], lw[1], lw[2], lw[3]));
                }
            }
            fence_proxy_async_smem();
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarPFull]);
            // warp 0's lane 0 issues PV of this tile and QK of the next one while the other
            // softmax warps wait for that S^T
            if (issuer && mma.pv(i) && i + 1 < n) mma.qk(i + 1);
            __syncwarp();
        }
        // the last PV is complete before the epilogue reads O^T
        if (!failed && n > 0) {
            const bool ok = warp_wait_phase(&bars[kBarKvFree + 3], (n - 1) & 1, abort_flag, p, lane);
            (void)barrier_or(kBarIdSoftmax, kSoftmaxThreads, !ok);
        }
        // every MMA issued must be complete before tensor memory is released
        if (issuer) mma.drain();
        __syncwarp();
        tc_fence_after_sync();
        // per-head sums over this warp's 32 token lanes
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            float l[16];
            if (n > 0 && !failed) {
                tmem_ld16(tmem + lane_base + kTmemL + 32 * hh + 16 * half, l);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int h = 0; h < 16; ++h) l[h] = 0.0f;
            }
            const float ls = warp_transpose_reduce<false, 16>(l, lane);
            if ((lane & 1) == 0) red[q * 64 + 32 * hh + 16 * half + (lane >> 1)] = ls;
        }
    } else {
        // ================================================================ producers
        const int pt = tid - kSoftmaxThreads;
        const uint32_t kv_s = smem_addr(sKV);
        TileRegs tr;
        if (n > 0) load_tile(pt, codes, p.cache, tr);
        for (int i = 0; i < n; ++i) {
            const int buf = i & 1;
            // translation of tile i+2, first step: its topk indices
            const int slot2 = (t_begin + i + 2) * kTile + pt;
            int idx_next = -1;
            if (pt < kTile && i + 2 < n && slot2 < p.topk) idx_next = __ldg(idx_row + slot2);
            bool ok = produce_tile(i, pt, lane, kv_s, bars, abort_flag, p, tr);
            // second step: the block-table entries
            int page_next = -1;
            const bool in_range = idx_next >= 0 && idx_next < seq_len && (idx_next >> 8) < p.max_blocks;
            if (in_range) page_next = __ldg(bt_row + (idx_next >> 8));
            // the rows of tile i+1 go in flight
            if (ok && i + 1 < n) load_tile(pt, codes + (buf ^ 1) * kTile, p.cache, tr);
            // tile i+2's codes replace tile i's (the loads above read the other buffer)
            if (pt < kTile && i + 2 < n) {
                int code = -1;
                if (in_range) {
                    if (page_next < 0 || static_cast<long long>(page_next) >= p.num_pages)
                        atomicOr(p.err, SMLA_FLAG_BAD_PAGE);
                    else
                        code = page_next * kPageTokens + (idx_next & (kPageTokens - 1));
                }
                codes[buf * kTile + pt] = code;
                const uint32_t bits = __ballot_sync(0xffffffffu, code >= 0);
                if (lane == 0) mask[((i + 2) & 3) * 4 + (pt >> 5)] = bits;
            }
            if (barrier_or(kBarIdProducer, kProducerThreads, !ok)) break;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const bool ok = !*abort_flag;

    // ---- epilogue: per-head sums (red holds them per TMEM quadrant), then O/l or the cluster merge
    float *l_head = head_alpha;
    if (tid < kHeads) l_head[tid] = (red[tid] + red[64 + tid]) + (red[128 + tid] + red[192 + tid]);
    __syncthreads();
    if (p.cluster_merge) {
        cluster_epilogue(p, b, ok, n, tid, warp, lane, tmem, smem, &bars[kBarXch], head_m, l_head, red);
    } else if (ok) {
        if (tid < kHeads) {
            const float l = l_head[tid];
            const float val = (l > 0.0f) ? (head_m[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
            if (p.nsplit == 1)
                p.lse[static_cast<size_t>(b) * kHeads + tid] = val;
            else
                p.part_lse[(static_cast<size_t>(b) * kHeads + tid) * p.nsplit + split] = val;
        }
        if (tid < kHeads) {
            const float l = l_head[tid];
            red[tid] = (l > 0.0f) ? 1.0f / l : 0.0f;  // 1/l per head
        }
        __syncthreads();
        if (warp < kSoftmaxWarps) {
            const int q = warp & 3;
            const int hh = warp >> 2;
            const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
            // the nsplit > 1 partials are [b][head][split][dim]
            const size_t head_stride = static_cast<size_t>(p.nsplit) * kDim;
            float *base = (p.nsplit == 1) ? p.out + static_cast<size_t>(b) * kHeads * kDim
                                          : p.part_o + static_cast<size_t>(b) * kHeads * head_stride + split * kDim;
#pragma unroll 1
            for (int part = 0; part < 8; ++part) {  // 4 chunks x 2 halves of 16 heads
                const int mc = part >> 1, h0 = 32 * hh + 16 * (part & 1);
                float o[16];
                if (n > 0) {
                    tmem_ld16(tmem + lane_base + 64 * mc + h0, o);
                    tmem_wait_ld();
                }
                float *dst = base + static_cast<size_t>(h0) * head_stride + 128 * mc + 32 * q + lane;
#pragma unroll
                for (int h = 0; h < 16; ++h) dst[h * head_stride] = (n > 0) ? o[h] * red[h0 + h] : 0.0f;
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

// Up to this many splits of a request merge inside a thread-block cluster (exchanging
// through the workspace, ordered by the cluster barrier); beyond it they go through
// normalised global partials and the merge kernel.
constexpr int kMaxClusterSplits = 4;

// Workspace after the header: nsplit == 1: nothing.  2..4 (cluster merge): the
// (m, l) rows [B][nsplit][128] f32, then the exchanged O^T chunks
// [B][4][nsplit-1][64][128] f32.  Above 4: part_lse [B][64][nsplit] f32, then
// part_o [B][64][nsplit][512] f32.
size_t workspace_for(int B, int topk, int nsplit) {
    size_t bytes = SMLA_WORKSPACE_HEADER;
    if (nsplit > kMaxClusterSplits) {
        const size_t rows = static_cast<size_t>(B) * SMLA_HEADS * nsplit;
        bytes += round256(rows * sizeof(float)) + rows * SMLA_DIM * sizeof(float);
    } else if (nsplit > 1) {
        bytes += round256(static_cast<size_t>(B) * nsplit * 128 * sizeof(float)) +
                 static_cast<size_t>(B) * 4 * (nsplit - 1) * 128 * SMLA_HEADS * sizeof(float);
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
    const size_t rows = (nsplit > kMaxClusterSplits) ? static_cast<size_t>(B) * SMLA_HEADS * nsplit
                                                             : static_cast<size_t>(B) * nsplit * 128;
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

