// smla.cu -- sparse MLA decode over an FP8 paged latent cache on B200 (sm_100a):
// the decode kernel (gather -> dequant -> tcgen05 QK^T -> fp32 online softmax ->
// tcgen05 PV -> split-K merge), the split-K LSE-merge kernel, the gather debug
// kernel and the C ABI declared in include/smla.h.
//
// Method ("The Turning Point: Architecting a Custom MMA Sparse-MLA Decode
// Kernel"): one program per (request, topk split) handles all 64 heads, so each
// gathered KV tile is read once for every head (Step 3), the two contractions
// run on tensor cores with fp32 accumulation, and split partials are merged by
// their log-sum-exp (Step 5).
//
// B200 mapping, per CTA (one per SM, 16 worker warps + 1 control warp):
//   * Q[b] (64 heads x 512, bf16) sits in shared memory (one TMA load) for the
//     whole kernel: every tile's score MMA reads it there.
//   * The worker warps hold the FP8 rows of the next 128-slot tile in registers
//     (16-byte loads) while the rows of the tile after it are already on their
//     way into L2 (bulk prefetches issued two tiles ahead), and dequantise a tile
//     into a bf16 [128 x 512] buffer in the 128-byte-swizzled layout the tensor
//     core reads, in two 256-dim halves as the previous tile's PV releases them.
//   * S^T[128 tokens x 64 heads] = K_tile . Q^T: tcgen05.mma M=128 N=64, fp32 in
//     tensor memory.  Tokens fill the 128-row M dimension, not the 64 heads.
//   * The worker warps then read S^T from tensor memory (one token lane and 16
//     heads per thread), raise the running max of a head only when a score passes
//     it by more than kRescaleThreshold (then O^T and the sums are rescaled in
//     tensor memory), and write P^T as two bf16 terms (P = P_hi + P_lo).
//   * O^T[512 x 64] += V^T . P^T with V = the same bf16 tile read MN-major: per
//     16-token step, dims chunks 0-1 take one N=128 MMA each over [P_hi | P_lo],
//     chunks 2-3 two N=64 MMAs each, so P carries ~16 significant bits (a single
//     bf16 P is not accurate enough when a few large latents dominate).
//   * The control warp owns tensor memory and the mbarriers, loads Q and issues
//     every MMA from one thread.
//   * The epilogue writes O/l and LSE = (m + log2 l) ln 2.  When the topk range of
//     a request is split in two, the two CTAs of a cluster swap their per-head
//     log-sum-exps and each adds its scaled O^T into the output (zeroed half by
//     each at entry) with fp32 atomic adds straight from tensor memory; more
//     splits, or a bf16 output, write fp32 partials that combine_kernel merges.
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

constexpr int kTile = 128;                     // topk slots per MMA tile (the M of S^T)
constexpr int kWorkerWarps = 16;               // gather, dequantisation, softmax, epilogue
constexpr int kWorkers = 32 * kWorkerWarps;    // 512
constexpr int kCtlWarp = kWorkerWarps;         // warp 16: tensor memory, mbarriers, TMA, MMA issue
constexpr int kThreads = kWorkers + 32;        // 544 threads: at most 120 registers each
constexpr int kGatherThreads = 256;            // threads of the gather debug kernel
constexpr uint32_t kBarIdWorkers = 1;          // named barrier of the 512 worker threads
constexpr int kWaiter = 32;                    // the worker that waits on behalf of all workers
// Two splits of a request merge inside the kernel (a CTA pair in one cluster, two terms
// per output element: the sum does not depend on their order); more go through global
// partials and the merge kernel, whose fixed order keeps the result reproducible.
constexpr int kMaxClusterSplits = 2;

// Dynamic shared memory map (bytes from a 1024-aligned base).
constexpr int kSmemQ = 0;                         // 64 KB: 8 K-blocks x [64 heads x 128 B], TMA-written
constexpr int kSmemKV = kSmemQ + 65536;           // 128 KB: 8 K-blocks x [128 tokens x 128 B]
constexpr int kSmemPhi = kSmemKV + 131072;        // 16 KB: P_hi^T [128 tokens x 64 heads] bf16
constexpr int kSmemPlo = kSmemPhi + 16384;        // 16 KB: P_lo^T
constexpr int kSmemCodes = kSmemPlo + 16384;      // [2][128] int32 token codes (tile ring)
constexpr int kSmemRed = kSmemCodes + 1024;       // [4][64] f32: per-quadrant maxima or sums; merge weights
constexpr int kSmemMask = kSmemRed + 1024;        // [4][4] u32: valid-token bits of a tile, ring of 4 tiles
constexpr int kSmemHeadM = kSmemMask + 64;        // [64] running max per head (log2 units)
constexpr int kSmemHeadAlpha = kSmemHeadM + 256;  // [64] rescale factor of the last max update; then the sums
constexpr int kSmemPeerLam = kSmemHeadAlpha + 256;  // [64] the other split's per-head log-sum-exp (2 splits)
constexpr int kSmemBars = kSmemPeerLam + 256;     // mbarriers (8 B each)

enum Bar : int {
    kBarQ = 0,          // Q landed (TMA transaction bytes)
    kBarKvFull = 1,     // + c (c = 0..3): dims chunk c of the tile written (16 worker-warp arrivals;
                        //   chunks 0-1 with the first 256-dim half, 2-3 with the second)
    kBarKvFree = 5,     // + c: PV chunk c of the tile done (MMA commit): chunk c may be overwritten
    kBarSFull = 9,      // + (i & 1): S^T of tile i complete (MMA commit; the two barriers alternate
                        //   over the tiles, each completing once every second tile)
    kBarPFull = 11,     // P^T written (16 worker-warp arrivals)
    kBarDrain = 12,     // final commit before tensor memory is released
    kBarSpare = 13,     // test hook target
    kBarMl = 14,        // pair merge: the peer's log-sum-exp row is in (256 transaction bytes)
    kNumBars = 15,
};
constexpr int kSmemTmemSlot = kSmemBars + kNumBars * 8;
constexpr int kSmemAbort = kSmemTmemSlot + 4;
constexpr int kSmemBytes = kSmemAbort + 4;
static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-block shared memory limit");
static_assert(kSmemBars % 8 == 0, "mbarriers need 8-byte alignment");

// Tensor memory (lane = dim of an O^T chunk, or token row of S^T and L; column = head):
//   [0, 256)   O^T dims chunks 0 and 1, 128 columns each: V^T.P_hi^T | V^T.P_lo^T
//              (one N = 128 MMA per step reads V^T once for both terms)
//   [256, 384) O^T dims chunks 2 and 3, 64 columns each: both terms accumulate in place
//   [384, 448) S^T of the current tile (dead before the next tile's QK^T is issued:
//              that waits for the dequantisation, which waits for this tile's PV)
//   [448, 512) per-lane running sums L
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO2 = 256;
constexpr uint32_t kTmemS = 384;
constexpr uint32_t kTmemL = 448;
constexpr uint32_t kIdescQK = idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16(128, 64, true, true);
constexpr uint32_t kIdescPV2 = idesc_bf16(128, 128, true, true);
// log2 units: the running max m of a head is raised (and O^T, the sums rescaled) only when a
// score exceeds it by more than this, so p = 2^(s - m) stays below 2^64.  P_hi + P_lo keep
// their relative precision at any magnitude, and fp32 sums of p x |v| over at most 2^16 slots
// stay finite for |v| < 2^48.  A high threshold makes the rescale (two CTA barriers and a
// pass over O^T in tensor memory) rare after the first tile, even when a few latents are
// much larger than the rest.
constexpr float kRescaleThreshold = 64.0f;

// The CTA's dynamic shared memory.  Every function addresses it through these
// accessors (constant offsets from the shared window), so no 64-bit pointer to
// shared memory has to live in a register.
extern __shared__ __align__(1024) uint8_t g_smem[];
__device__ __forceinline__ uint64_t *sm_bars() { return reinterpret_cast<uint64_t *>(g_smem + kSmemBars); }
__device__ __forceinline__ int *sm_codes() { return reinterpret_cast<int *>(g_smem + kSmemCodes); }
__device__ __forceinline__ uint32_t *sm_mask() { return reinterpret_cast<uint32_t *>(g_smem + kSmemMask); }
__device__ __forceinline__ float *sm_head_m() { return reinterpret_cast<float *>(g_smem + kSmemHeadM); }
__device__ __forceinline__ float *sm_head_alpha() { return reinterpret_cast<float *>(g_smem + kSmemHeadAlpha); }
__device__ __forceinline__ float *sm_red() { return reinterpret_cast<float *>(g_smem + kSmemRed); }
__device__ __forceinline__ volatile int *sm_abort() { return reinterpret_cast<volatile int *>(g_smem + kSmemAbort); }
__device__ __forceinline__ float *sm_peer_lam() { return reinterpret_cast<float *>(g_smem + kSmemPeerLam); }

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

// What the decode kernel writes, fixed at compile time so each instantiation carries only
// its own epilogue (and gets its own register allocation):
//   kEpiF32   fp32 O and LSE with one split; fp32 partials for the merge kernel with more
//   kEpiBf16  bf16 O (round to nearest even) and fp32 LSE, one split
//   kEpiPair  two splits in a CTA pair (cluster) adding into the fp32 output
enum Epilogue : int { kEpiF32 = 0, kEpiBf16 = 1, kEpiPair = 2 };

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
__device__ __forceinline__ bool wait_phase_poll(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                const DecodeParams &p, uint32_t backoff_ns) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t k = 1;; ++k) {
        if (backoff_ns) __nanosleep(backoff_ns);
        if (mbar_test_wait(bar, parity)) return true;
        if ((k & 31u) != 0) continue;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > p.timeout_ns) {
            *abort_flag = 1;
            atomicOr(p.err, SMLA_FLAG_TIMEOUT);
            return false;
        }
    }
}
__device__ __noinline__ bool wait_phase_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             const DecodeParams &p, uint32_t backoff_ns) {
    return wait_phase_poll(bar, parity, abort_flag, p, backoff_ns);
}
// The MMA-issuing thread spins (backoff 0); waiting worker threads back off between
// polls so they take few issue slots from the warps that share their scheduler.
constexpr uint32_t kWorkerBackoffNs = 32;
// kInline (here and in the functions below that take it): the rare paths -- the polling
// loop of a wait that does not complete at once, the rescale of the softmax -- inline, or
// as calls.  Measured per kernel on B200: the CTA-pair kernel runs faster with them inline
// (B=64 x topk 512: 26.7 vs 28.0 us), the single-split kernel with calls, whose smaller
// worker code spills less (B=256 x topk 512: 74.8 vs 76.8 us).
template <bool kInline>
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                           const DecodeParams &p, uint32_t backoff_ns = 0) {
    if (mbar_test_wait(bar, parity)) return true;
    if constexpr (kInline)
        return wait_phase_poll(bar, parity, abort_flag, p, backoff_ns);
    else
        return wait_phase_slow(bar, parity, abort_flag, p, backoff_ns);
}

// Warp-uniform version: lane 0 waits (acquire), the verdict is broadcast, and the warp
// synchronisation orders the other lanes after its observation.
template <bool kInline>
__device__ __forceinline__ bool warp_wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                const DecodeParams &p, int lane,
                                                uint32_t backoff_ns = kWorkerBackoffNs) {
    int ok = 1;
    if (lane == 0) ok = wait_phase<kInline>(bar, parity, abort_flag, p, backoff_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Worker-wide waits: one worker thread (in warp 1, so it does not share a scheduler
// with the MMA-issuing warp 16) waits on the mbarrier phase, with acquire semantics,
// while the other workers block in a named barrier; the barrier then orders every
// worker after that observation (the others do not poll the mbarrier word, which would
// serialise 512 accesses to one address).  `enabled` false skips the wait but keeps
// the barrier (every worker calls these with the same arguments).  Returns false if
// the wait failed or was skipped.
template <bool kInline>
__device__ __forceinline__ bool workers_wait(uint64_t *bar, uint32_t parity, const DecodeParams &p, int t,
                                             bool enabled = true, uint32_t backoff_ns = kWorkerBackoffNs,
                                             bool failed_before = false) {
    bool ok = enabled;
    if (t == kWaiter && enabled) ok = wait_phase<kInline>(bar, parity, sm_abort(), p, backoff_ns);
    return !barrier_or(kBarIdWorkers, kWorkers, !ok || failed_before);
}

// ------------------------------------------------------------------ gather + dequant
// A tile's 128 token rows are dealt out to the 512 worker threads t, 9 sixteen-byte
// chunks each, grouped by dims chunk c (dims [128c, 128c+128)):
//   chunks 0..2: nope chunk 8c + (t & 7) of the tokens (t >> 3) and (t >> 3) + 64
//   chunk 3:     nope chunk 24 + (t & 3) of the token t >> 2, and rope chunk
//                28 + (t & 7) of the tokens (t >> 3) and (t >> 3) + 64
// Consecutive threads take consecutive chunks of a token row (coalesced loads).
// A Slot holds those bytes and their UE8M0 scales in registers between the load and
// the dequantisation.
struct Slot {
    uint4 raw[3][2];  // nope chunks of dims chunks 0..2, tokens (t >> 3) + 64u
    uint4 rope[2];    // rope chunk of the same tokens
    uint4 nope3;      // nope chunk 24 + (t & 3) of token t >> 2
    uint2 srow[2];    // scale rows of tokens (t >> 3) + 64u
    uint32_t sc3;     // scale byte 6 of token t >> 2
};

// The loads of one dims chunk's items of a tile (part 0..3), so that a tile's rows can
// go in flight chunk by chunk as the registers of the previous tile's chunk free up.
// Part 2 also loads the scale rows (their last use is chunk 2), part 3 the rest.
__device__ __forceinline__ void load_part(int part, int t, const int *codes, const uint8_t *cache, Slot &s) {
    const int k8 = t & 7;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int code = codes[(t >> 3) + 64 * u];
        const uint8_t *row = token_row(cache, code >= 0 ? code : 0);
        if (part == 0) s.raw[0][u] = (code >= 0) ? ld_stream_v4(row + k8 * 16) : make_uint4(0u, 0u, 0u, 0u);
        if (part == 1) s.raw[1][u] = (code >= 0) ? ld_stream_v4(row + (8 + k8) * 16) : make_uint4(0u, 0u, 0u, 0u);
        if (part == 2) {
            s.raw[2][u] = (code >= 0) ? ld_stream_v4(row + (16 + k8) * 16) : make_uint4(0u, 0u, 0u, 0u);
            s.srow[u] = (code >= 0) ? ld_stream_v2(token_scales(cache, code)) : make_uint2(0u, 0u);
        }
        if (part == 3) s.rope[u] = (code >= 0) ? ld_stream_v4(row + (28 + k8) * 16) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (part == 3) {
        const int code3 = codes[t >> 2];
        s.nope3 = (code3 >= 0) ? ld_stream_v4(token_row(cache, code3) + (24 + (t & 3)) * 16) : make_uint4(0u, 0u, 0u, 0u);
        s.sc3 = (code3 >= 0) ? ld_stream_u8(token_scales(cache, code3) + 6) : 0u;
    }
}

__device__ __forceinline__ void load_slot(int t, const int *codes, const uint8_t *cache, Slot &s) {
    const int k8 = t & 7;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int code = codes[(t >> 3) + 64 * u];
        s.raw[0][u] = s.raw[1][u] = s.raw[2][u] = s.rope[u] = make_uint4(0u, 0u, 0u, 0u);
        s.srow[u] = make_uint2(0u, 0u);
        if (code >= 0) {
            const uint8_t *row = token_row(cache, code);
            s.raw[0][u] = ld_stream_v4(row + k8 * 16);
            s.raw[1][u] = ld_stream_v4(row + (8 + k8) * 16);
            s.raw[2][u] = ld_stream_v4(row + (16 + k8) * 16);
            s.rope[u] = ld_stream_v4(row + (28 + k8) * 16);
            s.srow[u] = ld_stream_v2(token_scales(cache, code));
        }
    }
    const int code3 = codes[t >> 2];
    s.nope3 = make_uint4(0u, 0u, 0u, 0u);
    s.sc3 = 0u;
    if (code3 >= 0) {
        s.nope3 = ld_stream_v4(token_row(cache, code3) + (24 + (t & 3)) * 16);
        s.sc3 = ld_stream_u8(token_scales(cache, code3) + 6);
    }
}

// Asks L2 to fetch a token's row and scale row ahead of the register loads.
__device__ __forceinline__ void prefetch_token_l2(const uint8_t *cache, int code) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], 576;" ::"l"(token_row(cache, code)) : "memory");
    asm volatile("prefetch.global.L2 [%0];" ::"l"(token_scales(cache, code)) : "memory");
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

// Dequantisation of tile i: each half of the dims is written as soon as the PV of tile
// i-1 has released it, and its registers then take the same dims' rows of tile i+1
// (`next`, null for the last tile): the load issue, which stalls while the memory
// pipeline is full, overlaps the waits for the PV instead of delaying the softmax.
template <bool kInline>
__device__ __forceinline__ bool dequant_tile(int i, int t, int lane, const DecodeParams &p, Slot &s,
                                             const int *next, bool &late_ok) {
    const uint32_t kv = smem_addr(g_smem + kSmemKV);
    uint64_t *bars = sm_bars();
    const int k8 = t & 7;
    // Two halves of 256 dims, each written in one go and published with one fence: half 0
    // (dims chunks 0-1) after a worker-wide wait on chunk 1's release (the PV commits
    // complete in issue order, so chunk 0 is free too; the barrier also orders the previous
    // step's writes of tile i+1's codes before every thread's loads below), half 1 (chunks
    // 2-3) after a warp-by-warp wait on chunk 3's.  A failed warp wait keeps the warp in
    // step (it still stores and publishes) and is folded into the next worker-wide wait,
    // where every worker sees it.  Fewer, larger hand-overs than one per 128-dim chunk: the
    // waits, fences and arrivals cost more than the later start of the first half.
    late_ok = true;
    if (i > 0 && !workers_wait<kInline>(&bars[kBarKvFree + 1], (i - 1) & 1, p, t)) return false;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int kb = 2 * c + (k8 >> 2);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint4 raw = (c == 0) ? s.raw[0][u] : s.raw[1][u];
            const uint32_t w = (kb < 4) ? s.srow[u].x : s.srow[u].y;
            store_item(kv, (t >> 3) + 64 * u, kb, 2 * (k8 & 3), true, raw, (w >> (8 * (kb & 3))) & 0xFFu);
        }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        mbar_arrive(&bars[kBarKvFull + 0]);
        mbar_arrive(&bars[kBarKvFull + 1]);
    }
    if (next) {
        load_part(0, t, next, p.cache, s);
        load_part(1, t, next, p.cache, s);
    }
    if (i > 0)
        late_ok = warp_wait_phase<kInline>(&bars[kBarKvFree + 3], (i - 1) & 1, sm_abort(), p, lane, 0u) && late_ok;
    {
        const int kb = 4 + (k8 >> 2);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint32_t w = (kb < 4) ? s.srow[u].x : s.srow[u].y;
            store_item(kv, (t >> 3) + 64 * u, kb, 2 * (k8 & 3), true, s.raw[2][u], (w >> (8 * (kb & 3))) & 0xFFu);
        }
    }
    store_item(kv, t >> 2, 6, 2 * (t & 3), true, s.nope3, s.sc3);
#pragma unroll
    for (int u = 0; u < 2; ++u) store_item(kv, (t >> 3) + 64 * u, 7, k8, false, s.rope[u], 0u);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        mbar_arrive(&bars[kBarKvFull + 2]);
        mbar_arrive(&bars[kBarKvFull + 3]);
    }
    if (next) {
        load_part(2, t, next, p.cache, s);
        load_part(3, t, next, p.cache, s);
    }
    return true;
}

// ------------------------------------------------------------------ MMA issue
// The tensor-core side of the pipeline, run by one thread of the control warp, with
// every descriptor in registers and each chunk's MMAs unrolled: a single thread issues
// all of them, so instructions between two MMAs directly slow the tensor core.  Every
// wait is bounded; a failed wait stops the issue.
//
// Descriptor words (128-byte swizzle, see sw128_desc): the high word holds SBO = 1024
// (8 rows of 128 bytes), the version and the swizzle mode; the low word holds the
// address (16-byte units) and LBO.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr, uint32_t lbo) {
    return ((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}

// S^T += K.Q^T over dims chunk cp: 2 K-blocks x 4 steps of K = 16 (the K rows are
// 128 bytes per K-block, K-blocks 16 KB apart; Q K-blocks 8 KB apart).
__device__ __forceinline__ void issue_qk_chunk(uint32_t d, uint32_t a_lo, uint32_t b_lo, bool first) {
    if (first)
        mma_bf16_ss(d, desc_from(a_lo, kDescHi), desc_from(b_lo, kDescHi), kIdescQK, 0u);
    else
        mma_bf16_ss_acc(d, desc_from(a_lo, kDescHi), desc_from(b_lo, kDescHi), kIdescQK);
#pragma unroll
    for (int k = 1; k < 8; ++k) {
        const uint32_t ao = (k >> 2) * ((kTile * 128) >> 4) + (k & 3) * 2;
        const uint32_t bo = (k >> 2) * (8192 >> 4) + (k & 3) * 2;
        mma_bf16_ss_acc(d, desc_from(a_lo + ao, kDescHi), desc_from(b_lo + bo, kDescHi), kIdescQK);
    }
}

// O^T chunk += V^T.P_hi^T + V^T.P_lo^T over the tile's 128 tokens: 8 steps of 16 tokens
// (2 KB apart in the MN-major V^T and P^T), two N = 64 MMAs per step.
__device__ __forceinline__ void issue_pv_chunk(uint32_t d, uint32_t a_lo, uint32_t bh_lo, uint32_t bl_lo,
                                               bool accumulate) {
    if (accumulate)
        mma_bf16_ss_acc(d, desc_from(a_lo, kDescHi), desc_from(bh_lo, kDescHi), kIdescPV);
    else
        mma_bf16_ss(d, desc_from(a_lo, kDescHi), desc_from(bh_lo, kDescHi), kIdescPV, 0u);
    mma_bf16_ss_acc(d, desc_from(a_lo, kDescHi), desc_from(bl_lo, kDescHi), kIdescPV);
#pragma unroll
    for (int ks = 1; ks < 8; ++ks) {
        const uint32_t o = ks * (2048 >> 4);
        mma_bf16_ss_acc(d, desc_from(a_lo + o, kDescHi), desc_from(bh_lo + o, kDescHi), kIdescPV);
        mma_bf16_ss_acc(d, desc_from(a_lo + o, kDescHi), desc_from(bl_lo + o, kDescHi), kIdescPV);
    }
}

// [O^T_hi | O^T_lo] chunk += V^T.[P_hi | P_lo]^T: one N = 128 MMA per step of 16 tokens,
// whose B operand is the two P^T arrays as two 64-column MN blocks 16 KB apart.
__device__ __forceinline__ void issue_pv_wide(uint32_t d, uint32_t a_lo, uint32_t b_lo, bool accumulate) {
    if (accumulate)
        mma_bf16_ss_acc(d, desc_from(a_lo, kDescHi), desc_from(b_lo, kDescHi), kIdescPV2);
    else
        mma_bf16_ss(d, desc_from(a_lo, kDescHi), desc_from(b_lo, kDescHi), kIdescPV2, 0u);
#pragma unroll
    for (int ks = 1; ks < 8; ++ks) {
        const uint32_t o = ks * (2048 >> 4);
        mma_bf16_ss_acc(d, desc_from(a_lo + o, kDescHi), desc_from(b_lo + o, kDescHi), kIdescPV2);
    }
}

// For each tile i: S^T = K.Q^T chunk by chunk as the workers publish the
// tile's dims chunks, then, once every worker has written P^T, O^T += V^T.P^T with a
// commit per 128-dim chunk (freeing that chunk of the tile buffer; in the last tile it
// makes that chunk of O^T final).
template <bool kInline>
__device__ __forceinline__ void mma_issue_loop(uint32_t tmem, const DecodeParams &p, int n) {
    uint64_t *bars = sm_bars();
    volatile int *abort_flag = sm_abort();
    const uint32_t kv = smem_addr(g_smem + kSmemKV);
    const uint32_t qk_a = desc_lo(kv, 16), qk_b = desc_lo(smem_addr(g_smem + kSmemQ), 16);
    const uint32_t pv_a = desc_lo(kv, kTile * 128);
    const uint32_t pv_bh = desc_lo(smem_addr(g_smem + kSmemPhi), 8192);
    const uint32_t pv_bl = desc_lo(smem_addr(g_smem + kSmemPlo), 8192);
    const uint32_t pv_b2 = desc_lo(smem_addr(g_smem + kSmemPhi), kSmemPlo - kSmemPhi);
    bool ok = true, spare_used = false;
    for (int i = 0; i < n && ok; ++i) {
        const uint32_t s_col = tmem + kTmemS;
#pragma unroll 1
        for (int cp = 0; cp < 4 && ok; ++cp) {
            ok = (i > 0 || cp > 0 || wait_phase<kInline>(&bars[kBarQ], 0, abort_flag, p)) &&
                 wait_phase<kInline>(&bars[kBarKvFull + cp], i & 1, abort_flag, p);
            if (!ok) break;
            tc_fence_after_sync();
            issue_qk_chunk(s_col, qk_a + cp * 2 * ((kTile * 128) >> 4), qk_b + cp * 2 * (8192 >> 4), cp == 0);
        }
        if (!ok) break;
        const bool hook = (i == 0) && (p.debug_flags & SMLA_DEBUG_SKIP_FIRST_COMMIT);
        mma_commit(hook ? &bars[kBarSpare] : &bars[kBarSFull + (i & 1)]);
        spare_used = spare_used || hook;
        ok = wait_phase<kInline>(&bars[kBarPFull], i & 1, abort_flag, p);
        if (!ok) break;
        tc_fence_after_sync();
#pragma unroll 1
        for (int mc = 0; mc < 2; ++mc) {
            issue_pv_wide(tmem + 128 * mc, pv_a + mc * 2 * ((kTile * 128) >> 4), pv_b2, i > 0);
            mma_commit(&bars[kBarKvFree + mc]);
        }
#pragma unroll 1
        for (int mc = 2; mc < 4; ++mc) {
            issue_pv_chunk(tmem + kTmemO2 + 64 * (mc - 2), pv_a + mc * 2 * ((kTile * 128) >> 4), pv_bh, pv_bl, i > 0);
            mma_commit(&bars[kBarKvFree + mc]);
        }
    }
    // every MMA issued must be complete before tensor memory is released
    if (spare_used) (void)mbar_wait(&bars[kBarSpare], 0, p.timeout_ns);
    mma_commit(&bars[kBarDrain]);
    (void)mbar_wait(&bars[kBarDrain], 0, p.timeout_ns);
}

// ------------------------------------------------------------------ worker state
// Per-thread view of the CTA for the worker warps.  Warp w reads tensor-memory lanes
// 32q.. (q = w & 3: the tokens 32q..32q+31 of S^T, or dims 32q.. of an O^T chunk)
// and the 16 heads 16hq.. (hq = w >> 2).
struct Worker {
    const DecodeParams &p;
    uint32_t tmem;
    int t, warp, lane, q, hq;
    uint32_t lane_base;

    // Softmax of tile i: p = 2^(s c - m) against the running max m, which is raised (with
    // a rescale of O^T and of the sums) only when a score exceeds it by more than
    // kRescaleThreshold; P^T is written as bf16 hi + lo terms.  The scores are read from
    // tensor memory once; the running sums, which the PV does not read, are updated
    // after P^T has been handed to the tensor core.
    template <bool kInline>
    __device__ __forceinline__ bool softmax(int i, bool failed_before = false) {
        // the tensor core is idle until P^T is written: wake up without backoff
        if (!workers_wait<kInline>(&sm_bars()[kBarSFull + (i & 1)], (i >> 1) & 1, p, t, true, 0u, failed_before))
            return false;
        tc_fence_after_sync();
        const float c = p.scale_log2;
        const bool valid = (sm_mask()[(i & 3) * 4 + q] >> lane) & 1u;
        const uint32_t s_col = tmem + lane_base + kTmemS + 16 * hq;
        const float *hm = sm_head_m() + 16 * hq;
        float x[16], mm[16];
        tmem_ld16(s_col, x);
        load16(hm, mm);
        tmem_wait_ld();
        // does any score exceed its head's running max by more than the threshold?
        bool over = false;
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            x[h] = valid ? x[h] * c : -INFINITY;
            over |= (x[h] - mm[h]) > kRescaleThreshold;
        }
        if (barrier_or(kBarIdWorkers, kWorkers, over)) {
            if constexpr (kInline)
                rescale(i, valid, s_col);
            else
                rescale_call(i, valid, s_col);
            load16(hm, mm);
        }
        // p = 2^(s c - m) (0 for a masked token); P^T row r as bf16 hi + lo
        const int r = 32 * q + lane;
        const uint32_t phi = smem_addr(g_smem + kSmemPhi), plo = smem_addr(g_smem + kSmemPlo);
#pragma unroll
        for (int h = 0; h < 16; ++h) x[h] = valid ? fast_exp2(x[h] - mm[h]) : 0.0f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a0 = x[8 * half + 2 * e], a1 = x[8 * half + 2 * e + 1];
                // hi = bf16(p), lo = bf16(p - hi) (p - hi is exact in fp32): |p - hi - lo| <= 2^-17 p
                hw[e] = pack_bf16x2(a0, a1);
                lw[e] = pack_bf16x2(a0 - __uint_as_float(hw[e] << 16), a1 - __uint_as_float(hw[e] & 0xFFFF0000u));
            }
            const uint32_t off = r * 128 + (((2 * hq + half) ^ (r & 7)) << 4);
            sts_v4(phi + off, make_uint4(hw[0], hw[1], hw[2], hw[3]));
            sts_v4(plo + off, make_uint4(lw[0], lw[1], lw[2], lw[3]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm_bars()[kBarPFull]);
        // running sums (per token lane and head) += p
        const uint32_t l_col = tmem + lane_base + kTmemL + 16 * hq;
        if (i > 0) {
            float l[16];
            tmem_ld16(l_col, l);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 16; ++h) x[h] += l[h];
        }
        tmem_st16(l_col, x);
        tmem_wait_st();
        return true;
    }

    // Raises each head's running max to max(m, tile max) and rescales what was
    // accumulated (O^T and the sums) by 2^(m_old - m_new).  Rare: the max moves only
    // past kRescaleThreshold, and on the first tile with a valid token.  rescale_call is
    // the same as an out-of-line call.
    __device__ __noinline__ void rescale_call(int i, bool valid, uint32_t s_col) { rescale(i, valid, s_col); }
    __device__ __forceinline__ void rescale(int i, bool valid, uint32_t s_col) {
        const float c = p.scale_log2;
        float y[16];
        tmem_ld16(s_col, y);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 16; ++h) y[h] = valid ? y[h] * c : -INFINITY;
        const float tmax = warp_transpose_reduce<true, 16>(y, lane);
        if ((lane & 1) == 0) sm_red()[q * 64 + 16 * hq + (lane >> 1)] = tmax;
        named_barrier_sync(kBarIdWorkers, kWorkers);
        if (t < kHeads) {
            const float *red = sm_red();
            const float tm = fmaxf(fmaxf(red[t], red[64 + t]), fmaxf(red[128 + t], red[192 + t]));
            const float mo = sm_head_m()[t];
            const float mn = fmaxf(mo, tm);
            sm_head_alpha()[t] = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
            sm_head_m()[t] = mn;
        }
        named_barrier_sync(kBarIdWorkers, kWorkers);
        if (i == 0) return;  // nothing accumulated yet
        // the PV of tile i-1 is complete (the S^T commit of tile i covers it): rescale the
        // six 64-column groups of O^T and the sums, unless none of this warp's 16 heads moved
        float al[16];
        load16(sm_head_alpha() + 16 * hq, al);
        bool moved = false;
#pragma unroll
        for (int h = 0; h < 16; ++h) moved |= al[h] != 1.0f;
        if (!moved) return;
#pragma unroll 1
        for (int mc = 0; mc < 7; ++mc) {
            const uint32_t col = tmem + lane_base + (mc < 6 ? 64 * mc : kTmemL) + 16 * hq;
            float o[16];
            tmem_ld16(col, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 16; ++h) o[h] *= al[h];
            tmem_st16(col, o);
        }
        tmem_wait_st();
    }

    // Per-head sums over all 128 token lanes into the head_alpha array (every worker calls it;
    // `have` is false when no tile was completed, the sums are then zero).
    __device__ __forceinline__ void reduce_sums(bool have) {
        float v[16];
        if (have) {
            tmem_ld16(tmem + lane_base + kTmemL + 16 * hq, v);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int h = 0; h < 16; ++h) v[h] = 0.0f;
        }
        const float s = warp_transpose_reduce<false, 16>(v, lane);
        if ((lane & 1) == 0) sm_red()[q * 64 + 16 * hq + (lane >> 1)] = s;
        named_barrier_sync(kBarIdWorkers, kWorkers);
        if (t < kHeads) sm_head_alpha()[t] = (sm_red()[t] + sm_red()[64 + t]) + (sm_red()[128 + t] + sm_red()[192 + t]);
        named_barrier_sync(kBarIdWorkers, kWorkers);
    }
};

// One step of the worker pipeline for tile i: dequantise it from the register slot while
// refilling the slot with tile i+1 (from L2: its rows were prefetched one step earlier,
// at kernel entry for tile 1), run the softmax of tile i, then translate tile i+2 and
// prefetch its rows.
// Translation runs two tiles ahead in stages so no thread waits on a dependent load:
// the topk index of a slot is loaded one step before its block-table entry, which is
// loaded before the token code is formed (threads t < 128 own slot t of every tile).
struct Translator {
    int idx_a = -1;   // topk index of slot t of tile i+2
    int idx_b = -1;   // of tile i+3
    int page_a = -1;  // block-table entry for idx_a
};

__device__ __forceinline__ int slot_index(const DecodeParams &p, int t_begin, int tile, int t) {
    return (t_begin + tile) * kTile + t;
}

template <bool kInline>
__device__ __forceinline__ bool worker_step(Worker &w, int i, int n, int t_begin, int seq_len, const int32_t *bt_row,
                                            const int32_t *idx_row, Translator &tr, Slot &cur) {
    const DecodeParams &p = w.p;
    const int t = w.t;
    if (t < kTile && i + 2 < n) {
        tr.page_a = slot_in_range(tr.idx_a, seq_len, p.max_blocks) ? __ldg(bt_row + (tr.idx_a >> 8)) : -1;
        const int s3 = slot_index(p, t_begin, i + 3, t);
        tr.idx_b = (i + 3 < n && s3 < p.topk) ? __ldg(idx_row + s3) : -1;
    }
    const int *next = (i + 1 < n) ? sm_codes() + ((i + 1) & 1) * kTile : nullptr;
    bool late_ok;
    if (!dequant_tile<kInline>(i, t, w.lane, p, cur, next, late_ok)) return false;  // uniform over the workers
    if (!w.softmax<kInline>(i, !late_ok)) return false;                           // uniform too
    if (t < kTile && i + 2 < n) {
        // tile i's codes are dead (its rows were loaded one step ago): tile i+2 takes the buffer
        const int code = slot_in_range(tr.idx_a, seq_len, p.max_blocks)
                             ? slot_code(tr.idx_a, tr.page_a, p.num_pages, p.err)
                             : -1;
        sm_codes()[(i & 1) * kTile + t] = code;
        const uint32_t bits = __ballot_sync(0xffffffffu, code >= 0);
        if (w.lane == 0) sm_mask()[((i + 2) & 3) * 4 + (t >> 5)] = bits;
        if (code >= 0) prefetch_token_l2(p.cache, code);
    }
    tr.idx_a = tr.idx_b;
    return true;
}

// ------------------------------------------------------------------ epilogues
// This lane's dim of O^T dims chunk c for the 16 heads 16hq..: chunks 0 and 1 keep the
// P_hi and P_lo products in separate halves, added here.
__device__ __forceinline__ void load_o16(uint32_t lane_addr, int c, int hq, float (&v)[16]) {
    if (c < 2) {
        float lo[16];
        tmem_ld16(lane_addr + 128 * c + 16 * hq, v);
        tmem_ld16(lane_addr + 128 * c + 64 + 16 * hq, lo);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 16; ++h) v[h] += lo[h];
    } else {
        tmem_ld16(lane_addr + kTmemO2 + 64 * (c - 2) + 16 * hq, v);
        tmem_wait_ld();
    }
}

// Writes dims chunk c of this CTA's O^T, each head h scaled by scale[h] (16 heads 16hq..,
// in registers), to dst + h * head_stride + 128c + dim.  Lane l of warp (q, hq) holds dim
// 32q + l of its 16 heads, so each store or atomic add of a head covers 32 consecutive
// floats per warp (128 bytes, coalesced) without staging through shared memory, whose
// bandwidth the tensor core is using meanwhile.  What is written: kChunkTmem the scaled
// O^T, kChunkZero zeros (no tile, or weight 0), kChunkNan NaN (a failed wait: the result
// is invalid).
enum ChunkSource : int { kChunkNan = 0, kChunkZero = 1, kChunkTmem = 2 };
__device__ __forceinline__ uint16_t to_bf16_rn(float x) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}
// kMode: kStoreF32 plain fp32 stores, kAddF32 atomic adds, kStoreBf16 bf16 stores.
enum StoreMode : int { kStoreF32 = 0, kAddF32 = 1, kStoreBf16 = 2 };
template <int kMode>
__device__ __forceinline__ void write_chunk(const Worker &w, int c, const float (&scale)[16], void *dst,
                                            size_t head_stride, int source) {
    float v[16];
    if (source == kChunkTmem) load_o16(w.tmem + w.lane_base, c, w.hq, v);
    const size_t off = static_cast<size_t>(16 * w.hq) * head_stride + 128 * c + 32 * w.q + w.lane;
#pragma unroll
    for (int h = 0; h < 16; ++h) {
        const float x = (source == kChunkTmem) ? v[h] * scale[h] : (source == kChunkZero) ? 0.0f : NAN;
        if (kMode == kStoreBf16)
            static_cast<uint16_t *>(dst)[off + h * head_stride] = to_bf16_rn(x);
        else if (kMode == kAddF32)
            asm volatile("red.global.add.f32 [%0], %1;" ::"l"(static_cast<float *>(dst) + off + h * head_stride), "f"(x)
                         : "memory");
        else
            static_cast<float *>(dst)[off + h * head_stride] = x;
    }
}

template <int kEpi>
__device__ __forceinline__ void epilogue_direct(Worker &w, int b, int split, int n, bool ok) {
    const DecodeParams &p = w.p;
    if (n > 0) ok = workers_wait<false>(&sm_bars()[kBarKvFree + 3], (n - 1) & 1, p, w.t, ok);
    float *inv = sm_red();
    if (w.t < kHeads) {
        const float l = sm_head_alpha()[w.t];
        const float val = !ok ? NAN : (l > 0.0f) ? (sm_head_m()[w.t] + log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (p.nsplit == 1)
            p.lse[static_cast<size_t>(b) * kHeads + w.t] = val;
        else
            p.part_lse[(static_cast<size_t>(b) * kHeads + w.t) * p.nsplit + split] = val;
        inv[w.t] = !ok ? NAN : (l > 0.0f) ? 1.0f / l : 0.0f;
    }
    named_barrier_sync(kBarIdWorkers, kWorkers);
    // the nsplit > 1 partials are [b][head][split][dim] fp32; one split writes out (fp32 or bf16)
    const size_t head_stride = static_cast<size_t>(p.nsplit) * kDim;
    constexpr bool bf16 = kEpi == kEpiBf16;
    void *base = (p.nsplit > 1) ? static_cast<void *>(p.part_o + static_cast<size_t>(b) * kHeads * head_stride +
                                                      split * kDim)
                 : bf16 ? static_cast<void *>(reinterpret_cast<uint16_t *>(p.out) + static_cast<size_t>(b) * kHeads * kDim)
                        : static_cast<void *>(p.out + static_cast<size_t>(b) * kHeads * kDim);
    float sc[16];
    load16(inv + 16 * w.hq, sc);
    const int source = !ok ? kChunkNan : (n > 0) ? kChunkTmem : kChunkZero;
    if constexpr (bf16) {
#pragma unroll 1
        for (int mc = 0; mc < 4; ++mc) write_chunk<kStoreBf16>(w, mc, sc, base, head_stride, source);
    } else {
#pragma unroll 1
        for (int mc = 0; mc < 4; ++mc) write_chunk<kStoreF32>(w, mc, sc, base, head_stride, source);
    }
}

// nsplit = 2 in one cluster.  With lambda_s = m_s + log2 l_s (the log-sum-exp of split s
// in log2 units) and L = log2(2^lambda_0 + 2^lambda_1), the merged output is
// O = sum_s 2^(lambda_s - L) O^T_s / l_s and LSE = L ln 2 (the split-K log-sum-exp
// merge).  Each CTA sends its 64 lambdas to the other (asynchronous stores into a row
// kept for them, counted as transaction bytes on the receiver's mbarrier), and, chunk
// by chunk as its last PV finishes, adds its scaled O^T into the output, which both
// CTAs zeroed half of at entry (two terms: the sum does not depend on their order).
__device__ __forceinline__ void epilogue_pair(Worker &w, int b, int n, bool ok) {
    const DecodeParams &p = w.p;
    const int me = static_cast<int>(cluster_ctarank());
    const int t = w.t;
    uint64_t *bars = sm_bars();
    float lam = NAN;
    if (t < kHeads) {
        const float l = sm_head_alpha()[t];
        lam = !ok ? NAN : (n > 0 && l > 0.0f) ? sm_head_m()[t] + log2f(l) : -INFINITY;
        const uint32_t dst = map_to_rank(sm_peer_lam() + t, me ^ 1);
        const uint32_t bar = map_to_rank(&bars[kBarMl], me ^ 1);
        asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(dst),
                     "r"(__float_as_uint(lam)), "r"(bar)
                     : "memory");
    }
    const bool got = workers_wait<true>(&bars[kBarMl], 0, p, t);
    float *scale = sm_red();
    if (t < kHeads) {
        const float other = got ? sm_peer_lam()[t] : NAN;
        const float mx = fmaxf(lam, other);
        const bool bad = isnan(lam) || isnan(other);
        const float L = (mx == -INFINITY) ? -INFINITY : mx + log2f(exp2f(lam - mx) + exp2f(other - mx));
        const float l = sm_head_alpha()[t];
        scale[t] = bad ? NAN : (lam == -INFINITY) ? 0.0f : exp2f(lam - L) / l;
        if (me == 0) p.lse[static_cast<size_t>(b) * kHeads + t] = bad ? NAN : L * 0.69314718055994531f;
    }
    named_barrier_sync(kBarIdWorkers, kWorkers);
    float sc[16];
    load16(scale + 16 * w.hq, sc);
    float *base = p.out + static_cast<size_t>(b) * kHeads * kDim;
    // the two CTAs add into the same output, in chunk orders two chunks apart, so that
    // their atomic adds do not meet on the same lines at the same time
#pragma unroll 1
    for (int k = 0; k < 4; ++k) {
        const int c = (k + 2 * me) & 3;
        const bool chunk_ok = workers_wait<true>(&bars[kBarKvFree + c], (n - 1) & 1, p, t, ok && n > 0);
        // a split without tiles adds zeros; a failed wait NaN
        const int source = chunk_ok ? kChunkTmem : (ok && n == 0) ? kChunkZero : kChunkNan;
        write_chunk<kAddF32>(w, c, sc, base, kDim, source);
    }
}

// ------------------------------------------------------------------ the decode kernel
// One CTA per (topk split, request).  The 16 worker warps move one 128-slot tile at a
// time through dequantisation and softmax while the rows of the next two tiles are in
// flight; the control warp issues the MMAs (S^T of tile i as its dims chunks land,
// PV of tile i once P^T is written, each PV chunk releasing that chunk of the tile
// buffer to the next tile's dequantisation).
template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_q) {
    constexpr bool kPair = kEpi == kEpiPair;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int split = blockIdx.x;
    const int b = blockIdx.y;

    // The shared-memory tiles need a 1024-byte aligned base (128-byte swizzle atoms).  The
    // dynamic shared memory base is the same for every CTA of the launch, so this exit is
    // taken by all CTAs or none.
    if (smem_addr(g_smem) & 1023u) {
        if (tid == 0) atomicOr(p.err, SMLA_FLAG_SMEM);
        // the result is invalid: NaN where this CTA's output goes (the merge kernel turns a
        // NaN partial log-sum-exp into NaN rows)
        if (kPair || p.nsplit == 1) {
            for (int k = tid; k < kHeads * kDim; k += kThreads) {
                if (kEpi == kEpiBf16)
                    reinterpret_cast<uint16_t *>(p.out)[static_cast<size_t>(b) * kHeads * kDim + k] = 0x7FC0u;
                else
                    p.out[static_cast<size_t>(b) * kHeads * kDim + k] = NAN;
            }
            if (tid < kHeads) p.lse[static_cast<size_t>(b) * kHeads + tid] = NAN;
        } else if (tid < kHeads) {
            p.part_lse[(static_cast<size_t>(b) * kHeads + tid) * p.nsplit + split] = NAN;
        }
        // a CTA of a pair still takes part in both cluster barriers, so its peer (which
        // takes this same exit: every CTA of a launch has the same shared-memory base)
        // never waits on it
        if constexpr (kPair) {
            cluster_arrive();
            cluster_wait();
            cluster_arrive();
            cluster_wait();
        }
        return;
    }
    uint64_t *bars = sm_bars();
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(g_smem + kSmemTmemSlot);
    int *codes = sm_codes();
    uint32_t *mask = sm_mask();
    float *head_m = sm_head_m();

    const int num_tiles = (p.topk + kTile - 1) / kTile;
    const int t_begin = split * p.tiles_per_split;
    const int n = max(0, min(num_tiles, t_begin + p.tiles_per_split) - t_begin);
    const int seq_len = __ldg(p.seq_lens + b);
    const int32_t *bt_row = p.block_table + static_cast<size_t>(b) * p.max_blocks;
    const int32_t *idx_row = p.topk_idx + static_cast<size_t>(b) * p.topk;

    // ---- setup
    Translator tr;
    if (warp == kCtlWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
        if (lane == 0) {
            mbar_init(&bars[kBarQ], 1);
            for (int c = 0; c < 4; ++c) {
                mbar_init(&bars[kBarKvFull + c], kWorkerWarps);
                mbar_init(&bars[kBarKvFree + c], 1);
            }
            mbar_init(&bars[kBarSFull], 1);
            mbar_init(&bars[kBarSFull + 1], 1);
            mbar_init(&bars[kBarPFull], kWorkerWarps);
            mbar_init(&bars[kBarDrain], 1);
            mbar_init(&bars[kBarSpare], 1);
            mbar_init(&bars[kBarMl], 1);
            // the peer's row of 64 log-sum-exps arrives as 256 transaction bytes
            if (kPair) mbar_arrive_expect_tx(&bars[kBarMl], kHeads * 4);
            fence_barrier_init();
            *sm_abort() = 0;
            mbar_arrive_expect_tx(&bars[kBarQ], kHeads * kDim * 2);
#pragma unroll
            for (int kb = 0; kb < 8; ++kb) tma_load_2d(g_smem + kSmemQ + kb * 8192, &tmap_q, 64 * kb, kHeads * b, &bars[kBarQ]);
        }
    } else if (tid < 2 * kTile) {
        // index translation of tiles 0 and 1 (worker t: tile t / 128, slot t % 128)
        const int ti = tid >> 7;
        const int s = slot_index(p, t_begin, ti, tid & (kTile - 1));
        int code = -1;
        if (ti < n && s < p.topk)
            code = translate_slot(bt_row, p.max_blocks, seq_len, p.num_pages, __ldg(idx_row + s), p.err);
        codes[tid] = code;
        const uint32_t bits = __ballot_sync(0xffffffffu, code >= 0);
        if (lane == 0) mask[ti * 4 + ((tid >> 5) & 3)] = bits;
        if (tid < kTile && n > 2) {
            const int s2 = slot_index(p, t_begin, 2, tid);
            tr.idx_a = (s2 < p.topk) ? __ldg(idx_row + s2) : -1;
        }
    }
    if (tid < kHeads) head_m[tid] = -INFINITY;
    if constexpr (kPair) {
        // two splits add their weighted partials into the output: each CTA zeroes 32 heads of
        // out[b] now; the barriers below order these stores before either CTA's additions
        float4 *z = reinterpret_cast<float4 *>(p.out + (static_cast<size_t>(b) * kHeads + 32 * split) * kDim);
        for (int k = tid; k < 32 * kDim / 4; k += kThreads) z[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if constexpr (kPair) cluster_arrive();  // peers may address this CTA's mbarriers from now on
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == kCtlWarp) {
        // ================================================================ MMA issue
        if (lane == 0 && n > 0) mma_issue_loop<kPair>(tmem, p, n);
        __syncwarp();
        if constexpr (kPair) cluster_wait();
    } else {
        // ================================================================ workers
        Worker w{p, tmem, tid, warp, lane, warp & 3, warp >> 2, static_cast<uint32_t>(32 * (warp & 3)) << 16};
        Slot slot;
        if (n > 0) load_slot(tid, codes, p.cache, slot);
        // tile 1's rows head for L2 right behind tile 0's (its register loads come later)
        if (tid >= kTile && tid < 2 * kTile && codes[tid] >= 0) prefetch_token_l2(p.cache, codes[tid]);
        for (int i = 0; i < n && ok; ++i)
            ok = worker_step<kPair>(w, i, n, t_begin, seq_len, bt_row, idx_row, tr, slot);
        ok = ok && !*sm_abort();
        ok = !barrier_or(kBarIdWorkers, kWorkers, !ok);
        w.reduce_sums(ok && n > 0);
        if constexpr (kPair) {
            cluster_wait();  // the peer has initialised its mbarriers and zeroed its half of out
            epilogue_pair(w, b, n, ok);
        } else {
            epilogue_direct<kEpi>(w, b, split, n, ok);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (kPair) {
        // no CTA leaves while a peer may still write into its shared memory
        cluster_arrive();
        cluster_wait();
    }
    if (warp == kCtlWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Split-K merge: one CTA of 128 threads per (b, h), 4 output dims per thread.
__device__ __forceinline__ void store_row4(void *out, size_t bh, int tid, float4 v, int out_bf16) {
    if (out_bf16) {
        const uint32_t lo = to_bf16_rn(v.x) | (static_cast<uint32_t>(to_bf16_rn(v.y)) << 16);
        const uint32_t hi = to_bf16_rn(v.z) | (static_cast<uint32_t>(to_bf16_rn(v.w)) << 16);
        reinterpret_cast<uint2 *>(static_cast<uint16_t *>(out) + bh * kDim)[tid] = make_uint2(lo, hi);
    } else {
        reinterpret_cast<float4 *>(static_cast<float *>(out) + bh * kDim)[tid] = v;
    }
}

__global__ void __launch_bounds__(128) combine_kernel(const float *__restrict__ part_o,
                                                      const float *__restrict__ part_lse, void *__restrict__ out,
                                                      float *__restrict__ lse, int nsplit, int out_bf16) {
    const size_t bh = blockIdx.x;
    const int tid = threadIdx.x;
    const float *L = part_lse + bh * nsplit;
    float lmax = -INFINITY;
    bool invalid = false;  // a NaN partial LSE marks a split whose CTA aborted
    for (int s = 0; s < nsplit; ++s) {
        const float ls = __ldg(L + s);
        invalid = invalid || isnan(ls);
        lmax = fmaxf(lmax, ls);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (invalid) {
        store_row4(out, bh, tid, make_float4(NAN, NAN, NAN, NAN), out_bf16);
        if (tid == 0) lse[bh] = NAN;
        return;
    }
    if (lmax == -INFINITY) {
        store_row4(out, bh, tid, acc, out_bf16);
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
    store_row4(out, bh, tid, acc, out_bf16);
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
            (cudaFuncSetAttribute(smla::decode_kernel<smla::kEpiF32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smla::kSmemBytes) != cudaSuccess ||
             cudaFuncSetAttribute(smla::decode_kernel<smla::kEpiBf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smla::kSmemBytes) != cudaSuccess ||
             cudaFuncSetAttribute(smla::decode_kernel<smla::kEpiPair>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smla::kSmemBytes) != cudaSuccess))
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

// Two splits of a request merge inside the decode kernel (a CTA pair: the log-sum-exp
// rows cross through distributed shared memory, the fp32 outputs are added into out);
// more, or a bf16 output, go through normalised global partials and the merge kernel.
//
// Workspace after the header: nsplit == 1: nothing.  nsplit >= 2: part_lse [B][64][nsplit]
// f32, then part_o [B][64][nsplit][512] f32 (unused by the fp32 pair merge).
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
                           static_cast<cudaStream_t>(stream)>>>(part_o, part_lse, out, lse, nsplit, 0);
    return cudaGetLastError() == cudaSuccess ? SMLA_OK : SMLA_ERR_LAUNCH;
}

int smla_decode_ex(const void *q, const uint8_t *kv_cache, const int32_t *block_table, const int32_t *topk_idx,
                   const int32_t *seq_lens, float sm_scale, void *out, float *lse, int B, int H, int topk,
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
    p.out = static_cast<float *>(out);
    const bool out_bf16 = opts && opts->out_bf16;
    p.lse = lse;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    p.err = reinterpret_cast<uint32_t *>(ws);
    if (nsplit > 1) {
        const size_t rows = static_cast<size_t>(B) * SMLA_HEADS * nsplit;
        p.part_lse = reinterpret_cast<float *>(ws + SMLA_WORKSPACE_HEADER);
        p.part_o = reinterpret_cast<float *>(ws + SMLA_WORKSPACE_HEADER + round256(rows * sizeof(float)));
    }
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
    // two splits merge inside the kernel (fp32 output); more, or a bf16 output with splits,
    // go through fp32 partials and the merge kernel
    const bool pair = nsplit > 1 && nsplit <= smla::kMaxClusterSplits && !out_bf16;
    const int epi = pair ? smla::kEpiPair : (out_bf16 && nsplit == 1) ? smla::kEpiBf16 : smla::kEpiF32;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(nsplit, B);
    cfg.blockDim = dim3(smla::kThreads);
    cfg.dynamicSmemBytes = smla::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pair ? nsplit : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t launched =
        epi == smla::kEpiPair   ? cudaLaunchKernelEx(&cfg, smla::decode_kernel<smla::kEpiPair>, p, tmap_q)
        : epi == smla::kEpiBf16 ? cudaLaunchKernelEx(&cfg, smla::decode_kernel<smla::kEpiBf16>, p, tmap_q)
                                : cudaLaunchKernelEx(&cfg, smla::decode_kernel<smla::kEpiF32>, p, tmap_q);
    if (launched != cudaSuccess) return SMLA_ERR_LAUNCH;
    if (cudaGetLastError() != cudaSuccess) return SMLA_ERR_LAUNCH;
    if (nsplit > 1 && !pair) {
        smla::combine_kernel<<<static_cast<unsigned>(B) * SMLA_HEADS, 128, 0, st>>>(p.part_o, p.part_lse, out, lse,
                                                                                   nsplit, out_bf16 ? 1 : 0);
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

