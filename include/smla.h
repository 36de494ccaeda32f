/*
 * smla.h -- C ABI of libsmla.so: sparse Multi-head Latent Attention decode over an
 * FP8 paged latent cache, for NVIDIA B200 (sm_100a).
 *
 * The operation (source blog pages, cited by title and section):
 *   "The Turning Point: Architecting a Custom MMA Sparse-MLA Decode Kernel",
 *   Step 1 and Output Knowledge item 2: each of B decode queries has H = 64 bf16
 *   heads of a 512-d latent (448 "nope" + 64 "rope"); all heads attend over one
 *   shared latent KV head gathered at topk sparse token positions; the step
 *   dequantises, concatenates, multiplies, takes the softmax and returns the
 *   softmax-weighted latent O[B,H,512] and the log-sum-exp LSE[B,H].
 *   Step 5: split-K over the topk dimension with partial (O, LSE) merged by the
 *   standard online-softmax combine.
 *   "The Validation Gate: Writing a Standalone Correctness Test ...", section
 *   "The Test Design": the cache byte layout below.
 *   "The Validation Moment", smoke-test section: the page indexing logic.
 *
 * Cache layout (uint8, [num_pages][149504]): page p starts at p*149504; token
 * slot t of the page has its 576-byte row at +t*576 (448 e4m3 nope bytes, then
 * 64 little-endian bf16 rope values) and its 8-byte scale row at
 * +147456+t*8 (UE8M0 bytes for nope dims [64g,64g+64), g = 0..6; byte 7 unused).
 * Nope value d = e4m3(byte d) * 2^(scale[d/64] - 127).
 *
 * Slot validity: topk slot i of request b, idx = topk_idx[b][i], is valid iff
 * 0 <= idx < seq_lens[b], idx/256 < max_blocks and page = block_table[b][idx/256]
 * lies in [0, num_pages).  Invalid slots (the -1 padding among them) contribute
 * nothing.  A request with no valid slot gets O = 0 and LSE = -inf.  Duplicate
 * indices count with multiplicity.  LSE = ln sum_j exp(sm_scale * <q, k_j>).
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers must be device memory of the current
 *     device; the caller owns all memory.  The library never allocates or frees
 *     memory and never synchronises (except smla_read_error), so smla_decode can
 *     be captured in a CUDA graph.
 *   - "stream" is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - All arrays are dense and row-major.  kv_cache must be 16-byte aligned,
 *     q/out 16-byte aligned, the int32 arrays 4-byte aligned.
 *   - Return value: SMLA_OK, or a negative SMLA_ERR_* code; on error nothing is
 *     launched.
 *   - Problems found on the device (a block-table entry outside [0,num_pages), a
 *     wait that ran out) do not fault: the affected token is masked, or the CTA
 *     gives up and writes NaN into its requests' rows of out and lse (so the result
 *     is visibly invalid even if the error word is never read), and a bit is set in
 *     the sticky error word at the start of the workspace, read (and cleared) with
 *     smla_read_error.
 *   - Input domain: the cache holds no e4m3 NaN codes (0x7F/0xFF); dequantised
 *     nope values are exact in bf16 for scale bytes 10..254 as long as they lie
 *     in the bf16 range (larger ones become +-inf; scale bytes below 10 can round
 *     values below 2^-126); a 0xFF scale byte yields NaN.
 */
#ifndef SMLA_H
#define SMLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SMLA_OK 0
#define SMLA_ERR_INVALID (-1)   /* bad argument: null pointer, H != 64, sizes, alignment, workspace */
#define SMLA_ERR_DEVICE (-2)    /* current device is not sm_100 (B200 class) */
#define SMLA_ERR_CUDA (-3)      /* a CUDA runtime call failed */
#define SMLA_ERR_LAUNCH (-4)    /* kernel launch failed */
#define SMLA_ERR_SCRATCH (-5)   /* smla_decode_noalloc: the call needs more than SMLA_STATIC_SCRATCH_BYTES */

/* Bits of the device error word. */
#define SMLA_FLAG_BAD_PAGE 0x1u  /* a block-table entry outside [0, num_pages) was met and masked */
#define SMLA_FLAG_TIMEOUT 0x2u   /* a pipeline wait ran out of time; that CTA's out/lse rows are NaN */
#define SMLA_FLAG_SMEM 0x4u      /* dynamic shared memory was not 1024-byte aligned; rows are NaN */

#define SMLA_HEADS 64
#define SMLA_DIM 512
#define SMLA_PAGE_TOKENS 256
#define SMLA_PAGE_BYTES 149504
#define SMLA_MAX_TOPK 65536
#define SMLA_WORKSPACE_HEADER 256

/* Tuning and test options for smla_decode_ex.  Zero-initialise for defaults. */
typedef struct smla_options {
    int nsplit;                  /* topk splits per request; 0 = built-in heuristic */
    int out_bf16;                /* 0: out is fp32; 1: out is bf16 (see smla_decode_ex) */
    uint64_t wait_timeout_ns;    /* bound on every in-kernel wait; 0 = 1 s */
    uint32_t debug_flags;        /* test hooks, 0 in normal use (see SMLA_DEBUG_*) */
    uint32_t reserved1;
} smla_options;

/* Test hook: the first score MMA batch signals a spare barrier instead of the one
 * the CTA waits on, so that wait runs out; the CTA then drains its MMAs through
 * the spare barrier, releases its tensor memory, sets SMLA_FLAG_TIMEOUT and exits. */
#define SMLA_DEBUG_SKIP_FIRST_COMMIT 0x1u

/*
 * smla_decode -- one sparse MLA decode step.
 *   q           device, bf16 [B][H][512]
 *   kv_cache    device, uint8 [num_pages][149504] (layout above)
 *   block_table device, int32 [B][max_blocks], logical block -> physical page
 *   topk_idx    device, int32 [B][topk], logical token indices (-1 = padding)
 *   seq_lens    device, int32 [B]
 *   sm_scale    softmax scale applied to q.k
 *   out         device, fp32 [B][H][512]   (written)
 *   lse         device, fp32 [B][H]        (written, natural log)
 *   H must be 64; 1 <= topk <= SMLA_MAX_TOPK; B >= 1; max_blocks >= 1;
 *   1 <= num_pages < 2^23.
 *   workspace   device scratch of at least smla_workspace_bytes(B, H, topk)
 *               bytes, 256-byte aligned.  Its first 4 bytes are the sticky error
 *               word: zero it once (cudaMemset or smla_read_error) before first use.
 *               The rest holds the split-K partials of a call that splits a request
 *               (between the decode and the merge kernel: 3 or more parts, or a
 *               bf16 output); concurrent calls must not share a workspace.
 * Launches the decode kernel on `stream`.  A request whose topk range is split
 * in 2 parts is merged inside the kernel by its CTA pair (one thread-block
 * cluster: each adds its weighted part into out, two terms, so the result does
 * not depend on their order); with 3 or more parts the combine kernel follows
 * (a fixed summation order).  Results are reproducible bit for bit.
 */
int smla_decode(const void *q, const uint8_t *kv_cache, const int32_t *block_table, const int32_t *topk_idx,
                const int32_t *seq_lens, float sm_scale, float *out, float *lse, int B, int H, int topk,
                int max_blocks, int num_pages, void *workspace, size_t workspace_bytes, void *stream);

/* smla_decode with explicit options (opts may be NULL).  With opts->nsplit set,
 * the workspace must hold smla_workspace_bytes_ex(B, H, topk, opts->nsplit).
 * With opts->out_bf16 = 1, out is bf16 [B][H][512] (16-byte aligned): the fp32
 * result rounded to nearest even (|dO| up to 2^-9 |O| more than the fp32 output;
 * the pages give no bf16 tolerance), lse stays fp32.  A split request then merges
 * through the merge kernel (fp32 partials, one bf16 rounding), never through
 * atomic adds, so the result stays reproducible. */
int smla_decode_ex(const void *q, const uint8_t *kv_cache, const int32_t *block_table, const int32_t *topk_idx,
                   const int32_t *seq_lens, float sm_scale, void *out, float *lse, int B, int H, int topk,
                   int max_blocks, int num_pages, void *workspace, size_t workspace_bytes,
                   const smla_options *opts, void *stream);

/*
 * smla_combine -- split-K LSE merge ("The Turning Point", Step 5):
 *   L = ln sum_s exp(L_s),  O = sum_s exp(L_s - L) * O_s,
 * splits with L_s = -inf weigh 0; if all are -inf, O = 0 and L = -inf.
 *   part_o   device, fp32 [B][H][nsplit][512] normalised partial outputs
 *   part_lse device, fp32 [B][H][nsplit] partial log-sum-exps (natural log)
 *   out, lse device, fp32 [B][H][512], [B][H]
 *   1 <= nsplit <= 1024, B >= 1, H >= 1.
 */
int smla_combine(const float *part_o, const float *part_lse, int nsplit, float *out, float *lse, int B, int H,
                 void *stream);

/* Number of topk splits smla_decode uses for (B, topk) on the current device. */
int smla_num_splits(int B, int H, int topk);

/* Workspace bytes smla_decode needs (header + split-K partials for any split count
 * above 1, whatever the output type); 0 on bad sizes. */
size_t smla_workspace_bytes(int B, int H, int topk);

/* Workspace bytes for an explicit split count (1 <= nsplit <= ceil(topk/128)). */
size_t smla_workspace_bytes_ex(int B, int H, int topk, int nsplit);

/* Synchronises `stream`, copies the error word into *flags and clears it. */
int smla_read_error(void *workspace, void *stream, uint32_t *flags);

/*
 * smla_debug_gather -- the gather and dequantisation stages alone, for bit-exact
 * checks of index translation and FP8/UE8M0 decoding.
 *   latents   device, fp32 [B][topk][512]: the bf16 latent the decode kernel
 *             feeds to the tensor cores, widened to fp32 (zeros when invalid)
 *   page_slot device, int32 [B][topk][2]: (page, slot), (-1,-1) when invalid
 *   workspace as for smla_decode (only the error word is used).
 */
int smla_debug_gather(const uint8_t *kv_cache, const int32_t *block_table, const int32_t *topk_idx,
                      const int32_t *seq_lens, int B, int topk, int max_blocks, int num_pages, float *latents,
                      int32_t *page_slot, void *workspace, size_t workspace_bytes, void *stream);

/*
 * smla_decode_noalloc -- smla_decode for callers that cannot allocate device
 * memory.  (No counterpart on the source pages: this is a library-usage addition.)
 *
 * Who needs it: a serving engine that has frozen its device memory pool after
 * capturing its decode step into CUDA graphs, or a plugin host that owns every
 * device allocation, cannot give this library a workspace.  This entry point
 * takes the same arguments as smla_decode minus the workspace and uses instead
 * a scratch array of SMLA_STATIC_SCRATCH_BYTES (32 MiB) that is part of the
 * library's device image: every GPU that loads the library holds those bytes
 * until the process exits.  It allocates and frees nothing (no cudaMalloc, no
 * allocating library call).
 *
 *   - Limit: calls whose split-K exchange needs more than the array (what
 *     smla_workspace_bytes reports for the built-in split count) return
 *     SMLA_ERR_SCRATCH without launching.  On a 148-SM B200 the built-in split
 *     count keeps every call under 20 MB.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress with that device current); make that first call
 *     before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it has to start at zero (every partial is written before it is
 *     read), but calls whose kernels overlap on the GPU (for example calls on
 *     two streams of one device) race on it: serialise them.
 *   - Device-side error flags land in the array's error word and are not
 *     reported; use smla_decode with a workspace to read them.
 */
#define SMLA_STATIC_SCRATCH_BYTES (32u << 20)
int smla_decode_noalloc(const void *q, const uint8_t *kv_cache, const int32_t *block_table, const int32_t *topk_idx,
                        const int32_t *seq_lens, float sm_scale, float *out, float *lse, int B, int H, int topk,
                        int max_blocks, int num_pages, void *stream);

/*
 * smla_write_kv -- the KV-cache writer: quantise n new latents into the cache format
 * above and store each at position pos[i] of request req[i], i.e. at page
 * block_table[req[i]][pos[i] / 256], slot pos[i] % 256 (the page indexing of "The
 * Validation Moment"; the byte layout of "The Validation Gate", "The Test Design").
 * The pages do not say how the scales are chosen; the rule here is that of the
 * synthetic caches: per 64-dim nope group g, e = the smallest integer with
 * max|x| <= 448 * 2^e, clamped to [-127, 127] (-127 for an all-zero group); scale
 * byte g = e + 127 (byte 7 = 0); nope byte d = e4m3 of x[d] / 2^e, round to nearest
 * even; rope value r = bf16 of x[448 + r], round to nearest even.  Non-finite
 * inputs: a group holding an infinity or NaN takes e = 127, +-inf becomes +-448
 * (0x7E / 0xFE) and NaN 0x7F; a NaN rope value becomes 0x7FC0.
 *   latents     device, [n][512], fp32 (latents_bf16 = 0) or bf16 (latents_bf16 = 1),
 *               16-byte aligned
 *   req, pos    device, int32 [n]: request and position of each token
 *   block_table device, int32 [B][max_blocks]
 *   kv_cache    device, uint8 [num_pages][149504], 16-byte aligned (written)
 *   err         device uint32 or NULL: SMLA_FLAG_BAD_PAGE is or-ed in when a token
 *               is skipped (req outside [0, B), pos < 0, pos / 256 >= max_blocks, or
 *               a page outside [0, num_pages)); nothing is written for it
 *   n >= 0 (0: nothing is launched), B >= 1, max_blocks >= 1, 1 <= num_pages < 2^23.
 * Two tokens with the same destination in one call: one of them is stored (which one
 * is unspecified).  One launch on `stream`, one warp per token.
 */
int smla_write_kv(const void *latents, int latents_bf16, int n, const int32_t *req, const int32_t *pos,
                  const int32_t *block_table, int B, int max_blocks, int num_pages, uint8_t *kv_cache,
                  uint32_t *err, void *stream);

/* Build identification string (static storage). */
const char *smla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SMLA_H */
