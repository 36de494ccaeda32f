/*
 * smla_oracle.c -- plain fp64 CPU oracle for the sparse MLA decode step over an
 * FP8 paged latent cache.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the CUDA path: the byte layout, the
 * e4m3 / UE8M0 / bf16 decoders and the attention arithmetic are all written out
 * again here, in double precision, in the order the method states them.
 *
 * What it follows (page titles of the source blog pages):
 *  - "The Validation Gate: Writing a Standalone Correctness Test for a Custom MMA
 *    Sparse-Decode Kernel", section "The Test Design": the cache is a flat uint8
 *    array of 256-token pages; one page holds all 256 token rows of 576 bytes
 *    (448 FP8 nope bytes, then the rope part in bf16) followed by all 256 scale
 *    rows of 8 bytes.
 *  - "The Turning Point: Architecting a Custom MMA Sparse-MLA Decode Kernel",
 *    Step 1 (Q is [B,H,512] = 448 nope + 64 rope, one shared latent KV head),
 *    Input Knowledge (nope in FP8 with UE8M0 scales, rope in bf16), Output
 *    Knowledge item 2 (dequantize -> concat -> matmul -> softmax -> weighted sum)
 *    and Step 5 (partial outputs with log-sum-exp, merged by the standard
 *    online-softmax combine).
 *  - "The Validation Moment", section on the smoke test: the page-indexing logic
 *    (logical token index -> block table -> physical page and slot).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - e4m3 is the OCP "fn" flavour (bias 7, no infinities, 0x7F/0xFF are NaN).
 *  - A UE8M0 byte b encodes 2^(b-127); 0xFF is NaN.
 *  - Scale byte g (g = 0..6) covers nope dims [64g, 64g+64); byte 7 is padding.
 *  - The rope part is 64 little-endian bf16 values (128 bytes, so 448+128 = 576).
 *  - V is the whole 512-d dequantised latent; O is [B,H,512].
 *  - A topk slot is valid iff 0 <= idx < seq_len[b], idx/256 < max_blocks and the
 *    physical page lies in [0, num_pages).  Duplicates count with multiplicity.
 *  - No valid slot: O = 0 and LSE = -inf.  LSE is a natural log of the sum of
 *    exp(sm_scale * q.k).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_PAGE_TOKENS 256
#define ORC_ROW_BYTES 576
#define ORC_SCALE_ROW_BYTES 8
#define ORC_NOPE 448
#define ORC_ROPE 64
#define ORC_DIM 512
#define ORC_GROUP 64
/* 256 rows of 576 bytes, then 256 scale rows of 8 bytes */
#define ORC_SCALE_BLOCK_OFFSET ((int64_t)ORC_PAGE_TOKENS * ORC_ROW_BYTES)
#define ORC_PAGE_BYTES ((int64_t)ORC_PAGE_TOKENS * (ORC_ROW_BYTES + ORC_SCALE_ROW_BYTES))

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* OCP e4m3 (fn): sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
 * subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is no infinity. */
double orc_e4m3(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 15;
    int m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* UE8M0: an unsigned biased exponent with no mantissa, 2^(b-127); 0xFF is NaN. */
double orc_ue8m0(uint8_t b) {
    if (b == 255) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* bf16: the upper half of an IEEE binary32. */
double orc_bf16(uint16_t u) {
    uint32_t bits = (uint32_t)u << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Logical token index -> (physical page, slot).  Returns 1 if the slot is valid. */
int orc_translate_one(const int32_t *bt_row, int max_blocks, int seq_len, int64_t num_pages,
                      int32_t idx, int32_t *page, int32_t *slot) {
    int32_t blk, p;
    if (idx < 0 || idx >= seq_len) return 0;
    blk = idx / ORC_PAGE_TOKENS;
    if (blk >= max_blocks) return 0;
    p = bt_row[blk];
    if (p < 0 || (int64_t)p >= num_pages) return 0;
    *page = p;
    *slot = idx % ORC_PAGE_TOKENS;
    return 1;
}

/* Decode one cached token into its 512-d latent: nope[d] = e4m3(byte d) *
 * ue8m0(scale byte d/64), rope[r] = bf16 at bytes 448+2r, 449+2r. */
void orc_token_latent(const uint8_t *cache, int64_t page, int slot, double *k) {
    const uint8_t *page_base = cache + page * ORC_PAGE_BYTES;
    const uint8_t *row = page_base + (int64_t)slot * ORC_ROW_BYTES;
    const uint8_t *scales = page_base + ORC_SCALE_BLOCK_OFFSET + (int64_t)slot * ORC_SCALE_ROW_BYTES;
    int d, r;
    for (d = 0; d < ORC_NOPE; d++) k[d] = orc_e4m3(row[d]) * orc_ue8m0(scales[d / ORC_GROUP]);
    for (r = 0; r < ORC_ROPE; r++) {
        uint16_t u = (uint16_t)(row[ORC_NOPE + 2 * r] | (row[ORC_NOPE + 2 * r + 1] << 8));
        k[ORC_NOPE + r] = orc_bf16(u);
    }
}

/* Gather: page/slot for every topk slot ([B,topk,2], -1 when invalid) and the
 * dequantised latent ([B,topk,512], zeros when invalid). */
int orc_gather(const uint8_t *cache, int64_t num_pages, const int32_t *block_table, int max_blocks,
               const int32_t *topk_idx, const int32_t *seq_lens, int B, int topk,
               double *latents, int32_t *page_slot) {
    int b;
    if (B < 0 || topk < 0 || max_blocks < 0) return -1;
#pragma omp parallel for schedule(dynamic)
    for (b = 0; b < B; b++) {
        int i;
        for (i = 0; i < topk; i++) {
            int32_t page = -1, slot = -1;
            int64_t o = (int64_t)b * topk + i;
            int ok = orc_translate_one(block_table + (int64_t)b * max_blocks, max_blocks, seq_lens[b],
                                       num_pages, topk_idx[o], &page, &slot);
            if (page_slot) {
                page_slot[2 * o] = ok ? page : -1;
                page_slot[2 * o + 1] = ok ? slot : -1;
            }
            if (latents) {
                if (ok)
                    orc_token_latent(cache, page, slot, latents + o * ORC_DIM);
                else
                    memset(latents + o * ORC_DIM, 0, sizeof(double) * ORC_DIM);
            }
        }
    }
    return 0;
}

/* Softmax-weighted latent and log-sum-exp for one head over the gathered set:
 *   s_j = sm_scale * <q, k_j>,  M = max_j s_j,
 *   O   = sum_j exp(s_j - M) k_j / sum_j exp(s_j - M),
 *   LSE = M + ln sum_j exp(s_j - M). */
static void orc_attend_one(const double *qh, const double *K, int n, double sm_scale,
                           double *o, double *lse, double *s) {
    int j, d;
    double M = -INFINITY, l = 0.0;
    for (d = 0; d < ORC_DIM; d++) o[d] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return;
    }
    for (j = 0; j < n; j++) {
        double acc = 0.0;
        for (d = 0; d < ORC_DIM; d++) acc += qh[d] * K[(int64_t)j * ORC_DIM + d];
        s[j] = sm_scale * acc;
        if (s[j] > M) M = s[j];
    }
    for (j = 0; j < n; j++) {
        double w = exp(s[j] - M);
        l += w;
        for (d = 0; d < ORC_DIM; d++) o[d] += w * K[(int64_t)j * ORC_DIM + d];
    }
    for (d = 0; d < ORC_DIM; d++) o[d] /= l;
    *lse = M + log(l);
}

/* The decode step.  q: bf16 bits [B,H,512].  If rows is NULL every (b,h) is
 * computed and out/lse are [B,H,512] / [B,H]; otherwise rows holds nrows pairs
 * (b,h) and out/lse are [nrows,512] / [nrows] in that order. */
int orc_decode(const uint16_t *q, const uint8_t *cache, int64_t num_pages, const int32_t *block_table,
               int max_blocks, const int32_t *topk_idx, const int32_t *seq_lens, double sm_scale,
               int B, int H, int topk, const int32_t *rows, int nrows, double *out, double *lse) {
    int b;
    if (B < 0 || H <= 0 || topk < 0 || max_blocks < 0) return -1;
    if (rows) {
        int r;
        for (r = 0; r < nrows; r++)
            if (rows[2 * r] < 0 || rows[2 * r] >= B || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= H) return -1;
    }
#pragma omp parallel for schedule(dynamic)
    for (b = 0; b < B; b++) {
        int i, n = 0, h, r, d;
        int want = (rows == NULL);
        double *K, *s, *qh;
        if (!want)
            for (r = 0; r < nrows; r++)
                if (rows[2 * r] == b) want = 1;
        if (!want) continue;
        K = (double *)malloc(sizeof(double) * ORC_DIM * (size_t)(topk > 0 ? topk : 1));
        s = (double *)malloc(sizeof(double) * (size_t)(topk > 0 ? topk : 1));
        qh = (double *)malloc(sizeof(double) * ORC_DIM);
        /* gather the valid slots once per request (a multiset, in slot order) */
        for (i = 0; i < topk; i++) {
            int32_t page, slot;
            if (orc_translate_one(block_table + (int64_t)b * max_blocks, max_blocks, seq_lens[b], num_pages,
                                  topk_idx[(int64_t)b * topk + i], &page, &slot)) {
                orc_token_latent(cache, page, slot, K + (int64_t)n * ORC_DIM);
                n++;
            }
        }
        if (rows == NULL) {
            for (h = 0; h < H; h++) {
                for (d = 0; d < ORC_DIM; d++) qh[d] = orc_bf16(q[((int64_t)b * H + h) * ORC_DIM + d]);
                orc_attend_one(qh, K, n, sm_scale, out + ((int64_t)b * H + h) * ORC_DIM, lse + (int64_t)b * H + h, s);
            }
        } else {
            for (r = 0; r < nrows; r++) {
                if (rows[2 * r] != b) continue;
                h = rows[2 * r + 1];
                for (d = 0; d < ORC_DIM; d++) qh[d] = orc_bf16(q[((int64_t)b * H + h) * ORC_DIM + d]);
                orc_attend_one(qh, K, n, sm_scale, out + (int64_t)r * ORC_DIM, lse + r, s);
            }
        }
        free(K);
        free(s);
        free(qh);
    }
    return 0;
}

/* Split-K merge ("standard online softmax combine"): given per-split normalised
 * outputs O_s and log-sum-exps L_s of disjoint parts of the gathered set,
 *   L = ln sum_s exp(L_s),  O = sum_s exp(L_s - L) O_s.
 * A split with L_s = -inf has weight 0; if every split is -inf, O = 0, L = -inf.
 * part_o: [B,H,nsplit,512], part_lse: [B,H,nsplit]. */
int orc_combine(const double *part_o, const double *part_lse, int B, int H, int nsplit,
                double *out, double *lse) {
    int64_t bh;
    if (B < 0 || H <= 0 || nsplit <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (bh = 0; bh < (int64_t)B * H; bh++) {
        const double *L = part_lse + bh * nsplit;
        double Lmax = -INFINITY, W = 0.0;
        int s, d;
        double *o = out + bh * ORC_DIM;
        for (d = 0; d < ORC_DIM; d++) o[d] = 0.0;
        for (s = 0; s < nsplit; s++)
            if (L[s] > Lmax) Lmax = L[s];
        if (Lmax == -INFINITY) {
            lse[bh] = -INFINITY;
            continue;
        }
        for (s = 0; s < nsplit; s++) {
            double w;
            if (L[s] == -INFINITY) continue;
            w = exp(L[s] - Lmax);
            W += w;
            for (d = 0; d < ORC_DIM; d++) o[d] += w * part_o[(bh * nsplit + s) * ORC_DIM + d];
        }
        for (d = 0; d < ORC_DIM; d++) o[d] /= W;
        lse[bh] = Lmax + log(W);
    }
    return 0;
}

/* ------------------------------------------------------------------ cache writer
 * The inverse of orc_token_latent, for the synthetic-cache quantisation the pages
 * leave open (reading: scale exponent e = ceil(log2(amax / 448)) per 64-dim nope
 * group, i.e. the smallest e with amax <= 448 * 2^e, clamped to [-127, 127] and -127
 * for an all-zero group; scale byte e + 127; nope byte = e4m3 of x / 2^e rounded to
 * nearest, ties to even; rope = bf16 of x rounded to nearest, ties to even).
 * Non-finite inputs (not produced by the generators; fixed here so that two writers
 * can be compared byte for byte): a group holding an infinity or NaN takes e = 127;
 * +-inf saturates to +-448, NaN becomes 0x7F; a NaN rope value becomes 0x7FC0. */

/* Nearest e4m3 (fn) code to x by search over the 127 non-negative finite codes; a
 * tie goes to the code whose last mantissa bit is 0; |x| >= 448 gives 448 (0x7E). */
uint8_t orc_e4m3_encode(double x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x), best_d = INFINITY;
    int c, best = 0;
    if (isnan(x)) return 0x7F;
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    for (c = 0; c <= 0x7E; c++) {
        double d = fabs(orc_e4m3((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best_d = d;
            best = c;
        }
    }
    return (uint8_t)(sign | best);
}

/* bf16 of a binary32 value: the nearer of the two bf16 values around it (its upper
 * half truncated, and the next one away from zero), a tie to the one whose last bit
 * is 0.  The truncation is exact for values that are already bf16. */
uint16_t orc_bf16_encode(float f) {
    uint32_t bits;
    uint16_t lo, hi;
    double dlo, dhi, v = (double)f;
    if (isnan(f)) return 0x7FC0;
    memcpy(&bits, &f, sizeof bits);
    lo = (uint16_t)(bits >> 16);
    if ((bits & 0xFFFF) == 0) return lo;
    hi = (uint16_t)(lo + 1); /* next magnitude up; past the largest finite it is the infinity, */
    dlo = fabs(orc_bf16(lo) - v); /* which rounding treats as the value 2^128 */
    dhi = ((hi & 0x7FFF) == 0x7F80) ? fabs(copysign(ldexp(1.0, 128), v) - v) : fabs(orc_bf16(hi) - v);
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo & 1) ? hi : lo;
}

/* The scale exponent of one nope group (see the reading above). */
int orc_scale_exponent(const float *x) {
    double amax = 0.0;
    int d, e;
    for (d = 0; d < ORC_GROUP; d++) {
        if (!isfinite(x[d])) return 127;
        if (fabs((double)x[d]) > amax) amax = fabs((double)x[d]);
    }
    if (amax == 0.0) return -127;
    e = -127;
    while (e < 127 && ldexp(448.0, e) < amax) e++;
    return e;
}

/* One 512-d latent -> its 576-byte row and 8-byte scale row (byte 7 = 0). */
void orc_quantize_token(const float *x, uint8_t *row, uint8_t *scale_row) {
    int g, d, r;
    for (g = 0; g < ORC_NOPE / ORC_GROUP; g++) {
        int e = orc_scale_exponent(x + g * ORC_GROUP);
        scale_row[g] = (uint8_t)(e + 127);
        for (d = g * ORC_GROUP; d < (g + 1) * ORC_GROUP; d++) row[d] = orc_e4m3_encode(ldexp((double)x[d], -e));
    }
    scale_row[ORC_NOPE / ORC_GROUP] = 0;
    for (r = 0; r < ORC_ROPE; r++) {
        uint16_t u = orc_bf16_encode(x[ORC_NOPE + r]);
        row[ORC_NOPE + 2 * r] = (uint8_t)(u & 0xFF);
        row[ORC_NOPE + 2 * r + 1] = (uint8_t)(u >> 8);
    }
}

/* Writes n latents [n,512] at positions pos[i] of requests req[i]: page =
 * block_table[req][pos / 256], slot = pos % 256 (the page indexing of "The
 * Validation Moment").  A token whose request, position or page is out of range
 * is skipped.  Returns the number of skipped tokens. */
int orc_write_kv(const float *latents, int n, const int32_t *req, const int32_t *pos,
                 const int32_t *block_table, int B, int max_blocks, int64_t num_pages, uint8_t *cache) {
    int i, skipped = 0;
    for (i = 0; i < n; i++) {
        int32_t b = req[i], p = pos[i], page;
        uint8_t *page_base;
        if (b < 0 || b >= B || p < 0 || p / ORC_PAGE_TOKENS >= max_blocks) {
            skipped++;
            continue;
        }
        page = block_table[(int64_t)b * max_blocks + p / ORC_PAGE_TOKENS];
        if (page < 0 || (int64_t)page >= num_pages) {
            skipped++;
            continue;
        }
        page_base = cache + (int64_t)page * ORC_PAGE_BYTES;
        orc_quantize_token(latents + (int64_t)i * ORC_DIM,
                           page_base + (int64_t)(p % ORC_PAGE_TOKENS) * ORC_ROW_BYTES,
                           page_base + ORC_SCALE_BLOCK_OFFSET + (int64_t)(p % ORC_PAGE_TOKENS) * ORC_SCALE_ROW_BYTES);
    }
    return skipped;
}
