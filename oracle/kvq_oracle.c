/*
 * kvq_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, single-threaded CPU restatement of the SAW-INT4 KV-cache
 * write path (block-diagonal Hadamard rotation followed by token-wise
 * asymmetric INT4 quantisation, appended through a page table) and read path
 * (paged GQA decode attention over the dequantised cache).  Only the test
 * suite, the package smoke check and the benchmark's CPU-baseline leg may load
 * it.  The CUDA library never does, and the two share no source, header,
 * constant or helper.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (see
 * oracle/__init__.py).  FP contraction is off so every float operation below
 * is one IEEE-754 binary32 operation rounded to nearest-even, in the order
 * written.
 *
 * Sources (pages about "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for
 * Real-World LLM Serving", arXiv 2604.19157):
 *  [ABS]  the paper's abstract (fugumt.com paper check, "Abstract"):
 *         token-wise INT4 quantisation with block-diagonal Hadamard rotation;
 *         a fused rotation-quantisation kernel that writes into paged KV-cache
 *         layouts; fused attention execution.
 *  [WIS2] wispaper.ai blog on the paper, section 2 ("core intuition:
 *         rotation"): head_dim is split into blocks of 16 to 128 that are
 *         rotated independently by a Hadamard matrix.
 *  [WIS3] same blog, section 3 ("methodology"), the formula
 *         K~ = quant(K H_blk), V~ = quant(V H_blk); the rotation is fused into
 *         the KV-cache write; the query is rotated in step so that the dot
 *         product is the same as in the original space.
 *  [WIS4] same blog, section 4 ("experiments"): ablations over key-only versus
 *         key+value rotation and over the block size.
 *
 * Readings where the pages are silent:
 *  R1 H_b is Sylvester's Hadamard matrix in natural order,
 *     H[i][j] = (-1)^popcount(i & j), normalised by 1/sqrt(b).
 *  R2 The fp32 FWHT runs its butterfly stages with increasing stride
 *     h = 1, 2, ..., b/2, pairs (i, i+h) with (i & h) == 0 becoming
 *     (x_i + x_{i+h}, x_i - x_{i+h}); the result is then multiplied by
 *     r_b = (float)(1.0 / sqrt((double)b)).
 *  R3 "Token-wise": one scale and one zero per (token, KV head), taken over the
 *     whole head_dim (rotation blocks do not get their own scales).
 *  R4 Asymmetric min/max quantiser with a float offset:
 *     scale = fp16(fl(max - min) / 15), zero = fp16(min), signed zeros of min
 *     and max canonicalised to +0 first; inv = fl(1 / float(scale)) or 0 when
 *     scale is not positive; code = clamp(rint_even(fl(y - zero) * inv), 0, 15)
 *     where the product fl(y - zero) * inv is taken exactly (not rounded to
 *     fp32 before the rounding to an integer).  A row holding a NaN has NaN
 *     min and max: scale = zero = fp16 quiet NaN 0x7E00 and every code 0.
 *     Dequantised value = code * scale + zero.
 *  2-bit variant (optional): the same quantiser with range/3, codes 0..3, four
 *     codes per byte, code k of a byte in bits 2k and 2k+1.
 *  Fused RoPE (optional): a caller-given table of (cos, sin) per position and
 *     rotate-half pair turns the keys (fp32, before the block rotation; BF16
 *     pages store the turned row rounded to bf16) and the query, at position
 *     seq_len - 1, the newest token; positions outside the table are skipped.
 *  R5 Packing: byte j holds code 2j in its low nibble and code 2j+1 in its
 *     high nibble.
 *  R6 Page layout: codes uint8 [pages, H_kv, page_size, D/2]; scale/zero as
 *     fp16 pairs [pages, H_kv, page_size, 2]; BF16 cache bf16
 *     [pages, H_kv, page_size, D].  Token at position p of sequence s lives in
 *     page page_table[s * pt_stride + p / page_size], slot p % page_size.
 *  R7 Decode: query head j reads KV head j / (H_q / H_kv); scores are
 *     (q' . k^) / sqrt(D); exact softmax over all seq_len cached tokens; when V
 *     was rotated the output is rotated back with the same H_blk (self-inverse).
 *     An empty sequence yields a zero output row.
 *  R8 Out-of-range page ids, positions or sequence ids are skipped and counted
 *     (the count is the return value), never dereferenced.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KVQO_BF16 0
#define KVQO_INT4 1
#define KVQO_INT4_BDR 2

int oracle_version(void) { return 1; }

/* ---- scalar conversions -------------------------------------------------- */

static float bf16_bits_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16; /* bf16 is the top half of a binary32 */
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* IEEE binary32 -> binary16, round to nearest even (the compiler's own
 * conversion of the C23/TS 18661-3 _Float16 type). */
static uint16_t f32_to_f16_bits(float f) {
    _Float16 h = (_Float16)f;
    uint16_t u;
    memcpy(&u, &h, 2);
    return u;
}

static float f16_bits_to_f32(uint16_t u) {
    _Float16 h;
    memcpy(&h, &u, 2);
    return (float)h;
}

void oracle_f32_to_f16(const float* x, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; i++) out[i] = f32_to_f16_bits(x[i]);
}

/* ---- rotation (C2, [WIS2], [WIS3]; readings R1, R2) ---------------------- */

/* The normalisation constant r_b of reading R2. */
static float rb_f32(int b) { return (float)(1.0 / sqrt((double)b)); }

/* In-place fp32 fast Walsh-Hadamard transform of each length-b block of x[0..D),
 * stages in increasing stride; normalised by r_b when normalise != 0. */
/* fp32 -> bf16 bits, round to nearest even; NaN -> 0x7FC0. */
static uint16_t f32_to_bf16_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0x7FC0;
    return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

/* Rotary position embedding, rotate-half layout (reading for the fused RoPE):
 * element i and i + D/2 (i < D/2) turn by the angle of pair i at the row's
 * position, given as cs[2i] = cos, cs[2i+1] = sin (the caller's table row):
 *   x'_i       = fl(fl(x_i cos) - fl(x_{i+D/2} sin))
 *   x'_{i+D/2} = fl(fl(x_{i+D/2} cos) + fl(x_i sin))
 * one IEEE op each, no FMA contraction. */
void oracle_rope_f32(float* x, int D, const float* cs) {
    int half = D / 2;
    for (int i = 0; i < half; i++) {
        float c = cs[2 * i], s = cs[2 * i + 1];
        float a = x[i], b = x[i + half];
        float ac = a * c, bs = b * s, bc = b * c, as = a * s;
        x[i] = ac - bs;
        x[i + half] = bc + as;
    }
}

void oracle_rotate_f32(float* x, int D, int b, int normalise) {
    for (int base = 0; base < D; base += b) {
        float* blk = x + base;
        for (int h = 1; h < b; h <<= 1) {
            for (int i = 0; i < b; i++) {
                if ((i & h) == 0) {
                    float a = blk[i];
                    float c = blk[i + h];
                    blk[i] = a + c;
                    blk[i + h] = a - c;
                }
            }
        }
        if (normalise) {
            float r = rb_f32(b);
            for (int i = 0; i < b; i++) blk[i] = blk[i] * r;
        }
    }
}

/* The same rotation in float64 with the exact normaliser 1/sqrt(b); used on
 * the read side (query and output), which the pages fix to no precision. */
void oracle_rotate_f64(double* x, int D, int b) {
    double r = 1.0 / sqrt((double)b);
    for (int base = 0; base < D; base += b) {
        double* blk = x + base;
        for (int h = 1; h < b; h <<= 1) {
            for (int i = 0; i < b; i++) {
                if ((i & h) == 0) {
                    double a = blk[i];
                    double c = blk[i + h];
                    blk[i] = a + c;
                    blk[i + h] = a - c;
                }
            }
        }
        for (int i = 0; i < b; i++) blk[i] = blk[i] * r;
    }
}

/* ---- token-wise asymmetric INT4 (C1, [ABS], [WIS3]; readings R3-R5) ------ */

/* Quantise one (already rotated) row y[0..D) into D*bits/8 packed bytes and an
 * (scale, zero) fp16 pair: bits = 4 (codes 0..15, two per byte) or 2 (codes
 * 0..3, four per byte; reading for the 2-bit variant: the same token-wise
 * asymmetric quantiser with range/3, code k of a byte in bits 2k, 2k+1). */
void oracle_quant_row_bits(const float* y, int D, int bits, uint8_t* codes, uint16_t* scale_zero) {
    const int levels = (1 << bits) - 1;
    const int per_byte = 8 / bits;
    const int nbytes = D / per_byte;
    /* a NaN anywhere makes the row's min and max NaN (reading): scale and zero are the
     * fp16 quiet NaN 0x7E00 and every code is 0 */
    for (int i = 0; i < D; i++) {
        if (y[i] != y[i]) {
            for (int j = 0; j < nbytes; j++) codes[j] = 0;
            scale_zero[0] = scale_zero[1] = 0x7E00;
            return;
        }
    }
    float mn = y[0], mx = y[0];
    for (int i = 1; i < D; i++) {
        if (y[i] < mn) mn = y[i];
        if (y[i] > mx) mx = y[i];
    }
    mn = mn + 0.0f; /* -0 + +0 = +0: signed zeros made canonical */
    mx = mx + 0.0f;
    float range = mx - mn;
    float s32 = range / (float)levels;
    uint16_t scale_h = f32_to_f16_bits(s32);
    uint16_t zero_h = f32_to_f16_bits(mn);
    float scale = f16_bits_to_f32(scale_h);
    float zero = f16_bits_to_f32(zero_h);
    float inv = (scale > 0.0f) ? 1.0f / scale : 0.0f;
    for (int j = 0; j < nbytes; j++) codes[j] = 0;
    for (int e = 0; e < D; e++) {
        float t = y[e] - zero;
        /* R4: rint (ties to even) of the exact product fl(y - zero) * fl(1/scale),
         * one rounding straight to an integer (not the product rounded to fp32 first,
         * and not the exact quotient (y - zero) / scale).  The product of two floats is
         * exact in double (24 + 24 < 53 significant bits). */
        double v = (double)t * (double)inv;
        double r = rint(v); /* default rounding mode: nearest, ties to even */
        int code;
        if (!(r > 0.0)) code = 0; /* also NaN */
        else if (r > (double)levels) code = levels;
        else code = (int)r;
        codes[e / per_byte] |= (uint8_t)(code << (bits * (e % per_byte)));
    }
    scale_zero[0] = scale_h;
    scale_zero[1] = zero_h;
}

void oracle_quant_row(const float* y, int D, uint8_t* codes, uint16_t* scale_zero) {
    oracle_quant_row_bits(y, D, 4, codes, scale_zero);
}

void oracle_quant_rows_bits(const uint16_t* x, int64_t n, int D, int b, int bits, uint8_t* codes, uint16_t* sz) {
    float* y = (float*)malloc(sizeof(float) * (size_t)D);
    for (int64_t r = 0; r < n; r++) {
        for (int i = 0; i < D; i++) y[i] = bf16_bits_to_f32(x[r * D + i]);
        if (b > 0) oracle_rotate_f32(y, D, b, 1);
        oracle_quant_row_bits(y, D, bits, codes + r * (D * bits / 8), sz + r * 2);
    }
    free(y);
}

void oracle_quant_rows(const uint16_t* x, int64_t n, int D, int b, uint8_t* codes, uint16_t* sz) {
    oracle_quant_rows_bits(x, n, D, b, 4, codes, sz);
}

/* ---- append into the paged cache (C3, C5, C6; reading R6, R8) ------------ */

/* Appends num_tokens tokens.  k, v: bf16 [num_tokens, H, D].  Token i goes to
 * sequence tok_seq[i] at position tok_pos[i].  Returns the number of
 * (token) writes skipped because an index was out of range. */
int64_t oracle_append(int mode, int bdr_block, int rotate_v, int num_pages, int page_size,
                      int H, int D, uint8_t* k_pool, uint8_t* v_pool, uint16_t* k_sz,
                      uint16_t* v_sz, const uint16_t* k, const uint16_t* v, int num_tokens,
                      const int32_t* tok_seq, const int32_t* tok_pos, const int32_t* page_table,
                      int pt_stride, int num_seqs, const float* rope, int rope_positions, int bits) {
    int64_t skipped = 0;
    float* y = (float*)malloc(sizeof(float) * (size_t)D);
    const int row_bytes = D * bits / 8;
    for (int i = 0; i < num_tokens; i++) {
        int s = tok_seq[i], p = tok_pos[i];
        if (s < 0 || s >= num_seqs || p < 0 || p / page_size >= pt_stride || (rope && p >= rope_positions)) {
            skipped++;
            continue;
        }
        int page = page_table[(int64_t)s * pt_stride + p / page_size];
        if (page < 0 || page >= num_pages) {
            skipped++;
            continue;
        }
        int slot = p % page_size;
        for (int h = 0; h < H; h++) {
            int64_t row = ((int64_t)page * H + h) * page_size + slot;
            for (int kv = 0; kv < 2; kv++) {
                const uint16_t* src = (kv == 0 ? k : v) + ((int64_t)i * H + h) * D;
                int rotary = rope && kv == 0; /* RoPE turns the keys only */
                if (mode == KVQO_BF16) {
                    uint16_t* dst = (uint16_t*)(kv == 0 ? k_pool : v_pool) + row * D;
                    if (!rotary) {
                        memcpy(dst, src, sizeof(uint16_t) * (size_t)D);
                    } else {
                        for (int e = 0; e < D; e++) y[e] = bf16_bits_to_f32(src[e]);
                        oracle_rope_f32(y, D, rope + (int64_t)p * D);
                        for (int e = 0; e < D; e++) dst[e] = f32_to_bf16_bits(y[e]);
                    }
                    continue;
                }
                for (int e = 0; e < D; e++) y[e] = bf16_bits_to_f32(src[e]);
                if (rotary) oracle_rope_f32(y, D, rope + (int64_t)p * D);
                int rotate = (mode == KVQO_INT4_BDR) && (kv == 0 || rotate_v);
                if (rotate) oracle_rotate_f32(y, D, bdr_block, 1);
                uint8_t* cdst = (kv == 0 ? k_pool : v_pool) + row * row_bytes;
                uint16_t* sdst = (kv == 0 ? k_sz : v_sz) + row * 2;
                oracle_quant_row_bits(y, D, bits, cdst, sdst);
            }
        }
    }
    free(y);
    return skipped;
}

/* ---- decode attention over the paged cache (C4, C7; readings R6-R8) ------ */

/* Dequantised element e of the cached row (page, h, slot), as float64. */
static double cached_value(int mode, int bits, const void* pool, const uint16_t* sz, int64_t row, int D, int e) {
    if (mode == KVQO_BF16) return (double)bf16_bits_to_f32(((const uint16_t*)pool)[row * D + e]);
    const int per_byte = 8 / bits;
    uint8_t byte = ((const uint8_t*)pool)[row * (D / per_byte) + e / per_byte];
    int code = (byte >> (bits * (e % per_byte))) & ((1 << bits) - 1);
    double scale = (double)f16_bits_to_f32(sz[row * 2 + 0]);
    double zero = (double)f16_bits_to_f32(sz[row * 2 + 1]);
    return (double)code * scale + zero;
}

/* Computes out[r, :] for each requested (sequence, query head) pair
 * rows[2r], rows[2r+1] (all B*Hq pairs in order when rows == NULL).
 * q: bf16 [batch, Hq, D].  out: float64 [num_rows, D].  Returns the number of
 * cached tokens skipped because their page id was out of range. */
int64_t oracle_decode(int mode, int bdr_block, int rotate_v, int num_pages, int page_size, int H,
                      int Hq, int D, const void* k_pool, const void* v_pool, const uint16_t* k_sz,
                      const uint16_t* v_sz, const uint16_t* q, const int32_t* seq_lens,
                      const int32_t* page_table, int pt_stride, int batch, const int32_t* rows,
                      int num_rows, double* out, const float* rope, int rope_positions, int bits) {
    int64_t skipped = 0;
    int G = Hq / H;
    int n = rows ? num_rows : batch * Hq;
    double* qr = (double*)malloc(sizeof(double) * (size_t)D);
    double* o = (double*)malloc(sizeof(double) * (size_t)D);
    for (int r = 0; r < n; r++) {
        int s = rows ? rows[2 * r] : r / Hq;
        int j = rows ? rows[2 * r + 1] : r % Hq;
        int h = j / G;
        for (int e = 0; e < D; e++) qr[e] = (double)bf16_bits_to_f32(q[((int64_t)s * Hq + j) * D + e]);
        int L = seq_lens[s];
        if (L < 0) L = 0;
        if (rope && L > 0) {
            /* the query is the newest token, at position L - 1 (reading); a position outside the
             * table skips the sequence: zero output */
            if (L > rope_positions) {
                skipped += L;
                for (int e = 0; e < D; e++) out[(int64_t)r * D + e] = 0.0;
                continue;
            }
            const float* cs = rope + (int64_t)(L - 1) * D;
            for (int i = 0; i < D / 2; i++) {
                double c = (double)cs[2 * i], sn = (double)cs[2 * i + 1];
                double a = qr[i], b = qr[i + D / 2];
                qr[i] = a * c - b * sn;
                qr[i + D / 2] = b * c + a * sn;
            }
        }
        if (mode == KVQO_INT4_BDR) oracle_rotate_f64(qr, D, bdr_block);
        if (L > pt_stride * page_size) { /* positions beyond the page table */
            skipped += L - pt_stride * page_size;
            L = pt_stride * page_size;
        }
        double* z = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        int64_t* rowid = (int64_t*)malloc(sizeof(int64_t) * (size_t)(L > 0 ? L : 1));
        double zmax = -INFINITY;
        for (int t = 0; t < L; t++) {
            int page = page_table[(int64_t)s * pt_stride + t / page_size];
            if (page < 0 || page >= num_pages) {
                rowid[t] = -1;
                skipped++;
                continue;
            }
            int64_t row = ((int64_t)page * H + h) * page_size + t % page_size;
            rowid[t] = row;
            double dot = 0.0;
            for (int e = 0; e < D; e++) dot += qr[e] * cached_value(mode, bits, k_pool, k_sz, row, D, e);
            z[t] = dot / sqrt((double)D);
            if (z[t] > zmax) zmax = z[t];
        }
        for (int e = 0; e < D; e++) o[e] = 0.0;
        double l = 0.0;
        for (int t = 0; t < L; t++) {
            if (rowid[t] < 0) continue;
            double p = exp(z[t] - zmax);
            l += p;
            for (int e = 0; e < D; e++) o[e] += p * cached_value(mode, bits, v_pool, v_sz, rowid[t], D, e);
        }
        if (l > 0.0)
            for (int e = 0; e < D; e++) o[e] /= l;
        if (mode == KVQO_INT4_BDR && rotate_v) oracle_rotate_f64(o, D, bdr_block);
        memcpy(out + (int64_t)r * D, o, sizeof(double) * (size_t)D);
        free(z);
        free(rowid);
    }
    free(qr);
    free(o);
    return skipped;
}
