/*
 * kvq.h -- C ABI of libkvq.so: a paged KV cache holding keys and values as
 * token-wise asymmetric INT4 after a block-diagonal Hadamard rotation (BDR),
 * with the fused append (write) kernel and the paged GQA decode-attention
 * (read) kernels, for NVIDIA B200 (sm_100a).
 *
 * The method is SAW-INT4 ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization
 * for Real-World LLM Serving", arXiv 2604.19157).  Passages cited below:
 *  [ABS]  the paper's abstract: token-wise INT4 quantisation with
 *         block-diagonal Hadamard rotation; a fused rotation-quantisation
 *         kernel that integrates directly into paged KV-cache layouts; paged
 *         memory, regular access and fused attention as serving constraints.
 *  [WIS1] wispaper.ai blog on the paper, section 1: PagedAttention needs
 *         fixed-size pages; channel-wise scales break contiguous access.
 *  [WIS2] same blog, section 2: head_dim split into independent blocks of
 *         16..128, each rotated by a Hadamard matrix before quantisation.
 *  [WIS3] same blog, section 3: K~ = quant(K H_blk), V~ = quant(V H_blk); the
 *         rotation is fused into the KV-cache write operator (no separate
 *         kernel); the query is rotated in step at inference, so the dot
 *         product equals the one in the original space.
 *  [WIS4] same blog, section 4: key-only rotation versus key+value; block 128.
 *
 * Conventions the pages leave open, fixed here:
 *  - H_b is Sylvester's Hadamard matrix in natural order,
 *    H[i][j] = (-1)^popcount(i & j), scaled by 1/sqrt(b); the fp32 transform
 *    runs butterfly stages of stride 1, 2, ..., b/2 ((a, c) -> (a + c, a - c))
 *    and then multiplies by (float)(1/sqrt((double)b)).
 *  - One fp16 scale and one fp16 zero per (token, KV head) over all head_dim
 *    elements: scale = fp16(fl(max - min) / 15), zero = fp16(min);
 *    code = clamp(rint_even(fl(y - zero) * fl(1 / scale)), 0, 15), the product
 *    rounded to an integer from its exact value (inverse 0 when scale == 0);
 *    dequantised value = code * scale + zero.
 *  - Byte j of a row holds code 2j in its low nibble, code 2j+1 in its high one.
 *  - Query head j reads KV head j / (num_q_heads / num_kv_heads); the softmax
 *    scale is 1/sqrt(head_dim); when values are rotated, the attention output
 *    is rotated back with the same H_blk (it is its own inverse).
 *
 * Memory layout (all buffers are caller-owned device memory):
 *  INT4 pools   uint8  [num_pages, num_kv_heads, page_size, head_dim/2]
 *               (head_dim/4 with code_bits = 2: four 2-bit codes per byte)
 *  scale/zero   fp16x2 [num_pages, num_kv_heads, page_size] (scale, zero)
 *  BF16 pools   bf16   [num_pages, num_kv_heads, page_size, head_dim]
 *  page_table   int32  [num_seqs, pt_stride]; token p of sequence s lives in
 *               page page_table[s * pt_stride + p / page_size], slot
 *               p % page_size.
 *
 * Devices: a handle belongs to the device that was current when kv_create_paged
 * made it; every later call on the handle makes that device current while it runs
 * and restores the caller's device before returning.
 *
 * Ownership and errors: the library owns only the opaque handle and one
 * device error word.  Every call is asynchronous on the given stream
 * (a cudaStream_t passed as void*, NULL = legacy default stream).  Arguments
 * are validated on the host before any launch (KV_ERR_INVALID /
 * KV_ERR_UNSUPPORTED, nothing launched).  Inside the kernels, a page id,
 * sequence id or position that falls outside the pool or page table is never
 * dereferenced: that token's work is skipped and a bit is set in the device
 * error word, which kv_get_error() reports as KV_ERR_OOB.  No kernel traps.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KV_OK = 0,
    KV_ERR_INVALID = -1,     /* bad argument (null pointer, bad size, misalignment) */
    KV_ERR_UNSUPPORTED = -2, /* valid but not built (e.g. head_dim != 128) */
    KV_ERR_CUDA = -3,        /* a CUDA runtime call failed */
    KV_ERR_OOB = -4,         /* a kernel skipped work on an out-of-range index */
    KV_ERR_TIMEOUT = -5,     /* a kernel gave up a bounded wait (should never happen) */
    KV_ERR_SCRATCH_TOO_SMALL = -6 /* kv_decode_attn_noalloc: the call needs more than
                                     KV_NOALLOC_SCRATCH_BYTES of scratch; nothing launched */
} kv_status;

typedef enum {
    KV_BF16 = 0,     /* unquantised bf16 pages (comparator) */
    KV_INT4 = 1,     /* token-wise INT4, no rotation ("naive INT4") */
    KV_INT4_BDR = 2  /* token-wise INT4 after the block-diagonal Hadamard rotation */
} kv_mode;

typedef struct {
    int num_pages;    /* pages in each pool; num_pages * num_kv_heads * page_size < 2^32 */
    int page_size;    /* tokens per page, 1..1024 */
    int num_kv_heads; /* H_kv: 1, 2, 4, 8, 16 or 32 */
    int num_q_heads;  /* H_q = G * H_kv with G in {1, 2, 4, 8} */
    int head_dim;     /* must be 128 */
    int mode;         /* kv_mode */
    int bdr_block;    /* 16, 32, 64 or 128 for KV_INT4_BDR (ignored otherwise) */
    int rotate_v;     /* KV_INT4_BDR only: 0 = rotate keys only, 1 = keys and values */
    void* k_pool;     /* device pools, layouts above; 32-byte aligned */
    void* v_pool;
    void* k_sz;       /* device fp16x2 scale/zero arrays (INT4 modes), 16-byte aligned; NULL for BF16 */
    void* v_sz;
    /* Optional fused rotary embedding: NULL = off.  Else a device float32 table
     * [rope_positions][head_dim/2][2] (cos, sin) of each position's angle for the
     * rotate-half pairs (i, i + head_dim/2), 16-byte aligned, owned by the caller.
     * kv_append_quant turns each key row at its tok_pos (fp32, before the block
     * rotation; BF16 pages store the turned row rounded to nearest even);
     * kv_decode_attn turns q at position seq_len - 1 (the newest token).  A
     * position outside the table skips the token (append) or the sequence (decode:
     * zero output), flagged KV_ERR_OOB. */
    const float* rope;
    int rope_positions; /* rows of the table (>= 1 when rope is set) */
    /* Code width of the INT4 modes: 0 or 4 = 4-bit codes; 2 = the 2-bit variant (the
     * same token-wise asymmetric quantiser with range/3, codes 0..3, four per byte,
     * code k of a byte in bits 2k and 2k+1; the pages leave 2-bit open). */
    int code_bits;
} kv_desc;

typedef struct kv_cache kv_cache; /* opaque host handle */

/* Validate a descriptor and create a handle (host only, no kernel).
 * [ABS] (paged layouts), [WIS1] (fixed-size pages).  The handle records the
 * caller's pool pointers; the caller keeps the pools alive until kv_free. */
kv_status kv_create_paged(const kv_desc* desc, kv_cache** out);

/* Append num_tokens new tokens: one launch of the fused kernel that rotates
 * (keys, and values if rotate_v) with H_blk, quantises each (token, KV head)
 * row to INT4 with its own scale and zero, packs the nibbles and stores codes
 * and scale/zero into the page slot -- K~ = quant(K H_blk), V~ = quant(V H_blk)
 * fused into the KV-cache write ([WIS3], [ABS]).  In KV_BF16 mode the rows are
 * copied unchanged.
 *  k, v        device bf16 [num_tokens, num_kv_heads, head_dim], 16-B aligned
 *  tok_seq     device int32 [num_tokens]: sequence (page-table row) of token i
 *  tok_pos     device int32 [num_tokens]: its position within that sequence
 *  page_table  device int32 [num_seqs, pt_stride]
 * Two tokens must not target the same slot in one call.  num_tokens == 0 is a
 * no-op; num_tokens * num_kv_heads above INT32_MAX rows is KV_ERR_INVALID.
 * Out-of-range sequence ids, positions or page ids are skipped and flagged
 * (KV_ERR_OOB via kv_get_error). */
kv_status kv_append_quant(kv_cache* cache, const void* k, const void* v, int num_tokens,
                          const int32_t* tok_seq, const int32_t* tok_pos, const int32_t* page_table,
                          int pt_stride, int num_seqs, void* stream);

/* Bytes of device workspace kv_decode_attn needs for this batch and bound on
 * sequence length (split-K partial outputs and softmax statistics). */
size_t kv_decode_workspace_bytes(const kv_cache* cache, int batch, int max_seq_len);

/* Paged GQA decode attention, one query token per sequence: rotate q with the
 * same H_blk ([WIS3]: query rotated in step), walk the sequence's pages,
 * dequantise K/V in registers, softmax(q' k^T / sqrt(D)) v over all
 * seq_lens[b] cached tokens, split-K with a log-sum-exp merge, rotate the
 * output back when values are rotated ([ABS]: fused attention execution over
 * the paged INT4 cache).
 *  q           device bf16 [batch, num_q_heads, head_dim]
 *  seq_lens    device int32 [batch], each in [0, max_seq_len]; 0 gives a zero row
 *  page_table  device int32 [batch, pt_stride]
 *  out         device [batch, num_q_heads, head_dim], bf16 (out_fp32 == 0) or
 *              fp32 (out_fp32 != 0); the bf16 output is the fp32 one rounded
 *              to nearest even
 *  workspace   device, >= kv_decode_workspace_bytes(cache, batch, max_seq_len)
 *              bytes, 16-B aligned (may be NULL when that size is 0) */
kv_status kv_decode_attn(kv_cache* cache, const void* q, const int32_t* seq_lens,
                         const int32_t* page_table, int pt_stride, int batch, int max_seq_len,
                         void* out, int out_fp32, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Size of the fixed device scratch array behind kv_decode_attn_noalloc. */
#define KV_NOALLOC_SCRATCH_BYTES (8u << 20) /* 8 MiB, held on every GPU that loads the library */

/* kv_decode_attn without a workspace argument, for callers that cannot allocate
 * device memory when they decode: code running inside an allocator or memory pool
 * that must not re-enter itself, runtimes that fix their device-memory budget up
 * front, and plain-C hosts with no device allocator of their own.  (This entry
 * point has no counterpart in the SAW-INT4 paper; it only changes where the
 * split-K scratch lives.)
 *
 * Same arguments, kernels and results as kv_decode_attn, but the split-K scratch
 * is a library-owned, file-scope device array of KV_NOALLOC_SCRATCH_BYTES; the
 * call allocates nothing.  Calls whose scratch need,
 * kv_decode_workspace_bytes(cache, batch, max_seq_len), exceeds that size return
 * KV_ERR_SCRATCH_TOO_SMALL before launching anything.
 *  - The first call for a handle on a given device looks up the array's device
 *    address there with cudaGetSymbolAddress (the call makes the handle's device
 *    current while it runs); make that first call before any stream capture on
 *    the device.
 *  - Every call shares the one array: calls whose kernels may overlap on the GPU
 *    (different streams, unsynchronised threads) race on it; order them on one
 *    stream.  No part of the array needs to start at zero: each call writes all
 *    the scratch it later reads. */
kv_status kv_decode_attn_noalloc(kv_cache* cache, const void* q, const int32_t* seq_lens,
                                 const int32_t* page_table, int pt_stride, int batch, int max_seq_len,
                                 void* out, int out_fp32, void* stream);

/* Extend (chunked-prefill) attention over the INT4 cache: the n_s newest tokens of
 * sequence s, already written by kv_append_quant, attend causally to the cached
 * tokens ([ABS]: fused attention execution over the paged quantised cache, which
 * chunked prefill in mixed serving reads this way).  Query i (0-based) of sequence s
 * sits at position p = seq_lens[s] - n_s + i and its output row is exactly what
 * kv_decode_attn gives for that query with seq_len = p + 1: q turned by the rotary
 * table at position p (when set), rotated with H_blk ([WIS3]), softmax over tokens
 * 0 .. p, output rotated back when values are rotated.
 *  q           device bf16 [total_q, num_q_heads, head_dim], total_q = q_indptr[batch]
 *  q_indptr    device int32 [batch + 1], non-decreasing, q_indptr[0] = 0: the queries
 *              of sequence s are rows q_indptr[s] .. q_indptr[s + 1] - 1 of q and out
 *  seq_lens    device int32 [batch]: cached tokens of s, its new ones included
 *  page_table  device int32 [batch, pt_stride]
 *  max_q_len   >= every n_s (host bound; sizes the grid), max_seq_len >= every seq_len
 *  out         device [total_q, num_q_heads, head_dim], bf16 (round to nearest even of
 *              the fp32 value) or fp32 (out_fp32 != 0)
 * No workspace; one launch.  KV_BF16 pages or batch > 65535: KV_ERR_UNSUPPORTED.  Flagged
 * (KV_ERR_OOB via kv_get_error): n_s > max_q_len (the queries before the last
 * max_q_len ones are not computed), p < 0 (n_s > seq_len: zero row), p outside the
 * rotary table (zero row), p + 1 beyond the page table or max_seq_len (clamped as in
 * kv_decode_attn), page ids outside the pool (token skipped). */
kv_status kv_extend_attn(kv_cache* cache, const void* q, const int32_t* q_indptr, const int32_t* seq_lens,
                         const int32_t* page_table, int pt_stride, int batch, int max_q_len, int max_seq_len,
                         void* out, int out_fp32, void* stream);

/* Synchronise the stream, then read and clear the device error word:
 * KV_OK, KV_ERR_OOB or KV_ERR_TIMEOUT (KV_ERR_CUDA if the runtime failed). */
kv_status kv_get_error(kv_cache* cache, void* stream);

/* Release the handle and its device error word.  NULL is a no-op. */
void kv_free(kv_cache* cache);

/* Static, human-readable name of a kv_status value. */
const char* kv_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
