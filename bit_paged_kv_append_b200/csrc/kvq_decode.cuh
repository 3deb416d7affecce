// kvq_decode.cuh -- what the decode kernels share: the parameter block, the
// workspace layout and the fragment-slot -> head_dim permutation.
//
// A decode call is two kernels on one stream:
//   split  one CTA per (split k, KV head h, sequence s): attention of the G query
//          heads of group h over cached tokens [k * item_tokens, (k+1) * item_tokens)
//          of sequence s -> unnormalised partial output + softmax statistics
//          (kvq_decode_mma.cu for INT4 pages, kvq_decode.cu for BF16 pages);
//          CTAs past the end of their sequence exit at once.
//   merge  one warp per (sequence, query head): log-sum-exp merge of its splits,
//          output rotation, bf16/fp32 store (kvq_decode.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq_internal.h"

namespace kvq {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxGroup = 8;  // query heads per KV head

struct DecodeParams {
    CacheGeom g;
    DecodeArgs a;
    int item_tokens;  // cached tokens per split, a multiple of 64
    int max_splits;   // ceil(max_seq_len / item_tokens), >= 1
    float qscale;     // 1/sqrt(D) * log2(e): scores live in the log2 domain
    int ps_shift;     // log2(page_size) when it is a power of two, else -1
    float* ws_o;      // [B][max_splits][Hq][D] unnormalised partial outputs
    float2* ws_ml;    // [B][max_splits][Hq] (running max, sum of weights)
    int* err;
};

// Row of the partial arrays for (sequence s, split k, query head j).
__host__ __device__ inline int64_t partial_row(const DecodeParams& p, int s, int k, int j) {
    return (int64_t(s) * p.max_splits + k) * p.g.Hq + j;
}

// Dimension d that column k of q.K k-step j stands for.  Thread-in-group pp of
// an mma reads bytes [16 pp, 16 pp + 16) of a packed code row (dims 32 pp ..
// 32 pp + 31); word i = j / 2 of them yields the code pairs (n0, n4), (n1, n5)
// of k-step 2i and (n2, n6), (n3, n7) of k-step 2i + 1, the second of each
// from the high nibbles (x16, so those dims carry a factor 1/16 in A).
__host__ __device__ constexpr int dpos(int j, int k) {
    return 32 * ((k & 7) >> 1) + 8 * (j >> 1) + ((j & 1) ? 2 : 0) + (k >> 3) + 4 * (k & 1);
}

#ifdef __CUDACC__
// Cached length of sequence s, clamped to what the page table and the bound allow; 0 when
// the fused rotary embedding has no table row for the query's position L - 1.
__device__ __forceinline__ int decode_len(const DecodeParams& p, int s) {
    const int L = __ldg(p.a.seq_lens + s);
    if (p.g.rope && L > p.g.rope_positions) return 0;
    const int cap = min(p.a.pt_stride * p.g.page_size, p.a.max_seq_len);
    return L < 0 ? 0 : (L > cap ? cap : L);
}

// Page-table index and slot of token position t (shifts for power-of-two page sizes).
__device__ __forceinline__ int page_of_pos(const DecodeParams& p, int t) {
    return p.ps_shift >= 0 ? (t >> p.ps_shift) : t / p.g.page_size;
}
__device__ __forceinline__ int slot_of_pos(const DecodeParams& p, int t) {
    return p.ps_shift >= 0 ? (t & (p.g.page_size - 1)) : t % p.g.page_size;
}

__device__ __forceinline__ float fast_exp2(float x) {  // MUFU ex2; exp2(-inf) = +0
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
#endif

// Tensor-core split kernel for the INT4 modes (grid: max_splits x H x B).
cudaError_t launch_decode_mma(const DecodeParams& p, cudaStream_t s);
// Tensor-core split kernel for BF16 pages (grid: max_splits x H x B).
cudaError_t launch_decode_bf16(const DecodeParams& p, cudaStream_t s);

}  // namespace kvq
