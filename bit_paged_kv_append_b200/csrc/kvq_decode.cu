// kvq_decode.cu -- paged GQA decode attention: planning and the split-K merge
// kernel.  The split kernels (tensor cores) are in kvq_decode_mma.cu (INT4 pages)
// and kvq_decode_bf16.cu (BF16 pages).
//
// SAW-INT4 (wispaper.ai blog, section 3): the query is rotated in step with
// H_blk at inference, so (q H)(k H)^T = q k^T and attention runs directly on
// the rotated, quantised keys; the abstract keeps fused attention over the
// paged layout.  When values are rotated too, the output is rotated back with
// the same H_blk (it is its own inverse).
//
// Work is cut into splits of item_tokens cached tokens of one (sequence, KV
// head): one CTA each, CTAs past the end of their sequence exit at once, and the
// merge reads only the splits a sequence has.  Scores are kept in the log2
// domain (q is pre-scaled by log2(e) / sqrt(D)); partial outputs are
// unnormalised.
#include "kvq_common.cuh"
#include "kvq_decode.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
using Params = DecodeParams;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------- merge --------

// One CTA per (sequence, query head): merge the sequence's splits (statistics
// fetched once, 128 splits at a time, partial outputs loaded 8 at a time),
// normalise, rotate back
// when values were rotated (o H_blk; H_blk is its own inverse), store bf16 (round
// to nearest even of the fp32 value) or fp32.  An empty sequence gives zeros.
__global__ void __launch_bounds__(kThreads) merge_kernel(Params p, int rotate_out) {
    __shared__ float wts[kThreads];
    __shared__ float red[2][kWarps];
    __shared__ float buf[kHeadDim];
    const int row = blockIdx.x;  // s * Hq + j
    const int Hq = p.g.Hq;
    const int s = row / Hq, j = row % Hq;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dep_wait();  // the split kernel's partials
    grid_dep_launch();
    const int n = (decode_len(p, s) + p.item_tokens - 1) / p.item_tokens;
    const int64_t stride = int64_t(Hq) * kHeadDim;  // next split, same query head
    float acc = 0.0f, l = 0.0f, M = -INFINITY;
    // splits in tiles of 128: thread t fetches the statistics of split k0 + t, the tile's
    // weights go through shared memory, every thread then sums its dimension over the tile
    for (int k0 = 0; k0 < n; k0 += kThreads) {
        const int cnt = min(kThreads, n - k0);
        const float2 ml = tid < cnt ? p.ws_ml[partial_row(p, s, k0 + tid, j)] : make_float2(-INFINITY, 0.0f);
        float tm = warp_max(ml.x);
        if (lane == 0) red[0][warp] = tm;
        __syncthreads();
        tm = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
        const float Mn = fmaxf(M, tm);
        const float f = (ml.x == -INFINITY) ? 0.0f : fast_exp2(ml.x - Mn);
        wts[tid] = f;
        const float lt = warp_sum(f * ml.y);
        if (lane == 0) red[1][warp] = lt;
        __syncthreads();
        const float rescale = (M == -INFINITY) ? 0.0f : fast_exp2(M - Mn);
        l = l * rescale + (red[1][0] + red[1][1] + red[1][2] + red[1][3]);
        acc *= rescale;
        M = Mn;
        const float* src = p.ws_o + partial_row(p, s, k0, j) * kHeadDim + tid;
        int t = 0;
        for (; t + 8 <= cnt; t += 8) {
            float o[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) o[u] = src[(t + u) * stride];
#pragma unroll
            for (int u = 0; u < 8; ++u) acc += wts[t + u] * o[u];
        }
        for (; t < cnt; ++t) acc += wts[t] * src[t * stride];
        __syncthreads();
    }
    float res = l > 0.0f ? acc / l : 0.0f;
    if (rotate_out) {
        buf[tid] = res;
        __syncthreads();
        for (int hs = 1; hs < p.g.bdr_block; hs <<= 1) {
            const float mine = buf[tid], other = buf[tid ^ hs];
            const float nv = (tid & hs) ? other - mine : mine + other;
            __syncthreads();
            buf[tid] = nv;
            __syncthreads();
        }
        res = buf[tid] * rsqrtf(float(p.g.bdr_block));
    }
    const int64_t o = int64_t(row) * kHeadDim + tid;
    if (p.a.out_fp32)
        static_cast<float*>(p.a.out)[o] = res;
    else
        static_cast<__nv_bfloat16*>(p.a.out)[o] = __float2bfloat16_rn(res);
}

template <int G>
cudaError_t launch_group(const Params& p, cudaStream_t st) {
    const cudaError_t e = p.g.mode == 0 ? launch_decode_bf16(p, st) : launch_decode_mma(p, st);
    if (e != cudaSuccess) return e;
    return launch_overlapped(merge_kernel, dim3(p.a.batch * p.g.Hq), dim3(kThreads), 0, st, p,
                             int(p.g.mode == 2 && p.g.rotate_v));
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

DecodePlan plan_decode(const CacheGeom& g, int batch, int max_seq_len, int num_sms) {
    // Splits of a multiple of 64 tokens (4 warps x 16-token chunks), between 512 and 4096
    // tokens, sized so that a full batch at the length bound gives about 2.75 waves of
    // resident split CTAs (5 per SM).  Measured on B200 over batch sizes 1..256 and
    // lengths 2k..1M: shorter splits pay their start-up and merge more often, longer ones
    // leave a tail; 4096 also bounds how many steps one warp accumulates.
    DecodePlan pl;
    const int64_t L = max_seq_len > 0 ? max_seq_len : 1;
    const int64_t slots = int64_t(num_sms > 0 ? num_sms : 148) * 5;
    int64_t it = (int64_t(batch) * g.H * L * 4 + 11 * slots - 1) / (11 * slots);
    it = ((it + 63) / 64) * 64;
    if (it < 512) it = 512;
    // BF16 pages move 4 KiB a token and their split kernel holds 2 CTAs per SM: splits of at
    // least 2048 tokens (measured: batch16 40.0 -> 37.8 us, the long workloads unchanged)
    if (g.mode == 0 && it < 2048) it = 2048;
    if (it > 4096) it = 4096;
    pl.item_tokens = int(it);
    pl.max_splits = int((L + it - 1) / it);
    pl.max_items = batch * pl.max_splits;
    pl.num_sms = num_sms;
    const size_t rows = size_t(pl.max_items) * size_t(g.Hq);
    pl.ws_bytes = align256(rows * kHeadDim * sizeof(float)) + rows * sizeof(float2);
    return pl;
}

cudaError_t launch_decode(const CacheGeom& g, const DecodeArgs& a, const DecodePlan& plan, int* err_word,
                          cudaStream_t s) {
    if (a.batch == 0) return cudaSuccess;
    const size_t rows = size_t(plan.max_items) * size_t(g.Hq);
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    Params p;
    p.g = g;
    p.a = a;
    p.item_tokens = plan.item_tokens;
    p.max_splits = plan.max_splits;
    p.qscale = float(1.0 / sqrt(double(kHeadDim))) * kLog2e;
    p.ps_shift = -1;
    for (int sh = 0; sh < 11; ++sh)
        if ((1 << sh) == g.page_size) p.ps_shift = sh;
    p.ws_o = reinterpret_cast<float*>(ws);
    p.ws_ml = reinterpret_cast<float2*>(ws + align256(rows * kHeadDim * sizeof(float)));
    p.err = err_word;
    switch (g.Hq / g.H) {
        case 1: return launch_group<1>(p, s);
        case 2: return launch_group<2>(p, s);
        case 4: return launch_group<4>(p, s);
        case 8: return launch_group<8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
