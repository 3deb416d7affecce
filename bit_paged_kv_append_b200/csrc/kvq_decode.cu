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

constexpr int kMergeWarps = 4;  // (sequence, query head) rows per merge CTA, one warp each
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

// One warp per (sequence, query head) row, lane l owning dims 4l .. 4l + 3: merge the
// sequence's splits (statistics 32 splits at a time, one per lane, their maximum and
// weighted sum by shuffles, the next pass's statistics fetched before this pass's rows;
// partial outputs 8 splits at a time as float4), normalise, rotate back when values were
// rotated (o H_blk; H_blk is its own inverse: butterflies of stride 1 and 2 within a
// lane, 4 .. 64 across lanes), store bf16 (round to nearest even of the fp32 value) or
// fp32.  An empty sequence gives zeros.  With share_rows (few rows of many splits) the
// CTA's warps share one row, warp w taking passes w, w + 4, ..., and warp 0 combines
// their (max, sum, vector) through shared memory; otherwise each warp finishes its row
// alone, with no block barrier.
__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(Params p, int rotate_out, int share_rows) {
    __shared__ float4 part_v[kMergeWarps][32];
    __shared__ float2 part_ml[kMergeWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hq = p.g.Hq;
    const int row = share_rows ? blockIdx.x : blockIdx.x * kMergeWarps + warp;  // s * Hq + j
    const int k_first = share_rows ? 32 * warp : 0;
    const int k_step = share_rows ? 32 * kMergeWarps : 32;
    grid_dep_wait();  // the split kernel's partials
    grid_dep_launch();
    if (row >= p.a.batch * Hq) return;  // whole warps (with share_rows, the whole CTA)
    const int s = row / Hq, j = row % Hq;
    const int n = (decode_len(p, s) + p.item_tokens - 1) / p.item_tokens;
    const int64_t stride4 = int64_t(Hq) * (kHeadDim / 4);  // next split, same query head, in float4
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float l = 0.0f, M = -INFINITY;
    float2 ml = k_first + lane < n ? p.ws_ml[partial_row(p, s, k_first + lane, j)] : make_float2(-INFINITY, 0.0f);
    for (int k0 = k_first; k0 < n; k0 += k_step) {
        const int cnt = min(32, n - k0);
        const int kn = k0 + k_step + lane;
        const float2 ml_next = kn < n ? p.ws_ml[partial_row(p, s, kn, j)] : make_float2(-INFINITY, 0.0f);
        const float Mn = fmaxf(M, warp_max(ml.x));
        const float f = (ml.x == -INFINITY) ? 0.0f : fast_exp2(ml.x - Mn);  // this lane's split weight
        const float rescale = (M == -INFINITY) ? 0.0f : fast_exp2(M - Mn);
        l = l * rescale + warp_sum(f * ml.y);
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] *= rescale;
        M = Mn;
        ml = ml_next;
        const float4* src = reinterpret_cast<const float4*>(p.ws_o + partial_row(p, s, k0, j) * kHeadDim) + lane;
        int t = 0;
        for (; t + 8 <= cnt; t += 8) {
            float4 o[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) o[u] = src[(t + u) * stride4];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float w = __shfl_sync(0xffffffffu, f, t + u);
                v[0] += w * o[u].x;
                v[1] += w * o[u].y;
                v[2] += w * o[u].z;
                v[3] += w * o[u].w;
            }
        }
        for (; t < cnt; ++t) {
            const float4 o = src[t * stride4];
            const float w = __shfl_sync(0xffffffffu, f, t);
            v[0] += w * o.x;
            v[1] += w * o.y;
            v[2] += w * o.z;
            v[3] += w * o.w;
        }
    }
    if (share_rows) {
        part_v[warp][lane] = make_float4(v[0], v[1], v[2], v[3]);
        if (lane == 0) part_ml[warp] = make_float2(M, l);
        __syncthreads();
        if (warp != 0) return;
        float Mt = part_ml[0].x;
#pragma unroll
        for (int w = 1; w < kMergeWarps; ++w) Mt = fmaxf(Mt, part_ml[w].x);
        l = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = 0.0f;
#pragma unroll
        for (int w = 0; w < kMergeWarps; ++w) {
            const float2 wm = part_ml[w];
            const float f = (wm.x == -INFINITY) ? 0.0f : fast_exp2(wm.x - Mt);
            const float4 pv = part_v[w][lane];
            l += f * wm.y;
            v[0] += f * pv.x;
            v[1] += f * pv.y;
            v[2] += f * pv.z;
            v[3] += f * pv.w;
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) v[c] = l > 0.0f ? v[c] / l : 0.0f;
    if (rotate_out) {
        const int b = p.g.bdr_block;  // 16 .. 128
        // element 4 lane + c; at stride hs the lower element of each pair takes a + d, the
        // upper a - d
#pragma unroll
        for (int hs = 1; hs < 4; hs <<= 1) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if ((c & hs) == 0) {
                    const float a = v[c], d = v[c + hs];
                    v[c] = a + d;
                    v[c + hs] = a - d;
                }
            }
        }
        for (int hs = 4; hs < b; hs <<= 1) {
            const int ls = hs >> 2;  // partner lane distance
            const bool upper = (lane & ls) != 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float other = __shfl_xor_sync(0xffffffffu, v[c], ls);
                v[c] = upper ? other - v[c] : v[c] + other;
            }
        }
        const float r = rsqrtf(float(b));
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] *= r;
    }
    const int64_t o = int64_t(row) * kHeadDim + 4 * lane;  // out is 16-byte aligned (checked by the API)
    if (p.a.out_fp32) {
        *reinterpret_cast<float4*>(static_cast<float*>(p.a.out) + o) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t*>(&lo);
        w.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.a.out) + o) = w;
    }
}

template <int G>
cudaError_t launch_group(const Params& p, int num_sms, cudaStream_t st) {
    const cudaError_t e = p.g.mode == 0 ? launch_decode_bf16(p, st) : launch_decode_mma(p, st);
    if (e != cudaSuccess) return e;
    // few rows of more than one pass of splits (long sequences, small batches): the CTA's
    // warps share a row
    const int rows = p.a.batch * p.g.Hq;
    const int share = p.max_splits > 32 && rows <= 4 * (num_sms > 0 ? num_sms : 148);
    const int grid = share ? rows : (rows + kMergeWarps - 1) / kMergeWarps;
    return launch_overlapped(merge_kernel, dim3(grid), dim3(kMergeWarps * 32), 0, st, p,
                             int(p.g.mode == 2 && p.g.rotate_v), share);
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
        case 1: return launch_group<1>(p, plan.num_sms, s);
        case 2: return launch_group<2>(p, plan.num_sms, s);
        case 4: return launch_group<4>(p, plan.num_sms, s);
        case 8: return launch_group<8>(p, plan.num_sms, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
