// kvq_decode.cu -- paged GQA decode attention: planning, the CUDA-core split
// kernel used for BF16 pages and the split-K merge kernel.  The INT4 split
// kernel (tensor cores) is in kvq_decode_mma.cu.
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

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

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

// ---------------------------------------------------- CUDA-core split (BF16) ---

// One CTA per (split k, KV head h, sequence s) over bf16 pages.  Lanes own tokens
// for q.k and head_dim slices for P.V (staged per warp), online softmax per query
// head, the 4 warps merged in shared memory.
template <int G>
struct Bf16Smem {
    float qs[G][kHeadDim];
    union {
        struct {
            float pt[kWarps][32][G];
            uint32_t v[kWarps][32][65];  // staged V rows (+1 word: no bank conflicts)
        } loop;
        struct {
            float m[kWarps][G];
            float l[kWarps][G];
            float o[kWarps][G][kHeadDim];
        } merge;
    } u;
};

template <int G>
__global__ void __launch_bounds__(kThreads) bf16_split_kernel(Params p) {
    __shared__ Bf16Smem<G> sm;
    const int k = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.g.H, Hq = p.g.Hq, ps = p.g.page_size;
    const int L = decode_len(p, s);
    if (k == 0 && h == 0 && tid == 0 && L != __ldg(p.a.seq_lens + s)) flag_error(p.err, kErrOOB);
    const int t0 = k * p.item_tokens;
    if (t0 >= L) {  // past the end of the sequence
        grid_dep_wait();  // still: no grid here completes before the one it follows
        grid_dep_launch();
        return;
    }
    const int t1 = min(L, t0 + p.item_tokens);
    const int64_t out_row0 = partial_row(p, s, k, h * G);

    const uint16_t* q = static_cast<const uint16_t*>(p.a.q) + (int64_t(s) * Hq + h * G) * kHeadDim;
    if (p.g.rope) {  // fused rotary embedding at position seq_len - 1: pairs (i, i + 64)
#pragma unroll
        for (int g = 0; g < G; ++g) sm.qs[g][tid] = __uint_as_float(uint32_t(q[g * kHeadDim + tid]) << 16);
        __syncthreads();
        const int pos = __ldg(p.a.seq_lens + s) - 1;
        const int i = tid & 63;
        const float c = __ldg(p.g.rope + int64_t(pos) * kHeadDim + 2 * i);
        const float sn = __ldg(p.g.rope + int64_t(pos) * kHeadDim + 2 * i + 1);
        float turned[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float own = sm.qs[g][tid], other = sm.qs[g][tid ^ 64];
            turned[g] = tid < 64 ? fmaf(own, c, -other * sn) : fmaf(own, c, other * sn);
        }
        __syncthreads();
#pragma unroll
        for (int g = 0; g < G; ++g) sm.qs[g][tid] = turned[g] * p.qscale;
    } else {
#pragma unroll
        for (int g = 0; g < G; ++g) sm.qs[g][tid] = __uint_as_float(uint32_t(q[g * kHeadDim + tid]) << 16) * p.qscale;
    }
    __syncthreads();

    float m[G], lsum[G], o[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        lsum[g] = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) o[g][e] = 0.0f;
    }
    const int32_t* pt = p.a.page_table + int64_t(s) * p.a.pt_stride;
    grid_dep_wait();  // the cache as the previous grid (an append) left it
    grid_dep_launch();

    for (int base = t0 + 32 * warp; base < t1; base += 32 * kWarps) {
        const int t = base + lane;
        bool valid = t < t1;
        int64_t row = 0;
        if (valid) {
            const int page = __ldg(pt + page_of_pos(p, t));
            if (page < 0 || page >= p.g.num_pages) {
                flag_error(p.err, kErrOOB);
                valid = false;
            } else {
                row = (int64_t(page) * H + h) * ps + slot_of_pos(p, t);
            }
        }
        float sc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) sc[g] = -INFINITY;
        if (valid) {
            float acc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = 0.0f;
            const uint4* kr = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.g.k_pool) + row * 256);
#pragma unroll 4
            for (int j = 0; j < 16; ++j) {
                const uint4 w = __ldg(kr + j);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float k0 = bf16_lo(ww[e]), k1 = bf16_hi(ww[e]);
                    const int d = 8 * j + 2 * e;
#pragma unroll
                    for (int g = 0; g < G; ++g) acc[g] += sm.qs[g][d] * k0 + sm.qs[g][d + 1] * k1;
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) sc[g] = acc[g];
        }
        float pg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mnew = fmaxf(m[g], warp_max(sc[g]));
            const float alpha = (mnew == -INFINITY) ? 1.0f : exp2f(m[g] - mnew);
            pg[g] = valid ? exp2f(sc[g] - mnew) : 0.0f;
            m[g] = mnew;
            lsum[g] = lsum[g] * alpha + pg[g];
#pragma unroll
            for (int e = 0; e < 4; ++e) o[g][e] *= alpha;
        }
        uint32_t* vs = sm.u.loop.v[warp][lane];
        if (valid) {
            const uint4* vr = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.g.v_pool) + row * 256);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint4 w = __ldg(vr + j);
                vs[4 * j + 0] = w.x;
                vs[4 * j + 1] = w.y;
                vs[4 * j + 2] = w.z;
                vs[4 * j + 3] = w.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) vs[j] = 0u;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) sm.u.loop.pt[warp][lane][g] = pg[g];
        __syncwarp();
        const int ntok = min(32, t1 - base);
        for (int j = 0; j < ntok; ++j) {
            const uint32_t w0 = sm.u.loop.v[warp][j][2 * lane], w1 = sm.u.loop.v[warp][j][2 * lane + 1];
            const float vv[4] = {bf16_lo(w0), bf16_hi(w0), bf16_lo(w1), bf16_hi(w1)};
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float wgt = sm.u.loop.pt[warp][j][g];
#pragma unroll
                for (int e = 0; e < 4; ++e) o[g][e] += wgt * vv[e];
            }
        }
        __syncwarp();
    }
#pragma unroll
    for (int g = 0; g < G; ++g) lsum[g] = warp_sum(lsum[g]);
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (lane == 0) {
            sm.u.merge.m[warp][g] = m[g];
            sm.u.merge.l[warp][g] = lsum[g];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) sm.u.merge.o[warp][g][4 * lane + e] = o[g][e];
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.u.merge.m[w][g]);
        float acc = 0.0f, lt = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float mw = sm.u.merge.m[w][g];
            const float f = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
            acc += f * sm.u.merge.o[w][g][tid];
            lt += f * sm.u.merge.l[w][g];
        }
        p.ws_o[(out_row0 + g) * kHeadDim + tid] = acc;
        if (tid == 0) p.ws_ml[out_row0 + g] = make_float2(M, lt);
    }
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
    const int B = p.a.batch, H = p.g.H;
    cudaError_t e;
    if (p.g.mode == 0) {
        e = launch_overlapped(bf16_split_kernel<G>, dim3(p.max_splits, H, B), dim3(kThreads), 0, st, p);
    } else {
        e = launch_decode_mma(p, st);
    }
    if (e != cudaSuccess) return e;
    return launch_overlapped(merge_kernel, dim3(B * p.g.Hq), dim3(kThreads), 0, st, p,
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
