// kvq_decode.cu -- paged GQA decode attention over the INT4 (or BF16) cache,
// split-K over the context with a log-sum-exp merge.
//
// SAW-INT4 (wispaper.ai blog, section 3): the query is rotated in step with
// H_blk at inference, so (q H)(k H)^T = q k^T and attention can run directly on
// the rotated, quantised keys; the abstract names fused attention execution
// over the paged layout as a serving constraint the method keeps.  INT4 K/V
// are dequantised in registers; nothing is expanded to memory.
//
// Kernel 1 (decode_split_kernel): one CTA per (split, KV head, sequence), 4
// warps.  The prologue loads the G = Hq / H_kv query rows of the head group,
// rotates them (fp32 FWHT in shared memory, same block as the cache) and folds
// in the softmax scale 1/sqrt(D) * log2(e).  Each warp then walks 32-token
// groups of its split: lanes own tokens for q.k (factored dequantisation:
// s = scale * (q'.c) + zero * sum(q')), an online softmax per query head, then
// lanes own head_dim slices for P.V out of a per-warp staging buffer.  The 4
// warps merge in shared memory and write one unnormalised partial
// (o, m, l) per (split, sequence, query head) to the workspace.
// Kernel 2 (merge_kernel): per (sequence, query head), merge the splits,
// normalise, rotate the output back when values were rotated, store bf16 or
// fp32.
#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
    CacheGeom g;
    DecodeArgs a;
    int num_splits;
    int chunk;
    float qscale;  // 1/sqrt(D) * log2(e)
    float* ws_o;   // [splits, B, Hq, D]
    float2* ws_ml; // [splits, B, Hq]: (max, sum) in the log2 domain
    int* err;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Nibble k of w as the exact float 1 + c/16 (c in 0..15).
__device__ __forceinline__ float nib1p(uint32_t w, int k) {
    const uint32_t c = (w >> (4 * k)) & 15u;
    return __uint_as_float(0x3F800000u | (c << 19));
}

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

template <int MODE, int G>
struct DecodeSmem {
    static constexpr int kVWords = MODE == 0 ? 64 : 16;  // words per staged V row
    float qs[G][kHeadDim];
    float qsum[G];
    union {
        struct {
            float pt[kWarps][32][G];                // p (BF16) or p * scale_v (INT4) per token
            uint32_t v[kWarps][32][kVWords + 1];     // staged V rows (+1 word: no bank conflicts)
        } loop;
        struct {
            float m[kWarps][G];
            float l[kWarps][G];
            float o[kWarps][G][kHeadDim];
        } merge;
    } u;
};

template <int MODE, int G>
__global__ void __launch_bounds__(kThreads) decode_split_kernel(Params p) {
    using Smem = DecodeSmem<MODE, G>;
    __shared__ Smem sm;
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.g.H, Hq = p.g.Hq, ps = p.g.page_size;
    const int B = p.a.batch;

    int L = __ldg(p.a.seq_lens + b);
    const int cap = p.a.pt_stride * ps;
    if (L > cap || L > p.a.max_seq_len || L < 0) {
        if (split == 0 && h == 0 && tid == 0) flag_error(p.err, kErrOOB);
        L = L < 0 ? 0 : min(L, min(cap, p.a.max_seq_len));
    }
    const int t0 = split * p.chunk;
    const int t1 = min(L, t0 + p.chunk);
    const int64_t out_row0 = (int64_t(split) * B + b) * Hq + h * G;  // first query head of the group

    if (t0 >= t1) {  // empty split: neutral partial
        for (int i = tid; i < G * kHeadDim; i += kThreads) p.ws_o[out_row0 * kHeadDim + i] = 0.0f;
        if (tid < G) p.ws_ml[out_row0 + tid] = make_float2(-INFINITY, 0.0f);
        return;
    }

    // ---- prologue: q' = q H_blk (mode 2), times 1/sqrt(D) log2(e) ----
    const uint16_t* q = static_cast<const uint16_t*>(p.a.q) + (int64_t(b) * Hq + h * G) * kHeadDim;
#pragma unroll
    for (int g = 0; g < G; ++g) sm.qs[g][tid] = __uint_as_float(uint32_t(q[g * kHeadDim + tid]) << 16);
    __syncthreads();
    if (MODE == 2) {
        for (int hs = 1; hs < p.g.bdr_block; hs <<= 1) {
            float nv[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float mine = sm.qs[g][tid], other = sm.qs[g][tid ^ hs];
                nv[g] = (tid & hs) ? other - mine : mine + other;
            }
            __syncthreads();
#pragma unroll
            for (int g = 0; g < G; ++g) sm.qs[g][tid] = nv[g];
            __syncthreads();
        }
    }
    {
        const float sc = (MODE == 2 ? rsqrtf(float(p.g.bdr_block)) : 1.0f) * p.qscale;
#pragma unroll
        for (int g = 0; g < G; ++g) sm.qs[g][tid] *= sc;
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float s = 0.0f;
            for (int d = lane; d < kHeadDim; d += 32) s += sm.qs[g][d];
            s = warp_sum(s);
            if (lane == 0) sm.qsum[g] = s;
        }
    }
    __syncthreads();

    // ---- main loop ----
    float m[G], lsum[G], zsum[G], psum[G], o[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        lsum[g] = zsum[g] = psum[g] = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) o[g][k] = 0.0f;
    }
    const int32_t* pt = p.a.page_table + int64_t(b) * p.a.pt_stride;

    for (int base = t0 + 32 * warp; base < t1; base += 32 * kWarps) {
        const int t = base + lane;
        bool valid = t < t1;
        int64_t row = 0;
        if (valid) {
            const int page = __ldg(pt + t / ps);
            if (page < 0 || page >= p.g.num_pages) {
                flag_error(p.err, kErrOOB);
                valid = false;
            } else {
                row = (int64_t(page) * H + h) * ps + (t % ps);
            }
        }
        // q . k for this lane's token
        float s[G];
#pragma unroll
        for (int g = 0; g < G; ++g) s[g] = -INFINITY;
        float vscale = 0.0f, vzero = 0.0f;
        if (valid) {
            float acc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = 0.0f;
            if (MODE == 0) {
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
                for (int g = 0; g < G; ++g) s[g] = acc[g];
            } else {
                const uint4* kr = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.g.k_pool) + row * 64);
                const uint32_t ksz = __ldg(p.g.k_sz + row);
                const float kscale = __half2float(__ushort_as_half(uint16_t(ksz & 0xFFFF)));
                const float kzero = __half2float(__ushort_as_half(uint16_t(ksz >> 16)));
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 w = __ldg(kr + j);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float c1 = nib1p(ww[e], k);
                            const int d = 32 * j + 8 * e + k;
#pragma unroll
                            for (int g = 0; g < G; ++g) acc[g] += sm.qs[g][d] * c1;
                        }
                    }
                }
                // sum q'(1 + c/16) = sum q' + (q'.c)/16
#pragma unroll
                for (int g = 0; g < G; ++g)
                    s[g] = kscale * (16.0f * (acc[g] - sm.qsum[g])) + kzero * sm.qsum[g];
            }
            if (MODE != 0) {
                const uint32_t vsz = __ldg(p.g.v_sz + row);
                vscale = __half2float(__ushort_as_half(uint16_t(vsz & 0xFFFF)));
                vzero = __half2float(__ushort_as_half(uint16_t(vsz >> 16)));
            }
        }
        // online softmax (log2 domain)
        float pg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mnew = fmaxf(m[g], warp_max(s[g]));
            const float alpha = (mnew == -INFINITY) ? 1.0f : exp2f(m[g] - mnew);
            pg[g] = valid ? exp2f(s[g] - mnew) : 0.0f;
            m[g] = mnew;
            lsum[g] = lsum[g] * alpha + pg[g];
            zsum[g] = zsum[g] * alpha + pg[g] * vzero;
            psum[g] = psum[g] * alpha + pg[g] * vscale;
#pragma unroll
            for (int k = 0; k < 4; ++k) o[g][k] *= alpha;
        }
        // stage V rows + weights
        constexpr int kVW = Smem::kVWords;
        uint32_t* vs = sm.u.loop.v[warp][lane];
        if (valid) {
            const uint4* vr = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.g.v_pool) +
                                                             row * (MODE == 0 ? 256 : 64));
#pragma unroll
            for (int j = 0; j < kVW / 4; ++j) {
                const uint4 w = __ldg(vr + j);
                vs[4 * j + 0] = w.x;
                vs[4 * j + 1] = w.y;
                vs[4 * j + 2] = w.z;
                vs[4 * j + 3] = w.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < kVW; ++j) vs[j] = 0u;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) sm.u.loop.pt[warp][lane][g] = MODE == 0 ? pg[g] : pg[g] * vscale;
        __syncwarp();
        // P . V, lanes own d = 4 lane .. 4 lane + 3
        const int ntok = min(32, t1 - base);
        for (int j = 0; j < ntok; ++j) {
            float vv[4];
            if (MODE == 0) {
                const uint32_t w0 = sm.u.loop.v[warp][j][2 * lane], w1 = sm.u.loop.v[warp][j][2 * lane + 1];
                vv[0] = bf16_lo(w0);
                vv[1] = bf16_hi(w0);
                vv[2] = bf16_lo(w1);
                vv[3] = bf16_hi(w1);
            } else {
                const uint32_t w = sm.u.loop.v[warp][j][lane >> 1] >> ((lane & 1) * 16);
#pragma unroll
                for (int k = 0; k < 4; ++k) vv[k] = nib1p(w, k);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float wgt = sm.u.loop.pt[warp][j][g];
#pragma unroll
                for (int k = 0; k < 4; ++k) o[g][k] += wgt * vv[k];
            }
        }
        __syncwarp();
    }

    // ---- per-warp finish: o = sum p v (unnormalised), l = sum p ----
#pragma unroll
    for (int g = 0; g < G; ++g) {
        lsum[g] = warp_sum(lsum[g]);
        if (MODE != 0) {
            const float P = warp_sum(psum[g]);
            const float Z = warp_sum(zsum[g]);
#pragma unroll
            for (int k = 0; k < 4; ++k) o[g][k] = 16.0f * (o[g][k] - P) + Z;  // sum p (scale c + zero)
        }
    }
    __syncthreads();  // loop buffers are reused for the merge
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (lane == 0) {
            sm.u.merge.m[warp][g] = m[g];
            sm.u.merge.l[warp][g] = lsum[g];
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) sm.u.merge.o[warp][g][4 * lane + k] = o[g][k];
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
            const float sc = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
            acc += sc * sm.u.merge.o[w][g][tid];
            lt += sc * sm.u.merge.l[w][g];
        }
        p.ws_o[(out_row0 + g) * kHeadDim + tid] = acc;
        if (tid == 0) p.ws_ml[out_row0 + g] = make_float2(M, lt);
    }
}

// One CTA per (sequence, query head): merge splits, normalise, un-rotate V.
__global__ void __launch_bounds__(kThreads) merge_kernel(Params p, int rotate_out) {
    __shared__ float buf[kHeadDim];
    const int row = blockIdx.x;  // b * Hq + j
    const int tid = threadIdx.x;
    const int64_t rows = int64_t(p.a.batch) * p.g.Hq;
    float M = -INFINITY;
    for (int s = 0; s < p.num_splits; ++s) M = fmaxf(M, p.ws_ml[s * rows + row].x);
    float acc = 0.0f, l = 0.0f;
    for (int s = 0; s < p.num_splits; ++s) {
        const float2 ml = p.ws_ml[s * rows + row];
        const float sc = (ml.x == -INFINITY) ? 0.0f : exp2f(ml.x - M);
        acc += sc * p.ws_o[(s * rows + row) * kHeadDim + tid];
        l += sc * ml.y;
    }
    float res = l > 0.0f ? acc / l : 0.0f;
    if (rotate_out) {  // o H_blk: H_blk is symmetric and its own inverse
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
    if (p.a.out_fp32)
        static_cast<float*>(p.a.out)[int64_t(row) * kHeadDim + tid] = res;
    else
        static_cast<__nv_bfloat16*>(p.a.out)[int64_t(row) * kHeadDim + tid] = __float2bfloat16_rn(res);
}

template <int MODE>
cudaError_t launch_mode(const Params& p, dim3 grid, cudaStream_t s) {
    switch (p.g.Hq / p.g.H) {
        case 1: decode_split_kernel<MODE, 1><<<grid, kThreads, 0, s>>>(p); break;
        case 2: decode_split_kernel<MODE, 2><<<grid, kThreads, 0, s>>>(p); break;
        case 4: decode_split_kernel<MODE, 4><<<grid, kThreads, 0, s>>>(p); break;
        case 8: decode_split_kernel<MODE, 8><<<grid, kThreads, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

DecodePlan plan_decode(const CacheGeom& g, int batch, int max_seq_len, int num_sms) {
    DecodePlan pl;
    const int base_ctas = batch * g.H;
    const int min_chunk = 256;
    int by_len = (max_seq_len + min_chunk - 1) / min_chunk;
    if (by_len < 1) by_len = 1;
    int want = base_ctas > 0 ? (4 * num_sms + base_ctas - 1) / base_ctas : 1;
    if (want < 1) want = 1;
    pl.num_splits = want < by_len ? want : by_len;
    int chunk = (max_seq_len + pl.num_splits - 1) / pl.num_splits;
    chunk = ((chunk + 31) / 32) * 32;
    if (chunk < 32) chunk = 32;
    pl.chunk = chunk;
    const size_t rows = size_t(pl.num_splits) * size_t(batch) * size_t(g.Hq);
    pl.ws_bytes = rows * kHeadDim * sizeof(float) + rows * sizeof(float2);
    return pl;
}

cudaError_t launch_decode(const CacheGeom& g, const DecodeArgs& a, const DecodePlan& plan, int* err_word,
                          cudaStream_t s) {
    if (a.batch == 0) return cudaSuccess;
    Params p;
    p.g = g;
    p.a = a;
    p.num_splits = plan.num_splits;
    p.chunk = plan.chunk;
    p.qscale = float(1.0 / sqrt(double(kHeadDim))) * kLog2e;
    const size_t rows = size_t(plan.num_splits) * size_t(a.batch) * size_t(g.Hq);
    p.ws_o = static_cast<float*>(a.workspace);
    p.ws_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(a.workspace) + rows * kHeadDim * sizeof(float));
    p.err = err_word;
    dim3 grid(plan.num_splits, g.H, a.batch);
    cudaError_t e;
    if (g.mode == 0) e = launch_mode<0>(p, grid, s);
    else if (g.mode == 1) e = launch_mode<1>(p, grid, s);
    else e = launch_mode<2>(p, grid, s);
    if (e != cudaSuccess) return e;
    merge_kernel<<<a.batch * g.Hq, kThreads, 0, s>>>(p, g.mode == 2 && g.rotate_v);
    return cudaGetLastError();
}

}  // namespace kvq
