// kvq_decode_mma.cu -- paged GQA decode attention over the INT4 cache on the
// tensor cores (mma.sync m16n8k16, fp16 operands, fp32 accumulation).
//
// SAW-INT4 (wispaper.ai blog, section 3): the query is rotated in step with
// H_blk, so q' k^ needs no inverse rotation of the cache; the abstract keeps
// fused attention over the paged INT4 layout.  Dequantisation is factored:
//   q' . (scale c + zero) = scale (q' . c) + zero sum(q')
//   sum_t p_t (scale_t c_t + zero_t) = sum_t (p_t scale_t) c_t + sum_t p_t zero_t
// so both contractions run on raw 4-bit codes, which are exact in fp16.
//
// One CTA = (split, KV head, sequence), 4 warps; each warp walks 16-token
// chunks of its split (round robin), with its own online-softmax state.  The
// CTA issues its first copies before anything else, then rotates q (one warp
// per head, FWHT with shuffles) straight into mma fragment order, so the
// prologue hides under the first memory latency.
//   * Staging: per warp a ring of 4 shared-memory stages; one lane issues 1-D
//     bulk async copies (cp.async.bulk, no multicast) of the chunk's K codes,
//     V codes and scale/zero words (2176 B) on an mbarrier; every wait is
//     bounded.  Page sizes that are not a multiple of 16 take a per-token
//     gather instead.
//   * q.K: D[16 x 8] = A[16 x 16] B[16 x 8] per (n-tile of 8 tokens, 16 dims).
//     A = the G rotated query heads, each split into an fp16 high part (rows
//     0..7) and low part (rows 8..15), so q' keeps ~22 bits; B = codes.  A
//     code nibble c is masked in place into an fp16 lane, which makes it the
//     exact subnormal c * 2^-24 (16 c * 2^-24 for the high nibble of a byte,
//     whose A entries carry a factor 1/16): one AND per two codes, no bias to
//     cancel, every product exact; the scores are scaled back by 2^24.
//   * P.V: D[16 dims x 8 heads] = A[16 x 16 tokens] B[16 tokens x 8 heads].  A =
//     V codes of four tokens (PRMT + AND), centred to c - 8 by one exact fp16
//     add, B = p * scale_v, taken straight from the q.K accumulator layout (the
//     thread that holds a score also holds the matching B element), so no
//     shuffle or transpose.  Centring keeps the accumulator small: the tensor
//     cores' fp32 accumulation does not round to nearest, and over thousands of
//     tokens sum (p scale) c and sum p zero would otherwise nearly cancel.  B
//     is split into fp16 high and low parts accumulated by two mmas, since a
//     single fp16 rounding of p * scale would cost ~1e-3 of the output.
//   * Which dimension d and which token each fragment slot stands for is a
//     fixed permutation chosen so every thread reads contiguous bytes and the
//     shared-memory reads are conflict-free; the output mapping undoes it.
#include "kvq_common.cuh"
#include "kvq_decode.cuh"

namespace kvq {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = 4;
constexpr int kStages = 4;
constexpr int kChunk = 16;                 // tokens per chunk
constexpr int kCodeBytes = kChunk * 64;    // 1 KiB of codes per chunk, K or V
constexpr int kOffV = kCodeBytes;          // stage layout: K codes | V codes | K sz | V sz
constexpr int kOffKs = 2 * kCodeBytes;
constexpr int kOffVs = 2 * kCodeBytes + kChunk * 4;
constexpr int kStageBytes = 2 * kCodeBytes + 2 * kChunk * 4;  // 2176
constexpr float kTwo24 = 16777216.0f;  // a masked nibble c in an fp16 lane is the subnormal c * 2^-24
constexpr float kTwo20 = 1048576.0f;   // ... and a masked high nibble is 16 c * 2^-24 = c * 2^-20

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// fp16x2 add of raw words (exact here: every operand and sum is a small multiple of 2^-24)
__device__ __forceinline__ uint32_t hadd2u(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
constexpr uint32_t kMinus8 = 0x80088008u;    // fp16x2 (-8 2^-24, -8 2^-24)
constexpr uint32_t kMinus128 = 0x80808080u;  // fp16x2 (-128 2^-24, -128 2^-24)

__device__ __forceinline__ float half_lo(uint32_t w) { return __half2float(__ushort_as_half(uint16_t(w & 0xFFFF))); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half(uint16_t(w >> 16))); }

// Token (within an 8-token n-tile) that column n stands for: the four rows one
// P.V load touches then fall on both 64-byte halves of the bank space.
__device__ __forceinline__ int sigma(int n) { return n ^ ((n >> 2) & 1); }

template <int G>
__global__ void __launch_bounds__(kThreads, 4) decode_mma_kernel(DecodeParams p) {
    __shared__ __align__(128) uint8_t ring[kWarps][kStages][kStageBytes];
    __shared__ __align__(8) uint64_t bars[kWarps][kStages];
    __shared__ uint32_t smask[kWarps][kStages];
    __shared__ float2 szf[kWarps][2][kChunk];  // (scale, zero) of the current chunk: [warp][K / V][token]
    __shared__ uint32_t As[8 * 4 * 32];         // q.K A operand in fragment order: [k-step][reg][lane]
    __shared__ float qsum_s[kMaxGroup];

    const int k = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, pq = lane & 3;  // mma group id / thread in group
    const int H = p.g.H, Hq = p.g.Hq, ps = p.g.page_size;

    const int L = decode_len(p, s);
    if (k == 0 && h == 0 && tid == 0 && L != __ldg(p.a.seq_lens + s)) flag_error(p.err, kErrOOB);
    const int t0 = k * p.item_tokens;
    if (t0 >= L) return;  // past the end of the sequence: no partial (the merge reads only real splits)
    const int t1 = min(L, t0 + p.item_tokens);

    const bool fast = (ps % kChunk) == 0;
    const uint8_t* kpool = static_cast<const uint8_t*>(p.g.k_pool);
    const uint8_t* vpool = static_cast<const uint8_t*>(p.g.v_pool);
    const uint32_t* ksz = p.g.k_sz;
    const uint32_t* vsz = p.g.v_sz;
    const int32_t* pt = p.a.page_table + int64_t(s) * p.a.pt_stride;
    const int nchunks = (t1 - t0 + kChunk - 1) / kChunk;
    const int nw = nchunks > warp ? (nchunks - warp + kWarps - 1) / kWarps : 0;  // this warp's chunks

    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < kStages; ++st) mbar_init(&bars[warp][st], 1);
        fence_mbar_init();
    }
    for (int w = tid; w < 8 * 4 * 32; w += kThreads) As[w] = 0u;
    __syncthreads();

    // ---------------- start streaming this warp's chunks ----------------
    const uint64_t pol = policy_evict_first();
    int win = -1, mypage = -1;
    auto page_of = [&](int iw) {  // page of this warp's chunk iw (all lanes; 32 ids per window)
        if ((iw >> 5) != win) {
            win = iw >> 5;
            const int ci = 32 * win + lane;
            mypage = ci < nw ? __ldg(pt + page_of_pos(p, t0 + (warp + kWarps * ci) * kChunk)) : -1;
        }
        return __shfl_sync(0xffffffffu, mypage, iw & 31);
    };
    auto issue = [&](int iw, int slot) {  // this warp's chunk number iw into ring slot
        uint8_t* st = ring[warp][slot];
        const int tb = t0 + (warp + kWarps * iw) * kChunk;
        if (fast) {
            const int page = page_of(iw);
            if (lane == 0) {
                if (page >= 0 && page < p.g.num_pages) {
                    const int64_t row = (int64_t(page) * H + h) * ps + slot_of_pos(p, tb);
                    smask[warp][slot] = 0xFFFFu;
                    fence_proxy_async();
                    mbar_expect_tx(&bars[warp][slot], kStageBytes);
                    bulk_g2s(st, kpool + row * 64, kCodeBytes, &bars[warp][slot], pol);
                    bulk_g2s(st + kOffV, vpool + row * 64, kCodeBytes, &bars[warp][slot], pol);
                    bulk_g2s(st + kOffKs, ksz + row, kChunk * 4, &bars[warp][slot], pol);
                    bulk_g2s(st + kOffVs, vsz + row, kChunk * 4, &bars[warp][slot], pol);
                } else {
                    smask[warp][slot] = 0u;
                    flag_error(p.err, kErrOOB);
                }
                mbar_arrive(&bars[warp][slot]);
            }
        } else {
            // gather: lanes 0..15 fetch K rows, lanes 16..31 V rows of tokens tb + (lane & 15)
            const int i = lane & 15;
            const bool isv = lane >= 16;
            const int t = tb + i;
            bool ok = false;
            if (t < t1) {
                const int page = __ldg(pt + page_of_pos(p, t));
                ok = page >= 0 && page < p.g.num_pages;
                if (ok) {
                    const int64_t row = (int64_t(page) * H + h) * ps + slot_of_pos(p, t);
                    const uint4* src = reinterpret_cast<const uint4*>((isv ? vpool : kpool) + row * 64);
                    uint4* dst = reinterpret_cast<uint4*>(st + (isv ? kOffV : 0) + i * 64);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) dst[q4] = __ldg(src + q4);
                    reinterpret_cast<uint32_t*>(st + (isv ? kOffVs : kOffKs))[i] = __ldg((isv ? vsz : ksz) + row);
                } else if (!isv) {
                    flag_error(p.err, kErrOOB);
                }
            }
            const uint32_t m = __ballot_sync(0xffffffffu, ok) & 0xFFFFu;
            __syncwarp();
            if (lane == 0) {
                smask[warp][slot] = m;
                mbar_arrive(&bars[warp][slot]);
            }
        }
    };
    const int pre = nw < kStages ? nw : kStages;
    for (int i = 0; i < pre; ++i) issue(i, i);

    // ---------------- q' = q H_blk * log2(e)/sqrt(D) as fp16 hi/lo, fragment order ----------------
    for (int row = warp; row < G; row += kWarps) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.a.q) +
                                                               (int64_t(s) * Hq + h * G + row) * kHeadDim) + lane);
        float x[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                      __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};  // dims 4 lane + c
        float sc = p.qscale;
        if (p.g.mode == 2) {
            const int b = p.g.bdr_block;
            // strides 1 and 2 inside the lane, 4 .. 64 across lanes (lane bit = stride / 4)
            float y0 = x[0] + x[1], y1 = x[0] - x[1], y2 = x[2] + x[3], y3 = x[2] - x[3];
            x[0] = y0 + y2;
            x[2] = y0 - y2;
            x[1] = y1 + y3;
            x[3] = y1 - y3;
            for (int hs = 4; hs < b; hs <<= 1) {
                const bool upper = (lane & (hs >> 2)) != 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float other = __shfl_xor_sync(0xffffffffu, x[c], hs >> 2);
                    x[c] = upper ? other - x[c] : x[c] + other;
                }
            }
            sc *= rsqrtf(float(b));
        }
        float tsum = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            x[c] *= sc;
            tsum += x[c];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tsum += __shfl_xor_sync(0xffffffffu, tsum, o);
        if (lane == 0) qsum_s[row] = tsum;
        uint16_t* A16 = reinterpret_cast<uint16_t*>(As);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int d = 4 * lane + c;
            const float v = x[c] * ((d & 1) ? 0.0625f : 1.0f);  // odd d pairs with a high nibble (x16)
            const __half hi = __float2half_rn(v);
            const __half lo = __float2half_rn(v - __half2float(hi));
            // inverse of dpos: d = 32 pp + 8 i + off
            const int pp = d >> 5, i = (d >> 3) & 3, off = d & 7;
            const int j = 2 * i + ((off >> 1) & 1), h8 = off & 1, e = off >> 2;
            const int base = (j * 4 + 2 * h8) * 32 + 4 * row + pp;  // hi part: register 2 h8; lo part: + 1
            A16[2 * base + e] = __half_as_ushort(hi);
            A16[2 * (base + 32) + e] = __half_as_ushort(lo);
        }
    }
    __syncthreads();
    uint32_t A[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int r = 0; r < 4; ++r) A[j][r] = As[(j * 4 + r) * 32 + lane];
    const float qsh = qsum_s[gq < G ? gq : 0];

    // ---------------- main loop over this warp's chunks ----------------
    float m = -INFINITY, l = 0.0f, Z = 0.0f;  // softmax state of head gq (q.K layout)
    float O[8][4];                            // P.V accumulators: dims x heads (2 pq, 2 pq + 1)
#pragma unroll
    for (int j = 0; j < 8; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.0f;
    const int tokA = sigma(2 * pq), tokB = sigma(2 * pq + 1), tokK = sigma(gq);

    for (int i = 0; i < nw; ++i) {
        const int slot = i % kStages;
        if (!mbar_wait(&bars[warp][slot], (i / kStages) & 1)) {
            flag_error(p.err, kErrTimeout);
            break;
        }
        const uint8_t* st = ring[warp][slot];
        const uint32_t vmask = smask[warp][slot];
        const int tb = t0 + (warp + kWarps * i) * kChunk;
        {  // each lane converts one (scale, zero) word: lanes 0..15 K, 16..31 V
            const uint32_t w = reinterpret_cast<const uint32_t*>(st + kOffKs)[lane];
            const float sc = half_lo(w), zr = half_hi(w);
            // values use centred codes c - 8, so their offset is zero + 8 scale
            szf[warp][lane >> 4][lane & 15] = make_float2(sc, lane < 16 ? zr : zr + 8.0f * sc);
            __syncwarp();
        }

        // ---- scores: q' . codes for the two 8-token n-tiles ----
        float C[2][4];
#pragma unroll
        for (int tau = 0; tau < 2; ++tau) {
            const uint4 kw = *reinterpret_cast<const uint4*>(st + (8 * tau + tokK) * 64 + 16 * pq);
            const uint32_t w[4] = {kw.x, kw.y, kw.z, kw.w};
            C[tau][0] = C[tau][1] = C[tau][2] = C[tau][3] = 0.0f;
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                const uint32_t ws = w[wi] >> 8;
                mma16816(C[tau], A[2 * wi], w[wi] & 0x000F000Fu, w[wi] & 0x00F000F0u);
                mma16816(C[tau], A[2 * wi + 1], ws & 0x000F000Fu, ws & 0x00F000F0u);
            }
        }
        float sc[2][2];
        int loc[2][2];
#pragma unroll
        for (int tau = 0; tau < 2; ++tau) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int lt = 8 * tau + (e ? tokB : tokA);
                loc[tau][e] = lt;
                const float2 kz = szf[warp][0][lt];
                const float S = (C[tau][e] + C[tau][2 + e]) * kTwo24;
                const float v = kz.x * S + kz.y * qsh;
                const bool valid = (gq < G) && (tb + lt < t1) && ((vmask >> lt) & 1u);
                sc[tau][e] = valid ? v : -INFINITY;
            }
        }
        // ---- online softmax (log2 domain) for head gq ----
        float cm = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
        const float mn = fmaxf(m, cm);
        if (__any_sync(0xffffffffu, mn > m)) {
            const float alpha = (mn > m) ? fast_exp2(m - mn) : 1.0f;
            l *= alpha;
            Z *= alpha;
            m = mn;
            const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * pq);
            const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * pq + 4);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                O[j][0] *= a0;
                O[j][1] *= a1;
                O[j][2] *= a0;
                O[j][3] *= a1;
            }
        }
        float pt_[2][2];
#pragma unroll
        for (int tau = 0; tau < 2; ++tau) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                // masked tokens (past the end, skipped pages, stale slots) may hold any bits in
                // their scale/zero word: never let them reach an operand, even times 0
                const bool live = sc[tau][e] != -INFINITY;
                const float pr = live ? fast_exp2(sc[tau][e] - m) : 0.0f;
                const float2 vz = live ? szf[warp][1][loc[tau][e]] : make_float2(0.0f, 0.0f);
                l += pr;
                Z += pr * vz.y;
                pt_[tau][e] = pr * vz.x;
            }
        }
        const uint32_t b0 = pack_half2(pt_[0][0], pt_[0][1]);
        const uint32_t b1 = pack_half2(pt_[1][0], pt_[1][1]);
        const uint32_t b0l = pack_half2(pt_[0][0] - half_lo(b0), pt_[0][1] - half_hi(b0));
        const uint32_t b1l = pack_half2(pt_[1][0] - half_lo(b1), pt_[1][1] - half_hi(b1));

        // ---- P . V: A = codes of tokens (tokA, tokB), (8+tokA, 8+tokB), bytes [8 gq, 8 gq + 8) ----
        const uint8_t* vc = st + kOffV + 8 * gq;
        const uint2 v00 = *reinterpret_cast<const uint2*>(vc + tokA * 64);
        const uint2 v01 = *reinterpret_cast<const uint2*>(vc + tokB * 64);
        const uint2 v10 = *reinterpret_cast<const uint2*>(vc + (8 + tokA) * 64);
        const uint2 v11 = *reinterpret_cast<const uint2*>(vc + (8 + tokB) * 64);
#pragma unroll
        for (int wq = 0; wq < 2; ++wq) {
            const uint32_t x00 = wq ? v00.y : v00.x, x01 = wq ? v01.y : v01.x;
            const uint32_t x10 = wq ? v10.y : v10.x, x11 = wq ? v11.y : v11.x;
#pragma unroll
            for (int bp = 0; bp < 2; ++bp) {
                const uint32_t sel = bp ? 0x7632u : 0x5410u;
                uint32_t P0 = prmt(x00, x01, sel), P1 = prmt(x10, x11, sel);
#pragma unroll
                for (int sh = 0; sh < 2; ++sh) {
                    const int jv = 4 * wq + 2 * bp + sh;  // byte of the thread's 8-byte slice
                    // centred codes (c - 8) 2^-24 and 16 (c - 8) 2^-24: exact subnormal fp16
                    const uint32_t a[4] = {hadd2u(P0 & 0x000F000Fu, kMinus8), hadd2u(P0 & 0x00F000F0u, kMinus128),
                                           hadd2u(P1 & 0x000F000Fu, kMinus8), hadd2u(P1 & 0x00F000F0u, kMinus128)};
                    mma16816(O[jv], a, b0, b1);
                    mma16816(O[jv], a, b0l, b1l);
                    P0 >>= 8;
                    P1 >>= 8;
                }
            }
        }
        __syncwarp();
        if (i + kStages < nw) issue(i + kStages, slot);
    }

    // ---------------- per-head totals, undo the 2^-24 code scale, merge the warps ----------------
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    Z += __shfl_xor_sync(0xffffffffu, Z, 1);
    Z += __shfl_xor_sync(0xffffffffu, Z, 2);
    const float Z0 = __shfl_sync(0xffffffffu, Z, 8 * pq), Z1 = __shfl_sync(0xffffffffu, Z, 8 * pq + 4);
    __syncthreads();  // every ring is drained; reuse it for the merge
    float* mo = reinterpret_cast<float*>(&ring[0][0][0]);  // [warp][G][128]
    float* mm = mo + kWarps * G * kHeadDim;                // [warp][G]
    float* ml = mm + kWarps * G;                           // [warp][G]
    const int h0 = 2 * pq, h1 = 2 * pq + 1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int d = 16 * gq + 2 * j;
        if (h0 < G) {
            mo[(warp * G + h0) * kHeadDim + d] = O[j][0] * kTwo24 + Z0;
            mo[(warp * G + h0) * kHeadDim + d + 1] = O[j][2] * kTwo20 + Z0;
        }
        if (h1 < G) {
            mo[(warp * G + h1) * kHeadDim + d] = O[j][1] * kTwo24 + Z1;
            mo[(warp * G + h1) * kHeadDim + d + 1] = O[j][3] * kTwo20 + Z1;
        }
    }
    if (pq == 0 && gq < G) {
        mm[warp * G + gq] = m;
        ml[warp * G + gq] = l;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * G + g]);
        float acc = 0.0f, lt = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float mw = mm[w * G + g];
            const float f = (mw == -INFINITY) ? 0.0f : fast_exp2(mw - M);
            acc += f * mo[(w * G + g) * kHeadDim + tid];
            lt += f * ml[w * G + g];
        }
        const int64_t r = partial_row(p, s, k, h * G + g);
        p.ws_o[r * kHeadDim + tid] = acc;
        if (tid == 0) p.ws_ml[r] = make_float2(M, lt);
    }
}

}  // namespace

cudaError_t launch_decode_mma(const DecodeParams& p, cudaStream_t s) {
    const dim3 grid(p.max_splits, p.g.H, p.a.batch);
    switch (p.g.Hq / p.g.H) {
        case 1: decode_mma_kernel<1><<<grid, kThreads, 0, s>>>(p); break;
        case 2: decode_mma_kernel<2><<<grid, kThreads, 0, s>>>(p); break;
        case 4: decode_mma_kernel<4><<<grid, kThreads, 0, s>>>(p); break;
        case 8: decode_mma_kernel<8><<<grid, kThreads, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace kvq
