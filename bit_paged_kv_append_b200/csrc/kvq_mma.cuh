// kvq_mma.cuh -- what the tensor-core attention kernels over the INT4 cache share
// (decode in kvq_decode_mma.cu and kvq_decode_bf16.cu; the extend in kvq_extend_tc.cu takes
// the rotated query loader's constants and the 2-bit spreading): mma.sync wrappers, the
// per-warp ring of 16-token chunk stages and its cp.async copies, the rotated query,
// the 23-bit fixed-point q digits, the key-code B fragments and the V-code A tiles.
//
// Dequantisation is factored (SAW-INT4, wispaper.ai blog, section 3: the query is
// rotated in step with H_blk, so no inverse rotation of the cache is needed):
//   q' . (scale c + zero) = scale (q' . c) + zero sum(q')
//   sum_t p_t (scale_t c_t + zero_t) = sum_t (p_t scale_t) c_t + sum_t p_t zero_t
// so both contractions run on raw codes.
#pragma once

#include "kvq_common.cuh"
#include "kvq_decode.cuh"

namespace kvq {
constexpr int kThreads = 128;
constexpr int kWarps = 4;
constexpr int kStages = 4;
constexpr int kChunk = 16;                 // tokens per chunk
constexpr int kCodeBytes = kChunk * 64;    // 1 KiB of codes per chunk, K or V
constexpr int kOffV = kCodeBytes;          // stage layout: K codes | V codes | K sz | V sz
constexpr int kOffKs = 2 * kCodeBytes;
constexpr int kOffVs = 2 * kCodeBytes + kChunk * 4;
constexpr int kStageBytes = 2 * kCodeBytes + 2 * kChunk * 4;  // 2176
// Stage layout for CB-bit codes: K codes | V codes | K sz | V sz (2-bit rows are 32 bytes;
// the 4-bit layout above is Stage<4>).
template <int CB>
struct Stage {
    static constexpr int kRowBytes = 16 * CB;
    static constexpr int kCode = kChunk * kRowBytes;
    static constexpr int kOffV = kCode;
    static constexpr int kOffKs = 2 * kCode;
    static constexpr int kOffVs = 2 * kCode + kChunk * 4;
};
constexpr float kTwo24 = 16777216.0f;  // a masked nibble c in an fp16 lane is the subnormal c * 2^-24
constexpr float kTwo20 = 1048576.0f;   // ... and a masked high nibble is 16 c * 2^-24 = c * 2^-20
constexpr int kQFix = 8355711;  // |q_int| bound: 65536 hi + 256 mid + lo with hi, mid, lo in [-128, 127]
constexpr uint32_t kFull = 0xffffffffu;

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

// D[16 x 8] += A[16 x 32] (s8) B[32 x 8] (u8), int32 accumulation
__device__ __forceinline__ void mma16832_s8u8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D[16 x 8] += A[16 x 32] (u8) B[32 x 8] (s8), int32 accumulation
__device__ __forceinline__ void mma16832_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte asynchronous global -> shared copy (L2 only), completed by the copy-group waits below
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async16_s(uint32_t dst, const void* src, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// this thread's copy groups, all but the n most recent, have landed
template <int n>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory");
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

// Token (within an 8-token group) that slot n stands for: the four rows one
// P.V load touches then fall on both 64-byte halves of the bank space.
__device__ __forceinline__ int sigma(int n) { return n ^ ((n >> 2) & 1); }

// Byte offset of byte b of V-code row r in a stage: rows with bit 1 set swap their
// 32-byte halves, so the four rows (two even, two odd, one of each pair with bit 1
// set) that one 8-byte P.V load reads in each half-warp hit four distinct 32-byte
// bank groups.
__device__ __forceinline__ int vrow_off(int r, int b) { return kOffV + 64 * r + (b ^ ((r & 2) << 4)); }

// 2-bit codes -> the 4-bit nibble layout: byte b of w (codes of dims 4b .. 4b + 3 in bits
// 2k, 2k + 1) becomes bytes 2b, 2b + 1 (dims 4b, 4b + 1 | 4b + 2, 4b + 3 in the low / high
// nibbles), so the 4-bit fragment mappings apply unchanged.
__device__ __forceinline__ uint32_t spread2(uint32_t t) {  // two bytes in 16-bit lanes
    t = (t | (t << 4)) & 0x0F0F0F0Fu;
    return (t | (t << 2)) & 0x33333333u;
}
__device__ __forceinline__ uint2 expand2(uint32_t w) {
    return make_uint2(spread2(prmt(w, 0u, 0x4140u)), spread2(prmt(w, 0u, 0x4342u)));
}

// q' in fixed point (23 bits: q_int = rint(q' kQFix / max|q'|)) as three balanced signed
// bytes, q_int = 65536 hi + 256 mid + lo.  Fewer bits (16: two bytes) cost up to ~2e-3
// of the output on keys with outlier channels; 23 bits cost ~5e-6.
__device__ __forceinline__ void q_digits(int q, int& hi, int& mid, int& lo) {
    q = min(max(q, -kQFix), kQFix);
    lo = ((q + 128) & 255) - 128;
    const int q1 = (q - lo) >> 8;  // exact
    mid = ((q1 + 128) & 255) - 128;
    hi = (q1 - mid) >> 8;          // exact, in [-127, 127]
}

// Score sum from the three digit partial sums (|each| < 2^18): 65536 hi + 256 mid + lo.
__device__ __forceinline__ float q_dot(int dhi, int dmid, int dlo) {
    return fmaf(float(dhi), 65536.0f, float(dmid * 256 + dlo));
}

// What a CTA keeps in shared memory for its warps' chunk streams.
struct CtaRing {
    uint8_t stage[kWarps][kStages][kStageBytes];
    uint32_t mask[kWarps][kStages];     // tokens of the staged chunk on valid pages (bit per token)
    float2 szf[kWarps][2][kChunk];      // (scale, offset) of the current chunk: [warp][K / V][token]
};

// One warp's 16-token chunks: chunk iw starts at token t0 + (first + step iw) 16 (decode:
// a split's chunks round robin over the warps; extend: every chunk of the warp's range).
// Pool rows (one page-table lookup per lane, 32 chunks a window) and the copies of chunk
// iw into a ring stage.
template <int CB>
struct ChunkStream {
    using L = Stage<CB>;
    CtaRing* r;
    const int32_t* pt;  // this sequence's page-table row
    int t0, t1, nw, warp, lane, h;
    int first, step;    // chunk iw is the (first + step iw)-th 16-token chunk after t0
    bool fast;          // page size a multiple of 16: a chunk is 16 consecutive slots of one page
    uint64_t pol;
    int win;
    uint32_t myrow;     // pool row of this lane's chunk of the window, or kNoRow
    // per-lane sources (fast path): byte 16 lane of the K / V code blocks, and the
    // scale/zero words lanes 0..7 copy (4 K words per lane for lanes 0..3, V for 4..7)
    const uint8_t* kc;
    const uint8_t* vc;
    const uint32_t* sz;
    uint32_t dst0;      // shared address of this lane's K destination in slot 0

    static constexpr uint32_t kNoRow = 0xFFFFFFFFu;

    __device__ __forceinline__ void init(const DecodeParams& p) {
        win = -1;
        myrow = kNoRow;
        kc = static_cast<const uint8_t*>(p.g.k_pool) + 16 * lane;
        vc = static_cast<const uint8_t*>(p.g.v_pool) + 16 * lane;
        sz = (lane < 4 ? p.g.k_sz : p.g.v_sz) + 4 * (lane & 3);
        dst0 = smem_u32(r->stage[warp][0]) + 16 * lane;
    }

    // Pool row (page H + h) ps + slot of chunk iw's first token (all lanes; kNoRow for a
    // bad page, flagged once when its window is loaded).
    __device__ __forceinline__ uint32_t row_of(const DecodeParams& p, int iw) {
        if ((iw >> 5) != win) {
            win = iw >> 5;
            const int ci = 32 * win + lane;
            myrow = kNoRow;
            if (ci < nw) {
                const int tb = t0 + (first + step * ci) * kChunk;
                const int page = __ldg(pt + page_of_pos(p, tb));
                if (page >= 0 && page < p.g.num_pages)
                    myrow = (uint32_t(page) * uint32_t(p.g.H) + uint32_t(h)) * uint32_t(p.g.page_size) +
                            uint32_t(slot_of_pos(p, tb));
                else
                    flag_error(p.err, kErrOOB);
            }
        }
        return __shfl_sync(kFull, myrow, iw & 31);
    }

    // Copies of chunk iw into ring slot by all 32 lanes (16-byte cp.async, no divergent
    // issuer); the caller commits one copy group per chunk slot.
    __device__ __forceinline__ void issue(const DecodeParams& p, int iw, int slot) {
        if (fast) {
            // 16 consecutive slots of one page: 1 KiB of K codes, 1 KiB of V codes, 64 B of
            // scale/zero words each; lane L copies bytes 16 L and 512 + 16 L of both code
            // blocks (V rows swizzled, vrow_off), lanes 0..3 / 4..7 the K / V words
            const uint32_t row = row_of(p, iw);
            const bool ok = row != kNoRow;
            if (ok) {
                const uint32_t d = dst0 + uint32_t(slot) * kStageBytes;
                const uint8_t* ks = kc + size_t(row) * L::kRowBytes;
                const uint8_t* vs = vc + size_t(row) * L::kRowBytes;
                if (CB == 4) {
                    const int vsw = 16 * ((lane >> 2) & 2);  // this lane's V unit moves by 32 bytes
                    cp_async16_s(d, ks, pol);
                    cp_async16_s(d + 512, ks + 512, pol);
                    cp_async16_s((d + kOffV) ^ vsw, vs, pol);
                    cp_async16_s(((d + kOffV) ^ vsw) + 512, vs + 512, pol);
                } else {  // 512 bytes each: one copy per lane
                    cp_async16_s(d, ks, pol);
                    cp_async16_s(d + L::kOffV, vs, pol);
                }
                if (lane < 8) cp_async16_s(d + L::kOffKs, sz + row, pol);  // V words follow the K words
            }
            r->mask[warp][slot] = ok ? 0xFFFFu : 0u;  // the same value from every lane
        } else {
            // gather: lane L copies half L & 1 of token tb + (L >> 1)'s K and V code rows and
            // its K (even L) or V (odd L) scale/zero word
            uint8_t* st = r->stage[warp][slot];
            const int tb = t0 + (first + step * iw) * kChunk;
            const uint8_t* kpool = static_cast<const uint8_t*>(p.g.k_pool);
            const uint8_t* vpool = static_cast<const uint8_t*>(p.g.v_pool);
            const int i = lane >> 1, hf = lane & 1;
            const int t = tb + i;
            bool ok = false;
            if (t < t1) {
                const int page = __ldg(pt + page_of_pos(p, t));
                ok = page >= 0 && page < p.g.num_pages;
                if (ok) {
                    const int64_t row = (int64_t(page) * p.g.H + h) * p.g.page_size + slot_of_pos(p, t);
                    if (CB == 4) {
                        const int off = i * 64 + 32 * hf;
                        const int voff = i * 64 + 32 * (hf ^ ((i >> 1) & 1));  // V rows swizzled (vrow_off)
                        const uint8_t* kcp = kpool + row * 64 + 32 * hf;
                        const uint8_t* vcp = vpool + row * 64 + 32 * hf;
                        cp_async16(st + off, kcp, pol);
                        cp_async16(st + off + 16, kcp + 16, pol);
                        cp_async16(st + kOffV + voff, vcp, pol);
                        cp_async16(st + kOffV + voff + 16, vcp + 16, pol);
                    } else {  // 32-byte rows: 16 bytes per lane of each
                        const int off = i * 32 + 16 * hf;
                        cp_async16(st + off, kpool + row * 32 + 16 * hf, pol);
                        cp_async16(st + L::kOffV + off, vpool + row * 32 + 16 * hf, pol);
                    }
                    cp_async4(st + (hf ? L::kOffVs : L::kOffKs) + 4 * i, (hf ? p.g.v_sz : p.g.k_sz) + row);
                } else if (hf == 0) {
                    flag_error(p.err, kErrOOB);
                }
            }
            uint32_t m = __ballot_sync(kFull, ok);
            m = (m & 0x55555555u);  // one bit per token (even lanes) -> compact to bit i
            m = (m | (m >> 1)) & 0x33333333u;
            m = (m | (m >> 2)) & 0x0F0F0F0Fu;
            m = (m | (m >> 4)) & 0x00FF00FFu;
            m = (m | (m >> 8)) & 0x0000FFFFu;
            if (lane == 0) r->mask[warp][slot] = m;
        }
    }
};

// Unnormalised FWHT of the 128-dim row a warp holds 4 dims per lane (dims 4 lane ..
// 4 lane + 3), in blocks of b: butterflies of stride 1 and 2 inside the lane, then 4 ..
// b / 2 across lanes (lane bit = stride / 4), (a, c) -> (a + c, a - c) at every stage.
__device__ __forceinline__ void fwht_lanes(float (&x)[4], int lane, int b) {
    float y0 = x[0] + x[1], y1 = x[0] - x[1], y2 = x[2] + x[3], y3 = x[2] - x[3];
    x[0] = y0 + y2;
    x[2] = y0 - y2;
    x[1] = y1 + y3;
    x[3] = y1 - y3;
    for (int hs = 4; hs < b; hs <<= 1) {
        const bool upper = (lane & (hs >> 2)) != 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float other = __shfl_xor_sync(kFull, x[c], hs >> 2);
            x[c] = upper ? other - x[c] : x[c] + other;
        }
    }
}

// Query row qrow (bf16, 128 dims) as q H_blk * log2(e)/sqrt(D), after the fused rotary
// embedding at position pos when a table is set (the caller checks pos against the table):
// lane holds dims 4 lane .. 4 lane + 3, and lanes l, l ^ 16 hold the rotate-half pairs
// (i, i + 64).
__device__ __forceinline__ void load_q_rotated(const DecodeParams& p, int64_t qrow, int pos, int lane,
                                               float (&x)[4]) {
    const uint2 raw =
        __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.a.q) + qrow * kHeadDim) + lane);
    x[0] = __uint_as_float(raw.x << 16);
    x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    x[2] = __uint_as_float(raw.y << 16);
    x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    if (p.g.rope) {
        const float4* cs = reinterpret_cast<const float4*>(p.g.rope + int64_t(pos) * kHeadDim) + 2 * (lane & 15);
        const float4 c01 = __ldg(cs), c23 = __ldg(cs + 1);  // pairs 4 (lane & 15) .. + 3: (cos, sin) each
        const float c[4] = {c01.x, c01.z, c23.x, c23.z}, sn[4] = {c01.y, c01.w, c23.y, c23.w};
        const bool upper = lane >= 16;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float other = __shfl_xor_sync(kFull, x[e], 16);
            x[e] = upper ? fmaf(x[e], c[e], other * sn[e]) : fmaf(x[e], c[e], -other * sn[e]);
        }
    }
    float sc = p.qscale;
    if (p.g.mode == 2) {
        const int b = p.g.bdr_block;
        fwht_lanes(x, lane, b);
        sc *= rsqrtf(float(b));
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) x[c] *= sc;
}

// Chunk's (scale, zero) words into floats, one word per lane (0..15 K, 16..31 V).
// Values use centred codes c - 8, so their offset is zero + 8 scale; kscale
// multiplies the key scales and vscale the value scales (exactly: powers of two).
template <int CB>
__device__ __forceinline__ void stage_szf(CtaRing& R, const uint8_t* st, int warp, int lane, float kscale,
                                          float vscale) {
    const uint32_t w = reinterpret_cast<const uint32_t*>(st + Stage<CB>::kOffKs)[lane];
    const float sc = half_lo(w), zr = half_hi(w);
    R.szf[warp][lane >> 4][lane & 15] =
        lane < 16 ? make_float2(sc * kscale, zr) : make_float2(sc * vscale, zr + 8.0f * sc);
    __syncwarp();
}

// Lazily moved softmax reference: a row's reference max moves only when a chunk's max
// passes it by kTau (log2 units), so p = 2^(s - m) stays below 2^kTau and most chunks skip
// the rescale of the accumulators.  The decode multiplies value scales by kPScale so that
// p scale 2^-kTau <= scale stays inside fp16; its output undoes the factor (kPOut).
constexpr float kTau = 8.0f;
constexpr float kPScale = 1.0f / 256.0f;  // 2^-kTau
constexpr float kPOut = 256.0f;

// V codes of one chunk as P.V A operands: for each 16-dim tile jv, f(jv, a) with
// a = A[16 dims x 16 tokens], tokens (tokA, tokB), (8 + tokA, 8 + tokB) from bytes
// [8 gq, 8 gq + 8) of each row; row gq of tile jv is dim 16 gq + 2 jv (low nibble),
// row gq + 8 is dim 16 gq + 2 jv + 1 (high nibble, x16).
template <int CB, class F>
__device__ __forceinline__ void v_tiles(const uint8_t* st, int gq, int tokA, int tokB, F&& f) {
    uint2 v00, v01, v10, v11;
    if (CB == 4) {
        v00 = *reinterpret_cast<const uint2*>(st + vrow_off(tokA, 8 * gq));
        v01 = *reinterpret_cast<const uint2*>(st + vrow_off(tokB, 8 * gq));
        v10 = *reinterpret_cast<const uint2*>(st + vrow_off(8 + tokA, 8 * gq));
        v11 = *reinterpret_cast<const uint2*>(st + vrow_off(8 + tokB, 8 * gq));
    } else {  // dims 16 gq .. 16 gq + 15: 4 bytes of a 32-byte row, spread to the 4-bit layout
        const uint8_t* vb = st + Stage<2>::kOffV + 4 * gq;
        v00 = expand2(*reinterpret_cast<const uint32_t*>(vb + 32 * tokA));
        v01 = expand2(*reinterpret_cast<const uint32_t*>(vb + 32 * tokB));
        v10 = expand2(*reinterpret_cast<const uint32_t*>(vb + 32 * (8 + tokA)));
        v11 = expand2(*reinterpret_cast<const uint32_t*>(vb + 32 * (8 + tokB)));
    }
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
                // centred codes (c - 8) 2^-24 and 16 (c - 8) 2^-24: exact subnormal fp16
                const uint32_t a[4] = {hadd2u(P0 & 0x000F000Fu, kMinus8), hadd2u(P0 & 0x00F000F0u, kMinus128),
                                       hadd2u(P1 & 0x000F000Fu, kMinus8), hadd2u(P1 & 0x00F000F0u, kMinus128)};
                f(4 * wq + 2 * bp + sh, a);  // jv = byte of the thread's 8-byte slice
                P0 >>= 8;
                P1 >>= 8;
            }
        }
    }
}

// P.V of one chunk into O[16-dim tile jv][4] (tiles as in v_tiles) with B = (b0, b1);
// with kLow, (b0l, b1l) is accumulated by a second mma with the same A.
template <bool kLow, int CB>
__device__ __forceinline__ void pv_chunk(float (&O)[8][4], const uint8_t* st, int gq, int tokA, int tokB, uint32_t b0,
                                         uint32_t b1, uint32_t b0l, uint32_t b1l) {
    v_tiles<CB>(st, gq, tokA, tokB, [&](int jv, const uint32_t(&a)[4]) {
        mma16816(O[jv], a, b0, b1);
        if (kLow) mma16816(O[jv], a, b0l, b1l);
    });
}

// Codes of dims 32 pq .. 32 pq + 31 of token row tok in the 4-bit nibble layout (16 bytes).
template <int CB>
__device__ __forceinline__ uint4 key_codes(const uint8_t* st, int tok, int pq) {
    if (CB == 4) return *reinterpret_cast<const uint4*>(st + tok * 64 + 16 * pq);
    const uint2 r = *reinterpret_cast<const uint2*>(st + tok * 32 + 8 * pq);
    const uint2 a = expand2(r.x), b = expand2(r.y);
    return make_uint4(a.x, a.y, b.x, b.y);
}

}  // namespace kvq
