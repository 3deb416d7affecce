// kvq_append.cu -- the fused KV-cache write: block-diagonal Hadamard rotation +
// token-wise asymmetric INT4 quantisation + nibble packing + store into the
// page slot, in one kernel (SAW-INT4 abstract: a fused rotation-quantisation
// kernel integrated into paged KV-cache layouts; wispaper.ai blog section 3:
// K~ = quant(K H_blk), V~ = quant(V H_blk), the rotation fused into the
// KV-cache write operator with no separate kernel).
//
// Work unit: one (token, KV head) row of head_dim = 128 bf16 values, handled
// entirely by one thread.  The whole 128-element transform, the min/max, the
// quantiser and the packing then run in registers with no shuffles; the fp32
// butterflies use sm_100's packed f32x2 adds, pairing element i with element
// i + 64 so every stage of stride < 64 is one packed op per pair.  The compiler
// contracts the packed multiply intrinsic followed by a packed add into one fused
// op even when both carry an explicit rounding mode, so the 1/sqrt(b)
// normalisation is a packed multiply written in PTX, which it leaves alone.  K
// and V rows that take the same path (no rotation, or both rotated) share one
// instantiation of it: half the hot code, fewer instruction-fetch stalls.
//
// Data movement: a persistent grid (one CTA per SM); per CTA a ring of three
// 56 KiB shared-memory stages filled by TMA tensor loads (128-byte swizzle,
// L2 evict-first, no multicast) issued by a producer warp, which also resolves
// each token's page slot (ids loaded one tile ahead, page lookups overlapped
// with the tile's copies, a 2-slot meta ring).  Seven consumer warps (224
// threads = 224 rows per stage; with the producer, two warps per SM
// sub-partition, so a thread may hold ~200 registers) read their row from the
// swizzled stage without bank conflicts, write 64 B of codes + 4 B of (scale,
// zero) per row straight to the pool, and free the stage on an mbarrier: no
// block-wide barrier in the loop.  A tile = up to 224 consecutive rows of the
// [T, H, D] input = up to 224 / H tokens (H divides 32); its K rows fill one stage
// and its V rows the next.
//
// Schedule: CTA c owns the contiguous chunk of ceil(T / SMs) tokens starting at
// c * that, so no CTA holds more than one token above the mean.  A chunk that is
// not a whole number of tiles starts with its remainder as one short tile, copied
// by a second pair of tensor maps whose box is that remainder's rows, then whole
// tiles: with 4.01 tiles of work per SM every CTA runs four whole tiles and one
// short one, not two CTAs five whole ones.
//
// Every wait is bounded (kWaitLimitNs); out-of-range sequence ids, positions
// and page ids are skipped and flagged in the device error word.
#include <cudaTypedefs.h>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kRows = 224;                   // (token, head) rows per stage = consumer threads (7 warps)
constexpr int kThreads = kRows + 32;         // + one producer warp: 8 warps, two per SM sub-partition
constexpr int kStages = 3;
constexpr int kHalfBytes = kRows * 128;      // one 128-byte half-row per row
constexpr int kStageBytes = 2 * kHalfBytes;  // 56 KiB (a multiple of 1 KiB: swizzle atoms stay aligned)
constexpr int kMaxTileTokens = kRows;        // H == 1
constexpr size_t kSmemBytes = 1024 /*align slack*/ + size_t(kStages) * kStageBytes +
                              2 * size_t(kMaxTileTokens) * (sizeof(int2) + sizeof(int)) +
                              2 * kStages * sizeof(uint64_t) + 16 /*abort flag*/;

// Magic constant 1.5 * 2^23: for |v| < 2^22, the fp32 sum v + kMagic (rounded to
// nearest even) carries rint_even(v) in its low mantissa bits.
constexpr float kMagic = 12582912.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;
// Sum over k = 0..7 of kMagicBits << 4k (mod 2^32): the offset the packing
// Horner chain below accumulates from the magic bias of eight codes.
constexpr uint32_t magic_pack_offset() {
    uint32_t c = 0;
    for (int k = 0; k < 8; ++k) c += kMagicBits << (4 * k);
    return c;
}
constexpr uint32_t kMagicPackOffset = magic_pack_offset();
// ... and the offset of sixteen 2-bit codes packed with shifts of 2
constexpr uint32_t magic_pack_offset2() {
    uint32_t c = 0;
    for (int k = 0; k < 16; ++k) c += kMagicBits << (2 * k);
    return c;
}
constexpr uint32_t kMagicPackOffset2 = magic_pack_offset2();

struct Params {
    CacheGeom g;
    AppendArgs a;
    int tile_tokens;   // kRows / H: tokens of a whole tile
    int chunk_tokens;  // tokens per CTA (the last CTA's chunk may be shorter)
    int short_tokens;  // tokens the short-tile maps' box covers (0: no short maps)
    float r_b;         // (float)(1 / sqrt((double)bdr_block))
    int* err;
};

struct Tile {
    int first, count;  // first token, tokens (count 0: past the end of the chunk)
};

// Tile j of the chunk [c0, c0 + len): the remainder len % TT first, then whole tiles.
__device__ __forceinline__ Tile tile_of(int c0, int len, int TT, int j) {
    const int rem = len % TT;
    const int first = rem ? (j == 0 ? c0 : c0 + rem + (j - 1) * TT) : c0 + j * TT;
    const int count = (rem && j == 0) ? rem : TT;
    return first < c0 + len ? Tile{first, count} : Tile{0, 0};
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Eight codes (as magic-biased float bits, element k in u[k]) -> one packed word,
// element k in nibble k.
__device__ __forceinline__ uint32_t pack8(const uint32_t (&u)[8]) {
    uint32_t acc = u[7];
#pragma unroll
    for (int k = 6; k >= 0; --k) acc = (acc << 4) + u[k];
    return acc - kMagicPackOffset;
}

// Sixteen 2-bit codes (magic-biased float bits, element k in u[k]) -> one word, element k
// in bits 2k, 2k + 1.
__device__ __forceinline__ uint32_t pack16(const uint32_t (&u)[16]) {
    uint32_t acc = u[15];
#pragma unroll
    for (int k = 14; k >= 0; --k) acc = (acc << 2) + u[k];
    return acc - kMagicPackOffset2;
}

// Loads this thread's row from the swizzled stage into R[i] = (x_i, x_{i+64}).
__device__ __forceinline__ void load_row(const uint8_t* stage, int row, float2 (&R)[64]) {
    const uint4* h0 = reinterpret_cast<const uint4*>(stage + row * 128);
    const uint4* h1 = reinterpret_cast<const uint4*>(stage + kHalfBytes + row * 128);
    const int sw = row & 7;  // 128-byte swizzle: chunk j of line L sits at chunk j ^ (L & 7)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint4 a = h0[j ^ sw];
        const uint4 b = h1[j ^ sw];
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            R[8 * j + 2 * q] = make_float2(bf16_lo(aw[q]), bf16_lo(bw[q]));
            R[8 * j + 2 * q + 1] = make_float2(bf16_hi(aw[q]), bf16_hi(bw[q]));
        }
    }
}

// fp32x2 multiply as packed PTX: the compiler keeps it a separate rounding from the adds
// that follow (it contracts the packed multiply intrinsic with a following packed add)
__device__ __forceinline__ float2 f2_mul_rn(float2 a, float s) {
    unsigned long long v = (static_cast<unsigned long long>(__float_as_uint(a.y)) << 32) | __float_as_uint(a.x);
    const unsigned long long m = (static_cast<unsigned long long>(__float_as_uint(s)) << 32) | __float_as_uint(s);
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(v) : "l"(v), "l"(m));
    return make_float2(__uint_as_float(uint32_t(v)), __uint_as_float(uint32_t(v >> 32)));
}

// Block-diagonal normalised Sylvester-Hadamard rotation of one row, fp32,
// stages of increasing stride, then the 1/sqrt(b) multiply.  The butterflies
// are packed adds (no multiply anywhere to contract with); the normalisation
// is a packed multiply in PTX that is never merged into a later add.
template <int BLK>
__device__ __forceinline__ void rotate_row(float2 (&R)[64], float r_b) {
    constexpr int kPacked = BLK < 64 ? BLK : 64;  // strides below 64 stay within a packed lane
#pragma unroll
    for (int hs = 1; hs < kPacked; hs <<= 1) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if ((i & hs) == 0) {
                const float2 a = R[i], c = R[i + hs];
                R[i] = __fadd2_rn(a, c);
                R[i + hs] = __fadd2_rn(a, make_float2(-c.x, -c.y));  // a - c, exactly
            }
        }
    }
    if (BLK == 128) {  // stride 64 pairs the two lanes of each packed register
#pragma unroll
        for (int i = 0; i < 64; ++i) R[i] = make_float2(__fadd_rn(R[i].x, R[i].y), __fsub_rn(R[i].x, R[i].y));
    }
#pragma unroll
    for (int i = 0; i < 64; ++i) R[i] = f2_mul_rn(R[i], r_b);
}

// Codes of a row into 16 packed words: wa = elements 0..63, wb = elements 64..127.
// u = fma(y - zero, inv, 1.5 * 2^23) rounds the exact product fl(y - zero) * inv to the
// nearest integer (ties to even) in its low mantissa bits: the fma adds the unrounded
// product to the magic constant and rounds once.  CLAMP maps products below 0
// (or NaN) to 0 and above 15 to 15; rows whose extreme codes are in range skip it.
template <bool CLAMP>
__device__ __forceinline__ void quantise_pack(const float2 (&R)[64], float zf, float inv, uint32_t (&wa)[8],
                                              uint32_t (&wb)[8]) {
    const float2 nz = make_float2(-zf, -zf), ii = make_float2(inv, inv), mm = make_float2(kMagic, kMagic);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        uint32_t ulo[8], uhi[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float2 u = __ffma2_rn(__fadd2_rn(R[8 * m + k], nz), ii, mm);
            if (CLAMP) {
                u.x = u.x > kMagic ? fminf(u.x, kMagic + 15.0f) : kMagic;
                u.y = u.y > kMagic ? fminf(u.y, kMagic + 15.0f) : kMagic;
            }
            ulo[k] = __float_as_uint(u.x);
            uhi[k] = __float_as_uint(u.y);
        }
        wa[m] = pack8(ulo);  // elements 8m .. 8m+7 -> bytes 4m .. 4m+3
        wb[m] = pack8(uhi);  // elements 64+8m .. 64+8m+7 -> bytes 32+4m .. 32+4m+3
    }
}

// 2-bit codes of a row into 8 packed words (the row's 32 bytes): word m < 4 holds elements
// 16 m .. 16 m + 15 (R[.].x), word 4 + m elements 64 + 16 m .. (R[.].y).
template <bool CLAMP>
__device__ __forceinline__ void quantise_pack2(const float2 (&R)[64], float zf, float inv, uint32_t (&w)[8]) {
    const float2 nz = make_float2(-zf, -zf), ii = make_float2(inv, inv), mm = make_float2(kMagic, kMagic);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        uint32_t ulo[16], uhi[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float2 u = __ffma2_rn(__fadd2_rn(R[16 * m + k], nz), ii, mm);
            if (CLAMP) {
                u.x = u.x > kMagic ? fminf(u.x, kMagic + 3.0f) : kMagic;
                u.y = u.y > kMagic ? fminf(u.y, kMagic + 3.0f) : kMagic;
            }
            ulo[k] = __float_as_uint(u.x);
            uhi[k] = __float_as_uint(u.y);
        }
        w[m] = pack16(ulo);
        w[4 + m] = pack16(uhi);
    }
}

// min / max that return NaN when any input is NaN
__device__ __forceinline__ float min_nan(float a, float b) {
    float d;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ float max_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ float min3_nan(float a, float b, float c) {
    float d;
    asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
    float d;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Token-wise asymmetric quantisation of one row with CB-bit codes (4: 64 bytes, 2: 32
// bytes) and the (scale, zero) word.  A NaN anywhere in the row makes its min and max
// NaN: every code 0, scale = zero = fp16 quiet NaN.
template <int CB>
__device__ __forceinline__ void quantise_store(const float2 (&R)[64], uint8_t* codes_dst, uint32_t* sz_dst) {
    constexpr float kLevels = CB == 4 ? 15.0f : 3.0f;
    float mn4[4], mx4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        mn4[k] = min_nan(R[k].x, R[k].y);
        mx4[k] = max_nan(R[k].x, R[k].y);
    }
#pragma unroll
    for (int i = 4; i < 64; ++i) {
        mn4[i & 3] = min3_nan(mn4[i & 3], R[i].x, R[i].y);
        mx4[i & 3] = max3_nan(mx4[i & 3], R[i].x, R[i].y);
    }
    float mn = min3_nan(mn4[0], mn4[1], min_nan(mn4[2], mn4[3]));
    float mx = max3_nan(mx4[0], mx4[1], max_nan(mx4[2], mx4[3]));
    if (mn != mn) {
        const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        st_global_v8(codes_dst, z);
        if (CB == 4) st_global_v8(codes_dst + 32, z);
        *sz_dst = 0x7E007E00u;
        return;
    }
    mn = __fadd_rn(mn, 0.0f);  // -0 + +0 = +0: canonical signed zero
    mx = __fadd_rn(mx, 0.0f);
    const float range = __fsub_rn(mx, mn);
    const float s32 = __fdiv_rn(range, kLevels);
    const __half sh = __float2half_rn(s32);
    const __half zh = __float2half_rn(mn);
    const float sf = __half2float(sh);
    const float zf = __half2float(zh);
    const float inv = sf > 0.0f ? __frcp_rn(sf) : 0.0f;
    // The quantiser is monotone in y, so the row's extreme codes decide whether any
    // element needs clamping (an infinite scale or zero fails the test).
    const float umin = __fmaf_rn(__fsub_rn(mn, zf), inv, kMagic);
    const float umax = __fmaf_rn(__fsub_rn(mx, zf), inv, kMagic);
    const bool in_range = (umin >= kMagic) && (umax <= kMagic + kLevels);
    if (CB == 4) {
        uint32_t wa[8], wb[8];
        if (in_range)
            quantise_pack<false>(R, zf, inv, wa, wb);
        else
            quantise_pack<true>(R, zf, inv, wa, wb);
        st_global_v8(codes_dst, wa);
        st_global_v8(codes_dst + 32, wb);
    } else {
        uint32_t w[8];
        if (in_range)
            quantise_pack2<false>(R, zf, inv, w);
        else
            quantise_pack2<true>(R, zf, inv, w);
        st_global_v8(codes_dst, w);
    }
    *sz_dst = uint32_t(__half_as_ushort(sh)) | (uint32_t(__half_as_ushort(zh)) << 16);
}

// Rotary embedding of one row, rotate-half pairs: R[i] = (x_i, x_{i+64}) turns by the
// angle of pair i at the token's position, cs = that position's (cos, sin) table row:
// x_i' = fl(fl(x_i c) - fl(x_{i+64} s)), x_{i+64}' = fl(fl(x_{i+64} c) + fl(x_i s)),
// scalar IEEE ops (never contracted).
__device__ __forceinline__ void rope_row(float2 (&R)[64], const float* cs) {
    const float4* t = reinterpret_cast<const float4*>(cs);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float4 w = __ldg(t + j);  // pairs 2j and 2j + 1: (cos, sin, cos, sin)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float c = e ? w.z : w.x, s = e ? w.w : w.y;
            const float x = R[2 * j + e].x, y = R[2 * j + e].y;
            R[2 * j + e] = make_float2(__fsub_rn(__fmul_rn(x, c), __fmul_rn(y, s)),
                                       __fadd_rn(__fmul_rn(y, c), __fmul_rn(x, s)));
        }
    }
}

// fp32 -> bf16 bits, round to nearest even; NaN -> 0x7FC0
__device__ __forceinline__ uint32_t bf16_rn_bits(float f) {
    const uint32_t u = __float_as_uint(f);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0x7FC0u;
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

// BF16 cache with RoPE: the turned key row, rounded to bf16, into the pool row.
__device__ __forceinline__ void copy_row_rope(const uint8_t* stage, int row, const float* cs, uint8_t* dst) {
    float2 R[64];
    load_row(stage, row, R);
    rope_row(R, cs);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 16 elements (32 bytes) per store
            uint32_t w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int i = 16 * q + 2 * k;
                const float a = half ? R[i].y : R[i].x, b = half ? R[i + 1].y : R[i + 1].x;
                w[k] = bf16_rn_bits(a) | (bf16_rn_bits(b) << 16);
            }
            st_global_v8(dst + half * 128 + q * 32, w);
        }
    }
}

template <bool ROT, int BLK, int CB>
__device__ __forceinline__ void process_row(const uint8_t* stage, int row, float r_b, const float* cs,
                                            uint8_t* cdst, uint32_t* sdst) {
    float2 R[64];
    load_row(stage, row, R);
    if (cs) rope_row(R, cs);
    if (ROT) rotate_row<BLK>(R, r_b);
    quantise_store<CB>(R, cdst, sdst);
}

// BF16 cache: copy the row unchanged.
__device__ __forceinline__ void copy_row(const uint8_t* stage, int row, uint8_t* dst) {
    const uint4* h0 = reinterpret_cast<const uint4*>(stage + row * 128);
    const uint4* h1 = reinterpret_cast<const uint4*>(stage + kHalfBytes + row * 128);
    const int sw = row & 7;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const uint4* src = half ? h1 : h0;
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const uint4 a = src[j ^ sw], b = src[(j + 1) ^ sw];
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            st_global_v8(dst + half * 128 + j * 16, w);
        }
    }
}

template <int MODE, int BLK, bool ROTV, bool ROPE, int CB>
__global__ void __launch_bounds__(kThreads, 1)
    append_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                  const __grid_constant__ CUtensorMap kmap_s, const __grid_constant__ CUtensorMap vmap_s, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    int2* meta = reinterpret_cast<int2*>(smem + kStages * kStageBytes);  // [tile parity][tile token] = (page, slot)
    int* mpos = reinterpret_cast<int*>(meta + 2 * kMaxTileTokens);       // [tile parity][tile token] = position
    uint64_t* full = reinterpret_cast<uint64_t*>(mpos + 2 * kMaxTileTokens);
    uint64_t* empty = full + kStages;
    // set by the producer when it gives up a wait: a stage released after that carries no
    // tile and its consumers leave without reading it
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int TT = p.tile_tokens;
    const int H = p.g.H;
    const int c0 = blockIdx.x * p.chunk_tokens;  // this CTA's chunk of tokens
    const int len = min(p.chunk_tokens, p.a.num_tokens - c0);
    const int ntiles = len > 0 ? (len + TT - 1) / TT : 0;
    if (tid == 0) {
        for (int e = 0; e < kStages; ++e) {
            mbar_init(&full[e], 1);
            mbar_init(&empty[e], kRows / 32);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    grid_dep_wait();  // inputs and cache as the previous grid left them
    grid_dep_launch();

    if (warp == kRows / 32) {
        // ---------------- producer warp ----------------
        // Per tile: load the next tile's (sequence, position) ids, issue this tile's K and V
        // stage copies, resolve this tile's page slots (one dependent load, overlapped with
        // the copies) into its meta slot, then release both stages.
        const uint64_t pol = policy_evict_first();
        constexpr int kPerLane = (kMaxTileTokens + 31) / 32;
        int sq[kPerLane], po[kPerLane];
        auto load_ids = [&](int j, int (&a)[kPerLane], int (&b)[kPerLane]) {
            const Tile tl = tile_of(c0, len, TT, j);
#pragma unroll
            for (int r = 0; r < kPerLane; ++r) {
                const int tt = lane + 32 * r;
                const int t = tl.first + tt;
                const bool in = tt < tl.count;
                a[r] = in ? __ldg(p.a.tok_seq + t) : -1;
                b[r] = in ? __ldg(p.a.tok_pos + t) : -1;
            }
        };
        // Before the warp leaves: every stage copy it issued (issued = fills so far) has
        // landed, waited for with the usual bound, so the CTA never exits while a bulk copy
        // into its shared memory is in flight.
        auto drain = [&](int issued) {
            for (int e = 0; e < kStages; ++e) {
                if (issued > e && !mbar_wait(&full[e], ((issued - 1 - e) / kStages) & 1))
                    flag_error(p.err, kErrTimeout);
            }
        };
        load_ids(0, sq, po);
        int seqno = 0;
        for (int n = 0; n < ntiles; ++n) {
            const Tile tl = tile_of(c0, len, TT, n);
            // a short tile within the short maps' box takes them: its copy is its own rows
            const bool short_box = tl.count <= p.short_tokens;
            int nsq[kPerLane], npo[kPerLane];
            load_ids(n + 1, nsq, npo);
            int es[2];
            for (int kv = 0; kv < 2; ++kv, ++seqno) {
                const int e = seqno % kStages;
                const uint32_t fill = seqno / kStages;
                es[kv] = e;
                if (fill > 0 && !mbar_wait(&empty[e], (fill - 1) & 1)) {
                    flag_error(p.err, kErrTimeout);
                    // release the K stage this tile already filled (its arrival completes the
                    // phase; the flag tells its consumers to skip it), then drain and leave
                    if (lane == 0) {
                        *abort_flag = 1;
                        if (kv == 1) mbar_arrive(&full[es[0]]);
                    }
                    __syncwarp();
                    drain(seqno);
                    return;
                }
                if (lane == 0) {
                    const CUtensorMap* map = short_box ? (kv ? &vmap_s : &kmap_s) : (kv ? &vmap : &kmap);
                    uint8_t* dst = stages + e * kStageBytes;
                    // a box counts its full size in bytes, rows past the input's end included
                    mbar_expect_tx(&full[e], short_box ? uint32_t(p.short_tokens * H) * 256u : uint32_t(kStageBytes));
                    tma_load_3d(dst, map, &full[e], 0, 0, tl.first * H, pol);
                    tma_load_3d(dst + kHalfBytes, map, &full[e], 0, 1, tl.first * H, pol);
                }
            }
            // the meta slot of tile n was last read for tile n - 2, whose stages the waits above freed
            int2* mt = meta + (n & 1) * kMaxTileTokens;
            int* mp = mpos + (n & 1) * kMaxTileTokens;
#pragma unroll
            for (int r = 0; r < kPerLane; ++r) {
                const int tt = lane + 32 * r;
                if (tt < TT) {
                    int2 m = make_int2(-1, 0);
                    if (tt < tl.count) {
                        const int sid = sq[r], pos = po[r];
                        bool ok = sid >= 0 && sid < p.a.num_seqs && pos >= 0 && pos / p.g.page_size < p.a.pt_stride &&
                                  (!ROPE || pos < p.g.rope_positions);
                        if (ok) {
                            const int page = __ldg(p.a.page_table + int64_t(sid) * p.a.pt_stride + pos / p.g.page_size);
                            ok = page >= 0 && page < p.g.num_pages;
                            if (ok) m = make_int2(page, pos % p.g.page_size);
                        }
                        if (!ok) flag_error(p.err, kErrOOB);
                    }
                    mt[tt] = m;
                    if (ROPE) mp[tt] = po[r];
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&full[es[0]]);
                mbar_arrive(&full[es[1]]);
            }
#pragma unroll
            for (int r = 0; r < kPerLane; ++r) {
                sq[r] = nsq[r];
                po[r] = npo[r];
            }
        }
        drain(seqno);
        return;
    }

    // ---------------- consumer warps: thread tid owns row tid of each stage ----------------
    const int tt = tid / H, h = tid % H;
    int seqno = 0;
    for (int n = 0; n < ntiles; ++n) {
        const Tile tl = tile_of(c0, len, TT, n);
        int2 m = make_int2(-1, 0);
#pragma unroll 1
        for (int kv = 0; kv < 2; ++kv, ++seqno) {
            const int e = seqno % kStages;
            const uint32_t fill = seqno / kStages;
            if (!mbar_wait(&full[e], fill & 1)) {
                flag_error(p.err, kErrTimeout);
                return;
            }
            if (*abort_flag) return;  // the producer gave up: this stage holds no tile
            if (kv == 0) m = meta[(n & 1) * kMaxTileTokens + tt];
            // key rows turn at the token's position (the position was checked by the producer)
            const float* cs = (ROPE && kv == 0 && m.x >= 0)
                                  ? p.g.rope + int64_t(mpos[(n & 1) * kMaxTileTokens + tt]) * kHeadDim
                                  : nullptr;
            if (tt < tl.count && m.x >= 0) {
                const uint8_t* stage = stages + e * kStageBytes;
                const int64_t row = (int64_t(m.x) * H + h) * p.g.page_size + m.y;
                if (MODE == 0) {
                    uint8_t* dst = static_cast<uint8_t*>(kv ? p.g.v_pool : p.g.k_pool) + row * 256;
                    if (ROPE && cs)
                        copy_row_rope(stage, tid, cs, dst);
                    else
                        copy_row(stage, tid, dst);
                } else {
                    uint8_t* cdst = static_cast<uint8_t*>(kv ? p.g.v_pool : p.g.k_pool) + row * (16 * CB);
                    uint32_t* sdst = (kv ? p.g.v_sz : p.g.k_sz) + row;
                    if (MODE != 2 || ROTV)  // K and V rows take the same path: one copy of it
                        process_row<MODE == 2, BLK, CB>(stage, tid, p.r_b, ROPE ? cs : nullptr, cdst, sdst);
                    else if (kv == 0)
                        process_row<true, BLK, CB>(stage, tid, p.r_b, ROPE ? cs : nullptr, cdst, sdst);
                    else
                        process_row<false, BLK, CB>(stage, tid, p.r_b, nullptr, cdst, sdst);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[e]);
        }
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [T*H rows, 2 halves, 64 bf16] view of a [T, H, 128] bf16 input; box = one
// 128-byte half of box_rows consecutive rows, 128-byte swizzle.
bool make_row_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {64, 2, cuuint64_t(rows)};
    cuuint64_t strides[2] = {128, 256};
    cuuint32_t box[3] = {64, 1, cuuint32_t(box_rows)};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Maps {
    CUtensorMap k, v;    // whole tiles: kRows rows
    CUtensorMap ks, vs;  // short tiles: short_tokens * H rows
};

template <int MODE, int BLK, bool ROTV, bool ROPE, int CB>
cudaError_t launch_r(const Maps& m, const Params& p, int grid, cudaStream_t s) {
    constexpr auto kern = append_kernel<MODE, BLK, ROTV, ROPE, CB>;
    const cudaError_t e = ensure_smem_opt_in<kern>(kSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_overlapped(kern, dim3(grid), dim3(kThreads), kSmemBytes, s, m.k, m.v, m.ks, m.vs, p);
}

template <int MODE, int BLK, bool ROTV, bool ROPE>
cudaError_t launch_c(const Maps& m, const Params& p, int grid, cudaStream_t s) {
    if (MODE != 0 && p.g.code_bits == 2) return launch_r<MODE, BLK, ROTV, ROPE, 2>(m, p, grid, s);
    return launch_r<MODE, BLK, ROTV, ROPE, 4>(m, p, grid, s);
}

template <int MODE, int BLK, bool ROTV>
cudaError_t launch_t(const Maps& m, const Params& p, int grid, cudaStream_t s) {
    return p.g.rope ? launch_c<MODE, BLK, ROTV, true>(m, p, grid, s) : launch_c<MODE, BLK, ROTV, false>(m, p, grid, s);
}

}  // namespace

cudaError_t launch_append(const CacheGeom& g, const AppendArgs& a, int* err_word, int num_sms, cudaStream_t s) {
    if (a.num_tokens == 0) return cudaSuccess;
    if (num_sms < 1) return cudaErrorInvalidValue;
    const int64_t rows = int64_t(a.num_tokens) * g.H;
    Params p;
    p.g = g;
    p.a = a;
    p.tile_tokens = kRows / g.H;
    // equal chunks of ceil(T / SMs) tokens; grid = the chunks that hold tokens
    p.chunk_tokens = (a.num_tokens + num_sms - 1) / num_sms;
    const int grid = (a.num_tokens + p.chunk_tokens - 1) / p.chunk_tokens;
    p.short_tokens = p.chunk_tokens % p.tile_tokens;
    p.r_b = g.mode == 2 ? float(1.0 / sqrt(double(g.bdr_block))) : 1.0f;
    p.err = err_word;
    Maps m;
    if (!make_row_map(&m.k, a.k, rows, kRows) || !make_row_map(&m.v, a.v, rows, kRows)) return cudaErrorInvalidValue;
    if (p.short_tokens > 0) {
        if (!make_row_map(&m.ks, a.k, rows, p.short_tokens * g.H) ||
            !make_row_map(&m.vs, a.v, rows, p.short_tokens * g.H))
            return cudaErrorInvalidValue;
    } else {  // never taken (no tile has count <= 0); passed so that every parameter is a valid map
        m.ks = m.k;
        m.vs = m.v;
    }
    if (g.mode == 0) return launch_t<0, 128, false>(m, p, grid, s);
    if (g.mode == 1) return launch_t<1, 128, false>(m, p, grid, s);
    switch (g.bdr_block * 2 + (g.rotate_v ? 1 : 0)) {
        case 32: return launch_t<2, 16, false>(m, p, grid, s);
        case 33: return launch_t<2, 16, true>(m, p, grid, s);
        case 64: return launch_t<2, 32, false>(m, p, grid, s);
        case 65: return launch_t<2, 32, true>(m, p, grid, s);
        case 128: return launch_t<2, 64, false>(m, p, grid, s);
        case 129: return launch_t<2, 64, true>(m, p, grid, s);
        case 256: return launch_t<2, 128, false>(m, p, grid, s);
        case 257: return launch_t<2, 128, true>(m, p, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
