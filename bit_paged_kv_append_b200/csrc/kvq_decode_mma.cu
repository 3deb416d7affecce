// kvq_decode_mma.cu -- paged GQA decode attention over the INT4 cache on the
// tensor cores (mma.sync: int8 and fp16 operands, int32 / fp32 accumulation).
//
// SAW-INT4 (wispaper.ai blog, section 3): the query is rotated in step with
// H_blk, so q' k^ needs no inverse rotation of the cache; the abstract keeps
// fused attention over the paged INT4 layout.  Dequantisation is factored:
//   q' . (scale c + zero) = scale (q' . c) + zero sum(q')
//   sum_t p_t (scale_t c_t + zero_t) = sum_t (p_t scale_t) c_t + sum_t p_t zero_t
// so both contractions run on raw 4-bit codes.
//
// One CTA = (split, KV head, sequence), 4 warps; each warp walks 16-token
// chunks of its split (round robin), with its own online-softmax state.  The
// CTA prepares q first (it may overlap the end of the previous grid in the
// stream: programmatic dependent launch), then waits for that grid and starts
// its copies.
//   * Staging: per warp a ring of 4 shared-memory stages, 4 chunks in flight;
//     all 32 lanes copy a chunk's K codes, V codes and scale/zero words (2176
//     B) with 16-byte cp.async (one copy group per chunk), so no lane runs a
//     divergent issue path.  Page sizes that are not a multiple of 16 take a
//     per-token gather of the same form.
//   * P.V (both tiles): D[16 dims x 8 cols] += A[16 dims x 16 tokens] B[16 tokens
//     x 8 cols].  A = V codes of two tokens per register (PRMT + AND) masked
//     into fp16 lanes, where a nibble c is the exact subnormal c 2^-24, and
//     centred to c - 8 by one exact fp16 add.  Centring keeps the accumulator
//     small: the tensor cores' fp32 accumulation does not round to nearest, and
//     over thousands of tokens sum (p scale) c and sum p zero would otherwise
//     nearly cancel.  B = p scale_v as an fp16 high part plus an fp16 low part
//     (one fp16 rounding of p scale would cost ~1e-3 of the output).
//
// Two tiles, by the number G of query heads per KV head:
//   G = 8, heads on M (decode_mma_kernel): q.K is D[16 x 8 tokens] = A[16 x 32
//     dims] B[32 dims x 8 tokens] on the int8 tensor path: A = q' as 23-bit
//     fixed point in three signed bytes (m-tile 0: the 8 heads' high bytes in
//     rows 0..7, middle bytes in rows 8..15; m-tile 1: the low bytes), B = codes
//     as bytes (AND / shift-AND); the int32 accumulation is exact.  The score of
//     (head, token) then sits in the thread that needs it as the P.V B operand;
//     the low part of B is a second mma.
//   G <= 4, tokens on M (decode_tok_kernel): q.K is D[16 tokens x 8 cols] =
//     A[16 tokens x 32 dims] B[32 dims x 8 cols] on the int8 tensor path: A =
//     codes as bytes (AND / shift-AND, 8 codes for 3 instructions), B = q' as
//     23-bit fixed point per head in three signed bytes (n-tile 0: 4 heads x
//     {high, middle}; n-tile 1: the low bytes); the int32 accumulation is exact.
//     Every lane holds two real scores (no idle rows at G = 4), and the P.V B
//     operand takes its 8 columns as 4 heads x {high, low part of p scale}, so
//     the low part costs no extra mma; two shuffles move each score from the
//     q.K layout to the B layout.
//   * 2-bit codes (the pages leave 2-bit open): the stage holds 32-byte rows; each
//     load site reads half as many bytes and spreads them into the 4-bit nibble
//     layout in registers, so every fragment mapping above is shared.
//   * Which dimension and which token each fragment slot stands for is a fixed
//     permutation chosen so that every thread reads contiguous bytes and the
//     shared-memory reads are conflict-free; the output mapping undoes it.
#include <type_traits>

#include "kvq_mma.cuh"

namespace kvq {
namespace {

// Merge scratch mo [warp][G][128]: each 16-byte chunk of a head's row is stored at chunk
// c ^ mo_swz(g), so the four 16-byte stores per lane of a 16-dim segment (the 8 lanes of
// one store phase: two segments x four heads) hit distinct bank groups.
template <int G>
__device__ __forceinline__ int mo_swz(int g) { return G == 8 ? (g >> 1) & 3 : g & 3; }
template <int G>
__device__ __forceinline__ int mo_idx(int row, int g, int d) {
    return row * kHeadDim + ((((d >> 2) ^ mo_swz<G>(g))) << 2) + (d & 3);
}
// dims 16 gq .. 16 gq + 15 of head g (v[i] = dim 16 gq + i) into the merge scratch row
template <int G>
__device__ __forceinline__ void mo_store16(float* mo, int row, int g, int gq, const float (&v)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
        *reinterpret_cast<float4*>(mo + mo_idx<G>(row, g, 16 * gq + 4 * c)) =
            make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

// Merge the 4 warps' partial states (mo [warp][G][128] outputs incl. the offset
// term, mm / ml [warp][G] max and weight sum) and store the split's partial rows.
template <int G>
__device__ __forceinline__ void store_partials(const DecodeParams& p, const float* mo, const float* mm,
                                               const float* ml, int s, int k, int h, int tid) {
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
            acc += f * mo[mo_idx<G>(w * G + g, g, tid)];
            lt += f * ml[w * G + g];
        }
        const int64_t r = partial_row(p, s, k, h * G + g);
        p.ws_o[r * kHeadDim + tid] = acc;
        if (tid == 0) p.ws_ml[r] = make_float2(M, lt);
    }
}

// Common start of a CTA: split bounds and the chunk stream.  False: no tokens.
template <int CB>
__device__ __forceinline__ bool begin_split(const DecodeParams& p, CtaRing& R, ChunkStream<CB>& cs, int warp, int lane,
                                            int tid) {
    const int k = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int L = decode_len(p, s);
    if (k == 0 && h == 0 && tid == 0 && L != __ldg(p.a.seq_lens + s)) flag_error(p.err, kErrOOB);
    const int t0 = k * p.item_tokens;
    if (t0 >= L) {  // past the end of the sequence: no partial (the merge reads only real splits)
        grid_dep_wait();  // still: no grid here completes before the one it follows
        grid_dep_launch();
        return false;
    }
    cs.r = &R;
    cs.pt = p.a.page_table + int64_t(s) * p.a.pt_stride;
    cs.t0 = t0;
    cs.t1 = min(L, t0 + p.item_tokens);
    const int nchunks = (cs.t1 - t0 + kChunk - 1) / kChunk;
    cs.nw = nchunks > warp ? (nchunks - warp + kWarps - 1) / kWarps : 0;  // this warp's chunks
    cs.warp = warp;
    cs.first = warp;
    cs.step = kWarps;
    cs.lane = lane;
    cs.h = h;
    cs.fast = (p.g.page_size % kChunk) == 0;
    cs.pol = policy_evict_first();
    cs.init(p);
    return true;
}

// =====================================================================================
// G = 8: heads on M, fp16 q.K
// =====================================================================================
template <int G, int CB>
__global__ void __launch_bounds__(kThreads, 4) decode_mma_kernel(DecodeParams p) {
    __shared__ __align__(128) CtaRing R;
    // q.K A operands (4 x s8 per word) in fragment order: m-tile 0 (rows hi | mid), [k-step][reg][lane];
    // m-tile 1 (rows lo | zero), [k-step][even / odd dims][lane]
    __shared__ uint32_t As[4 * 4 * 32 + 4 * 2 * 32];
    __shared__ float qsc_s[kMaxGroup], qsn_s[kMaxGroup];  // per head: fixed-point step, sum of q_int

    const int k = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, pq = lane & 3;  // mma group id / thread in group
    ChunkStream<CB> cs;
    if (!begin_split(p, R, cs, warp, lane, tid)) return;
    for (int w = tid; w < 4 * 4 * 32 + 4 * 2 * 32; w += kThreads) As[w] = 0u;
    __syncthreads();
    const int nw = cs.nw, t1 = cs.t1;

    // ---------------- q' as 23-bit fixed point per head, A fragment order ----------------
    // k-step j, k-slot 4 pq + i (registers 0, 1) / 16 + 4 pq + i (registers 2, 3) stand for
    // dim 32 pq + 8 j + 2 i (+ 1); m-tile 0: rows 0..7 hi, rows 8..15 mid; m-tile 1: rows
    // 0..7 lo, rows 8..15 zero.
    for (int row = warp; row < G; row += kWarps) {
        float x[4];
        load_q_rotated(p, int64_t(s) * p.g.Hq + h * G + row, __ldg(p.a.seq_lens + s) - 1, lane, x);
        float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
        const float inv = amax > 0.0f ? float(kQFix) / amax : 0.0f;
        int qi[4], isum = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            qi[c] = min(max(__float2int_rn(x[c] * inv), -kQFix), kQFix);
            isum += qi[c];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(kFull, isum, o);
        if (lane == 0) {
            qsc_s[row] = amax / float(kQFix);
            qsn_s[row] = float(isum);
        }
        uint8_t* A8 = reinterpret_cast<uint8_t*>(As);
        uint8_t* A8lo = reinterpret_cast<uint8_t*>(As + 4 * 4 * 32);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int d = 4 * lane + c;
            const int dp = d >> 5, j = (d >> 3) & 3, i = (d >> 1) & 3, odd = d & 1;
            int hi, mid, lo;
            q_digits(qi[c], hi, mid, lo);
            const int lw = 4 * row + dp;  // lane of row gq = row
            A8[((j * 4 + 2 * odd) * 32 + lw) * 4 + i] = uint8_t(hi);
            A8[((j * 4 + 2 * odd + 1) * 32 + lw) * 4 + i] = uint8_t(mid);
            A8lo[((j * 2 + odd) * 32 + lw) * 4 + i] = uint8_t(lo);
        }
    }
    // q only (never written by an append) so far; the cache after the previous grid
    grid_dep_wait();
    grid_dep_launch();
    for (int i = 0; i < kStages; ++i) {
        if (i < nw) cs.issue(p, i, i);
        cp_async_commit();
    }
    __syncthreads();
    uint32_t A[4][4], Alo[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int r = 0; r < 4; ++r) A[j][r] = As[(j * 4 + r) * 32 + lane];
#pragma unroll
        for (int r = 0; r < 2; ++r) Alo[j][r] = As[4 * 4 * 32 + (j * 2 + r) * 32 + lane];
    }
    const float qsc = gq < G ? qsc_s[gq] : 0.0f, qsn = gq < G ? qsn_s[gq] : 0.0f;

    // ---------------- main loop over this warp's chunks ----------------
    // softmax state of head gq (q.K layout); rows gq >= G stand for no head: their m stays 0
    // and every score -inf, so they never trigger a rescale and their weights are 0
    const bool gval = gq < G;
    float m = gval ? -INFINITY : 0.0f, l = 0.0f, Z = 0.0f;
    float O[8][4];  // P.V accumulators: dims x heads (2 pq, 2 pq + 1)
#pragma unroll
    for (int j = 0; j < 8; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.0f;
    const int tokA = sigma(2 * pq), tokB = sigma(2 * pq + 1), tokK = sigma(gq);

    for (int i = 0; i < nw; ++i) {
        const int slot = i % kStages;
        cp_async_wait<kStages - 1>();  // chunk i's group (the stream keeps kStages groups)
        __syncwarp();                   // ... and every lane's copies of it
        const uint8_t* st = R.stage[warp][slot];
        const uint32_t vmask = R.mask[warp][slot];
        const int tb = cs.t0 + (warp + kWarps * i) * kChunk;
        stage_szf<CB>(R, st, warp, lane, 1.0f, kPScale);

        // ---- scores: q_int . codes for the two 8-token n-tiles (column gq: token 8 tau + tokK) ----
        float C[2][2];
#pragma unroll
        for (int tau = 0; tau < 2; ++tau) {
            const uint4 kw = key_codes<CB>(st, 8 * tau + tokK, pq);
            const uint32_t w[4] = {kw.x, kw.y, kw.z, kw.w};
            int D[4] = {0, 0, 0, 0}, E[4] = {0, 0, 0, 0};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t b0 = w[j] & 0x0F0F0F0Fu, b1 = (w[j] >> 4) & 0x0F0F0F0Fu;
                const uint32_t alo[4] = {Alo[j][0], 0u, Alo[j][1], 0u};
                mma16832_s8u8(D, A[j], b0, b1);
                mma16832_s8u8(E, alo, b0, b1);
            }
            C[tau][0] = q_dot(D[0], D[2], E[0]);  // head gq, column 2 pq
            C[tau][1] = q_dot(D[1], D[3], E[1]);  // head gq, column 2 pq + 1
        }
        // A chunk whose 16 tokens all lie before the end and on valid pages (FULL, the common
        // case) needs no per-token masks; the two cases are separate code paths.
        uint32_t b0, b1, b0l, b1l;
        auto softmax = [&](auto full_c) {
            constexpr bool FULL = decltype(full_c)::value;
            float sc[2][2];
#pragma unroll
            for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int lt = 8 * tau + (e ? tokB : tokA);
                    const float2 kz = R.szf[warp][0][lt];
                    const float v = qsc * fmaf(kz.x, C[tau][e], kz.y * qsn);
                    const bool valid = gval && (FULL || ((tb + lt < t1) && ((vmask >> lt) & 1u)));
                    sc[tau][e] = valid ? v : -INFINITY;
                }
            // ---- online softmax (log2 domain) for head gq ----
            float cm = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
            cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 1));
            cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 2));
            const bool up = cm > m + kTau;  // lazily moved reference (m = -inf: any finite cm)
            const float mn = up ? cm : m;
            if (__any_sync(kFull, up)) {
                const float alpha = up ? fast_exp2(m - mn) : 1.0f;
                l *= alpha;
                Z *= alpha;
                m = mn;
                const float a0 = __shfl_sync(kFull, alpha, 8 * pq);
                const float a1 = __shfl_sync(kFull, alpha, 8 * pq + 4);
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
                    const int lt = 8 * tau + (e ? tokB : tokA);
                    float pr;
                    float2 vz;
                    if (FULL) {  // rows past the group hold m = 0 and scores -inf: weight 0
                        pr = fast_exp2(sc[tau][e] - m);
                        vz = R.szf[warp][1][lt];
                    } else {
                        // masked tokens (past the end, skipped pages, stale slots) may hold any
                        // bits in their scale/zero word: never let them reach an operand, even times 0
                        const bool live = sc[tau][e] != -INFINITY;
                        pr = live ? fast_exp2(sc[tau][e] - m) : 0.0f;
                        vz = live ? R.szf[warp][1][lt] : make_float2(0.0f, 0.0f);
                    }
                    l += pr;
                    Z += pr * vz.y;
                    pt_[tau][e] = pr * vz.x;
                }
            }
            b0 = pack_half2(pt_[0][0], pt_[0][1]);
            b1 = pack_half2(pt_[1][0], pt_[1][1]);
            b0l = pack_half2(pt_[0][0] - half_lo(b0), pt_[0][1] - half_hi(b0));
            b1l = pack_half2(pt_[1][0] - half_lo(b1), pt_[1][1] - half_hi(b1));
        };
        if ((tb + kChunk <= t1) && (vmask == 0xFFFFu))
            softmax(std::true_type{});
        else
            softmax(std::false_type{});
        pv_chunk<true, CB>(O, st, gq, tokA, tokB, b0, b1, b0l, b1l);
        __syncwarp();  // every lane is done with this slot
        if (i + kStages < nw) cs.issue(p, i + kStages, slot);
        cp_async_commit();
    }

    // ---------------- per-head totals, undo the 2^-24 code scale, merge the warps ----------------
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    Z += __shfl_xor_sync(kFull, Z, 1);
    Z += __shfl_xor_sync(kFull, Z, 2);
    const float Z0 = __shfl_sync(kFull, Z, 8 * pq), Z1 = __shfl_sync(kFull, Z, 8 * pq + 4);
    __syncthreads();  // every ring is drained; reuse it for the merge
    float* mo = reinterpret_cast<float*>(&R.stage[0][0][0]);  // [warp][G][128]
    float* mm = mo + kWarps * G * kHeadDim;                   // [warp][G]
    float* ml = mm + kWarps * G;                              // [warp][G]
    const int h0 = 2 * pq, h1 = 2 * pq + 1;
    if (h0 < G) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            v[2 * j] = O[j][0] * (kTwo24 * kPOut) + Z0;
            v[2 * j + 1] = O[j][2] * (kTwo20 * kPOut) + Z0;
        }
        mo_store16<G>(mo, warp * G + h0, h0, gq, v);
    }
    if (h1 < G) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            v[2 * j] = O[j][1] * (kTwo24 * kPOut) + Z1;
            v[2 * j + 1] = O[j][3] * (kTwo20 * kPOut) + Z1;
        }
        mo_store16<G>(mo, warp * G + h1, h1, gq, v);
    }
    if (pq == 0 && gq < G) {
        mm[warp * G + gq] = m;
        ml[warp * G + gq] = l;
    }
    __syncthreads();
    store_partials<G>(p, mo, mm, ml, s, k, h, tid);
}

// =====================================================================================
// G <= 4: tokens on M, int8 q.K
// =====================================================================================
template <int G, int CB>
__global__ void __launch_bounds__(kThreads, 5) decode_tok_kernel(DecodeParams p) {
    static_assert(G >= 1 && G <= 4, "tokens-on-M tile serves up to 4 query heads per KV head");
    __shared__ __align__(128) CtaRing R;
    // q.K B operands (4 x s8 per word) in fragment order, [k-step][reg][lane]: n-tile 0
    // (columns 2 head: hi, 2 head + 1: mid), n-tile 1 (columns 2 head: lo, odd columns zero)
    __shared__ uint32_t Bs[2 * 4 * 2 * 32];
    __shared__ float qsc_s[4], qsn_s[4];  // per head: fixed-point step of q', sum of the fixed-point q'

    const int k = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, pq = lane & 3;
    ChunkStream<CB> cs;
    if (!begin_split(p, R, cs, warp, lane, tid)) return;
    for (int w = tid; w < 2 * 4 * 2 * 32; w += kThreads) Bs[w] = 0u;
    __syncthreads();
    const int nw = cs.nw, t1 = cs.t1;

    // ---------------- q' as 23-bit fixed point per head, B fragment order ----------------
    // k-step j, k-slot 4 pq + i (register 0) / 16 + 4 pq + i (register 1) stand for dim
    // 32 pq + 8 j + 2 i (+ 1): the low / high nibbles of bytes 16 pq + 4 j + i.
    // n-tile 0, column 2 head + part: part 0 holds hi, part 1 mid; n-tile 1, column
    // 2 head: lo.
    for (int row = warp; row < G; row += kWarps) {
        float x[4];
        load_q_rotated(p, int64_t(s) * p.g.Hq + h * G + row, __ldg(p.a.seq_lens + s) - 1, lane, x);
        float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
        const float inv = amax > 0.0f ? float(kQFix) / amax : 0.0f;
        int qi[4], isum = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            qi[c] = min(max(__float2int_rn(x[c] * inv), -kQFix), kQFix);
            isum += qi[c];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(kFull, isum, o);
        if (lane == 0) {
            qsc_s[row] = amax / float(kQFix);
            qsn_s[row] = float(isum);
        }
        uint8_t* B8 = reinterpret_cast<uint8_t*>(Bs);
        uint8_t* B8lo = reinterpret_cast<uint8_t*>(Bs + 4 * 2 * 32);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int d = 4 * lane + c;
            const int dp = d >> 5, j = (d >> 3) & 3, i = (d >> 1) & 3, r = d & 1;
            int hi, mid, lo;
            q_digits(qi[c], hi, mid, lo);
            B8[((j * 2 + r) * 32 + 4 * (2 * row) + dp) * 4 + i] = uint8_t(hi);
            B8[((j * 2 + r) * 32 + 4 * (2 * row + 1) + dp) * 4 + i] = uint8_t(mid);
            B8lo[((j * 2 + r) * 32 + 4 * (2 * row) + dp) * 4 + i] = uint8_t(lo);
        }
    }
    // q only (never written by an append) so far; the cache after the previous grid
    grid_dep_wait();
    grid_dep_launch();
    for (int i = 0; i < kStages; ++i) {
        if (i < nw) cs.issue(p, i, i);
        cp_async_commit();
    }
    __syncthreads();
    uint32_t Bq[4][2], Blo[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            Bq[j][r] = Bs[(j * 2 + r) * 32 + lane];
            Blo[j][r] = Bs[4 * 2 * 32 + (j * 2 + r) * 32 + lane];
        }

    // ---------------- main loop over this warp's chunks ----------------
    // Thread (gq, pq) scores tokens tk, tk + 8 against head pq; heads >= G hold m = 0 and
    // scores -inf, so they never trigger a rescale and their weights are 0.
    const bool hv = pq < G;
    const float qsc = hv ? qsc_s[pq] : 0.0f, qsn = hv ? qsn_s[pq] : 0.0f;
    float m = hv ? -INFINITY : 0.0f, l = 0.0f, Z = 0.0f;
    float O[8][4];  // P.V accumulators: dims x (head pq high, head pq low)
#pragma unroll
    for (int j = 0; j < 8; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.0f;
    const int tk = sigma(gq), tokA = sigma(2 * pq), tokB = sigma(2 * pq + 1);
    // P.V B column gq = (head gq >> 1, part gq & 1) wants tokens tokA, tokB (+ 8) of that head,
    // which q.K left in lanes srcA = (row 2 pq, head) and srcB = (row 2 pq + 1, head).
    // Even rows send their high words first, odd rows their low words, so each
    // shuffle serves both parts.
    const bool part = (gq & 1) != 0;
    const int srcA = 4 * (2 * pq) + (gq >> 1), srcB = srcA + 4;
    const int src1 = part ? srcB : srcA, src2 = part ? srcA : srcB;
    const uint32_t sel0 = part ? 0x1054u : 0x5410u, sel1 = part ? 0x3276u : 0x7632u;

    for (int i = 0; i < nw; ++i) {
        const int slot = i % kStages;
        cp_async_wait<kStages - 1>();  // chunk i's group (the stream keeps kStages groups)
        __syncwarp();                   // ... and every lane's copies of it
        const uint8_t* st = R.stage[warp][slot];
        const uint32_t vmask = R.mask[warp][slot];
        const int tb = cs.t0 + (warp + kWarps * i) * kChunk;
        stage_szf<CB>(R, st, warp, lane, 1.0f, kPScale);

        // ---- scores: codes (tokens tk, tk + 8; bytes [16 pq, 16 pq + 16)) . q_int ----
        const uint4 k0 = key_codes<CB>(st, tk, pq);
        const uint4 k1 = key_codes<CB>(st, tk + 8, pq);
        const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w}, w1[4] = {k1.x, k1.y, k1.z, k1.w};
        int D[4] = {0, 0, 0, 0}, E[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t a[4] = {w0[j] & 0x0F0F0F0Fu, w1[j] & 0x0F0F0F0Fu, (w0[j] >> 4) & 0x0F0F0F0Fu,
                                   (w1[j] >> 4) & 0x0F0F0F0Fu};
            mma16832_u8s8(D, a, Bq[j][0], Bq[j][1]);
            mma16832_u8s8(E, a, Blo[j][0], Blo[j][1]);
        }
        const float S0 = q_dot(D[0], D[1], E[0]), S1 = q_dot(D[2], D[3], E[2]);
        const float2 kz0 = R.szf[warp][0][tk], kz1 = R.szf[warp][0][tk + 8];
        const float v0 = qsc * fmaf(kz0.x, S0, kz0.y * qsn), v1 = qsc * fmaf(kz1.x, S1, kz1.y * qsn);
        const bool full = (tb + kChunk <= t1) && (vmask == 0xFFFFu);
        const bool ok0 = hv && (full || ((tb + tk < t1) && ((vmask >> tk) & 1u)));
        const bool ok1 = hv && (full || ((tb + tk + 8 < t1) && ((vmask >> (tk + 8)) & 1u)));
        const float sc0 = ok0 ? v0 : -INFINITY, sc1 = ok1 ? v1 : -INFINITY;

        // ---- online softmax (log2 domain) for head pq: the 16 tokens sit in lanes pq + 4 n ----
        float cm = fmaxf(sc0, sc1);
        cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 4));
        cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 8));
        cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 16));
        const bool up = cm > m + kTau;  // lazily moved reference (m = -inf: any finite cm)
        const float mn = up ? cm : m;
        if (__any_sync(kFull, up)) {
            const float alpha = up ? fast_exp2(m - mn) : 1.0f;
            l *= alpha;
            Z *= alpha;
            m = mn;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                O[j][0] *= alpha;
                O[j][1] *= alpha;
                O[j][2] *= alpha;
                O[j][3] *= alpha;
            }
        }
        float p0, p1;
        float2 vz0, vz1;
        if (full) {
            p0 = fast_exp2(sc0 - m);
            p1 = fast_exp2(sc1 - m);
            vz0 = R.szf[warp][1][tk];
            vz1 = R.szf[warp][1][tk + 8];
        } else {
            // masked tokens (past the end, skipped pages, stale slots) may hold any bits
            // in their scale/zero word: never let them reach an operand, even times 0
            const float2 zz = make_float2(0.0f, 0.0f);
            p0 = ok0 ? fast_exp2(sc0 - m) : 0.0f;
            p1 = ok1 ? fast_exp2(sc1 - m) : 0.0f;
            vz0 = ok0 ? R.szf[warp][1][tk] : zz;
            vz1 = ok1 ? R.szf[warp][1][tk + 8] : zz;
        }
        l += p0 + p1;
        Z = fmaf(p0, vz0.y, fmaf(p1, vz1.y, Z));
        const float P0 = p0 * vz0.x, P1 = p1 * vz1.x;
        const uint32_t HI = pack_half2(P0, P1);
        const uint32_t LO = pack_half2(P0 - half_lo(HI), P1 - half_hi(HI));
        // ---- to the P.V B layout: (tokA, tokB) and (tokA + 8, tokB + 8) of column gq ----
        const uint32_t R1 = __shfl_sync(kFull, part ? LO : HI, src1);
        const uint32_t R2 = __shfl_sync(kFull, part ? HI : LO, src2);
        pv_chunk<false, CB>(O, st, gq, tokA, tokB, prmt(R1, R2, sel0), prmt(R1, R2, sel1), 0u, 0u);
        __syncwarp();  // every lane is done with this slot
        if (i + kStages < nw) cs.issue(p, i + kStages, slot);
        cp_async_commit();
    }

    // ---------------- per-head totals, undo the 2^-24 code scale, merge the warps ----------------
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l += __shfl_xor_sync(kFull, l, o);
        Z += __shfl_xor_sync(kFull, Z, o);
    }
    __syncthreads();  // every ring is drained; reuse it for the merge
    float* mo = reinterpret_cast<float*>(&R.stage[0][0][0]);  // [warp][G][128]
    float* mm = mo + kWarps * G * kHeadDim;                   // [warp][G]
    float* ml = mm + kWarps * G;                              // [warp][G]
    if (hv) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            v[2 * j] = (O[j][0] + O[j][1]) * (kTwo24 * kPOut) + Z;
            v[2 * j + 1] = (O[j][2] + O[j][3]) * (kTwo20 * kPOut) + Z;
        }
        mo_store16<G>(mo, warp * G + pq, pq, gq, v);
        if (gq == 0) {
            mm[warp * G + pq] = m;
            ml[warp * G + pq] = l;
        }
    }
    __syncthreads();
    store_partials<G>(p, mo, mm, ml, s, k, h, tid);
}

}  // namespace

cudaError_t launch_decode_mma(const DecodeParams& p, cudaStream_t s) {
    const dim3 grid(p.max_splits, p.g.H, p.a.batch);
    const bool two = p.g.code_bits == 2;
    switch (p.g.Hq / p.g.H) {
        case 1: return two ? launch_overlapped(decode_tok_kernel<1, 2>, grid, dim3(kThreads), 0, s, p)
                           : launch_overlapped(decode_tok_kernel<1, 4>, grid, dim3(kThreads), 0, s, p);
        case 2: return two ? launch_overlapped(decode_tok_kernel<2, 2>, grid, dim3(kThreads), 0, s, p)
                           : launch_overlapped(decode_tok_kernel<2, 4>, grid, dim3(kThreads), 0, s, p);
        case 4: return two ? launch_overlapped(decode_tok_kernel<4, 2>, grid, dim3(kThreads), 0, s, p)
                           : launch_overlapped(decode_tok_kernel<4, 4>, grid, dim3(kThreads), 0, s, p);
        case 8: return two ? launch_overlapped(decode_mma_kernel<8, 2>, grid, dim3(kThreads), 0, s, p)
                           : launch_overlapped(decode_mma_kernel<8, 4>, grid, dim3(kThreads), 0, s, p);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
