// kvq_extend.cu -- extend (chunked-prefill) attention over the paged cache with 2-bit codes
// on the mma.sync tensor cores (4-bit codes take the tcgen05 kernel in kvq_extend_tc.cu):
// the queries of a sequence's newest tokens, whose keys and values the append has already
// written, attend causally to the cached tokens.
//
// SAW-INT4's abstract keeps fused attention over the paged quantised layout as a
// serving constraint; chunked prefill in mixed serving reads the cache this way.  Query
// i of the n new queries of a sequence with L cached tokens sits at position
// L - n + i and attends to tokens 0 .. L - n + i: exactly a decode of length
// L - n + i + 1, with q turned by the rotary table at that position, rotated in step
// with H_blk (wispaper.ai blog, section 3) and the output rotated back when values
// are rotated.
//
// Work: one CTA = (KV head, sequence, block of 64 / G consecutive queries), 4 warps;
// a warp owns 16 (query, head) rows (16 / G queries x the G heads of the KV head) and
// walks every 16-token chunk up to its last query's position with its own ring of
// chunk stages and online-softmax state, so warps never wait on one another.  Blocks
// are numbered from each sequence's last query backwards, so the longest rows start
// first, and the query block is the grid's fastest index: the CTAs in flight at any time
// belong to few (sequence, KV head) pairs, whose codes then stay in L2 for all of them.
//   * q.K: D[16 rows x 8 tokens] += A[16 x 32 dims] B[32 dims x 8 tokens] on the int8
//     tensor path, with q' in 23-bit fixed point as three signed bytes per row (m-tile
//     0: rows 0..7 high | middle bytes, m-tile 1: rows 8..15, m-tile 2: the low bytes
//     of all 16) and B = the key codes as bytes; the int32 sums are exact.
//   * P.V: D[16 dims x 8 rows] += A[16 dims x 16 tokens] B[16 tokens x 8 rows]: A = the
//     centred V codes (shared with the decode tiles), B = p scale_v as fp16 high and low
//     parts for each of the two 8-row halves: four mmas per V tile.
//   * Causal mask: per row, tokens at or past its length are masked; chunks below every
//     row's length on valid pages take no per-token test.
//   * Long rows: the tensor cores' fp32 accumulation does not round to nearest, so over
//     thousands of chunks its bias grows (5.6e-3 of the output at 34k tokens).  Every 32
//     chunks the P.V accumulators are folded into a shared-memory copy with ordinary fp32
//     arithmetic (scaled to the current row maxima) and restarted from zero, which bounds
//     each accumulator's run as the decode's split length does.
#include <type_traits>

#include "kvq_mma.cuh"

namespace kvq {
namespace {

constexpr int kRows = 16;     // (query, head) rows per warp
constexpr int kFoldEvery = 32;  // chunks between folds of the P.V accumulators into shared memory
constexpr int kOWords = 2 * 8 * 4;  // P.V accumulators per thread
// dynamic shared memory: the ring, then per warp the folded accumulators [kOWords][32 lanes]
constexpr size_t kSmemBytes = sizeof(CtaRing) + size_t(kWarps) * kOWords * 32 * sizeof(float);
static_assert(sizeof(CtaRing) % 16 == 0, "the folded accumulators start 16-byte aligned");

struct ExtendParams {
    DecodeParams d;           // cache, q / seq_lens / page table / out, qscale, error word
    const int32_t* q_indptr;  // [batch + 1]
    int max_q_len;
};

// q fragments: 3 m-tiles x 4 k-steps x 4 registers x 32 lanes (words)
constexpr int kAWords = 3 * 4 * 4 * 32;
static_assert(kAWords * 4 <= kStages * kStageBytes, "q fragments are staged in the warp's ring");
static_assert(kRows * kHeadDim * 4 <= kStages * kStageBytes, "output rows are staged in the warp's ring");

// Output row staging [16 rows][128 dims] fp32: 16-byte chunk c of row r is stored at
// chunk c ^ ((r >> 1) & 3), so the eight 16-byte stores of one phase (two 16-dim
// segments x four rows) and the row-wise reads hit distinct bank groups.
__device__ __forceinline__ int ob_idx(int r, int d) { return r * kHeadDim + 4 * ((d >> 2) ^ ((r >> 1) & 3)) + (d & 3); }

template <int G, int CB>
__global__ void __launch_bounds__(kThreads, 3) extend_kernel(ExtendParams ep) {
    static_assert(kRows % G == 0, "a warp holds whole query groups");
    constexpr int QW = kRows / G;   // queries per warp
    constexpr int QB = kWarps * QW;  // queries per CTA
    extern __shared__ __align__(128) uint8_t dsm[];
    CtaRing& R = *reinterpret_cast<CtaRing*>(dsm);
    const DecodeParams& p = ep.d;
    const int z = blockIdx.x, h = blockIdx.y, s = blockIdx.z;  // z: query block, from the last
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, pq = lane & 3;

    const int q0 = __ldg(ep.q_indptr + s);
    int n = __ldg(ep.q_indptr + s + 1) - q0;
    if (z == 0 && h == 0 && tid == 0 && (n < 0 || n > ep.max_q_len)) flag_error(p.err, kErrOOB);
    n = max(n, 0);
    const int qhi = n - QB * z;  // this CTA's queries end here (exclusive)
    if (qhi <= 0) {
        grid_dep_wait();  // no grid here completes before the one it follows
        grid_dep_launch();
        return;
    }
    const int qw0 = qhi - QB + QW * warp;  // query of the warp's first row (may be < 0: no row)
    const int64_t L = __ldg(p.a.seq_lens + s);
    const int cap = min(p.a.pt_stride * p.g.page_size, p.a.max_seq_len);

    // ---- row r = lane (lanes 0..15): length = its decode length (position + 1), 0 when the
    // row has no cached tokens or no rotary-table row; -1 when there is no such query ----
    int rowlen = -1;
    if (lane < kRows) {
        const int qi = qw0 + lane / G;
        if (qi >= 0) {
            const int64_t Lr = L - n + qi + 1;
            const bool no_rope = p.g.rope && Lr > p.g.rope_positions;
            rowlen = (Lr <= 0 || no_rope) ? 0 : int(min(Lr, int64_t(cap)));
            if (Lr <= 0 || no_rope || Lr > cap) flag_error(p.err, kErrOOB);
        }
    }
    int t1 = max(rowlen, 0), tmin = lane < kRows ? max(rowlen, 0) : 0x7FFFFFFF;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        t1 = max(t1, __shfl_xor_sync(kFull, t1, o));
        tmin = min(tmin, __shfl_xor_sync(kFull, tmin, o));
    }

    // ---------------- q' of the 16 rows as 23-bit fixed point, A fragment order ----------------
    // k-step j, k-slot 4 pq + i (registers 0, 1) / 16 + 4 pq + i (registers 2, 3) stand for
    // dim 32 pq + 8 j + 2 i (+ 1): the low / high nibbles of key bytes 16 pq + 4 j + i.
    uint8_t* wbuf = &R.stage[warp][0][0];  // the warp's ring, free until the first copy
    uint32_t* As = reinterpret_cast<uint32_t*>(wbuf);
    for (int w = lane; w < kAWords; w += 32) As[w] = 0u;
    __syncwarp();
    float qsc_r = 0.0f, qsn_r = 0.0f;  // lane r: fixed-point step of row r, sum of its q_int
    for (int r = 0; r < kRows; ++r) {
        if (__shfl_sync(kFull, rowlen, r) <= 0) continue;  // no row or no tokens: A rows stay 0
        const int qi = qw0 + r / G;
        float x[4];
        load_q_rotated(p, int64_t(q0 + qi) * p.g.Hq + h * G + r % G, int(L - n + qi), lane, x);
        float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
        const float inv = amax > 0.0f ? float(kQFix) / amax : 0.0f;
        int qv[4], isum = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            qv[c] = min(max(__float2int_rn(x[c] * inv), -kQFix), kQFix);
            isum += qv[c];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(kFull, isum, o);
        if (lane == r) {
            qsc_r = amax / float(kQFix);
            qsn_r = float(isum);
        }
        const int mt = r >> 3, g = r & 7;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int d = 4 * lane + c;
            const int dp = d >> 5, j = (d >> 3) & 3, i = (d >> 1) & 3, odd = d & 1;
            int hi, mid, lo;
            q_digits(qv[c], hi, mid, lo);
            uint8_t* A8 = reinterpret_cast<uint8_t*>(As);
            A8[(((mt * 4 + j) * 4 + 2 * odd) * 32 + 4 * g + dp) * 4 + i] = uint8_t(hi);
            A8[(((mt * 4 + j) * 4 + 1 + 2 * odd) * 32 + 4 * g + dp) * 4 + i] = uint8_t(mid);
            A8[(((2 * 4 + j) * 4 + mt + 2 * odd) * 32 + 4 * g + dp) * 4 + i] = uint8_t(lo);
        }
    }
    __syncwarp();
    uint32_t A[3][4][4];
#pragma unroll
    for (int mt = 0; mt < 3; ++mt)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r) A[mt][j][r] = As[((mt * 4 + j) * 4 + r) * 32 + lane];
    __syncwarp();  // the ring is the copies' again
    // this thread's score rows: gq (half 0) and gq + 8 (half 1)
    const float qsc[2] = {__shfl_sync(kFull, qsc_r, gq), __shfl_sync(kFull, qsc_r, gq + 8)};
    const float qsn[2] = {__shfl_sync(kFull, qsn_r, gq), __shfl_sync(kFull, qsn_r, gq + 8)};
    const int len[2] = {__shfl_sync(kFull, rowlen, gq), __shfl_sync(kFull, rowlen, gq + 8)};

    ChunkStream<CB> cs;
    cs.r = &R;
    cs.pt = p.a.page_table + int64_t(s) * p.a.pt_stride;
    cs.t0 = 0;
    cs.t1 = t1;
    cs.nw = (t1 + kChunk - 1) / kChunk;
    cs.warp = warp;
    cs.lane = lane;
    cs.h = h;
    cs.first = 0;
    cs.step = 1;
    cs.fast = (p.g.page_size % kChunk) == 0;
    cs.pol = policy_evict_normal();  // every warp of the sequence's blocks reads these tokens
    cs.init(p);
    const int nw = cs.nw;
    // q only (never written by an append) so far; the cache after the previous grid
    grid_dep_wait();
    grid_dep_launch();
    for (int i = 0; i < kStages; ++i) {
        if (i < nw) cs.issue(p, i, i);
        cp_async_commit();
    }

    // ---------------- main loop over the warp's chunks ----------------
    float* fold = reinterpret_cast<float*>(dsm + sizeof(CtaRing)) + warp * kOWords * 32 + lane;  // [word][lane]
#pragma unroll
    for (int w = 0; w < kOWords; ++w) fold[w * 32] = 0.0f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f}, Z[2] = {0.0f, 0.0f};
    float mf[2] = {-INFINITY, -INFINITY};  // row maxima the folded accumulators are relative to
    float O[2][8][4];  // P.V accumulators [row half][dim tile]: dims x rows (2 pq, 2 pq + 1)
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int j = 0; j < 8; ++j) O[t][j][0] = O[t][j][1] = O[t][j][2] = O[t][j][3] = 0.0f;
    const int tokA = sigma(2 * pq), tokB = sigma(2 * pq + 1), tokK = sigma(gq);
    // fold = fold * 2^(mf - m) + O (row by row, ordinary fp32), O = 0, mf = m
    auto fold_acc = [&]() {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const float beta = (mf[t] == -INFINITY) ? 0.0f : fast_exp2(mf[t] - m[t]);
            const float b0 = __shfl_sync(kFull, beta, 8 * pq);      // row 8 t + 2 pq
            const float b1 = __shfl_sync(kFull, beta, 8 * pq + 4);  // row 8 t + 2 pq + 1
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float* f = fold + ((t * 8 + j) * 4 + c) * 32;
                    *f = fmaf(*f, (c & 1) ? b1 : b0, O[t][j][c]);
                    O[t][j][c] = 0.0f;
                }
            mf[t] = m[t];
        }
    };

    for (int i = 0; i < nw; ++i) {
        const int slot = i % kStages;
        cp_async_wait<kStages - 1>();  // chunk i's group (the stream keeps kStages groups)
        __syncwarp();                   // ... and every lane's copies of it
        const uint8_t* st = R.stage[warp][slot];
        const uint32_t vmask = R.mask[warp][slot];
        const int tb = i * kChunk;
        stage_szf<CB>(R, st, warp, lane, 1.0f, 1.0f);

        // ---- q_int . codes: column gq of n-tile tau is token 8 tau + tokK ----
        int X[2][4], Y[2][4], W[2][4];
        uint32_t kwv[2][4];
#pragma unroll
        for (int tau = 0; tau < 2; ++tau) {
            const uint4 kw = key_codes<CB>(st, 8 * tau + tokK, pq);
            kwv[tau][0] = kw.x;
            kwv[tau][1] = kw.y;
            kwv[tau][2] = kw.z;
            kwv[tau][3] = kw.w;
#pragma unroll
            for (int c = 0; c < 4; ++c) X[tau][c] = Y[tau][c] = W[tau][c] = 0;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int tau = 0; tau < 2; ++tau) {  // six independent accumulators between dependent mmas
                const uint32_t b0 = kwv[tau][j] & 0x0F0F0F0Fu, b1 = (kwv[tau][j] >> 4) & 0x0F0F0F0Fu;
                mma16832_s8u8(X[tau], A[0][j], b0, b1);
                mma16832_s8u8(Y[tau], A[1][j], b0, b1);
                mma16832_s8u8(W[tau], A[2][j], b0, b1);
            }
        // Scores, online softmax and weights; a chunk below every row's length and on valid
        // pages (FULL, the common case) takes no per-token test.
        uint32_t bh[2][2], bl[2][2];  // P.V B operands per row half: fp16 high / low parts
        auto softmax = [&](auto full_c) {
            constexpr bool FULL = decltype(full_c)::value;
            float sc[2][2][2];  // [row half][tau][column 2 pq + e]
#pragma unroll
            for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int lt = 8 * tau + (e ? tokB : tokA);
                    const float2 kz = R.szf[warp][0][lt];
                    const float c0 = q_dot(X[tau][e], X[tau][2 + e], W[tau][e]);
                    const float c1 = q_dot(Y[tau][e], Y[tau][2 + e], W[tau][2 + e]);
                    sc[0][tau][e] = qsc[0] * fmaf(kz.x, c0, kz.y * qsn[0]);
                    sc[1][tau][e] = qsc[1] * fmaf(kz.x, c1, kz.y * qsn[1]);
                    if (!FULL) {
                        const bool page_ok = ((vmask >> lt) & 1u) != 0;
                        if (!(page_ok && tb + lt < len[0])) sc[0][tau][e] = -INFINITY;
                        if (!(page_ok && tb + lt < len[1])) sc[1][tau][e] = -INFINITY;
                    }
                }
            // online softmax (log2 domain) per row; a row's 16 scores sit in one lane quad
            float mn[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                float cm = fmaxf(fmaxf(sc[t][0][0], sc[t][0][1]), fmaxf(sc[t][1][0], sc[t][1][1]));
                cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 1));
                cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 2));
                mn[t] = fmaxf(m[t], cm);
            }
            if (__any_sync(kFull, (mn[0] > m[0]) || (mn[1] > m[1]))) {
                float alpha[2];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    alpha[t] = (mn[t] > m[t]) ? fast_exp2(m[t] - mn[t]) : 1.0f;
                    l[t] *= alpha[t];
                    Z[t] *= alpha[t];
                    m[t] = mn[t];
                }
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const float a0 = __shfl_sync(kFull, alpha[t], 8 * pq);      // row 8 t + 2 pq
                    const float a1 = __shfl_sync(kFull, alpha[t], 8 * pq + 4);  // row 8 t + 2 pq + 1
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        O[t][j][0] *= a0;
                        O[t][j][1] *= a1;
                        O[t][j][2] *= a0;
                        O[t][j][3] *= a1;
                    }
                }
            }
            float pv[2][2][2];
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int lt = 8 * tau + (e ? tokB : tokA);
                        float pr;
                        float2 vz;
                        if (FULL) {
                            pr = fast_exp2(sc[t][tau][e] - m[t]);
                            vz = R.szf[warp][1][lt];
                        } else {
                            // masked tokens (past a row's end, skipped pages, stale slots) may hold
                            // any bits in their scale/zero word: never let them reach an operand,
                            // even times 0
                            const bool live = sc[t][tau][e] != -INFINITY;
                            pr = live ? fast_exp2(sc[t][tau][e] - m[t]) : 0.0f;
                            vz = live ? R.szf[warp][1][lt] : make_float2(0.0f, 0.0f);
                        }
                        l[t] += pr;
                        Z[t] = fmaf(pr, vz.y, Z[t]);
                        pv[t][tau][e] = pr * vz.x;
                    }
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int tau = 0; tau < 2; ++tau) {
                    bh[t][tau] = pack_half2(pv[t][tau][0], pv[t][tau][1]);
                    bl[t][tau] =
                        pack_half2(pv[t][tau][0] - half_lo(bh[t][tau]), pv[t][tau][1] - half_hi(bh[t][tau]));
                }
        };
        if ((tb + kChunk <= tmin) && (vmask == 0xFFFFu))
            softmax(std::true_type{});
        else
            softmax(std::false_type{});
        v_tiles<CB>(st, gq, tokA, tokB, [&](int jv, const uint32_t(&a)[4]) {
            mma16816(O[0][jv], a, bh[0][0], bh[0][1]);
            mma16816(O[1][jv], a, bh[1][0], bh[1][1]);
            mma16816(O[0][jv], a, bl[0][0], bl[0][1]);
            mma16816(O[1][jv], a, bl[1][0], bl[1][1]);
        });
        if ((i % kFoldEvery) == kFoldEvery - 1) fold_acc();
        __syncwarp();  // every lane is done with this slot
        if (i + kStages < nw) cs.issue(p, i + kStages, slot);
        cp_async_commit();
    }
    fold_acc();
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int c = 0; c < 4; ++c) O[t][j][c] = fold[((t * 8 + j) * 4 + c) * 32];

    // ---------------- normalise, undo the 2^-24 code scale, rotate back, store ----------------
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        l[t] += __shfl_xor_sync(kFull, l[t], 1);
        l[t] += __shfl_xor_sync(kFull, l[t], 2);
        Z[t] += __shfl_xor_sync(kFull, Z[t], 1);
        Z[t] += __shfl_xor_sync(kFull, Z[t], 2);
    }
    cp_async_wait<0>();
    __syncwarp();  // the ring is free: stage the 16 output rows there
    float* ob = reinterpret_cast<float*>(wbuf);
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = 8 * t + 2 * pq + e;
            const float lr = __shfl_sync(kFull, l[t], 4 * (2 * pq + e));
            const float zr = __shfl_sync(kFull, Z[t], 4 * (2 * pq + e));
            const float inv = lr > 0.0f ? 1.0f / lr : 0.0f;
            float v[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                v[2 * j] = fmaf(O[t][j][e], kTwo24, zr) * inv;
                v[2 * j + 1] = fmaf(O[t][j][2 + e], kTwo20, zr) * inv;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<float4*>(ob + ob_idx(r, 16 * gq + 4 * c)) =
                    make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
    __syncwarp();
    const bool rot = p.g.mode == 2 && p.g.rotate_v;
    for (int r = 0; r < kRows; ++r) {
        const int qi = qw0 + r / G;
        if (qi < 0) continue;
        const float4 o4 = *reinterpret_cast<const float4*>(ob + ob_idx(r, 4 * lane));
        float x[4] = {o4.x, o4.y, o4.z, o4.w};
        if (rot) {
            fwht_lanes(x, lane, p.g.bdr_block);
            const float sc = rsqrtf(float(p.g.bdr_block));
#pragma unroll
            for (int c = 0; c < 4; ++c) x[c] *= sc;
        }
        const int64_t o = (int64_t(q0 + qi) * p.g.Hq + h * G + r % G) * kHeadDim + 4 * lane;
        if (p.a.out_fp32) {
            *reinterpret_cast<float4*>(static_cast<float*>(p.a.out) + o) = make_float4(x[0], x[1], x[2], x[3]);
        } else {
            const __nv_bfloat162 b01 = __floats2bfloat162_rn(x[0], x[1]);
            const __nv_bfloat162 b23 = __floats2bfloat162_rn(x[2], x[3]);
            uint2 u;
            u.x = *reinterpret_cast<const uint32_t*>(&b01);
            u.y = *reinterpret_cast<const uint32_t*>(&b23);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.a.out) + o) = u;
        }
    }
}

template <int G, int CB>
cudaError_t launch_k(const ExtendParams& ep, dim3 grid, cudaStream_t s) {
    constexpr auto kern = extend_kernel<G, CB>;
    const cudaError_t e = ensure_smem_opt_in<kern>(kSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_overlapped(kern, grid, dim3(kThreads), kSmemBytes, s, ep);
}

template <int G>
cudaError_t launch_group(const ExtendParams& ep, dim3 grid, cudaStream_t s) {
    return launch_k<G, 2>(ep, grid, s);  // only 2-bit codes reach this kernel
}

}  // namespace

int extend_queries_per_cta(const CacheGeom& g) { return kWarps * kRows / (g.Hq / g.H); }

cudaError_t launch_extend(const CacheGeom& g, const ExtendArgs& a, int* err_word, cudaStream_t s) {
    if (a.batch == 0 || a.max_q_len == 0) return cudaSuccess;
    ExtendParams ep;
    ep.d.g = g;
    ep.d.a = DecodeArgs{a.q, a.seq_lens, a.page_table, a.pt_stride, a.batch, a.max_seq_len, a.out, a.out_fp32,
                        nullptr, 0};
    ep.d.item_tokens = 0;
    ep.d.max_splits = 0;
    ep.d.qscale = float(1.0 / sqrt(double(kHeadDim))) * kLog2e;
    ep.d.ps_shift = -1;
    for (int sh = 0; sh < 11; ++sh)
        if ((1 << sh) == g.page_size) ep.d.ps_shift = sh;
    ep.d.ws_o = nullptr;
    ep.d.ws_ml = nullptr;
    ep.d.err = err_word;
    ep.q_indptr = a.q_indptr;
    ep.max_q_len = a.max_q_len;
    // 4-bit codes: the tcgen05 kernel (kvq_extend_tc.cu); 2-bit codes: the mma.sync kernel below
    if (g.code_bits == 4) return launch_extend_tc(ep.d, a.q_indptr, a.max_q_len, s);
    const int qb = extend_queries_per_cta(g);
    const dim3 grid((a.max_q_len + qb - 1) / qb, g.H, a.batch);
    switch (g.Hq / g.H) {
        case 1: return launch_group<1>(ep, grid, s);
        case 2: return launch_group<2>(ep, grid, s);
        case 4: return launch_group<4>(ep, grid, s);
        case 8: return launch_group<8>(ep, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
