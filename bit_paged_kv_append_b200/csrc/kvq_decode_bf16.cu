// kvq_decode_bf16.cu -- paged GQA decode attention over BF16 pages (the unquantised cache
// the pages compare INT4 against), built the same way as the INT4 split kernels: one CTA
// per (split, KV head, sequence), 4 warps walking 16-token chunks round robin, each warp
// with its own ring of cp.async-filled shared-memory stages and its own online softmax, the
// contractions on the tensor cores, the warps merged in shared memory and the split's
// partial rows stored for the log-sum-exp merge kernel.
//
// A chunk is 16 tokens of one (page, KV head) block: 4 KiB of K rows and 4 KiB of V rows
// (bf16, 256 bytes a token).  Every lane copies 16-byte units of both with cp.async; unit c
// of token row t lands at 16-byte slot c ^ (t & 7) of the row, so the eight rows one
// ldmatrix phase reads sit in eight different bank groups.
//
//   q.K   S[16 rows x 8 tokens] += A[16 rows x 16 dims] B[16 dims x 8 tokens]
//         (mma.m16n8k16, bf16 operands, fp32 accumulation).  Rows 0..7 hold the high bf16
//         part of the query of heads 0..G-1, rows 8..15 the low part (q - high, rounded to
//         bf16): with the rotary embedding the turned query is fp32, and the two parts carry
//         it to ~16 bits; without it the query is bf16 already and its low part is zero.  B
//         = the K rows, loaded with ldmatrix (no transpose).  16 mmas a chunk.
//   P.V   O[16 rows x 8 dims] += A[16 rows x 16 tokens] B[16 tokens x 8 dims]: the score
//         accumulator of q.K is already the A layout of P.V (flash-attention register reuse).
//         Rows 0..7 carry the high bf16 part of p, rows 8..15 the low part, so a head's output
//         is the sum of its two rows and p keeps ~16 bits.  B = the V rows, loaded with
//         ldmatrix.trans.  16 mmas a chunk.
//
// Scores are kept in the log2 domain (scaled by log2(e)/sqrt(D) after the mma).  The warps
// merge into the same partial layout as the INT4 kernels, and the same merge kernel
// finishes the call.
#include "kvq_mma.cuh"

namespace kvq {
namespace {

constexpr int kBfStages = 3;
constexpr int kBfRow = 256;                // bytes of one bf16 row (128 dims)
constexpr int kBfRows = kChunk * kBfRow;   // 4 KiB: the K (or V) rows of one chunk
constexpr int kBfStage = 2 * kBfRows;      // K rows | V rows

struct BfRing {
    uint8_t stage[kWarps][kBfStages][kBfStage];
    uint32_t mask[kWarps][kBfStages];  // tokens of the staged chunk on valid pages (bit per token)
};
constexpr size_t kBfSmem = sizeof(BfRing);
// the merge reuses the ring: mo [warp][G][kMoStride] floats, then max and weight sum [warp][G]
constexpr int kMoStride = kHeadDim + 4;
static_assert(kWarps * kMaxGroup * (kMoStride + 2) * 4 <= int(sizeof(BfRing)), "merge scratch fits the ring");

// Byte offset of 16-byte unit c of token row t in a stage half.
__device__ __forceinline__ uint32_t bf_swz(int t, int c) { return uint32_t(t * kBfRow + ((c ^ (t & 7)) << 4)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// fp32 pair -> bf16x2 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// One warp's 16-token chunks of bf16 rows: chunk iw starts at token t0 + (warp + 4 iw) 16.
struct BfStream {
    BfRing* r;
    const int32_t* pt;
    int t0, t1, nw, warp, lane, h;
    bool fast;  // page size a multiple of 16: a chunk is 16 consecutive slots of one page
    uint64_t pol;
    int win;
    uint32_t myrow;
    uint32_t base;  // shared address of this warp's stage 0

    static constexpr uint32_t kNoRow = 0xFFFFFFFFu;

    // Pool row (page H + h) ps + slot of chunk iw's first token (window of 32 chunks, one
    // page-table lookup per lane; kNoRow for a bad page, flagged when its window is loaded).
    __device__ __forceinline__ uint32_t row_of(const DecodeParams& p, int iw) {
        if ((iw >> 5) != win) {
            win = iw >> 5;
            const int ci = 32 * win + lane;
            myrow = kNoRow;
            if (ci < nw) {
                const int tb = t0 + (warp + kWarps * ci) * kChunk;
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

    // Copies of chunk iw into ring slot `slot` by all 32 lanes; the caller commits the group.
    __device__ __forceinline__ void issue(const DecodeParams& p, int iw, int slot) {
        const uint8_t* kpool = static_cast<const uint8_t*>(p.g.k_pool);
        const uint8_t* vpool = static_cast<const uint8_t*>(p.g.v_pool);
        const uint32_t d = base + uint32_t(slot) * kBfStage;
        if (fast) {
            // 16 consecutive rows: 4 KiB of K and 4 KiB of V, 256 units of 16 bytes each;
            // lane L copies units L + 32 i (token (L + 32 i) / 16)
            const uint32_t row = row_of(p, iw);
            const bool ok = row != kNoRow;
            if (ok) {
                const uint8_t* ks = kpool + size_t(row) * kBfRow;
                const uint8_t* vs = vpool + size_t(row) * kBfRow;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int u = lane + 32 * i;
                    const uint32_t off = bf_swz(u >> 4, u & 15);
                    cp_async16_s(d + off, ks + 16 * u, pol);
                    cp_async16_s(d + kBfRows + off, vs + 16 * u, pol);
                }
            }
            r->mask[warp][slot] = ok ? 0xFFFFu : 0u;  // the same value from every lane
        } else {
            // gather: lane L copies half L & 1 (8 units) of token tb + (L >> 1)'s K and V rows
            const int tb = t0 + (warp + kWarps * iw) * kChunk;
            const int i = lane >> 1, hf = lane & 1;
            const int t = tb + i;
            bool ok = false;
            if (t < t1) {
                const int page = __ldg(pt + page_of_pos(p, t));
                ok = page >= 0 && page < p.g.num_pages;
                if (ok) {
                    const int64_t row = (int64_t(page) * p.g.H + h) * p.g.page_size + slot_of_pos(p, t);
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        const int c = 8 * hf + c8;
                        const uint32_t off = bf_swz(i, c);
                        cp_async16_s(d + off, kpool + row * kBfRow + 16 * c, pol);
                        cp_async16_s(d + kBfRows + off, vpool + row * kBfRow + 16 * c, pol);
                    }
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

template <int G>
__global__ void __launch_bounds__(kThreads, 2) decode_bf16_kernel(DecodeParams p) {
    extern __shared__ __align__(128) uint8_t dsm[];
    BfRing& R = *reinterpret_cast<BfRing*>(dsm);
    const int k = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, pq = lane & 3;
    const int L = decode_len(p, s);
    if (k == 0 && h == 0 && tid == 0 && L != __ldg(p.a.seq_lens + s)) flag_error(p.err, kErrOOB);
    const int t0 = k * p.item_tokens;
    if (t0 >= L) {  // past the end of the sequence: no partial (the merge reads only real splits)
        grid_dep_wait();  // still: no grid here completes before the one it follows
        grid_dep_launch();
        return;
    }
    const int t1 = min(L, t0 + p.item_tokens);
    const int nchunks = (t1 - t0 + kChunk - 1) / kChunk;
    const int nw = nchunks > warp ? (nchunks - warp + kWarps - 1) / kWarps : 0;  // this warp's chunks

    // ---------------- query A fragments: head gq's dims 16 j + 2 pq + {0, 1, 8, 9} ----------------
    // rows 0..7: high bf16 part, rows 8..15: low part; heads >= G stay zero
    const bool gval = gq < G;
    uint32_t A[8][4];
    {
        float x[8][4];  // [k-step j][e]: dims 16 j + 2 pq + (0, 1, 8, 9)
        if (gval) {
            const uint32_t* qw = reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.a.q) +
                                                                   (int64_t(s) * p.g.Hq + h * G + gq) * kHeadDim);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t w0 = __ldg(qw + 8 * j + pq), w1 = __ldg(qw + 8 * j + 4 + pq);
                x[j][0] = bf_lo(w0);
                x[j][1] = bf_hi(w0);
                x[j][2] = bf_lo(w1);
                x[j][3] = bf_hi(w1);
            }
            if (p.g.rope) {  // turn at position seq_len - 1: pairs (i, i + 64) = k-steps (j, j + 4)
                const float* cs = p.g.rope + int64_t(__ldg(p.a.seq_lens + s) - 1) * kHeadDim;
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = 16 * j + 2 * pq + (e & 1) + 8 * (e >> 1);  // pair index
                        const float2 c = __ldg(reinterpret_cast<const float2*>(cs) + i);
                        const float a = x[j][e], b = x[j + 4][e];
                        x[j][e] = fmaf(a, c.x, -b * c.y);
                        x[j + 4][e] = fmaf(b, c.x, a * c.y);
                    }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j][0] = x[j][1] = x[j][2] = x[j][3] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t h01 = pack_bf162(x[j][0], x[j][1]), h89 = pack_bf162(x[j][2], x[j][3]);
            A[j][0] = h01;
            A[j][2] = h89;
            A[j][1] = pack_bf162(x[j][0] - bf_lo(h01), x[j][1] - bf_hi(h01));
            A[j][3] = pack_bf162(x[j][2] - bf_lo(h89), x[j][3] - bf_hi(h89));
        }
    }

    BfStream cs;
    cs.r = &R;
    cs.pt = p.a.page_table + int64_t(s) * p.a.pt_stride;
    cs.t0 = t0;
    cs.t1 = t1;
    cs.nw = nw;
    cs.warp = warp;
    cs.lane = lane;
    cs.h = h;
    cs.fast = (p.g.page_size % kChunk) == 0;
    cs.pol = policy_evict_first();
    cs.win = -1;
    cs.myrow = BfStream::kNoRow;
    cs.base = smem_u32(R.stage[warp][0]);
    // q only (never written by an append) so far; the cache after the previous grid
    grid_dep_wait();
    grid_dep_launch();
#pragma unroll
    for (int i = 0; i < kBfStages; ++i) {
        if (i < nw) cs.issue(p, i, i);
        cp_async_commit();
    }

    // ldmatrix row addresses (lane L names row L & 7 of matrix L >> 3)
    const int mi = lane >> 3, mr = lane & 7;
    // q.K: matrices (tokens 8 (mi >> 1) .. , dims 16 j + 8 (mi & 1) ..): unit 2 j + (mi & 1)
    const int k_tok = 8 * (mi >> 1) + mr, k_half = mi & 1;
    // P.V: matrices (tokens 8 (mi & 1) .., dims 8 (n + (mi >> 1)) ..): unit n + (mi >> 1)
    const int v_tok = 8 * (mi & 1) + mr, v_add = mi >> 1;

    float m = gval ? -INFINITY : 0.0f, l = 0.0f;
    float O[16][4];  // P.V accumulators [dim group n]: rows (gq: high p, gq + 8: low p) x dims 8 n + 2 pq + {0, 1}
#pragma unroll
    for (int n = 0; n < 16; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.0f;

    for (int i = 0; i < nw; ++i) {
        const int slot = i % kBfStages;
        cp_async_wait<kBfStages - 1>();  // chunk i's group (the stream keeps kBfStages groups)
        __syncwarp();                     // ... and every lane's copies of it
        const uint32_t st = cs.base + uint32_t(slot) * kBfStage;
        const uint32_t vmask = R.mask[warp][slot];
        const int tb = t0 + (warp + kWarps * i) * kChunk;

        // ---- S = q K^T: n-tile 0 = tokens 0..7, n-tile 1 = tokens 8..15 ----
        float S[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t b00, b01, b10, b11;
            ldsm_x4(st + bf_swz(k_tok, 2 * j + k_half), b00, b01, b10, b11);
            mma_bf16(S[0], A[j], b00, b01);
            mma_bf16(S[1], A[j], b10, b11);
        }
        // ---- scores of head gq, tokens 8 t + 2 pq + e (log2 domain), masked ----
        const bool full = (tb + kChunk <= t1) && (vmask == 0xFFFFu);
        if (!full) {
            // rows of masked tokens (past the end, skipped pages) hold stale bits, maybe NaN or
            // inf: zero their V rows so that p = 0 times them stays 0 in the P.V mma
#pragma unroll
            for (int u8 = 0; u8 < 8; ++u8) {
                const int u = lane + 32 * u8, t = u >> 4;
                if (!((tb + t < t1) && ((vmask >> t) & 1u)))
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(st + kBfRows + bf_swz(t, u & 15)),
                                 "r"(0u)
                                 : "memory");
            }
            __syncwarp();
        }
        float sc[2][2];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int lt = 8 * t + 2 * pq + e;
                const bool ok = gval && (full || ((tb + lt < t1) && ((vmask >> lt) & 1u)));
                sc[t][e] = ok ? (S[t][e] + S[t][2 + e]) * p.qscale : -INFINITY;
            }
        // ---- online softmax for head gq: its 16 tokens sit in lanes 4 gq .. 4 gq + 3 ----
        float cm = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 1));
        cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 2));
        const float mn = fmaxf(m, cm);
        if (__any_sync(kFull, mn > m)) {
            const float alpha = (mn > m) ? fast_exp2(m - mn) : 1.0f;
            l *= alpha;
            m = mn;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                O[n][0] *= alpha;
                O[n][1] *= alpha;
                O[n][2] *= alpha;
                O[n][3] *= alpha;
            }
        }
        float pr[2][2];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                // masked scores give 0 (also while m is still -inf: no exp2 of -inf - -inf)
                pr[t][e] = (sc[t][e] == -INFINITY) ? 0.0f : fast_exp2(sc[t][e] - m);
                l += pr[t][e];
            }
        uint32_t Ap[4];
        Ap[0] = pack_bf162(pr[0][0], pr[0][1]);
        Ap[2] = pack_bf162(pr[1][0], pr[1][1]);
        Ap[1] = pack_bf162(pr[0][0] - bf_lo(Ap[0]), pr[0][1] - bf_hi(Ap[0]));
        Ap[3] = pack_bf162(pr[1][0] - bf_lo(Ap[2]), pr[1][1] - bf_hi(Ap[2]));
        // ---- O += P V: two 8-dim groups per ldmatrix.trans ----
#pragma unroll
        for (int n = 0; n < 16; n += 2) {
            uint32_t b00, b01, b10, b11;
            ldsm_x4_t(st + kBfRows + bf_swz(v_tok, n + v_add), b00, b01, b10, b11);
            mma_bf16(O[n], Ap, b00, b01);
            mma_bf16(O[n + 1], Ap, b10, b11);
        }
        __syncwarp();  // every lane is done with this slot
        if (i + kBfStages < nw) cs.issue(p, i + kBfStages, slot);
        cp_async_commit();
    }
    cp_async_wait<0>();

    // ---------------- per-head totals, merge the warps, store the split's partial rows ----------------
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
    __syncthreads();  // every ring is drained; reuse it for the merge
    float* mo = reinterpret_cast<float*>(dsm);        // [warp][G][kMoStride]
    float* mm = mo + kWarps * G * kMoStride;          // [warp][G]
    float* ml = mm + kWarps * G;                      // [warp][G]
    if (gval) {
        float* row = mo + (warp * G + gq) * kMoStride;
#pragma unroll
        for (int n = 0; n < 16; ++n)
            *reinterpret_cast<float2*>(row + 8 * n + 2 * pq) = make_float2(O[n][0] + O[n][2], O[n][1] + O[n][3]);
        if (pq == 0) {
            mm[warp * G + gq] = m;
            ml[warp * G + gq] = l;
        }
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
            acc += f * mo[(w * G + g) * kMoStride + tid];
            lt += f * ml[w * G + g];
        }
        const int64_t r = partial_row(p, s, k, h * G + g);
        p.ws_o[r * kHeadDim + tid] = acc;
        if (tid == 0) p.ws_ml[r] = make_float2(M, lt);
    }
}

template <int G>
cudaError_t launch_g(const DecodeParams& p, cudaStream_t s) {
    constexpr auto kern = decode_bf16_kernel<G>;
    const cudaError_t e = ensure_smem_opt_in<kern>(kBfSmem);
    if (e != cudaSuccess) return e;
    return launch_overlapped(kern, dim3(p.max_splits, p.g.H, p.a.batch), dim3(kThreads), kBfSmem, s, p);
}

}  // namespace

cudaError_t launch_decode_bf16(const DecodeParams& p, cudaStream_t s) {
    switch (p.g.Hq / p.g.H) {
        case 1: return launch_g<1>(p, s);
        case 2: return launch_g<2>(p, s);
        case 4: return launch_g<4>(p, s);
        case 8: return launch_g<8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
