// kvq_extend_tc.cu -- extend (chunked-prefill) attention over the paged INT4 (or 2-bit) cache
// on the 5th-generation tensor cores (tcgen05.mma, operands and accumulators in tensor memory).
//
// SAW-INT4's abstract keeps fused attention over the paged quantised layout as a serving
// constraint; chunked prefill in mixed serving reads the cache this way.  Query i of the n
// new queries of a sequence with L cached tokens sits at position L - n + i and attends to
// tokens 0 .. L - n + i: exactly a decode of length L - n + i + 1, with q turned by the
// rotary table at that position, rotated in step with H_blk (wispaper.ai blog, section 3)
// and the output rotated back when values are rotated.  Dequantisation stays factored:
//   q'.(scale c + zero) = scale (q'.c) + zero sum(q')
//   sum_t p_t (scale_t c_t + zero_t) = sum_t (p_t scale_t)(c_t - 8) + sum_t p_t (zero_t + 8 scale_t)
// so both contractions run on raw 4-bit codes.
//
// One CTA = 128 (query, head) rows of one KV head of one sequence (128 / G consecutive
// queries x the G heads), one CTA per SM (207 KB of shared memory, all 512 TMEM columns),
// three warp roles working on blocks of 128 key tokens:
//   * loaders (warps 8-11, thread = token): gather a block's key and value code rows through
//     the page table and write them as fp16 operand tiles: key codes as the exact
//     subnormals c 2^-24 (B of q.K, K-major), value codes centred, (c - 8) 2^-24 for 4-bit
//     codes and (c - 2) 2^-24 for 2-bit ones (B of P.V, N-major), with the tokens' scales and
//     zeros.  2-bit rows (32 bytes) are first spread to the 4-bit nibble layout.  Two stages; the key tile is released
//     when its q.K is done, the value tile when its P.V is done;
//   * one MMA thread (warp 12): S_j[128 x 128] = q_hi K_j^T + q_lo K_j^T (16 MMAs M128 N128
//     K16, kind::f16, q read from TMEM, the key tile from shared memory) into one of two TMEM
//     score buffers; then, once the softmax has written P_{j-1}, O_t += P_{j-1} V_{j-1} with P
//     read from TMEM (16 MMAs).  q' = rope(q) H_blk log2(e)/sqrt(D) is scaled per row by a
//     power of two to ~2^14 and split into fp16 high and low parts (~22 significant bits);
//   * softmax (warps 0-7; row r = TMEM lane r is shared by warps r / 32 and r / 32 + 4, each
//     thread taking one half of the block's tokens): reads its half row of S_j, forms the
//     scores, runs the online softmax with a lazily moved reference max (p = 2^(s - m_ref)
//     may reach 2^8 before the reference moves; the two halves of a row exchange their block
//     maxima through shared memory) and writes P = p scale_v 2^-k (k a per-block power of two
//     that keeps P below 2^15) as fp16 high and low parts over S_j in TMEM.
// The softmax of block j overlaps q.K of block j + 1 and P.V of block j - 1.  The tensor
// cores' fp32 accumulation does not round to nearest, and over thousands of tokens its bias
// would grow: O_t runs 4 blocks (512 tokens), then the softmax folds it into an fp32 copy O_f
// in shared memory with ordinary adds and the next P.V restarts O_t; a row whose reference
// moves rescales its part of O_t in place and of O_f.  Both operands of q.K in shared memory would take
// ~120 B per clock, the whole shared-memory port, while the softmax and the loaders need it
// too; with q in tensor memory q.K reads only the key tiles.
//
// Every mbarrier wait is bounded (kWaitLimitNs, and it gives up early once another role has
// given up); on expiry the CTA flags KV_ERR_TIMEOUT, each role leaves its loop, the MMA
// thread waits (bounded) for every MMA it issued, and the tensor memory is freed.  No
// hardware barrier is entered by only part of its threads.
#include "kvq_mma.cuh"

namespace kvq {
namespace {

constexpr int kXRows = 128;   // (query, head) rows per CTA = TMEM lanes
constexpr int kXBlk = 128;    // key tokens per block = loader threads
constexpr int kXSoftWarps = 8, kXLoadWarps = 4;
constexpr int kXSoftThreads = 32 * kXSoftWarps;  // two per row
constexpr int kXMmaWarp = kXSoftWarps + kXLoadWarps;
constexpr int kXThreads = 32 * (kXMmaWarp + 4);  // the MMA warp's warpgroup: the issuer + 3 idle warps
constexpr int kXCols = 512;                  // TMEM columns: S_0 | S_1 | O_t | q' (high, low)
constexpr uint32_t kColS = 0, kColOt = 256, kColQ = 384;
constexpr int kFoldEvery = 4;                // blocks accumulated in O_t between folds (512 tokens)
constexpr float kTau = 8.0f;                 // a row's reference moves once a score passes it by this (log2)
constexpr int kTile = kXBlk * kHeadDim * 2;  // one fp16 [128][128] operand tile, 32 KB

// Shared-memory operand tiles, no swizzle, "core matrices" of 8 rows x 16 bytes (128
// contiguous bytes): element (row r, column c) of a [128][128] fp16 tile sits at
// ((r / 8) 16 + c / 8) 128 + (r % 8) 16 + (c % 8) 2.  Read K-major (rows = M or N, columns
// = K: q, keys) the 8-row groups are 2048 B apart and the 8-column chunks 128 B; read
// N-major (rows = K, columns = N: values) the 8-K groups are 2048 B apart and the 8-N
// groups 128 B.
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
    return uint32_t(((r >> 3) * 16 + (c >> 3)) * 128 + (r & 7) * 16 + (c & 7) * 2);
}

struct XSmem {
    float4 of[kXRows][32];      // O_f: per row 128 fp32 columns; float4 k of row r sits at k ^ (r % 8)
    uint8_t k[2][kTile];        // per stage: key codes, tokens x dims
    uint8_t v[2][kTile];        // per stage: centred value codes, tokens x dims
    float2 ksz[2][kXBlk];       // per stage and token: key (scale, zero)
    float2 vsz[2][kXBlk];       // value (scale, zero + 8 scale)
    uint32_t vmask[2][4];       // tokens on valid pages, one word per loader warp
    float vmax[2][4];           // largest value scale, per loader warp
    float hm[2][2][kXRows];     // per block parity, half and row: the half row's block max
    float2 qx[kXRows];          // per row: (qexp, zq) of its q'
    float2 lz[2][kXRows];       // per half and row: (l, Z) after the last block
    uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];  // loaders <-> MMA, per stage
    uint64_t s_full[2], p_full[2];                          // MMA <-> softmax, per score buffer
    uint64_t pv_done;           // every P.V
    uint64_t fin;               // the MMA thread's last commit
    uint32_t tmem;
    int tmax, tmin;
    int abort;                  // a role gave up waiting
};
constexpr size_t kXSmem = sizeof(XSmem) + 1024;  // + alignment slack (tiles start 1024-aligned)

// Shared-memory matrix descriptor: no swizzle, Blackwell version bit, byte offsets >> 4.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return uint64_t((saddr >> 4) & 0x3FFF) | (uint64_t((lbo >> 4) & 0x3FFF) << 16) |
           (uint64_t((sbo >> 4) & 0x3FFF) << 32) | (uint64_t(1) << 46);
}
// Instruction descriptor of kind::f16: fp16 A and B, fp32 D, A K-major, B K- or N-major.
__host__ __device__ constexpr uint32_t idesc_f16(int n, int m, int b_nmajor) {
    return (1u << 4) | (uint32_t(b_nmajor) << 16) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}
constexpr uint32_t kIdQK = idesc_f16(kXBlk, kXRows, 0);     // S[128 x 128] = A[128 x 16] B[128 x 16]^T
constexpr uint32_t kIdPV = idesc_f16(kHeadDim, kXRows, 1);  // O[128 x 128] = A[128 x 16] B[16 x 128]

// A from tensor memory: lane = row, column c holds the fp16 pair (K index 2c, 2c + 1)
__device__ __forceinline__ void mma_ts(uint32_t dcol, uint32_t acol, uint64_t db, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(dcol),
        "r"(acol), "l"(db), "r"(id), "r"(acc), "r"(0u)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive TMEM columns of this warp's 32 lanes (no wait)
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(addr));
}
// 16 consecutive TMEM columns of this warp's 32 lanes (no wait)
__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(addr));
}
__device__ __forceinline__ void tmem_st16(uint32_t addr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::
            "r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// Register split (per thread): the launch gives 128 to each of the 16 warps (four per
// scheduler).  The loader warpgroup lowers its share to 104 and the MMA warpgroup (the
// issuing warp and three idle ones, there so that the group can give registers back) to
// 40; the two softmax warpgroups then raise theirs to 184.  8 x 32 x 184 + 4 x 32 x 104 +
// 4 x 32 x 40 = 65536 = 512 x 128, the launch's total, so the raise never waits for
// registers that do not exist (and no role spills).
constexpr int kXRegsSoft = 184, kXRegsLoad = 104, kXRegsMma = 40, kXRegsLaunch = 128;
static_assert(kXSoftThreads * kXRegsSoft + 32 * kXLoadWarps * kXRegsLoad + 128 * kXRegsMma <=
                  kXThreads * kXRegsLaunch,
              "register split exceeds the launch's registers");

// The two softmax warps that share TMEM lanes 32 q .. 32 q + 31 (warps q and q + 4, the two halves
// of the same rows) meet on named barrier 1 + q; both always take it the same number of times.
__device__ __forceinline__ void pair_bar(int warp) {
    asm volatile("barrier.sync %0, 64;" ::"r"(1 + (warp & 3)) : "memory");
}
// ... and the OR of pred over those 64 threads
__device__ __forceinline__ bool pair_any(int warp, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %2, 0;\n\t"
        "barrier.cta.red.or.pred q, %1, 64, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(1 + (warp & 3)), "r"(uint32_t(pred))
        : "memory");
    return r != 0;
}

// CTA-wide barrier 0 in its non-aligned form: each role reaches it from its own code.
__device__ __forceinline__ void cta_bar() { asm volatile("barrier.sync 0;" ::: "memory"); }

// Bounded wait that also gives up once another role has given up (abort set); on its own
// expiry it sets abort and flags KV_ERR_TIMEOUT.
__device__ __forceinline__ bool xwait(uint64_t* bar, uint32_t parity, volatile int* abort, int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            flag_error(err, kErrTimeout);
            return false;
        }
    }
}

// 2^k for an integer k in [-126, 127], exactly
__device__ __forceinline__ float pow2i(int k) { return __int_as_float((k + 127) << 23); }

// fp32 -> fp16 bits (round to nearest even)
__device__ __forceinline__ uint32_t h_bits(float x) { return __half_as_ushort(__float2half_rn(x)); }

// Four codes of one input word w (bytes b0..b3, two codes each, even dim in the low nibble)
// as fp16 pairs: out[i] = (lo nibble of b_i, hi nibble of b_i) as the subnormals c 2^-24,
// centred by `centre` (0 or fp16x2 (-8 2^-24, -8 2^-24), an exact add).
__device__ __forceinline__ void codes_to_f16(uint32_t w, uint32_t centre, uint32_t (&out)[4]) {
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    // PRMT puts byte i of lo in byte 0 and byte i of hi in byte 2; the AND clears bytes 1 and 3
    out[0] = prmt(lo, hi, 0x0400u) & 0x00FF00FFu;
    out[1] = prmt(lo, hi, 0x0501u) & 0x00FF00FFu;
    out[2] = prmt(lo, hi, 0x0602u) & 0x00FF00FFu;
    out[3] = prmt(lo, hi, 0x0703u) & 0x00FF00FFu;
    if (centre) {
#pragma unroll
        for (int i = 0; i < 4; ++i) out[i] = hadd2u(out[i], centre);
    }
}

template <int G, int CB>
__global__ void __maxnreg__(kXRegsLaunch) extend_tc_kernel(const __grid_constant__ DecodeParams p,
                                                                 const int32_t* __restrict__ q_indptr, int max_q_len) {
    constexpr int QB = kXRows / G;  // queries per CTA
    // value codes are centred at the middle of their range: c - 8 (4-bit) or c - 2 (2-bit)
    constexpr float kCentre = CB == 4 ? 8.0f : 2.0f;
    constexpr uint32_t kCentreF16 = CB == 4 ? kMinus8 : 0x80028002u;  // fp16x2 (-centre 2^-24, -centre 2^-24)
    constexpr uint32_t kCentreNib = CB == 4 ? 0x88888888u : 0x22222222u;  // every nibble at the centre
    extern __shared__ uint8_t dsm_raw[];
    XSmem& sm = *reinterpret_cast<XSmem*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    volatile int* abort = &sm.abort;
    const int z = blockIdx.x, h = blockIdx.y, s = blockIdx.z;  // z: query block, from the last
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int q0 = __ldg(q_indptr + s);
    int n = __ldg(q_indptr + s + 1) - q0;
    if (z == 0 && h == 0 && tid == 0 && (n < 0 || n > max_q_len)) flag_error(p.err, kErrOOB);
    n = max(n, 0);
    const int qhi = n - QB * z;  // this CTA's queries end here (exclusive)
    if (qhi <= 0) {
        grid_dep_wait();  // no grid here completes before the one it follows
        grid_dep_launch();
        return;
    }
    const int64_t L = __ldg(p.a.seq_lens + s);
    const int cap = min(p.a.pt_stride * p.g.page_size, p.a.max_seq_len);
    const bool soft = warp < kXSoftWarps;
    // The roles part here, each under its own register limit; the three CTA barriers (set-up done,
    // q tiles written, teardown) are reached by every role from its own code.
    if (soft) {
        // =============================== softmax ===============================
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kXRegsSoft));
        // ---- row r: query qi = qhi - QB + r / G, head g = r % G; its length = position + 1.  Half hf
        // of the row takes tokens 64 hf .. 64 hf + 63 of every block.  Only the last max_q_len
        // queries of a sequence are computed (the grid may cover more). ----
        const int row = tid & (kXRows - 1), hf = tid >> 7;
        const int qi0 = qhi - QB + row / G, g = row % G;
        const int qi = qi0 >= n - max_q_len ? qi0 : -1;
        int rowlen = -1;  // -1: no such query
        if (qi >= 0) {
            const int64_t Lr = L - n + qi + 1;
            const bool no_rope = p.g.rope && Lr > p.g.rope_positions;
            rowlen = (Lr <= 0 || no_rope) ? 0 : int(min(Lr, int64_t(cap)));
            if (hf == 0 && (Lr <= 0 || no_rope || Lr > cap)) flag_error(p.err, kErrOOB);
        }

        if (warp == 0) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                         "r"(kXCols));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
        if (tid == 0) {
            for (int i = 0; i < 2; ++i) {
                mbar_init(&sm.k_full[i], kXBlk);
                mbar_init(&sm.v_full[i], kXBlk);
                mbar_init(&sm.k_empty[i], 1);
                mbar_init(&sm.v_empty[i], 1);
                mbar_init(&sm.s_full[i], 1);
                mbar_init(&sm.p_full[i], kXSoftThreads);
            }
            mbar_init(&sm.pv_done, 1);
            mbar_init(&sm.fin, 1);
            fence_mbar_init();
            sm.tmax = 0;
            sm.tmin = 0x7FFFFFFF;
            sm.abort = 0;
        }
        tc_before_sync();
        cta_bar();  // barriers initialised, tensor memory allocated
        tc_after_sync();
        if (hf == 0 && rowlen > 0) atomicMax(&sm.tmax, rowlen);
        if (hf == 0 && rowlen >= 0) atomicMin(&sm.tmin, rowlen);

        // ---------------- q' of row r (first half): turned, rotated, scaled, split into fp16 parts ----------------
        // score of a token = qexp (ksc S + zq kz) in log2 units, S the q.K accumulator, (ksc, kz) the
        // key's scale and zero: qexp = 2^(24 - e) undoes the code scale and the row's power of two,
        // zq = sum(q') / qexp carries the zero term
        if (hf == 0) {
            float qsum = 0.0f, qexp = 1.0f;
            float x[kHeadDim];
            if (rowlen > 0) {
                const uint4* qr = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.a.q) +
                                                                 (int64_t(q0 + qi) * p.g.Hq + h * G + g) * kHeadDim);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint4 w = __ldg(qr + c);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        x[8 * c + 2 * e] = __uint_as_float(ww[e] << 16);
                        x[8 * c + 2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
                    }
                }
                if (p.g.rope) {  // rotate-half pairs (i, i + 64) at position L - n + qi
                    const float2* cs = reinterpret_cast<const float2*>(p.g.rope + (L - n + qi) * kHeadDim);
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        const float2 c = __ldg(cs + i);
                        const float a = x[i], b = x[i + 64];
                        x[i] = fmaf(a, c.x, -b * c.y);
                        x[i + 64] = fmaf(b, c.x, a * c.y);
                    }
                }
                float sc = p.qscale;
                if (p.g.mode == 2) {
                    const int b = p.g.bdr_block;
#pragma unroll
                    for (int hs = 1; hs < 128; hs <<= 1) {
                        if (hs < b) {
#pragma unroll
                            for (int i = 0; i < 128; ++i)
                                if ((i & hs) == 0) {
                                    const float a = x[i], c = x[i + hs];
                                    x[i] = a + c;
                                    x[i + hs] = a - c;
                                }
                        }
                    }
                    sc *= rsqrtf(float(b));
                }
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 128; ++i) {
                    x[i] *= sc;
                    qsum += x[i];
                    amax = fmaxf(amax, fabsf(x[i]));
                }
                // scale by 2^e so that the largest component sits in [2^13, 2^14): fp16 keeps both parts
                int e = 0;
                if (amax > 0.0f) e = 13 - (int((__float_as_uint(amax) >> 23) & 0xFF) - 127);
                e = max(-100, min(100, e));
                const float up = exp2f(float(e));
                qexp = exp2f(float(24 - e));
#pragma unroll
                for (int i = 0; i < 128; ++i) x[i] *= up;
            } else {
#pragma unroll
                for (int i = 0; i < 128; ++i) x[i] = 0.0f;
            }
            sm.qx[row] = make_float2(qexp, qsum / qexp);
            // row r of q' into TMEM lane r, the A operand of q.K: column c of the high (low) part holds
            // the fp16 pair (dims 2 c, 2 c + 1)
            const uint32_t qcol = sm.tmem + (uint32_t((warp & 3) * 32) << 16) + kColQ;
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // dims 32 c .. 32 c + 31
                uint32_t hw[16], lw[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float a = x[32 * c + 2 * e], b = x[32 * c + 2 * e + 1];
                    const uint32_t ha = h_bits(a), hb = h_bits(b);
                    hw[e] = ha | (hb << 16);
                    lw[e] = h_bits(a - __half2float(__ushort_as_half(uint16_t(ha)))) |
                            (h_bits(b - __half2float(__ushort_as_half(uint16_t(hb)))) << 16);
                }
                tmem_st16(qcol + 16 * c, hw);
                tmem_st16(qcol + 64 + 16 * c, lw);
            }
            tmem_wait_st();
        }
        tc_before_sync();
        cta_bar();  // q' in tensor memory, row lengths
        tc_after_sync();
        const uint32_t tm = sm.tmem;
        const int tmax = sm.tmax, tmin = sm.tmin;
        const int nblocks = (tmax + kXBlk - 1) / kXBlk;
        // q only (never written by an append) so far; the cache after the previous grid
        grid_dep_wait();
        grid_dep_launch();

        const uint32_t tm_row = tm + (uint32_t((warp & 3) * 32) << 16);  // this warp's lanes
        const float qexp = sm.qx[row].x, zq = sm.qx[row].y;
        const float tau = kTau / qexp;  // the reference threshold in the units of ksc S + zq kz
        float O[kHeadDim / 2];          // this half of the row's output columns, read after the last block
        float l = 0.0f, Zs = 0.0f;      // this half's share of the weight sum and the zero term
        bool ok = true;
        float m_ref = -INFINITY;
        int k_ref = 0;       // P = p scale_v 2^-k, k the same for every row of the CTA
        bool k_set = false;
        bool of_valid = false;
        for (int j = 0; j < nblocks; ++j) {
            const int b = j & 1;
            const uint32_t par = (j >> 1) & 1;
            const bool w = xwait(&sm.s_full[b], par, abort, p.err) && xwait(&sm.v_full[b], par, abort, p.err);
            tc_after_sync();
            // ---- pass 1: this half's scores (ksc S + zq kz, -inf when masked) and their max ----
            uint32_t sv[64];
            const uint32_t s_col = tm_row + kColS + 128 * b;
            tmem_ld32(s_col + 64 * hf, sv);
            tmem_ld32(s_col + 64 * hf + 32, sv + 32);
            tmem_wait_ld();
            const int tb = j * kXBlk + 64 * hf;  // position of this half's first token
            const bool full = (j * kXBlk + kXBlk <= tmin) &&
                              ((sm.vmask[b][0] & sm.vmask[b][1] & sm.vmask[b][2] & sm.vmask[b][3]) == 0xFFFFFFFFu);
            float mb4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            const float4* kz4 = reinterpret_cast<const float4*>(sm.ksz[b]) + 32 * hf;
#pragma unroll
            for (int c = 0; c < 2; ++c) {  // 32 tokens at a time: their 16 (scale, zero) loads issue together
                float4 kz[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) kz[i] = kz4[16 * c + i];
                const uint32_t vm = full ? 0xFFFFFFFFu : sm.vmask[b][2 * hf + c];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = 32 * c + 2 * i;
                    const float v0 = fmaf(kz[i].x, __uint_as_float(sv[t]), zq * kz[i].y);
                    const float v1 = fmaf(kz[i].z, __uint_as_float(sv[t + 1]), zq * kz[i].w);
                    const float m0 = (full || ((tb + t < rowlen) && ((vm >> (2 * i)) & 1u))) ? v0 : -INFINITY;
                    const float m1 = (full || ((tb + t + 1 < rowlen) && ((vm >> (2 * i + 1)) & 1u))) ? v1 : -INFINITY;
                    sv[t] = __float_as_uint(m0);
                    sv[t + 1] = __float_as_uint(m1);
                    mb4[i & 3] = fmaxf(mb4[i & 3], fmaxf(m0, m1));
                }
            }
            const float hmax = fmaxf(fmaxf(mb4[0], mb4[1]), fmaxf(mb4[2], mb4[3]));
            // the power of two for P, the same for every row: 2^8 * max scale 2^-k < 2^15.  It is set at
            // the first block with values, with room for scales 16 times larger, and raised only when a
            // block's values exceed that.
            int k_new = k_ref;
            {
                const float vmx = fmaxf(fmaxf(sm.vmax[b][0], sm.vmax[b][1]), fmaxf(sm.vmax[b][2], sm.vmax[b][3]));
                if (vmx > 0.0f && vmx < INFINITY) {
                    const int k_target = max(-100, min(100, int((__float_as_uint(vmx) >> 23) & 0xFF) - 127 - 6));
                    if (!k_set) {
                        k_new = min(100, k_target + 4);
                        k_set = true;
                    } else {
                        k_new = max(k_ref, k_target);
                    }
                }
            }
            // The two halves of a row exchange their maxima (the pair barrier also ends the loop for both
            // when a wait gave up).  A row's reference moves when the row's max passes it by tau, or k moves.
            sm.hm[b][hf][row] = hmax;
            if (pair_any(warp, !w || *abort)) {
                ok = false;
                break;
            }
            const float mblk = fmaxf(hmax, sm.hm[b][hf ^ 1][row]);
            const float m_new = (mblk > m_ref + tau || (m_ref == -INFINITY && mblk > -INFINITY)) ? mblk : m_ref;
            const bool move = (m_ref != -INFINITY) && (m_new != m_ref || k_new != k_ref);
            // ---- every 4 blocks O_t (blocks j - 4 .. j - 1) is folded into O_f and the next P.V restarts it;
            // a row whose reference moves rescales its part of O_t in place and of O_f.  Both need the P.V of
            // block j - 1 complete.  Warp-uniform (tcgen05.ld / st are warp-wide): lanes that do not move
            // scale by 1. ----
            const bool fold = j > 0 && (j % kFoldEvery) == 0;
            if (fold || __any_sync(0xffffffffu, move)) {
                const float alpha = move ? fast_exp2(qexp * (m_ref - m_new)) * pow2i(k_ref - k_new) : 1.0f;
                if (j > 0 && __all_sync(0xffffffffu, xwait(&sm.pv_done, (j - 1) & 1, abort, p.err))) {
                    tc_after_sync();
                    float4* ofr = sm.of[row];
#pragma unroll 1
                    for (int c = 64 * hf; c < 64 * hf + 64; c += 16) {
                        uint32_t a[16];
                        tmem_ld16(tm_row + kColOt + c, a);
                        tmem_wait_ld();
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            float4& dst = ofr[((c >> 2) + q4) ^ (row & 7)];
                            const float4 o = of_valid ? dst : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                            if (fold) {
                                dst = make_float4((o.x + __uint_as_float(a[4 * q4])) * alpha,
                                                  (o.y + __uint_as_float(a[4 * q4 + 1])) * alpha,
                                                  (o.z + __uint_as_float(a[4 * q4 + 2])) * alpha,
                                                  (o.w + __uint_as_float(a[4 * q4 + 3])) * alpha);
                            } else {
                                if (of_valid) dst = make_float4(o.x * alpha, o.y * alpha, o.z * alpha, o.w * alpha);
#pragma unroll
                                for (int e = 0; e < 4; ++e) a[4 * q4 + e] = __float_as_uint(__uint_as_float(a[4 * q4 + e]) * alpha);
                            }
                        }
                        if (!fold) tmem_st16(tm_row + kColOt + c, a);
                    }
                    if (!fold) tmem_wait_st();
                    if (fold) of_valid = true;
                }
                l *= alpha;
                Zs *= alpha;
            }
            m_ref = m_new;
            k_ref = k_new;
            // ---- pass 2: p 2^-k = 2^(qexp (v - m) - k); P = p scale_v 2^-k as fp16 high and low parts over
            // S: chunk c of 32 tokens keeps its high parts in columns 32 c .. 32 c + 15 (token pairs) and
            // its low parts in 32 c + 16 .. 32 c + 31, so each half writes only the columns it read ----
            const float cofs = (m_ref == -INFINITY) ? 0.0f : -qexp * m_ref - float(k_ref);
            const float4* vz4 = reinterpret_cast<const float4*>(sm.vsz[b]) + 32 * hf;
            float lb[4] = {0.0f, 0.0f, 0.0f, 0.0f}, zb[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // independent partial sums
#pragma unroll
            for (int c = 0; c < 2; ++c) {  // 32 tokens (chunk 2 hf + c of the block) at a time
                uint32_t hw[16], lw[16];
                float4 vzc[16];  // their 16 (scale, zero + 8 scale) loads issue together
#pragma unroll
                for (int i = 0; i < 16; ++i) vzc[i] = vz4[16 * c + i];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int t0 = 32 * c + 2 * e;
                    const float4 vz = vzc[e];
                    const float p0 = fast_exp2(fmaf(__uint_as_float(sv[t0]), qexp, cofs));
                    const float p1 = fast_exp2(fmaf(__uint_as_float(sv[t0 + 1]), qexp, cofs));
                    lb[e & 3] += p0 + p1;
                    zb[e & 3] = fmaf(p0, vz.y, fmaf(p1, vz.w, zb[e & 3]));
                    const float a = p0 * vz.x, bb = p1 * vz.z;
                    const __half2 hi2 = __floats2half2_rn(a, bb);
                    const float2 back = __half22float2(hi2);
                    const __half2 lo2 = __floats2half2_rn(a - back.x, bb - back.y);
                    hw[e] = *reinterpret_cast<const uint32_t*>(&hi2);
                    lw[e] = *reinterpret_cast<const uint32_t*>(&lo2);
                }
                // tokens 16 c .. 16 c + 15 of this half: chunk 2 hf + c / 2 of the block, its (c % 2)-th 8 pairs
                const uint32_t pc = s_col + 64 * hf + 32 * c;
                tmem_st16(pc, hw);
                tmem_st16(pc + 16, lw);
            }
            l += (lb[0] + lb[1]) + (lb[2] + lb[3]);
            Zs += (zb[0] + zb[1]) + (zb[2] + zb[3]);
            tmem_wait_st();
            tc_before_sync();
            mbar_arrive(&sm.p_full[b]);
        }
        // ---- this half's output columns: O_f + O_t once the last P.V is complete ----
#pragma unroll
        for (int d = 0; d < kHeadDim / 2; ++d) O[d] = 0.0f;
        if (ok && nblocks > 0) {
            if (__all_sync(0xffffffffu, xwait(&sm.pv_done, (nblocks - 1) & 1, abort, p.err))) {
                tc_after_sync();
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t a[32];
                    tmem_ld32(tm_row + kColOt + 64 * hf + 32 * c, a);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 o = of_valid ? sm.of[row][(16 * hf + 8 * c + q4) ^ (row & 7)]
                                                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        O[32 * c + 4 * q4 + 0] = __uint_as_float(a[4 * q4 + 0]) + o.x;
                        O[32 * c + 4 * q4 + 1] = __uint_as_float(a[4 * q4 + 1]) + o.y;
                        O[32 * c + 4 * q4 + 2] = __uint_as_float(a[4 * q4 + 2]) + o.z;
                        O[32 * c + 4 * q4 + 3] = __uint_as_float(a[4 * q4 + 3]) + o.w;
                    }
                }
            } else {
                ok = false;
            }
        }
        // ---- free the tensor memory (every role is past its last use) ----
        tc_before_sync();
        cta_bar();
        if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(kXCols));
        // ---- the row's weight sum and zero term from both halves; normalise ----
        sm.lz[hf][row] = make_float2(l, Zs);
        pair_bar(warp);
        const float2 lz2 = sm.lz[hf ^ 1][row];
        const float lt = l + lz2.x, zt = Zs + lz2.y;
        const float inv = lt > 0.0f ? 1.0f / lt : 0.0f;
#pragma unroll
        for (int d = 0; d < kHeadDim / 2; ++d) O[d] = fmaf(O[d], kTwo24, zt) * inv;
        // ---- rotate back: butterflies of stride < 64 stay inside a half; stride 64 pairs the halves
        // through shared memory (the key tiles, free now), laid out [half][column][row] ----
        if (p.g.mode == 2 && p.g.rotate_v) {
            const int bb = p.g.bdr_block;
#pragma unroll
            for (int hs = 1; hs < 64; hs <<= 1) {
                if (hs < bb) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if ((i & hs) == 0) {
                            const float a = O[i], c = O[i + hs];
                            O[i] = a + c;
                            O[i + hs] = a - c;
                        }
                }
            }
            if (bb == 128) {
                float* xo = reinterpret_cast<float*>(sm.k[0]);
#pragma unroll
                for (int i = 0; i < 64; ++i) xo[(hf * 64 + i) * kXRows + row] = O[i];
                pair_bar(warp);
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const float other = xo[((hf ^ 1) * 64 + i) * kXRows + row];
                    O[i] = hf == 0 ? O[i] + other : other - O[i];
                }
            }
            const float rs = rsqrtf(float(bb));
#pragma unroll
            for (int d = 0; d < kHeadDim / 2; ++d) O[d] *= rs;
        }
        if (qi < 0 || !ok || *abort) return;
        const int64_t orow = (int64_t(q0 + qi) * p.g.Hq + h * G + g) * kHeadDim + 64 * hf;
        if (p.a.out_fp32) {
            float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(p.a.out) + orow);
#pragma unroll
            for (int c = 0; c < 16; ++c) o4[c] = make_float4(O[4 * c], O[4 * c + 1], O[4 * c + 2], O[4 * c + 3]);
        } else {
            uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.a.out) + orow);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(O[8 * c + 2 * e], O[8 * c + 2 * e + 1]);
                    w[e] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                o4[c] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    } else if (warp < kXMmaWarp) {
        // =============================== loaders ===============================
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kXRegsLoad));
        cta_bar();  // barriers initialised
        cta_bar();  // row lengths
        const int tmax = sm.tmax;
        const int nblocks = (tmax + kXBlk - 1) / kXBlk;
        grid_dep_wait();
        grid_dep_launch();
        const int t = tid - 32 * kXSoftWarps;  // token of the block
        const int lw = warp - kXSoftWarps;
        const int32_t* pt = p.a.page_table + int64_t(s) * p.a.pt_stride;
        const uint8_t* kpool = static_cast<const uint8_t*>(p.g.k_pool);
        const uint8_t* vpool = static_cast<const uint8_t*>(p.g.v_pool);
        // page id of token t of block j, loaded one block before its codes
        auto page_id = [&](int j) -> int {
            const int T = j * kXBlk + t;
            return (j < nblocks && T < tmax) ? __ldg(pt + page_of_pos(p, T)) : -1;
        };
        int npage = page_id(0);
        for (int j = 0; j < nblocks; ++j) {
            if (__any_sync(0xffffffffu, *abort)) break;  // warp-uniform: the warp's shuffles follow
            const int b = j & 1;
            const int T = j * kXBlk + t;
            const int page = npage;
            npage = page_id(j + 1);
            // the token's key and value codes as 16 words of the 4-bit nibble layout (word n: dims
            // 8 n .. 8 n + 7); a masked token's values are the centre itself (centred zero)
            uint32_t nk[16], nv[16];
            uint32_t cks = 0, cvs = 0;
            bool tok = false;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                nk[n] = 0u;
                nv[n] = kCentreNib;
            }
            if (T < tmax) {
                if (page >= 0 && page < p.g.num_pages) {
                    const int64_t row = (int64_t(page) * p.g.H + h) * p.g.page_size + slot_of_pos(p, T);
                    const uint4* kr = reinterpret_cast<const uint4*>(kpool + row * (16 * CB));
                    const uint4* vr = reinterpret_cast<const uint4*>(vpool + row * (16 * CB));
#pragma unroll
                    for (int i = 0; i < CB; ++i) {  // 16-byte units of the row: 4 (4-bit) or 2 (2-bit)
                        const uint4 a = __ldg(kr + i), c = __ldg(vr + i);
                        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            if (CB == 4) {
                                nk[4 * i + e] = aw[e];
                                nv[4 * i + e] = cw[e];
                            } else {  // 16 two-bit codes (dims 16 m .. 16 m + 15) -> two nibble words
                                const uint2 ka = expand2(aw[e]), va = expand2(cw[e]);
                                nk[8 * i + 2 * e] = ka.x;
                                nk[8 * i + 2 * e + 1] = ka.y;
                                nv[8 * i + 2 * e] = va.x;
                                nv[8 * i + 2 * e + 1] = va.y;
                            }
                        }
                    }
                    cks = __ldg(p.g.k_sz + row);
                    cvs = __ldg(p.g.v_sz + row);
                    tok = true;
                } else {
                    flag_error(p.err, kErrOOB);
                }
            }
            // ---- key tile: free once q.K of block j - 2 is done ----
            bool w = true;
            if (j >= 2) {
                w = (lane == 0) ? xwait(&sm.k_empty[b], ((j >> 1) + 1) & 1, abort, p.err) : true;
                w = __shfl_sync(0xffffffffu, w, 0);
            }
            if (!w) break;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                uint32_t o4[4];
                codes_to_f16(nk[n], 0u, o4);
                *reinterpret_cast<uint4*>(sm.k[b] + tile_off(t, 8 * n)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
            fence_proxy_async();
            mbar_arrive(&sm.k_full[b]);
            // ---- value tile and the tokens' scales: free once P.V of block j - 2 is done ----
            if (j >= 2) {
                w = (lane == 0) ? xwait(&sm.v_empty[b], ((j >> 1) + 1) & 1, abort, p.err) : true;
                w = __shfl_sync(0xffffffffu, w, 0);
            }
            if (!w) break;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                uint32_t o4[4];
                codes_to_f16(nv[n], kCentreF16, o4);
                *reinterpret_cast<uint4*>(sm.v[b] + tile_off(t, 8 * n)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
            const float ksc = half_lo(cks), kzr = half_hi(cks);
            const float vsc = half_lo(cvs), vzr = half_hi(cvs);
            sm.ksz[b][t] = tok ? make_float2(ksc, kzr) : make_float2(0.0f, 0.0f);
            sm.vsz[b][t] = tok ? make_float2(vsc, vzr + kCentre * vsc) : make_float2(0.0f, 0.0f);
            float vmx = tok ? fabsf(vsc) : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, o));
            const uint32_t bal = __ballot_sync(0xffffffffu, tok);
            if (lane == 0) {
                sm.vmask[b][lw] = bal;
                sm.vmax[b][lw] = vmx;
            }
            fence_proxy_async();
            mbar_arrive(&sm.v_full[b]);
        }
        cta_bar();
    } else {
        // =============================== MMA issue ===============================
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kXRegsMma));
        cta_bar();  // barriers initialised
        cta_bar();  // q tiles, tensor memory, row lengths
        tc_after_sync();
        const uint32_t tm = sm.tmem;
        const int nblocks = (sm.tmax + kXBlk - 1) / kXBlk;
        grid_dep_wait();
        grid_dep_launch();
        if (warp == kXMmaWarp && lane == 0) {
            bool issued = false;
            for (int j = 0; j <= nblocks; ++j) {
                if (*abort) break;
                if (j < nblocks) {  // S_j = q K_j^T into score buffer j % 2
                    const int b = j & 1;
                    if (!xwait(&sm.k_full[b], (j >> 1) & 1, abort, p.err)) break;
                    // the buffer held P_{j-2}: its P.V must be complete
                    if (j >= 2 && !xwait(&sm.pv_done, (j - 2) & 1, abort, p.err)) break;
                    tc_after_sync();
                    const uint32_t kb = smem_u32(sm.k[b]);
                    const uint32_t d = tm + kColS + 128 * b;
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int ks = 0; ks < kHeadDim / 16; ++ks)
                            mma_ts(d, tm + kColQ + 64 * part + 8 * ks, sdesc(kb + 256 * ks, 128, 2048), kIdQK,
                                   (part | ks) ? 1u : 0u);
                    mma_commit(&sm.s_full[b]);
                    mma_commit(&sm.k_empty[b]);
                    issued = true;
                }
                if (j >= 1) {  // O_t += P_{j-1} V_{j-1}
                    const int i = j - 1, b = i & 1;
                    if (!xwait(&sm.p_full[b], (i >> 1) & 1, abort, p.err)) break;
                    if (!xwait(&sm.v_full[b], (i >> 1) & 1, abort, p.err)) break;
                    tc_after_sync();
                    const bool restart = (i % kFoldEvery) == 0;  // O_t was folded during the softmax of block i
                    const uint32_t pa = tm + kColS + 128 * b;
                    const uint32_t vb = smem_u32(sm.v[b]);
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int ks = 0; ks < kXBlk / 16; ++ks)
                            mma_ts(tm + kColOt, pa + 32 * (ks >> 1) + 8 * (ks & 1) + 16 * part, sdesc(vb + 4096 * ks, 2048, 128), kIdPV,
                                   (restart && part == 0 && ks == 0) ? 0u : 1u);
                    mma_commit(&sm.pv_done);
                    mma_commit(&sm.v_empty[b]);
                }
            }
            if (issued) {  // nothing this thread issued is still running when the tensor memory is freed
                mma_commit(&sm.fin);
                if (!mbar_wait(&sm.fin, 0)) flag_error(p.err, kErrTimeout);
            }
        }
        tc_before_sync();
        cta_bar();
    }
}

template <int G, int CB>
cudaError_t launch_g(const DecodeParams& dp, const int32_t* q_indptr, int max_q_len, dim3 grid, cudaStream_t s) {
    constexpr auto kern = extend_tc_kernel<G, CB>;
    const cudaError_t e = ensure_smem_opt_in<kern>(kXSmem);
    if (e != cudaSuccess) return e;
    return launch_overlapped(kern, grid, dim3(kXThreads), kXSmem, s, dp, q_indptr, max_q_len);
}

template <int CB>
cudaError_t launch_cb(const DecodeParams& dp, const int32_t* q_indptr, int max_q_len, dim3 grid, cudaStream_t s) {
    switch (dp.g.Hq / dp.g.H) {
        case 1: return launch_g<1, CB>(dp, q_indptr, max_q_len, grid, s);
        case 2: return launch_g<2, CB>(dp, q_indptr, max_q_len, grid, s);
        case 4: return launch_g<4, CB>(dp, q_indptr, max_q_len, grid, s);
        case 8: return launch_g<8, CB>(dp, q_indptr, max_q_len, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_extend(const CacheGeom& g, const ExtendArgs& a, int* err_word, cudaStream_t s) {
    if (a.batch == 0 || a.max_q_len == 0) return cudaSuccess;
    DecodeParams dp;
    dp.g = g;
    dp.a = DecodeArgs{a.q, a.seq_lens, a.page_table, a.pt_stride, a.batch, a.max_seq_len, a.out, a.out_fp32,
                      nullptr, 0};
    dp.item_tokens = 0;
    dp.max_splits = 0;
    dp.qscale = float(1.0 / sqrt(double(kHeadDim))) * kLog2e;
    dp.ps_shift = -1;
    for (int sh = 0; sh < 11; ++sh)
        if ((1 << sh) == g.page_size) dp.ps_shift = sh;
    dp.ws_o = nullptr;
    dp.ws_ml = nullptr;
    dp.err = err_word;
    const int qb = kXRows / (g.Hq / g.H);
    const dim3 grid((a.max_q_len + qb - 1) / qb, g.H, a.batch);
    return g.code_bits == 2 ? launch_cb<2>(dp, a.q_indptr, a.max_q_len, grid, s)
                            : launch_cb<4>(dp, a.q_indptr, a.max_q_len, grid, s);
}

}  // namespace kvq
