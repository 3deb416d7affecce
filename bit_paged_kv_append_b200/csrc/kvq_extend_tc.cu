// kvq_extend_tc.cu -- extend (chunked-prefill) attention over the paged INT4 cache on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in tensor memory).
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
// queries x the G heads), 4 warps; thread r owns row r, which is TMEM lane r (warp w reads
// lanes 32 w .. 32 w + 31).  Two CTAs share an SM (97 KB of shared memory and 256 TMEM
// columns each), so one CTA's softmax overlaps the other's tensor-core work.  Per block of
// 32 key tokens:
//   1. every thread copies a quarter of one token's K and V code rows (prefetched one block
//      ahead into registers) into the block's operand tiles: key codes as the exact fp16
//      subnormals c 2^-24 (B of q.K, K-major), value codes centred, (c - 8) 2^-24 (B of P.V,
//      N-major);
//   2. one thread issues q.K: S[128 x 32] (fp32, TMEM) = q_hi K^T + q_lo K^T, 16 MMAs of
//      M128 N32 K16 (kind::f16).  q' = rope(q) H_blk log2(e)/sqrt(D) is scaled per row by a
//      power of two to ~2^14 and split into fp16 high and low parts (~22 significant bits);
//   3. each thread reads its row of S, forms the scores, and runs the online softmax with a
//      lazily moved reference max: p = 2^(s - m_ref) may reach 2^8 before the reference
//      moves, and P = p scale_v 2^-k_ref carries a per-row power of two that keeps it below
//      2^15 in fp16.  P goes to shared memory as fp16 high and low parts;
//   4. one thread issues P.V: O[128 x 128] (fp32, TMEM) += P_hi V + P_lo V, 4 MMAs of M128
//      N128 K16.
// When any row's reference must move, and every 16 blocks, the CTA folds O into fp32
// registers (one row per thread, ordinary IEEE adds) and restarts the TMEM accumulation:
// the tensor cores' fp32 accumulation does not round to nearest, and over thousands of
// tokens its bias would grow; a fold bounds each accumulation run to 512 tokens.
//
// Waits on the MMA mbarrier are bounded (kWaitLimitNs; on expiry the CTA flags
// KV_ERR_TIMEOUT, stops issuing, waits once more for what it issued and frees its tensor
// memory).  The 2-bit variant keeps the mma.sync kernel (kvq_extend.cu).
#include "kvq_mma.cuh"

namespace kvq {
namespace {

constexpr int kTcRows = 128;    // (query, head) rows per CTA = threads = TMEM lanes
constexpr int kTcBlock = 32;    // key tokens per block
constexpr int kTcCols = 256;    // TMEM columns per CTA: S at 0 .. 31, O at 128 .. 255
constexpr int kTcOCol = 128;
constexpr int kFoldEvery = 16;  // blocks between forced folds (512 tokens)
constexpr float kTau = 8.0f;    // the reference max moves once a score passes it by this much (log2)

// Shared-memory operand tiles, no swizzle, "core matrices" of 8 rows x 16 bytes (128
// contiguous bytes).  K-major tiles: core (row group, 16-byte chunk of the K extent);
// N-major: core (8 K rows, 8 N elements).
constexpr int kQTile = kTcRows * kHeadDim * 2;   // 32 KB: q' part [128 rows][128 dims] fp16, K-major
constexpr int kKTile = kTcBlock * kHeadDim * 2;  // 8 KB: key codes [32 tokens][128 dims] fp16, K-major
constexpr int kVTile = kTcBlock * kHeadDim * 2;  // 8 KB: value codes [32 tokens][128 dims] fp16, N-major
constexpr int kPTile = kTcRows * kTcBlock * 2;   // 8 KB: P part [128 rows][32 tokens] fp16, K-major

struct TcSmem {
    uint8_t q[2][kQTile];   // high, low parts of q'
    uint8_t k[kKTile];
    uint8_t v[2][kVTile];   // double buffer: P.V of block j reads one while block j + 1 fills the other
    uint8_t p[2][kPTile];   // high, low parts of P
    float2 ksz[kTcBlock];   // (scale, zero) of the block's keys
    float2 vsz[kTcBlock];   // (scale, zero + 8 scale) of its values
    uint32_t vmask;         // tokens of the block on valid pages
    float vmax[4];          // per warp: the largest value scale of its eight tokens
    int tmax, tmin;         // longest / shortest row of the CTA
    uint64_t bar;           // MMA completion
    uint32_t tmem;          // TMEM base column
    int abort;              // a wait timed out
};
constexpr size_t kTcSmem = sizeof(TcSmem) + 1024;  // + alignment slack (tiles start 1024-aligned)

// K-major tile byte offset of element (row r, k index kk) for 2-byte elements, K extent kext
__device__ __forceinline__ uint32_t kmaj(int r, int kk, int kext) {
    return uint32_t(((r >> 3) * (kext >> 3) + (kk >> 3)) * 128 + (r & 7) * 16 + (kk & 7) * 2);
}
// N-major tile byte offset of element (k row kk, n index n) for 2-byte elements, N extent next
__device__ __forceinline__ uint32_t nmaj(int kk, int n, int next) {
    return uint32_t(((kk >> 3) * (next >> 3) + (n >> 3)) * 128 + (kk & 7) * 16 + (n & 7) * 2);
}

// Shared-memory matrix descriptor: no swizzle, Blackwell version bit, byte offsets >> 4.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return uint64_t((saddr >> 4) & 0x3FFF) | (uint64_t((lbo >> 4) & 0x3FFF) << 16) |
           (uint64_t((sbo >> 4) & 0x3FFF) << 32) | (uint64_t(1) << 46);
}
// Instruction descriptor of kind::f16: fp16 A and B, fp32 D, A K-major, B K- or N-major.
__host__ __device__ constexpr uint32_t idesc_f16(int n, int m, int b_nmajor) {
    return (1u << 4) | (uint32_t(b_nmajor) << 16) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}
constexpr uint32_t kIdQK = idesc_f16(kTcBlock, kTcRows, 0);  // S[128 x 32] = A[128 x 16] B[32 x 16]^T
constexpr uint32_t kIdPV = idesc_f16(kHeadDim, kTcRows, 1);  // O[128 x 128] = A[128 x 16] B[16 x 128]

__device__ __forceinline__ void mma_f16(uint32_t dcol, uint64_t da, uint64_t db, uint32_t id, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(dcol),
        "l"(da), "l"(db), "r"(id), "r"(acc), "r"(0u)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive TMEM columns of this warp's 32 lanes (lane = thread's row)
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(addr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16 consecutive TMEM columns of this warp's 32 lanes
__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(addr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Bounded wait for phase `parity` of the MMA barrier; false after kWaitLimitNs.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) { return mbar_wait(bar, parity); }

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

template <int G>
__global__ void __launch_bounds__(kTcRows, 2) extend_tc_kernel(const __grid_constant__ DecodeParams p,
                                                               const int32_t* __restrict__ q_indptr, int max_q_len) {
    constexpr int QB = kTcRows / G;  // queries per CTA
    extern __shared__ uint8_t dsm_raw[];
    TcSmem& sm = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    const int z = blockIdx.x, h = blockIdx.y, s = blockIdx.z;  // z: query block, from the last
    const int tid = threadIdx.x, warp = tid >> 5;

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

    // ---- row r = tid: query qi = qhi - QB + r / G, head g = r % G; its length = position + 1.
    // Only the last max_q_len queries of a sequence are computed (the grid may cover more). ----
    const int qi0 = qhi - QB + tid / G, g = tid % G;
    const int qi = qi0 >= n - max_q_len ? qi0 : -1;
    int rowlen = -1;  // -1: no such query
    if (qi >= 0) {
        const int64_t Lr = L - n + qi + 1;
        const bool no_rope = p.g.rope && Lr > p.g.rope_positions;
        rowlen = (Lr <= 0 || no_rope) ? 0 : int(min(Lr, int64_t(cap)));
        if (Lr <= 0 || no_rope || Lr > cap) flag_error(p.err, kErrOOB);
    }

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(kTcCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
        sm.tmax = 0;
        sm.tmin = 0x7FFFFFFF;
        sm.abort = 0;
    }
    __syncthreads();
    if (rowlen > 0) atomicMax(&sm.tmax, rowlen);
    if (rowlen >= 0) atomicMin(&sm.tmin, rowlen);

    // ---------------- q' of row r: turned, rotated, scaled, split into fp16 parts ----------------
    // score of a token = qexp (ksc S + zq kz) in log2 units, S the q.K accumulator, (ksc, kz) the
    // key's scale and zero: qexp = 2^(24 - e) undoes the code scale and the row's power of two,
    // zq = sum(q') / qexp carries the zero term
    float qsum = 0.0f, qexp = 1.0f;
    {
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
        // row r of the q tiles: 16 chunks of 8 dims, high and low parts
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = x[8 * c + 2 * e], b = x[8 * c + 2 * e + 1];
                const uint32_t ha = h_bits(a), hb = h_bits(b);
                hw[e] = ha | (hb << 16);
                lw[e] = h_bits(a - __half2float(__ushort_as_half(uint16_t(ha)))) |
                        (h_bits(b - __half2float(__ushort_as_half(uint16_t(hb)))) << 16);
            }
            const uint32_t off = kmaj(tid, 8 * c, kHeadDim);
            *reinterpret_cast<uint4*>(sm.q[0] + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(sm.q[1] + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
    }
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tm = sm.tmem;
    const uint32_t tm_row = tm + (uint32_t(warp * 32) << 16);  // this warp's lanes
    const int tmax = sm.tmax, tmin = sm.tmin;
    const int nblocks = (tmax + kTcBlock - 1) / kTcBlock;

    // q only (never written by an append) so far; the cache after the previous grid
    grid_dep_wait();
    grid_dep_launch();

    const float zq = qsum / qexp;
    const float tau = kTau / qexp;  // the reference threshold in the units of ksc S + zq kz

    // ---- block loader: lane L of warp w copies quarter L >> 3 of token 8 w + (L & 7) of each block
    // (the eight lanes of a store phase fill the eight rows of one core matrix) ----
    const int lane = tid & 31;
    const int tt = 8 * warp + (lane & 7), qq = lane >> 3;
    const int32_t* pt = p.a.page_table + int64_t(s) * p.a.pt_stride;
    const uint8_t* kpool = static_cast<const uint8_t*>(p.g.k_pool);
    const uint8_t* vpool = static_cast<const uint8_t*>(p.g.v_pool);
    uint4 nk = make_uint4(0, 0, 0, 0), nv = make_uint4(0, 0, 0, 0);
    uint32_t nks = 0, nvs = 0;
    bool nok = false;
    // page id of this thread's token in block j: loaded one block before the codes, so that the
    // code loads never wait for it
    auto page_id = [&](int j) -> int {
        const int T = j * kTcBlock + tt;
        return (j < nblocks && T < tmax) ? __ldg(pt + page_of_pos(p, T)) : -1;
    };
    int npage = page_id(0);
    auto fetch = [&](int j) {  // raw codes of block j into the prefetch registers; then block j + 1's page id
        const int T = j * kTcBlock + tt;
        const int page = npage;
        npage = page_id(j + 1);
        nok = false;
        if (j < nblocks && T < tmax) {
            if (page >= 0 && page < p.g.num_pages) {
                const int64_t row = (int64_t(page) * p.g.H + h) * p.g.page_size + slot_of_pos(p, T);
                nk = __ldg(reinterpret_cast<const uint4*>(kpool + row * 64) + qq);
                nv = __ldg(reinterpret_cast<const uint4*>(vpool + row * 64) + qq);
                if (qq == 0) {
                    nks = __ldg(p.g.k_sz + row);
                    nvs = __ldg(p.g.v_sz + row);
                }
                nok = true;
            } else if (qq == 0) {
                flag_error(p.err, kErrOOB);
            }
        }
    };
    fetch(0);

    // ---- per-row softmax state: O, l and Z in units of 2^-k, relative to the reference m ----
    float O[kHeadDim];  // folded output (fp32, ordinary rounding)
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) O[d] = 0.0f;
    float m_ref = -INFINITY, l = 0.0f, Zs = 0.0f;
    int k_ref = 0;       // P = p scale_v 2^-k, k the same for every row of the CTA
    bool k_set = false;
    uint32_t acc = 0;    // the next P.V accumulates onto TMEM O (0: restart)
    int since_fold = 0;  // blocks accumulated in TMEM O since it was last folded
    uint32_t phase = 0;
    bool ok = true;
    const uint32_t s_addr = tm_row + 0, o_addr = tm_row + kTcOCol;

    for (int j = 0; j < nblocks && ok; ++j) {
        // ---------------- 1. operand tiles of block j ----------------
        {
            const bool tok = nok;
            const uint4 ck = nk, cv = nv;
            const uint32_t cks = nks, cvs = nvs;
            uint8_t* vt = sm.v[j & 1];
            const uint32_t kw[4] = {ck.x, ck.y, ck.z, ck.w}, vw[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t ko[4], vo[4];
                codes_to_f16(tok ? kw[c] : 0u, 0u, ko);
                codes_to_f16(tok ? vw[c] : 0x88888888u, kMinus8, vo);  // masked values: centred zero
                const int d0 = 32 * qq + 8 * c;  // dims d0 .. d0 + 7
                *reinterpret_cast<uint4*>(sm.k + kmaj(tt, d0, kHeadDim)) = make_uint4(ko[0], ko[1], ko[2], ko[3]);
                *reinterpret_cast<uint4*>(vt + nmaj(tt, d0, kHeadDim)) = make_uint4(vo[0], vo[1], vo[2], vo[3]);
            }
            float vmx = 0.0f;
            if (qq == 0) {
                const float ksc = half_lo(cks), kzr = half_hi(cks);
                const float vsc = half_lo(cvs), vzr = half_hi(cvs);
                sm.ksz[tt] = tok ? make_float2(ksc, kzr) : make_float2(0.0f, 0.0f);
                sm.vsz[tt] = tok ? make_float2(vsc, vzr + 8.0f * vsc) : make_float2(0.0f, 0.0f);
                vmx = tok ? fabsf(vsc) : 0.0f;
            }
            vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, 1));
            vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, 2));
            vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, 4));
            const uint32_t bal = __ballot_sync(0xffffffffu, tok && qq == 0);  // lane i < 8: token 8 w + i
            if (lane == 0) {
                reinterpret_cast<volatile uint8_t*>(&sm.vmask)[warp] = uint8_t(bal & 0xFFu);
                sm.vmax[warp] = vmx;
            }
        }
        fetch(j + 1);  // in flight while the block is computed
        fence_proxy_async();
        tc_before_sync();
        __syncthreads();
        tc_after_sync();
        // ---------------- 2. q.K ----------------
        if (tid == 0) {
            const uint32_t kb = smem_u32(sm.k);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t qa = smem_u32(sm.q[part]);
#pragma unroll
                for (int ks = 0; ks < kHeadDim / 16; ++ks)
                    mma_f16(tm, sdesc(qa + 256 * ks, 128, 2048), sdesc(kb + 256 * ks, 128, 2048), kIdQK,
                            (part | ks) ? 1u : 0u);
            }
            mma_commit(&sm.bar);
        }
        // the power of two for P, the same for every row: 2^8 * max scale 2^-k < 2^15.  It is set at
        // the first block with values, with room for scales 16 times larger, and raised (which needs
        // a fold) only when a block's values exceed that.
        int k_new = k_ref;
        {
            const float vmx = fmaxf(fmaxf(sm.vmax[0], sm.vmax[1]), fmaxf(sm.vmax[2], sm.vmax[3]));
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
        if (!tc_wait(&sm.bar, phase)) {
            flag_error(p.err, kErrTimeout);
            sm.abort = 1;
        }
        phase ^= 1;
        tc_after_sync();
        // ---------------- 3. scores and the online softmax of row r ----------------
        uint32_t sc[kTcBlock];  // S, then ksc S + zq kz (the score / qexp) as float bits, -inf when masked
        tmem_ld32(s_addr, sc);
        const int tb = j * kTcBlock;
        const uint32_t vmask = sm.vmask;
        const bool full = (tb + kTcBlock <= tmin) && (vmask == 0xFFFFFFFFu);
        float mb4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int t = 0; t < kTcBlock; ++t) {
            const float2 kz = sm.ksz[t];
            const float v = fmaf(kz.x, __uint_as_float(sc[t]), zq * kz.y);
            const float vm = (full || ((tb + t < rowlen) && ((vmask >> t) & 1u))) ? v : -INFINITY;
            sc[t] = __float_as_uint(vm);
            mb4[t & 3] = fmaxf(mb4[t & 3], vm);
        }
        const float mblk = fmaxf(fmaxf(mb4[0], mb4[1]), fmaxf(mb4[2], mb4[3]));
        const float m_new = (mblk > m_ref + tau || (m_ref == -INFINITY && mblk > -INFINITY)) ? mblk : m_ref;
        const bool fold = __syncthreads_or((since_fold > 0 && (m_new != m_ref || k_new != k_ref)) ||
                                           since_fold >= kFoldEvery || sm.abort) != 0;
        if (sm.abort) {  // a wait gave up: let what was issued finish (bounded) before TMEM is freed
            tc_wait(&sm.bar, phase ^ 1);
            ok = false;
            break;
        }
        if (fold) {  // every P.V so far is complete: the q.K commit waited for above came after it
#pragma unroll
            for (int c0 = 0; c0 < kHeadDim; c0 += 16) {
                uint32_t ov[16];
                tmem_ld16(o_addr + c0, ov);
#pragma unroll
                for (int d = 0; d < 16; ++d) O[c0 + d] += __uint_as_float(ov[d]);
            }
            acc = 0;
            since_fold = 0;
        }
        if (m_new != m_ref || k_new != k_ref) {
            const float alpha =
                (m_ref == -INFINITY) ? 0.0f : fast_exp2(qexp * (m_ref - m_new)) * pow2i(k_ref - k_new);
#pragma unroll
            for (int d = 0; d < kHeadDim; ++d) O[d] *= alpha;
            l *= alpha;
            Zs *= alpha;
            m_ref = m_new;
            k_ref = k_new;
        }
        // p 2^-k = 2^(qexp (v - m) - k); P = p scale_v 2^-k as fp16 high and low parts, tokens 8 c .. 8 c + 7
        const float cofs = (m_ref == -INFINITY) ? 0.0f : -qexp * m_ref - float(k_ref);
        float lb[4] = {0.0f, 0.0f, 0.0f, 0.0f}, zb[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // independent partial sums
#pragma unroll
        for (int c = 0; c < kTcBlock / 8; ++c) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t0 = 8 * c + 2 * e;
                const float2 v0 = sm.vsz[t0], v1 = sm.vsz[t0 + 1];
                const float p0 = fast_exp2(fmaf(__uint_as_float(sc[t0]), qexp, cofs));
                const float p1 = fast_exp2(fmaf(__uint_as_float(sc[t0 + 1]), qexp, cofs));
                lb[e] += p0 + p1;
                zb[e] = fmaf(p0, v0.y, fmaf(p1, v1.y, zb[e]));
                const float a = p0 * v0.x, b = p1 * v1.x;
                const __half2 hi2 = __floats2half2_rn(a, b);
                const float2 back = __half22float2(hi2);
                const __half2 lo2 = __floats2half2_rn(a - back.x, b - back.y);
                hw[e] = *reinterpret_cast<const uint32_t*>(&hi2);
                lw[e] = *reinterpret_cast<const uint32_t*>(&lo2);
            }
            const uint32_t off = kmaj(tid, 8 * c, kTcBlock);
            *reinterpret_cast<uint4*>(sm.p[0] + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(sm.p[1] + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        l += (lb[0] + lb[1]) + (lb[2] + lb[3]);
        Zs += (zb[0] + zb[1]) + (zb[2] + zb[3]);
        ++since_fold;
        fence_proxy_async();
        tc_before_sync();
        __syncthreads();
        tc_after_sync();
        // ---------------- 4. P.V ----------------
        if (tid == 0) {
            const uint32_t vb = smem_u32(sm.v[j & 1]);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t pa = smem_u32(sm.p[part]);
#pragma unroll
                for (int ks = 0; ks < kTcBlock / 16; ++ks)
                    mma_f16(tm + kTcOCol, sdesc(pa + 256 * ks, 128, 512), sdesc(vb + 4096 * ks, 2048, 128), kIdPV,
                            (acc | part | ks) ? 1u : 0u);
            }
        }
        acc = 1;
    }

    // ---------------- final fold, normalise, rotate back, store ----------------
    if (tid == 0 && ok) mma_commit(&sm.bar);
    __syncthreads();
    if (ok) {
        if (!tc_wait(&sm.bar, phase)) {
            flag_error(p.err, kErrTimeout);
            ok = false;
        }
        tc_after_sync();
    }
    if (ok && nblocks > 0) {
#pragma unroll
        for (int c0 = 0; c0 < kHeadDim; c0 += 16) {
            uint32_t ov[16];
            tmem_ld16(o_addr + c0, ov);
#pragma unroll
            for (int d = 0; d < 16; ++d) O[c0 + d] += __uint_as_float(ov[d]);
        }
    }
    tc_before_sync();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(kTcCols));
    if (qi < 0 || !ok) return;
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) O[d] = fmaf(O[d], kTwo24, Zs) * inv;
    if (p.g.mode == 2 && p.g.rotate_v) {
        const int b = p.g.bdr_block;
#pragma unroll
        for (int hs = 1; hs < 128; hs <<= 1) {
            if (hs < b) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if ((i & hs) == 0) {
                        const float a = O[i], c = O[i + hs];
                        O[i] = a + c;
                        O[i + hs] = a - c;
                    }
            }
        }
        const float rs = rsqrtf(float(b));
#pragma unroll
        for (int d = 0; d < kHeadDim; ++d) O[d] *= rs;
    }
    const int64_t orow = (int64_t(q0 + qi) * p.g.Hq + h * G + g) * kHeadDim;
    if (p.a.out_fp32) {
        float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(p.a.out) + orow);
#pragma unroll
        for (int c = 0; c < 32; ++c) o4[c] = make_float4(O[4 * c], O[4 * c + 1], O[4 * c + 2], O[4 * c + 3]);
    } else {
        uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.a.out) + orow);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(O[8 * c + 2 * e], O[8 * c + 2 * e + 1]);
                w[e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            o4[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

template <int G>
cudaError_t launch_g(const DecodeParams& dp, const int32_t* q_indptr, int max_q_len, dim3 grid, cudaStream_t s) {
    constexpr auto kern = extend_tc_kernel<G>;
    const cudaError_t e = ensure_smem_opt_in<kern>(kTcSmem);
    if (e != cudaSuccess) return e;
    return launch_overlapped(kern, grid, dim3(kTcRows), kTcSmem, s, dp, q_indptr, max_q_len);
}

}  // namespace

cudaError_t launch_extend_tc(const DecodeParams& dp, const int32_t* q_indptr, int max_q_len, cudaStream_t s) {
    const int G = dp.g.Hq / dp.g.H;
    const int qb = kTcRows / G;
    const dim3 grid((max_q_len + qb - 1) / qb, dp.g.H, dp.a.batch);
    switch (G) {
        case 1: return launch_g<1>(dp, q_indptr, max_q_len, grid, s);
        case 2: return launch_g<2>(dp, q_indptr, max_q_len, grid, s);
        case 4: return launch_g<4>(dp, q_indptr, max_q_len, grid, s);
        case 8: return launch_g<8>(dp, q_indptr, max_q_len, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvq
