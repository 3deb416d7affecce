// kvq_api.cu -- the C ABI of libkvq.so (declared in include/kvq.h): host-side
// validation, the opaque handle, the device error word, and dispatch to the
// append / decode / extend launchers.  No kernel is launched before every argument has
// been checked; nothing here allocates on the per-call path.
#include <cuda_runtime.h>
#include <stdint.h>

#include <new>

#include "kvq.h"
#include "kvq_internal.h"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" {

const char* kv_status_string(int status) {
    switch (status) {
        case KV_OK: return "KV_OK";
        case KV_ERR_INVALID: return "KV_ERR_INVALID";
        case KV_ERR_UNSUPPORTED: return "KV_ERR_UNSUPPORTED";
        case KV_ERR_CUDA: return "KV_ERR_CUDA";
        case KV_ERR_OOB: return "KV_ERR_OOB";
        case KV_ERR_TIMEOUT: return "KV_ERR_TIMEOUT";
        case KV_ERR_SCRATCH_TOO_SMALL: return "KV_ERR_SCRATCH_TOO_SMALL";
        default: return "KV_ERR_UNKNOWN";
    }
}

kv_status kv_create_paged(const kv_desc* d, kv_cache** out) {
    if (!d || !out) return KV_ERR_INVALID;
    *out = nullptr;
    if (d->num_pages < 1 || d->page_size < 1 || d->page_size > 1024) return KV_ERR_INVALID;
    if (d->num_kv_heads < 1 || d->num_q_heads < 1 || d->num_q_heads % d->num_kv_heads) return KV_ERR_INVALID;
    if (d->head_dim != kvq::kHeadDim) return KV_ERR_UNSUPPORTED;
    if (32 % d->num_kv_heads) return KV_ERR_UNSUPPORTED;
    const int G = d->num_q_heads / d->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return KV_ERR_UNSUPPORTED;
    if (d->mode < KV_BF16 || d->mode > KV_INT4_BDR) return KV_ERR_INVALID;
    if (d->mode == KV_INT4_BDR && d->bdr_block != 16 && d->bdr_block != 32 && d->bdr_block != 64 &&
        d->bdr_block != 128)
        return KV_ERR_UNSUPPORTED;
    if (!d->k_pool || !d->v_pool || !aligned(d->k_pool, 32) || !aligned(d->v_pool, 32)) return KV_ERR_INVALID;
    if (d->mode != KV_BF16 && (!d->k_sz || !d->v_sz || !aligned(d->k_sz, 16) || !aligned(d->v_sz, 16)))
        return KV_ERR_INVALID;
    if (d->rope && (d->rope_positions < 1 || !aligned(d->rope, 16))) return KV_ERR_INVALID;
    const int code_bits = d->code_bits == 0 ? 4 : d->code_bits;
    if (code_bits != 4 && code_bits != 2) return KV_ERR_UNSUPPORTED;
    if (code_bits == 2 && d->mode == KV_BF16) return KV_ERR_INVALID;
    const int64_t rows = int64_t(d->num_pages) * d->num_kv_heads * d->page_size;
    if (rows >= (int64_t(1) << 32)) return KV_ERR_INVALID;  // slot indices are 32-bit in the kernels

    kv_cache* c = new (std::nothrow) kv_cache();
    if (!c) return KV_ERR_INVALID;
    c->g.num_pages = d->num_pages;
    c->g.page_size = d->page_size;
    c->g.H = d->num_kv_heads;
    c->g.Hq = d->num_q_heads;
    c->g.D = d->head_dim;
    c->g.mode = d->mode;
    c->g.bdr_block = d->mode == KV_INT4_BDR ? d->bdr_block : 0;
    c->g.rotate_v = d->mode == KV_INT4_BDR ? (d->rotate_v ? 1 : 0) : 0;
    c->g.k_pool = d->k_pool;
    c->g.v_pool = d->v_pool;
    c->g.k_sz = static_cast<uint32_t*>(d->mode == KV_BF16 ? nullptr : d->k_sz);
    c->g.v_sz = static_cast<uint32_t*>(d->mode == KV_BF16 ? nullptr : d->v_sz);
    c->g.rope = d->rope;
    c->g.rope_positions = d->rope ? d->rope_positions : 0;
    c->g.code_bits = d->mode == KV_BF16 ? 4 : code_bits;
    if (cudaGetDevice(&c->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess ||
        cudaMalloc(&c->err_dev, sizeof(int)) != cudaSuccess) {
        delete c;
        return KV_ERR_CUDA;
    }
    if (cudaMemset(c->err_dev, 0, sizeof(int)) != cudaSuccess) {
        cudaFree(c->err_dev);
        delete c;
        return KV_ERR_CUDA;
    }
    *out = c;
    return KV_OK;
}

kv_status kv_append_quant(kv_cache* c, const void* k, const void* v, int num_tokens, const int32_t* tok_seq,
                          const int32_t* tok_pos, const int32_t* page_table, int pt_stride, int num_seqs,
                          void* stream) {
    if (!c || num_tokens < 0) return KV_ERR_INVALID;
    if (num_tokens == 0) return KV_OK;
    if (!k || !v || !tok_seq || !tok_pos || !page_table) return KV_ERR_INVALID;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(tok_seq, 4) || !aligned(tok_pos, 4) ||
        !aligned(page_table, 4))
        return KV_ERR_INVALID;
    if (pt_stride < 1 || num_seqs < 1) return KV_ERR_INVALID;
    if (int64_t(num_tokens) * c->g.H > INT32_MAX) return KV_ERR_INVALID;  // rows index the TMA box as int32
    kvq::AppendArgs a{k, v, num_tokens, tok_seq, tok_pos, page_table, pt_stride, num_seqs};
    kvq::DeviceGuard dg(c->device);
    if (!dg.ok()) return KV_ERR_CUDA;
    cudaError_t e = kvq::launch_append(c->g, a, c->err_dev, c->num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

size_t kv_decode_workspace_bytes(const kv_cache* c, int batch, int max_seq_len) {
    if (!c || batch <= 0 || max_seq_len < 0) return 0;
    return kvq::plan_decode(c->g, batch, max_seq_len, c->num_sms).ws_bytes;
}

kv_status kv_decode_attn(kv_cache* c, const void* q, const int32_t* seq_lens, const int32_t* page_table,
                         int pt_stride, int batch, int max_seq_len, void* out, int out_fp32, void* workspace,
                         size_t workspace_bytes, void* stream) {
    if (!c || batch < 0 || max_seq_len < 0) return KV_ERR_INVALID;
    if (batch == 0) return KV_OK;
    if (!q || !seq_lens || !page_table || !out || pt_stride < 1) return KV_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(seq_lens, 4) || !aligned(page_table, 4) || !aligned(out, 16))
        return KV_ERR_INVALID;
    const kvq::DecodePlan plan = kvq::plan_decode(c->g, batch, max_seq_len, c->num_sms);
    if (!workspace || workspace_bytes < plan.ws_bytes || !aligned(workspace, 16)) return KV_ERR_INVALID;
    kvq::DecodeArgs a{q, seq_lens, page_table, pt_stride, batch, max_seq_len, out, out_fp32 ? 1 : 0,
                      workspace, workspace_bytes};
    kvq::DeviceGuard dg(c->device);
    if (!dg.ok()) return KV_ERR_CUDA;
    cudaError_t e = kvq::launch_decode(c->g, a, plan, c->err_dev, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

kv_status kv_extend_attn(kv_cache* c, const void* q, const int32_t* q_indptr, const int32_t* seq_lens,
                         const int32_t* page_table, int pt_stride, int batch, int max_q_len, int max_seq_len,
                         void* out, int out_fp32, void* stream) {
    if (!c || batch < 0 || max_q_len < 0 || max_seq_len < 0) return KV_ERR_INVALID;
    if (batch == 0 || max_q_len == 0) return KV_OK;
    if (!q || !q_indptr || !seq_lens || !page_table || !out || pt_stride < 1) return KV_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(q_indptr, 4) || !aligned(seq_lens, 4) || !aligned(page_table, 4) ||
        !aligned(out, 16))
        return KV_ERR_INVALID;
    if (c->g.mode == KV_BF16) return KV_ERR_UNSUPPORTED;
    if (batch > 65535) return KV_ERR_UNSUPPORTED;  // the grid's z extent
    kvq::ExtendArgs a{q, q_indptr, seq_lens, page_table, pt_stride, batch, max_q_len, max_seq_len, out,
                      out_fp32 ? 1 : 0};
    kvq::DeviceGuard dg(c->device);
    if (!dg.ok()) return KV_ERR_CUDA;
    cudaError_t e = kvq::launch_extend(c->g, a, c->err_dev, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

kv_status kv_get_error(kv_cache* c, void* stream) {
    if (!c) return KV_ERR_INVALID;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    kvq::DeviceGuard dg(c->device);
    if (!dg.ok()) return KV_ERR_CUDA;
    int h = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return KV_ERR_CUDA;
    if (cudaMemcpyAsync(&h, c->err_dev, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(c->err_dev, 0, sizeof(int), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
        return KV_ERR_CUDA;
    if (h & 2) return KV_ERR_TIMEOUT;
    if (h & 1) return KV_ERR_OOB;
    return KV_OK;
}

void kv_free(kv_cache* c) {
    if (!c) return;
    {
        kvq::DeviceGuard dg(c->device);
        cudaFree(c->err_dev);
    }
    delete c;
}

}  // extern "C"
