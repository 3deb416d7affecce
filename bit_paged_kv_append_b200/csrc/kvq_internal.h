// kvq_internal.h -- host-side view of libkvq.so's kernels: parameter blocks and
// launchers shared between the C-ABI layer (kvq_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kvq {

constexpr int kHeadDim = 128;

struct CacheGeom {
    int num_pages, page_size, H, Hq, D, mode, bdr_block, rotate_v;
    void* k_pool;
    void* v_pool;
    uint32_t* k_sz;  // (scale, zero) fp16 pairs as one 32-bit word, scale in the low half
    uint32_t* v_sz;
    const float* rope;   // (cos, sin) [rope_positions][D/2][2], or nullptr
    int rope_positions;
    int code_bits;       // INT4 modes: 4 or 2 (codes per byte: 8 / code_bits)
};

struct AppendArgs {
    const void* k;
    const void* v;
    int num_tokens;
    const int32_t* tok_seq;
    const int32_t* tok_pos;
    const int32_t* page_table;
    int pt_stride;
    int num_seqs;
};

struct DecodeArgs {
    const void* q;
    const int32_t* seq_lens;
    const int32_t* page_table;
    int pt_stride;
    int batch;
    int max_seq_len;
    void* out;
    int out_fp32;
    void* workspace;
    size_t workspace_bytes;
};

struct ExtendArgs {
    const void* q;
    const int32_t* q_indptr;  // [batch + 1]: queries of sequence s are rows q_indptr[s] .. q_indptr[s + 1] - 1
    const int32_t* seq_lens;
    const int32_t* page_table;
    int pt_stride;
    int batch;
    int max_q_len;
    int max_seq_len;
    void* out;
    int out_fp32;
};

// Split-K plan for one decode call: cached tokens per work item, the bound on
// items per sequence and in total, and the workspace they need.
struct DecodePlan {
    int item_tokens;
    int max_splits;
    int max_items;
    int num_sms;
    size_t ws_bytes;
};

DecodePlan plan_decode(const CacheGeom& g, int batch, int max_seq_len, int num_sms);

// Each returns cudaSuccess or the first launch error.
cudaError_t launch_append(const CacheGeom& g, const AppendArgs& a, int* err_word, int num_sms, cudaStream_t s);
cudaError_t launch_decode(const CacheGeom& g, const DecodeArgs& a, const DecodePlan& plan, int* err_word,
                          cudaStream_t s);
// INT4 modes only (the caller rejects BF16 pages); kvq_extend_tc.cu.
cudaError_t launch_extend(const CacheGeom& g, const ExtendArgs& a, int* err_word, cudaStream_t s);

// Makes the handle's device current for the duration of one C-ABI call (and restores the
// caller's device afterwards), so that launches, function attributes and symbol lookups
// all refer to the device the cache's pools live on.
class DeviceGuard {
  public:
    explicit DeviceGuard(int device) : prev_(-1) {
        int cur = -1;
        ok_ = cudaGetDevice(&cur) == cudaSuccess;
        if (ok_ && cur != device) {
            ok_ = cudaSetDevice(device) == cudaSuccess;
            if (ok_) prev_ = cur;
        }
    }
    ~DeviceGuard() {
        if (prev_ >= 0) cudaSetDevice(prev_);
    }
    bool ok() const { return ok_; }
    DeviceGuard(const DeviceGuard&) = delete;
    DeviceGuard& operator=(const DeviceGuard&) = delete;

  private:
    int prev_;
    bool ok_;
};

}  // namespace kvq

// The opaque handle of include/kvq.h (the only definition: kvq_api.cu and kvq_noalloc.cu
// both use this one).
struct kv_cache {
    kvq::CacheGeom g;
    int* err_dev;  // device error word (bit flags, see kvq_common.cuh)
    int device;    // the device current at kv_create_paged: every call runs there
    int num_sms;
};
