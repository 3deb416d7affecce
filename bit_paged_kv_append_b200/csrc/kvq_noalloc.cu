// kvq_noalloc.cu -- kv_decode_attn_noalloc: decode attention whose split-K
// scratch lives in a fixed, library-owned device array instead of a
// caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the point where
// they decode -- code running inside a custom allocator or memory pool that
// must not re-enter itself, runtimes that hand out a fixed memory budget up
// front and forbid allocation afterwards, and plain-C hosts that have no
// device allocator of their own (no torch, no caching allocator) and do not
// want a cudaMalloc / cudaFree pair around every call.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes
// (KV_NOALLOC_SCRATCH_BYTES in kvq.h).  Every GPU that loads this library
// holds it until the process exits.  In host code the array's name is only a
// host-side stand-in, so its device address is obtained once per device with
// cudaGetSymbolAddress (on the first call for a handle on that device, which the call
// makes current while it runs)
// and then passed to the kernels like any workspace pointer.  Nothing in the
// scratch has to start at zero: the split kernel writes every partial result
// the merge kernel reads, on every call.  All calls share the one array, so
// calls whose kernels overlap on the GPU (different streams, or threads
// without ordering) race on it and must be serialised by the caller.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kvq.h"
#include "kvq_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = KV_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on `device`, which must be current (looked up once
// per device, under a lock); nullptr on failure.
void* scratch_address(int device) {
    if (device < 0 || device >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[device]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[device] = ptr;
    }
    return g_scratch_addr[device];
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" kv_status kv_decode_attn_noalloc(kv_cache* c, const void* q, const int32_t* seq_lens,
                                            const int32_t* page_table, int pt_stride, int batch, int max_seq_len,
                                            void* out, int out_fp32, void* stream) {
    if (!c || batch < 0 || max_seq_len < 0) return KV_ERR_INVALID;
    if (batch == 0) return KV_OK;
    if (!q || !seq_lens || !page_table || !out || pt_stride < 1) return KV_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(seq_lens, 4) || !aligned(page_table, 4) || !aligned(out, 16))
        return KV_ERR_INVALID;
    const kvq::DecodePlan plan = kvq::plan_decode(c->g, batch, max_seq_len, c->num_sms);
    if (plan.ws_bytes > kNoAllocScratchBytes) return KV_ERR_SCRATCH_TOO_SMALL;
    // the handle's device, current while the address is looked up and the kernels launch
    kvq::DeviceGuard dg(c->device);
    if (!dg.ok()) return KV_ERR_CUDA;
    void* scratch = scratch_address(c->device);
    if (!scratch) return KV_ERR_CUDA;
    kvq::DecodeArgs a{q, seq_lens, page_table, pt_stride, batch, max_seq_len, out, out_fp32 ? 1 : 0,
                      scratch, kNoAllocScratchBytes};
    cudaError_t e = kvq::launch_decode(c->g, a, plan, c->err_dev, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}
