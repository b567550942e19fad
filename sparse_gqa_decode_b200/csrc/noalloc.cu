// noalloc.cu -- sgd_decode_attn_noalloc: the split-KV decode for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: a plugin hosted by a framework
// that owns every byte of device memory and exposes no allocator to its plugins, or a
// latency-critical loop that may not call cudaMalloc because it can synchronise the whole
// device and has no bounded latency.  This entry point runs the same plan, decode and merge
// kernels as sgd_decode_attn, with their scratch (plan arrays, per-chunk partial outputs and
// log-sum-exps, status word) placed in one file-scope device array instead of a caller
// workspace.  It calls no cudaMalloc, cudaFree or other allocating routine.
//
// The array is SGD_NOALLOC_SCRATCH_BYTES long; every GPU that loads the library holds its own
// copy until the process exits.  All calls on a device share that copy, and it keeps the
// previous call's contents, so calls whose GPU work overlaps (for example calls issued on two
// streams of one device) race on it: serialise them.
#include <mutex>

#include "internal.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[SGD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
void *g_scratch_addr[kMaxDev];  // device address of g_noalloc_scratch, per device
std::mutex g_scratch_mu;

// The name g_noalloc_scratch is a host-side stand-in in host code, not a device address:
// the address is looked up once per device, with that device current.
int scratch_address(void **addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return SGD_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SGD_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return SGD_OK;
}

}  // namespace

extern "C" int sgd_decode_attn_noalloc(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv,
                                       const int32_t *idx, const int32_t *cu_kept, int64_t kept_total,
                                       int schedule, int n_splits, int q_quant, float *out, float *lse, int32_t *status,
                                       void *stream) {
    void *scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != SGD_OK) return rc;
    const size_t need = sgd_workspace_size(SGD_OP_DECODE, kv, G, schedule, n_splits);
    if (need > SGD_NOALLOC_SCRATCH_BYTES) return SGD_ERR_SCRATCH_LIMIT;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return SGD_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The previous call's header is still in the array.  Nothing needs clearing here: the plan
    // kernel, the first launch of the decode, zeroes the status word and the per-row counters
    // before any other kernel of the call reads them, and a call rejected on the host launches
    // nothing at all.
    rc = sgd_decode_attn(q, q_dtype, G, kv, idx, cu_kept, kept_total, schedule, n_splits, q_quant, out, lse,
                         scratch, SGD_NOALLOC_SCRATCH_BYTES, stream);
    if (rc == SGD_OK && status) {
        if (cudaMemcpyAsync(status, static_cast<uint8_t *>(scratch) + SGD_WS_STATUS_OFFSET, sizeof(int32_t),
                            cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return SGD_ERR_CUDA;
    }
    return rc;
}
