// stream.cu -- sgd_stream_read: a read-only HBM streaming kernel, the ceiling the decode's
// mostly-read traffic is measured against (a copy moves as many bytes out as in, so its rate
// understates what a pure read stream reaches).
//
// Two ways of reading, both reducing every byte they read into one 64-bit word so that nothing
// can be elided:
//   method 0: every thread issues 16-byte loads (L1 bypassed), eight in flight per thread,
//             grid-stride over the buffer, XOR-reduced in registers;
//   method 1: one thread per CTA streams 32 KB chunks with bulk asynchronous copies
//             (cp.async.bulk) into a ring of shared-memory stages; each landed chunk is folded
//             into the word by the CTA's warp before the stage is refilled.
// Each CTA XORs its word into sink[0].
//
// sgd_gather_read, the same measurement for scattered rows: the rows a kept-token decode reads
// (one K row and one V row of codes per kept token), by a row index, 16-byte loads from every
// thread with the indices of a batch loaded before its rows.
#include "internal.h"

namespace sgd {

constexpr int kStreamUnroll = 8;
constexpr int kBulkChunk = 32 * 1024;
constexpr int kBulkStages = 6;

__global__ void __launch_bounds__(512) stream_vec_kernel(const uint4 *__restrict__ p, int64_t n,
                                                         unsigned long long *sink) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    uint32_t acc = 0u;
    for (; i + (kStreamUnroll - 1) * stride < n; i += kStreamUnroll * stride) {
        uint4 w[kStreamUnroll];
#pragma unroll
        for (int u = 0; u < kStreamUnroll; ++u) w[u] = __ldcs(p + i + u * stride);
#pragma unroll
        for (int u = 0; u < kStreamUnroll; ++u) acc ^= w[u].x ^ w[u].y ^ w[u].z ^ w[u].w;
    }
    for (; i < n; i += stride) {
        const uint4 w = __ldcs(p + i);
        acc ^= w.x ^ w.y ^ w.z ^ w.w;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0 && acc) atomicXor(sink, (unsigned long long)acc);
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// One warp per CTA.  Lane 0 issues; after a stage's chunk lands the warp folds it (each lane 32
// 16-byte words of the 32 KB, so every byte is read) and lane 0 refills the stage.
__global__ void __launch_bounds__(32) stream_bulk_kernel(const uint8_t *__restrict__ p, int64_t n_chunks,
                                                         int64_t bytes, unsigned long long *sink,
                                                         int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *buf = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t *full = reinterpret_cast<uint64_t *>(buf + kBulkStages * kBulkChunk);
    volatile int32_t *abort_flag = reinterpret_cast<int32_t *>(full + kBulkStages);
    const int lane = threadIdx.x;
    if (lane == 0) {
        for (int s = 0; s < kBulkStages; ++s) mbar_init(&full[s], 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncwarp();
    auto issue = [&](int64_t c, int s) {
        const int64_t off = c * kBulkChunk;
        const uint32_t len = (uint32_t)(bytes - off < kBulkChunk ? bytes - off : (int64_t)kBulkChunk);
        mbar_arrive_expect_tx(&full[s], len);
        bulk_load(buf + s * kBulkChunk, p + off, len, &full[s]);
    };
    // chunks of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int64_t first = blockIdx.x, step = gridDim.x;
    const int64_t mine = first < n_chunks ? (n_chunks - first + step - 1) / step : 0;
    int64_t issued = 0;  // chunks of this CTA issued so far (lane 0)
    if (lane == 0)
        for (; issued < kBulkStages && issued < mine; ++issued) issue(first + issued * step, (int)issued);
    uint32_t acc = 0u;
    bool ok = true;
    for (int64_t j = 0; j < mine; ++j) {
        const int s = (int)(j % kBulkStages);
        const uint32_t par = (uint32_t)((j / kBulkStages) & 1);
        ok = __all_sync(0xffffffffu, ok && mbar_wait(&full[s], par, status, abort_flag, kWaitLimit));
        if (ok) {
            const int64_t off = (first + j * step) * kBulkChunk;
            const int len = (int)(bytes - off < kBulkChunk ? bytes - off : (int64_t)kBulkChunk);
            const uint4 *w = reinterpret_cast<const uint4 *>(buf + s * kBulkChunk);
#pragma unroll 8
            for (int e = lane; e < len / 16; e += 32) {
                const uint4 x = w[e];
                acc ^= x.x ^ x.y ^ x.z ^ x.w;
            }
        }
        __syncwarp();
        if (lane == 0 && ok && issued < mine) {
            fence_proxy_async_shared();
            issue(first + issued * step, s);  // issued == j + kBulkStages: the stage just read
            ++issued;
        }
        if (!ok) break;
    }
    // nothing may still be landing when the CTA ends (only after a wait that gave up): the
    // chunks issued but not yet waited for are the last kBulkStages at most
    if (lane == 0 && !ok) {
        for (int64_t j = (issued > kBulkStages ? issued - kBulkStages : 0); j < issued; ++j)
            mbar_drain(&full[j % kBulkStages], (uint32_t)((j / kBulkStages) & 1), kWaitLimit);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0 && acc) atomicXor(sink, (unsigned long long)acc);
}

constexpr int kGatherUnroll = 8;

// Item i of the gather: chunk c (16 bytes) of tensor t (0: a, 1: b) of listed row j, with
// i = (j * nt + t) * C + c, so consecutive threads read consecutive chunks of one row.  C = 2^lc
// chunks per row and nt = 2^lt tensors, so the split is shifts and masks.
__global__ void __launch_bounds__(512) gather_read_kernel(const uint8_t *__restrict__ a, const uint8_t *__restrict__ b,
                                                          int64_t row_bytes, const int32_t *__restrict__ rows,
                                                          int64_t n_items, int lc, int lt, unsigned long long *sink) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t acc = 0u;
    for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i0 < n_items; i0 += kGatherUnroll * stride) {
        int32_t r[kGatherUnroll];
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) {  // every index of the batch first
            const int64_t i = i0 + u * stride;
            r[u] = (i < n_items) ? __ldg(rows + (i >> (lc + lt))) : 0;
        }
        uint4 w[kGatherUnroll];
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) {
            const int64_t i = i0 + u * stride;
            w[u] = make_uint4(0u, 0u, 0u, 0u);
            if (i < n_items) {
                const int c = (int)(i & ((1 << lc) - 1)), t = (int)((i >> lc) & ((1 << lt) - 1));
                const uint8_t *base = t ? b : a;
                w[u] = __ldcs(reinterpret_cast<const uint4 *>(base + (int64_t)r[u] * row_bytes) + c);
            }
        }
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) acc ^= w[u].x ^ w[u].y ^ w[u].z ^ w[u].w;
    }
    // one atomic per CTA (a small read must not wait on thousands of same-address atomics)
    __shared__ uint32_t part[16];
#pragma unroll
    for (int o = 16; o; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t x = 0u;
        for (int k = 0; k < (int)(blockDim.x >> 5); ++k) x ^= part[k];
        if (x) atomicXor(sink, (unsigned long long)x);
    }
}

int launch_gather_read(const void *a, const void *b, int64_t row_bytes, const int32_t *rows, int64_t n_rows,
                       unsigned long long *sink, int sm_count, cudaStream_t s) {
    int per = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, gather_read_kernel, 512, 0) != cudaSuccess || per < 1)
        per = 2;
    const int lt = b ? 1 : 0;
    int lc = 0;
    while ((int64_t(16) << lc) < row_bytes) ++lc;  // row_bytes = 16 * 2^lc (checked by the caller)
    const int64_t n_items = n_rows << (lc + lt);
    return (int)launch_k(gather_read_kernel, dim3(sm_count * per), dim3(512), 0, s, 1,
                         static_cast<const uint8_t *>(a), static_cast<const uint8_t *>(b), row_bytes, rows, n_items,
                         lc, lt, sink);
}

int launch_stream_read(const void *buf, size_t bytes, int method, unsigned long long *sink, int32_t *status,
                       int sm_count, cudaStream_t s) {
    if (method == 0) {
        int per = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, stream_vec_kernel, 512, 0) != cudaSuccess || per < 1)
            per = 2;
        return (int)launch_k(stream_vec_kernel, dim3(sm_count * per), dim3(512), 0, s, 1,
                             static_cast<const uint4 *>(buf), (int64_t)(bytes / 16), sink);
    }
    const size_t smem = 128 + (size_t)kBulkStages * kBulkChunk + kBulkStages * 8 + 16;
    cudaError_t e = cudaFuncSetAttribute(stream_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    const int64_t n_chunks = (int64_t)((bytes + kBulkChunk - 1) / kBulkChunk);
    return (int)launch_k(stream_bulk_kernel, dim3(sm_count), dim3(32), smem, s, 1,
                         static_cast<const uint8_t *>(buf), n_chunks, (int64_t)bytes, sink, status);
}

}  // namespace sgd
