// common.cuh -- device helpers shared by the sm_100a kernels of libsgd.so:
// inline-PTX wrappers for mbarriers, TMA (cp.async.bulk.tensor), cp.async,
// warp-level MMA fragments, and the internal launch interface.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/sgd.h"

namespace sgd {

// ------------------------------------------------------------------------------------------
// workspace header (first 256 bytes of every workspace)
// ------------------------------------------------------------------------------------------
struct WsHeader {
    int32_t status;       // SGD_STATUS_* bits, offset SGD_WS_STATUS_OFFSET
    int32_t pad0;
    uint32_t amax_bits[2];  // quantize: running max |K|, max |V| as float bits
    int64_t plan_W;       // plan: padded stream length
    int64_t plan_S;       // plan: CTA range length
    int32_t plan_ncta;    // plan: CTAs with work
    int32_t plan_nslots;  // plan: segments (partial results)
    int32_t n_parts;      // quantize/decode: partitions counted on the device
    float q_scale;        // decode with a per-tensor query scale: max|q| / 127
    int32_t pad1[52];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr int kGranule = 16;      // plan granularity (tokens)
constexpr int kMaxColGroups = 4;  // decode columns per KV head up to 4 x 16 (M * G <= 64)
constexpr int kPart = SGD_PARTITION;
constexpr long long kWaitLimit = 1 << 22;  // bounded mbarrier polls before giving up

__host__ __device__ inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// Per-launch timing (sgd_kernel_timing_start / _stop, api.cu): while it is on, every launch is
// bracketed by a pair of events on its stream.  kt_begin returns the launch's slot or -1.
int kt_begin(cudaStream_t s);
void kt_end(cudaStream_t s, int slot, const void *kern);

// ------------------------------------------------------------------------------------------
// host: launch `kern` through cudaLaunchKernelEx, as clusters of `cluster` CTAs along x when
// cluster > 1.  Returns the launch's cudaError_t.
// ------------------------------------------------------------------------------------------
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k_raw(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                unsigned cluster, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    unsigned n = 0;
    if (cluster > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        n = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            unsigned cluster, Args &&...args) {
    const int slot = kt_begin(s);
    const cudaError_t e = launch_k_raw(kern, grid, block, smem, s, cluster, std::forward<Args>(args)...);
    if (slot >= 0) kt_end(s, slot, reinterpret_cast<const void *>(kern));
    return e;
}

// ------------------------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity.  Every wait is bounded: after `limit` polls
// (kWaitLimit unless a test lowers it) the wait records SGD_STATUS_WAIT_TIMEOUT, raises the
// CTA's abort flag and returns false.  Once the flag is up every later wait of the CTA returns
// false at once, so all warps still run through the same (named) barriers and the kernel ends
// promptly instead of hanging.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int32_t *status,
                                          volatile int32_t *abort_flag, long long limit) {
    if (*abort_flag) return false;
    for (long long i = 0; i < limit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023) == 1023 && *abort_flag) return false;
    }
    *abort_flag = 1;
    atomicOr(status, SGD_STATUS_WAIT_TIMEOUT);
    return false;
}

// Bounded wait for a phase that a copy this thread issued completes, regardless of the abort
// flag: a producer calls it before it exits so that no copy is still writing into the CTA's
// shared memory when the CTA ends.  False if the limit ran out.
__device__ __forceinline__ bool mbar_drain(uint64_t *bar, uint32_t parity, long long limit) {
    for (long long i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Orders this thread's generic-proxy shared-memory accesses before later async-proxy ones (a
// stage read by the threads, then refilled by TMA or a bulk copy).
__device__ __forceinline__ void fence_proxy_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled TMA load of one box into shared memory, completing on `bar` (tx bytes).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 16-byte asynchronous global -> shared copy (L2 only), and its completion signal.
__device__ __forceinline__ void cp_async_16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Waits until every cp.async this thread issued has landed in shared memory.
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
    return r;
}

__device__ __forceinline__ void sts64(uint32_t addr, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(x), "r"(y) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(addr));
    return r;
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// D += A(16x16, row) * B(16x8, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A(16x32, s8) * B(32x8, s8), int32 accumulation
__device__ __forceinline__ void mma_s8(int32_t (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Four signed bytes -> two f16x2 (exact).  Each byte b is biased to u = b ^ 0x80 = b + 128,
// placed under the f16 exponent of 1024 (bits 0x64uu = 1024 + u, exact because f16 has a
// 10-bit mantissa), and 1152 = 1024 + 128 is subtracted.
__device__ __forceinline__ void s8x4_to_f16x2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
    const uint32_t u = w ^ 0x80808080u;
    lo = __byte_perm(u, 0x64646464u, 0x4140);  // bytes [u0, 0x64, u1, 0x64]
    hi = __byte_perm(u, 0x64646464u, 0x4342);  // bytes [u2, 0x64, u3, 0x64]
    const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
    __half2 l = __hsub2(*reinterpret_cast<__half2 *>(&lo), bias);
    __half2 h = __hsub2(*reinterpret_cast<__half2 *>(&hi), bias);
    lo = *reinterpret_cast<uint32_t *>(&l);
    hi = *reinterpret_cast<uint32_t *>(&h);
}

// Two already-biased bytes (u = b ^ 0x80) sitting in byte lanes `sel` of (a, b) -> f16x2.
__device__ __forceinline__ uint32_t biased_pair_to_f16x2(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t x = __byte_perm(a, b, sel);                 // bytes [ua, ub, *, *] in lanes 0, 1
    x = __byte_perm(x, 0x64646464u, 0x4140);             // [ua, 0x64, ub, 0x64]
    const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
    __half2 r = __hsub2(*reinterpret_cast<__half2 *>(&x), bias);
    return *reinterpret_cast<uint32_t *>(&r);
}

// max(|lo|, |hi|) of a running bf16x2 maximum folded into float (bf16 values are exact in float)
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t m, uint32_t w) {
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&w), b = *reinterpret_cast<__nv_bfloat162 *>(&m);
    __nv_bfloat162 r = __hmax2(__habs2(a), b);
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ float bf16x2_fold_max(uint32_t m) {
    return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
}

// ss += lo(w)^2 + hi(w)^2 for the two bf16 of w, as a packed f32x2 FMA on (even, odd) partial sums
__device__ __forceinline__ uint64_t bf16x2_sumsq(uint64_t acc, uint32_t w) {
    const uint64_t x = (uint64_t)(w << 16) | ((uint64_t)(w & 0xffff0000u) << 32);
    asm("fma.rn.f32x2 %0, %1, %1, %0;" : "+l"(acc) : "l"(x));
    return acc;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------------------------------------
// internal launch interface (host side)
// ------------------------------------------------------------------------------------------
struct RowInfo {        // per-row record written by the plan kernel (32 bytes)
    int32_t pos;        // padded stream position of the row
    int32_t len;        // attended tokens (kept count, or the sequence length)
    int32_t seq_start;  // cu_seqlens[b]
    int32_t seq_len;    // sequence length
    int32_t len_start;  // start of the attended row (cu_kept[b], or cu_seqlens[b])
    int32_t part0;      // scheme-A partition offset of the sequence
    int32_t slot0;      // first partial slot of the row
    int32_t nseg;       // segments (partial results) of the row
};
static_assert(sizeof(RowInfo) == 32, "row record is two int4");

struct PlanView {  // device arrays of a plan inside a workspace
    int32_t *row_pos;    // [R+1] padded stream position of each row
    int32_t *row_slot0;  // [R+1] first partial slot of each row
    int32_t *cta_begin;  // [N+1] stream position where each CTA starts
    int32_t *cta_slot0;  // [N+1] first partial slot of each CTA
    int32_t *cta_row0;   // [N] first row each CTA range reaches (R for an empty range)
    RowInfo *row_info;   // [R] per-row record
    int32_t *row_done;   // [R] decode: segments of the row finished (zeroed by the plan kernel), or NULL
    int32_t *seq_part0;  // [B+1] scheme-A partition offset of each sequence
};

}  // namespace sgd
