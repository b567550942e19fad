// oam.cu -- top-K token selection of output-aware token dropping.
//
// "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse attention),
// section 3: tokens with the lowest OAM score are dropped and the top-K kept; one
// index set serves all G query heads of a KV head.  Ties are broken by the lower
// token index (total order: score descending, index ascending) and the kept
// positions are emitted in ascending order.  The scores themselves come from the
// score mode of the decode pipeline (decode.cu).
//
// One thread-block cluster of 8 CTAs per (KV head, sequence) row, each CTA holding
// an eighth of the row's keys in shared memory: an exact radix select of the K-th
// largest order-preserving 32-bit key in three digit passes (11, 11, 10 bits) with
// warp-aggregated shared-memory histograms merged across the cluster through
// distributed shared memory, then one pass in token order that keeps every key
// above the threshold and the first `need` keys equal to it, each CTA writing at
// its cluster-wide prefix offset.  Cluster barriers are hardware barriers: no
// spinning on flags.
#include <cooperative_groups.h>

#include "internal.h"
#include "scan.cuh"

namespace cg = cooperative_groups;

namespace sgd {

__device__ __forceinline__ uint32_t score_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int32_t kept_of(int32_t L, int keep_num, int keep_den) {
    int64_t k = ((int64_t)L * keep_num + keep_den - 1) / keep_den;
    if (k < 1) k = 1;
    if (k > L) k = L;
    return (int32_t)k;
}

constexpr int kTopkCluster = 8;      // CTAs per (sequence, KV head) row
constexpr int kTopkThreads = 1024;
constexpr int kTopkCap = 16384;      // keys per CTA staged in shared memory (64 KB)

// One thread-block cluster per row; CTA `rank` owns the contiguous chunk
// [rank*C, (rank+1)*C) of the row's tokens, C = ceil(L / kTopkCluster).
__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkThreads)
    topk_cluster_kernel(const float *__restrict__ scores, const int32_t *__restrict__ cu, int B, int64_t T,
                        int keep_num, int keep_den, int32_t *__restrict__ idx, int32_t *__restrict__ cu_kept,
                        int64_t Kt, int32_t *status) {
    extern __shared__ uint32_t skeys[];  // [kTopkCap]
    __shared__ uint32_t hist[2048];
    __shared__ int32_t sm[33];
    __shared__ uint32_t sel[2];
    __shared__ int32_t cnt[2];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31;
    const int r = blockIdx.x / kTopkCluster, kvh = r / B, b = r % B;
    const int32_t L = cu[b + 1] - cu[b];

    // output offset of this sequence: sum of the kept counts of the sequences before it
    int32_t mine = 0;
    for (int bb = tid; bb < b; bb += blockDim.x) mine += kept_of(max(cu[bb + 1] - cu[bb], 1), keep_num, keep_den);
    int32_t off;
    block_exclusive_scan(mine, off, sm);
    // the two early exits depend on the row only, so every CTA of the cluster takes them together
    if (L < 1) {
        if (rank == 0 && tid == 0) atomicOr(status, SGD_STATUS_EMPTY_SEQUENCE);
        return;
    }
    const int32_t K = kept_of(L, keep_num, keep_den);
    if (kvh == 0 && rank == 0 && tid == 0) {
        cu_kept[b + 1] = off + K;
        if (b == 0) cu_kept[0] = 0;
    }
    if (off + (int64_t)K > Kt) {
        if (rank == 0 && tid == 0) atomicOr(status, SGD_STATUS_SIZE_MISMATCH);
        return;
    }
    const int32_t C = (L + kTopkCluster - 1) / kTopkCluster;
    const int32_t lo = min(rank * C, L), n = min(lo + C, L) - lo;
    const float *s = scores + (int64_t)kvh * T + cu[b] + lo;
    for (int32_t i = tid; i < min(n, kTopkCap); i += blockDim.x) skeys[i] = score_key(__ldg(s + i));
    __syncthreads();
    auto key_at = [&](int32_t i) -> uint32_t { return i < kTopkCap ? skeys[i] : score_key(__ldg(s + i)); };

    uint32_t prefix = 0, mask = 0;
    int32_t rem = K;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < nb; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        for (int32_t base = 0; base < n; base += blockDim.x) {
            const int32_t i = base + tid;
            uint32_t bin = 0xffffffffu;
            if (i < n) {
                const uint32_t key = key_at(i);
                if ((key & mask) == prefix) bin = (key >> shift) & (uint32_t)(nb - 1);
            }
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (bin != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
        }
        cluster.sync();  // every CTA's histogram of this pass is complete
        // merged counts of the bins this thread owns, in descending bin order
        const int per = nb / blockDim.x;
        uint32_t mc[2] = {0u, 0u};
        for (int i = 0; i < per; ++i) {
            const int j = nb - 1 - (tid * per + i);
#pragma unroll
            for (int rr = 0; rr < kTopkCluster; ++rr) mc[i] += cluster.map_shared_rank(hist, rr)[j];
        }
        int32_t tot;
        int32_t above = block_exclusive_scan((int32_t)(mc[0] + mc[1]), tot, sm);
        for (int i = 0; i < per; ++i) {
            const int j = nb - 1 - (tid * per + i);
            const int32_t h = (int32_t)mc[i];
            if (above < rem && rem <= above + h) {
                sel[0] = (uint32_t)j;
                sel[1] = (uint32_t)above;
            }
            above += h;
        }
        __syncthreads();
        rem -= (int32_t)sel[1];
        prefix |= sel[0] << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        cluster.sync();  // remote histograms read before the next pass clears them
    }
    // keys > thr: K - need of them; keys == thr: the first `need` in token order are kept
    const uint32_t thr = prefix;
    const int32_t need = rem;
    int32_t my_gt = 0, my_eq = 0;
    for (int32_t i = tid; i < n; i += blockDim.x) {
        const uint32_t key = key_at(i);
        my_gt += key > thr;
        my_eq += key == thr;
    }
    int32_t tot_gt, tot_eq;
    block_exclusive_scan(my_gt, tot_gt, sm);
    block_exclusive_scan(my_eq, tot_eq, sm);
    if (tid == 0) {
        cnt[0] = tot_gt;
        cnt[1] = tot_eq;
    }
    cluster.sync();
    int32_t written = 0, eq_seen = 0;  // over the chunks before this one
    for (int rr = 0; rr < rank; ++rr) {
        const int32_t *rc = cluster.map_shared_rank(cnt, rr);
        const int32_t g = rc[0], e = rc[1];
        written += g + min(max(need - eq_seen, 0), e);
        eq_seen += e;
    }
    cluster.sync();  // no CTA leaves while another still reads its counts
    int32_t *out = idx + (int64_t)kvh * Kt + off;
    for (int32_t base = 0; base < n; base += blockDim.x * 8) {
        const int32_t t0 = base + tid * 8;
        uint32_t gtm = 0, eqm = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int32_t t = t0 + i;
            if (t < n) {
                const uint32_t key = key_at(t);
                if (key > thr) gtm |= 1u << i;
                else if (key == thr) eqm |= 1u << i;
            }
        }
        int32_t te, tk;
        int32_t eq_before = block_exclusive_scan(__popc(eqm), te, sm) + eq_seen;
        uint32_t keep = gtm;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (eqm & (1u << i)) {
                if (eq_before < need) keep |= 1u << i;
                ++eq_before;
            }
        int32_t pos = block_exclusive_scan(__popc(keep), tk, sm) + written;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (keep & (1u << i)) {
                if (pos < K) out[pos] = lo + t0 + i;
                ++pos;
            }
        written += tk;
        eq_seen += te;
    }
    if (rank == kTopkCluster - 1 && tid == 0 && written != K) atomicOr(status, SGD_STATUS_SIZE_MISMATCH);
}

int launch_topk(const float *scores, const int32_t *cu, int B, int Hkv, int64_t T, int keep_num, int keep_den,
                int32_t *idx, int32_t *cu_kept, int64_t kept_total, int32_t *status, cudaStream_t s) {
    const int smem = kTopkCap * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    topk_cluster_kernel<<<B * Hkv * kTopkCluster, kTopkThreads, smem, s>>>(scores, cu, B, T, keep_num, keep_den, idx,
                                                                           cu_kept, kept_total, status);
    return (int)cudaGetLastError();
}

}  // namespace sgd
