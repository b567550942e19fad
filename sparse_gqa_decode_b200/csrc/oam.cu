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
constexpr int kCandCap = 2048;       // candidates of the threshold bin gathered per row

__device__ __forceinline__ float key_score(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// One thread-block cluster per row; CTA `rank` owns the contiguous chunk
// [rank*C, (rank+1)*C) of the row's tokens, C = ceil(L / kTopkCluster).
//
// Threshold search.  Fast path: the cluster's min and max score bound the row; scores are
// binned linearly into 2048 bins between them (a monotonic map, so the K-th largest lies in
// the first bin, counted from the top, whose cumulative count reaches K); the keys of that bin
// (usually a few hundred) are gathered through distributed shared memory and ranked exactly.
// Fallback (every score equal, a non-finite range, or a threshold bin with more than
// kCandCap keys): exact radix select over the order-preserving keys in three digit passes
// (11, 11, 10 bits).  Either way: thr = the K-th largest key, need = how many keys equal to
// thr are kept (the lowest-index ones).
__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkThreads)
    topk_cluster_kernel(const float *__restrict__ scores, const int32_t *__restrict__ cu, int B, int64_t T,
                        int keep_num, int keep_den, int32_t *__restrict__ idx, int32_t *__restrict__ cu_kept,
                        int64_t Kt, int32_t *status) {
    extern __shared__ uint32_t skeys[];  // [kTopkCap]
    __shared__ uint32_t hist[2][2048];   // linear histogram (hist[0]); radix passes alternate buffers
    __shared__ uint32_t cand[kCandCap];  // this CTA's keys in the threshold bin
    __shared__ uint32_t allc[kCandCap];  // every CTA's keys in the threshold bin
    __shared__ int32_t sm[33];
    __shared__ uint32_t sel[2];
    __shared__ int32_t cnt[2];
    __shared__ uint32_t ext[2];          // this CTA's smallest and largest key
    __shared__ uint32_t wmin[32], wmax[32];
    __shared__ uint32_t ncand;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
    const int32_t ns = min(n, kTopkCap);
    uint32_t kmin = 0xffffffffu, kmax = 0u;  // neutral for an empty chunk
    for (int32_t base = 0; base < ns; base += blockDim.x * 4) {  // four independent loads in flight
        float x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int32_t i = base + u * blockDim.x + tid;
            x[u] = (i < ns) ? __ldg(s + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int32_t i = base + u * blockDim.x + tid;
            if (i < ns) {
                const uint32_t k = score_key(x[u]);
                skeys[i] = k;
                kmin = min(kmin, k);
                kmax = max(kmax, k);
            }
        }
    }
    for (int32_t i = kTopkCap + tid; i < n; i += blockDim.x) {  // keys beyond the shared-memory stage
        const uint32_t k = score_key(__ldg(s + i));
        kmin = min(kmin, k);
        kmax = max(kmax, k);
    }
    auto key_at = [&](int32_t i) -> uint32_t { return i < kTopkCap ? skeys[i] : score_key(__ldg(s + i)); };
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
        wmin[warp] = kmin;
        wmax[warp] = kmax;
    }
    for (int i = tid; i < 2048; i += blockDim.x) hist[0][i] = 0u;
    if (tid == 0) ncand = 0u;
    __syncthreads();
    if (tid == 0) {
        uint32_t a0 = 0xffffffffu, a1 = 0u;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            a0 = min(a0, wmin[w]);
            a1 = max(a1, wmax[w]);
        }
        ext[0] = a0;
        ext[1] = a1;
    }
    cluster.sync();  // (1) every CTA's key range is published
    uint32_t gmin = 0xffffffffu, gmax = 0u;
#pragma unroll
    for (int rr = 0; rr < kTopkCluster; ++rr) {
        const uint32_t *e = cluster.map_shared_rank(ext, rr);
        gmin = min(gmin, e[0]);
        gmax = max(gmax, e[1]);
    }
    const float smin = key_score(gmin), span = key_score(gmax) - smin;
    // the same decision in every CTA of the cluster
    bool fast = (gmin < gmax) && isfinite(span) && span > 0.f && isfinite(smin);
    const float bscale = fast ? 2048.f / span : 0.f;
    auto lin_bin = [&](uint32_t key) -> int {  // non-decreasing in the score
        const float v = (key_score(key) - smin) * bscale;
        return min(2047, max(0, (int)v));
    };

    uint32_t thr = 0u;
    int32_t need = 0;
    if (fast) {
        for (int32_t i = tid; i < n; i += blockDim.x) atomicAdd(&hist[0][lin_bin(key_at(i))], 1u);
        cluster.sync();  // (2) every CTA's linear histogram is complete
        const int j0 = 2047 - 2 * tid, j1 = j0 - 1;  // this thread's bins, in descending order
        uint32_t m0 = 0u, m1 = 0u;
#pragma unroll
        for (int rr = 0; rr < kTopkCluster; ++rr) {
            const uint32_t *hr = cluster.map_shared_rank(&hist[0][0], rr);
            m0 += hr[j0];
            m1 += hr[j1];
        }
        int32_t tot;
        int32_t above = block_exclusive_scan((int32_t)(m0 + m1), tot, sm);
        if (above < K && K <= above + (int32_t)m0) {
            sel[0] = (uint32_t)j0;
            sel[1] = (uint32_t)above;
        }
        above += (int32_t)m0;
        if (above < K && K <= above + (int32_t)m1) {
            sel[0] = (uint32_t)j1;
            sel[1] = (uint32_t)above;
        }
        __syncthreads();
        const int bstar = (int)sel[0];
        const int32_t rem = K - (int32_t)sel[1];  // keys still to take inside bin bstar
        __syncthreads();
        for (int32_t i = tid; i < n; i += blockDim.x) {  // this CTA's keys of bin bstar
            const uint32_t key = key_at(i);
            if (lin_bin(key) == bstar) {
                const uint32_t at = atomicAdd(&ncand, 1u);
                if (at < (uint32_t)kCandCap) cand[at] = key;
            }
        }
        cluster.sync();  // (3) every CTA's candidate list is complete
        uint32_t cnts[kTopkCluster], tot_c = 0;
#pragma unroll
        for (int rr = 0; rr < kTopkCluster; ++rr) {
            cnts[rr] = *cluster.map_shared_rank(&ncand, rr);
            tot_c += cnts[rr];
        }
        fast = tot_c <= (uint32_t)kCandCap;
        if (fast) {
            // one copy of every CTA's candidates in this CTA's shared memory
            for (uint32_t ci = tid; ci < tot_c; ci += blockDim.x) {
                int own = 0;
                uint32_t at = ci;
#pragma unroll
                for (int rr = 0; rr < kTopkCluster - 1; ++rr)
                    if (own == rr && at >= cnts[rr]) {
                        at -= cnts[rr];
                        own = rr + 1;
                    }
                allc[ci] = cluster.map_shared_rank(cand, own)[at];
            }
            __syncthreads();
            // exact rank of every candidate among all candidates; thr = the rem-th largest key
            for (uint32_t ci = tid; ci < tot_c; ci += blockDim.x) {
                const uint32_t key = allc[ci];
                int32_t gt = 0, ge = 0;
                for (uint32_t i = 0; i < tot_c; ++i) {
                    const uint32_t o = allc[i];
                    gt += o > key;
                    ge += o >= key;
                }
                if (gt < rem && rem <= ge) {  // every candidate equal to thr writes the same values
                    sel[0] = key;
                    sel[1] = (uint32_t)(rem - gt);
                }
            }
        }
        __syncthreads();
        if (fast) {
            thr = sel[0];
            need = (int32_t)sel[1];
        }
        __syncthreads();  // sel may be rewritten by the radix path
    }
    if (!fast) {
        // exact radix select over the order-preserving keys (hist[1], hist[0], hist[1]: a buffer
        // is cleared only after every CTA has passed the cluster barrier that follows its last read)
        uint32_t prefix = 0, mask = 0;
        int32_t rem = K;
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const int nb = pass == 2 ? 1024 : 2048;
            uint32_t *h = hist[(pass + 1) & 1];
            for (int i = tid; i < nb; i += blockDim.x) h[i] = 0u;
            __syncthreads();
            for (int32_t base = 0; base < n; base += blockDim.x) {
                const int32_t i = base + tid;
                uint32_t bin = 0xffffffffu;
                if (i < n) {
                    const uint32_t key = key_at(i);
                    if ((key & mask) == prefix) bin = (key >> shift) & (uint32_t)(nb - 1);
                }
                const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                if (bin != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&h[bin], (uint32_t)__popc(peers));
            }
            cluster.sync();  // every CTA's histogram of this pass is complete
            int32_t tot, above;
            if (nb == 2048) {
                const int j0 = nb - 1 - 2 * tid;
                uint32_t a0 = 0u, a1 = 0u;
#pragma unroll
                for (int rr = 0; rr < kTopkCluster; ++rr) {
                    const uint32_t *hr = cluster.map_shared_rank(h, rr);
                    a0 += hr[j0];
                    a1 += hr[j0 - 1];
                }
                above = block_exclusive_scan((int32_t)(a0 + a1), tot, sm);
                if (above < rem && rem <= above + (int32_t)a0) {
                    sel[0] = (uint32_t)j0;
                    sel[1] = (uint32_t)above;
                }
                above += (int32_t)a0;
                if (above < rem && rem <= above + (int32_t)a1) {
                    sel[0] = (uint32_t)(j0 - 1);
                    sel[1] = (uint32_t)above;
                }
            } else {
                const int j0 = nb - 1 - tid;
                uint32_t a0 = 0u;
#pragma unroll
                for (int rr = 0; rr < kTopkCluster; ++rr) a0 += cluster.map_shared_rank(h, rr)[j0];
                above = block_exclusive_scan((int32_t)a0, tot, sm);
                if (above < rem && rem <= above + (int32_t)a0) {
                    sel[0] = (uint32_t)j0;
                    sel[1] = (uint32_t)above;
                }
            }
            __syncthreads();
            rem -= (int32_t)sel[1];
            prefix |= sel[0] << shift;
            mask |= (uint32_t)(nb - 1) << shift;
            __syncthreads();  // sel is rewritten by the next pass
        }
        thr = prefix;
        need = rem;
    }
    // keys > thr: K - need of them; keys == thr: the first `need` in token order are kept
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
    // all of the SM's unified L1/shared memory as shared: two 1024-thread CTAs per SM, one wave
    e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return (int)e;
    topk_cluster_kernel<<<B * Hkv * kTopkCluster, kTopkThreads, smem, s>>>(scores, cu, B, T, keep_num, keep_den, idx,
                                                                           cu_kept, kept_total, status);
    return (int)cudaGetLastError();
}

}  // namespace sgd
