// oam.cu -- top-K token selection of output-aware token dropping.
//
// "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse attention),
// section 3: tokens with the lowest OAM score are dropped and the top-K kept; one
// index set serves all G query heads of a KV head.  Ties are broken by the lower
// token index (total order: score descending, index ascending) and the kept
// positions are emitted in ascending order.  The scores themselves come from the
// score mode of the decode pipeline (decode.cu).
//
// One CTA per (KV head, sequence) row: an exact radix select of the K-th largest
// order-preserving 32-bit key in three digit passes (11, 11, 10 bits) over the
// row's scores (resident in L2), with warp-aggregated shared-memory histograms,
// then one pass in token order that keeps every key above the threshold and the
// first `need` keys equal to it.
#include "internal.h"
#include "scan.cuh"

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

__global__ void __launch_bounds__(1024) topk_kernel(const float *__restrict__ scores, const int32_t *__restrict__ cu,
                                                    int B, int64_t T, int keep_num, int keep_den,
                                                    int32_t *__restrict__ idx, int32_t *__restrict__ cu_kept,
                                                    int64_t Kt, int32_t *status) {
    __shared__ uint32_t hist[2048];
    __shared__ int32_t sm[33];
    __shared__ uint32_t sel[2];
    const int tid = threadIdx.x, lane = tid & 31;
    const int r = blockIdx.x, kvh = r / B, b = r % B;
    const int32_t L = cu[b + 1] - cu[b];

    // output offset of this sequence: sum of the kept counts of the sequences before it
    int32_t mine = 0;
    for (int bb = tid; bb < b; bb += blockDim.x) mine += kept_of(max(cu[bb + 1] - cu[bb], 1), keep_num, keep_den);
    int32_t off;
    block_exclusive_scan(mine, off, sm);
    if (L < 1) {
        if (tid == 0) atomicOr(status, SGD_STATUS_EMPTY_SEQUENCE);
        return;
    }
    const int32_t K = kept_of(L, keep_num, keep_den);
    if (kvh == 0 && tid == 0) {
        cu_kept[b + 1] = off + K;
        if (b == 0) cu_kept[0] = 0;
    }
    if (off + (int64_t)K > Kt) {
        if (tid == 0) atomicOr(status, SGD_STATUS_SIZE_MISMATCH);
        return;
    }
    const float *s = scores + (int64_t)kvh * T + cu[b];
    int32_t *out = idx + (int64_t)kvh * Kt + off;

    uint32_t prefix = 0, mask = 0;
    int32_t rem = K;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < nb; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        for (int32_t base = 0; base < L; base += blockDim.x) {
            const int32_t t = base + tid;
            uint32_t bin = 0xffffffffu;
            if (t < L) {
                const uint32_t key = score_key(__ldg(s + t));
                if ((key & mask) == prefix) bin = (key >> shift) & (uint32_t)(nb - 1);
            }
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (bin != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
        }
        __syncthreads();
        // bins in descending order: thread tid owns positions tid*per .. tid*per+per-1
        const int per = nb / blockDim.x;
        int32_t c = 0;
        for (int i = 0; i < per; ++i) c += (int32_t)hist[nb - 1 - (tid * per + i)];
        int32_t tot;
        int32_t above = block_exclusive_scan(c, tot, sm);
        for (int i = 0; i < per; ++i) {
            const int j = nb - 1 - (tid * per + i);
            const int32_t h = (int32_t)hist[j];
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
        __syncthreads();
    }
    // keys > prefix: K - rem of them; keys == prefix: take the first `rem` in token order
    const uint32_t thr = prefix;
    const int32_t need = rem;
    int32_t written = 0, eq_seen = 0;
    for (int32_t base = 0; base < L; base += blockDim.x * 8) {
        const int32_t t0 = base + tid * 8;
        uint32_t gtm = 0, eqm = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int32_t t = t0 + i;
            if (t < L) {
                const uint32_t key = score_key(__ldg(s + t));
                if (key > thr) gtm |= 1u << i;
                else if (key == thr) eqm |= 1u << i;
            }
        }
        int32_t tot_eq, tot_keep;
        int32_t eq_before = block_exclusive_scan(__popc(eqm), tot_eq, sm) + eq_seen;
        uint32_t keep = gtm;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (eqm & (1u << i)) {
                if (eq_before < need) keep |= 1u << i;
                ++eq_before;
            }
        int32_t pos = block_exclusive_scan(__popc(keep), tot_keep, sm) + written;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (keep & (1u << i)) {
                if (pos < K) out[pos] = t0 + i;
                ++pos;
            }
        written += tot_keep;
        eq_seen += tot_eq;
    }
    if (tid == 0 && written != K) atomicOr(status, SGD_STATUS_SIZE_MISMATCH);
}

int launch_topk(const float *scores, const int32_t *cu, int B, int Hkv, int64_t T, int keep_num, int keep_den,
                int32_t *idx, int32_t *cu_kept, int64_t kept_total, int32_t *status, cudaStream_t s) {
    topk_kernel<<<B * Hkv, 1024, 0, s>>>(scores, cu, B, T, keep_num, keep_den, idx, cu_kept, kept_total, status);
    return (int)cudaGetLastError();
}

}  // namespace sgd
