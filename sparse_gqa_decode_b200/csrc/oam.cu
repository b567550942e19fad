// oam.cu -- top-K token selection of output-aware token dropping.
//
// "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse attention),
// section 3: tokens with the lowest OAM score are dropped and the top-K kept; one
// index set serves all G query heads of a KV head.  Ties are broken by the lower
// token index (total order: score descending, index ascending) and the kept
// positions are emitted in ascending order.  The scores themselves come from the
// score mode of the decode pipeline (decode.cu).
//
// One thread-block cluster of CL CTAs per (KV head, sequence) row, each CTA holding a
// contiguous 1/CL of the row's order-preserving 32-bit keys in shared memory.
//
//   1. key range: every CTA publishes its smallest and largest key (cluster barrier 1);
//   2. linear histogram: 2048 bins between the row's smallest and largest score, a map
//      that never decreases with the score, so the K-th largest key lies in the first bin,
//      counted from the top, whose cumulative count reaches K (barrier 2);
//   3. distributed merge: CTA r sums bins [r*2048/CL, (r+1)*2048/CL) over the cluster
//      into its own shared memory, with the slice total (barrier 3); every CTA then finds
//      the slice from the slice totals and the bin b* inside it with one warp;
//   4. candidates: every CTA counts its keys in bins above b* and gathers its keys of b*
//      (barrier 4); each CTA copies every candidate, ranks them exactly (thr = the K-th
//      largest key, need = how many keys equal to thr are kept, the lowest-index ones)
//      and derives from the candidate lists and the above-b* counts how many kept tokens
//      the CTAs before it hold -- no further pass over the keys;
//   5. compaction in token order, one warp ballot per 32 tokens and one block scan,
//      each CTA writing at its cluster-wide offset.
//
// Fallback (every score equal, a non-finite range, or more than kCandCap keys in b*): an
// exact radix select over the keys in three digit passes (11, 11, 10 bits), then one
// counting pass whose per-CTA totals are exchanged through distributed shared memory.
// Cluster barriers are hardware barriers: no spinning on flags.
#include <cooperative_groups.h>

#include "internal.h"
#include "plan.cuh"
#include "scan.cuh"

namespace cg = cooperative_groups;

namespace sgd {

// Order-preserving key of a score; -0 and +0 compare equal, as they do as scores, so both map
// to the key of +0.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

__device__ __forceinline__ int32_t kept_of(int32_t L, int keep_num, int keep_den) {
    int64_t k = ((int64_t)L * keep_num + keep_den - 1) / keep_den;
    if (k < 1) k = 1;
    if (k > L) k = L;
    return (int32_t)k;
}

__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

constexpr int kTopkBins = 2048;   // linear bins of the fast path
constexpr int kCandCap = 1024;    // keys of the threshold bin ranked exactly (per row)
constexpr int kTopkChunk = 16384; // keys one compaction round covers (per CTA)

template <int NT, int CL>
struct TopkCfg {
    static constexpr int kThreads = NT;
    static constexpr int kCluster = CL;
    static constexpr int kWarps = NT / 32;
    static constexpr int kSlice = kTopkBins / CL;  // bins each CTA merges
    static constexpr int kPerLane = kSlice / 32;   // bins per lane of the warp that scans one slice
    static constexpr int kLoadUnroll = kTopkChunk / NT;
    static_assert(kPerLane % 4 == 0 && kSlice <= NT, "slice layout");
    static_assert(kTopkChunk % (32 * kWarps) == 0 && kTopkChunk / 32 <= NT, "compaction rounds");
};

// Compaction in token order from the keys themselves (radix path, or rows longer than the masks
// cover): warp w covers 32 * (kTopkChunk / NT) consecutive keys per chunk.  `written` / `eq_seen`
// enter as the kept tokens / keys equal to thr before this CTA and leave including it.
template <int NT, typename KeyAt>
__device__ __forceinline__ void compact_by_keys(const KeyAt &key_at, int32_t n, int32_t lo, uint32_t thr, int32_t need,
                                                int32_t K, int32_t &written, int32_t &eq_seen, int32_t *out,
                                                int32_t *sm) {
    constexpr int RW = kTopkChunk / NT;  // 32-token rounds per warp and chunk
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    for (int32_t base = 0; base < n; base += kTopkChunk) {
        const int32_t wbase = base + warp * 32 * RW;
        uint32_t g = 0u, e = 0u;
#pragma unroll 4
        for (int j = 0; j < RW; ++j) {
            const int32_t t = wbase + j * 32 + lane;
            const uint32_t key = t < n ? key_at(t) : 0u;
            g += __popc(__ballot_sync(0xffffffffu, t < n && key > thr));
            e += __popc(__ballot_sync(0xffffffffu, t < n && key == thr));
        }
        // packed (above, equal) counts: each half stays below 2^16 (kTopkChunk keys per round)
        int32_t tot;
        const int32_t pre = block_exclusive_scan(lane == 0 ? (int32_t)((g << 16) | e) : 0, tot, sm);
        const int32_t wpre = __shfl_sync(0xffffffffu, pre, 0);
        int32_t eq_run = eq_seen + (wpre & 0xffff);
        int32_t pos = written + (wpre >> 16) + min(need, eq_run) - min(need, eq_seen);
#pragma unroll 4
        for (int j = 0; j < RW; ++j) {
            const int32_t t = wbase + j * 32 + lane;
            const uint32_t key = t < n ? key_at(t) : 0u;
            const bool gt = t < n && key > thr, eq = t < n && key == thr;
            const uint32_t em = __ballot_sync(0xffffffffu, eq);
            const bool keep = gt || (eq && eq_run + __popc(em & lt) < need);
            const uint32_t km = __ballot_sync(0xffffffffu, keep);
            if (keep) {
                const int32_t p = pos + __popc(km & lt);
                if (p < K) out[p] = lo + t;
            }
            pos += __popc(km);
            eq_run += __popc(em);
        }
        const int32_t gtot = tot >> 16, etot = tot & 0xffff;
        written += gtot + min(need, eq_seen + etot) - min(need, eq_seen);
        eq_seen += etot;
    }
}

// grid: B*Hkv clusters of CL CTAs (cluster dimension set at launch), NT threads (at least MINB
// CTAs resident per SM), `cap` keys of dynamic shared memory per CTA (keys past `cap` are re-read
// from global memory).
template <int NT, int CL, int MINB>
__global__ void __launch_bounds__(NT, MINB)
    topk_cluster_kernel(const float *__restrict__ scores, const int32_t *__restrict__ cu, int B, int64_t T,
                        int keep_num, int keep_den, int32_t *__restrict__ idx, int32_t *__restrict__ cu_kept,
                        int64_t Kt, int32_t *status, int cap) {
    using Cfg = TopkCfg<NT, CL>;
    constexpr int NW = Cfg::kWarps, SLICE = Cfg::kSlice, PL = Cfg::kPerLane, U = Cfg::kLoadUnroll;
    extern __shared__ uint32_t skeys[];                   // [cap]
    __shared__ uint32_t hist[2][kTopkBins];               // linear histogram; radix passes alternate
    __shared__ __align__(16) uint32_t mh[SLICE];          // merged counts of this CTA's bin slice
    __shared__ uint32_t cand[kCandCap];                   // this CTA's keys of bin b*
    __shared__ uint32_t allc[kCandCap];                   // every CTA's keys of bin b*, rank order
    __shared__ uint32_t smask[kTopkChunk / 32];           // per 32-token round: keys in bins above b*
    __shared__ uint32_t cmask[kTopkChunk / 32];           // per 32-token round: keys in bin b*
    __shared__ uint32_t wred[3][NW];
    __shared__ uint32_t ext[2];                           // this CTA's smallest and largest key
    __shared__ uint32_t slice_tot, ncand, nabove;
    __shared__ int32_t sm[33];
    __shared__ uint32_t sel[2];
    __shared__ int32_t cnt[2];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = blockIdx.x / CL, kvh = r / B, b = r % B;
    const int32_t L = cu[b + 1] - cu[b];
    const int32_t C = (max(L, 0) + CL - 1) / CL;
    const int32_t lo = min(rank * C, max(L, 0)), n = max(min(lo + C, L) - lo, 0);
    const float *s = scores + (int64_t)kvh * T + cu[b] + lo;
    const int32_t ns = min(n, cap);

    // ---- 1. stage keys, this CTA's key range, output offset of the sequence ----
    uint32_t mine = 0;  // kept counts of the sequences before this one
    for (int bb = tid; bb < b; bb += NT) mine += kept_of(max(cu[bb + 1] - cu[bb], 1), keep_num, keep_den);
    uint32_t kmin = 0xffffffffu, kmax = 0u;  // neutral for an empty chunk
    for (int32_t base = 0; base < ns; base += NT * U) {  // U independent loads in flight
        float x[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int32_t i = base + u * NT + tid;
            x[u] = (i < ns) ? __ldg(s + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int32_t i = base + u * NT + tid;
            if (i < ns) {
                const uint32_t k = score_key(x[u]);
                skeys[i] = k;
                kmin = min(kmin, k);
                kmax = max(kmax, k);
            }
        }
    }
    for (int32_t i = cap + tid; i < n; i += NT) {  // keys beyond the shared-memory stage
        const uint32_t k = score_key(__ldg(s + i));
        kmin = min(kmin, k);
        kmax = max(kmax, k);
    }
    auto key_at = [&](int32_t i) -> uint32_t { return i < cap ? skeys[i] : score_key(__ldg(s + i)); };
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        mine += __shfl_xor_sync(0xffffffffu, mine, o);
    }
    if (lane == 0) {
        wred[0][warp] = kmin;
        wred[1][warp] = kmax;
        wred[2][warp] = mine;
    }
    for (int i = tid; i < kTopkBins; i += NT) hist[0][i] = 0u;
    if (tid == 0) slice_tot = ncand = nabove = 0u;
    __syncthreads();
    {  // every warp reduces the per-warp values itself
        uint32_t a0 = lane < NW ? wred[0][lane] : 0xffffffffu, a1 = lane < NW ? wred[1][lane] : 0u;
        uint32_t a2 = lane < NW ? wred[2][lane] : 0u;
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            a0 = min(a0, __shfl_xor_sync(0xffffffffu, a0, o));
            a1 = max(a1, __shfl_xor_sync(0xffffffffu, a1, o));
            a2 += __shfl_xor_sync(0xffffffffu, a2, o);
        }
        kmin = a0;
        kmax = a1;
        mine = a2;
    }
    const int32_t off = (int32_t)mine;
    // the early exits depend on the row only, so every CTA of the cluster takes them together
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
    if (tid == 0) {
        ext[0] = kmin;
        ext[1] = kmax;
    }
    cluster.sync();  // (1) every CTA's key range is published
    uint32_t gmin = 0xffffffffu, gmax = 0u;
#pragma unroll
    for (int rr = 0; rr < CL; ++rr) {
        const uint32_t *e = cluster.map_shared_rank(ext, rr);
        gmin = min(gmin, e[0]);
        gmax = max(gmax, e[1]);
    }
    const float smin = key_score(gmin), span = key_score(gmax) - smin;
    // the same decision in every CTA of the cluster
    bool fast = (gmin < gmax) && isfinite(span) && span > 0.f && isfinite(smin);
    const float bscale = fast ? 2048.f / span : 0.f;
    auto lin_bin = [&](uint32_t key) -> int {  // non-decreasing in the score; explicit roundings
        const float v = __fmul_rn(__fsub_rn(key_score(key), smin), bscale);
        return min(kTopkBins - 1, max(0, (int)v));
    };

    uint32_t thr = 0u;
    int32_t need = 0, written = 0, eq_seen = 0;  // kept tokens / keys equal to thr in the CTAs before
    if (fast) {
        for (int32_t i = tid; i < n; i += NT) atomicAdd(&hist[0][lin_bin(key_at(i))], 1u);
        cluster.sync();  // (2) every CTA's linear histogram is complete
        uint32_t m = 0u;
        if (tid < SLICE) {
            const int j = rank * SLICE + tid;
#pragma unroll
            for (int rr = 0; rr < CL; ++rr) m += cluster.map_shared_rank(&hist[0][0], rr)[j];
            mh[tid] = m;
        }
        m = warp_sum_u32(m);
        if (lane == 0 && m) atomicAdd(&slice_tot, m);
        cluster.sync();  // (3) every slice is merged
        // the slice holding the K-th largest key, counted from the top, and the keys above it
        int sstar = 0;
        int32_t above = 0;
        {
            bool found = false;
#pragma unroll
            for (int rr = CL - 1; rr >= 0; --rr) {
                const int32_t t = (int32_t)*cluster.map_shared_rank(&slice_tot, rr);
                if (!found) {
                    if (above + t >= K) {
                        sstar = rr;
                        found = true;
                    } else {
                        above += t;
                    }
                }
            }
        }
        if (warp == 0) {  // the bin inside the slice: lane 0 holds the slice's top PL bins
            const uint32_t *rm = cluster.map_shared_rank(mh, sstar);
            const int lb = (31 - lane) * PL;
            uint32_t c[PL];
#pragma unroll
            for (int v4 = 0; v4 < PL / 4; ++v4) {
                const uint4 t = *reinterpret_cast<const uint4 *>(rm + lb + 4 * v4);
                c[4 * v4] = t.x;
                c[4 * v4 + 1] = t.y;
                c[4 * v4 + 2] = t.z;
                c[4 * v4 + 3] = t.w;
            }
            int32_t lsum = 0;
#pragma unroll
            for (int u = 0; u < PL; ++u) lsum += (int32_t)c[u];
            const int32_t ex = above + warp_inclusive_scan(lsum) - lsum;
            if (ex < K && K <= ex + lsum) {  // exactly one lane
                int32_t acc = ex;
                bool done = false;
#pragma unroll
                for (int u = PL - 1; u >= 0; --u) {
                    if (!done) {
                        if (acc + (int32_t)c[u] >= K) {
                            sel[0] = (uint32_t)(sstar * SLICE + lb + u);
                            sel[1] = (uint32_t)acc;
                            done = true;
                        } else {
                            acc += (int32_t)c[u];
                        }
                    }
                }
            }
        }
        __syncthreads();
        const int bstar = (int)sel[0];
        const int32_t rem = K - (int32_t)sel[1];  // keys still to take inside bin b*
        // warp w takes the 32-token rounds w, w + NW, ...; a round's masks say which of its keys
        // lie above bin b* (kept whatever thr is) and which in it (decided by the exact rank)
        uint32_t my_above = 0u;
        for (int32_t rd = warp; rd * 32 < n; rd += NW) {
            const int32_t t = rd * 32 + lane;
            uint32_t key = 0u;
            int bin = -1;
            if (t < n) {
                key = key_at(t);
                bin = lin_bin(key);
            }
            const uint32_t above_m = __ballot_sync(0xffffffffu, bin > bstar);
            const uint32_t cand_m = __ballot_sync(0xffffffffu, bin == bstar);
            if (bin == bstar) {
                const uint32_t at = atomicAdd(&ncand, 1u);
                if (at < (uint32_t)kCandCap) cand[at] = key;
            }
            if (lane == 0) {
                my_above += __popc(above_m);
                if (rd < kTopkChunk / 32) {
                    smask[rd] = above_m;
                    cmask[rd] = cand_m;
                }
            }
        }
        if (lane == 0 && my_above) atomicAdd(&nabove, my_above);
        cluster.sync();  // (4) every CTA's candidates and above-b* count are published
        uint32_t nc[CL], tot_c = 0u, cand_before = 0u, above_before = 0u;
#pragma unroll
        for (int rr = 0; rr < CL; ++rr) {
            nc[rr] = *cluster.map_shared_rank(&ncand, rr);
            tot_c += nc[rr];
            if (rr < rank) {
                cand_before += nc[rr];
                above_before += *cluster.map_shared_rank(&nabove, rr);
            }
        }
        fast = tot_c <= (uint32_t)kCandCap;  // the same in every CTA
        if (fast) {
            for (uint32_t ci = tid; ci < tot_c; ci += NT) {  // every candidate, in rank order
                int own = 0;
                uint32_t at = ci;
#pragma unroll
                for (int rr = 0; rr < CL - 1; ++rr)
                    if (own == rr && at >= nc[rr]) {
                        at -= nc[rr];
                        own = rr + 1;
                    }
                allc[ci] = cluster.map_shared_rank(cand, own)[at];
            }
            cluster.barrier_arrive();  // this thread's last read of another CTA's shared memory
            __syncthreads();
            for (uint32_t ci = tid; ci < tot_c; ci += NT) {  // exact rank of every candidate
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
            __syncthreads();
            thr = sel[0];
            need = (int32_t)sel[1];
            // keys above thr / equal to thr among the candidates of the CTAs before this one
            uint32_t g = 0u, e = 0u;
            for (uint32_t ci = tid; ci < cand_before; ci += NT) {
                const uint32_t key = allc[ci];
                g += key > thr;
                e += key == thr;
            }
            g = warp_sum_u32(g);
            e = warp_sum_u32(e);
            if (lane == 0) {
                wred[0][warp] = g;
                wred[1][warp] = e;
            }
            __syncthreads();
            g = lane < NW ? wred[0][lane] : 0u;
            e = lane < NW ? wred[1][lane] : 0u;
            g = warp_sum_u32(g);
            e = warp_sum_u32(e);
            eq_seen = (int32_t)e;
            written = (int32_t)(above_before + g) + min(need, eq_seen);
        }
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
            for (int i = tid; i < nb; i += NT) h[i] = 0u;
            __syncthreads();
            for (int32_t base = 0; base < n; base += NT) {
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
            // thread t owns the digits nb-1-t*(nb/NT) .. downwards (descending order)
            constexpr int kMaxPer = 2048 / NT > 0 ? 2048 / NT : 1;
            const int per = nb / NT;
            uint32_t a[kMaxPer];
            int32_t my = 0;
#pragma unroll
            for (int u = 0; u < kMaxPer; ++u) {
                a[u] = 0u;
                if (u < per) {
                    const int j = nb - 1 - tid * per - u;
#pragma unroll
                    for (int rr = 0; rr < CL; ++rr) a[u] += cluster.map_shared_rank(h, rr)[j];
                    my += (int32_t)a[u];
                }
            }
            int32_t tot;
            int32_t above = block_exclusive_scan(my, tot, sm);
#pragma unroll
            for (int u = 0; u < kMaxPer; ++u) {
                if (u < per) {
                    if (above < rem && rem <= above + (int32_t)a[u]) {
                        sel[0] = (uint32_t)(nb - 1 - tid * per - u);
                        sel[1] = (uint32_t)above;
                    }
                    above += (int32_t)a[u];
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
        // keys > thr: K - need of them; keys == thr: the first `need` in token order are kept
        int32_t my_gt = 0, my_eq = 0;
        for (int32_t i = tid; i < n; i += NT) {
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
        for (int rr = 0; rr < rank; ++rr) {
            const int32_t *rc = cluster.map_shared_rank(cnt, rr);
            written += rc[0] + min(max(need - eq_seen, 0), rc[1]);
            eq_seen += rc[1];
        }
        cluster.barrier_arrive();  // this thread's last read of another CTA's shared memory
    }

    // ---- 5. compaction in token order ----
    int32_t *out = idx + (int64_t)kvh * Kt + off;
    if (fast && n <= kTopkChunk && n <= cap) {
        // from the masks: thread t owns round t; only keys of bin b* are looked at again
        uint32_t gtm = 0u, eqm = 0u;
        if (tid * 32 < n) {
            gtm = smask[tid];
            uint32_t cm = cmask[tid];
            while (cm) {
                const int bit = __ffs(cm) - 1;
                cm &= cm - 1u;
                const uint32_t key = skeys[tid * 32 + bit];
                if (key > thr) gtm |= 1u << bit;
                else if (key == thr) eqm |= 1u << bit;
            }
        }
        // packed (above, equal) counts: each half stays below 2^16 (kTopkChunk keys)
        int32_t tot;
        const int32_t pre = block_exclusive_scan((int32_t)((__popc(gtm) << 16) | __popc(eqm)), tot, sm);
        int32_t eq_run = eq_seen + (pre & 0xffff);
        int32_t pos = written + (pre >> 16) + min(need, eq_run) - min(need, eq_seen);
        uint32_t keep = gtm;
        while (eqm && eq_run < need) {  // the equal keys still within `need`, lowest index first
            const int bit = __ffs(eqm) - 1;
            eqm &= eqm - 1u;
            keep |= 1u << bit;
            ++eq_run;
        }
        while (keep) {
            const int bit = __ffs(keep) - 1;
            keep &= keep - 1u;
            if (pos < K) out[pos] = lo + tid * 32 + bit;
            ++pos;
        }
        written += (tot >> 16) + min(need, eq_seen + (tot & 0xffff)) - min(need, eq_seen);
        eq_seen += tot & 0xffff;
    } else {
        compact_by_keys<NT>(key_at, n, lo, thr, need, K, written, eq_seen, out, sm);
    }
    if (rank == CL - 1 && tid == 0 && written != K) atomicOr(status, SGD_STATUS_SIZE_MISMATCH);
    cluster.barrier_wait();  // no CTA leaves while another may still read its shared memory
}

// Launch one (NT, CL, MINB) variant.  cap = keys staged in shared memory per CTA.
template <int NT, int CL, int MINB>
int launch_topk_cfg(const float *scores, const int32_t *cu, int B, int Hkv, int64_t T, int keep_num, int keep_den,
                    int32_t *idx, int32_t *cu_kept, int64_t kept_total, int32_t *status, int cap, cudaStream_t s) {
    auto kern = topk_cluster_kernel<NT, CL, MINB>;
    const int smem = cap * 4;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return (int)e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return (int)e;
    if (CL > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return (int)e;
    }
    return (int)launch_k(kern, dim3((unsigned)(B * Hkv * CL)), dim3(NT), (size_t)smem, s, CL, scores, cu, B, T,
                           keep_num, keep_den, idx, cu_kept, kept_total, status, cap);
}

int launch_topk(const float *scores, const int32_t *cu, int B, int Hkv, int64_t T, int keep_num, int keep_den,
                int32_t *idx, int32_t *cu_kept, int64_t kept_total, int32_t *status, cudaStream_t s) {
    // 512 threads, 8-CTA clusters, two CTAs per SM: every row of a 32-row batch resident at once
    return launch_topk_cfg<512, 8, 2>(scores, cu, B, Hkv, T, keep_num, keep_den, idx, cu_kept, kept_total, status,
                                   kTopkChunk, s);
}

// ------------------------------------------------------------------------------------------
// block scores for block-granular selection ([NSA] section 2.1: 64-token selection blocks): each
// warp takes kBlocksPerWarp consecutive blocks of one KV head, finds the first one's sequence
// once, issues the loads of all its blocks together (two coalesced loads per lane and block) and
// reduces each block to its best token score
// ------------------------------------------------------------------------------------------
constexpr int kBlockMaxWarps = 8;
constexpr int kBlocksPerWarp = 4;

__global__ void __launch_bounds__(kBlockMaxWarps * 32)
    block_max_kernel(const float *__restrict__ scores, const int32_t *__restrict__ cu_seq,
                     const int32_t *__restrict__ cu_blk, int B, int Hkv, int64_t T, int64_t Tb,
                     float *__restrict__ bscores, int32_t *status) {
    const int64_t wpr = (Tb + kBlocksPerWarp - 1) / kBlocksPerWarp;  // warps per KV head
    const int64_t w = (int64_t)blockIdx.x * kBlockMaxWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= (int64_t)Hkv * wpr) return;
    const int h = (int)(w / wpr);
    const int32_t j0 = (int32_t)((w - (int64_t)h * wpr) * kBlocksPerWarp);
    if (j0 == 0 && h == 0 && lane == 0 && __ldg(cu_blk + B) != Tb) atomicOr(status, SGD_STATUS_SIZE_MISMATCH);
    int b = upper_bound_i32(cu_blk, B + 1, j0) - 1;  // sequence of block j0
    float v[kBlocksPerWarp][2];
    int32_t n[kBlocksPerWarp];
#pragma unroll
    for (int i = 0; i < kBlocksPerWarp; ++i) {
        const int32_t j = j0 + i;
        v[i][0] = v[i][1] = -INFINITY;
        n[i] = -1;  // no such block (past Tb, or past the lengths' blocks)
        if (j >= Tb) continue;
        while (b < B && __ldg(cu_blk + b + 1) <= j) ++b;  // blocks of empty sequences are skipped
        if (b < 0 || b >= B) continue;
        const int32_t s0 = __ldg(cu_seq + b), s1 = __ldg(cu_seq + b + 1);
        const int32_t t0 = s0 + (j - __ldg(cu_blk + b)) * kPart;
        n[i] = max(0, min(kPart, s1 - t0));
        const float *row = scores + (int64_t)h * T + t0;
        if (lane < n[i]) v[i][0] = __ldg(row + lane);
        if (lane + 32 < n[i]) v[i][1] = __ldg(row + lane + 32);
    }
#pragma unroll
    for (int i = 0; i < kBlocksPerWarp; ++i) {
        const int32_t j = j0 + i;
        if (j >= Tb) break;
        const float m = warp_max(fmaxf(v[i][0], v[i][1]));
        if (lane == 0) {
            bscores[(int64_t)h * Tb + j] = m;
            if (n[i] < 0) atomicOr(status, SGD_STATUS_SIZE_MISMATCH);  // the caller's count exceeds the lengths'
        }
    }
}

int launch_block_max(const float *scores, const int32_t *cu_seq, const int32_t *cu_blk, int B, int Hkv, int64_t T,
                     int64_t Tb, float *bscores, int32_t *status, cudaStream_t s) {
    const int64_t warps = (int64_t)Hkv * ((Tb + kBlocksPerWarp - 1) / kBlocksPerWarp);
    if (warps <= 0) return 0;
    const unsigned grid = (unsigned)((warps + kBlockMaxWarps - 1) / kBlockMaxWarps);
    return (int)launch_k(block_max_kernel, dim3(grid), dim3(kBlockMaxWarps * 32), 0, s, 1, scores, cu_seq, cu_blk,
                         B, Hkv, T, Tb, bscores, status);
}

}  // namespace sgd
