// plan.cu -- the split-KV partition kernel (one CTA) and its inspection kernel.
// The rule is stated in plan.cuh (granule 16 for decode; 64 for the fused score+quantize
// pass, whose tiles must coincide with the 64-token scheme-A partitions).
#include <algorithm>

#include "internal.h"
#include "plan.cuh"
#include "scan.cuh"

namespace sgd {

// staged arrays of plan_kernel: within the default 48 KB limit with room for its static arrays
constexpr size_t kPlanStageBytes = 47 * 1024;
// per-sequence arrays of plan_fast_kernel: the kernel opts into this much dynamic shared memory
constexpr size_t kPlanFastBytes = 160 * 1024;

// cu_len: lengths of the attended rows (cu_seqlens, or cu_kept for a kept set);
// cu_seq: cu_seqlens (for the scheme-A partition offsets of each sequence).
// With `staged`, the per-sequence values are read once into dynamic shared memory and row_pos,
// cta_begin and the partition offsets are built there (R + n_req + 2 + 5B int32) and copied out
// at the end, so no step waits on a global-memory round trip after the first loads.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t *__restrict__ cu_len,
                                                    const int32_t *__restrict__ cu_seq, int B, int Hkv,
                                                    int n_req, int min_chunk, int mode, int granule, int row_cost,
                                                    PlanView pv, WsHeader *hdr, int staged, float *out,
                                                    float *lse, int G, int D, const __nv_bfloat16 *q,
                                                    int64_t q_elems, int M, int len_unit, int ncg) {
    __shared__ int32_t sm[33];
    extern __shared__ int32_t stage[];
    const int tid = threadIdx.x;
    const int R = B * Hkv;
    int32_t *row_pos = staged ? stage : pv.row_pos;
    int32_t *cta_begin = staged ? stage + R + 1 : pv.cta_begin;
    int32_t *seqv = stage + R + n_req + 2;  // staged: [5][B] length, sequence length, starts, part0
    int32_t *part0 = staged ? seqv + 4 * B : pv.seq_part0;
    if (tid == 0) {
        hdr->status = 0;
        hdr->amax_bits[0] = hdr->amax_bits[1] = 0u;
    }
    if (q) {  // per-tensor query scale for the decode: max|q| / 127 (IEEE division)
        __shared__ uint32_t qmax;  // float bits: non-negative floats order as integers
        // q is 16-byte aligned and D a multiple of 8: 16-byte loads, four in flight per thread
        const uint4 *q4 = reinterpret_cast<const uint4 *>(q);
        const int64_t nv = q_elems / 8;
        uint32_t acc = 0u;  // |q| maxima as bf16x2 (exact)
        for (int64_t i = tid; i < nv; i += 4 * (int64_t)blockDim.x) {
            uint4 w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t k = i + (int64_t)u * blockDim.x;
                w[u] = (k < nv) ? __ldg(q4 + k) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                acc = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(acc, w[u].x), w[u].y), w[u].z), w[u].w);
        }
        float m = bf16x2_fold_max(acc);
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (tid == 0) qmax = 0u;
        __syncthreads();
        if ((tid & 31) == 0) atomicMax(&qmax, __float_as_uint(m));
        __syncthreads();
        if (tid == 0) hdr->q_scale = __fdiv_rn(__uint_as_float(qmax), 127.f);
    }
    if (staged) {
        for (int b = tid; b < B; b += blockDim.x) {  // all four loads of a thread in flight together
            const int32_t a0 = cu_len[b] * len_unit, a1 = cu_len[b + 1] * len_unit, s0 = cu_seq[b], s1 = cu_seq[b + 1];
            seqv[b] = a1 - a0;
            seqv[B + b] = s1 - s0;
            seqv[2 * B + b] = a0;
            seqv[3 * B + b] = s0;
        }
        __syncthreads();
    }
    auto len_of = [&](int b) -> int32_t { return staged ? seqv[b] : (cu_len[b + 1] - cu_len[b]) * len_unit; };
    auto seq_len_of = [&](int b) -> int32_t { return staged ? seqv[B + b] : cu_seq[b + 1] - cu_seq[b]; };
    auto len_start_of = [&](int b) -> int32_t { return staged ? seqv[2 * B + b] : cu_len[b] * len_unit; };
    auto seq_start_of = [&](int b) -> int32_t { return staged ? seqv[3 * B + b] : cu_seq[b]; };

    // 1. padded stream position of every row
    int32_t carry = 0;
    for (int base = 0; base < R; base += blockDim.x) {
        const int r = base + tid;
        int32_t v = 0;
        if (r < R) {
            const int32_t L = len_of(r % B);
            if (L < 1) atomicOr(&hdr->status, SGD_STATUS_EMPTY_SEQUENCE);
            v = (L > 0) ? (int32_t)align_up(L, granule) + row_cost : 0;
        }
        int32_t total;
        const int32_t ex = block_exclusive_scan(v, total, sm);
        if (r < R) row_pos[r] = carry + ex;
        carry += total;
    }
    const int32_t W = carry;
    if (tid == 0) row_pos[R] = W;

    int64_t S = 0;
    int ncta;
    if (mode == 0) {
        S = align_up((W + (int64_t)n_req - 1) / n_req, granule);
        if (S < min_chunk) S = min_chunk;
        ncta = (int)((W + S - 1) / S);
    } else {
        ncta = R;
    }
    __syncthreads();

    // 2. CTA ranges
    for (int i = tid; i <= n_req; i += blockDim.x) {
        int32_t a;
        if (mode == 0)
            a = (int32_t)(((int64_t)i * S < (int64_t)W) ? (int64_t)i * S : (int64_t)W);
        else
            a = row_pos[min(i, R)];
        cta_begin[i] = a;
    }
    __syncthreads();

    // 3. segments per CTA -> first slot and first row of each CTA
    carry = 0;
    for (int base = 0; base < n_req; base += blockDim.x) {
        const int i = base + tid;
        int32_t v = 0;
        if (i < n_req) {
            const int32_t a = cta_begin[i], e = cta_begin[i + 1];
            int r0 = R;
            if (a < e) {
                r0 = upper_bound_i32(row_pos, R + 1, a) - 1;
                for (int r = r0; r < R && row_pos[r] < e; ++r) {  // rows whose tokens meet [a, e)
                    const int32_t Lr = len_of(r % B);
                    v += (Lr > 0 && row_pos[r] + Lr > a) ? 1 : 0;
                }
            }
            pv.cta_row0[i] = r0;
        }
        int32_t total;
        const int32_t ex = block_exclusive_scan(v, total, sm);
        if (i < n_req) pv.cta_slot0[i] = carry + ex;
        carry += total;
    }
    const int32_t nslots_cta = carry;
    if (tid == 0) pv.cta_slot0[n_req] = nslots_cta;

    // 4. scheme-A partition offset of every sequence: sum_{b'<b} ceil(L_b' / 64)
    carry = 0;
    for (int base = 0; base < B; base += blockDim.x) {
        const int b = base + tid;
        int32_t v = 0;
        if (b < B) v = (int32_t)((max(seq_len_of(b), 0) + kPart - 1) / kPart);
        int32_t total;
        const int32_t ex = block_exclusive_scan(v, total, sm);
        if (b < B) {
            part0[b] = carry + ex;
            if (staged) pv.seq_part0[b] = carry + ex;
        }
        carry += total;
    }
    const int32_t n_parts = carry;
    if (tid == 0) pv.seq_part0[B] = n_parts;
    __syncthreads();  // part0 complete

    // 5. segments per row -> first slot of each row (same stream order); the row records
    carry = 0;
    for (int base = 0; base < R; base += blockDim.x) {
        const int r = base + tid;
        int32_t v = 0;
        if (r < R) {
            const int32_t p0 = row_pos[r];
            const int b = r % B;
            const int32_t L = max(len_of(b), 0);
            if (L > 0) v = (mode == 0) ? (int32_t)((p0 + L - 1) / S - p0 / S + 1) : 1;
        }
        int32_t total;
        const int32_t ex = block_exclusive_scan(v, total, sm);
        if (r < R) {
            const int b = r % B;
            pv.row_slot0[r] = carry + ex;
            int4 *ri = reinterpret_cast<int4 *>(pv.row_info + r);
            ri[0] = make_int4(row_pos[r], len_of(b), seq_start_of(b), seq_len_of(b));
            ri[1] = make_int4(len_start_of(b), part0[b], carry + ex, v);
            if (pv.row_done)  // one finished-segment counter per row and column group
                for (int j = 0; j < ncg; ++j) pv.row_done[r * ncg + j] = 0;
            if (out && v == 0) {  // a row with no tokens (reported above): zero output, lse -inf
                for (int m = 0; m < M; ++m) {
                    const int64_t h0 = ((int64_t)b * M + m) * Hkv * G + (r / B) * G;
                    for (int e = 0; e < G * D; ++e) out[h0 * D + e] = 0.f;
                    for (int g = 0; g < G; ++g) lse[h0 + g] = -INFINITY;
                }
            }
        }
        carry += total;
    }
    if (tid == 0) {
        pv.row_slot0[R] = carry;
        if (carry != nslots_cta) atomicOr(&hdr->status, SGD_STATUS_SIZE_MISMATCH);
        hdr->plan_W = W;
        hdr->plan_S = S;
        hdr->plan_ncta = ncta;
        hdr->plan_nslots = nslots_cta;
        hdr->n_parts = n_parts;
    }
    if (staged) {  // copy the staged arrays out
        __syncthreads();
        for (int i = tid; i <= R; i += blockDim.x) pv.row_pos[i] = row_pos[i];
        for (int i = tid; i <= n_req; i += blockDim.x) pv.cta_begin[i] = cta_begin[i];
    }
}

// The same plan with fewer block-wide steps (batches whose per-sequence values fit in shared
// memory): row positions follow from the prefix of the padded sequence lengths within one head
// (row r = kvh * B + b starts at kvh * Wh + P[b]), which one scan over the sequences gives together
// with the partition offsets; CTA ranges are closed forms; and the segment counts of CTA i and of
// row i are scanned together.  Writes the same arrays as plan_kernel.
__global__ void __launch_bounds__(1024) plan_fast_kernel(const int32_t *__restrict__ cu_len,
                                                         const int32_t *__restrict__ cu_seq, int B, int Hkv,
                                                         int n_req, int min_chunk, int mode, int granule,
                                                         int row_cost,
                                                         PlanView pv, WsHeader *hdr, float *out, float *lse, int G,
                                                         int D, const __nv_bfloat16 *q, int64_t q_elems, int M,
                                                         int len_unit, int ncg) {
    __shared__ int2 sm2[33];
    extern __shared__ int32_t st[];  // [6][B+1]: attended length, sequence length, attended start,
                                     // sequence start, padded prefix P, partition offset
    int32_t *len = st, *slen = st + (B + 1), *lstart = st + 2 * (B + 1), *sstart = st + 3 * (B + 1);
    int32_t *P = st + 4 * (B + 1), *part0 = st + 5 * (B + 1);
    const int tid = threadIdx.x, nt = blockDim.x;
    const int R = B * Hkv;
    if (tid == 0) {
        hdr->status = 0;
        hdr->amax_bits[0] = hdr->amax_bits[1] = 0u;
    }
    if (q) {  // per-tensor query scale for the decode: max|q| / 127 (IEEE division)
        __shared__ uint32_t qmax;
        const uint4 *q4 = reinterpret_cast<const uint4 *>(q);
        const int64_t nv = q_elems / 8;
        uint32_t acc = 0u;
        for (int64_t i = tid; i < nv; i += 4 * (int64_t)nt) {
            uint4 w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t k = i + (int64_t)u * nt;
                w[u] = (k < nv) ? __ldg(q4 + k) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                acc = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(acc, w[u].x), w[u].y), w[u].z), w[u].w);
        }
        float m = bf16x2_fold_max(acc);
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (tid == 0) qmax = 0u;
        __syncthreads();
        if ((tid & 31) == 0) atomicMax(&qmax, __float_as_uint(m));
        __syncthreads();
        if (tid == 0) hdr->q_scale = __fdiv_rn(__uint_as_float(qmax), 127.f);
    }
    for (int b = tid; b < B; b += nt) {  // all four loads of a thread in flight together
        const int32_t a0 = cu_len[b] * len_unit, a1 = cu_len[b + 1] * len_unit, s0 = cu_seq[b], s1 = cu_seq[b + 1];
        len[b] = a1 - a0;
        slen[b] = s1 - s0;
        lstart[b] = a0;
        sstart[b] = s0;
        if (a1 - a0 < 1) atomicOr(&hdr->status, SGD_STATUS_EMPTY_SEQUENCE);
    }
    __syncthreads();
    // 1. per sequence: padded length within a head (its prefix P) and scheme-A partitions (part0)
    int2 carry = make_int2(0, 0);
    for (int base = 0; base < B; base += nt) {
        const int b = base + tid;
        int32_t pad = 0, np = 0;
        if (b < B) {
            pad = (len[b] > 0) ? (int32_t)align_up(len[b], granule) + row_cost : 0;
            np = (max(slen[b], 0) + kPart - 1) / kPart;
        }
        int2 tot;
        const int2 ex = block_exclusive_scan2(pad, np, tot, sm2);
        if (b < B) {
            P[b] = carry.x + ex.x;
            part0[b] = carry.y + ex.y;
            pv.seq_part0[b] = carry.y + ex.y;
        }
        carry.x += tot.x;
        carry.y += tot.y;
    }
    const int32_t Wh = carry.x, n_parts = carry.y;
    if (tid == 0) {
        P[B] = Wh;
        pv.seq_part0[B] = n_parts;
    }
    const int32_t W = (int32_t)((int64_t)Wh * Hkv);
    int64_t S = 0;
    int ncta;
    if (mode == 0) {
        S = align_up((W + (int64_t)n_req - 1) / n_req, granule);
        if (S < min_chunk) S = min_chunk;
        ncta = (int)((W + S - 1) / S);
    } else {
        ncta = R;
    }
    __syncthreads();  // P complete
    auto row_pos = [&](int r) -> int32_t { return r >= R ? W : (r / B) * Wh + P[r % B]; };
    auto cta_begin = [&](int i) -> int32_t {
        if (mode == 0) return (int32_t)min((int64_t)i * S, (int64_t)W);
        return row_pos(min(i, R));
    };
    // 2. segments of CTA i and of row i, scanned together: first slot of each CTA and each row
    const int n_it = max(n_req, R);
    int2 acc = make_int2(0, 0);
    for (int base = 0; base < n_it; base += nt) {
        const int i = base + tid;
        int32_t vc = 0, vr = 0;
        if (i < n_req) {
            const int32_t a = cta_begin(i), e = cta_begin(i + 1);
            int r0 = R;
            if (a < e) {
                const int kvh = a / Wh;
                r0 = kvh * B + upper_bound_i32(P, B + 1, a - kvh * Wh) - 1;
                for (int r = r0; r < R && row_pos(r) < e; ++r) {  // rows whose tokens meet [a, e)
                    const int32_t Lr = len[r % B];
                    vc += (Lr > 0 && row_pos(r) + Lr > a) ? 1 : 0;
                }
            }
            pv.cta_row0[i] = r0;
            pv.cta_begin[i] = a;
        }
        int32_t p0 = 0, L = 0;
        if (i < R) {
            p0 = row_pos(i);
            L = max(len[i % B], 0);
            if (L > 0) vr = (mode == 0) ? (int32_t)((p0 + L - 1) / S - p0 / S + 1) : 1;
        }
        int2 tot;
        const int2 ex = block_exclusive_scan2(vc, vr, tot, sm2);
        if (i < n_req) pv.cta_slot0[i] = acc.x + ex.x;
        if (i < R) {
            const int b = i % B;
            pv.row_pos[i] = p0;
            pv.row_slot0[i] = acc.y + ex.y;
            int4 *ri = reinterpret_cast<int4 *>(pv.row_info + i);
            ri[0] = make_int4(p0, len[b], sstart[b], slen[b]);
            ri[1] = make_int4(lstart[b], part0[b], acc.y + ex.y, vr);
            if (pv.row_done)  // one finished-segment counter per row and column group
                for (int j = 0; j < ncg; ++j) pv.row_done[i * ncg + j] = 0;
            if (out && vr == 0) {  // a row with no tokens (reported above): zero output, lse -inf
                for (int m = 0; m < M; ++m) {
                    const int64_t h0 = ((int64_t)b * M + m) * Hkv * G + (i / B) * G;
                    for (int e = 0; e < G * D; ++e) out[h0 * D + e] = 0.f;
                    for (int g = 0; g < G; ++g) lse[h0 + g] = -INFINITY;
                }
            }
        }
        acc.x += tot.x;
        acc.y += tot.y;
    }
    if (tid == 0) {
        pv.cta_begin[n_req] = cta_begin(n_req);
        pv.cta_slot0[n_req] = acc.x;
        pv.row_pos[R] = W;
        pv.row_slot0[R] = acc.y;
        if (acc.x != acc.y) atomicOr(&hdr->status, SGD_STATUS_SIZE_MISMATCH);
        hdr->plan_W = W;
        hdr->plan_S = S;
        hdr->plan_ncta = ncta;
        hdr->plan_nslots = acc.x;
        hdr->n_parts = n_parts;
    }
}

// One thread per CTA: writes (cta, row, start, length) of its segments at their slots.
__global__ void plan_dump_kernel(PlanView pv, const int32_t *cu, int B, int Hkv, int n_req, int32_t *segs,
                                 int64_t max_segs, int32_t *n_segs, const WsHeader *hdr) {
    const int cta = blockIdx.x * blockDim.x + threadIdx.x;
    if (cta == 0) {
        n_segs[0] = pv.cta_slot0[n_req];
        n_segs[1] = hdr->plan_ncta;
    }
    if (cta >= n_req) return;
    SegCursor cur;
    cur.init(pv, B * Hkv, cta);
    int row, slot;
    int32_t t0, t1;
    while (cur.next(row, t0, t1, slot)) {
        if (slot < max_segs) {
            int32_t *o = segs + (int64_t)slot * 4;
            o[0] = cta;
            o[1] = row;
            o[2] = t0;
            o[3] = t1 - t0;
        }
    }
}

void launch_plan(const int32_t *cu_len, const int32_t *cu_seq, int B, int Hkv, int n_req, int min_chunk,
                 int mode, const PlanView &pv, WsHeader *hdr, cudaStream_t s, int granule, float *out, float *lse,
                 int G, int D, const void *q_bf16, int64_t q_elems, int M, int len_unit, int ncg, int row_cost) {
    // one thread per row / CTA / sequence where they fit: fewer warps make each of the kernel's
    // block barriers cheaper (the loops stride over anything larger)
    const int want = std::max(std::max(B * Hkv, n_req), B) + 1;
    const int nt = std::min(1024, std::max(64, (want + 31) / 32 * 32));
    const size_t seq_bytes = (size_t)6 * (B + 1) * sizeof(int32_t);
    if (seq_bytes <= kPlanFastBytes &&
        cudaFuncSetAttribute(plan_fast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPlanFastBytes) ==
            cudaSuccess) {
        launch_k(plan_fast_kernel, dim3(1), dim3(nt), seq_bytes, s, 1, cu_len, cu_seq, B, Hkv, n_req, min_chunk, mode,
                 granule, row_cost, pv, hdr, out, lse, G, D, static_cast<const __nv_bfloat16 *>(q_bf16), q_elems, M,
                 len_unit, ncg);
        return;
    }
    const size_t stage_bytes = (size_t)(B * Hkv + n_req + 2 + 5 * B) * sizeof(int32_t);
    const int staged = stage_bytes <= kPlanStageBytes;
    launch_k(plan_kernel, dim3(1), dim3(nt), staged ? stage_bytes : 0, s, 1, cu_len, cu_seq, B, Hkv, n_req,
             min_chunk, mode, granule, row_cost, pv, hdr, staged, out, lse, G, D,
             static_cast<const __nv_bfloat16 *>(q_bf16), q_elems, M, len_unit, ncg);
}

void launch_plan_dump(const PlanView &pv, const int32_t *cu, int B, int Hkv, int n_req, int32_t *segs,
                      int64_t max_segs, int32_t *n_segs, const WsHeader *hdr, cudaStream_t s) {
    launch_k(plan_dump_kernel, dim3((n_req + 127) / 128), dim3(128), 0, s, 1, pv, cu, B, Hkv, n_req, segs, max_segs,
               n_segs, hdr);
}

}  // namespace sgd
