// quantize.cu -- INT8 KV cache, schemes A and B.
//
// "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse attention),
// section 6: q_val = round(val / scale) with scale = max|x| / 127 over the group
// that shares it.  Scheme A ("fine-grained QK"): K has one scale per partition of
// 64 consecutive tokens (counted from each sequence's first token, per KV head),
// V one scale for the whole tensor.  Scheme B ("coarser KV"): one scale each for K
// and for V.  Readings: scale = float32 nearest to amax/127; the quotient is the
// correctly rounded float32 x/scale; rounding is half-to-even; codes clamp to
// [-127, 127]; a zero scale gives zero codes.
//
// Passes.  A per-tensor scale needs the tensor's max before any code, so V (and K
// for scheme B) is read twice:
//   scheme A: pass 1 quantises each K partition from registers (one read of K) and
//             accumulates max|V|; pass 2 quantises V.
//   scheme B: pass 1 accumulates max|K| and max|V|; pass 2 quantises both.
//
// Exact codes without a divide per element: q' = x * RN(1/s) differs from the
// correctly rounded quotient Q = RN(x/s) by at most |x/s| * 2^-23 + ulp(Q)/2 <= 2.3e-5
// (|x/s| <= 127 * (1 + 2^-23) because s is the group's own scale), so
// round_half_even(q') == round_half_even(Q) unless q' lies within 2.3e-5 of a
// half-integer.  Whenever q' is within 1e-4 of one (or is not finite) the IEEE
// division __fdiv_rn(x, s) is taken instead.
#include "internal.h"
#include "quant.cuh"
#include "scan.cuh"

namespace sgd {

__device__ __forceinline__ float block_max(float v, float *sm) {
    v = warp_max(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    __syncthreads();
    if (lane == 0) sm[warp] = v;
    __syncthreads();
    float r = 0.f;
    for (int w = 0; w < nw; ++w) r = fmaxf(r, sm[w]);
    return r;
}

// Zero the max accumulators, partition offsets of every sequence, consistency checks.
__global__ void __launch_bounds__(1024) quant_prep_kernel(const int32_t *cu, int B, int64_t n_parts_host,
                                                          int check_parts, int32_t *seq_part0, WsHeader *hdr) {
    __shared__ int32_t sm[33];
    const int tid = threadIdx.x;
    if (tid == 0) {
        hdr->status = 0;
        hdr->amax_bits[0] = hdr->amax_bits[1] = 0u;
    }
    int32_t carry = 0;
    for (int base = 0; base < B; base += blockDim.x) {
        const int b = base + tid;
        int32_t v = 0;
        if (b < B) {
            const int32_t L = cu[b + 1] - cu[b];
            if (L < 1) atomicOr(&hdr->status, SGD_STATUS_EMPTY_SEQUENCE);
            v = (max(L, 0) + kPart - 1) / kPart;
        }
        int32_t total;
        const int32_t ex = block_exclusive_scan(v, total, sm);
        if (b < B) seq_part0[b] = carry + ex;
        carry += total;
    }
    if (tid == 0) {
        seq_part0[B] = carry;
        hdr->n_parts = carry;
        if (check_parts && carry != n_parts_host) atomicOr(&hdr->status, SGD_STATUS_SIZE_MISMATCH);
    }
}

// Scheme A pass 1: one CTA per (KV head, partition): K codes and scale from registers, max|V|.
template <typename T, int D>
__global__ void __launch_bounds__(256) quant_k_partition_kernel(const T *__restrict__ k, const T *__restrict__ v,
                                                                const int32_t *__restrict__ cu,
                                                                const int32_t *__restrict__ seq_part0, int B,
                                                                int Hkv, int64_t Ttot, int64_t n_parts,
                                                                int8_t *__restrict__ kc,
                                                                float *__restrict__ k_scale, WsHeader *hdr) {
    constexpr int VE = Vec<T>::VE;
    constexpr int NV = (kPart * D / VE + 255) / 256;  // vectors per thread
    __shared__ float sm[32];
    if (hdr->n_parts != n_parts) return;  // sizes disagree: flagged by the prep kernel
    const int64_t total = (int64_t)Hkv * n_parts;
    float vmax = 0.f;
    for (int64_t p = blockIdx.x; p < total; p += gridDim.x) {
        const int kvh = (int)(p / n_parts);
        const int32_t lp = (int32_t)(p - (int64_t)kvh * n_parts);
        int lo = 0, hi = B;  // sequence b with seq_part0[b] <= lp < seq_part0[b+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (seq_part0[mid] <= lp) lo = mid;
            else hi = mid;
        }
        const int b = lo;
        const int32_t tok0 = cu[b] + (lp - seq_part0[b]) * kPart;
        const int32_t ntok = min(kPart, cu[b + 1] - tok0);
        const int64_t e0 = ((int64_t)kvh * Ttot + tok0) * D;
        const int nvec = ntok * D / VE;
        const uint4 *kp = reinterpret_cast<const uint4 *>(k + e0);
        const uint4 *vp = reinterpret_cast<const uint4 *>(v + e0);
        float x[NV][VE];
        float kmax = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int vi = threadIdx.x + 256 * i;
            uint4 kw = make_uint4(0, 0, 0, 0), vw = kw;
            if (vi < nvec) {
                kw = __ldcs(kp + vi);
                vw = __ldcs(vp + vi);
            }
            Vec<T>::unpack(kw, x[i]);
            float y[VE];
            Vec<T>::unpack(vw, y);
#pragma unroll
            for (int j = 0; j < VE; ++j) {
                kmax = fmaxf(kmax, fabsf(x[i][j]));
                vmax = fmaxf(vmax, fabsf(y[j]));
            }
        }
        kmax = block_max(kmax, sm);
        const float s = __fdiv_rn(kmax, 127.f);
        const float r = (s != 0.f) ? __frcp_rn(s) : 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int vi = threadIdx.x + 256 * i;
            if (vi < nvec) store_codes<VE>(kc + e0 + (int64_t)vi * VE, x[i], s, r);
        }
        if (threadIdx.x == 0) k_scale[p] = s;
    }
    vmax = block_max(vmax, sm);
    if (threadIdx.x == 0) atomicMax(&hdr->amax_bits[1], __float_as_uint(vmax));
}

// Scheme B pass 1: max|K| and max|V| over the whole tensors.
template <typename T>
__global__ void __launch_bounds__(256) quant_amax_kernel(const T *__restrict__ k, const T *__restrict__ v,
                                                         int64_t nvec, WsHeader *hdr) {
    constexpr int VE = Vec<T>::VE;
    __shared__ float sm[32];
    const uint4 *kp = reinterpret_cast<const uint4 *>(k);
    const uint4 *vp = reinterpret_cast<const uint4 *>(v);
    float km = 0.f, vm = 0.f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nvec; i += (int64_t)gridDim.x * blockDim.x) {
        float x[VE], y[VE];
        Vec<T>::unpack(__ldcs(kp + i), x);
        Vec<T>::unpack(__ldcs(vp + i), y);
#pragma unroll
        for (int j = 0; j < VE; ++j) {
            km = fmaxf(km, fabsf(x[j]));
            vm = fmaxf(vm, fabsf(y[j]));
        }
    }
    km = block_max(km, sm);
    vm = block_max(vm, sm);
    if (threadIdx.x == 0) {
        atomicMax(&hdr->amax_bits[0], __float_as_uint(km));
        atomicMax(&hdr->amax_bits[1], __float_as_uint(vm));
    }
}

constexpr int kGlobalUnroll = 4;  // independent 16-byte loads per thread and tensor

// Pass 2: codes of one or two whole tensors with their global scales.  Optionally also the L2
// norm of every row (token) of one of them (vnorm_of = 0 or 1: x0 or x1; -1: none) into vnorm:
// a row's vpr 16-byte vectors sit on vpr consecutive lanes of one warp (vpr divides 32; the
// grid-stride index keeps warps aligned), so the row's sum of squares is a shuffle tree over
// them.  Loop bounds are taken per warp so that every lane reaches every shuffle.
// SAT (calibrated scales): scale0 and scale1 are inputs, read instead of written, and the codes
// saturate (codes4_sat); otherwise each scale is max|x| / 127 from the header and is written out.
template <typename T, bool NORMS, bool SAT>
__global__ void __launch_bounds__(256) quant_global_kernel(const T *__restrict__ x0, int8_t *__restrict__ c0,
                                                           float *scale0, int which0, const T *__restrict__ x1,
                                                           int8_t *__restrict__ c1, float *scale1, int which1,
                                                           int64_t nvec, WsHeader *hdr,
                                                           float *__restrict__ vnorm, int vnorm_of, int vpr) {
    constexpr int VE = Vec<T>::VE;
    const bool report = blockIdx.x == 0 && threadIdx.x == 0;
    float s0, s1 = 0.f;
    if constexpr (SAT) {
        s0 = calibrated_scale(scale0, &hdr->status, report);
        if (x1) s1 = calibrated_scale(scale1, &hdr->status, report);
    } else {
        s0 = __fdiv_rn(__uint_as_float(hdr->amax_bits[which0]), 127.f);
        if (x1) s1 = __fdiv_rn(__uint_as_float(hdr->amax_bits[which1]), 127.f);
        if (report) {
            *scale0 = s0;
            if (x1) *scale1 = s1;
        }
    }
    const float r0 = (s0 != 0.f) ? __frcp_rn(s0) : 0.f, r1 = (s1 != 0.f) ? __frcp_rn(s1) : 0.f;
    const float cl0 = 127.f * s0, cl1 = 127.f * s1;  // saturation bounds (SAT)
    const int lane = NORMS ? (threadIdx.x & 31) : 0;  // without norms no loop bound is taken per warp
    auto row_norm = [&](const float (&x)[VE], int64_t iv, bool in) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < VE; ++e) ss = fmaf(x[e], x[e], ss);
        for (int o = vpr >> 1; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (in && lane % vpr == 0) vnorm[iv / vpr] = sqrtf(ss);
    };
    const uint4 *p0 = reinterpret_cast<const uint4 *>(x0);
    const uint4 *p1 = reinterpret_cast<const uint4 *>(x1);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // kGlobalUnroll vectors per thread in flight per tensor, then their codes
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    for (; (i - lane) + (NORMS ? 31 : 0) + (kGlobalUnroll - 1) * stride < nvec; i += kGlobalUnroll * stride) {
        uint4 w0[kGlobalUnroll], w1[kGlobalUnroll];
#pragma unroll
        for (int u = 0; u < kGlobalUnroll; ++u) w0[u] = __ldcs(p0 + i + u * stride);
        if (x1) {
#pragma unroll
            for (int u = 0; u < kGlobalUnroll; ++u) w1[u] = __ldcs(p1 + i + u * stride);
        }
#pragma unroll
        for (int u = 0; u < kGlobalUnroll; ++u) {
            float x[VE];
            Vec<T>::unpack(w0[u], x);
            store_codes<VE, SAT>(c0 + (i + u * stride) * VE, x, s0, r0, cl0);
            if (NORMS && vnorm_of == 0) row_norm(x, i + u * stride, true);
            if (x1) {
                Vec<T>::unpack(w1[u], x);
                store_codes<VE, SAT>(c1 + (i + u * stride) * VE, x, s1, r1, cl1);
                if (NORMS && vnorm_of == 1) row_norm(x, i + u * stride, true);
            }
        }
    }
    for (; i - lane < nvec; i += stride) {  // the rest (with norms: every lane of the warp together)
        const bool in = i < nvec;
        float x[VE];
        Vec<T>::unpack(in ? __ldcs(p0 + i) : make_uint4(0, 0, 0, 0), x);
        if (in) store_codes<VE, SAT>(c0 + i * VE, x, s0, r0, cl0);
        if (NORMS && vnorm_of == 0) row_norm(x, i, in);
        if (x1) {
            Vec<T>::unpack(in ? __ldcs(p1 + i) : make_uint4(0, 0, 0, 0), x);
            if (in) store_codes<VE, SAT>(c1 + i * VE, x, s1, r1, cl1);
            if (NORMS && vnorm_of == 1) row_norm(x, i, in);
        }
    }
}

// Resident CTAs per SM of one quant_global_kernel instantiation on the current device (cached
// per device and instantiation: the variant with norms holds more registers).
template <typename K>
static int ctas_per_sm(K kern, int slot) {
    static int cache[64][8] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || slot < 0 || slot >= 8) return 3;
    if (cache[dev][slot] == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 256, 0) != cudaSuccess || n < 1) n = 3;
        cache[dev][slot] = n;
    }
    return cache[dev][slot];
}

// One launch of quant_global_kernel over all of x0 (and x1): codes with per-tensor scales, the
// calibrated (`sat`) or the computed ones, and optionally the norms of one tensor's rows.  One
// CTA per resident slot: the grid-stride loop then ends in one wave.
template <typename T>
static cudaError_t launch_global(bool sat, const T *x0, int8_t *c0, float *scale0, int which0, const T *x1,
                                 int8_t *c1, float *scale1, int which1, int64_t nvec, WsHeader *hdr, float *vnorm,
                                 int vnorm_of, int vpr, int sm_count, cudaStream_t s) {
    auto kern = sat ? (vnorm ? quant_global_kernel<T, true, true> : quant_global_kernel<T, false, true>)
                    : (vnorm ? quant_global_kernel<T, true, false> : quant_global_kernel<T, false, false>);
    const int slot = (sizeof(T) == 2 ? 4 : 0) + (sat ? 2 : 0) + (vnorm ? 1 : 0);
    return launch_k(kern, dim3(sm_count * ctas_per_sm(kern, slot)), dim3(256), 0, s, 1, x0, c0, scale0, which0, x1,
                    c1, scale1, which1, nvec, hdr, vnorm, vnorm_of, vpr);
}

template <typename T, int D>
static int quantize_impl(const T *k, const T *v, const int32_t *cu, int B, int Hkv, int64_t Ttot,
                         sgd_scheme scheme, int64_t n_parts, int8_t *kc, int8_t *vc, float *k_scale,
                         float *v_scale, float *vnorm, WsHeader *hdr, int32_t *seq_part0, int sm_count,
                         cudaStream_t s) {
    constexpr int VE = Vec<T>::VE;
    const bool cal = scheme == SGD_SCHEME_A_CALIBRATED || scheme == SGD_SCHEME_B_CALIBRATED;
    const bool partitions = scheme == SGD_SCHEME_A || scheme == SGD_SCHEME_A_CALIBRATED;
    const int64_t nvec = (int64_t)Hkv * Ttot * D / VE;
    cudaError_t e = launch_k(quant_prep_kernel, dim3(1), dim3(1024), 0, s, 1, cu, B, n_parts, (int)partitions,
                             seq_part0, hdr);
    if (e != cudaSuccess) return (int)e;
    const int grid_stream = sm_count * 8;
    const T *none = nullptr;
    int8_t *no_codes = nullptr;
    float *no_scale = nullptr;
    if (partitions) {
        const int64_t total = (int64_t)Hkv * n_parts;
        const int grid = (int)std::min<int64_t>(total, (int64_t)sm_count * 8);
        if (grid > 0) {
            e = launch_k(quant_k_partition_kernel<T, D>, dim3(grid), dim3(256), 0, s, 1, k, v, cu,
                           (const int32_t *)seq_part0, B, Hkv, Ttot, n_parts, kc, k_scale, hdr);
            if (e != cudaSuccess) return (int)e;
        }
        e = launch_global(cal, v, vc, v_scale, 1, none, no_codes, no_scale, 0, nvec, hdr, vnorm, 0, D / VE, sm_count,
                          s);
    } else {
        if (!cal) {  // calibrated scales need no maxima
            e = launch_k(quant_amax_kernel<T>, dim3(grid_stream), dim3(256), 0, s, 1, k, v, nvec, hdr);
            if (e != cudaSuccess) return (int)e;
        }
        e = launch_global(cal, k, kc, k_scale, 0, v, vc, v_scale, 1, nvec, hdr, vnorm, 1, D / VE, sm_count, s);
    }
    return (int)e;
}

// The second pass of the fused quantise-and-select (dynamic scales only): the V codes (scheme
// A) or the K and V codes (scheme B) with the maxima the score pass took.
template <typename T>
static int quantize_global_impl(const T *k, const T *v, int Hkv, int D, int64_t Ttot, sgd_scheme scheme, int8_t *kc,
                                int8_t *vc, float *k_scale, float *v_scale, float *vnorm, WsHeader *hdr,
                                int sm_count, cudaStream_t s) {
    const int64_t nvec = (int64_t)Hkv * Ttot * D / Vec<T>::VE;
    const int vpr = D / Vec<T>::VE;
    if (scheme == SGD_SCHEME_A)
        return (int)launch_global<T>(false, v, vc, v_scale, 1, nullptr, nullptr, nullptr, 0, nvec, hdr, vnorm, 0,
                                     vpr, sm_count, s);
    return (int)launch_global<T>(false, k, kc, k_scale, 0, v, vc, v_scale, 1, nvec, hdr, vnorm, 1, vpr, sm_count, s);
}

int launch_quantize_global(const void *k, const void *v, sgd_dtype dt, int Hkv, int D, int64_t T,
                           sgd_scheme scheme, int8_t *kc, int8_t *vc, float *k_scale, float *v_scale,
                           float *vnorm, WsHeader *hdr, int sm_count, cudaStream_t s) {
    if (dt == SGD_BF16)
        return quantize_global_impl(static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v),
                                    Hkv, D, T, scheme, kc, vc, k_scale, v_scale, vnorm, hdr, sm_count, s);
    return quantize_global_impl(static_cast<const float *>(k), static_cast<const float *>(v), Hkv, D, T, scheme, kc,
                                vc, k_scale, v_scale, vnorm, hdr, sm_count, s);
}

int launch_quantize(const void *k, const void *v, sgd_dtype dt, const int32_t *cu, int B, int Hkv, int D,
                    int64_t T, sgd_scheme scheme, int64_t n_parts, int8_t *kc, int8_t *vc, float *k_scale,
                    float *v_scale, float *vnorm, WsHeader *hdr, int32_t *seq_part0, int sm_count, cudaStream_t s) {
    if (dt == SGD_BF16) {
        auto kk = static_cast<const __nv_bfloat16 *>(k), vv = static_cast<const __nv_bfloat16 *>(v);
        return D == 128 ? quantize_impl<__nv_bfloat16, 128>(kk, vv, cu, B, Hkv, T, scheme, n_parts, kc, vc, k_scale,
                                                            v_scale, vnorm, hdr, seq_part0, sm_count, s)
                        : quantize_impl<__nv_bfloat16, 64>(kk, vv, cu, B, Hkv, T, scheme, n_parts, kc, vc, k_scale,
                                                           v_scale, vnorm, hdr, seq_part0, sm_count, s);
    }
    auto kk = static_cast<const float *>(k), vv = static_cast<const float *>(v);
    return D == 128 ? quantize_impl<float, 128>(kk, vv, cu, B, Hkv, T, scheme, n_parts, kc, vc, k_scale, v_scale,
                                                vnorm, hdr, seq_part0, sm_count, s)
                    : quantize_impl<float, 64>(kk, vv, cu, B, Hkv, T, scheme, n_parts, kc, vc, k_scale, v_scale,
                                               vnorm, hdr, seq_part0, sm_count, s);
}

}  // namespace sgd
