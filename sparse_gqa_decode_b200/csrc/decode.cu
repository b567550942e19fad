// decode.cu -- split-KV flash-decoding kernels, the OAM score kernel that shares their
// pipeline, and the exact log-sum-exp merge.
//
// Sources: "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse
// attention) section 5 (split the KV of a row across CTAs; each chunk reports a
// partial result that an online-softmax reduction combines) and section 3 (OAM
// score); "注意力优化（Attention Optimization）" core principle (running max m and
// sum l with a rescaled accumulator, the FlashAttention recurrence); "共同设计 AI
// 模型注意力..." (Co-designing AI model attention), decode equations 5-7: decode
// reads every KV byte once at about 2G flops per byte, far below the tensor-core
// ridge, so the kernel is built around streaming HBM at full rate.
//
// Tensor-core decode kernel (kv BF16 with D in {64,128}, or INT8 codes with D = 128):
//   * one producer warp streams the CTA's token range through a 3-stage ring of
//     shared-memory tiles (K and V, ROWS tokens each).  Dense rows are fetched with
//     2-D TMA boxes (cp.async.bulk.tensor, 128-byte swizzle, L2 evict-first);
//     kept-index rows are gathered with 16-byte cp.async into the same swizzled
//     layout.  Full/empty mbarriers hand stages between producer and consumers; every
//     wait is bounded.
//   * four consumer warps each own 16-token sub-tiles.  QK: S^T[token, g] with
//     m16n8k16 MMAs (tokens as M, the G heads of the group as N, D as K); the fp32
//     logits get the dequantisation scales and 1/sqrt(D); online softmax in the log2
//     domain; P is transposed in registers (movmatrix) into the B operand of the
//     PV MMA O^T[d, g] += V^T[d, token] P^T[token, g].  INT8 codes are widened to f16
//     in registers (exact), Q is pre-scaled by a power of two into f16 range.
//   * rows of a 16-token MMA tile are permuted (0,5,2,7,4,1,6,3) so that the
//     swizzled shared-memory reads of both K and V are bank-conflict free.
//   * at the end of each (row, token range) segment the four warps' (m, l, O) are
//     combined through shared memory into one partial (o_c, lse_c).
// The same pipeline scores tokens (OAM, mode 1) and, with eight more warps that quantise
// each 64-token K tile (one scheme-A partition) while the consumer warps score it, runs the
// one-pass quantise-and-select (mode 2); with calibrated per-tensor scales those warps also
// write the V codes and the value norms.
// CUDA-core kernel: every other dtype/shape (F32 cache, INT8 with D = 64, ...).
#include <math.h>

#include <cudaTypedefs.h>

#include "internal.h"
#include "plan.cuh"
#include "quant.cuh"

namespace sgd {

constexpr float kLn2 = 0.69314718055994530942f;

__device__ __forceinline__ int mma_row_perm(int i) { return (i & 1) ? (i ^ 4) : i; }

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

constexpr int kQuantWarps = 8;  // K-quantising warps of the fused score + quantise pass

template <int D_, int GT_, bool I8_, bool IDX_, int MODE_, bool QI8_ = false, bool CAUSAL_ = false,
          bool BLK_ = false, bool CAL_ = false>
struct MmaCfg {
    static constexpr int D = D_, GT = GT_, NG = 8 * GT_;
    static constexpr bool I8 = I8_, IDX = IDX_;
    static constexpr bool QI8 = QI8_;  // INT8 query codes: S^T = K_codes . Q_codes^T on s8 MMAs
    static constexpr bool CAUSAL = CAUSAL_;  // several query tokens: causal limit per column
    static constexpr bool BLK = BLK_;  // kept 64-token blocks: one TMA box per block, at its start
    static constexpr int MODE = MODE_;  // 0 = decode, 1 = OAM score, 2 = OAM score + K quantise + max|V|
    static constexpr bool CAL = CAL_;   // mode 2 with calibrated per-tensor scales: every code in the pass
    static constexpr bool KONLY = I8 && MODE == 1;  // scores of an INT8 cache: K tiles only
    static constexpr int NW = 4;        // consumer warps
    static constexpr int SUB = I8 ? 2 : 1;  // 16-token sub-tiles per consumer warp per stage
    static constexpr int ROWS = NW * 16 * SUB;
    static constexpr int EB = I8 ? 1 : 2;
    static constexpr int ROWB = D * EB;
    static constexpr int BOXES = ROWB / 128;
    static constexpr int BOX_ELEMS = 128 / EB;
    static constexpr int BOX_ROWS = BLK ? kPart : ROWS;  // rows of one TMA box
    static constexpr int TILE = ROWS * ROWB;  // bytes of one tensor per stage
    static constexpr int STAGES = 3;
    // CTAs per SM the registers must allow: the K-only score of an INT8 cache has half-size stages
    // and is issue-bound, so a third CTA (more consumer warps) fits and pays
    static constexpr int MINB = KONLY ? 4 : 2;
    static constexpr int KB = D / 16;
    static constexpr int NQ = (MODE == 2) ? kQuantWarps : 0;  // K-quantising warps (mode 2)
    static constexpr int THREADS = (NW + NQ + 1) * 32;
    static constexpr int STAGE_BYTES = (KONLY ? 1 : 2) * TILE;  // K tile, then V tile
    static constexpr int SMEM_STAGES = STAGES * STAGE_BYTES;
    static constexpr bool ROW_SCALE = I8 && IDX;  // per-row K scales fetched by the producer
    static constexpr int SMEM_ROWSCALE = ROW_SCALE ? STAGES * ROWS * 4 : 0;
    static constexpr int SMEM_KMX = 2 * (NQ > 4 ? NQ : 4) * 4;  // [2][NQ] per-warp max|K| (mode 2)
    // two column tiles of the decode: the Q fragments wait in shared memory (each lane its own
    // 8 bytes per fragment pair) instead of 32-64 registers that the softmax and PV phases need
    static constexpr bool QS = GT == 2 && MODE == 0;
    static constexpr int SMEM_Q = QS ? GT * KB * 32 * 8 : 0;
    static constexpr int SMEM = 1024 + SMEM_STAGES + 2 * STAGES * 8 + NW * NG * 2 * 4 + 16 + SMEM_KMX + SMEM_ROWSCALE +
                                SMEM_Q;
    static_assert(ROWB % 128 == 0, "rows are whole 128-byte boxes");
    static_assert(NW * NG * D * 4 <= 2 * TILE, "epilogue fits in one stage");
    static_assert(!(I8 && MODE == 2), "the fused pass reads the unquantised cache");
    static_assert(!QI8 || (I8 && MODE == 0 && D == 128), "query codes meet INT8 keys in the decode");
    static_assert(!CAUSAL || MODE == 0, "several query tokens: decode only");
    static_assert(!BLK || (MODE == 0 && !IDX && !CAUSAL && ROWS % kPart == 0), "a tile is whole blocks");
    static_assert(MODE != 2 || ROWS == kPart, "a fused tile is one scheme-A partition");
    static_assert(!CAL || MODE == 2, "calibrated scales: the fused pass");
};

// ------------------------------------------------------------------------------------------
// producer warp
// ------------------------------------------------------------------------------------------
template <class C>
__device__ __forceinline__ void mma_producer(const CUtensorMap *tmK, const CUtensorMap *tmV, const DecodeArgs &a,
                                             uint8_t *smem, uint64_t *full, uint64_t *empty,
                                             volatile int32_t *abort_flag, float *row_scale,
                                             int cta, int lane) {
    if (!C::IDX && lane != 0) return;
    if (a.idle_producer) return;  // test aid: nothing is issued, so every consumer wait runs out
    uint64_t pol = 0;
    if constexpr (!C::IDX) {
        prefetch_tensormap(tmK);
        prefetch_tensormap(tmV);
        pol = l2_evict_first_policy();
    }
    SegCursor cur;
    cur.init(a.plan, a.B * a.Hkv, cta);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t filled = 0, fill_par = 0;  // per stage: filled at least once; parity of its last fill
    bool stop = false;
    int row, slot;
    int32_t t0, t1;
    while (!stop && cur.next(row, t0, t1, slot)) {
        const int b = row % a.B, kvh = row / a.B;
        const int64_t seq0 = (int64_t)kvh * a.T + cur.ri.seq_start;
        const int32_t Lb = cur.ri.seq_len;
        const int32_t *ip = nullptr;
        if constexpr (C::IDX) ip = a.idx + (int64_t)kvh * a.Kt + cur.ri.len_start;
        const float *ksc = nullptr;
        if constexpr (C::ROW_SCALE) ksc = a.k_scale + (int64_t)kvh * a.n_parts + cur.ri.part0;
        // Gathers: the row indices of the next kPrefetch tiles are loaded ahead in registers
        // (lane l holds those of rows l, l+32, ... of a tile), so a segment waits for its index
        // loads once and not before every tile.
        constexpr int RPL = C::IDX ? C::ROWS / 32 : 1;  // row indices held per lane and tile
        constexpr int kPrefetch = 2;
        int32_t tk[kPrefetch + 1][RPL];
        auto load_tile_idx = [&](int32_t (&dst)[RPL], int32_t tt) {
#pragma unroll
            for (int qi = 0; qi < RPL; ++qi)  // rows past the segment repeat its last token
                dst[qi] = (tt < t1) ? __ldg(ip + min(tt + lane + 32 * qi, t1 - 1)) : 0;
        };
        if constexpr (C::IDX) {
#pragma unroll
            for (int j = 0; j <= kPrefetch; ++j) load_tile_idx(tk[j], t0 + j * C::ROWS);
        }
        // kept blocks: the block numbers of this tile and the next (-1 past the segment), checked
        constexpr int NBT = C::BLK ? C::ROWS / kPart : 1;
        int32_t blk_cur[NBT], blk_nxt[NBT];
        const int32_t *bp = nullptr;
        if constexpr (C::BLK) bp = a.idx + (int64_t)kvh * a.Kt + cur.ri.len_start / kPart;
        const int32_t nblk = (Lb + kPart - 1) / kPart;
#pragma unroll
        for (int i = 0; i < NBT; ++i) blk_nxt[i] = -1;
        auto load_tile_blk = [&](int32_t tt) {
#pragma unroll
            for (int i = 0; i < NBT; ++i) {
                blk_cur[i] = blk_nxt[i];
                const int32_t u = tt + i * kPart;
                int32_t v = -1;
                if (u < t1) {
                    v = __ldg(bp + u / kPart);
                    if (v < 0 || v >= nblk) {  // out of range: reported, clamped (nothing loaded if none)
                        atomicOr(a.status, SGD_STATUS_BAD_INDEX);
                        v = (nblk > 0) ? min(max(v, 0), nblk - 1) : -1;
                    }
                }
                blk_nxt[i] = v;
            }
        };
        if constexpr (C::BLK) {
            load_tile_blk(t0);
            load_tile_blk(t0 + C::ROWS);
        }
        for (int32_t t = t0; t < t1; t += C::ROWS) {
            // a consumer that gave up still releases its stages: after any wait, the abort flag
            // (raised before that release) says whether the stage was really consumed
            bool ok = mbar_wait(&empty[stage], phase ^ 1, a.status, abort_flag, a.wait_limit) && !*abort_flag;
            if constexpr (C::IDX) ok = __all_sync(0xffffffffu, ok);  // the gathers need the whole warp
            if (!ok) {
                stop = true;
                break;
            }
            filled |= 1u << stage;
            fill_par = (fill_par & ~(1u << stage)) | (phase << stage);
            uint8_t *sk = smem + stage * C::STAGE_BYTES;
            uint8_t *sv = sk + C::TILE;
            if constexpr (C::BLK) {
                // the tile's kept blocks (t and t1 are multiples of 64 in the row's padded block
                // stream), each one box per tensor and 128-byte column, at its own cache row
                constexpr int NB = C::ROWS / kPart;
                int nload = 0;
#pragma unroll
                for (int i = 0; i < NB; ++i) nload += (blk_cur[i] >= 0) ? 1 : 0;
                mbar_arrive_expect_tx(&full[stage], nload * 2 * (C::TILE / NB));
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    if (blk_cur[i] < 0) continue;
                    const int y = (int)(seq0 + (int64_t)blk_cur[i] * kPart);
#pragma unroll
                    for (int bx = 0; bx < C::BOXES; ++bx) {
                        const int off = bx * C::ROWS * 128 + i * kPart * 128;
                        tma_load_2d(sk + off, tmK, &full[stage], bx * C::BOX_ELEMS, y, pol);
                        tma_load_2d(sv + off, tmV, &full[stage], bx * C::BOX_ELEMS, y, pol);
                    }
                }
                load_tile_blk(t + 2 * C::ROWS);
            } else if constexpr (!C::IDX) {
                mbar_arrive_expect_tx(&full[stage], (C::KONLY ? 1 : 2) * C::TILE);
                const int y = (int)(seq0 + t);
#pragma unroll
                for (int bx = 0; bx < C::BOXES; ++bx) {
                    tma_load_2d(sk + bx * C::ROWS * 128, tmK, &full[stage], bx * C::BOX_ELEMS, y, pol);
                    if constexpr (!C::KONLY)
                        tma_load_2d(sv + bx * C::ROWS * 128, tmV, &full[stage], bx * C::BOX_ELEMS, y, pol);
                }
            } else if (Lb >= 1) {
                // Row indices: lane l loads those of rows l, l+32, ...  Copies: one warp
                // instruction moves whole rows (CPR lanes per row, one 16-byte chunk each), so
                // every row reaches L2 as one contiguous request per tensor.
                constexpr int CPR = C::ROWB / 16;  // 16-byte chunks per row
                constexpr int RPI = 32 / CPR;      // rows per copy instruction
                int32_t toks[RPL];
#pragma unroll
                for (int qi = 0; qi < RPL; ++qi) {
                    int32_t tok = tk[0][qi];
                    if (tok < 0 || tok >= Lb) {
                        atomicOr(a.status, SGD_STATUS_BAD_INDEX);
                        tok = min(max(tok, 0), Lb - 1);
                    }
                    toks[qi] = tok;
                }
                const int c = lane % CPR, bx = c >> 3, cc = c & 7;
#pragma unroll
                for (int it = 0; it < C::ROWS / RPI; ++it) {
                    const int rr = it * RPI + lane / CPR;  // this lane's row in this instruction
                    const int32_t tok = __shfl_sync(0xffffffffu, toks[(it * RPI) / 32], rr & 31);
                    const int64_t src = (seq0 + tok) * C::ROWB + c * 16;
                    const int off = bx * C::ROWS * 128 + rr * 128 + ((cc ^ (rr & 7)) << 4);
                    cp_async_16(sk + off, static_cast<const uint8_t *>(a.k) + src);
                    cp_async_16(sv + off, static_cast<const uint8_t *>(a.v) + src);
                }
                if constexpr (C::ROW_SCALE) {
                    if (a.scheme == SGD_SCHEME_A) {
#pragma unroll
                        for (int qi = 0; qi < RPL; ++qi)
                            cp_async_4(row_scale + stage * C::ROWS + lane + 32 * qi, ksc + toks[qi] / kPart);
                    }
                }
                cp_async_mbar_arrive_noinc(&full[stage]);
            } else {
                // rows of an empty sequence (inconsistent kept counts): nothing to fetch
                if (lane == 0) atomicOr(a.status, SGD_STATUS_SIZE_MISMATCH);
                mbar_arrive(&full[stage]);
            }
            if constexpr (C::IDX) {
#pragma unroll
                for (int j = 0; j < kPrefetch; ++j)
#pragma unroll
                    for (int qi = 0; qi < RPL; ++qi) tk[j][qi] = tk[j + 1][qi];
                load_tile_idx(tk[kPrefetch], t + (kPrefetch + 1) * C::ROWS);
            }
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1;
            }
        }
    }
    // Before the producer (and with it, eventually, the CTA) ends, every copy it issued has
    // landed: the consumers may have given up on a stage whose copy is still in flight.
    if constexpr (C::IDX) {
        cp_async_wait_all();
    } else {
#pragma unroll
        for (int st = 0; st < C::STAGES; ++st)
            if ((filled >> st) & 1u) mbar_drain(&full[st], (fill_par >> st) & 1u, a.wait_limit);
    }
}

// ------------------------------------------------------------------------------------------
// consumer helpers
// ------------------------------------------------------------------------------------------
// Element offset of column n's row in q [B, M, Hq, D] (and out): the columns of KV head kvh are
// its M * G (query token, head) pairs, n = m * G + g.
__device__ __forceinline__ int64_t col_row(const DecodeArgs &a, int b, int kvh, int n) {
    const int m = (a.M == 1) ? 0 : n / a.G, g = n - m * a.G;
    return (((int64_t)b * a.M + m) * a.Hkv + kvh) * a.G + g;
}

// Q of one KV group as MMA B fragments (k <-> d order matching the K fragments) and the
// per-column logit factor (log2 units; INT8 also undoes the power-of-two Q pre-scale).
template <class C>
__device__ __forceinline__ void load_q_frags(const DecodeArgs &a, int b, int kvh, int g4, int t4,
                                             uint32_t (&qf)[C::GT][C::KB][2], float (&colf)[C::GT][2], int col0 = 0) {
#pragma unroll
    for (int gt = 0; gt < C::GT; ++gt) {
        const int g = col0 + 8 * gt + g4;  // column: this CTA's column group starts at col0
        const bool live = g < a.G * a.M;
        const __nv_bfloat16 *qrow = static_cast<const __nv_bfloat16 *>(a.q) + col_row(a, b, kvh, live ? g : 0) * C::D;
        if constexpr (!C::I8) {
#pragma unroll
            for (int h = 0; h < C::KB / 2; ++h) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (live) v = __ldg(reinterpret_cast<const uint4 *>(qrow) + (t4 + 4 * h));
                qf[gt][2 * h][0] = v.x;
                qf[gt][2 * h][1] = v.y;
                qf[gt][2 * h + 1][0] = v.z;
                qf[gt][2 * h + 1][1] = v.w;
            }
            colf[gt][0] = colf[gt][1] = a.sm_scale_log2;
        } else {
            float x[C::KB / 4][16];
            float mx = 0.f;
#pragma unroll
            for (int h = 0; h < C::KB / 4; ++h) {
                uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
                if (live) {
                    const uint4 *p = reinterpret_cast<const uint4 *>(qrow + 16 * (t4 + 4 * h));
                    v0 = __ldg(p);
                    v1 = __ldg(p + 1);
                }
                const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    x[h][2 * i] = __uint_as_float(w[i] << 16);
                    x[h][2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
                    mx = fmaxf(mx, fmaxf(fabsf(x[h][2 * i]), fabsf(x[h][2 * i + 1])));
                }
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            if constexpr (C::QI8) {
                // the head's query codes ([TD] section 6 on Q): scale max|q|/127 of this (sequence,
                // head) row, or the tensor's; the lane's chunk c = t4 + 4h gives two s8 MMAs (bytes
                // 0-7, 8-15), in the k order qk_subtile reads the K chunk in
                const float sq = a.q_quant == 2 ? __ldg(a.q_scale) : __fdiv_rn(mx, 127.f);
                const float rq = (sq != 0.f) ? __frcp_rn(sq) : 0.f;
#pragma unroll
                for (int h = 0; h < C::KB / 4; ++h)
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        qf[gt][2 * h + m][0] = (sq != 0.f) ? codes4(&x[h][8 * m], sq, rq) : 0u;
                        qf[gt][2 * h + m][1] = (sq != 0.f) ? codes4(&x[h][8 * m + 4], sq, rq) : 0u;
                    }
                const float s0 = __shfl_sync(0xffffffffu, sq, 4 * (2 * t4));
                const float s1 = __shfl_sync(0xffffffffu, sq, 4 * (2 * t4 + 1));
                float f = a.sm_scale_log2;
                if (a.scheme == SGD_SCHEME_B) f *= __ldg(a.k_scale);
                colf[gt][0] = f * s0;
                colf[gt][1] = f * s1;
                continue;
            }
            int ex = 0;
            if (mx > 0.f) frexpf(mx, &ex);
            const int sh = 14 - ex;  // max |q| * 2^sh < 2^14: inside f16 range
#pragma unroll
            for (int h = 0; h < C::KB / 4; ++h)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    qf[gt][4 * h + j][0] = pack_f16(ldexpf(x[h][4 * j], sh), ldexpf(x[h][4 * j + 1], sh));
                    qf[gt][4 * h + j][1] = pack_f16(ldexpf(x[h][4 * j + 2], sh), ldexpf(x[h][4 * j + 3], sh));
                }
            // column factor of this thread's columns g0 = 8gt + 2t4 and g0 + 1: their rows live on
            // lanes 4 * (2t4) and 4 * (2t4 + 1)
            const float inv = ldexpf(1.f, -sh);
            const float i0 = __shfl_sync(0xffffffffu, inv, 4 * (2 * t4));
            const float i1 = __shfl_sync(0xffffffffu, inv, 4 * (2 * t4 + 1));
            float f = a.sm_scale_log2;
            if (a.scheme == SGD_SCHEME_B) f *= __ldg(a.k_scale);
            colf[gt][0] = f * i0;
            colf[gt][1] = f * i1;
        }
    }
}

// S^T = K_tile(16 x D) * Q^T(D x NG) for this warp's sub-tile.
template <class C>
__device__ __forceinline__ void qk_subtile(uint32_t kbase, int rb, int pA, int t4,
                                           const uint32_t (&qf)[C::GT][C::KB][2], float (&sacc)[C::GT][4],
                                           uint32_t qsm = 0) {
    // fragment pair x of column tile gt: registers, or this lane's 8 bytes in shared memory
    auto qv = [&](int gt, int x) -> uint2 {
        if constexpr (C::QS) return lds64(qsm + (gt * C::KB + x) * 256);
        else return make_uint2(qf[gt][x][0], qf[gt][x][1]);
    };
#pragma unroll
    for (int gt = 0; gt < C::GT; ++gt) sacc[gt][0] = sacc[gt][1] = sacc[gt][2] = sacc[gt][3] = 0.f;
    const int rA = rb + pA, rB = rA + 8;
    if constexpr (!C::I8) {
#pragma unroll
        for (int h = 0; h < C::KB / 2; ++h) {
            const int c = t4 + 4 * h, bx = c >> 3, cc = c & 7;
            const uint32_t base = kbase + bx * C::ROWS * 128 + ((cc ^ pA) << 4);
            const uint4 ka = lds128(base + rA * 128), kb = lds128(base + rB * 128);
#pragma unroll
            for (int gt = 0; gt < C::GT; ++gt) {
                const uint2 q0 = qv(gt, 2 * h), q1 = qv(gt, 2 * h + 1);
                mma_bf16(sacc[gt], ka.x, kb.x, ka.y, kb.y, q0.x, q0.y);
                mma_bf16(sacc[gt], ka.z, kb.z, ka.w, kb.w, q1.x, q1.y);
            }
        }
    } else if constexpr (C::QI8) {
        // s8 x s8 -> s32: two m16n8k32 MMAs per 16-byte chunk of the row (its bytes 0-7 and 8-15 are
        // k 0..3 / 16..19 and so on of one MMA: the query codes follow the same order)
        int32_t ia[C::GT][4];
#pragma unroll
        for (int gt = 0; gt < C::GT; ++gt) ia[gt][0] = ia[gt][1] = ia[gt][2] = ia[gt][3] = 0;
#pragma unroll
        for (int h = 0; h < C::KB / 4; ++h) {
            const int c = t4 + 4 * h;
            const uint32_t base = kbase + ((c ^ pA) << 4);
            const uint4 ka = lds128(base + rA * 128), kb = lds128(base + rB * 128);
#pragma unroll
            for (int gt = 0; gt < C::GT; ++gt) {
                const uint2 q0 = qv(gt, 2 * h), q1 = qv(gt, 2 * h + 1);
                mma_s8(ia[gt], ka.x, kb.x, ka.y, kb.y, q0.x, q0.y);
                mma_s8(ia[gt], ka.z, kb.z, ka.w, kb.w, q1.x, q1.y);
            }
        }
#pragma unroll
        for (int gt = 0; gt < C::GT; ++gt)
#pragma unroll
            for (int j = 0; j < 4; ++j) sacc[gt][j] = (float)ia[gt][j];  // |sum| < 2^24: exact
    } else {
#pragma unroll
        for (int h = 0; h < C::KB / 4; ++h) {
            const int c = t4 + 4 * h;
            const uint32_t base = kbase + ((c ^ pA) << 4);
            const uint4 ka = lds128(base + rA * 128), kb = lds128(base + rB * 128);
            const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w}, wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t a0, a1, a2, a3;
                s8x4_to_f16x2x2(wa[j], a0, a2);
                s8x4_to_f16x2x2(wb[j], a1, a3);
#pragma unroll
                for (int gt = 0; gt < C::GT; ++gt) {
                    const uint2 q = qv(gt, 4 * h + j);
                    mma_f16(sacc[gt], a0, a1, a2, a3, q.x, q.y);
                }
            }
        }
    }
}

// O^T(D x NG) += V_tile^T(D x 16) * P^T(16 x NG)
template <class C>
__device__ __forceinline__ void pv_subtile(uint32_t vbase, int rb, int lane, const uint32_t (&pb)[C::GT][2],
                                           float (&o)[C::GT][C::KB][4]) {
    if constexpr (!C::I8) {
        const int lrow = rb + mma_row_perm(lane & 7) + ((lane >> 4) << 3);
        const int lhalf = (lane >> 3) & 1;
        const int sw = lrow & 7;
#pragma unroll
        for (int mt = 0; mt < C::KB; ++mt) {
            const int c = 2 * mt + lhalf, bx = c >> 3, cc = c & 7;
            uint32_t va[4];
            ldmatrix_x4_trans(va, vbase + bx * C::ROWS * 128 + lrow * 128 + ((cc ^ sw) << 4));
#pragma unroll
            for (int gt = 0; gt < C::GT; ++gt) mma_bf16(o[gt][mt], va[0], va[1], va[2], va[3], pb[gt][0], pb[gt][1]);
        }
    } else {
        const int g4 = lane >> 2, t4 = lane & 3;
        const int tA = rb + 2 * t4, tB = rb + ((2 * t4 + 1) ^ 4);
        const uint32_t off = (uint32_t)(g4 ^ (tA & 7)) << 4, offB = (uint32_t)(g4 ^ (tB & 7)) << 4;
        uint4 wA = lds128(vbase + tA * 128 + off), wA8 = lds128(vbase + (tA + 8) * 128 + off);
        uint4 wB = lds128(vbase + tB * 128 + offB), wB8 = lds128(vbase + (tB + 8) * 128 + offB);
        const uint32_t A[4] = {wA.x ^ 0x80808080u, wA.y ^ 0x80808080u, wA.z ^ 0x80808080u, wA.w ^ 0x80808080u};
        const uint32_t Bv[4] = {wB.x ^ 0x80808080u, wB.y ^ 0x80808080u, wB.z ^ 0x80808080u, wB.w ^ 0x80808080u};
        const uint32_t A8[4] = {wA8.x ^ 0x80808080u, wA8.y ^ 0x80808080u, wA8.z ^ 0x80808080u,
                                wA8.w ^ 0x80808080u};
        const uint32_t B8[4] = {wB8.x ^ 0x80808080u, wB8.y ^ 0x80808080u, wB8.z ^ 0x80808080u,
                                wB8.w ^ 0x80808080u};
#pragma unroll
        for (int mt = 0; mt < C::KB; ++mt) {
            const int w = mt >> 1;
            const uint32_t slo = (mt & 1) ? 0x0062u : 0x0040u, shi = (mt & 1) ? 0x0073u : 0x0051u;
            const uint32_t a0 = biased_pair_to_f16x2(A[w], Bv[w], slo);
            const uint32_t a1 = biased_pair_to_f16x2(A[w], Bv[w], shi);
            const uint32_t a2 = biased_pair_to_f16x2(A8[w], B8[w], slo);
            const uint32_t a3 = biased_pair_to_f16x2(A8[w], B8[w], shi);
#pragma unroll
            for (int gt = 0; gt < C::GT; ++gt) mma_f16(o[gt][mt], a0, a1, a2, a3, pb[gt][0], pb[gt][1]);
        }
    }
}

// Score mode for one 16-token sub-tile: OAM score of every token (max over the group's heads
// of the logit, plus beta * ln(|v| + eps)); mode 2 also accumulates max|V|.  Every score warp
// calls this for every tile.
template <class C>
__device__ __forceinline__ void score_subtile(const DecodeArgs &a, uint32_t kbase, uint32_t vbase, int rb,
                                              int32_t j0, int32_t t1, bool ready, int64_t tok_base, int pA,
                                              int t4, int lane, const uint32_t (&qf)[C::GT][C::KB][2],
                                              float &run_vmax) {
    const bool act = ready && j0 < t1;
    float sacc[C::GT][4];
    if (act) {
        qk_subtile<C>(kbase, rb, pA, t4, qf, sacc);
    } else {
#pragma unroll
        for (int gt = 0; gt < C::GT; ++gt) sacc[gt][0] = sacc[gt][1] = sacc[gt][2] = sacc[gt][3] = 0.f;
    }
    float mA = -INFINITY, mB = -INFINITY;
#pragma unroll
    for (int gt = 0; gt < C::GT; ++gt) {
        const int g0 = 8 * gt + 2 * t4;
        if (g0 < a.G * a.M) {  // (query token, head) columns
            mA = fmaxf(mA, sacc[gt][0]);
            mB = fmaxf(mB, sacc[gt][2]);
        }
        if (g0 + 1 < a.G * a.M) {
            mA = fmaxf(mA, sacc[gt][1]);
            mB = fmaxf(mB, sacc[gt][3]);
        }
    }
    mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
    mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
    mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
    mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
    // ||v||^2 of the sub-tile's 16 rows on the tensor cores, as the diagonal of V.V^T: the rows
    // take the MMA order of qk_subtile (row g4 at rb + pA, g4 + 8 at rb + pA + 8), and the B
    // operand of rows 0-7 (8-15) is the (a0, a2) ((a1, a3)) half of the A fragment, so no further
    // loads are needed; products are exact and sums f32.  The same registers give max|v| (mode 2).
    const int rA = rb + pA, rB = rA + 8;
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t vmA = 0, vmB = 0;  // running max |v| of rows rA and rB as bf16x2 (mode 2)
#pragma unroll
    for (int h = 0; h < C::KB / 2; ++h) {
        const int c = t4 + 4 * h, bx = c >> 3, cc = c & 7;
        const uint32_t base = vbase + bx * C::ROWS * 128 + ((cc ^ pA) << 4);
        const uint4 va = lds128(base + rA * 128), vb = lds128(base + rB * 128);
        mma_bf16(d0, va.x, vb.x, va.y, vb.y, va.x, va.y);
        mma_bf16(d1, va.x, vb.x, va.y, vb.y, vb.x, vb.y);
        mma_bf16(d0, va.z, vb.z, va.w, vb.w, va.z, va.w);
        mma_bf16(d1, va.z, vb.z, va.w, vb.w, vb.z, vb.w);
        if constexpr (C::MODE == 2) {
            vmA = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(vmA, va.x), va.y), va.z), va.w);
            vmB = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(vmB, vb.x), vb.y), vb.z), vb.w);
        }
    }
    // lane 4g + g/2 holds the diagonal of MMA rows g and g + 8
    const int g4 = lane >> 2;
    const float dlo = (g4 & 1) ? d0[1] : d0[0], dhi = (g4 & 1) ? d1[3] : d1[2];
    // row rb + rho of the tile is MMA row gm (rho < 8) or gm + 8, gm = perm(rho mod 8); lane rho
    // writes its score
    const int rho = lane & 15, half = lane >> 4;
    const int32_t j = j0 + rho;
    const bool vrow = act && j < t1;
    const int gm = mma_row_perm(rho & 7);
    const int src = 4 * gm, dsrc = 4 * gm + (gm >> 1);
    const float rAm = __shfl_sync(0xffffffffu, mA, src), rBm = __shfl_sync(0xffffffffu, mB, src);
    const float slo = __shfl_sync(0xffffffffu, dlo, dsrc), shi = __shfl_sync(0xffffffffu, dhi, dsrc);
    const float rmax = (rho < 8) ? rAm : rBm;
    const float ss = (rho < 8) ? slo : shi;
    if (half == 0 && vrow) {
        float sc = rmax * a.sm_scale + a.beta * logf(sqrtf(ss) + a.eps);
        if (sc == 0.f) sc = 0.f;  // one key for +0 and -0
        a.scores[tok_base + j] = sc;
    }
    if constexpr (C::MODE == 2) {
        const bool okA = act && j0 + pA < t1, okB = act && j0 + pA + 8 < t1;
        run_vmax = fmaxf(run_vmax, fmaxf(okA ? bf16x2_fold_max(vmA) : 0.f, okB ? bf16x2_fold_max(vmB) : 0.f));
    }
}

// OAM scores of a sub-tile of an INT8 cache (mode 1): khat = code * scale, so the logit of head g
// is sacc * colf_g (log2 units, with the head's Q pre-scale) times the sub-tile's partition scale
// rf >= 0 (scheme A; scheme B's scale is inside colf); ||v_t|| (vn, lanes 0-15: row rb + lane)
// comes from the norms stored when the cache was quantised, so the V codes are never read.
template <class C>
__device__ __forceinline__ void score_subtile_i8(const DecodeArgs &a, uint32_t kbase, int rb, int32_t j0, int32_t t1,
                                                 bool ready, int64_t tok_base, int pA, int t4, int lane,
                                                 const uint32_t (&qf)[C::GT][C::KB][2], const float (&colf)[C::GT][2],
                                                 float rf, float vn) {
    const bool act = ready && j0 < t1;
    const int rho = lane & 15, half = lane >> 4;
    const int32_t j = j0 + rho;
    const bool vrow = act && j < t1;
    float sacc[C::GT][4];
    if (act) {
        qk_subtile<C>(kbase, rb, pA, t4, qf, sacc);
    } else {
#pragma unroll
        for (int gt = 0; gt < C::GT; ++gt) sacc[gt][0] = sacc[gt][1] = sacc[gt][2] = sacc[gt][3] = 0.f;
    }
    float mA = -INFINITY, mB = -INFINITY;
#pragma unroll
    for (int gt = 0; gt < C::GT; ++gt) {
        const int g0 = 8 * gt + 2 * t4;
        if (g0 < a.G * a.M) {  // (query token, head) columns
            mA = fmaxf(mA, sacc[gt][0] * colf[gt][0]);
            mB = fmaxf(mB, sacc[gt][2] * colf[gt][0]);
        }
        if (g0 + 1 < a.G * a.M) {
            mA = fmaxf(mA, sacc[gt][1] * colf[gt][1]);
            mB = fmaxf(mB, sacc[gt][3] * colf[gt][1]);
        }
    }
    mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
    mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
    mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
    mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
    const int src = 4 * mma_row_perm(rho & 7);  // row rb + rho is MMA row perm(rho mod 8) (+ 8)
    const float rAm = __shfl_sync(0xffffffffu, mA, src), rBm = __shfl_sync(0xffffffffu, mB, src);
    const float rmax = (rho < 8) ? rAm : rBm;
    if (half == 0 && vrow) {
        float sc = rmax * rf * kLn2 + a.beta * logf(vn + a.eps);
        if (sc == 0.f) sc = 0.f;  // one key for +0 and -0
        a.scores[tok_base + j] = sc;
    }
}

// Codes of NH 16-byte bf16 chunks (8 values each) to NH / 2 16-byte stores at dst (SAT: under a
// calibrated scale, codes4_sat); s == 0 gives zero codes.
template <int NH, bool SAT>
__device__ __forceinline__ void store_code_chunks(int8_t *dst, const uint4 (&cw)[NH], float s, float r, float c) {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < NH; i += 2) {  // 16 codes per 16-byte store
        float x[8], y[8];
        Vec<__nv_bfloat16>::unpack(cw[i], x);
        Vec<__nv_bfloat16>::unpack(cw[i + 1], y);
        uint4 w;
        if constexpr (SAT) {
            w.x = (s != 0.f) ? codes4_sat<true>(x, s, r, c) : 0u;
            w.y = (s != 0.f) ? codes4_sat<true>(x + 4, s, r, c) : 0u;
            w.z = (s != 0.f) ? codes4_sat<true>(y, s, r, c) : 0u;
            w.w = (s != 0.f) ? codes4_sat<true>(y + 4, s, r, c) : 0u;
        } else {
            w.x = (s != 0.f) ? codes4<true>(x, s, r) : 0u;
            w.y = (s != 0.f) ? codes4<true>(x + 4, s, r) : 0u;
            w.z = (s != 0.f) ? codes4<true>(y, s, r) : 0u;
            w.w = (s != 0.f) ? codes4<true>(y + 4, s, r) : 0u;
        }
        d[i / 2] = w;
    }
}

// Mode 2, K-quantising warp qw: rows RW*qw .. RW*qw + RW-1 of every tile (a tile is one scheme-A
// partition, RW = 64 / NQ).  Scheme A: the tile's max|K| is met across the NQ warps through shared memory,
// then each warp writes the codes of its rows and warp 0 the partition scale.  Scheme B: only
// the running max|K|.  Every quantising warp takes every tile.
// With calibrated per-tensor scales the warps also write the codes of their V rows (and, scheme
// B, of their K rows) and, if asked, each V row's norm, summed in the order the V-codes pass
// sums it (per 16-byte chunk in element order, then chunk c with c ^ 8, ^ 4, ^ 2, ^ 1), so the
// norms are the same bits whichever call writes them.
template <class C>
__device__ __forceinline__ void quant_consumer(const DecodeArgs &a, uint8_t *smem, uint64_t *full, uint64_t *empty,
                                               volatile int32_t *abort_flag, float *kmxs,
                                               int cta, int qw, int lane) {
    SegCursor cur;
    cur.init(a.plan, a.B * a.Hkv, cta);
    int stage = 0, tile_no = 0;
    uint32_t phase = 0;
    int row, slot;
    int32_t t0, t1;
    float run_kmax = 0.f;
    // each warp takes RW rows of the 64-row tile, LPR lanes per row, NH 16-byte chunks per lane
    constexpr int RW = C::ROWS / C::NQ, LPR = 32 / RW, CPR = C::ROWB / 16, NH = CPR / LPR;
    static_assert(NH % 2 == 0 && RW * LPR == 32, "quantising lane map");
    const int rho = lane % RW, half = lane / RW;  // lane: row rho of the warp, part `half` of it
    const int vr = RW * qw + rho;
    auto chunk_at = [&](uint32_t base, int i) {  // chunk half * NH + i of tile row vr (128B swizzle)
        const int c = half * NH + i, bx = c >> 3, cc = c & 7;
        return lds128(base + bx * C::ROWS * 128 + vr * 128 + ((cc ^ (vr & 7)) << 4));
    };
    constexpr bool cal = C::CAL;
    float vs = 0.f, ks = 0.f;
    if constexpr (cal) {
        const bool report = cta == 0 && qw == 0 && lane == 0;
        vs = calibrated_scale(a.cal_v_scale, a.status, report);
        if (a.qscheme == SGD_SCHEME_B) ks = calibrated_scale(a.cal_k_scale, a.status, report);
    }
    const float vrc = (vs != 0.f) ? __frcp_rn(vs) : 0.f, vcl = 127.f * vs;
    const float krc = (ks != 0.f) ? __frcp_rn(ks) : 0.f, kcl = 127.f * ks;
    while (cur.next(row, t0, t1, slot)) {
        const int b = row % a.B, kvh = row / a.B;
        const int64_t row0 = (int64_t)kvh * a.T + cur.ri.seq_start;  // cache row of the sequence's token 0
        int8_t *codes_row0 = a.k_codes + row0 * C::D + half * (C::D / LPR);
        int8_t *vcodes_row0 = nullptr;
        if constexpr (cal) vcodes_row0 = a.v_codes_out + row0 * C::D + half * (C::D / LPR);
        float *scale_row0 = a.k_scale_out + (int64_t)kvh * a.n_parts + cur.ri.part0;
        for (int32_t t = t0; t < t1; t += C::ROWS, ++tile_no) {
            const bool ready = mbar_wait(&full[stage], phase, a.status, abort_flag, a.wait_limit);
            const uint32_t kbase = smem_u32(smem + stage * C::STAGE_BYTES);
            const int32_t j = t + vr;
            const bool vrow = ready && j < t1;
            uint4 kw[NH];
            uint32_t km2[4] = {0u, 0u, 0u, 0u};  // four independent running maxima
#pragma unroll
            for (int i = 0; i < NH; ++i) {
                kw[i] = chunk_at(kbase, i);
                km2[0] = bf16x2_absmax(km2[0], kw[i].x);
                km2[1] = bf16x2_absmax(km2[1], kw[i].y);
                km2[2] = bf16x2_absmax(km2[2], kw[i].z);
                km2[3] = bf16x2_absmax(km2[3], kw[i].w);
            }
            float kmx = fmaxf(fmaxf(bf16x2_fold_max(km2[0]), bf16x2_fold_max(km2[1])),
                              fmaxf(bf16x2_fold_max(km2[2]), bf16x2_fold_max(km2[3])));
            if (!vrow) kmx = 0.f;
            if (a.qscheme == SGD_SCHEME_B) {
                if constexpr (!cal) {
                    run_kmax = fmaxf(run_kmax, kmx);
                } else if (vrow) {  // K codes under the calibrated K scale
                    store_code_chunks<NH, true>(codes_row0 + (int64_t)j * C::D, kw, ks, krc, kcl);
                }
            } else {
                kmx = warp_max(kmx);
                const int parity = tile_no & 1;
                if (lane == 0) kmxs[parity * C::NQ + qw] = kmx;
                named_barrier_sync(2, C::NQ * 32);
                float tm = 0.f;
#pragma unroll
                for (int w = 0; w < C::NQ; ++w) tm = fmaxf(tm, kmxs[parity * C::NQ + w]);
                const float sc = __fdiv_rn(tm, 127.f);
                const float r = (sc != 0.f) ? __frcp_rn(sc) : 0.f;
                if (vrow) store_code_chunks<NH, false>(codes_row0 + (int64_t)j * C::D, kw, sc, r, 0.f);
                // (the partition count was checked against the host's n_parts before any write)
                if (qw == 0 && lane == 0 && ready) scale_row0[t / kPart] = sc;
            }
            if constexpr (cal) {  // V codes under the calibrated V scale, and the row norms
                uint4 vw[NH];
#pragma unroll
                for (int i = 0; i < NH; ++i) vw[i] = chunk_at(kbase + C::TILE, i);
                if (vrow) store_code_chunks<NH, true>(vcodes_row0 + (int64_t)j * C::D, vw, vs, vrc, vcl);
                if (a.v_norm_out) {
                    float p[NH];  // per-chunk sums of squares, in element order
#pragma unroll
                    for (int i = 0; i < NH; ++i) {
                        float x[8];
                        Vec<__nv_bfloat16>::unpack(vw[i], x);
                        float px = 0.f;
#pragma unroll
                        for (int e = 0; e < 8; ++e) px = fmaf(x[e], x[e], px);
                        p[i] = px;
                    }
                    // chunk c pairs with c ^ o: on the lane of half ^ (o / NH) for o >= NH, in
                    // this lane below
#pragma unroll
                    for (int o = CPR / 2; o >= NH; o >>= 1)
#pragma unroll
                        for (int i = 0; i < NH; ++i) p[i] += __shfl_xor_sync(0xffffffffu, p[i], RW * (o / NH));
#pragma unroll
                    for (int o = NH / 2; o; o >>= 1)
#pragma unroll
                        for (int i = 0; i < o; ++i) p[i] = p[i] + p[i + o];
                    if (vrow && half == 0) a.v_norm_out[row0 + j] = sqrtf(p[0]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1;
            }
        }
    }
    if (a.qscheme == SGD_SCHEME_B && !cal) {  // (calibrated: no maximum wanted)
        run_kmax = warp_max(run_kmax);
        if (lane == 0) atomicMax(&a.amax_bits[0], __float_as_uint(run_kmax));
    }
}

// ------------------------------------------------------------------------------------------
// in-kernel LSE merge of one row's partials (run by the CTA that finishes the row's last
// outstanding segment; the 128 consumer threads, `scratch` = one stage of shared memory):
// lse = ln sum_c exp(lse_c), out = sum_c exp(lse_c - lse) o_c, as merge_kernel computes it.
// ------------------------------------------------------------------------------------------
template <class C>
__device__ __forceinline__ void merge_row(const DecodeArgs &a, int slot0, int n, int b, int kvh, float *scratch,
                                          int col0 = 0) {
    constexpr int NT = C::NW * 32;
    // G here: this CTA's columns col0 .. col0 + G - 1 of the row's NCt (query token, head) pairs;
    // a slot holds all NCt columns
    const int NCt = a.G * a.M, G = min(C::NG, NCt - col0), tid = threadIdx.x;
    float *Ls = scratch;                       // [16] per head: running max, then the lse
    float *Ss = scratch + 16;                  // [16] running sum
    float *w = scratch + 32;                   // [chunk][G] lse, then weights
    const int chunk = (2 * C::TILE / 4 - 32) / G;
    const float *lp = a.lse_part + (int64_t)slot0 * NCt + col0;  // lse of (slot c, column j): lp[c * NCt + j]
    const float *op = a.o_part + ((int64_t)slot0 * NCt + col0) * C::D;
    auto lse_at = [&](int c, int p) { return __ldcg(lp + (int64_t)(c + p / G) * NCt + p % G); };
    constexpr int kQ4 = C::NG * C::D / 4 / NT;  // float4 columns per thread at the most columns
    const int Q = G * C::D / 4, QSt = NCt * C::D / 4;  // float4s of this CTA's columns / of a slot
    // float4 q of the CTA's [G][D] block -> its place in out (column col0 + 4q / D)
    auto dst4 = [&](int q) -> float4 & {
        const int n = (4 * q) / C::D;
        return *reinterpret_cast<float4 *>(a.out + col_row(a, b, kvh, col0 + n) * C::D + (4 * q - n * C::D));
    };
    if (n <= chunk) {
        // one round: every lse loaded once, the weights computed in place, then thread t reads
        // its float4 columns t, t + NT, ... of every slot, eight slots' loads in flight
        for (int p = tid; p < n * G; p += NT) w[p] = lse_at(0, p);
        named_barrier_sync(1, NT);
        if (tid < G) {
            float M = -INFINITY, S = 0.f;
            for (int c = 0; c < n; ++c) M = fmaxf(M, w[c * G + tid]);
            if (M > -INFINITY)  // else no partial saw a token (a query token past a short row)
                for (int c = 0; c < n; ++c) S += expf(w[c * G + tid] - M);
            Ls[tid] = (S > 0.f) ? M + logf(S) : -INFINITY;
        }
        named_barrier_sync(1, NT);
        for (int p = tid; p < n * G; p += NT) w[p] = (Ls[p % G] > -INFINITY) ? expf(w[p] - Ls[p % G]) : 0.f;
        named_barrier_sync(1, NT);
        const float4 *oc = reinterpret_cast<const float4 *>(op);
        float4 acc[kQ4];
#pragma unroll
        for (int j = 0; j < kQ4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int c = 0; c < n; ++c) {
#pragma unroll
            for (int j = 0; j < kQ4; ++j) {
                const int q = tid + j * NT;
                if (q < Q) {
                    const float4 x = __ldcg(oc + (int64_t)c * QSt + q);
                    const float wc = w[c * G + (4 * q) / C::D];
                    acc[j].x += wc * x.x;
                    acc[j].y += wc * x.y;
                    acc[j].z += wc * x.z;
                    acc[j].w += wc * x.w;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kQ4; ++j) {
            const int q = tid + j * NT;
            if (q < Q) dst4(q) = acc[j];
        }
        if (tid < G) a.lse[col_row(a, b, kvh, col0 + tid)] = Ls[tid];
        named_barrier_sync(1, NT);  // scratch is the stage's memory: free again
        return;
    }
    // more slots than one round of shared memory holds: running max and sum per head, then the
    // weighted sum round by round, adding to what this thread wrote
    if (tid < G) {
        Ls[tid] = -INFINITY;
        Ss[tid] = 0.f;
    }
    for (int c0 = 0; c0 < n; c0 += chunk) {  // pass 1: max and sum of exp per head, online
        const int m = min(chunk, n - c0);
        named_barrier_sync(1, NT);
        for (int p = tid; p < m * G; p += NT) w[p] = lse_at(c0, p);
        named_barrier_sync(1, NT);
        if (tid < G) {
            float M = Ls[tid], S = Ss[tid];
            for (int c = 0; c < m; ++c) {
                const float x = w[c * G + tid];
                if (x > M) {
                    S = S * expf(M - x) + 1.f;
                    M = x;
                } else if (x > -INFINITY) {
                    S += expf(x - M);
                }
            }
            Ls[tid] = M;
            Ss[tid] = S;
        }
    }
    named_barrier_sync(1, NT);
    if (tid < G) Ls[tid] = (Ss[tid] > 0.f) ? Ls[tid] + logf(Ss[tid]) : -INFINITY;
    // pass 2: thread t owns float4 columns t, t + NT, ... of the row's [G][D] block and reads
    // them from every slot of a chunk, kQ4 * 4 independent 16-byte loads in flight
    for (int c0 = 0; c0 < n; c0 += chunk) {
        const int m = min(chunk, n - c0);
        named_barrier_sync(1, NT);
        for (int p = tid; p < m * G; p += NT)
            w[p] = (Ls[p % G] > -INFINITY) ? expf(lse_at(c0, p) - Ls[p % G]) : 0.f;
        named_barrier_sync(1, NT);
        const float4 *oc = reinterpret_cast<const float4 *>(op + (int64_t)c0 * NCt * C::D);
        float4 acc[kQ4];
#pragma unroll
        for (int j = 0; j < kQ4; ++j) {
            const int q = tid + j * NT;
            acc[j] = (c0 > 0 && q < Q) ? dst4(q) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll 4
        for (int c = 0; c < m; ++c) {
#pragma unroll
            for (int j = 0; j < kQ4; ++j) {
                const int q = tid + j * NT;
                if (q < Q) {
                    const float4 x = __ldcg(oc + (int64_t)c * QSt + q);
                    const float wc = w[c * G + (4 * q) / C::D];
                    acc[j].x += wc * x.x;
                    acc[j].y += wc * x.y;
                    acc[j].z += wc * x.z;
                    acc[j].w += wc * x.w;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kQ4; ++j) {
            const int q = tid + j * NT;
            if (q < Q) dst4(q) = acc[j];
        }
    }
    if (tid < G) a.lse[col_row(a, b, kvh, col0 + tid)] = Ls[tid];
    named_barrier_sync(1, NT);  // scratch is the stage's memory: free again
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
template <class C>
__global__ void __launch_bounds__(C::THREADS, C::MINB)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const DecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::SMEM_STAGES);
    uint64_t *empty = full + C::STAGES;
    float *ml = reinterpret_cast<float *>(empty + C::STAGES);  // [NW][NG][2]: m, l
    volatile int32_t *abort_flag = reinterpret_cast<int32_t *>(ml + C::NW * C::NG * 2);
    float *kmxs = ml + C::NW * C::NG * 2 + 4;  // [2][NQ] per-warp max|K| of the current tile (mode 2)
    float *row_scale = kmxs + C::SMEM_KMX / 4;  // [STAGES][ROWS] K scale of each gathered row (INT8 gathers)
    // [GT][KB][32 lanes] uint2: the Q fragments of the current segment (two column tiles)
    const uint32_t qsm = smem_u32(row_scale + C::SMEM_ROWSCALE / 4) + (threadIdx.x & 31) * 8;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], C::IDX ? 32u : 1u);
            mbar_init(&empty[s], (uint32_t)(C::NW + C::NQ));
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // decode with more than 16 columns: ncg CTAs share each planned range, one group of 16 each
    const int ncg = (C::MODE == 0 && a.ncg > 1) ? a.ncg : 1;
    const int cta = blockIdx.x / ncg, cg = blockIdx.x - cta * ncg;
    const int col0 = cg * C::NG;
    if (a.plan.cta_begin[cta] >= a.plan.cta_begin[cta + 1]) return;
    if constexpr (C::MODE == 2) {
        // scheme-A scales are written at kvh * n_parts + (partition): the device count must agree
        if (a.qscheme == SGD_SCHEME_A && a.plan.seq_part0[a.B] != a.n_parts) {
            if (threadIdx.x == 0) atomicOr(a.status, SGD_STATUS_SIZE_MISMATCH);
            return;
        }
    }

    if (warp == C::NW + C::NQ) {
        mma_producer<C>(&tmK, &tmV, a, smem, full, empty, abort_flag, row_scale, cta, lane);
        return;
    }
    if constexpr (C::NQ > 0) {
        if (warp >= C::NW) {
            quant_consumer<C>(a, smem, full, empty, abort_flag, kmxs, cta, warp - C::NW, lane);
            return;
        }
    }

    const int g4 = lane >> 2, t4 = lane & 3;
    const int pA = mma_row_perm(g4);
    SegCursor cur;
    cur.init(a.plan, a.B * a.Hkv, cta);
    int stage = 0;
    uint32_t phase = 0;
    int row, slot;
    int32_t t0, t1;
    float run_kmax = 0.f, run_vmax = 0.f;  // mode 2
    int tile_no = 0;
    const float vfac = (C::I8 && C::MODE == 0) ? __ldg(a.v_scale) : 1.f;  // loaded once, used per segment
    while (cur.next(row, t0, t1, slot)) {
        const int b = row % a.B, kvh = row / a.B;
        const int32_t seq_start = cur.ri.seq_start;
        const int32_t Lb = cur.ri.seq_len;
        const int64_t tok_base = (int64_t)kvh * a.T + seq_start;  // cache row of token 0 of the sequence
        uint32_t qf[C::GT][C::KB][2];
        float colf[C::GT][2];
        load_q_frags<C>(a, b, kvh, g4, t4, qf, colf, col0);
        if constexpr (C::QS) {
            // each lane stores, and later reads, only its own slots; every consumer warp writes the
            // same values, and none still reads the previous segment's (the epilogue barriers)
#pragma unroll
            for (int gt = 0; gt < C::GT; ++gt)
#pragma unroll
                for (int x = 0; x < C::KB; ++x) sts64(qsm + (gt * C::KB + x) * 256, qf[gt][x][0], qf[gt][x][1]);
            __syncwarp();
        }
        float m[C::GT][2], l[C::GT][2], o[C::GT][C::KB][4];
#pragma unroll
        for (int gt = 0; gt < C::GT; ++gt) {
            m[gt][0] = m[gt][1] = -INFINITY;
            l[gt][0] = l[gt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < C::KB; ++mt) o[gt][mt][0] = o[gt][mt][1] = o[gt][mt][2] = o[gt][mt][3] = 0.f;
        }
        const float *ksc = nullptr;
        const int32_t *ip = nullptr;
        if constexpr (C::I8) ksc = a.k_scale + (int64_t)kvh * a.n_parts + cur.ri.part0;
        if constexpr (C::IDX) ip = a.idx + (int64_t)kvh * a.Kt + cur.ri.len_start;
        if constexpr (C::BLK) ip = a.idx + (int64_t)kvh * a.Kt + cur.ri.len_start / kPart;
        // scores of an INT8 cache: the value norms of each sub-tile row, loaded one tile ahead
        float vn_cur[C::SUB], vn_nxt[C::SUB];
        auto load_norms = [&](float (&dst)[C::SUB], int32_t tt) {
#pragma unroll
            for (int s = 0; s < C::SUB; ++s) {
                const int32_t j = tt + 16 * (s * C::NW + warp) + (lane & 15);
                dst[s] = (lane < 16 && j < t1) ? __ldg(a.v_norm + tok_base + j) : 0.f;
            }
        };
        if constexpr (C::KONLY) load_norms(vn_cur, t0);

        for (int32_t t = t0; t < t1; t += C::ROWS) {
            // dense scheme A: the K scale of each sub-tile's partition, loaded before the wait
            float rf_pre[C::SUB];
#pragma unroll
            for (int s = 0; s < C::SUB; ++s) rf_pre[s] = 1.f;
            // kept blocks: the sequence position of each sub-tile's row 0 (a 16-row sub-tile lies in
            // one block) and, for scheme A, that block's K scale (blocks are the K partitions)
            int32_t bpos[C::SUB];
            if constexpr (C::BLK) {
                const int32_t nb = (Lb + kPart - 1) / kPart;
#pragma unroll
                for (int s = 0; s < C::SUB; ++s) {
                    const int32_t u = t + 16 * (s * C::NW + warp);
                    int32_t v = (u < t1) ? __ldg(ip + u / kPart) : 0;
                    v = min(max(v, 0), max(nb - 1, 0));
                    bpos[s] = v * kPart + (u % kPart);
                    if constexpr (C::I8) {
                        if (a.scheme == SGD_SCHEME_A && nb > 0) rf_pre[s] = __ldg(ksc + v);
                    }
                }
            }
            if constexpr (C::I8 && !C::IDX && !C::BLK) {
                if (a.scheme == SGD_SCHEME_A) {
#pragma unroll
                    for (int s = 0; s < C::SUB; ++s)
                        rf_pre[s] = __ldg(ksc + min(t + 16 * (s * C::NW + warp), Lb - 1) / kPart);
                }
            }
            if constexpr (C::KONLY) load_norms(vn_nxt, t + C::ROWS);
            // warp-uniform: the MMAs and shuffles below need every lane
            const bool ready = __all_sync(0xffffffffu, mbar_wait(&full[stage], phase, a.status, abort_flag, a.wait_limit));
            uint8_t *sk = smem + stage * C::STAGE_BYTES;
            uint8_t *sv = sk + C::TILE;
            const uint32_t kbase = smem_u32(sk), vbase = smem_u32(sv);
            if constexpr (C::MODE >= 1) {
#pragma unroll
                for (int s = 0; s < C::SUB; ++s) {
                    const int rb = 16 * (s * C::NW + warp);
                    const int32_t j0 = t + rb;  // row-local position of sub-tile row 0
                    if constexpr (C::I8)
                        score_subtile_i8<C>(a, kbase, rb, j0, t1, ready, tok_base, pA, t4, lane, qf, colf, rf_pre[s],
                                            vn_cur[s]);
                    else
                        score_subtile<C>(a, kbase, vbase, rb, j0, t1, ready, tok_base, pA, t4, lane, qf, run_vmax);
                }
            } else if (ready) {
                // 1. logits of the warp's sub-tiles (log2 units, -inf where masked); 2. one running
                // max update per column for all of them; 3. probabilities and O += V^T P^T per sub-tile.
                // The sub-tiles' QK and PV chains are independent, so they overlap.
                float z[C::SUB][C::GT][4];
                bool live[C::SUB];
#pragma unroll
                for (int s = 0; s < C::SUB; ++s) {
                    const int rb = 16 * (s * C::NW + warp);
                    const int32_t j0 = t + rb;  // row-local position of sub-tile row 0
                    live[s] = j0 < t1;
#pragma unroll
                    for (int gt = 0; gt < C::GT; ++gt) z[s][gt][0] = z[s][gt][1] = z[s][gt][2] = z[s][gt][3] = -INFINITY;
                    if (!live[s]) continue;
                    float sacc[C::GT][4];
                    qk_subtile<C>(kbase, rb, pA, t4, qf, sacc, qsm);
                    bool vA = j0 + pA < t1, vB = j0 + pA + 8 < t1;
                    if constexpr (C::BLK) {  // the last block of a sequence is ragged
                        vA = bpos[s] + pA < Lb;
                        vB = bpos[s] + pA + 8 < Lb;
                    }
                    // several query tokens: token m sees sequence positions <= L_b - M + m; bit 4 gt + e
                    // keeps element e of column tile gt (only sub-tiles reaching the last M - 1
                    // positions mask anything)
                    uint32_t cm = ~0u;
                    if constexpr (C::CAUSAL) {
                        int32_t pa = j0 + pA, pb = pa + 8;
                        if constexpr (C::IDX) {
                            pa = vA ? __ldg(ip + j0 + pA) : 0;
                            pb = vB ? __ldg(ip + j0 + pA + 8) : 0;
                        }
                        const int32_t lim0 = Lb - a.M;
                        if (__any_sync(0xffffffffu, max(pa, pb) > lim0)) {
                            cm = 0u;
#pragma unroll
                            for (int gt = 0; gt < C::GT; ++gt)
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int32_t lim = lim0 + (col0 + 8 * gt + 2 * t4 + (e & 1)) / a.G;
                                    cm |= (uint32_t)((e < 2 ? pa : pb) <= lim) << (4 * gt + e);
                                }
                        }
                    }
                    // row (token) factors: scheme-A K scale of the token's 64-token partition
                    float rfA = rf_pre[s], rfB = rf_pre[s];
                    if constexpr (C::ROW_SCALE) {
                        if (a.scheme == SGD_SCHEME_A) {
                            rfA = row_scale[stage * C::ROWS + rb + pA];
                            rfB = row_scale[stage * C::ROWS + rb + pA + 8];
                        }
                    }
#pragma unroll
                    for (int gt = 0; gt < C::GT; ++gt) {
                        bool k0 = vA, k1 = vA, k2 = vB, k3 = vB;
                        if constexpr (C::CAUSAL) {
                            k0 = k0 && (cm >> (4 * gt) & 1u);
                            k1 = k1 && (cm >> (4 * gt + 1) & 1u);
                            k2 = k2 && (cm >> (4 * gt + 2) & 1u);
                            k3 = k3 && (cm >> (4 * gt + 3) & 1u);
                        }
                        if (k0) z[s][gt][0] = sacc[gt][0] * rfA * colf[gt][0];
                        if (k1) z[s][gt][1] = sacc[gt][1] * rfA * colf[gt][1];
                        if (k2) z[s][gt][2] = sacc[gt][2] * rfB * colf[gt][0];
                        if (k3) z[s][gt][3] = sacc[gt][3] * rfB * colf[gt][1];
                    }
                }
                float mu[C::GT][2];
#pragma unroll
                for (int gt = 0; gt < C::GT; ++gt) {
                    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                    for (int s = 0; s < C::SUB; ++s) {
                        mx0 = fmaxf(mx0, fmaxf(z[s][gt][0], z[s][gt][2]));
                        mx1 = fmaxf(mx1, fmaxf(z[s][gt][1], z[s][gt][3]));
                    }
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                    }
                    if (mx0 > m[gt][0]) {
                        const float al = exp2f(m[gt][0] - mx0);
                        m[gt][0] = mx0;
                        l[gt][0] *= al;
#pragma unroll
                        for (int mt = 0; mt < C::KB; ++mt) {
                            o[gt][mt][0] *= al;
                            o[gt][mt][2] *= al;
                        }
                    }
                    if (mx1 > m[gt][1]) {
                        const float al = exp2f(m[gt][1] - mx1);
                        m[gt][1] = mx1;
                        l[gt][1] *= al;
#pragma unroll
                        for (int mt = 0; mt < C::KB; ++mt) {
                            o[gt][mt][1] *= al;
                            o[gt][mt][3] *= al;
                        }
                    }
                    mu[gt][0] = (m[gt][0] == -INFINITY) ? 0.f : m[gt][0];
                    mu[gt][1] = (m[gt][1] == -INFINITY) ? 0.f : m[gt][1];
                }
#pragma unroll
                for (int s = 0; s < C::SUB; ++s) {
                    if (!live[s]) continue;
                    uint32_t pb[C::GT][2];
#pragma unroll
                    for (int gt = 0; gt < C::GT; ++gt) {
                        const float p0 = exp2f(z[s][gt][0] - mu[gt][0]), p2 = exp2f(z[s][gt][2] - mu[gt][0]);
                        const float p1 = exp2f(z[s][gt][1] - mu[gt][1]), p3 = exp2f(z[s][gt][3] - mu[gt][1]);
                        l[gt][0] += p0 + p2;
                        l[gt][1] += p1 + p3;
                        const uint32_t r0 = C::I8 ? pack_f16(p0, p1) : pack_bf16(p0, p1);
                        const uint32_t r1 = C::I8 ? pack_f16(p2, p3) : pack_bf16(p2, p3);
                        pb[gt][0] = movmatrix_trans(r0);
                        pb[gt][1] = movmatrix_trans(r1);
                    }
                    pv_subtile<C>(vbase, 16 * (s * C::NW + warp), lane, pb, o);
                }
            }
            ++tile_no;
            if constexpr (C::KONLY) {
#pragma unroll
                for (int s = 0; s < C::SUB; ++s) vn_cur[s] = vn_nxt[s];
            }
            const bool last = (t + C::ROWS >= t1);
            if (C::MODE == 0 && last) {
                // ---- segment epilogue: combine the four warps' (m, l, O) in this stage's memory ----
                named_barrier_sync(1, C::NW * 32);  // every warp is done reading the stage
                float *eo = reinterpret_cast<float *>(sk);  // [NW][NG][D]
#pragma unroll
                for (int gt = 0; gt < C::GT; ++gt)
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int off = 4; off < 32; off <<= 1) l[gt][j] += __shfl_xor_sync(0xffffffffu, l[gt][j], off);
#pragma unroll
                for (int gt = 0; gt < C::GT; ++gt) {
                    const int g0 = 8 * gt + 2 * t4;
                    float *e0 = eo + (warp * C::NG + g0) * C::D, *e1 = e0 + C::D;
#pragma unroll
                    for (int mt = 0; mt < C::KB; ++mt) {
                        const int da = C::I8 ? 16 * g4 + 2 * mt : 16 * mt + g4;
                        const int db = C::I8 ? da + 1 : da + 8;
                        e0[da] = o[gt][mt][0];
                        e1[da] = o[gt][mt][1];
                        e0[db] = o[gt][mt][2];
                        e1[db] = o[gt][mt][3];
                    }
                    if (g4 == 0) {
                        ml[(warp * C::NG + g0) * 2 + 0] = m[gt][0];
                        ml[(warp * C::NG + g0) * 2 + 1] = l[gt][0];
                        ml[(warp * C::NG + g0 + 1) * 2 + 0] = m[gt][1];
                        ml[(warp * C::NG + g0 + 1) * 2 + 1] = l[gt][1];
                    }
                }
                named_barrier_sync(1, C::NW * 32);
                const int tid = threadIdx.x;
                const int NCt = a.G * a.M;                 // columns of a row: (query token, head) pairs
                const int NC = min(C::NG, NCt - col0);     // this CTA's: col0 .. col0 + NC - 1
                if (tid < NC) {  // column n: the warps' weights replace their m in ml; the lse replaces warp 0's l
                    float M = -INFINITY, f[C::NW], L = 0.f;
#pragma unroll
                    for (int w = 0; w < C::NW; ++w) M = fmaxf(M, ml[(w * C::NG + tid) * 2]);
#pragma unroll
                    for (int w = 0; w < C::NW; ++w) {
                        f[w] = (M == -INFINITY) ? 0.f : exp2f(ml[(w * C::NG + tid) * 2] - M);
                        L += f[w] * ml[(w * C::NG + tid) * 2 + 1];
                    }
                    const float inv = (L > 0.f) ? vfac / L : 0.f;
#pragma unroll
                    for (int w = 0; w < C::NW; ++w) ml[(w * C::NG + tid) * 2] = f[w] * inv;
                    ml[tid * 2 + 1] = (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
                }
                named_barrier_sync(1, C::NW * 32);
                // a row's only segment is its result; otherwise a partial in the segment's slot
                const bool direct = cur.ri.nseg == 1;
                float *part = a.o_part + ((int64_t)slot * NCt + col0) * C::D;
                for (int e = tid; e < NC * C::D; e += C::NW * 32) {
                    const int g = e / C::D, d = e - g * C::D;
                    float O = 0.f;
#pragma unroll
                    for (int w = 0; w < C::NW; ++w) O += ml[(w * C::NG + g) * 2] * eo[(w * C::NG + g) * C::D + d];
                    if (direct) a.out[col_row(a, b, kvh, col0 + g) * C::D + d] = O;
                    else part[e] = O;
                }
                if (tid < NC) {
                    const float lv = ml[tid * 2 + 1];
                    if (direct) a.lse[col_row(a, b, kvh, col0 + tid)] = lv;
                    else a.lse_part[(int64_t)slot * NCt + col0 + tid] = lv;
                }
                if (!direct) {
                    // the CTA that finishes the row's last outstanding segment merges the row
                    volatile int *merge_flag = reinterpret_cast<volatile int *>(kmxs);
                    __threadfence();
                    named_barrier_sync(1, C::NW * 32);
                    if (tid == 0) *merge_flag = atomicAdd(a.plan.row_done + row * ncg + cg, 1) == cur.ri.nseg - 1;
                    named_barrier_sync(1, C::NW * 32);
                    if (*merge_flag) {
                        __threadfence();
                        merge_row<C>(a, cur.ri.slot0, cur.ri.nseg, b, kvh, reinterpret_cast<float *>(sk), col0);
                    }
                }
                fence_proxy_async_shared();
                named_barrier_sync(1, C::NW * 32);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == C::STAGES) {
                stage = 0;
                phase ^= 1;
            }
        }
    }
    if constexpr (C::MODE == 2) {
        run_vmax = warp_max(run_vmax);
        if (lane == 0) atomicMax(&a.amax_bits[1], __float_as_uint(run_vmax));
    }
}

// ------------------------------------------------------------------------------------------
// CUDA-core kernel: any dtype, D in {64, 128}, G <= 16
// ------------------------------------------------------------------------------------------
template <typename KT>
__device__ __forceinline__ float load_elem(const void *p, int64_t i) {
    if constexpr (sizeof(KT) == 4) return __ldg(static_cast<const float *>(p) + i);
    else if constexpr (sizeof(KT) == 2)
        return __bfloat162float(__ldg(static_cast<const __nv_bfloat16 *>(p) + i));
    else return (float)__ldg(static_cast<const int8_t *>(p) + i);
}

template <int D, typename KT, bool IDX, int MODE>
__global__ void __launch_bounds__(128) decode_generic_kernel(const DecodeArgs a) {
    constexpr int NW = 4, PER = D / 32, MG = 16;
    constexpr bool I8 = sizeof(KT) == 1;
    __shared__ float eo[NW][MG][D];
    __shared__ float eml[NW][MG][2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    if (a.plan.cta_begin[cta] >= a.plan.cta_begin[cta + 1]) return;
    const int Hq = a.Hkv * a.G;
    SegCursor cur;
    cur.init(a.plan, a.B * a.Hkv, cta);
    int row, slot;
    int32_t t0, t1;
    while (cur.next(row, t0, t1, slot)) {
        const int b = row % a.B, kvh = row / a.B;
        const int32_t Lb = cur.ri.seq_len;
        const int64_t seq0 = (int64_t)kvh * a.T + cur.ri.seq_start;
        float q[MG][PER];
#pragma unroll
        for (int g = 0; g < MG; ++g)
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                float x = 0.f;
                if (g < a.G) {
                    const int64_t qi = ((int64_t)b * Hq + kvh * a.G + g) * D + lane + 32 * i;
                    x = a.q_f32 ? __ldg(static_cast<const float *>(a.q) + qi)
                                : __bfloat162float(__ldg(static_cast<const __nv_bfloat16 *>(a.q) + qi));
                }
                q[g][i] = x;
            }
        float m[MG], l[MG], acc[MG][PER];
#pragma unroll
        for (int g = 0; g < MG; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
#pragma unroll
            for (int i = 0; i < PER; ++i) acc[g][i] = 0.f;
        }
        float kfac = 1.f, vfac = 1.f;
        const float *ksc = nullptr;
        if constexpr (I8) {
            vfac = __ldg(a.v_scale);
            if (a.scheme == SGD_SCHEME_B) kfac = __ldg(a.k_scale);
            else ksc = a.k_scale + (int64_t)kvh * a.n_parts + cur.ri.part0;
        }
        const int32_t *ip = IDX ? a.idx + (int64_t)kvh * a.Kt + cur.ri.len_start : nullptr;
        for (int32_t j = t0 + warp; j < t1; j += NW) {
            int32_t tok = j;
            if constexpr (IDX) {
                tok = __ldg(ip + j);
                if (tok < 0 || tok >= Lb) {
                    if (lane == 0) atomicOr(a.status, SGD_STATUS_BAD_INDEX);
                    tok = min(max(tok, 0), Lb - 1);
                }
            }
            const int64_t base = (seq0 + tok) * D;
            float kf = kfac;
            if (I8 && ksc) kf = __ldg(ksc + tok / kPart);
            float kk[PER], vv[PER];
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                kk[i] = load_elem<KT>(a.k, base + lane + 32 * i) * kf;
                vv[i] = load_elem<KT>(a.v, base + lane + 32 * i) * vfac;
            }
            if constexpr (MODE == 1) {
                float best = -INFINITY, ss = 0.f;
#pragma unroll
                for (int g = 0; g < MG; ++g) {
                    if (g < a.G) {
                        float dot = 0.f;
#pragma unroll
                        for (int i = 0; i < PER; ++i) dot = fmaf(q[g][i], kk[i], dot);
                        best = fmaxf(best, warp_sum(dot));
                    }
                }
#pragma unroll
                for (int i = 0; i < PER; ++i) ss = fmaf(vv[i], vv[i], ss);
                ss = warp_sum(ss);
                if (lane == 0) {
                    float sc = best * a.sm_scale + a.beta * logf(sqrtf(ss) + a.eps);
                    if (sc == 0.f) sc = 0.f;
                    a.scores[seq0 + j] = sc;
                }
            } else {
#pragma unroll
                for (int g = 0; g < MG; ++g) {
                    if (g < a.G) {
                        float dot = 0.f;
#pragma unroll
                        for (int i = 0; i < PER; ++i) dot = fmaf(q[g][i], kk[i], dot);
                        const float z = warp_sum(dot) * a.sm_scale_log2;
                        if (z > m[g]) {
                            const float al = exp2f(m[g] - z);
                            m[g] = z;
                            l[g] *= al;
#pragma unroll
                            for (int i = 0; i < PER; ++i) acc[g][i] *= al;
                        }
                        const float p = exp2f(z - m[g]);
                        l[g] += p;
#pragma unroll
                        for (int i = 0; i < PER; ++i) acc[g][i] = fmaf(p, vv[i], acc[g][i]);
                    }
                }
            }
        }
        if constexpr (MODE == 0) {
#pragma unroll
            for (int g = 0; g < MG; ++g) {
#pragma unroll
                for (int i = 0; i < PER; ++i) eo[warp][g][lane + 32 * i] = acc[g][i];
                if (lane == 0) {
                    eml[warp][g][0] = m[g];
                    eml[warp][g][1] = l[g];
                }
            }
            __syncthreads();
            for (int e = threadIdx.x; e < a.G * D; e += NW * 32) {
                const int g = e / D, d = e - g * D;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < NW; ++w) M = fmaxf(M, eml[w][g][0]);
                float L = 0.f, O = 0.f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int w = 0; w < NW; ++w) {
                        const float f = exp2f(eml[w][g][0] - M);
                        L += f * eml[w][g][1];
                        O += f * eo[w][g][d];
                    }
                }
                a.o_part[((int64_t)slot * a.G + g) * D + d] = (L > 0.f) ? O / L : 0.f;
                if (d == 0) a.lse_part[(int64_t)slot * a.G + g] = (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
            }
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------------------------------------
// exact LSE merge: per (sequence, query head), lse = ln sum_c exp(lse_c),
// out = sum_c exp(lse_c - lse) o_c
// ------------------------------------------------------------------------------------------
constexpr int kMergeThreads = 128;
constexpr int kMergeChunk = 512;  // combination weights staged in shared memory per round

__device__ __forceinline__ float block_reduce_128(float v, bool is_max, float *red) {
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const float w = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? fmaxf(v, w) : v + w;
    }
    const int warp = threadIdx.x >> 5;
    __syncthreads();  // red is reused
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    return is_max ? fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])) : (red[0] + red[1]) + (red[2] + red[3]);
}

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const DecodeArgs a, float *__restrict__ out,
                                                              float *__restrict__ lse) {
    // one block per (row, query head of the group): the row's partial LSEs are read by all
    // threads at once (no load waits on another), the weights exp(lse_c - lse) are staged in
    // shared memory and thread d accumulates channel d over the slots with independent loads
    __shared__ float w[kMergeChunk];
    __shared__ float red[4];
    const int r = blockIdx.x / a.G, g = blockIdx.x - r * a.G;
    const int b = r % a.B, kvh = r / a.B;
    const int s0 = a.plan.row_slot0[r], n = a.plan.row_slot0[r + 1] - s0;
    const int Hq = a.Hkv * a.G;
    const int64_t h = (int64_t)b * Hq + kvh * a.G + g;
    const float *lp = a.lse_part + (int64_t)s0 * a.G + g;
    const float *op = a.o_part + ((int64_t)s0 * a.G + g) * a.D;
    const int tid = threadIdx.x;
    if (n == 1) {  // one segment: its partial is the result
        for (int d = tid; d < a.D; d += kMergeThreads) out[h * a.D + d] = __ldg(op + d);
        if (tid == 0) lse[h] = __ldg(lp);
        return;
    }
    float M = -INFINITY;
    for (int c = tid; c < n; c += kMergeThreads) M = fmaxf(M, __ldg(lp + (int64_t)c * a.G));
    M = block_reduce_128(M, true, red);
    float S = 0.f;
    for (int c = tid; c < n; c += kMergeThreads) S += expf(__ldg(lp + (int64_t)c * a.G) - M);
    S = block_reduce_128(S, false, red);
    const float L = (n > 0) ? M + logf(S) : -INFINITY;
    float O = 0.f;
    for (int c0 = 0; c0 < n; c0 += kMergeChunk) {
        const int m = min(kMergeChunk, n - c0);
        __syncthreads();  // the previous round's weights are consumed
        for (int c = tid; c < m; c += kMergeThreads) w[c] = expf(__ldg(lp + (int64_t)(c0 + c) * a.G) - L);
        __syncthreads();
        if (tid < a.D) {
            const float *oc = op + (int64_t)c0 * a.G * a.D + tid;
#pragma unroll 8
            for (int c = 0; c < m; ++c) O += w[c] * __ldg(oc + (int64_t)c * a.G * a.D);
        }
    }
    if (tid < a.D) out[h * a.D + tid] = O;
    if (tid == 0) lse[h] = L;
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D map over a [rows, D] row-major tensor with boxes of (box_elems x box_rows), 128B swizzle.
static bool make_map(CUtensorMap *map, const void *base, bool i8, int D, int64_t rows, int box_elems, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int eb = i8 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * eb};
    cuuint32_t box[2] = {(cuuint32_t)box_elems, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, i8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                          const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <class C>
static cudaError_t set_smem_attrs() {
    auto k = decode_mma_kernel<C>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

template <class C>
static int ctas_per_sm_mma() {
    auto k = decode_mma_kernel<C>;
    if (set_smem_attrs<C>() != cudaSuccess) return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, C::THREADS, C::SMEM) != cudaSuccess) return 0;
    return n;
}

template <class C>
static int launch_mma(const DecodeArgs &a, int n_cta, cudaStream_t s) {
    CUtensorMap mk, mv;
    memset(&mk, 0, sizeof(mk));
    memset(&mv, 0, sizeof(mv));
    if constexpr (!C::IDX) {
        const int64_t rows = (int64_t)a.Hkv * a.T;
        if (!make_map(&mk, a.k, C::I8, C::D, rows, C::BOX_ELEMS, C::BOX_ROWS) ||
            !make_map(&mv, a.v, C::I8, C::D, rows, C::BOX_ELEMS, C::BOX_ROWS))
            return (int)cudaErrorInvalidValue;
    }
    auto k = decode_mma_kernel<C>;
    cudaError_t e = set_smem_attrs<C>();
    if (e != cudaSuccess) return (int)e;
    return (int)launch_k(k, dim3(n_cta), dim3(C::THREADS), C::SMEM, s, 1, mk, mv, a);
}

template <int D, int GT, bool I8, int MODE, bool QI8 = false>
static int launch_mma_idx(const DecodeArgs &a, bool indexed, int n_cta, cudaStream_t s) {
    if constexpr (MODE == 1) {
        return launch_mma<MmaCfg<D, GT, I8, false, MODE>>(a, n_cta, s);
    } else if (a.blk) {  // kept 64-token blocks: one TMA box per block
        return launch_mma<MmaCfg<D, GT, I8, false, MODE, QI8, false, true>>(a, n_cta, s);
    } else if (a.M > 1) {  // several query tokens per sequence: the causally masked instantiation
        return indexed ? launch_mma<MmaCfg<D, GT, I8, true, MODE, QI8, true>>(a, n_cta, s)
                       : launch_mma<MmaCfg<D, GT, I8, false, MODE, QI8, true>>(a, n_cta, s);
    } else {
        return indexed ? launch_mma<MmaCfg<D, GT, I8, true, MODE, QI8>>(a, n_cta, s)
                       : launch_mma<MmaCfg<D, GT, I8, false, MODE, QI8>>(a, n_cta, s);
    }
}

template <int D, typename KT, int MODE>
static int launch_generic(const DecodeArgs &a, bool indexed, int n_cta, cudaStream_t s) {
    if (indexed && MODE == 0)
        return (int)launch_k(decode_generic_kernel<D, KT, true, MODE>, dim3(n_cta), dim3(128), 0, s, 1, a);
    return (int)launch_k(decode_generic_kernel<D, KT, false, MODE>, dim3(n_cta), dim3(128), 0, s, 1, a);
}

Family decode_family(sgd_dtype kv, sgd_dtype q, int D, bool score) {
    if (q != SGD_BF16) return kFamilyGeneric;
    if (kv == SGD_BF16 && (D == 64 || D == 128)) return kFamilyMma;
    if (kv == SGD_I8 && D == 128) return kFamilyMma;
    return kFamilyGeneric;
}

int decode_ctas_per_sm(sgd_dtype kv, sgd_dtype q, int D, int G, bool indexed, bool score) {
    if (decode_family(kv, q, D, score) == kFamilyGeneric) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_generic_kernel<128, float, false, 0>, 128, 0) !=
            cudaSuccess)
            return 0;
        return n;
    }
    const bool g2 = G > 8;
    // the shared-memory and register footprint decide residency
    if (kv == SGD_I8 && score)
        return g2 ? ctas_per_sm_mma<MmaCfg<128, 2, true, false, 1>>() : ctas_per_sm_mma<MmaCfg<128, 1, true, false, 1>>();
    if (kv == SGD_I8 && indexed)
        return g2 ? ctas_per_sm_mma<MmaCfg<128, 2, true, true, 0>>() : ctas_per_sm_mma<MmaCfg<128, 1, true, true, 0>>();
    if (kv == SGD_I8) return g2 ? ctas_per_sm_mma<MmaCfg<128, 2, true, false, 0>>() : ctas_per_sm_mma<MmaCfg<128, 1, true, false, 0>>();
    if (D == 128) return g2 ? ctas_per_sm_mma<MmaCfg<128, 2, false, false, 0>>() : ctas_per_sm_mma<MmaCfg<128, 1, false, false, 0>>();
    return g2 ? ctas_per_sm_mma<MmaCfg<64, 2, false, false, 0>>() : ctas_per_sm_mma<MmaCfg<64, 1, false, false, 0>>();
}

int score_quantize_ctas_per_sm(int D, int G) {
    const bool g2 = G > 8;
    if (D == 128) return g2 ? ctas_per_sm_mma<MmaCfg<128, 2, false, false, 2>>() : ctas_per_sm_mma<MmaCfg<128, 1, false, false, 2>>();
    return g2 ? ctas_per_sm_mma<MmaCfg<64, 2, false, false, 2>>() : ctas_per_sm_mma<MmaCfg<64, 1, false, false, 2>>();
}

int launch_decode(const DecodeArgs &a, sgd_dtype kv, sgd_dtype q, bool indexed, bool score, int n_cta,
                  cudaStream_t s) {
    if (n_cta <= 0) return 0;
    const bool g2 = std::min(a.G * a.M, 16) > 8;  // columns of one CTA: (query token, head) pairs
    if (decode_family(kv, q, a.D, score) == kFamilyMma) {
        if (score) {
            if (kv == SGD_I8) return g2 ? launch_mma_idx<128, 2, true, 1>(a, false, n_cta, s) : launch_mma_idx<128, 1, true, 1>(a, false, n_cta, s);
            if (a.D == 128) return g2 ? launch_mma_idx<128, 2, false, 1>(a, false, n_cta, s) : launch_mma_idx<128, 1, false, 1>(a, false, n_cta, s);
            return g2 ? launch_mma_idx<64, 2, false, 1>(a, false, n_cta, s) : launch_mma_idx<64, 1, false, 1>(a, false, n_cta, s);
        }
        if (kv == SGD_I8 && a.q_quant)
            return g2 ? launch_mma_idx<128, 2, true, 0, true>(a, indexed, n_cta, s) : launch_mma_idx<128, 1, true, 0, true>(a, indexed, n_cta, s);
        if (kv == SGD_I8)
            return g2 ? launch_mma_idx<128, 2, true, 0>(a, indexed, n_cta, s) : launch_mma_idx<128, 1, true, 0>(a, indexed, n_cta, s);
        if (a.D == 128)
            return g2 ? launch_mma_idx<128, 2, false, 0>(a, indexed, n_cta, s) : launch_mma_idx<128, 1, false, 0>(a, indexed, n_cta, s);
        return g2 ? launch_mma_idx<64, 2, false, 0>(a, indexed, n_cta, s) : launch_mma_idx<64, 1, false, 0>(a, indexed, n_cta, s);
    }
    if (score) {
        if (kv == SGD_F32) return a.D == 128 ? launch_generic<128, float, 1>(a, false, n_cta, s) : launch_generic<64, float, 1>(a, false, n_cta, s);
        return a.D == 128 ? launch_generic<128, __nv_bfloat16, 1>(a, false, n_cta, s) : launch_generic<64, __nv_bfloat16, 1>(a, false, n_cta, s);
    }
    switch (kv) {
        case SGD_F32:
            return a.D == 128 ? launch_generic<128, float, 0>(a, indexed, n_cta, s) : launch_generic<64, float, 0>(a, indexed, n_cta, s);
        case SGD_BF16:
            return a.D == 128 ? launch_generic<128, __nv_bfloat16, 0>(a, indexed, n_cta, s) : launch_generic<64, __nv_bfloat16, 0>(a, indexed, n_cta, s);
        default:
            return a.D == 128 ? launch_generic<128, int8_t, 0>(a, indexed, n_cta, s) : launch_generic<64, int8_t, 0>(a, indexed, n_cta, s);
    }
}

template <bool CAL>
static int launch_score_quantize_cfg(const DecodeArgs &a, int n_cta, cudaStream_t s) {
    const bool g2 = a.G * a.M > 8;  // columns: the (query token, head) pairs
    if (a.D == 128)
        return g2 ? launch_mma<MmaCfg<128, 2, false, false, 2, false, false, false, CAL>>(a, n_cta, s)
                  : launch_mma<MmaCfg<128, 1, false, false, 2, false, false, false, CAL>>(a, n_cta, s);
    return g2 ? launch_mma<MmaCfg<64, 2, false, false, 2, false, false, false, CAL>>(a, n_cta, s)
              : launch_mma<MmaCfg<64, 1, false, false, 2, false, false, false, CAL>>(a, n_cta, s);
}

int launch_score_quantize(const DecodeArgs &a, int n_cta, cudaStream_t s) {
    if (n_cta <= 0) return 0;
    return a.cal_v_scale ? launch_score_quantize_cfg<true>(a, n_cta, s) : launch_score_quantize_cfg<false>(a, n_cta, s);
}

int launch_merge(const DecodeArgs &a, float *out, float *lse, cudaStream_t s) {
    return (int)launch_k(merge_kernel, dim3(a.B * a.Hkv * a.G), dim3(kMergeThreads), 0, s, 1, a, out, lse);
}

}  // namespace sgd
