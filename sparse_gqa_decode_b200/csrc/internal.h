// internal.h -- host-side interface between the C ABI (api.cu) and the kernels.
#pragma once

#include "common.cuh"

namespace sgd {

// Arguments of the decode / score kernels (device pointers unless noted).
struct DecodeArgs {
    const void *q;           // [B, M, Hq, D]
    const int32_t *cu_seq;   // cu_seqlens [B+1]
    const int32_t *cu_kept;  // kept-set prefix sums [B+1] (indexed mode)
    const int32_t *idx;      // [Hkv, Kt] kept positions (indexed mode)
    const void *k, *v;       // [Hkv, T, D]
    const float *k_scale;    // I8
    const float *v_scale;    // I8
    int scheme;              // I8: SGD_SCHEME_A / SGD_SCHEME_B
    int q_quant;             // I8 decode: 0 bf16 query, 1 query codes per (sequence, head), 2 per tensor
    const float *q_scale;    // q_quant == 2: the per-tensor query scale (in the workspace header)
    int B, Hkv, G, D;
    int M;                   // decode: query tokens per sequence (>= 1), causal over the cache's last M;
                             // the kernel's columns are the M * G (token, head) pairs of a KV head
    int blk;                 // decode: idx / cu_kept / Kt list kept 64-token blocks, not tokens
    int ncg;                 // decode: CTAs per planned range, one per group of 16 columns (M * G > 16)
    int64_t T, Kt, n_parts;
    int q_f32;               // q is float32 (otherwise bf16)
    float sm_scale_log2;     // log2(e) / sqrt(D)
    float sm_scale;          // 1 / sqrt(D)
    float beta, eps;         // score mode
    float *scores;           // score mode output [Hkv, T]
    const float *v_norm;     // score mode over an I8 cache: [Hkv, T] ||v_t||
    // score + quantize mode (fused first pass of sgd_quantize_select)
    int qscheme;             // SGD_SCHEME_A: K codes and partition scales here; B: max|K| only
    int8_t *k_codes;         // [Hkv, T, D]
    float *k_scale_out;      // [Hkv, n_parts]
    uint32_t *amax_bits;     // [2]: max|K| (scheme B), max|V| as float bits
    // mode 2 with calibrated per-tensor scales (cal_v_scale non-NULL): the pass also writes the V
    // codes (and, scheme B, the K codes with cal_k_scale) and, if v_norm_out, every ||v_t||
    const float *cal_k_scale;
    const float *cal_v_scale;
    int8_t *v_codes_out;     // [Hkv, T, D]
    float *v_norm_out;       // [Hkv, T] or NULL
    PlanView plan;
    float *o_part;           // [slots, M * G, D]
    float *lse_part;         // [slots, M * G]
    float *out;              // decode: [B, M, Hq, D] result (written by the kernel itself on the MMA path)
    float *lse;              // decode: [B, M, Hq]
    int32_t *status;
    long long wait_limit;    // polls before a pipeline wait gives up (kWaitLimit unless a test lowers it)
    int idle_producer;       // test aid: the producer warps issue no copies (every consumer wait runs out)
};

// The test hooks of sgd_test_pipeline_timeout (api.cu) applied to a launch's arguments.
void apply_test_hooks(DecodeArgs &a);

// kernel families
enum Family { kFamilyMma = 0, kFamilyGeneric = 1 };

// plan.cu
// out/lse (decode only, else NULL): rows without tokens get out = 0 and lse = -inf here.
// q_bf16 (decode with a per-tensor query scale, else NULL): hdr->q_scale = max|q| / 127.
// M: query tokens per sequence of the decode (out is [B, M, Hkv * G, D]).
// len_unit: tokens per unit of cu_len (64 when cu_len counts kept 64-token blocks).
void launch_plan(const int32_t *cu_len, const int32_t *cu_seq, int B, int Hkv, int n_req, int min_chunk,
                 int mode, const PlanView &pv, WsHeader *hdr, cudaStream_t s, int granule = kGranule,
                 float *out = nullptr, float *lse = nullptr, int G = 0, int D = 0, const void *q_bf16 = nullptr,
                 int64_t q_elems = 0, int M = 1, int len_unit = 1, int ncg = 1, int row_cost = 0);
void launch_plan_dump(const PlanView &pv, const int32_t *cu, int B, int Hkv, int n_req, int32_t *segs,
                      int64_t max_segs, int32_t *n_segs, const WsHeader *hdr, cudaStream_t s);

// decode.cu
// Family the decode/score of these arguments runs on.
Family decode_family(sgd_dtype kv_dtype, sgd_dtype q_dtype, int D, bool score);
// CTAs resident per SM for that kernel (0 on error).
int decode_ctas_per_sm(sgd_dtype kv_dtype, sgd_dtype q_dtype, int D, int G, bool indexed, bool score);
// Launches the split decode (or score) kernel over n_cta CTAs; returns a cudaError_t.
int launch_decode(const DecodeArgs &a, sgd_dtype kv_dtype, sgd_dtype q_dtype, bool indexed, bool score,
                  int n_cta, cudaStream_t s);
// CTAs resident per SM for the fused first pass of sgd_quantize_select (0 on error).
int score_quantize_ctas_per_sm(int D, int G);
// Fused first pass of sgd_quantize_select (bf16 cache, bf16 q): OAM scores, scheme-A K codes
// and scales (or max|K| for scheme B) and max|V|.  Needs a plan built with granule kPart.
int launch_score_quantize(const DecodeArgs &a, int n_cta, cudaStream_t s);
int launch_merge(const DecodeArgs &a, float *out, float *lse, cudaStream_t s);

// quantize.cu
// Second pass: codes of V (and of K for scheme B) with the global scales in hdr->amax_bits.
// vnorm (NULL: not wanted): [Hkv, T] L2 norm of every V row, written by the V-codes pass.
int launch_quantize_global(const void *k, const void *v, sgd_dtype dt, int Hkv, int D, int64_t T,
                           sgd_scheme scheme, int8_t *kc, int8_t *vc, float *k_scale, float *v_scale,
                           float *vnorm, WsHeader *hdr, int sm_count, cudaStream_t s);
int launch_quantize(const void *k, const void *v, sgd_dtype dt, const int32_t *cu, int B, int Hkv, int D,
                    int64_t T, sgd_scheme scheme, int64_t n_parts, int8_t *kc, int8_t *vc, float *k_scale,
                    float *v_scale, float *vnorm, WsHeader *hdr, int32_t *seq_part0, int sm_count, cudaStream_t s);

// oam.cu
int launch_topk(const float *scores, const int32_t *cu, int B, int Hkv, int64_t T, int keep_num, int keep_den,
                int32_t *idx, int32_t *cu_kept, int64_t kept_total, int32_t *status, cudaStream_t s);
// Block scores of 64-token blocks: bscores[h * Tb + j] = max of the token scores of block j
// (sequence b's blocks are cu_blk[b] .. cu_blk[b+1]; its last block may be ragged).
int launch_block_max(const float *scores, const int32_t *cu_seq, const int32_t *cu_blk, int B, int Hkv, int64_t T,
                     int64_t Tb, float *bscores, int32_t *status, cudaStream_t s);

// stream.cu
// Read-only streaming of `bytes` bytes (method 0: 16-byte loads; 1: bulk copies into shared
// memory), every byte XOR-folded into *sink.
int launch_stream_read(const void *buf, size_t bytes, int method, unsigned long long *sink, int32_t *status,
                       int sm_count, cudaStream_t s);
// Scattered-row read (sgd_gather_read): n_rows rows of row_bytes at a (and b) by row index.
int launch_gather_read(const void *a, const void *b, int64_t row_bytes, const int32_t *rows, int64_t n_rows,
                       unsigned long long *sink, int sm_count, cudaStream_t s);

}  // namespace sgd
