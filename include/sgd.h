/*
 * sgd.h -- C ABI of libsgd.so: single-token GQA decode attention over a long,
 * ragged KV cache on NVIDIA B200 (sm_100a), with output-aware token dropping
 * (OAM), an INT8 KV cache and split-KV flash-decoding with an exact
 * log-sum-exp merge.
 *
 * Sources (web pages, cited by title and section):
 *   [TD] "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse
 *        attention), lzwjava.github.io -- section 3 (OAM score and token
 *        dropping), section 5 (split-KV load balancing and the cross-chunk
 *        online-softmax merge), section 6 (INT8 KV cache, schemes A and B),
 *        section 7 (the three stack: OAM -> INT8 -> split-KV).
 *   [AO] "注意力优化（Attention Optimization）", learnagent.wiki -- scaled
 *        dot-product attention; GQA (query head h uses KV head h / G).
 *   [CD] "共同设计 AI 模型注意力，实现快速的交互式长上下文推理" (Co-designing AI
 *        model attention for fast interactive long-context inference), NVIDIA
 *        developer blog -- decode equations 5-7 (decode streams the KV cache
 *        and is HBM-bound; arithmetic intensity about 2G); speculative decoding
 *        raises the decode's GEMM M from G to (1 + n_draft) * G.
 *   [NSA] "硬件对齐的稀疏注意力机制：原理、优化与实践" (hardware-aligned sparse
 *        attention, NSA) -- section 2.1: selection shared by a GQA group,
 *        64-token selection blocks read contiguously.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  A packed ragged cache of B sequences and Hkv KV heads:
 *     k, v        [Hkv, T, D] row-major, T = cu_seqlens[B]; sequence b is tokens
 *                 cu_seqlens[b] .. cu_seqlens[b+1]-1 of every head.
 *     q           [B, Hq, D], Hq = Hkv * G; query head h = kvh * G + g reads KV
 *                 head kvh ([AO], GQA example).
 *     out         [B, Hq, D] float32; lse [B, Hq] float32, the natural log of
 *                 sum_t exp(q.k_t / sqrt(D)) over the tokens attended.
 * Pointers.  Every array argument is a DEVICE pointer of the current device
 * unless its comment says "host".  Arrays must start on a 16-byte boundary.
 * Ownership.  The caller allocates and frees every buffer, including the
 * workspace; the library never allocates, frees or synchronises (except
 * sgd_workspace_status and the measurement aid sgd_kernel_timing_*), and never
 * changes the current device.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream).  All work is enqueued on it; results are ready when it completes.
 * Errors.  Every int-returning call returns SGD_OK (0) or a negative SGD_ERR_*
 * code; invalid arguments are rejected on the host before anything is
 * launched.  Conditions only the device can see (a sequence of length 0 in a
 * device array, a bounded wait that ran out) set bits in the 32-bit status word
 * at the start of the workspace (SGD_WS_STATUS_OFFSET), read it with
 * sgd_workspace_status after the stream completes.  No call aborts, traps or
 * throws.
 * Limits.  1 <= G <= 16 (query heads per KV head); D in {64, 128}; Hkv * T < 2^31; B >= 1,
 * Hkv >= 1; several query tokens: G * M <= 64 for the decode, <= 16 for the selection.
 */
#ifndef SGD_H_
#define SGD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types of q and of the cache */
typedef enum { SGD_F32 = 0, SGD_BF16 = 1, SGD_I8 = 2 } sgd_dtype;

/* INT8 scale granularity ([TD] section 6):
 *   A: one K scale per (KV head, sequence, 64-token partition counted from
 *      the sequence's first token; the last partition takes the remainder),
 *      one V scale for the whole tensor;
 *   B: one K scale and one V scale, each for the whole tensor.
 * The _CALIBRATED forms, for sgd_quantize_kv and sgd_quantize_select only, take
 * every per-tensor scale as an input instead of computing it: [TD] section 6 names
 * per-tensor static quantisation and credits INT8's small error to calibrated
 * scales.  A_CALIBRATED reads the V scale from v_scale (the K partition scales are
 * still computed); B_CALIBRATED reads k_scale[0] and v_scale[0].  Values beyond
 * 127.5 * scale saturate to +-127.  The codes they give are scheme A or B codes:
 * an sgd_kv describing them names SGD_SCHEME_A or SGD_SCHEME_B. */
typedef enum {
    SGD_SCHEME_A = 0,
    SGD_SCHEME_B = 1,
    SGD_SCHEME_A_CALIBRATED = 2,
    SGD_SCHEME_B_CALIBRATED = 3
} sgd_scheme;

#define SGD_PARTITION 64 /* scheme-A partition length in tokens */
/* tokens of work the automatic split-KV partition charges each row beside its tokens (its
 * segment setup, epilogue and merge), so that CTAs covering many short rows take fewer tokens */
#define SGD_ROW_COST 512

/* status codes */
#define SGD_OK 0
#define SGD_ERR_NULL -1          /* a required pointer is NULL */
#define SGD_ERR_SHAPE -2         /* B, Hkv, T, D, G or a size out of range */
#define SGD_ERR_DTYPE -3         /* unsupported dtype / scheme combination */
#define SGD_ERR_ALIGN -4         /* an array is not 16-byte aligned */
#define SGD_ERR_WORKSPACE -5     /* workspace smaller than sgd_workspace_size */
#define SGD_ERR_CUDA -6          /* a CUDA runtime call or launch failed */
#define SGD_ERR_DEVICE -7        /* current device is not sm_100 */
#define SGD_ERR_ARG -8           /* any other invalid argument */
#define SGD_ERR_SCRATCH_LIMIT -9 /* needs more scratch than SGD_NOALLOC_SCRATCH_BYTES */

/* device status bits (status word at the start of the workspace) */
#define SGD_STATUS_EMPTY_SEQUENCE 0x1 /* a sequence has length < 1 */
#define SGD_STATUS_WAIT_TIMEOUT 0x2   /* a bounded pipeline wait gave up */
#define SGD_STATUS_SIZE_MISMATCH 0x4  /* device lengths disagree with host sizes */
#define SGD_STATUS_BAD_INDEX 0x8      /* a kept index or block number was outside its sequence */
#define SGD_STATUS_BAD_SCALE 0x10     /* a calibrated scale was negative or not finite: its codes are 0 */

#define SGD_WS_STATUS_OFFSET 0

/* A packed ragged KV cache (all pointers device pointers). */
typedef struct {
    sgd_dtype dtype;            /* of k and v: F32, BF16 or I8 (codes) */
    int32_t B;                  /* sequences */
    int32_t Hkv;                /* KV heads */
    int32_t D;                  /* head dim, 64 or 128 */
    int64_t T;                  /* total tokens = cu_seqlens[B] (host value) */
    const int32_t *cu_seqlens;  /* [B+1] prefix sums of the sequence lengths */
    const void *k;              /* [Hkv, T, D] */
    const void *v;              /* [Hkv, T, D] */
    /* I8 only */
    sgd_scheme scheme;
    const float *k_scale;       /* A: [Hkv, n_parts], sequence b's partitions start at
                                   sum_{b'<b} ceil(L_b'/64); B: [1] */
    const float *v_scale;       /* [1] */
    int64_t n_parts;            /* A: sum_b ceil(L_b / 64) (host value); B: ignored */
    const float *v_norm;        /* I8, for sgd_oam_select: [Hkv, T] ||v_t||_2 of the values
                                   before quantisation (the v_norm output of sgd_quantize_kv or
                                   sgd_quantize_select); NULL otherwise */
} sgd_kv;

/* operations, for sgd_workspace_size */
#define SGD_OP_QUANTIZE 0
#define SGD_OP_OAM_SELECT 1
#define SGD_OP_DECODE 2
#define SGD_OP_QUANTIZE_SELECT 3

/*
 * sgd_quantize_kv -- INT8 KV cache ([TD] section 6).
 *   scale = max|x| / 127 over the group sharing it (float32, IEEE division);
 *   code  = clamp(round_half_even(x / scale), -127, 127), with x / scale the
 *           correctly rounded float32 quotient; a zero scale gives zero codes.
 *   Scheme A: K groups are (KV head, sequence, 64-token partition); V is one
 *   group.  Scheme B: K is one group and V is one group.
 * in       cache to quantise: dtype BF16 or F32 (k_scale/v_scale/scheme ignored)
 * k_codes, v_codes   [Hkv, T, D] int8 outputs
 * k_scale  A: [Hkv, n_parts] (n_parts = sum_b ceil(L_b/64), passed below), B: [1]; output,
 *          except with B_CALIBRATED: input, the calibrated K scale
 * v_scale  [1]: output, except with A_CALIBRATED / B_CALIBRATED: input, the calibrated V scale
 *          (a zero scale gives zero codes; a negative or non-finite one sets
 *          SGD_STATUS_BAD_SCALE in the workspace status and gives zero codes)
 * v_norm   optional [Hkv, T] float32 output (NULL: not written): ||v_t||_2 of every value row,
 *          so that sgd_oam_select can later score the INT8 cache without the original values
 * Codes and scales are bit-exact functions of the input (and of the calibrated scales).
 */
int sgd_quantize_kv(const sgd_kv *in, sgd_scheme scheme, int64_t n_parts,
                    int8_t *k_codes, int8_t *v_codes, float *k_scale, float *v_scale, float *v_norm,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_oam_select -- output-aware token dropping ([TD] section 3).
 *   For every token t of sequence b and KV head kvh:
 *     s_t = max_g (q[b, kvh*G+g] . k_t) / sqrt(D) + beta * ln(||v_t||_2 + eps)
 *   (one index set per KV head, shared by its G query heads); keep the
 *   K_b = clamp(ceil(L_b * keep_num / keep_den), 1, L_b) highest-scoring
 *   tokens, ties broken by the lower token index.
 * q        [B, Hq, D], BF16 or F32 (q_dtype)
 * kv       BF16 or F32: the cache as the caller holds it before quantisation; or
 *          I8 (BF16 q, D = 128): the quantised cache, scored on khat = code * scale with
 *          ||v_t|| taken from kv->v_norm (required), so that only the K codes are read
 * idx      [Hkv, kept_total] int32 output: row (b, kvh) is
 *          idx[kvh, cu_kept[b] .. cu_kept[b+1]-1], kept token positions local
 *          to sequence b, ascending
 * cu_kept  [B+1] int32 output, prefix sums of K_b
 * kept_total  sum_b K_b (host value; the library checks it on the device)
 */
int sgd_oam_select(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv,
                   float beta, float eps, int keep_num, int keep_den,
                   int32_t *idx, int32_t *cu_kept, int64_t kept_total,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_oam_select_multi -- sgd_oam_select for M query tokens per sequence (the speculative step
 * of sgd_decode_attn_multi): one kept set per (sequence, KV head) serves all M * G query rows,
 * so the group maximum runs over all of them:
 *   s_t = max_{m,g} (q[b, m, kvh*G+g] . k_t) / sqrt(D) + beta * ln(||v_t||_2 + eps).
 * q        [B, M, Hq, D] BF16;  1 <= M, G * M <= 16;  the cache BF16 (D 64 or 128) or I8 (D 128,
 *          with kv->v_norm) -- SGD_ERR_DTYPE otherwise
 * workspace   sgd_workspace_size(SGD_OP_OAM_SELECT, kv, G * M, 0, 0) bytes
 * Outputs and errors as in sgd_oam_select; M = 1 is sgd_oam_select.
 */
int sgd_oam_select_multi(const void *q, sgd_dtype q_dtype, int G, int M, const sgd_kv *kv,
                         float beta, float eps, int keep_num, int keep_den,
                         int32_t *idx, int32_t *cu_kept, int64_t kept_total,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_oam_select_blocks -- block-granular token dropping: whole 64-token blocks are kept
 * ([NSA] section 2.1 selects 64-token blocks so that the kept KV is read contiguously; here a
 * block is ranked by the best OAM score s_t of its tokens).  Block j of sequence b holds tokens
 * 64j .. min(64j + 63, L_b - 1) (the last block may be ragged).  Per (b, kvh) the
 * NB_b = clamp(ceil(nb_b * keep_num / keep_den), 1, nb_b) best of the nb_b = ceil(L_b / 64)
 * blocks are kept, ties broken by the lower block index.
 * q, kv, beta, eps, keep_num, keep_den   as in sgd_oam_select
 * n_blocks        sum_b nb_b (host value; checked on the device)
 * blk             [Hkv, kept_blocks_total] int32 output: row (b, kvh) is
 *                 blk[kvh, cu_kept_blocks[b] .. cu_kept_blocks[b+1]-1], block numbers local
 *                 to sequence b, ascending
 * cu_kept_blocks  [B+1] int32 output, prefix sums of NB_b;  kept_blocks_total = sum_b NB_b
 * workspace       sgd_workspace_size(SGD_OP_OAM_SELECT, kv, G, 0, 0) bytes
 */
int sgd_oam_select_blocks(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv,
                          float beta, float eps, int keep_num, int keep_den, int64_t n_blocks,
                          int32_t *blk, int32_t *cu_kept_blocks, int64_t kept_blocks_total,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_quantize_select -- sgd_quantize_kv and sgd_oam_select of one cache in one call, with the
 * same outputs ([TD] sections 6 and 3; the pages' pipeline, section 7, runs both on the same
 * cache).  With a BF16 cache and BF16 q (D in {64, 128}) the K and V of every token are read
 * from HBM once for both: the OAM score pass also writes the scheme-A K codes and scales (or
 * takes max|K| for scheme B) and max|V|; a second pass writes the V codes (and the scheme-B K
 * codes), then the top-K runs.  With calibrated scales (SGD_SCHEME_A_CALIBRATED /
 * B_CALIBRATED) no scale waits for a maximum over the tensor, so the score pass writes every
 * code (and v_norm) itself and the second pass does not run: K and V are read once in all.
 * Other dtypes run the two calls one after the other.
 * Arguments as in sgd_quantize_kv and sgd_oam_select; kv must be BF16 or F32.
 * Workspace: sgd_workspace_size(SGD_OP_QUANTIZE_SELECT, ...).
 */
int sgd_quantize_select(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv,
                        float beta, float eps, int keep_num, int keep_den,
                        sgd_scheme scheme, int64_t n_parts,
                        int8_t *k_codes, int8_t *v_codes, float *k_scale, float *v_scale, float *v_norm,
                        int32_t *idx, int32_t *cu_kept, int64_t kept_total,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_quantize_select_multi -- sgd_quantize_select with the selection of sgd_oam_select_multi:
 * one kept set per (sequence, KV head) for M query tokens, s_t = max over the M * G query rows
 * (q [B, M, Hq, D] BF16 for the fused pass; 1 <= M, G * M <= 16).  The codes, scales and norms
 * are those of sgd_quantize_kv (they do not depend on q).
 * workspace   sgd_workspace_size(SGD_OP_QUANTIZE_SELECT, kv, G * M, 0, 0) bytes
 * Other arguments, outputs and errors as in sgd_quantize_select; M = 1 is sgd_quantize_select.
 */
int sgd_quantize_select_multi(const void *q, sgd_dtype q_dtype, int G, int M, const sgd_kv *kv,
                              float beta, float eps, int keep_num, int keep_den, sgd_scheme scheme,
                              int64_t n_parts, int8_t *k_codes, int8_t *v_codes, float *k_scale,
                              float *v_scale, float *v_norm, int32_t *idx, int32_t *cu_kept,
                              int64_t kept_total, void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_quantize_select_blocks -- sgd_quantize_select with the selection of sgd_oam_select_blocks:
 * whole 64-token blocks ranked by their best token's OAM score ([NSA] section 2.1), the token
 * scores taken in the same pass over K and V that quantises them.
 * n_blocks, blk, cu_kept_blocks, kept_blocks_total   as in sgd_oam_select_blocks
 * Other arguments, outputs and errors as in sgd_quantize_select.
 */
int sgd_quantize_select_blocks(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv,
                               float beta, float eps, int keep_num, int keep_den, sgd_scheme scheme,
                               int64_t n_parts, int8_t *k_codes, int8_t *v_codes, float *k_scale,
                               float *v_scale, float *v_norm, int64_t n_blocks, int32_t *blk,
                               int32_t *cu_kept_blocks, int64_t kept_blocks_total, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * sgd_decode_attn -- split-KV flash-decoding ([TD] section 5, [CD] eq. 5-7).
 *   out[b, h] = sum_t softmax_t(z_t) vhat_t, z_t = q[b, h] . khat_t / sqrt(D),
 *   over every token of sequence b (idx == NULL) or over the kept tokens
 *   idx[kvh, cu_kept[b] ..] (softmax renormalised over that set); khat, vhat
 *   are the cache values (I8: code * scale).  The work of all (sequence, KV
 *   head) rows is cut into equal token ranges, one per CTA (schedule 0: as many
 *   CTAs as fill the GPU, or n_splits when > 0; schedule 1: one CTA per row);
 *   each range emits partial (o_c, lse_c) per row it touches and they are
 *   combined exactly: lse = ln sum_c exp(lse_c), out = sum_c exp(lse_c - lse) o_c.
 * q        [B, Hq, D], BF16 (F32 only with an F32 cache)
 * idx, cu_kept, kept_total   as produced by sgd_oam_select, or NULL/NULL/0
 * q_quant  query-side INT8 ([TD] section 6, schemes A and B quantise Q too), I8 cache with
 *          D = 128 and a BF16 q only: 0 = q as given; 1 = q replaced by code * scale with one
 *          scale per (sequence, query head) row, max|q_row| / 127; 2 = one scale for all of q
 *          (the per-tensor baseline).  Codes follow the K rule (IEEE quotient, ties to even,
 *          clamp to +-127); q.k is then an exact integer dot product of the codes.
 * out      [B, Hq, D] float32;  lse [B, Hq] float32
 */
int sgd_decode_attn(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv,
                    const int32_t *idx, const int32_t *cu_kept, int64_t kept_total,
                    int schedule, int n_splits, int q_quant, float *out, float *lse,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_decode_attn_multi -- M query tokens per sequence in one step ([CD] "decode": speculative
 * decoding verifies n_draft drafted tokens at once, raising the GEMM M dimension of decode from
 * G to (1 + n_draft) * G).  The M new tokens' keys and values are the last M entries of each
 * sequence's cache; query token m (0-based) attends causally, to sequence positions
 * p <= L_b - M + m (of the kept tokens when idx is given).  A query token that sees no token
 * (L_b < M - m) gets out = 0 and lse = -inf.  M = 1 is sgd_decode_attn.
 * q        [B, M, Hq, D] BF16;  out [B, M, Hq, D] float32;  lse [B, M, Hq] float32
 * M        1 <= M and G * M <= 64; with M > 1 the cache is BF16 (D 64 or 128) or I8 (D 128)
 *          (SGD_ERR_DTYPE otherwise).  Above 16 columns (G * M), each split range is run by
 *          ceil(G * M / 16) CTAs, one per group of 16 (query token, head) columns, that read the
 *          same K/V tiles (the later ones from L2)
 * workspace   sgd_workspace_size(SGD_OP_DECODE, kv, G * M, schedule, n_splits) bytes (its G
 *          argument takes up to 64 for SGD_OP_DECODE)
 * Every other argument, and the error behaviour, as in sgd_decode_attn.
 */
int sgd_decode_attn_multi(const void *q, sgd_dtype q_dtype, int G, int M, const sgd_kv *kv,
                          const int32_t *idx, const int32_t *cu_kept, int64_t kept_total,
                          int schedule, int n_splits, int q_quant, float *out, float *lse,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_decode_attn_blocks -- sgd_decode_attn over kept 64-token blocks (the output of
 * sgd_oam_select_blocks): every row attends to all tokens of its kept blocks (a sequence's
 * ragged last block contributes only its L_b - 64 j tokens), renormalised over them.  Each
 * block is one contiguous run of the cache, fetched as whole tiles (no per-token gathers).
 * blk, cu_kept_blocks, kept_blocks_total   as produced by sgd_oam_select_blocks; a block number
 *          outside [0, nb_b) sets SGD_STATUS_BAD_INDEX and is clamped
 * The cache is BF16 (D 64 or 128) or I8 (D 128) with a BF16 q (SGD_ERR_DTYPE otherwise);
 * workspace, schedule, n_splits, q_quant, out, lse and errors as in sgd_decode_attn.
 */
int sgd_decode_attn_blocks(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv,
                           const int32_t *blk, const int32_t *cu_kept_blocks,
                           int64_t kept_blocks_total, int schedule, int n_splits, int q_quant,
                           float *out, float *lse, void *workspace, size_t workspace_bytes,
                           void *stream);

/* Workspace bytes an operation needs for this cache shape (>= 256). For
 * SGD_OP_DECODE, `schedule` and `n_splits` as in sgd_decode_attn and G the columns per KV
 * head (G * M of sgd_decode_attn_multi, up to 64); for the other ops they are ignored and
 * 1 <= G <= 16.  Returns 0 on invalid arguments. */
size_t sgd_workspace_size(int op, const sgd_kv *kv, int G, int schedule, int n_splits);

/* Number of CTAs sgd_decode_attn launches for these arguments (the partition's
 * n_req), or a negative SGD_ERR_* code. */
int sgd_decode_num_ctas(const sgd_kv *kv, int G, const int32_t *idx, int schedule,
                        int n_splits);

/*
 * sgd_plan_segments -- the split-KV partition used by sgd_decode_attn, for
 * inspection.  Rows are (KV head, sequence) pairs in memory order
 * (row = kvh * B + b) with lengths cu[b+1] - cu[b]; each row is padded to a
 * multiple of 16 tokens, followed by row_cost more positions (a fixed work
 * charge; rows of no tokens take none), and the rows are laid end to end;
 * mode 0 cuts this stream of W positions into CTA ranges of
 * S = max(min_chunk, round_up(ceil(W / n_req), 16)), mode 1 gives each row its
 * own CTA.  A segment is the intersection of one CTA range with the real
 * tokens of one row.  sgd_decode_attn's automatic split (schedule 0, no
 * n_splits, tokens rather than blocks) uses row_cost = SGD_ROW_COST and
 * min_chunk 256; a forced split uses row_cost 0.
 * cu        [B+1] device int32 (cu_seqlens, or cu_kept for a kept set)
 * row_cost  a multiple of 16 in [0, 65536]
 * segs      [max_segs, 4] device int32 output: (cta, row, row-local start, length)
 *           in stream order
 * n_segs    [2] device int32 output: number of segments, number of CTAs used
 * workspace device scratch, 16-byte aligned, of at least
 *           2048 + 4 * (B + 2 * B * Hkv + 3 * n_req + 6) + 32 * B * Hkv bytes
 *           (mode 1: n_req = B * Hkv); SGD_ERR_WORKSPACE when smaller
 */
int sgd_plan_segments(const int32_t *cu, int B, int Hkv, int n_req, int min_chunk, int mode, int row_cost,
                      int32_t *segs, int64_t max_segs, int32_t *n_segs,
                      void *workspace, size_t workspace_bytes, void *stream);

/*
 * sgd_decode_attn_noalloc -- sgd_decode_attn for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it serves callers, not the method.
 *   Some callers cannot provide a workspace: a plugin inside a framework that owns all device
 *   memory and offers its plugins no allocator, or a latency-critical loop that may not call
 *   cudaMalloc (it can synchronise the whole device and its latency is unbounded).  This call
 *   takes the same arguments as sgd_decode_attn minus the workspace and computes the same out
 *   and lse with the same kernels.  Their scratch lives in one device array inside the
 *   library, SGD_NOALLOC_SCRATCH_BYTES long, that every GPU which loads the library holds
 *   until the process exits.  Nothing is allocated or freed.
 * status   optional [1] int32 device output: the SGD_STATUS_* bits of this call (or NULL)
 * Returns SGD_ERR_SCRATCH_LIMIT, before launching anything, when the problem needs more scratch
 * than the array holds (sgd_workspace_size(SGD_OP_DECODE, ...) > SGD_NOALLOC_SCRATCH_BYTES).
 * The first call on a device looks up the array's device address (once per device, with that
 * device current); make that first call before any stream capture.  All calls on a device
 * share the array and each starts from the previous call's contents (the call clears the
 * status word itself), so calls whose GPU work overlaps, e.g. on two streams, race: serialise
 * them.
 */
#define SGD_NOALLOC_SCRATCH_BYTES (4u << 20)
int sgd_decode_attn_noalloc(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv,
                            const int32_t *idx, const int32_t *cu_kept, int64_t kept_total,
                            int schedule, int n_splits, int q_quant, float *out, float *lse, int32_t *status,
                            void *stream);

/* Copies the device status word of `workspace` to *status (host) after
 * synchronising `stream`.  The only call that synchronises. */
int sgd_workspace_status(const void *workspace, int32_t *status, void *stream);

/* Static text for a status code. */
const char *sgd_error_string(int code);

/*
 * Per-kernel timing, a measurement aid (not thread-safe; host state of the process).
 * sgd_kernel_timing_start: creates 2 * max_launches CUDA events (1 <= max_launches <= 4096);
 *   from then on every kernel the library launches, up to max_launches of them, is bracketed
 *   by a cudaEventRecord of an event pair on the stream it is launched on.  Calls made while a
 *   stream is captured into a graph add event-record nodes instead.
 * sgd_kernel_timing_stop: turns it off, waits for the recorded events, writes the elapsed
 *   milliseconds of launch k (in launch order) to ms[k] for k < max, the number of bracketed
 *   launches to *count, and frees the events.  SGD_ERR_CUDA if an event failed.
 * sgd_kernel_timing_name: the (mangled) name of launch k's kernel after _stop, or NULL.
 */
int sgd_kernel_timing_start(int max_launches);
int sgd_kernel_timing_stop(float *ms, int max, int *count);
const char *sgd_kernel_timing_name(int k);

/*
 * sgd_stream_read -- measurement aid: the read-only HBM ceiling.  Reads the `bytes` bytes at
 * `buf` (device, 16-byte aligned, bytes a positive multiple of 16) exactly once and XORs them,
 * folded to 32-bit words, into *sink (device, 8-byte aligned); the decode kernels mostly read,
 * so their bandwidth is compared with this rate as well as with a copy's.
 * method   0: 16-byte loads from every thread, eight in flight each, grid-stride;
 *          1: bulk asynchronous copies (cp.async.bulk) of 32 KB chunks into a six-stage
 *             shared-memory ring per SM, each chunk folded by the CTA's warp
 * status   device int32: SGD_STATUS_WAIT_TIMEOUT if a bounded wait of method 1 ran out
 * Time it with events around the call on `stream`; the pages have no counterpart.
 */
int sgd_stream_read(const void *buf, size_t bytes, int method, unsigned long long *sink, int32_t *status,
                    void *stream);

/*
 * sgd_gather_read -- measurement aid: the ceiling of reading scattered rows, as a decode over a
 * kept set does (one K row and one V row of codes per kept token).  For every i < n_rows reads
 * the row_bytes bytes at a + rows[i] * row_bytes and, if b is not NULL, at b + rows[i] *
 * row_bytes, each exactly once, and XORs them, folded to 32-bit words, into *sink (device,
 * 8-byte aligned).  16-byte loads from every thread; the indices of a batch of eight loads
 * are read before its rows.
 * a, b      device, 16-byte aligned (b may be NULL)
 * row_bytes a power of two in [16, 4096]
 * rows      device int32 [n_rows], row numbers (any order, repeats allowed; the caller keeps them
 *           inside the buffers: they are not checked)
 * Time it with events around the call on `stream`; the pages have no counterpart.
 */
int sgd_gather_read(const void *a, const void *b, int64_t row_bytes, const int32_t *rows, int64_t n_rows,
                    unsigned long long *sink, void *stream);

/*
 * sgd_test_pipeline_timeout -- test aid for the bounded pipeline waits (failure detection).
 * Every wait of the decode and score kernels on their shared-memory pipeline is bounded: when
 * it runs out, the kernel sets SGD_STATUS_WAIT_TIMEOUT in the workspace status word, each CTA
 * lets its copies already in flight land and the launch ends promptly with the context usable
 * (no trap, no fault); the outputs of that call are then undefined.
 * polls        > 0: from the next call on, a wait gives up after `polls` polls instead of the
 *              built-in limit (about 4 million); 0 restores the built-in limit
 * idle_producer != 0: the producer warps issue no copies at all, so every consumer wait runs out
 *              with nothing in flight -- how a test makes the timeout path run without a fault;
 *              0 restores normal operation
 * Host state of the process, not thread-safe; affects calls enqueued after it.  SGD_ERR_ARG for
 * polls < 0.  The pages have no counterpart: this serves testing only.
 */
int sgd_test_pipeline_timeout(int64_t polls, int idle_producer);

/* Library version, (major << 16) | minor. */
int sgd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SGD_H_ */
