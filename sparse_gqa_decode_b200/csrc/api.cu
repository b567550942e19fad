// api.cu -- the C ABI of libsgd.so (declared and documented in include/sgd.h).
//
// Each entry point validates its arguments on the host, lays out the caller's
// workspace, and enqueues its kernels on the caller's stream.  Nothing here
// allocates, frees or synchronises (except sgd_workspace_status, which reads the
// device status word).
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace sgd {

namespace {

constexpr int kMaxDevices = 64;
constexpr int kAutoMinChunk = 256;  // smallest CTA range when the split is automatic

struct DevInfo {
    int ok = -1;  // -1 unknown, 0 not sm_100, 1 ok
    int sms = 0;
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;

int current_device(DevInfo **info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SGD_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo &d = g_dev[dev];
    if (d.ok < 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return SGD_ERR_CUDA;
        d.ok = (major == 10 && minor == 0) ? 1 : 0;
        d.sms = sms;
    }
    *info = &d;
    return d.ok ? SGD_OK : SGD_ERR_DEVICE;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_kv(const sgd_kv *kv) {
    if (!kv || !kv->cu_seqlens || !kv->k || !kv->v) return SGD_ERR_NULL;
    if (kv->B < 1 || kv->Hkv < 1 || kv->T < 1) return SGD_ERR_SHAPE;
    if (kv->D != 64 && kv->D != 128) return SGD_ERR_SHAPE;
    if ((int64_t)kv->Hkv * kv->T >= (int64_t(1) << 31)) return SGD_ERR_SHAPE;
    if ((int64_t)kv->B * kv->Hkv >= (int64_t(1) << 24)) return SGD_ERR_SHAPE;
    if (kv->dtype != SGD_F32 && kv->dtype != SGD_BF16 && kv->dtype != SGD_I8) return SGD_ERR_DTYPE;
    if (!aligned16(kv->k) || !aligned16(kv->v)) return SGD_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(kv->cu_seqlens) & 3u) != 0) return SGD_ERR_ALIGN;
    return SGD_OK;
}

// workspace layout
struct Layout {
    size_t row_pos = 0, row_slot0 = 0, cta_begin = 0, cta_slot0 = 0, cta_row0 = 0, row_info = 0, row_done = 0;
    size_t seq_part0 = 0;
    size_t o_part = 0, lse_part = 0, scores = 0, bscores = 0, total = 0;
};

size_t take(size_t &off, size_t bytes) {
    const size_t at = off;
    off += (bytes + 255) / 256 * 256;
    return at;
}

Layout layout(int op, int B, int Hkv, int G, int D, int64_t T, int n_req) {
    Layout L;
    size_t off = sizeof(WsHeader);
    const int64_t R = (int64_t)B * Hkv;
    L.seq_part0 = take(off, (size_t)(B + 1) * 4);
    if (op != SGD_OP_QUANTIZE) {
        L.row_pos = take(off, (size_t)(R + 1) * 4);
        L.row_slot0 = take(off, (size_t)(R + 1) * 4);
        L.cta_begin = take(off, (size_t)(n_req + 1) * 4);
        L.cta_slot0 = take(off, (size_t)(n_req + 1) * 4);
        L.cta_row0 = take(off, (size_t)(n_req + 1) * 4);
        L.row_info = take(off, (size_t)R * sizeof(RowInfo));
    }
    if (op == SGD_OP_DECODE) {
        L.row_done = take(off, (size_t)R * kMaxColGroups * 4);  // per row and column group
        const int64_t slots = (int64_t)n_req + R;
        L.o_part = take(off, (size_t)slots * G * D * 4);
        L.lse_part = take(off, (size_t)slots * G * 4);
    }
    if (op == SGD_OP_OAM_SELECT) {
        L.scores = take(off, (size_t)Hkv * T * 4);
        L.bscores = take(off, (size_t)Hkv * (T / kPart + B) * 4);  // block selection: per-block scores
    }
    L.total = off;
    return L;
}

PlanView plan_view(uint8_t *ws, const Layout &L) {
    PlanView pv;
    pv.row_pos = reinterpret_cast<int32_t *>(ws + L.row_pos);
    pv.row_slot0 = reinterpret_cast<int32_t *>(ws + L.row_slot0);
    pv.cta_begin = reinterpret_cast<int32_t *>(ws + L.cta_begin);
    pv.cta_slot0 = reinterpret_cast<int32_t *>(ws + L.cta_slot0);
    pv.cta_row0 = reinterpret_cast<int32_t *>(ws + L.cta_row0);
    pv.row_info = reinterpret_cast<RowInfo *>(ws + L.row_info);
    pv.row_done = L.row_done ? reinterpret_cast<int32_t *>(ws + L.row_done) : nullptr;
    pv.seq_part0 = reinterpret_cast<int32_t *>(ws + L.seq_part0);
    return pv;
}

// CTAs requested from the partition for a decode / score launch.
// G: columns per KV head (the decode's M * G); above 16 each planned range is run by one CTA per
// group of 16 columns, so the automatic count is divided among the groups.
int decode_n_req(const DevInfo &dev, const sgd_kv *kv, sgd_dtype q_dtype, int G, bool indexed, bool score,
                 int schedule, int n_splits, int *n_req) {
    if (schedule == 1 && !score) {
        *n_req = kv->B * kv->Hkv;
        return SGD_OK;
    }
    if (schedule != 0) return SGD_ERR_ARG;
    if (n_splits > 0 && !score) {
        *n_req = n_splits;
        return SGD_OK;
    }
    if (n_splits < 0) return SGD_ERR_ARG;
    const int per = decode_ctas_per_sm(kv->dtype, q_dtype, kv->D, std::min(G, 16), indexed, score);
    if (per < 1) return SGD_ERR_CUDA;
    const int ncg = (G + 15) / 16;
    *n_req = (dev.sms * per + ncg - 1) / ncg;
    return SGD_OK;
}

// CTAs of the fused score + quantise pass of sgd_quantize_select: every SM's worth of them.
int fused_n_req(const DevInfo &dev, const sgd_kv *kv, int G) {
    const int per = score_quantize_ctas_per_sm(kv->D, G);
    return per > 0 ? dev.sms * per : 0;
}

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

// per-launch timing: event pairs around each launch while on (a measurement aid, one thread)
struct KernelTiming {
    bool on = false;
    int n = 0;
    std::vector<cudaEvent_t> ev;  // 2 per launch slot
    std::vector<const void *> fn;
    std::vector<std::string> names;
    void release() {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
        ev.clear();
        fn.clear();
    }
};
KernelTiming g_kt;

// sgd_test_pipeline_timeout: a lowered wait limit and idle producers (host state of the process)
struct TestHooks {
    long long wait_limit = 0;  // 0: kWaitLimit
    int idle_producer = 0;
};
TestHooks g_hooks;

}  // namespace

void apply_test_hooks(DecodeArgs &a) {
    a.wait_limit = g_hooks.wait_limit > 0 ? g_hooks.wait_limit : kWaitLimit;
    a.idle_producer = g_hooks.idle_producer;
}

int kt_begin(cudaStream_t s) {
    if (!g_kt.on || g_kt.n >= (int)g_kt.fn.size()) return -1;
    const int k = g_kt.n;
    return cudaEventRecord(g_kt.ev[2 * k], s) == cudaSuccess ? k : -1;
}

void kt_end(cudaStream_t s, int k, const void *kern) {
    if (cudaEventRecord(g_kt.ev[2 * k + 1], s) != cudaSuccess) return;
    g_kt.fn[k] = kern;
    g_kt.n = k + 1;
}

}  // namespace sgd

using namespace sgd;

namespace {

// The decode behind sgd_decode_attn, _multi and _blocks.  blocks: idx / cu_kept / kept_total
// list kept 64-token blocks (the tensor-core kernel reads each as one box per tensor).
int decode_impl(const void *q, sgd_dtype q_dtype, int G, int M, const sgd_kv *kv, const int32_t *idx,
                const int32_t *cu_kept, int64_t kept_total, bool blocks, int schedule, int n_splits, int q_quant,
                float *out, float *lse, void *workspace, size_t workspace_bytes, void *stream) {
    int rc = check_kv(kv);
    if (rc != SGD_OK) return rc;
    if (!q || !out || !lse || !workspace) return SGD_ERR_NULL;
    if (G < 1 || G > 16 || M < 1 || G * M > 16 * kMaxColGroups) return SGD_ERR_SHAPE;
    const int NC = G * M;  // the kernels' columns per KV head: (query token, head) pairs
    const int ncg = (NC + 15) / 16;  // CTAs per planned range, one per 16 columns
    // several query tokens, and kept blocks, run on the tensor-core kernel only
    if ((M > 1 || blocks) && decode_family(kv->dtype, q_dtype, kv->D, false) != kFamilyMma) return SGD_ERR_DTYPE;
    if (q_dtype != SGD_BF16 && q_dtype != SGD_F32) return SGD_ERR_DTYPE;
    if (q_dtype == SGD_F32 && kv->dtype != SGD_F32) return SGD_ERR_DTYPE;
    const bool listed = idx != nullptr;  // kept tokens or kept blocks
    if (listed != (cu_kept != nullptr)) return SGD_ERR_NULL;
    if (listed && (kept_total < kv->B || kept_total > (blocks ? kv->T / SGD_PARTITION + kv->B : kv->T)))
        return SGD_ERR_SHAPE;
    const bool indexed = listed && !blocks;  // token gathers
    if (kv->dtype == SGD_I8) {
        if (!kv->k_scale || !kv->v_scale) return SGD_ERR_NULL;
        if (kv->scheme != SGD_SCHEME_A && kv->scheme != SGD_SCHEME_B) return SGD_ERR_DTYPE;
        if (kv->scheme == SGD_SCHEME_A && (kv->n_parts < kv->B || kv->n_parts > kv->T / SGD_PARTITION + kv->B))
            return SGD_ERR_SHAPE;
    }
    if (q_quant < 0 || q_quant > 2) return SGD_ERR_ARG;
    if (q_quant != 0 && (kv->dtype != SGD_I8 || q_dtype != SGD_BF16)) return SGD_ERR_DTYPE;
    if (q_quant != 0 && kv->D != 128) return SGD_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return SGD_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (indexed && (reinterpret_cast<uintptr_t>(idx) & 3u)))
        return SGD_ERR_ALIGN;
    DevInfo *dev;
    if ((rc = current_device(&dev)) != SGD_OK) return rc;
    int n_req = 0;
    if ((rc = decode_n_req(*dev, kv, q_dtype, NC, indexed, false, schedule, n_splits, &n_req)) != SGD_OK) return rc;
    const Layout L = layout(SGD_OP_DECODE, kv->B, kv->Hkv, NC, kv->D, kv->T, n_req);
    if (workspace_bytes < L.total) return SGD_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    const PlanView pv = plan_view(ws, L);
    cudaStream_t s = as_stream(stream);
    // blocks: segments start and end on block boundaries (granule 64), lengths counted in blocks
    const int granule = blocks ? kPart : kGranule;
    const int min_chunk = (n_splits > 0 || schedule == 1) ? granule : kAutoMinChunk;
    // the automatic token split charges every row SGD_ROW_COST tokens of work (its segment setup,
    // epilogue and merge), while the stream positions stay below 2^31
    const int64_t R = (int64_t)kv->B * kv->Hkv;
    const bool charge = !blocks && schedule == 0 && n_splits == 0 &&
                        (int64_t)kv->Hkv * kv->T + R * (kGranule + SGD_ROW_COST) < (int64_t(1) << 31);
    launch_plan(listed ? cu_kept : kv->cu_seqlens, kv->cu_seqlens, kv->B, kv->Hkv, n_req, min_chunk, schedule, pv,
                hdr, s, granule, out, lse, G, kv->D, q_quant == 2 ? static_cast<const __nv_bfloat16 *>(q) : nullptr,
                (int64_t)kv->B * M * kv->Hkv * G * kv->D, M, blocks ? kPart : 1, ncg, charge ? SGD_ROW_COST : 0);
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q;
    a.q_f32 = q_dtype == SGD_F32;
    a.cu_seq = kv->cu_seqlens;
    a.cu_kept = cu_kept;
    a.idx = idx;
    a.k = kv->k;
    a.v = kv->v;
    a.k_scale = kv->k_scale;
    a.v_scale = kv->v_scale;
    a.scheme = kv->scheme;
    a.B = kv->B;
    a.Hkv = kv->Hkv;
    a.G = G;
    a.M = M;
    a.D = kv->D;
    a.T = kv->T;
    a.Kt = listed ? kept_total : 0;
    a.blk = blocks ? 1 : 0;
    a.ncg = ncg;
    a.n_parts = kv->dtype == SGD_I8 && kv->scheme == SGD_SCHEME_A ? kv->n_parts : 0;
    a.sm_scale = (float)(1.0 / sqrt((double)kv->D));
    a.sm_scale_log2 = (float)(1.4426950408889634 / sqrt((double)kv->D));
    a.plan = pv;
    a.o_part = reinterpret_cast<float *>(ws + L.o_part);
    a.lse_part = reinterpret_cast<float *>(ws + L.lse_part);
    a.out = out;
    a.lse = lse;
    a.status = &hdr->status;
    a.q_quant = q_quant;
    a.q_scale = &hdr->q_scale;
    apply_test_hooks(a);
    int e = launch_decode(a, kv->dtype, q_dtype, indexed, false, n_req * ncg, s);
    if (e != 0) return SGD_ERR_CUDA;
    // the tensor-core kernel merges each row itself (its last CTA); the CUDA-core one leaves partials
    if (decode_family(kv->dtype, q_dtype, kv->D, false) == kFamilyMma) return SGD_OK;
    e = launch_merge(a, out, lse, s);
    return e == 0 ? SGD_OK : SGD_ERR_CUDA;
}


// The selection behind sgd_oam_select and sgd_oam_select_blocks.  blocks: rank the 64-token
// blocks by their best token's score and keep whole blocks (n_blocks = sum_b ceil(L_b / 64)).
int select_impl(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv, float beta, float eps, int keep_num,
                int keep_den, bool blocks, int64_t n_blocks, int32_t *idx, int32_t *cu_kept, int64_t kept_total,
                void *workspace, size_t workspace_bytes, void *stream, int M = 1) {
    int rc = check_kv(kv);
    if (rc != SGD_OK) return rc;
    if (!q || !idx || !cu_kept || !workspace) return SGD_ERR_NULL;
    if (G < 1 || G > 16 || M < 1 || G * M > 16) return SGD_ERR_SHAPE;
    // several query tokens: the tensor-core score kernel, its columns the M * G query rows
    if (M > 1 && decode_family(kv->dtype, q_dtype, kv->D, true) != kFamilyMma) return SGD_ERR_DTYPE;
    if (q_dtype != SGD_BF16 && q_dtype != SGD_F32) return SGD_ERR_DTYPE;
    if (kv->dtype == SGD_I8) {
        // scoring the INT8 cache: khat = code * scale, ||v|| from the norms stored at quantisation
        if (q_dtype != SGD_BF16 || kv->D != 128) return SGD_ERR_DTYPE;
        if (!kv->k_scale || !kv->v_norm) return SGD_ERR_NULL;
        if (kv->scheme != SGD_SCHEME_A && kv->scheme != SGD_SCHEME_B) return SGD_ERR_DTYPE;
        if (kv->scheme == SGD_SCHEME_A && (kv->n_parts < kv->B || kv->n_parts > kv->T / SGD_PARTITION + kv->B))
            return SGD_ERR_SHAPE;
        if (reinterpret_cast<uintptr_t>(kv->v_norm) & 3u) return SGD_ERR_ALIGN;
    } else if (kv->dtype != SGD_BF16 && kv->dtype != SGD_F32) {
        return SGD_ERR_DTYPE;
    }
    if (keep_num < 0 || keep_den < 1 || keep_num > keep_den) return SGD_ERR_ARG;
    if (blocks && (n_blocks < kv->B || n_blocks > kv->T / SGD_PARTITION + kv->B)) return SGD_ERR_SHAPE;
    if (kept_total < kv->B || kept_total > (blocks ? n_blocks : kv->T)) return SGD_ERR_SHAPE;
    if (!isfinite(beta) || !isfinite(eps) || eps < 0.f) return SGD_ERR_ARG;
    if (!aligned16(q) || !aligned16(workspace)) return SGD_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(cu_kept) & 3u)) return SGD_ERR_ALIGN;
    DevInfo *dev;
    if ((rc = current_device(&dev)) != SGD_OK) return rc;
    int n_req = 0;
    if ((rc = decode_n_req(*dev, kv, q_dtype, G * M, false, true, 0, 0, &n_req)) != SGD_OK) return rc;
    const Layout L = layout(SGD_OP_OAM_SELECT, kv->B, kv->Hkv, G * M, kv->D, kv->T, n_req);
    if (workspace_bytes < L.total) return SGD_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    const PlanView pv = plan_view(ws, L);
    cudaStream_t s = as_stream(stream);
    launch_plan(kv->cu_seqlens, kv->cu_seqlens, kv->B, kv->Hkv, n_req, kAutoMinChunk, 0, pv, hdr, s);
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q;
    a.q_f32 = q_dtype == SGD_F32;
    a.cu_seq = kv->cu_seqlens;
    a.k = kv->k;
    a.v = kv->v;
    a.B = kv->B;
    a.Hkv = kv->Hkv;
    a.G = G;
    a.M = M;
    a.D = kv->D;
    a.T = kv->T;
    a.sm_scale = (float)(1.0 / sqrt((double)kv->D));
    a.sm_scale_log2 = (float)(1.4426950408889634 / sqrt((double)kv->D));
    a.beta = beta;
    a.eps = eps;
    if (kv->dtype == SGD_I8) {
        a.k_scale = kv->k_scale;
        a.scheme = kv->scheme;
        a.n_parts = kv->scheme == SGD_SCHEME_A ? kv->n_parts : 0;
        a.v_norm = kv->v_norm;
    }
    a.scores = reinterpret_cast<float *>(ws + L.scores);
    a.plan = pv;
    a.status = &hdr->status;
    apply_test_hooks(a);
    int e = launch_decode(a, kv->dtype, q_dtype, false, true, n_req, s);
    if (e != 0) return SGD_ERR_CUDA;
    if (blocks) {  // block scores, then the top blocks of each row (the plan's partition offsets = block offsets)
        float *bs = reinterpret_cast<float *>(ws + L.bscores);
        e = launch_block_max(a.scores, kv->cu_seqlens, pv.seq_part0, kv->B, kv->Hkv, kv->T, n_blocks, bs,
                             &hdr->status, s);
        if (e != 0) return SGD_ERR_CUDA;
        e = launch_topk(bs, pv.seq_part0, kv->B, kv->Hkv, n_blocks, keep_num, keep_den, idx, cu_kept, kept_total,
                        &hdr->status, s);
        return e == 0 ? SGD_OK : SGD_ERR_CUDA;
    }
    e = launch_topk(a.scores, kv->cu_seqlens, kv->B, kv->Hkv, kv->T, keep_num, keep_den, idx, cu_kept, kept_total,
                    &hdr->status, s);
    return e == 0 ? SGD_OK : SGD_ERR_CUDA;
}
bool quant_scheme_ok(sgd_scheme s) {
    return s == SGD_SCHEME_A || s == SGD_SCHEME_B || s == SGD_SCHEME_A_CALIBRATED || s == SGD_SCHEME_B_CALIBRATED;
}
// the scheme-A forms: K scales per 64-token partition
bool has_partitions(sgd_scheme s) { return s == SGD_SCHEME_A || s == SGD_SCHEME_A_CALIBRATED; }

}  // namespace

extern "C" {

int sgd_version(void) { return (1 << 16) | 0; }

int sgd_stream_read(const void *buf, size_t bytes, int method, unsigned long long *sink, int32_t *status,
                    void *stream) {
    if (!buf || !sink || !status) return SGD_ERR_NULL;
    if (bytes == 0 || bytes % 16 != 0) return SGD_ERR_SHAPE;
    if (method != 0 && method != 1) return SGD_ERR_ARG;
    if (!aligned16(buf) || (reinterpret_cast<uintptr_t>(sink) & 7u) || (reinterpret_cast<uintptr_t>(status) & 3u))
        return SGD_ERR_ALIGN;
    DevInfo *dev;
    int rc = current_device(&dev);
    if (rc != SGD_OK) return rc;
    return launch_stream_read(buf, bytes, method, sink, status, dev->sms, as_stream(stream)) == 0 ? SGD_OK
                                                                                                  : SGD_ERR_CUDA;
}

int sgd_gather_read(const void *a, const void *b, int64_t row_bytes, const int32_t *rows, int64_t n_rows,
                    unsigned long long *sink, void *stream) {
    if (!a || !rows || !sink) return SGD_ERR_NULL;
    if (row_bytes < 16 || row_bytes > 4096 || (row_bytes & (row_bytes - 1)) != 0 || n_rows < 1 ||
        n_rows >= (int64_t(1) << 40))
        return SGD_ERR_SHAPE;
    if (!aligned16(a) || (b && !aligned16(b)) || (reinterpret_cast<uintptr_t>(rows) & 3u) ||
        (reinterpret_cast<uintptr_t>(sink) & 7u))
        return SGD_ERR_ALIGN;
    DevInfo *dev;
    int rc = current_device(&dev);
    if (rc != SGD_OK) return rc;
    return launch_gather_read(a, b, row_bytes, rows, n_rows, sink, dev->sms, as_stream(stream)) == 0 ? SGD_OK
                                                                                                     : SGD_ERR_CUDA;
}

int sgd_test_pipeline_timeout(int64_t polls, int idle_producer) {
    if (polls < 0) return SGD_ERR_ARG;
    g_hooks.wait_limit = (long long)polls;
    g_hooks.idle_producer = idle_producer != 0;
    return SGD_OK;
}

int sgd_kernel_timing_start(int max_launches) {
    if (max_launches < 1 || max_launches > 4096) return SGD_ERR_ARG;
    g_kt.on = false;
    g_kt.release();
    g_kt.names.clear();
    g_kt.n = 0;
    g_kt.ev.assign(2 * (size_t)max_launches, nullptr);
    for (auto &e : g_kt.ev) {
        if (cudaEventCreate(&e) != cudaSuccess) {
            e = nullptr;
            for (auto &x : g_kt.ev)
                if (x) cudaEventDestroy(x);
            g_kt.ev.clear();
            return SGD_ERR_CUDA;
        }
    }
    g_kt.fn.assign((size_t)max_launches, nullptr);
    g_kt.on = true;
    return SGD_OK;
}

int sgd_kernel_timing_stop(float *ms, int max, int *count) {
    if (!ms || !count || max < 0) return SGD_ERR_NULL;
    g_kt.on = false;
    g_kt.names.clear();
    int rc = SGD_OK;
    for (int k = 0; k < g_kt.n; ++k) {
        float t = 0.f;
        if (cudaEventSynchronize(g_kt.ev[2 * k + 1]) != cudaSuccess ||
            cudaEventElapsedTime(&t, g_kt.ev[2 * k], g_kt.ev[2 * k + 1]) != cudaSuccess)
            rc = SGD_ERR_CUDA;
        if (k < max) ms[k] = t;
        const char *name = nullptr;
        if (cudaFuncGetName(&name, g_kt.fn[k]) != cudaSuccess || !name) name = "?";
        g_kt.names.emplace_back(name);
    }
    *count = g_kt.n;
    g_kt.release();
    return rc;
}

const char *sgd_kernel_timing_name(int k) {
    return (k >= 0 && k < (int)g_kt.names.size()) ? g_kt.names[k].c_str() : nullptr;
}

const char *sgd_error_string(int code) {
    switch (code) {
        case SGD_OK: return "ok";
        case SGD_ERR_NULL: return "a required pointer is NULL";
        case SGD_ERR_SHAPE: return "a size is out of range (B, Hkv, T, D in {64,128}, G in [1,16], Hkv*T < 2^31)";
        case SGD_ERR_DTYPE: return "unsupported dtype or scheme";
        case SGD_ERR_ALIGN: return "an array is not 16-byte aligned";
        case SGD_ERR_WORKSPACE: return "workspace smaller than sgd_workspace_size";
        case SGD_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
        case SGD_ERR_DEVICE: return "the current device is not an sm_100 GPU";
        case SGD_ERR_ARG: return "invalid argument";
        case SGD_ERR_SCRATCH_LIMIT: return "the problem needs more scratch than SGD_NOALLOC_SCRATCH_BYTES";
        default: return "unknown status";
    }
}

size_t sgd_workspace_size(int op, const sgd_kv *kv, int G, int schedule, int n_splits) {
    if (check_kv(kv) != SGD_OK) return 0;
    if (op == SGD_OP_QUANTIZE) return layout(op, kv->B, kv->Hkv, 0, kv->D, kv->T, 0).total;
    // G: query heads per KV head; for the decode, the columns M * G of sgd_decode_attn_multi
    if (G < 1 || G > (op == SGD_OP_DECODE ? 16 * kMaxColGroups : 16)) return 0;
    DevInfo *dev;
    if (current_device(&dev) != SGD_OK) return 0;
    int n_req = 0;
    const bool fused = op == SGD_OP_QUANTIZE_SELECT;
    if (fused) op = SGD_OP_OAM_SELECT;  // the fused call needs the select layout
    const bool score = op == SGD_OP_OAM_SELECT;
    if (op != SGD_OP_DECODE && !score) return 0;
    // the largest count over the kernels the call may pick: indexed or not, bf16 or f32 query
    if (decode_n_req(*dev, kv, SGD_BF16, G, false, score, score ? 0 : schedule, score ? 0 : n_splits, &n_req) !=
        SGD_OK)
        return 0;
    for (int ix = 0; ix < 2; ++ix) {
        for (sgd_dtype qd : {SGD_BF16, SGD_F32}) {
            int other = 0;
            if (decode_n_req(*dev, kv, qd, G, ix == 1, score, score ? 0 : schedule, score ? 0 : n_splits, &other) ==
                SGD_OK)
                n_req = std::max(n_req, other);
        }
    }
    if (fused) n_req = std::max(n_req, fused_n_req(*dev, kv, G));
    return layout(op, kv->B, kv->Hkv, G, kv->D, kv->T, n_req).total;
}

int sgd_decode_num_ctas(const sgd_kv *kv, int G, const int32_t *idx, int schedule, int n_splits) {
    int rc = check_kv(kv);
    if (rc != SGD_OK) return rc;
    DevInfo *dev;
    if ((rc = current_device(&dev)) != SGD_OK) return rc;
    int n_req = 0;
    rc = decode_n_req(*dev, kv, SGD_BF16, G, idx != nullptr, false, schedule, n_splits, &n_req);
    return rc == SGD_OK ? n_req : rc;
}

int sgd_quantize_kv(const sgd_kv *in, sgd_scheme scheme, int64_t n_parts, int8_t *k_codes, int8_t *v_codes,
                    float *k_scale, float *v_scale, float *v_norm, void *workspace, size_t workspace_bytes,
                    void *stream) {
    int rc = check_kv(in);
    if (rc != SGD_OK) return rc;
    if (!k_codes || !v_codes || !k_scale || !v_scale || !workspace) return SGD_ERR_NULL;
    if (in->dtype != SGD_BF16 && in->dtype != SGD_F32) return SGD_ERR_DTYPE;
    if (!quant_scheme_ok(scheme)) return SGD_ERR_DTYPE;
    if (has_partitions(scheme) && (n_parts < in->B || n_parts > in->T / SGD_PARTITION + in->B)) return SGD_ERR_SHAPE;
    if (!aligned16(k_codes) || !aligned16(v_codes) || !aligned16(workspace)) return SGD_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(v_norm) & 3u))
        return SGD_ERR_ALIGN;
    const Layout L = layout(SGD_OP_QUANTIZE, in->B, in->Hkv, 0, in->D, in->T, 0);
    if (workspace_bytes < L.total) return SGD_ERR_WORKSPACE;
    DevInfo *dev;
    if ((rc = current_device(&dev)) != SGD_OK) return rc;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int e = launch_quantize(in->k, in->v, in->dtype, in->cu_seqlens, in->B, in->Hkv, in->D, in->T, scheme,
                                  n_parts, k_codes, v_codes, k_scale, v_scale, v_norm, reinterpret_cast<WsHeader *>(ws),
                                  reinterpret_cast<int32_t *>(ws + L.seq_part0), dev->sms, as_stream(stream));
    return e == 0 ? SGD_OK : SGD_ERR_CUDA;
}

int sgd_oam_select(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv, float beta, float eps, int keep_num,
                   int keep_den, int32_t *idx, int32_t *cu_kept, int64_t kept_total, void *workspace,
                   size_t workspace_bytes, void *stream) {
    return select_impl(q, q_dtype, G, kv, beta, eps, keep_num, keep_den, false, 0, idx, cu_kept, kept_total, workspace,
                       workspace_bytes, stream);
}

int sgd_oam_select_multi(const void *q, sgd_dtype q_dtype, int G, int M, const sgd_kv *kv, float beta, float eps,
                         int keep_num, int keep_den, int32_t *idx, int32_t *cu_kept, int64_t kept_total,
                         void *workspace, size_t workspace_bytes, void *stream) {
    return select_impl(q, q_dtype, G, kv, beta, eps, keep_num, keep_den, false, 0, idx, cu_kept, kept_total, workspace,
                       workspace_bytes, stream, M);
}

int sgd_oam_select_blocks(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv, float beta, float eps,
                          int keep_num, int keep_den, int64_t n_blocks, int32_t *blk, int32_t *cu_kept_blocks,
                          int64_t kept_blocks_total, void *workspace, size_t workspace_bytes, void *stream) {
    return select_impl(q, q_dtype, G, kv, beta, eps, keep_num, keep_den, true, n_blocks, blk, cu_kept_blocks,
                       kept_blocks_total, workspace, workspace_bytes, stream);
}

// The quantisation and selection behind sgd_quantize_select, _multi (M query tokens, G * M <= 16
// columns) and _blocks (whole 64-token blocks ranked by their best token, n_blocks of them).
static int quantize_select_impl(const void *q, sgd_dtype q_dtype, int G, int M, const sgd_kv *kv, float beta,
                                float eps, int keep_num, int keep_den, sgd_scheme scheme, int64_t n_parts,
                                int8_t *k_codes, int8_t *v_codes, float *k_scale, float *v_scale, float *v_norm,
                                bool blocks, int64_t n_blocks, int32_t *idx, int32_t *cu_kept, int64_t kept_total,
                                void *workspace, size_t workspace_bytes, void *stream) {
    int rc = check_kv(kv);
    if (rc != SGD_OK) return rc;
    if (!q || !idx || !cu_kept || !workspace || !k_codes || !v_codes || !k_scale || !v_scale) return SGD_ERR_NULL;
    if (G < 1 || G > 16 || M < 1 || G * M > 16) return SGD_ERR_SHAPE;
    if (kv->dtype != SGD_BF16 && kv->dtype != SGD_F32) return SGD_ERR_DTYPE;
    if (q_dtype != SGD_BF16 && q_dtype != SGD_F32) return SGD_ERR_DTYPE;
    if (!quant_scheme_ok(scheme)) return SGD_ERR_DTYPE;
    if (has_partitions(scheme) && (n_parts < kv->B || n_parts > kv->T / SGD_PARTITION + kv->B)) return SGD_ERR_SHAPE;
    if (keep_num < 0 || keep_den < 1 || keep_num > keep_den) return SGD_ERR_ARG;
    if (blocks && (n_blocks < kv->B || n_blocks > kv->T / SGD_PARTITION + kv->B)) return SGD_ERR_SHAPE;
    if (kept_total < kv->B || kept_total > (blocks ? n_blocks : kv->T)) return SGD_ERR_SHAPE;
    if (!isfinite(beta) || !isfinite(eps) || eps < 0.f) return SGD_ERR_ARG;
    if (!aligned16(q) || !aligned16(workspace) || !aligned16(k_codes) || !aligned16(v_codes)) return SGD_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(cu_kept) & 3u) ||
        (reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(v_norm) & 3u))
        return SGD_ERR_ALIGN;
    if (decode_family(kv->dtype, q_dtype, kv->D, true) != kFamilyMma) {
        // no fused kernel for this dtype: the two passes one after the other
        rc = sgd_quantize_kv(kv, scheme, n_parts, k_codes, v_codes, k_scale, v_scale, v_norm, workspace,
                             workspace_bytes, stream);
        if (rc != SGD_OK) return rc;
        return select_impl(q, q_dtype, G, kv, beta, eps, keep_num, keep_den, blocks, n_blocks, idx, cu_kept,
                           kept_total, workspace, workspace_bytes, stream, M);
    }
    DevInfo *dev;
    if ((rc = current_device(&dev)) != SGD_OK) return rc;
    const int n_req = fused_n_req(*dev, kv, G * M);
    if (n_req < 1) return SGD_ERR_CUDA;
    const Layout L = layout(SGD_OP_OAM_SELECT, kv->B, kv->Hkv, G * M, kv->D, kv->T, n_req);
    if (workspace_bytes < L.total) return SGD_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    const PlanView pv = plan_view(ws, L);
    cudaStream_t s = as_stream(stream);
    // tiles of the fused pass must be whole 64-token partitions: plan granule 64
    launch_plan(kv->cu_seqlens, kv->cu_seqlens, kv->B, kv->Hkv, n_req, kAutoMinChunk, 0, pv, hdr, s, kPart);
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q;
    a.cu_seq = kv->cu_seqlens;
    a.k = kv->k;
    a.v = kv->v;
    a.B = kv->B;
    a.Hkv = kv->Hkv;
    a.G = G;
    a.M = M;
    a.D = kv->D;
    a.T = kv->T;
    const bool cal = scheme == SGD_SCHEME_A_CALIBRATED || scheme == SGD_SCHEME_B_CALIBRATED;
    const sgd_scheme base = has_partitions(scheme) ? SGD_SCHEME_A : SGD_SCHEME_B;
    a.n_parts = base == SGD_SCHEME_A ? n_parts : 0;
    a.sm_scale = (float)(1.0 / sqrt((double)kv->D));
    a.sm_scale_log2 = (float)(1.4426950408889634 / sqrt((double)kv->D));
    a.beta = beta;
    a.eps = eps;
    a.scores = reinterpret_cast<float *>(ws + L.scores);
    a.qscheme = base;
    a.k_codes = k_codes;
    a.k_scale_out = k_scale;
    a.amax_bits = hdr->amax_bits;
    if (cal) {  // every code (and norm) in the score pass: no second pass
        a.cal_v_scale = v_scale;
        a.cal_k_scale = base == SGD_SCHEME_B ? k_scale : nullptr;
        a.v_codes_out = v_codes;
        a.v_norm_out = v_norm;
    }
    a.plan = pv;
    a.status = &hdr->status;
    apply_test_hooks(a);
    int e = launch_score_quantize(a, n_req, s);
    if (e != 0) return SGD_ERR_CUDA;
    if (!cal) {
        e = launch_quantize_global(kv->k, kv->v, kv->dtype, kv->Hkv, kv->D, kv->T, base, k_codes, v_codes, k_scale,
                                   v_scale, v_norm, hdr, dev->sms, s);
        if (e != 0) return SGD_ERR_CUDA;
    }
    if (blocks) {  // block scores, then the top blocks of each row (the plan's partition offsets = block offsets)
        float *bs = reinterpret_cast<float *>(ws + L.bscores);
        e = launch_block_max(a.scores, kv->cu_seqlens, pv.seq_part0, kv->B, kv->Hkv, kv->T, n_blocks, bs,
                             &hdr->status, s);
        if (e != 0) return SGD_ERR_CUDA;
        e = launch_topk(bs, pv.seq_part0, kv->B, kv->Hkv, n_blocks, keep_num, keep_den, idx, cu_kept, kept_total,
                        &hdr->status, s);
        return e == 0 ? SGD_OK : SGD_ERR_CUDA;
    }
    e = launch_topk(a.scores, kv->cu_seqlens, kv->B, kv->Hkv, kv->T, keep_num, keep_den, idx, cu_kept, kept_total,
                    &hdr->status, s);
    return e == 0 ? SGD_OK : SGD_ERR_CUDA;
}

int sgd_quantize_select(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv, float beta, float eps,
                        int keep_num, int keep_den, sgd_scheme scheme, int64_t n_parts, int8_t *k_codes,
                        int8_t *v_codes, float *k_scale, float *v_scale, float *v_norm, int32_t *idx,
                        int32_t *cu_kept, int64_t kept_total, void *workspace, size_t workspace_bytes,
                        void *stream) {
    return quantize_select_impl(q, q_dtype, G, 1, kv, beta, eps, keep_num, keep_den, scheme, n_parts, k_codes, v_codes,
                                k_scale, v_scale, v_norm, false, 0, idx, cu_kept, kept_total, workspace,
                                workspace_bytes, stream);
}

int sgd_quantize_select_multi(const void *q, sgd_dtype q_dtype, int G, int M, const sgd_kv *kv, float beta, float eps,
                              int keep_num, int keep_den, sgd_scheme scheme, int64_t n_parts, int8_t *k_codes,
                              int8_t *v_codes, float *k_scale, float *v_scale, float *v_norm, int32_t *idx,
                              int32_t *cu_kept, int64_t kept_total, void *workspace, size_t workspace_bytes,
                              void *stream) {
    return quantize_select_impl(q, q_dtype, G, M, kv, beta, eps, keep_num, keep_den, scheme, n_parts, k_codes, v_codes,
                                k_scale, v_scale, v_norm, false, 0, idx, cu_kept, kept_total, workspace,
                                workspace_bytes, stream);
}

int sgd_quantize_select_blocks(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv, float beta, float eps,
                               int keep_num, int keep_den, sgd_scheme scheme, int64_t n_parts, int8_t *k_codes,
                               int8_t *v_codes, float *k_scale, float *v_scale, float *v_norm, int64_t n_blocks,
                               int32_t *blk, int32_t *cu_kept_blocks, int64_t kept_blocks_total, void *workspace,
                               size_t workspace_bytes, void *stream) {
    return quantize_select_impl(q, q_dtype, G, 1, kv, beta, eps, keep_num, keep_den, scheme, n_parts, k_codes, v_codes,
                                k_scale, v_scale, v_norm, true, n_blocks, blk, cu_kept_blocks, kept_blocks_total,
                                workspace, workspace_bytes, stream);
}

int sgd_decode_attn(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv, const int32_t *idx,
                    const int32_t *cu_kept, int64_t kept_total, int schedule, int n_splits, int q_quant, float *out,
                    float *lse, void *workspace, size_t workspace_bytes, void *stream) {
    return sgd_decode_attn_multi(q, q_dtype, G, 1, kv, idx, cu_kept, kept_total, schedule, n_splits, q_quant, out,
                                 lse, workspace, workspace_bytes, stream);
}

int sgd_decode_attn_multi(const void *q, sgd_dtype q_dtype, int G, int M, const sgd_kv *kv, const int32_t *idx,
                          const int32_t *cu_kept, int64_t kept_total, int schedule, int n_splits, int q_quant,
                          float *out, float *lse, void *workspace, size_t workspace_bytes, void *stream) {
    return decode_impl(q, q_dtype, G, M, kv, idx, cu_kept, kept_total, false, schedule, n_splits, q_quant, out, lse,
                       workspace, workspace_bytes, stream);
}

int sgd_decode_attn_blocks(const void *q, sgd_dtype q_dtype, int G, const sgd_kv *kv, const int32_t *blk,
                           const int32_t *cu_kept_blocks, int64_t kept_blocks_total, int schedule, int n_splits,
                           int q_quant, float *out, float *lse, void *workspace, size_t workspace_bytes,
                           void *stream) {
    if (!blk || !cu_kept_blocks) return SGD_ERR_NULL;
    return decode_impl(q, q_dtype, G, 1, kv, blk, cu_kept_blocks, kept_blocks_total, true, schedule, n_splits,
                       q_quant, out, lse, workspace, workspace_bytes, stream);
}

int sgd_plan_segments(const int32_t *cu, int B, int Hkv, int n_req, int min_chunk, int mode, int row_cost,
                      int32_t *segs, int64_t max_segs, int32_t *n_segs, void *workspace, size_t workspace_bytes,
                      void *stream) {
    if (!cu || !segs || !n_segs || !workspace) return SGD_ERR_NULL;
    if (B < 1 || Hkv < 1 || (int64_t)B * Hkv >= (int64_t(1) << 24)) return SGD_ERR_SHAPE;
    if (mode != 0 && mode != 1) return SGD_ERR_ARG;
    if (mode == 1) n_req = B * Hkv;
    if (n_req < 1 || min_chunk < kGranule || min_chunk % kGranule != 0 || max_segs < 0) return SGD_ERR_ARG;
    if (row_cost < 0 || row_cost > (1 << 16) || row_cost % kGranule != 0) return SGD_ERR_ARG;
    if (!aligned16(workspace)) return SGD_ERR_ALIGN;
    const Layout L = layout(SGD_OP_DECODE, B, Hkv, 1, 64, 1, n_req);
    if (workspace_bytes < L.row_done) return SGD_ERR_WORKSPACE;  // the plan arrays only
    DevInfo *dev;
    int rc = current_device(&dev);
    if (rc != SGD_OK) return rc;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    PlanView pv = plan_view(ws, L);
    pv.row_done = nullptr;  // no decode follows
    cudaStream_t s = as_stream(stream);
    launch_plan(cu, cu, B, Hkv, n_req, min_chunk, mode, pv, hdr, s, kGranule, nullptr, nullptr, 0, 0, nullptr, 0, 1, 1,
                1, row_cost);
    launch_plan_dump(pv, cu, B, Hkv, n_req, segs, max_segs, n_segs, hdr, s);
    return cudaGetLastError() == cudaSuccess ? SGD_OK : SGD_ERR_CUDA;
}

int sgd_workspace_status(const void *workspace, int32_t *status, void *stream) {
    if (!workspace || !status) return SGD_ERR_NULL;
    cudaStream_t s = as_stream(stream);
    if (cudaMemcpyAsync(status, static_cast<const uint8_t *>(workspace) + SGD_WS_STATUS_OFFSET, sizeof(int32_t),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SGD_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? SGD_OK : SGD_ERR_CUDA;
}

}  // extern "C"
