"""fp64 CPU oracle for single-token GQA decode with OAM token dropping, an INT8 KV cache
and split-KV merging.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg are the only callers.  The product (``sparse_gqa_decode_b200``) never imports
this package, and this package never imports the product: the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64, no fast-math); this module marshals
arrays and writes out the per-row / per-partition loops of each method step in the order the
pages state them.  Sources are cited by page title and section:

  [TD] "优化稀疏注意力中的令牌丢弃机制" (Optimizing token dropping in sparse attention):
       section 3 (OAM), section 5 (split-KV and its merge), section 6 (INT8 schemes A and B).
  [AO] "注意力优化（Attention Optimization）": GQA example (query head h uses KV head h // G).
  [CD] "共同设计 AI 模型注意力，实现快速的交互式长上下文推理": decode section (speculative decoding
       verifies several query tokens per step).
  [NSA] "硬件对齐的稀疏注意力机制：原理、优化与实践": section 2.1 (64-token selection blocks).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

PART = 64  # scheme-A K partition length in tokens ([TD] section 6: "e.g. 64 or 128 tokens")

_dp = ctypes.POINTER(ctypes.c_double)
_fp = ctypes.POINTER(ctypes.c_float)
_i8p = ctypes.POINTER(ctypes.c_int8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with plain gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load(path: str):
    """Open an oracle shared library at ``path`` and declare its C signatures."""
    L = ctypes.CDLL(path)
    L.orc_attend.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, _dp, _dp, _dp, _dp, _dp]
    L.orc_merge.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp]
    L.orc_amax.argtypes = [_fp, ctypes.c_int64]
    L.orc_amax.restype = ctypes.c_float
    L.orc_scale_from_amax.argtypes = [ctypes.c_float]
    L.orc_scale_from_amax.restype = ctypes.c_float
    L.orc_code.argtypes = [ctypes.c_float, ctypes.c_float]
    L.orc_code.restype = ctypes.c_int8
    L.orc_quantize.argtypes = [_fp, ctypes.c_int64, ctypes.c_float, _i8p]
    L.orc_quantize_partitions.argtypes = [_fp, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _fp, _i8p]
    L.orc_oam_scores.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, _dp, _dp, _dp,
                                 ctypes.c_double, ctypes.c_double, _dp]
    L.orc_topk.argtypes = [ctypes.c_int64, _dp, ctypes.c_int64, _i32p]
    L.orc_plan.argtypes = [ctypes.c_int, _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_int, ctypes.c_int64, _i32p, _i32p, _i64p, _i64p, _i32p]
    L.orc_plan.restype = ctypes.c_int64
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor: widen exactly through float32/float64
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


# ----------------------------------------------------------------------------------------------
# attention and merge
# ----------------------------------------------------------------------------------------------
def attend(q, k, v):
    """Softmax attention of G query heads over n tokens ([TD] section 2).

    q [G, D], k [n, D], v [n, D] -> (out [G, D], lse [G]) in float64; lse is the natural-log
    normaliser of the scaled logits q.k/sqrt(D).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    G, D = q.shape
    n = k.shape[0]
    out = np.empty((G, D), np.float64)
    lse = np.empty(G, np.float64)
    rc = lib().orc_attend(D, G, n, _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(out, _dp), _ptr(lse, _dp))
    if rc != 0:
        raise ValueError(f"orc_attend failed ({rc})")
    return out, lse


def merge(o_c, lse_c):
    """Exact LSE merge of split-KV partials ([TD] section 5): o_c [C, G, D], lse_c [C, G]."""
    o_c, lse_c = _f64(o_c), _f64(lse_c)
    C, G, D = o_c.shape
    out = np.empty((G, D), np.float64)
    lse = np.empty(G, np.float64)
    rc = lib().orc_merge(C, G, D, _ptr(o_c, _dp), _ptr(lse_c, _dp), _ptr(out, _dp), _ptr(lse, _dp))
    if rc != 0:
        raise ValueError(f"orc_merge failed ({rc})")
    return out, lse


# ----------------------------------------------------------------------------------------------
# INT8 quantisation ([TD] section 6)
# ----------------------------------------------------------------------------------------------
def amax(x) -> np.float32:
    x = _f32(x).ravel()
    return np.float32(lib().orc_amax(_ptr(x, _fp), x.size))


def scale_from_amax(a) -> np.float32:
    return np.float32(lib().orc_scale_from_amax(float(np.float32(a))))


def quantize(x, scale) -> np.ndarray:
    x = _f32(x)
    out = np.empty(x.shape, np.int8)
    lib().orc_quantize(_ptr(x, _fp), x.size, float(np.float32(scale)), _ptr(out, _i8p))
    return out


def quantize_q(q, mode: str):
    """Query-side INT8 ([TD] section 6: schemes A and B also quantise Q per token partition).

    A decode query is one token per sequence, so its partition is that token: ``mode`` "token"
    gives every (sequence, query head) row of q [B, Hq, D] its own scale over D; "tensor" gives
    all of q one scale (the per-tensor baseline).  Scale and code rules as for K and V.
    Returns (codes int8 [B, Hq, D], scales float32 [B, Hq] or [1])."""
    x = _f32(q)
    if mode == "tensor":
        s = scale_from_amax(amax(x))
        return quantize(x, s), np.array([s], np.float32)
    if mode != "token":
        raise ValueError("mode is 'token' or 'tensor'")
    B, Hq, D = x.shape
    codes = np.empty((B, Hq, D), np.int8)
    scales = np.empty((B, Hq), np.float32)
    for b in range(B):
        for h in range(Hq):
            scales[b, h] = scale_from_amax(amax(x[b, h]))
            codes[b, h] = quantize(x[b, h], scales[b, h])
    return codes, scales


def dequant_q(codes, scales) -> np.ndarray:
    """code * scale of a quantised query (float64, exact), scales [B, Hq] or [1]."""
    s = np.asarray(scales, np.float64)
    if s.size == 1:
        return np.asarray(codes, np.float64) * s[0]
    return np.asarray(codes, np.float64) * s[..., None]


def n_parts(lengths: Sequence[int], part: int = PART) -> np.ndarray:
    return np.array([(int(L) + part - 1) // part for L in lengths], dtype=np.int64)


def quantize_kv(k, v, cu_seqlens, scheme: str, part: int = PART, k_scale=None, v_scale=None):
    """Quantise a packed cache k, v [Hkv, T, D] (torch or numpy, bf16/f32 values).

    Scheme A: K gets one scale per (KV head, sequence, ``part``-token partition), laid out as
    k_scale [Hkv, sum_b ceil(L_b / part)] with sequence b's partitions starting at
    sum_{b'<b} ceil(L_b' / part); V gets one scale over the whole tensor.
    Scheme B: K and V each get one scale over the whole tensor (k_scale has shape [1]).
    Calibrated scales ([TD] section 6 names per-tensor static quantisation and credits INT8's
    small error to calibrated scales): a given ``v_scale`` (and, scheme B, ``k_scale``) replaces
    that tensor's max|x| / 127; the codes follow the same rule, so values beyond the scale's
    range saturate at +-127.  Scheme A's K partition scales are computed as always.
    Returns (k_codes int8 [Hkv,T,D], v_codes, k_scale float32, v_scale float32 [1]).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.size - 1
    Hkv, T, D = k.shape
    lengths = np.diff(cu)
    kc = np.empty((Hkv, T, D), np.int8)
    vc = np.empty((Hkv, T, D), np.int8)
    L = lib()
    # V: one scale over every element of the tensor (both schemes)
    if v_scale is None:
        v_amax = np.float32(0)
        for h in range(Hkv):
            v_amax = max(v_amax, amax(v[h]))
        v_scale = scale_from_amax(v_amax)
    v_scale = np.float32(v_scale)
    for h in range(Hkv):
        vc[h] = quantize(v[h], v_scale)
    if scheme == "A":
        if k_scale is not None:
            raise ValueError("scheme A computes its K partition scales")
        parts = n_parts(lengths, part)
        cu_parts = np.concatenate([[0], np.cumsum(parts)])
        k_scale = np.empty((Hkv, int(cu_parts[-1])), np.float32)
        for h in range(Hkv):
            kh = _f32(k[h])
            for b in range(B):
                s, e = int(cu[b]), int(cu[b + 1])
                rows = np.ascontiguousarray(kh[s:e])
                sc = np.empty(int(parts[b]), np.float32)
                codes = np.empty(rows.shape, np.int8)
                L.orc_quantize_partitions(_ptr(rows, _fp), e - s, D, part, _ptr(sc, _fp), _ptr(codes, _i8p))
                k_scale[h, cu_parts[b]:cu_parts[b + 1]] = sc
                kc[h, s:e] = codes
    elif scheme == "B":
        if k_scale is None:
            k_amax = np.float32(0)
            for h in range(Hkv):
                k_amax = max(k_amax, amax(k[h]))
            ks = scale_from_amax(k_amax)
        else:
            ks = np.float32(k_scale)
        for h in range(Hkv):
            kc[h] = quantize(k[h], ks)
        k_scale = np.array([ks], np.float32)
    else:
        raise ValueError("scheme must be 'A' or 'B'")
    return kc, vc, k_scale, np.array([v_scale], np.float32)


def dequant_rows(codes, scale_per_token) -> np.ndarray:
    """code * scale in float64 (exact: a 7-bit integer times a float32 fits 53 bits)."""
    return np.asarray(codes, np.float64) * np.asarray(scale_per_token, np.float64).reshape(-1, 1)


def k_scale_of_tokens(k_scale, scheme: str, h: int, b: int, L: int, cu_parts, part: int = PART):
    """Per-token K scale of sequence b, KV head h (length L)."""
    if scheme == "B":
        return np.full(L, k_scale[0], np.float32)
    t = np.arange(L)
    return k_scale[h, cu_parts[b] + t // part]


# ----------------------------------------------------------------------------------------------
# OAM scores and top-K ([TD] section 3)
# ----------------------------------------------------------------------------------------------
def oam_scores(q, k, v, beta: float, eps: float) -> np.ndarray:
    """s_t = max_g (q_g . k_t) / sqrt(D) + beta * ln(||v_t|| + eps), q [G, D], k, v [n, D]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    G, D = q.shape
    n = k.shape[0]
    s = np.empty(n, np.float64)
    rc = lib().orc_oam_scores(D, G, n, _ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), float(beta), float(eps), _ptr(s, _dp))
    if rc != 0:
        raise ValueError("orc_oam_scores failed")
    return s


def topk(s, K: int) -> np.ndarray:
    """Indices of the K best tokens under (score desc, index asc), returned ascending."""
    s = _f64(s)
    out = np.empty(int(K), np.int32)
    rc = lib().orc_topk(s.size, _ptr(s, _dp), int(K), _ptr(out, _i32p))
    if rc != 0:
        raise ValueError("orc_topk failed")
    return out


def kept_count(L: int, keep_num: int, keep_den: int) -> int:
    """Tokens kept of a length-L sequence when keeping the top keep_num/keep_den of them:
    ceil(L * keep_num / keep_den), at least 1 and at most L (12.5% -> ceil(L / 8))."""
    K = -(-int(L) * int(keep_num) // int(keep_den))
    return max(1, min(int(L), K))


def oam_select(q, k, v, cu_seqlens, G: int, beta: float, eps: float, keep_num: int, keep_den: int,
               rows: Optional[Sequence] = None):
    """Per (sequence, KV head): score every token, keep the top K_b (ascending positions).

    q [B, Hq, D], k, v [Hkv, T, D] -> (idx int32 [Hkv, sum_b K_b], cu_kept int32 [B+1]);
    row (b, h) occupies idx[h, cu_kept[b]:cu_kept[b+1]] with positions local to sequence b.
    With ``rows`` = [(b, h), ...] only those rows are filled (others stay -1).
    Also returns the scores of the computed rows as a dict {(b, h): s}.
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.size - 1
    Hkv = k.shape[0]
    kept = np.array([kept_count(int(cu[b + 1] - cu[b]), keep_num, keep_den) for b in range(B)], np.int64)
    cu_kept = np.concatenate([[0], np.cumsum(kept)]).astype(np.int32)
    idx = np.full((Hkv, int(cu_kept[-1])), -1, np.int32)
    scores = {}
    todo = rows if rows is not None else [(b, h) for h in range(Hkv) for b in range(B)]
    for b, h in todo:
        s0, e0 = int(cu[b]), int(cu[b + 1])
        qg = q[b, h * G:(h + 1) * G]
        s = oam_scores(qg, k[h, s0:e0], v[h, s0:e0], beta, eps)
        scores[(b, h)] = s
        idx[h, cu_kept[b]:cu_kept[b + 1]] = topk(s, int(kept[b]))
    return idx, cu_kept, scores


def oam_select_multi(q, k, v, cu_seqlens, G: int, M: int, beta: float, eps: float, keep_num: int,
                     keep_den: int, rows: Optional[Sequence] = None):
    """oam_select for M query tokens per sequence (q [B, M, Hq, D]; the speculative step of
    "共同设计 AI 模型注意力..." decode section, scored as "优化稀疏注意力中的令牌丢弃机制" section 3):
    one kept set per (sequence, KV head) serves all M * G query rows, so the group maximum of
    the score runs over all of them: s_t = max_{m,g} (q[b, m, kvh*G+g] . k_t) / sqrt(D) + beta * ln(||v_t|| + eps).
    Same outputs as oam_select."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.size - 1
    Hkv = k.shape[0]
    D = q.shape[-1]
    kept = np.array([kept_count(int(cu[b + 1] - cu[b]), keep_num, keep_den) for b in range(B)], np.int64)
    cu_kept = np.concatenate([[0], np.cumsum(kept)]).astype(np.int32)
    idx = np.full((Hkv, int(cu_kept[-1])), -1, np.int32)
    scores = {}
    todo = rows if rows is not None else [(b, h) for h in range(Hkv) for b in range(B)]
    for b, h in todo:
        s0, e0 = int(cu[b]), int(cu[b + 1])
        qg = _f64(q[b, :, h * G:(h + 1) * G]).reshape(M * G, D)
        s = oam_scores(qg, k[h, s0:e0], v[h, s0:e0], beta, eps)
        scores[(b, h)] = s
        idx[h, cu_kept[b]:cu_kept[b + 1]] = topk(s, int(kept[b]))
    return idx, cu_kept, scores


def value_norms(v) -> np.ndarray:
    """||v_t||_2 of every row of v [..., T, D] in float64 (the norm the OAM score takes)."""
    x = _f64(v)
    return np.sqrt(np.sum(x * x, axis=-1))


def oam_select_int8(q, k_codes, k_scale, v, cu_seqlens, scheme: str, G: int, beta: float, eps: float,
                    keep_num: int, keep_den: int, rows: Optional[Sequence] = None, part: int = PART):
    """oam_select over a quantised cache ([TD] section 3 score on the section 6 codes, the
    section 7 pipeline with the selection moved after quantisation): k_t is replaced by its
    dequantised value code * scale; ||v_t|| is that of the values before quantisation.
    Same outputs as oam_select."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.size - 1
    Hkv = k_codes.shape[0]
    lengths = np.diff(cu)
    cu_parts = np.concatenate([[0], np.cumsum((lengths + part - 1) // part)])
    kept = np.array([kept_count(int(cu[b + 1] - cu[b]), keep_num, keep_den) for b in range(B)], np.int64)
    cu_kept = np.concatenate([[0], np.cumsum(kept)]).astype(np.int32)
    idx = np.full((Hkv, int(cu_kept[-1])), -1, np.int32)
    scores = {}
    kc = np.asarray(k_codes)
    ks = np.asarray(k_scale, np.float32)
    todo = rows if rows is not None else [(b, h) for h in range(Hkv) for b in range(B)]
    for b, h in todo:
        s0, e0 = int(cu[b]), int(cu[b + 1])
        L = e0 - s0
        khat = dequant_rows(kc[h, s0:e0], k_scale_of_tokens(ks, scheme, h, b, L, cu_parts, part))
        s = oam_scores(q[b, h * G:(h + 1) * G], khat, v[h, s0:e0], beta, eps)
        scores[(b, h)] = s
        idx[h, cu_kept[b]:cu_kept[b + 1]] = topk(s, int(kept[b]))
    return idx, cu_kept, scores


def block_scores(s, block: int = PART) -> np.ndarray:
    """Block-granular importance ([NSA] section 2.1 selected attention: 64-token blocks scored as a
    whole): S_j = max of the token scores of block j (tokens j*block .. j*block + block - 1, the
    last block of a row ragged)."""
    s = _f64(s)
    nb = -(-s.size // block)
    return np.array([s[j * block:(j + 1) * block].max() for j in range(nb)], np.float64)


def select_blocks(scores, cu_seqlens, Hkv: int, keep_num: int, keep_den: int, block: int = PART):
    """Keep, per (sequence, KV head), the top ceil(nb * keep_num / keep_den) blocks of that row's
    token scores under (block score desc, block index asc), ascending.  ``scores`` = {(b, h): s}
    as the oam_select functions return it (rows not in it stay -1).

    -> (blk int32 [Hkv, sum_b NB_b], cu_kept_blocks int32 [B+1], {(b, h): block scores})."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.size - 1
    nblk = [-(-int(cu[b + 1] - cu[b]) // block) for b in range(B)]
    kept = np.array([kept_count(nblk[b], keep_num, keep_den) for b in range(B)], np.int64)
    cu_kept = np.concatenate([[0], np.cumsum(kept)]).astype(np.int32)
    blk = np.full((Hkv, int(cu_kept[-1])), -1, np.int32)
    bs = {}
    for (b, h), srow in scores.items():
        bs[(b, h)] = block_scores(srow, block)
        blk[h, cu_kept[b]:cu_kept[b + 1]] = topk(bs[(b, h)], int(kept[b]))
    return blk, cu_kept, bs


def decode_blocks(q, k, v, cu_seqlens, G: int, blk, cu_kept_blocks, block: int = PART, quant=None, rows=None):
    """Decode attending, per (sequence, KV head), to every token of that row's kept blocks
    ("硬件对齐的稀疏注意力机制" (NSA) section 2.1: selected attention keeps the original tokens of
    the chosen 64-token blocks; the attention itself is "优化稀疏注意力中的令牌丢弃机制" section 2
    over that subset).  The last block of a sequence holds fewer than ``block`` tokens.
    -> out [B, Hq, D], lse [B, Hq]."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    ckb = np.asarray(cu_kept_blocks, dtype=np.int64)
    B = cu.size - 1
    Hkv = (k if quant is None else quant[0]).shape[0]
    D = q.shape[-1]
    out = np.full((B, Hkv * G, D), np.nan)
    lse = np.full((B, Hkv * G), np.nan)
    todo = rows if rows is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        L = int(cu[b + 1] - cu[b])
        toks = np.concatenate([np.arange(j * block, min((j + 1) * block, L))
                               for j in np.asarray(blk[h, ckb[b]:ckb[b + 1]], np.int64)]).astype(np.int32)
        # one row's kept tokens as a one-row index list for decode_row
        idx = np.zeros((Hkv, toks.size), np.int32)
        idx[h] = toks
        cu_k = np.zeros(B + 1, np.int64)
        cu_k[b + 1:] = toks.size
        o, l = decode_row(q, k, v, cu, G, b, h, idx, cu_k, quant)
        out[b, h * G:(h + 1) * G] = o
        lse[b, h * G:(h + 1) * G] = l
    return out, lse


# ----------------------------------------------------------------------------------------------
# decode over a packed cache
# ----------------------------------------------------------------------------------------------
def decode_row(q, k, v, cu_seqlens, G: int, b: int, h: int, idx=None, cu_kept=None, quant=None):
    """Attention output of sequence b, KV head h: (out [G, D], lse [G]) in float64.

    ``quant`` = (k_codes, v_codes, k_scale, v_scale, scheme): attend over the dequantised
    cache code * scale instead of k, v.  ``idx``/``cu_kept``: attend only over the kept
    tokens of the row.
    """
    _, kr, vr = _row_kv(k, v, cu_seqlens, b, h, idx, cu_kept, quant)
    return attend(q[b, h * G:(h + 1) * G], kr, vr)


def _row_kv(k, v, cu_seqlens, b: int, h: int, idx=None, cu_kept=None, quant=None):
    """The attended tokens of row (b, h): (positions in the sequence, keys [n, D], values [n, D])
    in float64, dequantised when ``quant`` is given, restricted to the kept tokens with ``idx``."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    s0, e0 = int(cu[b]), int(cu[b + 1])
    L = e0 - s0
    sel = np.arange(L) if idx is None else np.asarray(idx[h, int(cu_kept[b]):int(cu_kept[b + 1])], np.int64)
    if quant is None:
        return sel, _f64(k[h, s0:e0])[sel], _f64(v[h, s0:e0])[sel]
    kc, vc, k_scale, v_scale, scheme = quant
    lengths = np.diff(cu)
    cu_parts = np.concatenate([[0], np.cumsum(n_parts(lengths))])
    ks = k_scale_of_tokens(np.asarray(k_scale), scheme, h, b, L, cu_parts)
    kr = dequant_rows(np.asarray(kc[h, s0:e0])[sel], ks[sel])
    vr = dequant_rows(np.asarray(vc[h, s0:e0])[sel], np.full(sel.size, np.asarray(v_scale).ravel()[0]))
    return sel, kr, vr


def decode(q, k, v, cu_seqlens, G: int, idx=None, cu_kept=None, quant=None, rows=None):
    """decode_row over every (b, h) (or the listed ``rows``): out [B, Hq, D], lse [B, Hq]
    (rows not computed are NaN)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.size - 1
    Hkv = (k if quant is None else quant[0]).shape[0]
    D = q.shape[-1]
    out = np.full((B, Hkv * G, D), np.nan)
    lse = np.full((B, Hkv * G), np.nan)
    todo = rows if rows is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        o, l = decode_row(q, k, v, cu, G, b, h, idx, cu_kept, quant)
        out[b, h * G:(h + 1) * G] = o
        lse[b, h * G:(h + 1) * G] = l
    return out, lse


# ----------------------------------------------------------------------------------------------
# equal-work partition ([TD] section 5)
def decode_multi(q, k, v, cu_seqlens, G: int, M: int, idx=None, cu_kept=None, quant=None, rows=None):
    """Decode of M query tokens per sequence in one step (speculative verification, [CD] "decode":
    the draft tokens raise the GEMM M dimension from G to (1 + n_draft) * G).

    The M new tokens' keys and values are the last M entries of each sequence's cache, and query
    token m (0-based) attends causally: sequence positions p <= L_b - M + m (of the kept tokens,
    with ``idx``).  A query that sees no token gets out 0 and lse -inf.
    q [B, M, Hq, D] -> out [B, M, Hq, D], lse [B, M, Hq] in float64 (rows not computed: NaN).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.size - 1
    Hkv = (k if quant is None else quant[0]).shape[0]
    D = q.shape[-1]
    out = np.full((B, M, Hkv * G, D), np.nan)
    lse = np.full((B, M, Hkv * G), np.nan)
    todo = rows if rows is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        L = int(cu[b + 1] - cu[b])
        pos, kr, vr = _row_kv(k, v, cu, b, h, idx, cu_kept, quant)
        for m in range(M):
            vis = pos <= L - M + m
            heads = slice(h * G, (h + 1) * G)
            if not vis.any():
                out[b, m, heads] = 0.0
                lse[b, m, heads] = -np.inf
                continue
            out[b, m, heads], lse[b, m, heads] = attend(q[b, m, heads], kr[vis], vr[vis])
    return out, lse


# ----------------------------------------------------------------------------------------------
def plan(row_lengths, n_req: int, granule: int, min_chunk: int, mode: int, row_cost: int = 0):
    """Segments (cta, row, start, length) of the split-KV partition, and the CTA count.  Each row
    occupies its length rounded up to ``granule`` plus ``row_cost`` positions of the stream."""
    lens = np.ascontiguousarray(row_lengths, dtype=np.int64)
    R = lens.size
    cap = int(max(1, n_req) + R + 8) if mode == 0 else R
    cta = np.empty(cap, np.int32)
    row = np.empty(cap, np.int32)
    start = np.empty(cap, np.int64)
    length = np.empty(cap, np.int64)
    ncta = ctypes.c_int32(0)
    n = lib().orc_plan(R, _ptr(lens, _i64p), int(n_req), int(granule), int(min_chunk), int(mode), int(row_cost), cap,
                       _ptr(cta, _i32p), _ptr(row, _i32p), _ptr(start, _i64p), _ptr(length, _i64p),
                       ctypes.byref(ncta))
    if n < 0:
        raise ValueError("orc_plan failed")
    if n > cap:
        raise RuntimeError("segment capacity exceeded")
    return {"cta": cta[:n], "row": row[:n], "start": start[:n], "len": length[:n], "n_cta": int(ncta.value)}
