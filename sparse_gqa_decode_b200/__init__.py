"""Single-token GQA decode attention for B200 (sm_100a): output-aware token dropping (OAM),
an INT8 KV cache and split-KV flash-decoding with an exact log-sum-exp merge.

This module is a thin binding over the C ABI of ``libsgd.so`` (``include/sgd.h``): it turns
torch tensors into device pointers, allocates outputs and the workspace with torch, and
passes the current CUDA stream.  Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and importing fails loudly when the library
has not been built (``python sparse_gqa_decode_b200/build.py``).

A decode step, as the benchmark runs it::

    kc, vc, ks, vs, idx, cu_kept, ws = quantize_select(q, k, v, cu, G, beta, eps, 1, 8, "A", lengths)
    out, lse, ws = decode_attn(q, G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                               n_parts_=n_parts(lengths), idx=idx, cu_kept=cu_kept,
                               kept_total_=idx.shape[1])

Variants: ``oam_select`` on a bf16/f32 cache or on the INT8 cache with stored value norms;
``decode_attn(..., q_quant="token"|"tensor")`` for INT8 query codes; ``oam_select_multi`` /
``decode_attn_multi`` for several query tokens per sequence (speculative decoding);
``oam_select_blocks`` / ``decode_attn_blocks`` for whole 64-token blocks.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "lib", "quantize_kv", "oam_select", "oam_select_multi", "oam_select_blocks", "quantize_select",
    "quantize_select_multi", "quantize_select_blocks", "decode_attn",
    "decode_attn_multi", "decode_attn_blocks", "decode_attn_noalloc", "plan_segments", "workspace_status",
    "workspace_size", "decode_num_ctas", "kept_total", "kept_blocks_total", "n_parts", "kernel_timing_start",
    "kernel_timing_stop", "test_pipeline_timeout", "stream_read", "gather_read", "SGD_F32", "SGD_BF16", "SGD_I8", "SCHEME_A", "SCHEME_B",
    "SCHEME_A_CALIBRATED", "SCHEME_B_CALIBRATED", "STATUS_BITS", "ROW_COST",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsgd.so")

SGD_F32, SGD_BF16, SGD_I8 = 0, 1, 2
SCHEME_A, SCHEME_B, SCHEME_A_CALIBRATED, SCHEME_B_CALIBRATED = 0, 1, 2, 3
ROW_COST = 512  # SGD_ROW_COST: the automatic split's work charge per row, in tokens
OP_QUANTIZE, OP_OAM_SELECT, OP_DECODE, OP_QUANTIZE_SELECT = 0, 1, 2, 3
PARTITION = 64
STATUS_BITS = {0x1: "empty sequence", 0x2: "wait timeout", 0x4: "size mismatch", 0x8: "bad index",
               0x10: "bad calibrated scale"}

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python sparse_gqa_decode_b200/build.py` "
                      "(there is no fallback implementation)")


class SgdKv(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("B", ctypes.c_int32),
        ("Hkv", ctypes.c_int32),
        ("D", ctypes.c_int32),
        ("T", ctypes.c_int64),
        ("cu_seqlens", ctypes.c_void_p),
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("scheme", ctypes.c_int),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("n_parts", ctypes.c_int64),
        ("v_norm", ctypes.c_void_p),
    ]


_vp, _sz, _i64, _i32, _f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int, ctypes.c_float
_kvp = ctypes.POINTER(SgdKv)

lib = ctypes.CDLL(LIB_PATH)
lib.sgd_version.restype = ctypes.c_int
lib.sgd_error_string.argtypes = [ctypes.c_int]
lib.sgd_error_string.restype = ctypes.c_char_p
lib.sgd_workspace_size.argtypes = [_i32, _kvp, _i32, _i32, _i32]
lib.sgd_workspace_size.restype = _sz
lib.sgd_decode_num_ctas.argtypes = [_kvp, _i32, _vp, _i32, _i32]
lib.sgd_quantize_kv.argtypes = [_kvp, _i32, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.sgd_oam_select.argtypes = [_vp, _i32, _i32, _kvp, _f, _f, _i32, _i32, _vp, _vp, _i64, _vp, _sz, _vp]
lib.sgd_decode_attn.argtypes = [_vp, _i32, _i32, _kvp, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp]
lib.sgd_decode_attn_multi.argtypes = [_vp, _i32, _i32, _i32, _kvp, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp,
                                      _sz, _vp]
lib.sgd_oam_select_multi.argtypes = [_vp, _i32, _i32, _i32, _kvp, _f, _f, _i32, _i32, _vp, _vp, _i64, _vp, _sz, _vp]
lib.sgd_oam_select_blocks.argtypes = [_vp, _i32, _i32, _kvp, _f, _f, _i32, _i32, _i64, _vp, _vp, _i64, _vp, _sz,
                                      _vp]
lib.sgd_decode_attn_blocks.argtypes = [_vp, _i32, _i32, _kvp, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _sz,
                                       _vp]
lib.sgd_test_pipeline_timeout.argtypes = [_i64, _i32]
lib.sgd_stream_read.argtypes = [_vp, _sz, _i32, _vp, _vp, _vp]
lib.sgd_gather_read.argtypes = [_vp, _vp, ctypes.c_int64, _vp, ctypes.c_int64, _vp, _vp]
lib.sgd_kernel_timing_start.argtypes = [_i32]
lib.sgd_kernel_timing_stop.argtypes = [ctypes.POINTER(ctypes.c_float), _i32, ctypes.POINTER(ctypes.c_int32)]
lib.sgd_kernel_timing_name.argtypes = [_i32]
lib.sgd_kernel_timing_name.restype = ctypes.c_char_p
lib.sgd_plan_segments.argtypes = [_vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _sz, _vp]
lib.sgd_workspace_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_int32), _vp]
lib.sgd_quantize_select.argtypes = [_vp, _i32, _i32, _kvp, _f, _f, _i32, _i32, _i32, _i64, _vp, _vp, _vp, _vp,
                                    _vp, _vp, _vp, _i64, _vp, _sz, _vp]
lib.sgd_quantize_select_multi.argtypes = [_vp, _i32, _i32, _i32, _kvp, _f, _f, _i32, _i32, _i32, _i64, _vp, _vp, _vp,
                                          _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp]
lib.sgd_quantize_select_blocks.argtypes = [_vp, _i32, _i32, _kvp, _f, _f, _i32, _i32, _i32, _i64, _vp, _vp, _vp,
                                           _vp, _vp, _i64, _vp, _vp, _i64, _vp, _sz, _vp]
lib.sgd_decode_attn_noalloc.argtypes = [_vp, _i32, _i32, _kvp, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp,
                                        _vp]

_DT = {torch.float32: SGD_F32, torch.bfloat16: SGD_BF16, torch.int8: SGD_I8}
_QQ = {"none": 0, "token": 1, "tensor": 2}


class SgdError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        raise SgdError(f"{what}: {lib.sgd_error_string(rc).decode()} ({rc})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def n_parts(lengths: Sequence[int]) -> int:
    """Scheme-A K partitions over all sequences: sum_b ceil(L_b / 64) (a buffer size)."""
    return int(sum((int(L) + PARTITION - 1) // PARTITION for L in lengths))


def kept_total(lengths: Sequence[int], keep_num: int, keep_den: int) -> int:
    """Size of the kept-index buffer per KV head: sum_b clamp(ceil(L_b*num/den), 1, L_b)."""
    return int(sum(max(1, min(int(L), -(-int(L) * keep_num // keep_den))) for L in lengths))


def kept_blocks_total(lengths: Sequence[int], keep_num: int, keep_den: int) -> int:
    """Size of the kept-block buffer per KV head: sum_b clamp(ceil(nb_b*num/den), 1, nb_b) with
    nb_b = ceil(L_b / 64) blocks."""
    return kept_total([(int(L) + PARTITION - 1) // PARTITION for L in lengths], keep_num, keep_den)


def _kv(k, v, cu_seqlens, k_scale=None, v_scale=None, scheme=SCHEME_A, parts=0, v_norm=None) -> SgdKv:
    if k.dim() != 3 or k.shape != v.shape or k.dtype != v.dtype:
        raise ValueError("k and v must both be [Hkv, T, D] of one dtype")
    if k.dtype not in _DT:
        raise ValueError(f"unsupported cache dtype {k.dtype}")
    if not (k.is_contiguous() and v.is_contiguous() and cu_seqlens.is_contiguous()):
        raise ValueError("k, v and cu_seqlens must be contiguous")
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    Hkv, T, D = k.shape
    return SgdKv(_DT[k.dtype], cu_seqlens.numel() - 1, Hkv, D, T, cu_seqlens.data_ptr(), k.data_ptr(),
                 v.data_ptr(), scheme, None if k_scale is None else k_scale.data_ptr(),
                 None if v_scale is None else v_scale.data_ptr(), int(parts),
                 None if v_norm is None else v_norm.data_ptr())


def workspace_size(op: int, kv: SgdKv, G: int = 1, schedule: int = 0, n_splits: int = 0) -> int:
    n = lib.sgd_workspace_size(op, ctypes.byref(kv), G, schedule, n_splits)
    if n == 0:
        raise SgdError("sgd_workspace_size rejected the arguments")
    return int(n)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise SgdError("workspace too small")
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Device status bits recorded by the last call that used ``workspace`` (synchronises)."""
    st = ctypes.c_int32(0)
    _check(lib.sgd_workspace_status(_ptr(workspace), ctypes.byref(st), _stream(stream)), "sgd_workspace_status")
    return int(st.value)


def _quant_scheme(scheme: str, k_scale_in, v_scale_in) -> int:
    """The C scheme value: A / B, or their calibrated forms when per-tensor scales are given."""
    if scheme not in ("A", "B"):
        raise ValueError("scheme must be 'A' or 'B'")
    if v_scale_in is None:
        if k_scale_in is not None:
            raise ValueError("a calibrated K scale goes with a calibrated V scale")
        return SCHEME_A if scheme == "A" else SCHEME_B
    if scheme == "A" and k_scale_in is not None:
        raise ValueError("scheme A computes its K partition scales: no k_scale_in")
    if scheme == "B" and k_scale_in is None:
        raise ValueError("scheme B with calibrated scales takes k_scale_in too")
    return SCHEME_A_CALIBRATED if scheme == "A" else SCHEME_B_CALIBRATED


def _scale_buffers(k, sch: int, parts: int, k_scale_in, v_scale_in):
    """k_scale / v_scale of a quantisation: the calibrated inputs where given, else new outputs."""
    Hkv = k.shape[0]
    if sch in (SCHEME_A, SCHEME_A_CALIBRATED):
        ks = torch.empty((Hkv, parts), dtype=torch.float32, device=k.device)
    else:
        ks = k_scale_in if k_scale_in is not None else torch.empty(1, dtype=torch.float32, device=k.device)
    vs = v_scale_in if v_scale_in is not None else torch.empty(1, dtype=torch.float32, device=k.device)
    return ks, vs


def quantize_kv(k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor, scheme: str,
                lengths: Sequence[int], out=None, workspace=None, stream=None, v_norm=None,
                k_scale_in=None, v_scale_in=None):
    """INT8 codes and scales of a bf16/f32 cache.  Returns (k_codes, v_codes, k_scale, v_scale, ws).

    ``lengths`` are the host copies of the sequence lengths (buffer sizes only).  ``v_norm``: an
    optional float32 [Hkv, T] tensor that receives ||v_t|| (for oam_select over the INT8 cache).
    ``v_scale_in`` (and, scheme B, ``k_scale_in``): calibrated per-tensor scales, float32 [1] device
    tensors, used instead of max|x| / 127; they are returned as the scales.
    """
    sch = _quant_scheme(scheme, k_scale_in, v_scale_in)
    Hkv, T, D = k.shape
    parts = n_parts(lengths) if sch in (SCHEME_A, SCHEME_A_CALIBRATED) else 0
    kv = _kv(k, v, cu_seqlens)
    if out is None:
        kc = torch.empty((Hkv, T, D), dtype=torch.int8, device=k.device)
        vc = torch.empty_like(kc)
        ks, vs = _scale_buffers(k, sch, parts, k_scale_in, v_scale_in)
    else:
        kc, vc, ks, vs = out
    ws = _workspace(workspace_size(OP_QUANTIZE, kv), k.device, workspace)
    _check(lib.sgd_quantize_kv(ctypes.byref(kv), sch, parts, _ptr(kc), _ptr(vc), _ptr(ks), _ptr(vs), _ptr(v_norm),
                               _ptr(ws), ws.numel(), _stream(stream)), "sgd_quantize_kv")
    return kc, vc, ks, vs, ws


def oam_select(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor, G: int,
               beta: float, eps: float, keep_num: int, keep_den: int, lengths: Sequence[int],
               out=None, workspace=None, stream=None, k_scale=None, v_scale=None, scheme: str = "A",
               n_parts_: int = 0, v_norm=None):
    """Kept token positions per (sequence, KV head).  Returns (idx [Hkv, Kt], cu_kept [B+1], ws).

    k, v bf16/f32: the cache before quantisation.  k, v int8: the quantised cache, scored on
    k_code * k_scale with ||v|| from ``v_norm`` (as written by quantize_kv / quantize_select)."""
    Hkv = k.shape[0]
    Kt = kept_total(lengths, keep_num, keep_den)
    kv = _kv(k, v, cu_seqlens, k_scale, v_scale, SCHEME_A if scheme == "A" else SCHEME_B, n_parts_, v_norm)
    if out is None:
        idx = torch.empty((Hkv, Kt), dtype=torch.int32, device=k.device)
        cu_kept = torch.empty(cu_seqlens.numel(), dtype=torch.int32, device=k.device)
    else:
        idx, cu_kept = out
    ws = _workspace(workspace_size(OP_OAM_SELECT, kv, G), k.device, workspace)
    _check(lib.sgd_oam_select(_ptr(q), _DT[q.dtype], G, ctypes.byref(kv), beta, eps, keep_num, keep_den, _ptr(idx),
                              _ptr(cu_kept), Kt, _ptr(ws), ws.numel(), _stream(stream)), "sgd_oam_select")
    return idx, cu_kept, ws


def oam_select_multi(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor, G: int,
                     beta: float, eps: float, keep_num: int, keep_den: int, lengths: Sequence[int],
                     out=None, workspace=None, stream=None, k_scale=None, v_scale=None, scheme: str = "A",
                     n_parts_: int = 0, v_norm=None):
    """One kept set per (sequence, KV head) for the M query tokens of q [B, M, Hq, D] (the group
    maximum over all M * G query rows).  Returns (idx [Hkv, Kt], cu_kept [B+1], ws)."""
    Hkv, M = k.shape[0], q.shape[1]
    Kt = kept_total(lengths, keep_num, keep_den)
    kv = _kv(k, v, cu_seqlens, k_scale, v_scale, SCHEME_A if scheme == "A" else SCHEME_B, n_parts_, v_norm)
    if out is None:
        idx = torch.empty((Hkv, Kt), dtype=torch.int32, device=k.device)
        cu_kept = torch.empty(cu_seqlens.numel(), dtype=torch.int32, device=k.device)
    else:
        idx, cu_kept = out
    ws = _workspace(workspace_size(OP_OAM_SELECT, kv, G * M), k.device, workspace)
    _check(lib.sgd_oam_select_multi(_ptr(q), _DT[q.dtype], G, M, ctypes.byref(kv), beta, eps, keep_num, keep_den,
                                    _ptr(idx), _ptr(cu_kept), Kt, _ptr(ws), ws.numel(), _stream(stream)),
           "sgd_oam_select_multi")
    return idx, cu_kept, ws


def oam_select_blocks(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor, G: int,
                      beta: float, eps: float, keep_num: int, keep_den: int, lengths: Sequence[int],
                      out=None, workspace=None, stream=None, k_scale=None, v_scale=None, scheme: str = "A",
                      n_parts_: int = 0, v_norm=None):
    """Kept 64-token blocks per (sequence, KV head), ranked by their best token's OAM score.
    Returns (blk [Hkv, NBt], cu_kept_blocks [B+1], ws); the cache arguments as in oam_select."""
    Hkv = k.shape[0]
    NBt = kept_blocks_total(lengths, keep_num, keep_den)
    kv = _kv(k, v, cu_seqlens, k_scale, v_scale, SCHEME_A if scheme == "A" else SCHEME_B, n_parts_, v_norm)
    if out is None:
        blk = torch.empty((Hkv, NBt), dtype=torch.int32, device=k.device)
        cu_kb = torch.empty(cu_seqlens.numel(), dtype=torch.int32, device=k.device)
    else:
        blk, cu_kb = out
    ws = _workspace(workspace_size(OP_OAM_SELECT, kv, G), k.device, workspace)
    _check(lib.sgd_oam_select_blocks(_ptr(q), _DT[q.dtype], G, ctypes.byref(kv), beta, eps, keep_num, keep_den,
                                     n_parts(lengths), _ptr(blk), _ptr(cu_kb), NBt, _ptr(ws), ws.numel(),
                                     _stream(stream)), "sgd_oam_select_blocks")
    return blk, cu_kb, ws


def _quantize_select(q, k, v, cu_seqlens, G, M, beta, eps, keep_num, keep_den, scheme, lengths, out, workspace,
                     stream, v_norm, k_scale_in, v_scale_in, blocks):
    sch = _quant_scheme(scheme, k_scale_in, v_scale_in)
    Hkv, T, D = k.shape
    nb = n_parts(lengths)
    parts = nb if sch in (SCHEME_A, SCHEME_A_CALIBRATED) else 0
    Kt = kept_blocks_total(lengths, keep_num, keep_den) if blocks else kept_total(lengths, keep_num, keep_den)
    kv = _kv(k, v, cu_seqlens)
    if out is None:
        kc = torch.empty((Hkv, T, D), dtype=torch.int8, device=k.device)
        vc = torch.empty_like(kc)
        ks, vs = _scale_buffers(k, sch, parts, k_scale_in, v_scale_in)
        idx = torch.empty((Hkv, Kt), dtype=torch.int32, device=k.device)
        cu_kept = torch.empty(cu_seqlens.numel(), dtype=torch.int32, device=k.device)
    else:
        kc, vc, ks, vs, idx, cu_kept = out
    ws = _workspace(workspace_size(OP_QUANTIZE_SELECT, kv, G * M), k.device, workspace)
    common = (beta, eps, keep_num, keep_den, sch, parts, _ptr(kc), _ptr(vc), _ptr(ks), _ptr(vs), _ptr(v_norm))
    tail = (_ptr(idx), _ptr(cu_kept), Kt, _ptr(ws), ws.numel(), _stream(stream))
    if blocks:
        rc = lib.sgd_quantize_select_blocks(_ptr(q), _DT[q.dtype], G, ctypes.byref(kv), *common, nb, *tail)
        name = "sgd_quantize_select_blocks"
    elif M > 1:
        rc = lib.sgd_quantize_select_multi(_ptr(q), _DT[q.dtype], G, M, ctypes.byref(kv), *common, *tail)
        name = "sgd_quantize_select_multi"
    else:
        rc = lib.sgd_quantize_select(_ptr(q), _DT[q.dtype], G, ctypes.byref(kv), *common, *tail)
        name = "sgd_quantize_select"
    _check(rc, name)
    return kc, vc, ks, vs, idx, cu_kept, ws


def quantize_select(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor, G: int,
                    beta: float, eps: float, keep_num: int, keep_den: int, scheme: str, lengths: Sequence[int],
                    out=None, workspace=None, stream=None, v_norm=None, k_scale_in=None, v_scale_in=None):
    """quantize_kv and oam_select of one cache in one call (K and V read once for both).
    Returns (k_codes, v_codes, k_scale, v_scale, idx, cu_kept, ws); ``v_norm``, ``k_scale_in`` and
    ``v_scale_in`` as in quantize_kv (with calibrated scales one pass writes every code)."""
    return _quantize_select(q, k, v, cu_seqlens, G, 1, beta, eps, keep_num, keep_den, scheme, lengths, out,
                            workspace, stream, v_norm, k_scale_in, v_scale_in, False)


def quantize_select_multi(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor, G: int,
                          beta: float, eps: float, keep_num: int, keep_den: int, scheme: str, lengths: Sequence[int],
                          out=None, workspace=None, stream=None, v_norm=None, k_scale_in=None, v_scale_in=None):
    """quantize_select for the M query tokens of q [B, M, Hq, D]: one kept set per (sequence, KV
    head) from the group maximum over all M * G query rows, as oam_select_multi."""
    return _quantize_select(q, k, v, cu_seqlens, G, q.shape[1], beta, eps, keep_num, keep_den, scheme, lengths, out,
                            workspace, stream, v_norm, k_scale_in, v_scale_in, False)


def quantize_select_blocks(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor, G: int,
                           beta: float, eps: float, keep_num: int, keep_den: int, scheme: str, lengths: Sequence[int],
                           out=None, workspace=None, stream=None, v_norm=None, k_scale_in=None, v_scale_in=None):
    """quantize_select keeping whole 64-token blocks, as oam_select_blocks.  Returns (k_codes,
    v_codes, k_scale, v_scale, blk [Hkv, NBt], cu_kept_blocks [B+1], ws)."""
    return _quantize_select(q, k, v, cu_seqlens, G, 1, beta, eps, keep_num, keep_den, scheme, lengths, out,
                            workspace, stream, v_norm, k_scale_in, v_scale_in, True)


def decode_attn(q: torch.Tensor, G: int, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                k_scale=None, v_scale=None, scheme: str = "A", n_parts_: int = 0,
                idx=None, cu_kept=None, kept_total_: int = 0, schedule: int = 0, n_splits: int = 0,
                out=None, workspace=None, stream=None, q_quant: str = "none"):
    """Attention output and log-sum-exp per query head.  Returns (out [B,Hq,D] f32, lse [B,Hq] f32, ws).

    ``q_quant`` (INT8 cache, bf16 q, D = 128): "none", "token" (one query scale per (sequence,
    head) row) or "tensor" (one scale for all of q); q.k then runs on the INT8 codes."""
    sch = SCHEME_A if scheme == "A" else SCHEME_B
    kv = _kv(k, v, cu_seqlens, k_scale, v_scale, sch, n_parts_)
    B = cu_seqlens.numel() - 1
    Hq = k.shape[0] * G
    D = k.shape[2]
    if out is None:
        o = torch.empty((B, Hq, D), dtype=torch.float32, device=k.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=k.device)
    else:
        o, lse = out
    ws = _workspace(workspace_size(OP_DECODE, kv, G, schedule, n_splits), k.device, workspace)
    _check(lib.sgd_decode_attn(_ptr(q), _DT[q.dtype], G, ctypes.byref(kv), _ptr(idx), _ptr(cu_kept),
                               int(kept_total_), schedule, n_splits, _QQ[q_quant], _ptr(o), _ptr(lse), _ptr(ws),
                               ws.numel(),
                               _stream(stream)), "sgd_decode_attn")
    return o, lse, ws


def decode_attn_multi(q: torch.Tensor, G: int, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                      k_scale=None, v_scale=None, scheme: str = "A", n_parts_: int = 0,
                      idx=None, cu_kept=None, kept_total_: int = 0, schedule: int = 0, n_splits: int = 0,
                      out=None, workspace=None, stream=None, q_quant: str = "none"):
    """M query tokens per sequence, q [B, M, Hq, D]; token m attends causally to positions
    <= L_b - M + m.  Returns (out [B, M, Hq, D] f32, lse [B, M, Hq] f32, ws)."""
    sch = SCHEME_A if scheme == "A" else SCHEME_B
    kv = _kv(k, v, cu_seqlens, k_scale, v_scale, sch, n_parts_)
    B, M = q.shape[0], q.shape[1]
    Hq = k.shape[0] * G
    D = k.shape[2]
    if out is None:
        o = torch.empty((B, M, Hq, D), dtype=torch.float32, device=k.device)
        lse = torch.empty((B, M, Hq), dtype=torch.float32, device=k.device)
    else:
        o, lse = out
    ws = _workspace(workspace_size(OP_DECODE, kv, G * M, schedule, n_splits), k.device, workspace)
    _check(lib.sgd_decode_attn_multi(_ptr(q), _DT[q.dtype], G, M, ctypes.byref(kv), _ptr(idx), _ptr(cu_kept),
                                     int(kept_total_), schedule, n_splits, _QQ[q_quant], _ptr(o), _ptr(lse),
                                     _ptr(ws), ws.numel(), _stream(stream)), "sgd_decode_attn_multi")
    return o, lse, ws


def decode_attn_blocks(q: torch.Tensor, G: int, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                       blk: torch.Tensor, cu_kept_blocks: torch.Tensor, k_scale=None, v_scale=None,
                       scheme: str = "A", n_parts_: int = 0, schedule: int = 0, n_splits: int = 0, out=None,
                       workspace=None, stream=None, q_quant: str = "none"):
    """Decode over kept 64-token blocks (as oam_select_blocks returns them).
    Returns (out [B, Hq, D] f32, lse [B, Hq] f32, ws)."""
    sch = SCHEME_A if scheme == "A" else SCHEME_B
    kv = _kv(k, v, cu_seqlens, k_scale, v_scale, sch, n_parts_)
    B = cu_seqlens.numel() - 1
    Hq = k.shape[0] * G
    D = k.shape[2]
    if out is None:
        o = torch.empty((B, Hq, D), dtype=torch.float32, device=k.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=k.device)
    else:
        o, lse = out
    ws = _workspace(workspace_size(OP_DECODE, kv, G, schedule, n_splits), k.device, workspace)
    _check(lib.sgd_decode_attn_blocks(_ptr(q), _DT[q.dtype], G, ctypes.byref(kv), _ptr(blk), _ptr(cu_kept_blocks),
                                      int(blk.shape[1]), schedule, n_splits, _QQ[q_quant], _ptr(o), _ptr(lse),
                                      _ptr(ws), ws.numel(), _stream(stream)), "sgd_decode_attn_blocks")
    return o, lse, ws


def decode_attn_noalloc(q: torch.Tensor, G: int, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                        k_scale=None, v_scale=None, scheme: str = "A", n_parts_: int = 0,
                        idx=None, cu_kept=None, kept_total_: int = 0, schedule: int = 0, n_splits: int = 0,
                        out=None, status=None, stream=None, q_quant: str = "none"):
    """decode_attn without a workspace: the library's built-in device scratch array is used
    (for callers that cannot allocate).  ``out`` = (out, lse) and ``status`` ([1] int32) are
    optional preallocated device outputs.  Returns (out, lse)."""
    sch = SCHEME_A if scheme == "A" else SCHEME_B
    kv = _kv(k, v, cu_seqlens, k_scale, v_scale, sch, n_parts_)
    B = cu_seqlens.numel() - 1
    if out is None:
        o = torch.empty((B, k.shape[0] * G, k.shape[2]), dtype=torch.float32, device=k.device)
        lse = torch.empty((B, k.shape[0] * G), dtype=torch.float32, device=k.device)
    else:
        o, lse = out
    _check(lib.sgd_decode_attn_noalloc(_ptr(q), _DT[q.dtype], G, ctypes.byref(kv), _ptr(idx), _ptr(cu_kept),
                                       int(kept_total_), schedule, n_splits, _QQ[q_quant], _ptr(o), _ptr(lse),
                                       _ptr(status),
                                       _stream(stream)), "sgd_decode_attn_noalloc")
    return o, lse


def stream_read(buf: torch.Tensor, method: int = 0, sink=None, status=None, stream=None):
    """Measurement aid: read every byte of ``buf`` once (method 0: 16-byte loads, 1: bulk copies
    into shared memory), XOR-folded into ``sink`` ([1] int64).  Returns (sink, status)."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int64, device=buf.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=buf.device)
    nbytes = buf.numel() * buf.element_size() // 16 * 16
    _check(lib.sgd_stream_read(_ptr(buf), nbytes, int(method), _ptr(sink), _ptr(status), _stream(stream)),
           "sgd_stream_read")
    return sink, status


def gather_read(a: torch.Tensor, rows: torch.Tensor, row_bytes: int, b=None, sink=None, stream=None,
                check: bool = True):
    """Measurement aid: read rows ``rows`` (int32 row numbers) of ``row_bytes`` bytes from ``a``
    (and ``b``) once, XOR-folded into ``sink`` ([1] int64).  ``check`` first verifies on the host
    that every row lies inside the tensors (a synchronising reduction: leave it to an untimed
    first call).  Returns sink."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int64, device=a.device)
    if check and rows.numel():
        lo, hi = int(rows.min()), int(rows.max())
        for t in (a, b):
            if t is not None and (lo < 0 or (hi + 1) * row_bytes > t.numel() * t.element_size()):
                raise ValueError("a row lies outside the tensor")
    _check(lib.sgd_gather_read(_ptr(a), _ptr(b), int(row_bytes), _ptr(rows), rows.numel(), _ptr(sink),
                               _stream(stream)), "sgd_gather_read")
    return sink


def test_pipeline_timeout(polls: int, idle_producer: bool) -> None:
    """Test aid: lower the bounded pipeline-wait limit to ``polls`` polls (0 = the built-in limit)
    and, with ``idle_producer``, keep the kernels' producer warps from issuing copies, so that the
    waits run out and report SGD_STATUS_WAIT_TIMEOUT.  Affects calls made afterwards."""
    _check(lib.sgd_test_pipeline_timeout(int(polls), 1 if idle_producer else 0), "sgd_test_pipeline_timeout")


def kernel_timing_start(max_launches: int = 256) -> None:
    """Bracket each kernel the library launches from now on with a CUDA event pair (a
    measurement aid; see kernel_timing_stop)."""
    _check(lib.sgd_kernel_timing_start(int(max_launches)), "sgd_kernel_timing_start")


def kernel_timing_stop(max_launches: int = 4096):
    """Stop bracketing; returns [(mangled kernel name, milliseconds), ...] in launch order."""
    ms = (ctypes.c_float * max_launches)()
    n = ctypes.c_int32(0)
    _check(lib.sgd_kernel_timing_stop(ms, max_launches, ctypes.byref(n)), "sgd_kernel_timing_stop")
    return [(lib.sgd_kernel_timing_name(k).decode(), float(ms[k])) for k in range(min(n.value, max_launches))]


def decode_num_ctas(k, v, cu_seqlens, G: int, indexed: bool = False, schedule: int = 0, n_splits: int = 0) -> int:
    kv = _kv(k, v, cu_seqlens)
    n = lib.sgd_decode_num_ctas(ctypes.byref(kv), G, ctypes.c_void_p(1) if indexed else None, schedule, n_splits)
    _check(min(n, 0), "sgd_decode_num_ctas")
    return int(n)


def plan_segments(cu: torch.Tensor, B: int, Hkv: int, n_req: int, min_chunk: int, mode: int, row_cost: int = 0,
                  stream=None):
    """The split-KV partition: int32 [n_segs, 4] rows (cta, row, start, length), and the CTA count.
    ``row_cost``: positions charged to each row beside its tokens (the decode's automatic split
    uses ROW_COST)."""
    R = B * Hkv
    cap = n_req + R + 8
    segs = torch.full((cap, 4), -1, dtype=torch.int32, device=cu.device)
    nseg = torch.zeros(2, dtype=torch.int32, device=cu.device)
    n = R if mode == 1 else n_req
    nbytes = 2048 + 4 * (B + 2 * R + 3 * n + 6) + 32 * R  # the bound sgd.h states
    ws = torch.empty(nbytes, dtype=torch.uint8, device=cu.device)
    _check(lib.sgd_plan_segments(_ptr(cu), B, Hkv, n_req, min_chunk, mode, int(row_cost), _ptr(segs), cap, _ptr(nseg),
                                 _ptr(ws), ws.numel(), _stream(stream)), "sgd_plan_segments")
    n, ncta = (int(x) for x in nseg.tolist())
    return segs[:n].cpu(), ncta
