"""The C ABI without a GPU: the library loads, exports every function include/sgd.h declares,
and rejects invalid arguments on the host before anything touches a device."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sgd.h")


@pytest.fixture(scope="module")
def sgd():
    from conftest import build_library
    m = build_library()
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sgd_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sgd_oam_select", "sgd_quantize_kv", "sgd_decode_attn", "sgd_workspace_size",
                     "sgd_error_string", "sgd_plan_segments", "sgd_workspace_status", "sgd_decode_attn_multi"):
        assert required in names


def test_library_exports_every_declared_symbol(sgd):
    for name in declared_functions():
        assert hasattr(sgd.lib, name), f"{name} not exported"


def test_error_strings_and_version(sgd):
    assert sgd.lib.sgd_version() == (1 << 16)
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        assert sgd.lib.sgd_error_string(code)
    assert sgd.lib.sgd_error_string(-99) == b"unknown status"


def test_struct_layout_matches_header(sgd):
    # dtype, B, Hkv, D (4 x 4 bytes), T (8), 3 pointers, scheme (+pad), 2 pointers, n_parts, v_norm
    assert ctypes.sizeof(sgd.SgdKv) == 4 * 4 + 8 + 3 * 8 + 8 + 2 * 8 + 8 + 8
    assert sgd.SgdKv.T.offset == 16 and sgd.SgdKv.k_scale.offset == 56 and sgd.SgdKv.n_parts.offset == 72
    assert sgd.SgdKv.v_norm.offset == 80


def _kv(sgd, **kw):
    base = dict(dtype=sgd.SGD_BF16, B=2, Hkv=2, D=128, T=100, cu_seqlens=0x1000, k=0x10000, v=0x20000,
                scheme=0, k_scale=None, v_scale=None, n_parts=0, v_norm=None)
    base.update(kw)
    return sgd.SgdKv(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), -1), (dict(cu_seqlens=None), -1), (dict(B=0), -2), (dict(D=96), -2),
    (dict(T=2**31), -2), (dict(dtype=7), -3), (dict(k=0x10008), -4),
])
def test_decode_rejects_bad_cache_on_host(sgd, kw, code):
    kv = _kv(sgd, **kw)
    rc = sgd.lib.sgd_decode_attn(ctypes.c_void_p(0x3000), sgd.SGD_BF16, 8, ctypes.byref(kv), None, None, 0, 0, 0, 0,
                                 ctypes.c_void_p(0x4000), ctypes.c_void_p(0x5000), ctypes.c_void_p(0x6000), 1 << 20,
                                 None)
    assert rc == code


def test_decode_rejects_bad_args_on_host(sgd):
    kv = _kv(sgd)
    L = sgd.lib

    def call(q=0x3000, qdt=sgd.SGD_BF16, G=8, idx=None, cu_kept=None, kt=0, out=0x4000, lse=0x5000, ws=0x6000,
             qq=0, cache=kv):
        return L.sgd_decode_attn(ctypes.c_void_p(q) if q else None, qdt, G, ctypes.byref(cache),
                                 ctypes.c_void_p(idx) if idx else None, ctypes.c_void_p(cu_kept) if cu_kept else None,
                                 kt, 0, 0, qq, ctypes.c_void_p(out) if out else None,
                                 ctypes.c_void_p(lse) if lse else None, ctypes.c_void_p(ws) if ws else None,
                                 1 << 20, None)

    assert call(q=0) == -1
    assert call(out=0) == -1
    assert call(G=0) == -2 and call(G=17) == -2
    assert call(qdt=sgd.SGD_F32) == -3  # an f32 query needs an f32 cache
    assert call(idx=0x7000) == -1  # idx without cu_kept
    assert call(idx=0x7000, cu_kept=0x8000, kt=1) == -2  # fewer kept tokens than sequences
    assert call(q=0x3004) == -4
    kv8 = _kv(sgd, dtype=sgd.SGD_I8)
    assert L.sgd_decode_attn(ctypes.c_void_p(0x3000), sgd.SGD_BF16, 8, ctypes.byref(kv8), None, None, 0, 0, 0, 0,
                             ctypes.c_void_p(0x4000), ctypes.c_void_p(0x5000), ctypes.c_void_p(0x6000), 1 << 20,
                             None) == -1  # int8 cache without scales
    # query codes: an INT8 cache with D = 128 and a bf16 query only; modes 0..2
    kv8s = _kv(sgd, dtype=sgd.SGD_I8, k_scale=0x30000, v_scale=0x40000, scheme=1)
    assert call(qq=3, cache=kv8s) == -8 and call(qq=-1, cache=kv8s) == -8
    assert call(qq=1) == -3  # bf16 cache
    assert call(qq=2, cache=_kv(sgd, dtype=sgd.SGD_I8, k_scale=0x30000, v_scale=0x40000, scheme=1, D=64)) == -2


def test_multi_token_decode_rejects_bad_args_on_host(sgd):
    L = sgd.lib
    p = ctypes.c_void_p

    def call(G=8, M=2, cache=None, qdt=sgd.SGD_BF16):
        kv = cache or _kv(sgd)
        return L.sgd_decode_attn_multi(p(0x3000), qdt, G, M, ctypes.byref(kv), None, None, 0, 0, 0, 0, p(0x4000),
                                       p(0x5000), p(0x6000), 1 << 20, None)

    assert call(M=0) == -2 and call(M=9) == -2 and call(G=16, M=5) == -2  # G * M <= 64
    assert call(cache=_kv(sgd, dtype=sgd.SGD_F32), qdt=sgd.SGD_F32) == -3  # tensor-core path only
    assert call(cache=_kv(sgd, dtype=sgd.SGD_I8, k_scale=0x30000, v_scale=0x40000, scheme=1, D=64)) == -3


def test_quantize_and_select_reject_bad_args_on_host(sgd):
    L = sgd.lib
    kv = _kv(sgd)
    p = ctypes.c_void_p
    assert L.sgd_quantize_kv(ctypes.byref(kv), 0, 3, None, p(0x1000), p(0x2000), p(0x3000), None, p(0x4000), 4096,
                             None) == -1
    assert L.sgd_quantize_kv(ctypes.byref(_kv(sgd, dtype=sgd.SGD_I8)), 0, 3, p(0x1000), p(0x1000), p(0x2000),
                             p(0x3000), None, p(0x4000), 4096, None) == -3
    assert L.sgd_quantize_kv(ctypes.byref(kv), 5, 3, p(0x1000), p(0x1000), p(0x2000), p(0x3000), None, p(0x4000), 4096,
                             None) == -3
    assert L.sgd_quantize_kv(ctypes.byref(kv), 0, 1, p(0x1000), p(0x1000), p(0x2000), p(0x3000), None, p(0x4000), 4096,
                             None) == -2  # fewer partitions than sequences
    assert L.sgd_quantize_kv(ctypes.byref(kv), 0, 3, p(0x1000), p(0x1000), p(0x2000), p(0x3000), None, p(0x4000), 16,
                             None) == -5  # workspace too small
    # the calibrated schemes: A_CALIBRATED checks the partitions like A, B_CALIBRATED takes none;
    # both pass the host checks (no device here: the call then fails on the device query)
    quant = lambda sch, parts: L.sgd_quantize_kv(ctypes.byref(kv), sch, parts, p(0x1000), p(0x1000), p(0x2000),
                                                 p(0x3000), None, p(0x4000), 4096, None)
    assert sgd.SCHEME_A_CALIBRATED == 2 and sgd.SCHEME_B_CALIBRATED == 3
    assert quant(2, 1) == -2 and quant(4, 3) == -3 and quant(-1, 3) == -3
    assert quant(2, 3) not in (-1, -2, -3, -4, -5, -8) and quant(3, 0) not in (-1, -2, -3, -4, -5, -8)
    sel = lambda **kw: L.sgd_oam_select(p(0x3000), kw.get("qdt", sgd.SGD_BF16), kw.get("G", 8), ctypes.byref(kv),
                                        kw.get("beta", 1.0), 1e-6, kw.get("num", 1), kw.get("den", 8), p(0x1000),
                                        p(0x2000), kw.get("kt", 20), p(0x4000), 1 << 20, None)
    assert sel(num=9, den=8) == -8
    assert sel(den=0) == -8
    assert sel(kt=1) == -2
    assert sel(beta=float("nan")) == -8
    assert sel(G=20) == -2
    # scoring an INT8 cache needs its K scales and the value norms, a bf16 query and D = 128
    kv8 = _kv(sgd, dtype=sgd.SGD_I8, k_scale=0x7000, v_scale=0x7100, n_parts=3)
    sel8 = lambda k8, qdt=sgd.SGD_BF16: L.sgd_oam_select(p(0x3000), qdt, 8, ctypes.byref(k8), 1.0, 1e-6, 1, 8,
                                                         p(0x1000), p(0x2000), 20, p(0x4000), 1 << 20, None)
    assert sel8(kv8) == -1  # no v_norm
    assert sel8(_kv(sgd, dtype=sgd.SGD_I8, v_norm=0x7200, n_parts=3)) == -1  # no k_scale
    assert sel8(_kv(sgd, dtype=sgd.SGD_I8, k_scale=0x7000, v_norm=0x7200, n_parts=3, D=64)) == -3
    assert sel8(_kv(sgd, dtype=sgd.SGD_I8, k_scale=0x7000, v_norm=0x7200, n_parts=3), sgd.SGD_F32) == -3
    assert sel8(_kv(sgd, dtype=sgd.SGD_I8, k_scale=0x7000, v_norm=0x7202, n_parts=3)) == -4


def test_block_entry_points_reject_bad_args_on_host(sgd):
    L = sgd.lib
    p = ctypes.c_void_p
    kv = _kv(sgd)  # B = 2, T = 100: at most 100 / 64 + 2 = 3 blocks

    def sel(n_blocks=3, kept=2, blk=0x7000):
        return L.sgd_oam_select_blocks(p(0x3000), sgd.SGD_BF16, 8, ctypes.byref(kv), 1.0, 1e-6, 1, 8, n_blocks,
                                       p(blk) if blk else None, p(0x8000), kept, p(0x6000), 1 << 20, None)

    assert sel(n_blocks=1) == -2 and sel(n_blocks=4) == -2  # between B and T / 64 + B
    assert sel(kept=4) == -2 and sel(kept=1) == -2  # kept blocks between B and n_blocks
    assert sel(blk=0) == -1

    def dec(blk=0x7000, cache=kv, kept=2):
        return L.sgd_decode_attn_blocks(p(0x3000), sgd.SGD_BF16, 8, ctypes.byref(cache), p(blk) if blk else None,
                                        p(0x8000), kept, 0, 0, 0, p(0x4000), p(0x5000), p(0x6000), 1 << 20, None)

    assert dec(blk=0) == -1
    assert dec(kept=4) == -2
    assert dec(cache=_kv(sgd, dtype=sgd.SGD_F32)) == -3  # tensor-core path only


def test_kernel_timing_rejects_bad_args_and_needs_a_device(sgd):
    L = sgd.lib
    assert L.sgd_kernel_timing_start(0) == -8 and L.sgd_kernel_timing_start(5000) == -8
    assert L.sgd_kernel_timing_stop(None, 0, None) == -1
    assert L.sgd_kernel_timing_name(0) is None
    if not torch.cuda.is_available():  # no device here: creating the events fails, nothing is left on
        assert L.sgd_kernel_timing_start(4) == L.sgd_kernel_timing_start(4) != 0


def test_multi_token_selection_and_plan_reject_bad_args_on_host(sgd):
    L = sgd.lib
    p = ctypes.c_void_p
    kv = _kv(sgd)

    def sel(G=8, M=2, cache=kv, qdt=sgd.SGD_BF16):
        return L.sgd_oam_select_multi(p(0x3000), qdt, G, M, ctypes.byref(cache), 1.0, 1e-6, 1, 8, p(0x1000),
                                      p(0x2000), 20, p(0x4000), 1 << 20, None)

    assert sel(M=0) == -2 and sel(M=3) == -2 and sel(G=16, M=2) == -2  # G * M <= 16 for the selection
    assert sel(cache=_kv(sgd, dtype=sgd.SGD_F32), qdt=sgd.SGD_F32) == -3  # tensor-core score kernel only

    def plan(cu=0x1000, B=2, Hkv=2, n_req=8, min_chunk=16, mode=0, ws=0x6000, nbytes=1 << 20, row_cost=0):
        n = ctypes.c_int32(0)
        return L.sgd_plan_segments(p(cu) if cu else None, B, Hkv, n_req, min_chunk, mode, row_cost, p(0x7000), 64,
                                   ctypes.byref(n), p(ws) if ws else None, nbytes, None)

    assert plan(cu=0) == -1 and plan(ws=0) == -1
    assert plan(B=0) == -2 and plan(mode=2) == -8
    assert plan(min_chunk=8) == -8 and plan(min_chunk=24) == -8 and plan(n_req=0) == -8
    assert plan(row_cost=-16) == -8 and plan(row_cost=24) == -8 and plan(row_cost=1 << 17) == -8
    assert plan(row_cost=sgd.ROW_COST) not in (-1, -2, -4, -5, -8)
    assert plan(ws=0x6004) == -4 and plan(nbytes=64) == -5
    # the workspace bound include/sgd.h states passes the size check for any shape (no device here,
    # so the call then fails on the device query); a few hundred bytes less does not
    for B, Hkv, n_req, mode in ((1, 1, 1, 0), (2, 2, 8, 0), (37, 8, 296, 0), (5000, 3, 148, 0), (9, 8, 0, 1)):
        n = B * Hkv if mode == 1 else n_req
        bound = 2048 + 4 * (B + 2 * B * Hkv + 3 * n + 6) + 32 * B * Hkv
        assert plan(B=B, Hkv=Hkv, n_req=max(n_req, 1), mode=mode, nbytes=bound) != -5
        assert plan(B=B, Hkv=Hkv, n_req=max(n_req, 1), mode=mode, nbytes=bound - 2048) == -5


def test_workspace_size_limits(sgd):
    kv = _kv(sgd)
    L = sgd.lib
    assert L.sgd_workspace_size(sgd.OP_QUANTIZE, ctypes.byref(kv), 1, 0, 0) >= 256  # no device needed
    assert L.sgd_workspace_size(sgd.OP_DECODE, ctypes.byref(kv), 65, 0, 0) == 0  # decode columns <= 64
    assert L.sgd_workspace_size(sgd.OP_OAM_SELECT, ctypes.byref(kv), 17, 0, 0) == 0  # selection G <= 16
    assert L.sgd_workspace_size(sgd.OP_DECODE, ctypes.byref(kv), 0, 0, 0) == 0


def test_pipeline_timeout_hook_is_host_state_only(sgd):
    # the test aid of the bounded waits: a negative limit is rejected, 0 restores the built-in one
    assert sgd.lib.sgd_test_pipeline_timeout(-1, 0) == -8
    assert sgd.lib.sgd_test_pipeline_timeout(4096, 1) == 0
    assert sgd.lib.sgd_test_pipeline_timeout(0, 0) == 0


def test_binding_picks_the_calibrated_scheme(sgd):
    qs = sgd._quant_scheme
    one = object()  # stands for a device scale tensor (only its presence matters here)
    assert qs("A", None, None) == sgd.SCHEME_A and qs("B", None, None) == sgd.SCHEME_B
    assert qs("A", None, one) == sgd.SCHEME_A_CALIBRATED and qs("B", one, one) == sgd.SCHEME_B_CALIBRATED
    for bad in (("A", one, one), ("B", None, one), ("A", one, None), ("C", None, None)):
        with pytest.raises(ValueError):
            qs(*bad)


def test_gather_read_rejects_bad_args_on_host(sgd):
    L = sgd.lib
    p = ctypes.c_void_p
    g = lambda a=0x1000, b=0x2000, rb=128, rows=0x3000, n=10, sink=0x4000: L.sgd_gather_read(
        p(a) if a else None, p(b) if b else None, rb, p(rows) if rows else None, n, p(sink) if sink else None, None)
    assert g(a=0) == -1 and g(rows=0) == -1 and g(sink=0) == -1
    assert g(rb=0) == -2 and g(rb=24) == -2 and g(rb=48) == -2 and g(rb=8192) == -2 and g(n=0) == -2
    assert g(a=0x1008) == -4 and g(b=0x2008) == -4 and g(rows=0x3002) == -4 and g(sink=0x4004) == -4
    assert g(b=0) not in (-1, -2, -4)  # b is optional; no device here, so the call fails later


def test_quantize_select_multi_and_blocks_reject_bad_args_on_host(sgd):
    L = sgd.lib
    p = ctypes.c_void_p
    kv = _kv(sgd)
    outs = (p(0x1000), p(0x1000), p(0x2000), p(0x3000), None)

    def multi(G=8, M=2, kt=20):
        return L.sgd_quantize_select_multi(p(0x3000), sgd.SGD_BF16, G, M, ctypes.byref(kv), 1.0, 1e-6, 1, 8, 0, 3,
                                           *outs, p(0x5000), p(0x6000), kt, p(0x4000), 1 << 20, None)

    def blocks(nb=3, kt=3):
        return L.sgd_quantize_select_blocks(p(0x3000), sgd.SGD_BF16, 8, ctypes.byref(kv), 1.0, 1e-6, 1, 4, 0, 3,
                                            *outs, nb, p(0x5000), p(0x6000), kt, p(0x4000), 1 << 20, None)

    assert multi(M=0) == -2 and multi(G=8, M=3) == -2 and multi(G=16, M=2) == -2
    assert multi(G=4, M=4) not in (-1, -2, -3, -4, -8)  # 16 columns pass the host checks
    assert blocks(nb=1) == -2  # fewer blocks than sequences
    assert blocks(kt=4) == -2  # more kept blocks than blocks
    assert blocks() not in (-1, -2, -3, -4, -8)


def test_binding_constants_match_the_header(sgd):
    text = open(HEADER).read()

    def define(name):
        m = re.search(r"#define\s+" + name + r"\s+\(?(\w+)", text)
        return int(m.group(1).rstrip("u"), 0)

    assert define("SGD_ROW_COST") == sgd.ROW_COST
    assert define("SGD_PARTITION") == 64
    for bit, name in ((0x1, "SGD_STATUS_EMPTY_SEQUENCE"), (0x2, "SGD_STATUS_WAIT_TIMEOUT"),
                      (0x4, "SGD_STATUS_SIZE_MISMATCH"), (0x8, "SGD_STATUS_BAD_INDEX"), (0x10, "SGD_STATUS_BAD_SCALE")):
        assert define(name) == bit and bit in sgd.STATUS_BITS
    enum = re.search(r"typedef enum \{(.*?)\} sgd_scheme;", text, re.S).group(1)
    values = dict(re.findall(r"(SGD_SCHEME_\w+)\s*=\s*(\d+)", enum))
    assert {k: int(v) for k, v in values.items()} == {
        "SGD_SCHEME_A": sgd.SCHEME_A, "SGD_SCHEME_B": sgd.SCHEME_B,
        "SGD_SCHEME_A_CALIBRATED": sgd.SCHEME_A_CALIBRATED, "SGD_SCHEME_B_CALIBRATED": sgd.SCHEME_B_CALIBRATED}
