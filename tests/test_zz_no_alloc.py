"""sgd_decode_attn_noalloc: the decode for callers that cannot allocate device memory.

Such callers (a plugin inside a framework that owns all device memory, a latency-critical loop
that may not call cudaMalloc) get no workspace to pass; this entry point keeps its scratch in a
device array built into the library.  The test calls it through the C ABI twice in a row, on two
different batches, and checks each result against sgd_decode_attn with a caller workspace, using
the parity tolerances of the other GPU tests.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2  # bf16 / INT8 inputs
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def sgd():
    from conftest import build_library
    m = build_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _batch(lengths, seed, dist="normal"):
    wl = workloads.Workload("noalloc", B=len(lengths), Hkv=4, G=8, D=128, kv_dtype="bf16", dist=dist,
                            lengths=tuple(lengths))
    bt = workloads.generate(wl, seed)
    return bt, [t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens)]


def _noalloc_via_abi(sgd, q, G, k, v, cu, **kw):
    """Direct C-ABI call (no workspace argument exists)."""
    kv = sgd._kv(k, v, cu, kw.get("k_scale"), kw.get("v_scale"), sgd.SCHEME_A, kw.get("n_parts", 0))
    B, Hq, D = cu.numel() - 1, k.shape[0] * G, k.shape[2]
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device=k.device)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=k.device)
    status = torch.full((1,), -1, dtype=torch.int32, device=k.device)
    rc = sgd.lib.sgd_decode_attn_noalloc(
        ctypes.c_void_p(q.data_ptr()), sgd.SGD_BF16, G, ctypes.byref(kv), None, None, 0, 0, 0, 0,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, out, lse, status


def _close(a, b, tol):
    scale = b.abs().max().item()
    return (a - b).abs().max().item() <= tol * scale


def test_noalloc_matches_workspace_decode_on_two_calls(sgd):
    bt1, (q1, k1, v1, cu1) = _batch((1, 700, 2053, 4096), seed=101)
    bt2, (q2, k2, v2, cu2) = _batch((3000, 65, 9), seed=202)
    ref1 = sgd.decode_attn(q1, 8, k1, v1, cu1)
    ref2 = sgd.decode_attn(q2, 8, k2, v2, cu2)
    rc1, o1, l1, s1 = _noalloc_via_abi(sgd, q1, 8, k1, v1, cu1)
    rc2, o2, l2, s2 = _noalloc_via_abi(sgd, q2, 8, k2, v2, cu2)
    torch.cuda.synchronize()
    assert rc1 == 0 and rc2 == 0
    assert s1.item() == 0 and s2.item() == 0
    assert _close(o1, ref1[0], OUT_TOL) and (l1 - ref1[1]).abs().max().item() <= LSE_TOL
    assert _close(o2, ref2[0], OUT_TOL) and (l2 - ref2[1]).abs().max().item() <= LSE_TOL


def test_noalloc_int8_matches_workspace_decode(sgd):
    bt, (q, k, v, cu) = _batch((100, 5000), seed=303, dist="outlier")
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    parts = sgd.n_parts(bt.lengths)
    ref = sgd.decode_attn(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A", n_parts_=parts)
    for _ in range(2):
        rc, o, l, s = _noalloc_via_abi(sgd, q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, n_parts=parts)
        torch.cuda.synchronize()
        assert rc == 0 and s.item() == 0
        assert _close(o, ref[0], OUT_TOL) and (l - ref[1]).abs().max().item() <= LSE_TOL


def test_noalloc_rejects_problems_beyond_its_scratch(sgd):
    # 2048 rows of G = 16 heads need far more partial-result scratch than the built-in array
    lengths = [64] * 512
    wl = workloads.Workload("big", B=512, Hkv=4, G=16, D=128, kv_dtype="bf16", dist="normal",
                            lengths=tuple(lengths))
    bt = workloads.generate(wl, 7)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    kv = sgd._kv(k, v, cu)
    assert sgd.workspace_size(sgd.OP_DECODE, kv, 16) > (4 << 20)
    rc, o, _, status = _noalloc_via_abi(sgd, q, 16, k, v, cu)
    torch.cuda.synchronize()
    assert rc == -9
    assert sgd.lib.sgd_error_string(rc) == b"the problem needs more scratch than SGD_NOALLOC_SCRATCH_BYTES"
    assert torch.isnan(o).all() and status.item() == -1  # nothing was launched
