"""sgd_decode_attn_noalloc: the decode for callers that cannot allocate device memory.

Such callers (a plugin inside a framework that owns all device memory and hands its plugins no
allocator, a latency-critical loop that may not call cudaMalloc because it can synchronise the
device) have no workspace to pass; this entry point keeps its scratch in a device array built into
the library.  Each test calls it through the C ABI, twice in a row where it matters (the second call
starts from the first one's leftovers in the shared array), and checks the result against
sgd_decode_attn with a caller workspace and against the fp64 oracle, with the parity tolerances of
the other GPU tests.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2  # bf16 / INT8 inputs
LSE_TOL = 1e-3
SGD_ERR_NULL = -1
SGD_ERR_SCRATCH_LIMIT = -9
SGD_STATUS_EMPTY_SEQUENCE = 0x1


@pytest.fixture(scope="module")
def sgd():
    from conftest import build_library
    m = build_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _batch(lengths, seed, dist="normal", Hkv=4):
    wl = workloads.Workload("noalloc", B=len(lengths), Hkv=Hkv, G=8, D=128, kv_dtype="bf16", dist=dist,
                            lengths=tuple(lengths))
    bt = workloads.generate(wl, seed)
    return bt, [t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens)]


def _noalloc_via_abi(sgd, q, G, k, v, cu, idx=None, cu_kept=None, kept_total=0, out_ptr=True, **kw):
    """Direct C-ABI call (the entry point has no workspace argument)."""
    kv = sgd._kv(k, v, cu, kw.get("k_scale"), kw.get("v_scale"), sgd.SCHEME_A, kw.get("n_parts", 0))
    B, Hq, D = cu.numel() - 1, k.shape[0] * G, k.shape[2]
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device=k.device)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=k.device)
    status = torch.full((1,), -1, dtype=torch.int32, device=k.device)
    rc = sgd.lib.sgd_decode_attn_noalloc(
        ctypes.c_void_p(q.data_ptr()), sgd.SGD_BF16, G, ctypes.byref(kv),
        None if idx is None else ctypes.c_void_p(idx.data_ptr()),
        None if cu_kept is None else ctypes.c_void_p(cu_kept.data_ptr()), int(kept_total), 0, 0, 0,
        ctypes.c_void_p(out.data_ptr()) if out_ptr else None, ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, out, lse, status


def _close(a, b, tol):
    scale = b.abs().max().item()
    return (a - b).abs().max().item() <= tol * scale


def _vs_oracle(out, lse, bt, G, **kw):
    ref_out, ref_lse = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, G, **kw)
    o, l = out.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.abs(o - ref_out).max() <= OUT_TOL * np.abs(ref_out).max()
    assert np.abs(l - ref_lse).max() <= LSE_TOL


def test_noalloc_matches_workspace_decode_and_oracle_on_two_calls(sgd):
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
    _vs_oracle(o1, l1, bt1, 8)
    _vs_oracle(o2, l2, bt2, 8)


def test_noalloc_int8_matches_workspace_decode_and_oracle(sgd):
    bt, (q, k, v, cu) = _batch((100, 5000), seed=303, dist="outlier")
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    parts = sgd.n_parts(bt.lengths)
    ref = sgd.decode_attn(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A", n_parts_=parts)
    quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A"), "A")
    for _ in range(2):
        rc, o, l, s = _noalloc_via_abi(sgd, q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, n_parts=parts)
        torch.cuda.synchronize()
        assert rc == 0 and s.item() == 0
        assert _close(o, ref[0], OUT_TOL) and (l - ref[1]).abs().max().item() <= LSE_TOL
        _vs_oracle(o, l, bt, 8, quant=quant)


def test_noalloc_over_a_kept_set(sgd):
    # the indexed path (kept positions from oam_select) through the built-in scratch
    bt, (q, k, v, cu) = _batch((513, 4100, 77), seed=404, dist="outlier", Hkv=2)
    idx, cu_kept, _ = sgd.oam_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, bt.lengths)
    Kt = idx.shape[1]
    ref = sgd.decode_attn(q, 8, k, v, cu, idx=idx, cu_kept=cu_kept, kept_total_=Kt)
    for _ in range(2):
        rc, o, l, s = _noalloc_via_abi(sgd, q, 8, k, v, cu, idx=idx, cu_kept=cu_kept, kept_total=Kt)
        torch.cuda.synchronize()
        assert rc == 0 and s.item() == 0
        assert _close(o, ref[0], OUT_TOL) and (l - ref[1]).abs().max().item() <= LSE_TOL
        _vs_oracle(o, l, bt, 8, idx=idx.cpu().numpy(), cu_kept=cu_kept.cpu().numpy())


def test_noalloc_reports_an_empty_sequence_in_the_callers_status_word(sgd):
    # sequence 1 has no tokens (cu_seqlens repeats a value): its status bit reaches the caller's
    # int32, the empty row gets out 0 and lse -inf, the other rows are still exact
    bt, (q, k, v, _) = _batch((300, 701), seed=505, Hkv=2)
    cu = torch.tensor([0, 300, 300, 1001], dtype=torch.int32, device="cuda")
    q3 = torch.cat([q[:1], q[:1], q[1:]])
    rc, o, l, s = _noalloc_via_abi(sgd, q3, 8, k, v, cu)
    torch.cuda.synchronize()
    assert rc == 0 and s.item() == SGD_STATUS_EMPTY_SEQUENCE
    assert torch.isinf(l[1]).all() and (o[1] == 0).all()
    ref_out, ref_lse = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8)
    keep = [0, 2]
    assert np.abs(o[keep].double().cpu().numpy() - ref_out).max() <= OUT_TOL * np.abs(ref_out).max()
    assert np.abs(l[keep].double().cpu().numpy() - ref_lse).max() <= LSE_TOL
    # the next call starts from a clear status word although the array still holds this one's
    bt2, (q2, k2, v2, cu2) = _batch((64, 1000), seed=506, Hkv=2)
    rc, o, l, s = _noalloc_via_abi(sgd, q2, 8, k2, v2, cu2)
    torch.cuda.synchronize()
    assert rc == 0 and s.item() == 0
    _vs_oracle(o, l, bt2, 8)


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
    assert rc == SGD_ERR_SCRATCH_LIMIT
    assert sgd.lib.sgd_error_string(rc) == b"the problem needs more scratch than SGD_NOALLOC_SCRATCH_BYTES"
    assert torch.isnan(o).all() and status.item() == -1  # nothing was launched


def test_noalloc_rejects_a_null_output_before_launching(sgd):
    bt, (q, k, v, cu) = _batch((100, 200), seed=606, Hkv=2)
    rc, o, l, status = _noalloc_via_abi(sgd, q, 8, k, v, cu, out_ptr=False)
    torch.cuda.synchronize()
    assert rc == SGD_ERR_NULL
    assert torch.isnan(l).all() and status.item() == -1  # nothing was launched, status untouched
