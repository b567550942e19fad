"""Failure detection without a fault: the bounded pipeline waits of the decode and score kernels.

With sgd_test_pipeline_timeout the kernels' producer warps issue no copies and the wait limit is
lowered, so every consumer wait on the shared-memory pipeline runs out with nothing in flight.
The call must then end promptly, report SGD_STATUS_WAIT_TIMEOUT in its workspace status word and
leave the context usable: the same call made afterwards with the hooks off is exact again.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

WAIT_TIMEOUT = 0x2
POLLS = 4096


@pytest.fixture(scope="module")
def sgd():
    from conftest import build_library
    m = build_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


@pytest.fixture(scope="module")
def batch():
    wl = workloads.Workload("timeout", B=3, Hkv=2, G=8, D=128, kv_dtype="bf16", dist="outlier",
                            lengths=(300, 2100, 70))
    bt = workloads.generate(wl, 91)
    return bt, [t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens)]


def _run(sgd, bt, dev, path):
    """One call of the given path; returns (workspace, outputs to check)."""
    q, k, v, cu = dev
    G = bt.wl.G
    if path == "decode_bf16":
        out, lse, ws = sgd.decode_attn(q, G, k, v, cu)
        return ws, (out, lse)
    if path == "decode_int8_kept":
        kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
        torch.cuda.synchronize()
        idx, cu_kept, _ = sgd.oam_select(q, k, v, cu, G, 1.0, 1e-6, 1, 4, bt.lengths)
        torch.cuda.synchronize()
        return kc, vc, ks, vs, idx, cu_kept
    if path == "select":
        idx, cu_kept, ws = sgd.oam_select(q, k, v, cu, G, 1.0, 1e-6, 1, 4, bt.lengths)
        return ws, (idx, cu_kept)
    if path == "quantize_select":
        *_, idx, cu_kept, ws = sgd.quantize_select(q, k, v, cu, G, 1.0, 1e-6, 1, 4, "A", bt.lengths)
        return ws, (idx, cu_kept)
    raise ValueError(path)


def _timed_out_call(sgd, fn):
    sgd.test_pipeline_timeout(POLLS, True)
    try:
        t0 = time.perf_counter()
        ws = fn()
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
        status = sgd.workspace_status(ws)
    finally:
        sgd.test_pipeline_timeout(0, False)
    return status, dt


@pytest.mark.parametrize("path", ["decode_bf16", "select", "quantize_select"])
def test_a_wait_that_runs_out_is_reported_and_the_call_ends(sgd, batch, path):
    bt, dev = batch
    status, dt = _timed_out_call(sgd, lambda: _run(sgd, bt, dev, path)[0])
    assert status & WAIT_TIMEOUT
    assert dt < 20.0
    # the context is still usable: the same call with the hooks off is exact
    ws, res = _run(sgd, bt, dev, path)
    assert sgd.workspace_status(ws) == 0
    if path == "decode_bf16":
        ref_out, ref_lse = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, bt.wl.G)
        out, lse = (x.double().cpu().numpy() for x in res)
        assert np.abs(out - ref_out).max() <= 1e-2 * np.abs(ref_out).max()
        assert np.abs(lse - ref_lse).max() <= 1e-3
    else:
        _, ref_cu, _ = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, bt.wl.G, 1.0, 1e-6, 1, 4)
        assert res[1].cpu().tolist() == ref_cu.tolist()


def test_the_gather_decode_times_out_with_nothing_in_flight(sgd, batch):
    # the INT8 decode over a kept set (cp.async row gathers instead of TMA boxes)
    bt, dev = batch
    q, _, _, cu = dev
    kc, vc, ks, vs, idx, cu_kept = _run(sgd, bt, dev, "decode_int8_kept")
    kw = dict(k_scale=ks, v_scale=vs, scheme="A", n_parts_=sgd.n_parts(bt.lengths), idx=idx, cu_kept=cu_kept,
              kept_total_=idx.shape[1])
    status, dt = _timed_out_call(sgd, lambda: sgd.decode_attn(q, bt.wl.G, kc, vc, cu, **kw)[2])
    assert status & WAIT_TIMEOUT and dt < 20.0
    out, lse, ws = sgd.decode_attn(q, bt.wl.G, kc, vc, cu, **kw)
    assert sgd.workspace_status(ws) == 0
    quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A"), "A")
    ref_out, ref_lse = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, bt.wl.G, idx=idx.cpu().numpy(),
                                     cu_kept=cu_kept.cpu().numpy(), quant=quant)
    o, l = out.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.abs(o - ref_out).max() <= 1e-2 * np.abs(ref_out).max()
    assert np.abs(l - ref_lse).max() <= 1e-3
