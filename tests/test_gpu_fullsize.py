"""Full-size workloads in the launch configuration bench.py times (automatic split over all SMs),
CUDA path vs the fp64 oracle.  The GPU computes every row; the oracle recomputes sampled
(sequence, KV head) rows one by one (including the shortest and longest), and the INT8 codes and
scales and the kept index sets are compared in full."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def sgd():
    from conftest import build_library
    m = build_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def sample_rows(bt, n_extra=3, seed=0):
    L = bt.lengths
    rows = {(int(np.argmin(L)), 0), (int(np.argmax(L)), bt.wl.Hkv - 1)}
    rng = np.random.default_rng(seed)
    while len(rows) < 2 + n_extra:
        rows.add((int(rng.integers(bt.wl.B)), int(rng.integers(bt.wl.Hkv))))
    return sorted(rows)


def compare_rows(out, lse, ref_out, ref_lse, rows, G):
    out = out.double().cpu().numpy()
    lse = lse.double().cpu().numpy()
    for b, h in rows:
        sl = slice(h * G, (h + 1) * G)
        scale = np.abs(ref_out[b, sl]).max()
        assert np.abs(out[b, sl] - ref_out[b, sl]).max() <= OUT_TOL * scale, (b, h)
        assert np.abs(lse[b, sl] - ref_lse[b, sl]).max() <= LSE_TOL, (b, h)


def test_config2_bf16_32k(sgd):
    bt = workloads.generate(workloads.config(2))
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    out, lse, ws = sgd.decode_attn(q, 8, k, v, cu)
    assert sgd.workspace_status(ws) == 0
    rows = sample_rows(bt)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, rows=rows)
    compare_rows(out, lse, *ref, rows, 8)


def test_config3_ragged_both_schedules(sgd):
    bt = workloads.generate(workloads.config(3))
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    o0, l0, ws0 = sgd.decode_attn(q, 8, k, v, cu, schedule=0)
    o1, l1, ws1 = sgd.decode_attn(q, 8, k, v, cu, schedule=1)
    assert sgd.workspace_status(ws0) == 0 and sgd.workspace_status(ws1) == 0
    rows = sample_rows(bt, n_extra=4)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, rows=rows)
    compare_rows(o0, l0, *ref, rows, 8)
    compare_rows(o1, l1, *ref, rows, 8)
    # the two schedules agree on every row
    scale = o1.abs().max().item()
    assert (o0 - o1).abs().max().item() <= OUT_TOL * scale
    assert (l0 - l1).abs().max().item() <= LSE_TOL


@pytest.mark.parametrize("scheme", ["A", "B"])
def test_config4_int8_128k(sgd, scheme):
    bt = workloads.generate(workloads.config(4))
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    kc, vc, ks, vs, wsq = sgd.quantize_kv(k, v, cu, scheme, bt.lengths)
    del k, v
    out, lse, ws = sgd.decode_attn(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme=scheme,
                                   n_parts_=sgd.n_parts(bt.lengths))
    assert sgd.workspace_status(wsq) == 0 and sgd.workspace_status(ws) == 0
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
    assert np.array_equal(ks.cpu().numpy().reshape(quant[2].shape), quant[2])
    assert np.array_equal(vs.cpu().numpy(), quant[3])
    for h in range(bt.wl.Hkv):  # every code, one head at a time
        assert np.array_equal(kc[h].cpu().numpy(), quant[0][h]), h
        assert np.array_equal(vc[h].cpu().numpy(), quant[1][h]), h
    rows = sample_rows(bt, n_extra=2)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, quant=(*quant, scheme), rows=rows)
    compare_rows(out, lse, *ref, rows, 8)


def test_config5_oam_int8a(sgd):
    wl = workloads.config(5)
    bt = workloads.generate(wl)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    idx, cu_kept, wss = sgd.oam_select(q, k, v, cu, wl.G, wl.beta, wl.eps, wl.keep_num, wl.keep_den, bt.lengths)
    out, lse, ws = sgd.decode_attn(q, wl.G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                   n_parts_=sgd.n_parts(bt.lengths), idx=idx, cu_kept=cu_kept,
                                   kept_total_=idx.shape[1])
    assert sgd.workspace_status(wss) == 0 and sgd.workspace_status(ws) == 0
    # every row's kept set against the oracle's top-K (near-ties within 1e-4 exempt)
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, wl.beta, wl.eps,
                                                wl.keep_num, wl.keep_den)
    assert cu_kept.cpu().tolist() == ref_cu.tolist()
    got = idx.cpu().numpy()
    n_diff = 0
    for (b, h), s in scores.items():
        a, e = int(ref_cu[b]), int(ref_cu[b + 1])
        kth = np.sort(s)[::-1][e - a - 1]
        g, w = set(got[h, a:e].tolist()), set(ref_idx[h, a:e].tolist())
        assert (np.diff(got[h, a:e]) > 0).all()
        for t in g ^ w:
            assert abs(s[t] - kth) <= 1e-4, (b, h, t)
        n_diff += len(g ^ w)
    assert n_diff <= 8
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    rows = sample_rows(bt, n_extra=3)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, idx=ref_idx, cu_kept=ref_cu,
                        quant=(*quant, "A"), rows=rows)
    compare_rows(out, lse, *ref, rows, wl.G)
    # the same selection decoded with INT8 query codes, one scale per (sequence, head): the
    # query-codes workload (same sizes, q_quant = "token")
    assert workloads.config(7).with_(name=wl.name, q_quant=None, seed=None) == wl
    out, lse, ws = sgd.decode_attn(q, wl.G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                   n_parts_=sgd.n_parts(bt.lengths), idx=idx, cu_kept=cu_kept,
                                   kept_total_=idx.shape[1], q_quant="token")
    assert sgd.workspace_status(ws) == 0
    qd = oracle.dequant_q(*oracle.quantize_q(bt.q, "token"))
    ref = oracle.decode(qd, bt.k, bt.v, bt.cu_seqlens, wl.G, idx=ref_idx, cu_kept=ref_cu,
                        quant=(*quant, "A"), rows=rows)
    compare_rows(out, lse, *ref, rows, wl.G)


def test_config8_two_query_tokens_int8_128k(sgd):
    # the speculative-decode workload: workload 4's cache, two query tokens per sequence
    wl = workloads.config(8)
    bt = workloads.generate(wl)
    assert bt.q.shape == (wl.B, 2, wl.Hq, wl.D)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    kc, vc, ks, vs, wsq = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    del k, v
    out, lse, ws = sgd.decode_attn_multi(q, wl.G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                         n_parts_=sgd.n_parts(bt.lengths))
    assert sgd.workspace_status(wsq) == 0 and sgd.workspace_status(ws) == 0
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    rows = sample_rows(bt, n_extra=1)
    ref_out, ref_lse = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, 2, quant=(*quant, "A"), rows=rows)
    for m in range(2):
        compare_rows(out[:, m], lse[:, m], ref_out[:, m], ref_lse[:, m], rows, wl.G)


@pytest.mark.parametrize("n", [6, 9])
def test_config6_and_9_selection_over_the_int8_cache(sgd, n):
    # workload 6 keeps tokens, workload 9 whole 64-token blocks, both scored on the INT8 K codes
    wl = workloads.config(n)
    bt = workloads.generate(wl)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    vn = torch.empty(k.shape[:2], dtype=torch.float32, device="cuda")
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths, v_norm=vn)
    del k, v
    parts = sgd.n_parts(bt.lengths)
    kw = dict(k_scale=ks, v_scale=vs, scheme="A", n_parts_=parts)
    select = sgd.oam_select_blocks if wl.blocks else sgd.oam_select
    idx, cu_kept, wss = select(q, kc, vc, cu, wl.G, wl.beta, wl.eps, wl.keep_num, wl.keep_den, bt.lengths,
                               v_norm=vn, **kw)
    assert sgd.workspace_status(wss) == 0
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    ref_idx, ref_cu, scores = oracle.oam_select_int8(bt.q, quant[0], quant[2], bt.v, bt.cu_seqlens, "A", wl.G,
                                                     wl.beta, wl.eps, wl.keep_num, wl.keep_den)
    if wl.blocks:
        ref_idx, ref_cu, scores = oracle.select_blocks(scores, bt.cu_seqlens, wl.Hkv, wl.keep_num, wl.keep_den)
    assert cu_kept.cpu().tolist() == ref_cu.tolist()
    got = idx.cpu().numpy()
    for (b, h), s in scores.items():
        a, e = int(ref_cu[b]), int(ref_cu[b + 1])
        kth = np.sort(s)[::-1][e - a - 1]
        assert (np.diff(got[h, a:e]) > 0).all()
        for t in set(got[h, a:e].tolist()) ^ set(ref_idx[h, a:e].tolist()):
            assert abs(s[t] - kth) <= 1e-4, (b, h, t)
    # the decode over the oracle's selection, in the bench's launch configuration
    ti, tc = torch.from_numpy(ref_idx).cuda(), torch.from_numpy(ref_cu).cuda()
    rows = sample_rows(bt, n_extra=2)
    if wl.blocks:
        out, lse, ws = sgd.decode_attn_blocks(q, wl.G, kc, vc, cu, ti, tc, **kw)
        ref = oracle.decode_blocks(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, ref_idx, ref_cu, quant=(*quant, "A"),
                                   rows=rows)
    else:
        out, lse, ws = sgd.decode_attn(q, wl.G, kc, vc, cu, idx=ti, cu_kept=tc, kept_total_=ref_idx.shape[1], **kw)
        ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, idx=ref_idx, cu_kept=ref_cu,
                            quant=(*quant, "A"), rows=rows)
    assert sgd.workspace_status(ws) == 0
    compare_rows(out, lse, *ref, rows, wl.G)


def test_config10_four_query_tokens_int8_128k(sgd):
    # 32 columns per KV head: two CTAs per split range, one per group of 16 columns
    wl = workloads.config(10)
    bt = workloads.generate(wl)
    assert bt.q.shape == (wl.B, 4, wl.Hq, wl.D)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    kc, vc, ks, vs, wsq = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    del k, v
    out, lse, ws = sgd.decode_attn_multi(q, wl.G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                         n_parts_=sgd.n_parts(bt.lengths))
    assert sgd.workspace_status(wsq) == 0 and sgd.workspace_status(ws) == 0
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    rows = sample_rows(bt, n_extra=0)
    ref_out, ref_lse = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, 4, quant=(*quant, "A"), rows=rows)
    for m in range(4):
        compare_rows(out[:, m], lse[:, m], ref_out[:, m], ref_lse[:, m], rows, wl.G)


@pytest.mark.parametrize("n", [12, 13])
def test_config12_13_query_codes_int8_128k(sgd, n):
    # the scheme table: per-tensor Q/K/V (scheme B, one query scale) and scheme A with query codes
    wl = workloads.config(n)
    bt = workloads.generate(wl)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    kc, vc, ks, vs, wsq = sgd.quantize_kv(k, v, cu, wl.scheme, bt.lengths)
    del k, v
    out, lse, ws = sgd.decode_attn(q, wl.G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme=wl.scheme,
                                   n_parts_=sgd.n_parts(bt.lengths), q_quant=wl.q_quant)
    assert sgd.workspace_status(wsq) == 0 and sgd.workspace_status(ws) == 0
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, wl.scheme)
    qd = oracle.dequant_q(*oracle.quantize_q(bt.q, wl.q_quant))
    rows = sample_rows(bt, n_extra=1)
    ref = oracle.decode(qd, bt.k, bt.v, bt.cu_seqlens, wl.G, quant=(*quant, wl.scheme), rows=rows)
    compare_rows(out, lse, *ref, rows, wl.G)


def check_kept_sets(idx, cu_kept, ref_idx, ref_cu, scores, max_diff):
    """Every row's kept set against the oracle's top-K: identical except tokens whose oracle score
    lies within 1e-4 of the row's K-th score; positions ascending."""
    assert cu_kept.cpu().tolist() == ref_cu.tolist()
    got = idx.cpu().numpy()
    n_diff = 0
    for (b, h), s in scores.items():
        a, e = int(ref_cu[b]), int(ref_cu[b + 1])
        kth = np.sort(s)[::-1][e - a - 1]
        g, w = set(got[h, a:e].tolist()), set(ref_idx[h, a:e].tolist())
        assert (np.diff(got[h, a:e]) > 0).all(), (b, h)
        for t in g ^ w:
            assert abs(s[t] - kth) <= 1e-4, (b, h, t)
        n_diff += len(g ^ w)
    assert n_diff <= max_diff


@pytest.mark.parametrize("n,scheme", [(5, "A"), (4, "A"), (4, "B")])
def test_fused_quantize_select_full_size(sgd, n, scheme):
    """The call the benchmark times, sgd_quantize_select, at full size: workload 5 (4 sequences of
    32K-128K tokens) and workload 4's 8 x 128K cache, where a bf16 tensor is 2 GiB and byte offsets
    pass 2^31.  Every K and V code and every scale bit-exact, the stored value norms, every row's
    kept set, then the decode over the kept tokens on sampled rows, all against the oracle."""
    wl = workloads.config(n)
    bt = workloads.generate(wl)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    vn = torch.empty(k.shape[:2], dtype=torch.float32, device="cuda")
    kc, vc, ks, vs, idx, cu_kept, wsq = sgd.quantize_select(q, k, v, cu, wl.G, wl.beta, wl.eps, wl.keep_num,
                                                            wl.keep_den, scheme, bt.lengths, v_norm=vn)
    del k, v
    assert sgd.workspace_status(wsq) == 0
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
    assert np.array_equal(ks.cpu().numpy().reshape(quant[2].shape), quant[2])
    assert np.array_equal(vs.cpu().numpy(), quant[3])
    for h in range(wl.Hkv):  # every code and value norm, one head at a time
        assert np.array_equal(kc[h].cpu().numpy(), quant[0][h]), h
        assert np.array_equal(vc[h].cpu().numpy(), quant[1][h]), h
        ref_vn = oracle.value_norms(bt.v[h])
        assert np.allclose(vn[h].double().cpu().numpy(), ref_vn, rtol=1e-5, atol=0), h
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, wl.beta, wl.eps,
                                                wl.keep_num, wl.keep_den)
    check_kept_sets(idx, cu_kept, ref_idx, ref_cu, scores, max_diff=4 * wl.B * wl.Hkv)
    out, lse, ws = sgd.decode_attn(q, wl.G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme=scheme,
                                   n_parts_=sgd.n_parts(bt.lengths), idx=idx, cu_kept=cu_kept,
                                   kept_total_=idx.shape[1])
    assert sgd.workspace_status(ws) == 0
    rows = sample_rows(bt, n_extra=2)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, idx=ref_idx, cu_kept=ref_cu,
                        quant=(*quant, scheme), rows=rows)
    compare_rows(out, lse, *ref, rows, wl.G)


@pytest.mark.parametrize("n,scheme", [(5, "A"), (4, "B")])
def test_fused_quantize_select_calibrated_full_size(sgd, n, scheme):
    """sgd_quantize_select with calibrated per-tensor scales at full size, where one pass writes
    every code: the scales are 1/4 of the computed ones (the largest values saturate).  Every code
    and scale bit-exact against the oracle with the same scales; the value norms and every kept
    set the same bits as the call with computed scales."""
    wl = workloads.config(n)
    bt = workloads.generate(wl)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    dyn_quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
    k_cal = np.float32(dyn_quant[2].ravel()[0] * np.float32(0.25)) if scheme == "B" else None
    v_cal = np.float32(dyn_quant[3][0] * np.float32(0.25))
    del dyn_quant
    cal = dict(v_scale_in=torch.tensor([float(v_cal)], dtype=torch.float32, device="cuda"))
    if scheme == "B":
        cal["k_scale_in"] = torch.tensor([float(k_cal)], dtype=torch.float32, device="cuda")
    vn = torch.empty(k.shape[:2], dtype=torch.float32, device="cuda")
    kc, vc, ks, vs, idx, cu_kept, wsq = sgd.quantize_select(q, k, v, cu, wl.G, wl.beta, wl.eps, wl.keep_num,
                                                            wl.keep_den, scheme, bt.lengths, v_norm=vn, **cal)
    assert sgd.workspace_status(wsq) == 0
    vn_dyn = torch.empty_like(vn)
    dyn = sgd.quantize_select(q, k, v, cu, wl.G, wl.beta, wl.eps, wl.keep_num, wl.keep_den, scheme, bt.lengths,
                              v_norm=vn_dyn)
    assert torch.equal(idx, dyn[4]) and torch.equal(cu_kept, dyn[5]) and torch.equal(vn, vn_dyn)
    del dyn, k, v
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme, k_scale=k_cal, v_scale=v_cal)
    assert np.array_equal(ks.cpu().numpy().reshape(quant[2].shape), quant[2])
    assert np.array_equal(vs.cpu().numpy(), quant[3])
    saturated = 0
    for h in range(wl.Hkv):
        assert np.array_equal(kc[h].cpu().numpy(), quant[0][h]), h
        assert np.array_equal(vc[h].cpu().numpy(), quant[1][h]), h
        saturated += int((np.abs(quant[1][h].astype(np.int32)) == 127).sum())
    assert saturated > 0


def test_config14_ragged_int8_decode(sgd):
    """The ragged INT8 batch (16 log-uniform lengths in [512, 128K] over the scheme-A cache) in the
    bench's launch configuration: every code and scale bit-exact, sampled rows (shortest and longest
    included) of the equal-work split decode against the oracle, and the one-CTA-per-row schedule
    agreeing with it on every row."""
    wl = workloads.config(14)
    bt = workloads.generate(wl)
    q, k, v, cu = (t.cuda() for t in (bt.q, bt.k, bt.v, bt.cu_seqlens))
    kc, vc, ks, vs, wsq = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    del k, v
    kw = dict(k_scale=ks, v_scale=vs, scheme="A", n_parts_=sgd.n_parts(bt.lengths))
    o0, l0, ws0 = sgd.decode_attn(q, wl.G, kc, vc, cu, schedule=0, **kw)
    o1, l1, ws1 = sgd.decode_attn(q, wl.G, kc, vc, cu, schedule=1, **kw)
    assert sgd.workspace_status(wsq) == 0 and sgd.workspace_status(ws0) == 0 and sgd.workspace_status(ws1) == 0
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    assert np.array_equal(ks.cpu().numpy().reshape(quant[2].shape), quant[2])
    assert np.array_equal(vs.cpu().numpy(), quant[3])
    assert np.array_equal(kc.cpu().numpy(), quant[0]) and np.array_equal(vc.cpu().numpy(), quant[1])
    rows = sample_rows(bt, n_extra=4)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, wl.G, quant=(*quant, "A"), rows=rows)
    compare_rows(o0, l0, *ref, rows, wl.G)
    compare_rows(o1, l1, *ref, rows, wl.G)
    scale = o1.abs().max().item()
    assert (o0 - o1).abs().max().item() <= OUT_TOL * scale
    assert (l0 - l1).abs().max().item() <= LSE_TOL
