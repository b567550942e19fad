"""CUDA path vs the fp64 oracle on the same seeded inputs, through the C ABI.

Tolerances (the stated acceptance bar): outputs max-abs error <= 1e-2 * max|out| for bf16 (and
INT8) inputs, <= 1e-3 * max|out| for fp32 inputs; lse <= 1e-3 absolute; INT8 codes and scales
bit-exact; the work partition bit-exact; kept index sets exact except tokens whose oracle score is
within 1e-4 of the K-th score.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

OUT_TOL = {"f32": 1e-3, "bf16": 1e-2}
LSE_TOL = 1e-3
TIE_WINDOW = 1e-4


@pytest.fixture(scope="module")
def sgd():
    from conftest import build_library
    m = build_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def dev(bt):
    return (bt.q.cuda(), bt.k.cuda(), bt.v.cuda(), bt.cu_seqlens.cuda())


def make(lengths, G=8, D=128, Hkv=2, dtype="bf16", dist="normal", seed=0):
    wl = workloads.Workload("t", B=len(lengths), Hkv=Hkv, G=G, D=D, kv_dtype=dtype, dist=dist,
                            lengths=tuple(lengths))
    return workloads.generate(wl, seed)


def assert_close(out, lse, ref_out, ref_lse, tol, rows=None):
    out = out.double().cpu().numpy()
    lse = lse.double().cpu().numpy()
    if rows is not None:  # compare only the computed (b, kvh) rows
        mask = ~np.isnan(ref_lse)
        out, lse, ref_out, ref_lse = out[mask], lse[mask], ref_out[mask], ref_lse[mask]
    scale = np.abs(ref_out).max()
    err = np.abs(out - ref_out).max()
    lerr = np.abs(lse - ref_lse).max()
    assert err <= tol * scale, f"out error {err:.3e} > {tol} * {scale:.3e}"
    assert lerr <= LSE_TOL, f"lse error {lerr:.3e}"
    return err / scale, lerr


def check_status(sgd, ws):
    assert sgd.workspace_status(ws) == 0


# ---------------------------------------------------------------------------------------------
# dense decode
# ---------------------------------------------------------------------------------------------
def test_config1_fp32_four_chunks(sgd):
    bt = workloads.generate(workloads.config(1))
    q, k, v, cu = dev(bt)
    out, lse, ws = sgd.decode_attn(q, 4, k, v, cu, n_splits=4)
    segs, ncta = sgd.plan_segments(cu, 1, 1, 4, 16, 0)
    assert ncta == 4 and segs[:, 3].tolist() == [64, 64, 64, 64]
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 4)
    assert_close(out, lse, *ref, OUT_TOL["f32"])
    check_status(sgd, ws)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_dense_decode_shapes(sgd, dtype, D, G):
    bt = make((1, 63, 64, 65, 1000, 2053), G=G, D=D, Hkv=2, dtype=dtype, seed=G * 7 + D)
    q, k, v, cu = dev(bt)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, G)
    for n_splits in (0, 3, 37):
        out, lse, ws = sgd.decode_attn(q, G, k, v, cu, n_splits=n_splits)
        assert_close(out, lse, *ref, OUT_TOL[dtype])
        check_status(sgd, ws)


def test_bf16_multi_tile_several_ctas(sgd):
    # config-2 shapes with shorter rows: many 64-token tiles per CTA and CTA ranges crossing rows
    bt = workloads.generate(workloads.config(2, lengths=(4096 + 37,) * 3, B=3), seed=2)
    q, k, v, cu = dev(bt)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8)
    out, lse, ws = sgd.decode_attn(q, 8, k, v, cu)
    assert_close(out, lse, *ref, OUT_TOL["bf16"])
    check_status(sgd, ws)


@pytest.mark.parametrize("G", [16, 3])
def test_row_merged_from_hundreds_of_segments(sgd, G):
    # 800 requested CTAs: ranges of 16 tokens, so the 11500-token row has 719 segments and the
    # CTA finishing its last one merges them, in more than one shared-memory round at G = 16
    bt = make((11500, 40), G=G, D=128, Hkv=1, seed=91)
    q, k, v, cu = dev(bt)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, G)
    out, lse, ws = sgd.decode_attn(q, G, k, v, cu, n_splits=800)
    assert_close(out, lse, *ref, OUT_TOL["bf16"])
    check_status(sgd, ws)
    segs, _ = sgd.plan_segments(cu, 2, 1, 800, 16, 0)
    assert int((segs[:, 1] == 0).sum()) > 510


def test_ragged_equal_work_equals_one_cta_per_row(sgd):
    wl = workloads.config(3, length_range=(17, 6000))
    bt = workloads.generate(wl, seed=3)
    q, k, v, cu = dev(bt)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8)
    o0, l0, ws0 = sgd.decode_attn(q, 8, k, v, cu, schedule=0)
    o1, l1, ws1 = sgd.decode_attn(q, 8, k, v, cu, schedule=1)
    assert_close(o0, l0, *ref, OUT_TOL["bf16"])
    assert_close(o1, l1, *ref, OUT_TOL["bf16"])
    assert (o0 - o1).abs().max().item() <= 1e-2 * np.abs(ref[0]).max()
    check_status(sgd, ws0)
    check_status(sgd, ws1)


def test_identical_keys_give_mean_of_v(sgd):
    bt = make((300,), G=4, D=128, Hkv=1)
    bt.k[:] = bt.k[:, :1]  # every key equal
    q, k, v, cu = dev(bt)
    out, lse, _ = sgd.decode_attn(q, 4, k, v, cu, n_splits=5)
    mean = bt.v[0].double().mean(dim=0)
    assert (out[0].double().cpu() - mean).abs().max().item() <= 1e-2 * mean.abs().max().item()


# ---------------------------------------------------------------------------------------------
# partition
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("row_cost", [0, 256, 48])
@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("mode", [0, 1])
def test_plan_matches_oracle_bit_exact(sgd, seed, mode, row_cost):
    rng = np.random.default_rng(seed)
    B, Hkv = int(rng.integers(1, 20)), int(rng.integers(1, 9))
    lens = np.rint(np.exp(rng.uniform(0, 11, B))).astype(np.int64)
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).cuda()
    n_req = int(rng.integers(1, 400))
    min_chunk = 16 * int(rng.integers(1, 20))
    segs, ncta = sgd.plan_segments(cu, B, Hkv, n_req, min_chunk, mode, row_cost)
    row_len = np.tile(lens, Hkv)  # row = kvh * B + b
    ref = oracle.plan(row_len, n_req, 16, min_chunk, mode, row_cost)
    got = segs.numpy()
    assert ncta == ref["n_cta"]
    assert got[:, 0].tolist() == ref["cta"].tolist()
    assert got[:, 1].tolist() == ref["row"].tolist()
    assert got[:, 2].tolist() == ref["start"].tolist()
    assert got[:, 3].tolist() == ref["len"].tolist()


@pytest.mark.parametrize("B,Hkv,n_req", [(6825, 1, 296), (6826, 1, 296), (2600, 3, 900), (40, 60, 2000)])
def test_plan_of_large_batches_matches_oracle(sgd, B, Hkv, n_req):
    # batches on both sides of the per-sequence staging limit (6825 sequences: the plan kernel
    # with closed-form row positions, else the one that scans rows) and with more rows and CTAs
    # than one block of threads
    rng = np.random.default_rng(B + Hkv)
    lens = rng.integers(1, 300, B).astype(np.int64)
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).cuda()
    for mode, row_cost in ((0, 0), (1, 0), (0, sgd.ROW_COST)):
        segs, ncta = sgd.plan_segments(cu, B, Hkv, n_req, 64, mode, row_cost)
        ref = oracle.plan(np.tile(lens, Hkv), n_req, 16, 64, mode, row_cost)
        got = segs.numpy()
        assert ncta == ref["n_cta"]
        for j, key in enumerate(("cta", "row", "start", "len")):
            assert got[:, j].tolist() == ref[key].tolist(), (key, mode, row_cost)


# ---------------------------------------------------------------------------------------------
# INT8 cache
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("scheme", ["A", "B"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_bit_exact(sgd, scheme, dtype):
    bt = make((1, 63, 64, 65, 700, 4099), G=8, D=128, Hkv=3, dtype=dtype, dist="outlier", seed=11)
    # plant exact rounding ties in partition 1 of sequence 5 (tokens 64..127) of head 1
    s0 = int(bt.cu_seqlens[5])
    bt.k[1, s0 + 64:s0 + 128] = 0
    if dtype == "f32":  # max |x| = 889 -> scale 7: quotients 6.5, 12.5, 14.5, -22.5
        ties, want = [45.5, 87.5, 101.5, -157.5, 889.0], [6, 12, 14, -22, 127]
    else:  # bf16 holds these exactly; max |x| = 127 -> scale 1
        ties, want = [2.5, 3.5, -2.5, 126.5, 127.0, -0.5], [2, 4, -2, 126, 127, 0]
    bt.k[1, s0 + 64, :len(ties)] = torch.tensor(ties).to(bt.k.dtype)
    q, k, v, cu = dev(bt)
    kc, vc, ks, vs, ws = sgd.quantize_kv(k, v, cu, scheme, bt.lengths)
    rkc, rvc, rks, rvs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
    assert np.array_equal(ks.cpu().numpy().reshape(rks.shape), rks)
    assert np.array_equal(vs.cpu().numpy(), rvs)
    assert np.array_equal(kc.cpu().numpy(), rkc)
    assert np.array_equal(vc.cpu().numpy(), rvc)
    if scheme == "A":
        assert kc[1, s0 + 64, :len(want)].tolist() == want
    check_status(sgd, ws)


@pytest.mark.parametrize("scheme", ["A", "B"])
@pytest.mark.parametrize("G", [4, 8, 16])
def test_int8_decode(sgd, scheme, G):
    bt = make((1, 65, 700, 3000), G=G, D=128, Hkv=2, dist="outlier", seed=21 + G)
    q, k, v, cu = dev(bt)
    rkc, rvc, rks, rvs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, G, quant=(rkc, rvc, rks, rvs, scheme))
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths)
    parts = sgd.n_parts(bt.lengths)
    for n_splits in (0, 7):
        out, lse, ws = sgd.decode_attn(q, G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme=scheme, n_parts_=parts,
                                       n_splits=n_splits)
        assert_close(out, lse, *ref, OUT_TOL["bf16"])
        check_status(sgd, ws)


# query codes: q.k becomes an exact integer dot product of the codes times the two scales, so
# the result is compared with the oracle attending with the dequantised query code * scale; the
# oracle with the unquantised query must sit measurably further away (the kernel really used codes)
@pytest.mark.parametrize("mode", ["token", "tensor"])
@pytest.mark.parametrize("G", [8, 16])
@pytest.mark.parametrize("indexed", [False, True])
def test_int8_decode_query_codes(sgd, mode, G, indexed):
    bt = make((1, 65, 700, 3000), G=G, D=128, Hkv=2, dist="outlier", seed=91 + G)
    q, k, v, cu = dev(bt)
    scheme = "A" if mode == "token" else "B"
    quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme), scheme)
    sel = {}
    if indexed:
        ref_idx, ref_cu, _ = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, G, 1.0, 1e-6, 1, 4)
        sel = dict(idx=ref_idx, cu_kept=ref_cu)
    qd = oracle.dequant_q(*oracle.quantize_q(bt.q, mode))
    ref = oracle.decode(qd, bt.k, bt.v, bt.cu_seqlens, G, quant=quant, **sel)
    ref_raw = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, G, quant=quant, **sel)
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths)
    extra = {}
    if indexed:
        extra = dict(idx=torch.from_numpy(ref_idx).int().cuda(), cu_kept=torch.from_numpy(ref_cu).int().cuda(),
                     kept_total_=ref_idx.shape[1])
    for n_splits in (0, 7):
        out, lse, ws = sgd.decode_attn(q, G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme=scheme,
                                       n_parts_=sgd.n_parts(bt.lengths), n_splits=n_splits, q_quant=mode, **extra)
        _, lerr = assert_close(out, lse, *ref, OUT_TOL["bf16"])
        check_status(sgd, ws)
        gap = np.abs(ref[1] - ref_raw[1]).max()
        assert lerr < 0.25 * gap, f"lse error {lerr:.2e} vs quantisation effect {gap:.2e}"


def test_query_codes_of_an_all_zero_query_row(sgd):
    # scale 0 -> every code 0: the row's logits are all 0 and its output the mean of the dequantised V
    bt = make((300, 45), G=8, D=128, Hkv=2, dist="outlier", seed=17)
    bt.q[0, 3] = 0  # sequence 0, KV head 0, query head 3
    bt.q[1, 8:16] = 0  # every query head of sequence 1, KV head 1
    q, k, v, cu = dev(bt)
    quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A"), "A")
    ref = oracle.decode(oracle.dequant_q(*oracle.quantize_q(bt.q, "token")), bt.k, bt.v, bt.cu_seqlens, 8,
                        quant=quant)
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    out, lse, ws = sgd.decode_attn(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                   n_parts_=sgd.n_parts(bt.lengths), n_splits=5, q_quant="token")
    assert_close(out, lse, *ref, OUT_TOL["bf16"])
    check_status(sgd, ws)
    assert abs(float(lse[0, 3]) - np.log(300)) < 1e-3 and abs(float(lse[1, 8]) - np.log(45)) < 1e-3


def test_int8_d64_uses_cuda_core_path(sgd):
    bt = make((5, 300), G=8, D=64, Hkv=2, dist="outlier", seed=5)
    q, k, v, cu = dev(bt)
    rkc, rvc, rks, rvs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, quant=(rkc, rvc, rks, rvs, "A"))
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    assert np.array_equal(kc.cpu().numpy(), rkc)
    out, lse, _ = sgd.decode_attn(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                  n_parts_=sgd.n_parts(bt.lengths))
    assert_close(out, lse, *ref, OUT_TOL["bf16"])


# ---------------------------------------------------------------------------------------------
# OAM selection
# ---------------------------------------------------------------------------------------------
def check_selection(idx, cu_kept, ref_idx, ref_cu, scores, B, Hkv):
    assert cu_kept.tolist() == ref_cu.tolist()
    idx = idx.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            a, e = int(ref_cu[b]), int(ref_cu[b + 1])
            got, want = set(idx[h, a:e].tolist()), set(ref_idx[h, a:e].tolist())
            assert (np.diff(idx[h, a:e]) > 0).all(), "kept positions must ascend"
            s = scores[(b, h)]
            kth = np.sort(s)[::-1][e - a - 1]
            for t in got ^ want:
                assert abs(s[t] - kth) <= TIE_WINDOW, f"token {t} differs and is not a near-tie"


@pytest.mark.parametrize("G,D", [(8, 128), (4, 64), (16, 128), (1, 128)])
def test_oam_select_matches_oracle(sgd, G, D):
    bt = make((1, 7, 64, 500, 5000), G=G, D=D, Hkv=2, dist="outlier", seed=31 + G)
    q, k, v, cu = dev(bt)
    idx, cu_kept, ws = sgd.oam_select(q, k, v, cu, G, 1.0, 1e-6, 1, 8, bt.lengths)
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, G, 1.0, 1e-6, 1, 8)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, bt.wl.B, 2)
    check_status(sgd, ws)


def test_oam_select_f32_cache(sgd):
    bt = make((40, 333), G=4, D=64, Hkv=1, dtype="f32", seed=41)
    q, k, v, cu = dev(bt)
    idx, cu_kept, _ = sgd.oam_select(q, k, v, cu, 4, 0.5, 1e-6, 3, 10, bt.lengths)
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, 4, 0.5, 1e-6, 3, 10)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, 2, 1)


def test_oam_ties_keep_lowest_indices(sgd):
    # q = 0 and every value row of the same norm: all scores equal -> tokens 0 .. K-1
    bt = make((100, 9, 1000), G=8, D=128, Hkv=2, seed=51)
    bt.q.zero_()
    bt.v[:] = 0
    bt.v[..., 0] = 2.0
    q, k, v, cu = dev(bt)
    idx, cu_kept, _ = sgd.oam_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, bt.lengths)
    assert cu_kept.tolist() == [0, 13, 15, 140]
    for h in range(2):
        assert idx[h, :13].tolist() == list(range(13))
        assert idx[h, 13:15].tolist() == [0, 1]
        assert idx[h, 15:].tolist() == list(range(125))


def test_oam_few_distinct_scores_take_the_radix_path(sgd):
    # q = 0 and value-row norms cycling through 1, 2, 4: three distinct scores spread apart, so the
    # threshold bin of the linear histogram holds thousands of keys and the exact radix select
    # decides; the kept set is the first K tokens of the top score, across all 8 CTAs of the row
    bt = make((20000, 7), G=4, D=64, Hkv=2, seed=52)
    bt.q.zero_()
    bt.v[:] = 0
    cu = bt.cu_seqlens.tolist()
    norms = torch.tensor([1.0, 2.0, 4.0])
    for h in range(2):
        for b in range(2):
            t = torch.arange(cu[b + 1] - cu[b])
            bt.v[h, cu[b]:cu[b + 1], 0] = norms[(t + h) % 3].to(bt.v.dtype)
    q, k, v, cu_d = dev(bt)
    idx, cu_kept, ws = sgd.oam_select(q, k, v, cu_d, 4, 1.0, 1e-6, 1, 8, bt.lengths)
    check_status(sgd, ws)
    assert cu_kept.tolist() == [0, 2500, 2501]
    for h in range(2):
        top = [t for t in range(20000) if (t + h) % 3 == 2][:2500]
        assert idx[h, :2500].tolist() == top
        assert idx[h, 2500:].tolist() == [[2, 1][h]]


def test_oam_long_row_beyond_the_shared_memory_stage(sgd):
    # 140000 tokens: each of the row's 8 CTAs holds more keys than it stages in shared memory,
    # so the rest is read again from global memory and the compaction works from the keys
    bt = make((140000, 300), G=8, D=128, Hkv=1, dist="outlier", seed=53)
    q, k, v, cu = dev(bt)
    idx, cu_kept, ws = sgd.oam_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, bt.lengths)
    check_status(sgd, ws)
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, 1.0, 1e-6, 1, 8)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, 2, 1)


def test_oam_keep_all_then_decode_equals_dense(sgd):
    bt = make((33, 700), G=8, D=128, Hkv=2, seed=61)
    q, k, v, cu = dev(bt)
    idx, cu_kept, _ = sgd.oam_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 1, bt.lengths)
    assert idx[0, :33].tolist() == list(range(33))
    dense = sgd.decode_attn(q, 8, k, v, cu)
    sel = sgd.decode_attn(q, 8, k, v, cu, idx=idx, cu_kept=cu_kept, kept_total_=idx.shape[1])
    assert (dense[0] - sel[0]).abs().max().item() <= 1e-5
    assert (dense[1] - sel[1]).abs().max().item() <= 1e-5


@pytest.mark.parametrize("kvdt", ["bf16", "int8A", "int8B"])
def test_oam_then_decode_over_kept(sgd, kvdt):
    bt = make((1, 90, 2000, 4500), G=8, D=128, Hkv=2, dist="outlier", seed=71)
    q, k, v, cu = dev(bt)
    idx, cu_kept, _ = sgd.oam_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, bt.lengths)
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, 1.0, 1e-6, 1, 8)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, 4, 2)
    Kt = idx.shape[1]
    if kvdt == "bf16":
        ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, idx=ref_idx, cu_kept=ref_cu)
        out, lse, ws = sgd.decode_attn(q, 8, k, v, cu, idx=idx, cu_kept=cu_kept, kept_total_=Kt)
    else:
        scheme = kvdt[-1]
        quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
        ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, idx=ref_idx, cu_kept=ref_cu, quant=(*quant, scheme))
        kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths)
        out, lse, ws = sgd.decode_attn(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme=scheme,
                                       n_parts_=sgd.n_parts(bt.lengths), idx=idx, cu_kept=cu_kept, kept_total_=Kt)
    assert_close(out, lse, *ref, OUT_TOL["bf16"])
    check_status(sgd, ws)


# ---------------------------------------------------------------------------------------------
# OAM over the INT8 cache: value norms stored at quantisation, scores on code * scale
# ---------------------------------------------------------------------------------------------
# fp32 sum of D exact squares: relative error below D * 2^-24; the square root halves it
VNORM_RTOL = 1e-5


@pytest.mark.parametrize("scheme", ["A", "B"])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 128), ("f32", 64)])
def test_quantize_writes_value_norms(sgd, scheme, dtype, D):
    bt = make((1, 63, 64, 65, 700, 2053), G=8, D=D, Hkv=2, dtype=dtype, dist="outlier", seed=21 + D)
    q, k, v, cu = dev(bt)
    vn = torch.full((2, int(bt.cu_seqlens[-1])), -1.0, dtype=torch.float32, device="cuda")
    _, _, _, _, ws = sgd.quantize_kv(k, v, cu, scheme, bt.lengths, v_norm=vn)
    check_status(sgd, ws)
    ref = oracle.value_norms(bt.v)
    rel = np.abs(vn.cpu().numpy() - ref) / np.maximum(ref, 1e-30)
    assert rel.max() <= VNORM_RTOL, rel.max()


def test_quantize_select_writes_the_same_value_norms(sgd):
    bt = make((7, 64, 500, 3000), G=8, D=128, Hkv=2, dist="outlier", seed=23)
    q, k, v, cu = dev(bt)
    T = int(bt.cu_seqlens[-1])
    vn1 = torch.empty((2, T), dtype=torch.float32, device="cuda")
    vn2 = torch.empty((2, T), dtype=torch.float32, device="cuda")
    sgd.quantize_kv(k, v, cu, "A", bt.lengths, v_norm=vn1)
    sgd.quantize_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, "A", bt.lengths, v_norm=vn2)
    assert torch.equal(vn1, vn2)


@pytest.mark.parametrize("scheme", ["A", "B"])
@pytest.mark.parametrize("G", [8, 16, 1])
def test_oam_select_over_the_int8_cache(sgd, scheme, G):
    bt = make((1, 7, 64, 500, 5000), G=G, D=128, Hkv=2, dist="outlier", seed=33 + G)
    q, k, v, cu = dev(bt)
    vn = torch.empty((2, int(bt.cu_seqlens[-1])), dtype=torch.float32, device="cuda")
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths, v_norm=vn)
    parts = sgd.n_parts(bt.lengths) if scheme == "A" else 0
    idx, cu_kept, ws = sgd.oam_select(q, kc, vc, cu, G, 1.0, 1e-6, 1, 8, bt.lengths, k_scale=ks, v_scale=vs,
                                      scheme=scheme, n_parts_=parts, v_norm=vn)
    check_status(sgd, ws)
    rkc, _, rks, _ = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
    ref_idx, ref_cu, scores = oracle.oam_select_int8(bt.q, rkc, rks, bt.v, bt.cu_seqlens, scheme, G, 1.0, 1e-6,
                                                     1, 8)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, bt.wl.B, 2)


def test_int8_cache_selection_then_decode(sgd):
    bt = make((90, 2000, 4500), G=8, D=128, Hkv=2, dist="outlier", seed=73)
    q, k, v, cu = dev(bt)
    vn = torch.empty((2, int(bt.cu_seqlens[-1])), dtype=torch.float32, device="cuda")
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths, v_norm=vn)
    parts = sgd.n_parts(bt.lengths)
    idx, cu_kept, _ = sgd.oam_select(q, kc, vc, cu, 8, 1.0, 1e-6, 1, 8, bt.lengths, k_scale=ks, v_scale=vs,
                                     scheme="A", n_parts_=parts, v_norm=vn)
    out, lse, ws = sgd.decode_attn(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A", n_parts_=parts, idx=idx,
                                   cu_kept=cu_kept, kept_total_=idx.shape[1])
    check_status(sgd, ws)
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    ref_idx, ref_cu, scores = oracle.oam_select_int8(bt.q, quant[0], quant[2], bt.v, bt.cu_seqlens, "A", 8, 1.0,
                                                     1e-6, 1, 8)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, 3, 2)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, idx=ref_idx, cu_kept=ref_cu, quant=(*quant, "A"))
    assert_close(out, lse, *ref, OUT_TOL["bf16"])


# ---------------------------------------------------------------------------------------------
# fused quantise + select
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("scheme", ["A", "B"])
@pytest.mark.parametrize("G,D,dtype", [(8, 128, "bf16"), (4, 64, "bf16"), (16, 128, "bf16"), (1, 128, "bf16"),
                                       (8, 128, "f32")])
def test_quantize_select_equals_separate_calls(sgd, scheme, G, D, dtype):
    bt = make((1, 63, 64, 65, 700, 4099), G=G, D=D, Hkv=3, dtype=dtype, dist="outlier", seed=91 + G + D)
    # exact rounding ties in partition 1 of sequence 5, head 2 (max |x| = 127: scale 1)
    s0 = int(bt.cu_seqlens[5])
    bt.k[2, s0 + 64:s0 + 128] = 0
    bt.k[2, s0 + 64:s0 + 80, :6] = torch.tensor([2.5, 3.5, -2.5, 126.5, 127.0, -0.5]).to(bt.k.dtype)
    q, k, v, cu = dev(bt)
    if dtype == "f32":
        q = q.float()
    fused = sgd.quantize_select(q, k, v, cu, G, 1.0, 1e-6, 1, 8, scheme, bt.lengths)
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths)
    idx, cu_kept, _ = sgd.oam_select(q, k, v, cu, G, 1.0, 1e-6, 1, 8, bt.lengths)
    for a, b in zip(fused[:6], (kc, vc, ks, vs, idx, cu_kept)):
        assert torch.equal(a, b)
    if scheme == "A":
        assert fused[0][2, s0 + 64, :6].tolist() == [2, 4, -2, 126, 127, 0]
    check_status(sgd, fused[6])
    rkc, rvc, rks, rvs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
    assert np.array_equal(fused[0].cpu().numpy(), rkc) and np.array_equal(fused[1].cpu().numpy(), rvc)
    assert np.array_equal(fused[2].cpu().numpy().reshape(rks.shape), rks)
    assert np.array_equal(fused[3].cpu().numpy(), rvs)
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, G, 1.0, 1e-6, 1, 8)
    check_selection(fused[4], fused[5].cpu(), ref_idx, ref_cu, scores, bt.wl.B, 3)


# ---------------------------------------------------------------------------------------------
# calibrated per-tensor scales ([TD] section 6, static quantisation): the given scale replaces
# max|x| / 127 and values beyond its range saturate; scales are fractions of the oracle's own
# computed ones, so frac < 1 makes the largest values saturate
# ---------------------------------------------------------------------------------------------
def _calibrated(bt, scheme, frac):
    _, _, rks, rvs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
    k_cal = np.float32(rks[0] * np.float32(frac)) if scheme == "B" else None
    return k_cal, np.float32(rvs[0] * np.float32(frac))


def _on_device(x):
    return None if x is None else torch.tensor([float(x)], dtype=torch.float32, device="cuda")


@pytest.mark.parametrize("frac", [1.0, 0.375])
@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 128)])
@pytest.mark.parametrize("scheme", ["A", "B"])
def test_quantize_calibrated_bit_exact(sgd, scheme, dtype, D, frac):
    bt = make((1, 63, 64, 65, 700, 4099), G=8, D=D, Hkv=3, dtype=dtype, dist="outlier", seed=131 + D)
    q, k, v, cu = dev(bt)
    T = int(bt.cu_seqlens[-1])
    k_cal, v_cal = _calibrated(bt, scheme, frac)
    vn = torch.empty((3, T), dtype=torch.float32, device="cuda")
    kc, vc, ks, vs, ws = sgd.quantize_kv(k, v, cu, scheme, bt.lengths, v_norm=vn, k_scale_in=_on_device(k_cal),
                                         v_scale_in=_on_device(v_cal))
    check_status(sgd, ws)
    rkc, rvc, rks, rvs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme, k_scale=k_cal, v_scale=v_cal)
    assert np.array_equal(kc.cpu().numpy(), rkc) and np.array_equal(vc.cpu().numpy(), rvc)
    assert np.array_equal(ks.cpu().numpy().reshape(rks.shape), rks) and vs.cpu().numpy()[0] == rvs[0]
    if frac < 1:
        assert (np.abs(rvc.astype(np.int32)) == 127).sum() > 10  # saturation exercised
    vn_dyn = torch.empty_like(vn)
    sgd.quantize_kv(k, v, cu, scheme, bt.lengths, v_norm=vn_dyn)
    assert torch.equal(vn, vn_dyn)


@pytest.mark.parametrize("G,D,dtype", [(8, 128, "bf16"), (16, 128, "bf16"), (4, 64, "bf16"), (8, 128, "f32")])
@pytest.mark.parametrize("scheme", ["A", "B"])
def test_quantize_select_calibrated(sgd, scheme, G, D, dtype):
    bt = make((1, 63, 64, 65, 700, 4099), G=G, D=D, Hkv=3, dtype=dtype, dist="outlier", seed=141 + G + D)
    s0 = int(bt.cu_seqlens[5])  # scheme A: exact rounding ties in one K partition (scale 1)
    bt.k[2, s0 + 64:s0 + 128] = 0
    bt.k[2, s0 + 64:s0 + 80, :6] = torch.tensor([2.5, 3.5, -2.5, 126.5, 127.0, -0.5]).to(bt.k.dtype)
    q, k, v, cu = dev(bt)
    if dtype == "f32":
        q = q.float()
    T = int(bt.cu_seqlens[-1])
    k_cal, v_cal = _calibrated(bt, scheme, 0.5)
    cal = dict(k_scale_in=_on_device(k_cal), v_scale_in=_on_device(v_cal))
    vn = torch.empty((3, T), dtype=torch.float32, device="cuda")
    fused = sgd.quantize_select(q, k, v, cu, G, 1.0, 1e-6, 1, 8, scheme, bt.lengths, v_norm=vn, **cal)
    check_status(sgd, fused[6])
    rkc, rvc, rks, rvs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme, k_scale=k_cal, v_scale=v_cal)
    assert np.array_equal(fused[0].cpu().numpy(), rkc) and np.array_equal(fused[1].cpu().numpy(), rvc)
    assert np.array_equal(fused[2].cpu().numpy().reshape(rks.shape), rks)
    assert fused[3].cpu().numpy()[0] == rvs[0]
    if scheme == "A":
        assert fused[0][2, s0 + 64, :6].tolist() == [2, 4, -2, 126, 127, 0]
    # the separate calibrated call gives the same bits; the kept sets and norms are the dynamic call's
    sep = sgd.quantize_kv(k, v, cu, scheme, bt.lengths, **cal)
    assert torch.equal(fused[0], sep[0]) and torch.equal(fused[1], sep[1]) and torch.equal(fused[2], sep[2])
    vn_dyn = torch.empty_like(vn)
    dyn = sgd.quantize_select(q, k, v, cu, G, 1.0, 1e-6, 1, 8, scheme, bt.lengths, v_norm=vn_dyn)
    assert torch.equal(fused[4], dyn[4]) and torch.equal(fused[5], dyn[5]) and torch.equal(vn, vn_dyn)
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, G, 1.0, 1e-6, 1, 8)
    check_selection(fused[4], fused[5].cpu(), ref_idx, ref_cu, scores, bt.wl.B, 3)


@pytest.mark.parametrize("call", ["quantize_kv", "quantize_select"])
def test_calibrated_scale_that_is_not_a_scale(sgd, call):
    bt = make((65, 700), G=8, D=128, Hkv=2, dist="outlier", seed=151)
    q, k, v, cu = dev(bt)
    for bad, status in ((-1.0, 0x10), (float("nan"), 0x10), (float("inf"), 0x10), (0.0, 0)):
        if call == "quantize_kv":
            kc, vc, ks, vs, ws = sgd.quantize_kv(k, v, cu, "A", bt.lengths, v_scale_in=_on_device(bad))
        else:
            kc, vc, ks, vs, _, _, ws = sgd.quantize_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, "A", bt.lengths,
                                                           v_scale_in=_on_device(bad))
        assert sgd.workspace_status(ws) == status, bad
        assert not vc.any() and kc.any()  # V codes zero, K codes (own partition scales) written


# ---------------------------------------------------------------------------------------------
# batches of many short sequences: hundreds of rows per CTA range, both schedules, the whole path
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("B", [256, 257, 300, 7000])
def test_batches_of_many_short_sequences(sgd, B):
    rng = np.random.default_rng(B)
    lengths = [int(x) for x in rng.integers(1, 260, size=B)]
    lengths[3] = 64  # a row of whole granules
    bt = make(lengths, G=8, D=128, Hkv=2, dist="outlier", seed=70 + B)
    q, k, v, cu = dev(bt)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8)
    for schedule, n_splits in ((0, 0), (0, 37), (1, 0)):
        out, lse, ws = sgd.decode_attn(q, 8, k, v, cu, schedule=schedule, n_splits=n_splits)
        assert_close(out, lse, *ref, OUT_TOL["bf16"])
        check_status(sgd, ws)
    idx, cu_kept, wss = sgd.oam_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 4, bt.lengths)
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, 1.0, 1e-6, 1, 4)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, B, 2)
    check_status(sgd, wss)
    kc, vc, ks, vs, idx2, cu2, wsq = sgd.quantize_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 4, "A", bt.lengths)
    check_status(sgd, wsq)
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    assert np.array_equal(kc.cpu().numpy(), quant[0]) and np.array_equal(ks.cpu().numpy(), quant[2])
    check_selection(idx2, cu2.cpu(), ref_idx, ref_cu, scores, B, 2)
    out, lse, ws = sgd.decode_attn(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                   n_parts_=sgd.n_parts(bt.lengths), idx=idx2, cu_kept=cu2, kept_total_=idx2.shape[1])
    check_status(sgd, ws)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, idx=idx2.cpu().numpy(), cu_kept=cu2.cpu().numpy(),
                        quant=(*quant, "A"))
    assert_close(out, lse, *ref, OUT_TOL["bf16"])


# ---------------------------------------------------------------------------------------------
# a mid-size batch: 32 rows of 700-31000 tokens over every SM, so rows span many CTA ranges and the
# row merges, the fused pass and the selection all run in the automatic split the bench uses
# ---------------------------------------------------------------------------------------------
MID_LENGTHS = (20000, 9001, 31000, 700)


def test_mid_size_decode_selection_and_fused_pass(sgd):
    bt = make(MID_LENGTHS, G=8, D=128, Hkv=8, dist="outlier", seed=404)
    q, k, v, cu = dev(bt)
    out, lse, ws = sgd.decode_attn(q, 8, k, v, cu)
    check_status(sgd, ws)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8)
    assert_close(out, lse, *ref, OUT_TOL["bf16"])
    kc, vc, ks, vs, idx, cu_kept, wsq = sgd.quantize_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, "A", bt.lengths)
    check_status(sgd, wsq)
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    for h in range(8):
        assert np.array_equal(kc[h].cpu().numpy(), quant[0][h]) and np.array_equal(vc[h].cpu().numpy(), quant[1][h])
    assert np.array_equal(ks.cpu().numpy(), quant[2]) and np.array_equal(vs.cpu().numpy(), quant[3])
    ref_idx, ref_cu, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, 1.0, 1e-6, 1, 8)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, bt.wl.B, 8)
    sidx, scu, wss = sgd.oam_select(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, bt.lengths)
    check_status(sgd, wss)
    check_selection(sidx, scu.cpu(), ref_idx, ref_cu, scores, bt.wl.B, 8)
    kw = dict(k_scale=ks, v_scale=vs, scheme="A", n_parts_=sgd.n_parts(bt.lengths))
    out, lse, ws = sgd.decode_attn(q, 8, kc, vc, cu, **kw)  # dense INT8
    check_status(sgd, ws)
    assert_close(out, lse, *oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, quant=(*quant, "A")), OUT_TOL["bf16"])
    out, lse, ws = sgd.decode_attn(q, 8, kc, vc, cu, idx=idx, cu_kept=cu_kept, kept_total_=idx.shape[1], **kw)
    check_status(sgd, ws)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, idx=idx.cpu().numpy(), cu_kept=cu_kept.cpu().numpy(),
                        quant=(*quant, "A"))
    assert_close(out, lse, *ref, OUT_TOL["bf16"])


def test_mid_size_with_column_groups(sgd):
    # four query tokens of G = 8: two CTAs per range, one per group of 16 (query token, head) columns
    bt = make_multi(MID_LENGTHS, M=4, G=8, Hkv=8, seed=405)
    q, k, v, cu = dev(bt)
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    out, lse, ws = sgd.decode_attn_multi(q, 8, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                         n_parts_=sgd.n_parts(bt.lengths))
    check_status(sgd, ws)
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    ref = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, 4, quant=(*quant, "A"))
    assert_close_multi(out, lse, *ref, OUT_TOL["bf16"])


# ---------------------------------------------------------------------------------------------
# device status reporting
# ---------------------------------------------------------------------------------------------
def test_empty_sequence_is_reported(sgd):
    bt = make((5, 40), G=8, D=128, Hkv=1, seed=81)
    q, k, v, _ = dev(bt)
    cu = torch.tensor([0, 5, 5, 45], dtype=torch.int32, device="cuda")  # sequence 1 is empty
    q3 = torch.cat([q[:1], q[:1], q[1:]])
    out, lse, ws = sgd.decode_attn(q3, 8, k, v, cu)
    assert sgd.workspace_status(ws) & 0x1
    assert torch.isinf(lse[1]).all() and (out[1] == 0).all()


# ---------------------------------------------------------------------------------------------
# multi-token (speculative) decode: M query tokens per sequence, causal over the last M entries
# ---------------------------------------------------------------------------------------------
def make_multi(lengths, M, G, D=128, Hkv=2, dist="outlier", seed=0):
    wl = workloads.Workload("t-multi", B=len(lengths), Hkv=Hkv, G=G, D=D, kv_dtype="bf16", dist=dist,
                            lengths=tuple(lengths), M=M)
    return workloads.generate(wl, seed)


def assert_close_multi(out, lse, ref_out, ref_lse, tol):
    """Queries that see no token: exactly out 0 and lse -inf; the rest as assert_close."""
    o, l = out.double().cpu().numpy(), lse.double().cpu().numpy()
    blind = np.isneginf(ref_lse)
    assert np.isneginf(l[blind]).all() and (o[blind] == 0).all()
    seen = ~blind
    scale = np.abs(ref_out[seen]).max()
    err = np.abs(o[seen] - ref_out[seen]).max()
    lerr = np.abs(l[seen] - ref_lse[seen]).max()
    assert err <= tol * scale, f"out error {err:.3e} > {tol} * {scale:.3e}"
    assert lerr <= LSE_TOL, f"lse error {lerr:.3e}"


def kept_with_tail(lengths, Hkv, M, seed):
    """A seeded kept set per (sequence, KV head): a random eighth of the positions plus the last
    M (so the causal limit cuts through kept tokens), ascending."""
    rng = np.random.default_rng(seed)
    rows, counts = {}, []
    for b, L in enumerate(lengths):
        K = max(min(L, M), (L + 7) // 8)
        counts.append(K)
        for h in range(Hkv):
            tail = np.arange(max(0, L - M), L)
            rest = np.setdiff1d(np.arange(L), tail)
            pick = rng.choice(rest, size=K - tail.size, replace=False) if K > tail.size else []
            rows[(b, h)] = np.sort(np.concatenate([tail, pick]).astype(np.int32))
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    idx = np.zeros((Hkv, int(cu[-1])), np.int32)
    for (b, h), r in rows.items():
        idx[h, cu[b]:cu[b + 1]] = r
    return idx, cu


@pytest.mark.parametrize("kvdt", ["bf16", "int8A"])
@pytest.mark.parametrize("M,G", [(2, 8), (4, 4), (16, 1), (4, 8), (3, 16), (8, 8)])
@pytest.mark.parametrize("indexed", [False, True])
def test_multi_token_decode(sgd, kvdt, M, G, indexed):
    # up to 16 columns (M * G) one CTA per range; 32, 48 and 64 columns: 2, 3 and 4 CTAs per range
    lengths = (1, 3, 70, 700, 3001)
    bt = make_multi(lengths, M, G, seed=31 + M)
    q, k, v, cu = dev(bt)
    sel, extra = {}, {}
    if indexed:
        idx, cu_kept = kept_with_tail(lengths, 2, M, seed=7)
        sel = dict(idx=idx, cu_kept=cu_kept)
        extra = dict(idx=torch.from_numpy(idx).cuda(), cu_kept=torch.from_numpy(cu_kept).cuda(),
                     kept_total_=idx.shape[1])
    quant, kw = None, {}
    kk, vv = k, v
    if kvdt == "int8A":
        quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A"), "A")
        kk, vv, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
        kw = dict(k_scale=ks, v_scale=vs, scheme="A", n_parts_=sgd.n_parts(bt.lengths))
    ref = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, G, M, quant=quant, **sel)
    for n_splits in (0, 7, 300):
        out, lse, ws = sgd.decode_attn_multi(q, G, kk, vv, cu, n_splits=n_splits, **kw, **extra)
        assert_close_multi(out, lse, *ref, OUT_TOL["bf16"])
        check_status(sgd, ws)


@pytest.mark.parametrize("D", [64, 128])
def test_multi_token_bf16_head_dims_and_one_token_equals_decode(sgd, D):
    bt = make_multi((5, 129, 1000), 2, 8, D=D, dist="normal", seed=3)
    q, k, v, cu = dev(bt)
    ref = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, 8, 2)
    out, lse, _ = sgd.decode_attn_multi(q, 8, k, v, cu)
    assert_close_multi(out, lse, *ref, OUT_TOL["bf16"])
    # M = 1 through the multi entry is the single-token decode, bit for bit
    q1 = q[:, :1].contiguous()
    o1, l1, _ = sgd.decode_attn_multi(q1, 8, k, v, cu)
    o0, l0, _ = sgd.decode_attn(q1[:, 0].contiguous(), 8, k, v, cu)
    assert torch.equal(o1[:, 0], o0) and torch.equal(l1[:, 0], l0)


def test_multi_token_with_query_codes(sgd):
    M, G = 2, 8
    lengths = (2, 90, 2500)
    bt = make_multi(lengths, M, G, seed=77)
    q, k, v, cu = dev(bt)
    quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A"), "A")
    qd = oracle.dequant_q(*oracle.quantize_q(bt.q.reshape(len(lengths) * M, 2 * G, 128), "token"))
    ref = oracle.decode_multi(qd.reshape(len(lengths), M, 2 * G, 128), bt.k, bt.v, bt.cu_seqlens, G, M, quant=quant)
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    out, lse, ws = sgd.decode_attn_multi(q, G, kc, vc, cu, k_scale=ks, v_scale=vs, scheme="A",
                                         n_parts_=sgd.n_parts(bt.lengths), n_splits=9, q_quant="token")
    assert_close_multi(out, lse, *ref, OUT_TOL["bf16"])
    check_status(sgd, ws)


# ---------------------------------------------------------------------------------------------
# block-granular selection (64-token blocks ranked by their best token) and decode over blocks
# ---------------------------------------------------------------------------------------------
BLOCK_LENGTHS = (1, 64, 65, 130, 700, 4099)


@pytest.mark.parametrize("cache", ["bf16", "int8A", "int8B"])
@pytest.mark.parametrize("G,D", [(8, 128), (4, 64)])
def test_block_selection_matches_oracle(sgd, cache, G, D):
    bt = make(BLOCK_LENGTHS, G=G, D=D, Hkv=2, dist="outlier", seed=41 + G)
    q, k, v, cu = dev(bt)
    if cache != "bf16" and D != 128:
        # the INT8 cache is scored at D = 128 only: the call is rejected on the host
        scheme = cache[-1]
        vn = torch.empty((2, bt.T), dtype=torch.float32, device="cuda")
        kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths, v_norm=vn)
        with pytest.raises(sgd.SgdError, match=r"\(-3\)"):
            sgd.oam_select_blocks(q, kc, vc, cu, G, 1.0, 1e-6, 1, 4, bt.lengths, k_scale=ks, v_scale=vs,
                                  scheme=scheme, n_parts_=sgd.n_parts(bt.lengths), v_norm=vn)
        return
    if cache == "bf16":
        blk, cu_kb, ws = sgd.oam_select_blocks(q, k, v, cu, G, 1.0, 1e-6, 1, 4, bt.lengths)
        _, _, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, G, 1.0, 1e-6, 1, 4)
    else:
        scheme = cache[-1]
        vn = torch.empty((2, bt.T), dtype=torch.float32, device="cuda")
        kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths, v_norm=vn)
        blk, cu_kb, ws = sgd.oam_select_blocks(q, kc, vc, cu, G, 1.0, 1e-6, 1, 4, bt.lengths, k_scale=ks,
                                               v_scale=vs, scheme=scheme, n_parts_=sgd.n_parts(bt.lengths),
                                               v_norm=vn)
        rkc, _, rks, _ = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
        _, _, scores = oracle.oam_select_int8(bt.q, rkc, rks, bt.v, bt.cu_seqlens, scheme, G, 1.0, 1e-6, 1, 4)
    ref_blk, ref_cu, bscores = oracle.select_blocks(scores, bt.cu_seqlens, 2, 1, 4)
    check_selection(blk, cu_kb.cpu(), ref_blk, ref_cu, bscores, bt.wl.B, 2)
    check_status(sgd, ws)


@pytest.mark.parametrize("cache", ["bf16", "int8A", "int8B"])
@pytest.mark.parametrize("G,D", [(8, 128), (16, 128), (4, 64)])
def test_decode_over_blocks_matches_oracle(sgd, cache, G, D):
    bt = make(BLOCK_LENGTHS, G=G, D=D, Hkv=2, dist="outlier", seed=43 + G)
    q, k, v, cu = dev(bt)
    if cache != "bf16" and D != 128:
        # kept blocks of an INT8 cache decode on the tensor cores at D = 128 only: rejected on the host
        scheme = cache[-1]
        kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths)
        tb = torch.zeros((2, bt.wl.B), dtype=torch.int32, device="cuda")
        tcu = torch.arange(bt.wl.B + 1, dtype=torch.int32, device="cuda")
        with pytest.raises(sgd.SgdError, match=r"\(-3\)"):
            sgd.decode_attn_blocks(q, G, kc, vc, cu, tb, tcu, k_scale=ks, v_scale=vs, scheme=scheme,
                                   n_parts_=sgd.n_parts(bt.lengths))
        return
    # a seeded kept-block set: a quarter of each row's blocks, always with its ragged last block
    rng = np.random.default_rng(5)
    nb = [-(-int(L) // 64) for L in BLOCK_LENGTHS]
    keep = [max(1, -(-n // 4)) for n in nb]
    cu_kb = np.concatenate([[0], np.cumsum(keep)]).astype(np.int32)
    blk = np.zeros((2, int(cu_kb[-1])), np.int32)
    for b, (n, K) in enumerate(zip(nb, keep)):
        for h in range(2):
            pick = rng.choice(n - 1, size=K - 1, replace=False) if K > 1 else []
            blk[h, cu_kb[b]:cu_kb[b + 1]] = np.sort(np.concatenate([pick, [n - 1]])).astype(np.int32)
    quant, kw, kk, vv = None, {}, k, v
    if cache != "bf16":
        scheme = cache[-1]
        quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme), scheme)
        kk, vv, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths)
        kw = dict(k_scale=ks, v_scale=vs, scheme=scheme, n_parts_=sgd.n_parts(bt.lengths))
    ref = oracle.decode_blocks(bt.q, bt.k, bt.v, bt.cu_seqlens, G, blk, cu_kb, quant=quant)
    tb, tcu = torch.from_numpy(blk).cuda(), torch.from_numpy(cu_kb).cuda()
    for n_splits in (0, 7, 300):
        out, lse, ws = sgd.decode_attn_blocks(q, G, kk, vv, cu, tb, tcu, n_splits=n_splits, **kw)
        assert_close(out, lse, *ref, OUT_TOL["bf16"])
        check_status(sgd, ws)
    # every block kept: the dense decode
    allb = np.concatenate([np.arange(n, dtype=np.int32) for n in nb])
    cu_all = np.concatenate([[0], np.cumsum(nb)]).astype(np.int32)
    tall = torch.from_numpy(np.stack([allb, allb])).cuda()
    out, lse, _ = sgd.decode_attn_blocks(q, G, kk, vv, cu, tall, torch.from_numpy(cu_all).cuda(), **kw)
    dense = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, G, quant=quant)
    assert_close(out, lse, *dense, OUT_TOL["bf16"])


def test_decode_over_blocks_reports_a_block_number_out_of_range(sgd):
    bt = make((130, 300), G=8, D=128, Hkv=1, seed=3)
    q, k, v, cu = dev(bt)
    blk = torch.tensor([[0, 7, 1]], dtype=torch.int32, device="cuda")  # sequence 0 has blocks 0..2
    cu_kb = torch.tensor([0, 2, 3], dtype=torch.int32, device="cuda")
    out, lse, ws = sgd.decode_attn_blocks(q, 8, k, v, cu, blk, cu_kb)
    assert sgd.workspace_status(ws) & 0x8  # bad index
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()


def test_kernel_timing_brackets_each_launch(sgd):
    bt = make((700, 3000), G=8, D=128, Hkv=2, seed=2)
    q, k, v, cu = dev(bt)
    sgd.decode_attn(q, 8, k, v, cu)  # warm
    torch.cuda.synchronize()
    sgd.kernel_timing_start(8)
    out, lse, _ = sgd.decode_attn(q, 8, k, v, cu)
    got = sgd.kernel_timing_stop()
    assert [("plan_" in n and "_kernel" in n, "decode_mma_kernel" in n) for n, _ in got] == [(True, False), (False, True)]
    assert all(ms > 0 for _, ms in got)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 8)
    assert_close(out, lse, *ref, OUT_TOL["bf16"])
    # off again: nothing more is recorded
    sgd.decode_attn(q, 8, k, v, cu)
    sgd.kernel_timing_start(1)
    assert sgd.kernel_timing_stop() == []


@pytest.mark.parametrize("cache", ["bf16", "int8A"])
@pytest.mark.parametrize("M,G", [(2, 8), (4, 4), (2, 4)])
def test_multi_token_selection_then_decode(sgd, cache, M, G):
    # one kept set for the M query tokens (group max over M * G rows), then the causal multi-token
    # decode over it; the decode is checked on the oracle's own selection
    lengths = (5, 300, 2500)
    bt = make_multi(lengths, M, G, seed=61 + M)
    q, k, v, cu = dev(bt)
    kw, kk, vv, quant, vn = {}, k, v, None, None
    if cache == "int8A":
        vn = torch.empty((2, bt.T), dtype=torch.float32, device="cuda")
        kk, vv, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths, v_norm=vn)
        kw = dict(k_scale=ks, v_scale=vs, scheme="A", n_parts_=sgd.n_parts(bt.lengths))
        quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A"), "A")
    idx, cu_kept, ws = sgd.oam_select_multi(q, kk, vv, cu, G, 1.0, 1e-6, 1, 8, bt.lengths, v_norm=vn, **kw)
    check_status(sgd, ws)
    if cache == "bf16":
        ref_idx, ref_cu, scores = oracle.oam_select_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, G, M, 1.0, 1e-6, 1, 8)
    else:  # scored on code * scale: the oracle's dequantised keys, the unquantised value norms
        khat = torch.from_numpy(np.stack([oracle.dequant_rows(quant[0][h], np.concatenate(
            [oracle.k_scale_of_tokens(quant[2], "A", h, b, L, np.concatenate([[0], np.cumsum(oracle.n_parts(lengths))]))
             for b, L in enumerate(lengths)])) for h in range(2)]))
        ref_idx, ref_cu, scores = oracle.oam_select_multi(bt.q, khat, bt.v, bt.cu_seqlens, G, M, 1.0, 1e-6, 1, 8)
    check_selection(idx, cu_kept.cpu(), ref_idx, ref_cu, scores, len(lengths), 2)
    ref = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, G, M, idx=ref_idx, cu_kept=ref_cu, quant=quant)
    out, lse, ws = sgd.decode_attn_multi(q, G, kk, vv, cu, idx=torch.from_numpy(ref_idx).cuda(),
                                         cu_kept=torch.from_numpy(ref_cu).cuda(), kept_total_=ref_idx.shape[1], **kw)
    assert_close_multi(out, lse, *ref, OUT_TOL["bf16"])
    check_status(sgd, ws)


@pytest.mark.parametrize("mode", ["token", "tensor"])
def test_decode_over_blocks_with_query_codes(sgd, mode):
    lengths = (64, 130, 3001)
    bt = make(lengths, G=8, D=128, Hkv=2, dist="outlier", seed=57)
    q, k, v, cu = dev(bt)
    nb = [-(-L // 64) for L in lengths]
    keep = [1, 2, 12]
    cu_kb = np.concatenate([[0], np.cumsum(keep)]).astype(np.int32)
    rng = np.random.default_rng(9)
    blk = np.zeros((2, int(cu_kb[-1])), np.int32)
    for b, (n, K) in enumerate(zip(nb, keep)):
        for h in range(2):
            blk[h, cu_kb[b]:cu_kb[b + 1]] = np.sort(rng.choice(n, size=K, replace=False))
    quant = (*oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A"), "A")
    qd = oracle.dequant_q(*oracle.quantize_q(bt.q, mode))
    ref = oracle.decode_blocks(qd, bt.k, bt.v, bt.cu_seqlens, 8, blk, cu_kb, quant=quant)
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, "A", bt.lengths)
    out, lse, ws = sgd.decode_attn_blocks(q, 8, kc, vc, cu, torch.from_numpy(blk).cuda(), torch.from_numpy(cu_kb).cuda(),
                                          k_scale=ks, v_scale=vs, scheme="A", n_parts_=sgd.n_parts(bt.lengths),
                                          n_splits=11, q_quant=mode)
    assert_close(out, lse, *ref, OUT_TOL["bf16"])
    check_status(sgd, ws)


# ---------------------------------------------------------------------------------------------
# measurement aids: the read-only stream and the scattered-row read fold every byte they read
# ---------------------------------------------------------------------------------------------
def _xor_words(x: np.ndarray) -> int:
    return int(np.bitwise_xor.reduce(x.view(np.uint32).ravel())) if x.size else 0


@pytest.mark.parametrize("method", [0, 1])
def test_stream_read_folds_every_byte(sgd, method):
    rng = np.random.default_rng(3 + method)
    host = rng.integers(0, 256, size=(3 << 20) + 4096, dtype=np.uint8)  # not a whole number of chunks
    buf = torch.from_numpy(host).cuda()
    sink, status = sgd.stream_read(buf, method)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert (int(sink.item()) & 0xffffffff) == _xor_words(host)


def test_gather_read_folds_the_listed_rows(sgd):
    rng = np.random.default_rng(11)
    a = rng.integers(0, 256, size=(5000, 128), dtype=np.uint8)
    b = rng.integers(0, 256, size=(5000, 128), dtype=np.uint8)
    rows = rng.integers(0, 5000, size=9999).astype(np.int32)  # repeats allowed; a ragged last batch
    da, db, dr = (torch.from_numpy(x).cuda() for x in (a, b, rows))
    sink = sgd.gather_read(da, dr, 128, b=db)
    torch.cuda.synchronize()
    assert (int(sink.item()) & 0xffffffff) == _xor_words(np.concatenate([a[rows], b[rows]]))
    sink1 = sgd.gather_read(da, dr[:7], 128)
    torch.cuda.synchronize()
    assert (int(sink1.item()) & 0xffffffff) == _xor_words(a[rows[:7]])
    for row_bytes in (16, 4096):  # the smallest and the largest rows
        flat = rng.integers(0, 256, size=row_bytes * 300, dtype=np.uint8)
        rr = rng.integers(0, 300, size=517).astype(np.int32)
        s2 = sgd.gather_read(torch.from_numpy(flat).cuda(), torch.from_numpy(rr).cuda(), row_bytes)
        torch.cuda.synchronize()
        assert (int(s2.item()) & 0xffffffff) == _xor_words(flat.reshape(300, row_bytes)[rr]), row_bytes
    with pytest.raises(ValueError):
        sgd.gather_read(da, torch.tensor([5000], dtype=torch.int32, device="cuda"), 128)


# ---------------------------------------------------------------------------------------------
# quantise and select in one call for several query tokens, or by 64-token blocks: the same codes,
# scales and norms as sgd_quantize_kv and the same kept sets as oam_select_multi / _blocks, which
# are checked against the oracle
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("scheme", ["A", "B", "B-calibrated"])
@pytest.mark.parametrize("M,G", [(2, 8), (4, 4), (2, 4), (16, 1)])
def test_quantize_select_multi_equals_separate_calls(sgd, scheme, M, G):
    lengths = (5, 64, 300, 2500)
    bt = make_multi(lengths, M, G, seed=71 + M + G)
    q, k, v, cu = dev(bt)
    base, cal = scheme[0], {}
    if scheme.endswith("calibrated"):
        k_cal, v_cal = _calibrated(bt, base, 0.5)
        cal = dict(k_scale_in=_on_device(k_cal), v_scale_in=_on_device(v_cal))
    scheme = base
    vn = torch.empty((2, bt.T), dtype=torch.float32, device="cuda")
    fused = sgd.quantize_select_multi(q, k, v, cu, G, 1.0, 1e-6, 1, 8, scheme, bt.lengths, v_norm=vn, **cal)
    check_status(sgd, fused[6])
    vn2 = torch.empty_like(vn)
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, scheme, bt.lengths, v_norm=vn2, **cal)
    idx, cu_kept, _ = sgd.oam_select_multi(q, k, v, cu, G, 1.0, 1e-6, 1, 8, bt.lengths)
    for a, b in zip(fused[:6], (kc, vc, ks, vs, idx, cu_kept)):
        assert torch.equal(a, b)
    assert torch.equal(vn, vn2)
    okw = {} if not cal else dict(k_scale=k_cal, v_scale=v_cal)
    rkc, rvc, rks, rvs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme, **okw)
    assert np.array_equal(fused[0].cpu().numpy(), rkc) and np.array_equal(fused[1].cpu().numpy(), rvc)
    ref_idx, ref_cu, scores = oracle.oam_select_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, G, M, 1.0, 1e-6, 1, 8)
    check_selection(fused[4], fused[5].cpu(), ref_idx, ref_cu, scores, len(lengths), 2)


@pytest.mark.parametrize("scheme", ["A", "B", "A-calibrated"])
@pytest.mark.parametrize("G,D", [(8, 128), (4, 64), (16, 128)])
def test_quantize_select_blocks_equals_separate_calls(sgd, scheme, G, D):
    bt = make(BLOCK_LENGTHS, G=G, D=D, Hkv=2, dist="outlier", seed=81 + G + D)
    q, k, v, cu = dev(bt)
    base = scheme[0]
    cal = {}
    if scheme.endswith("calibrated"):
        cal = dict(v_scale_in=_on_device(_calibrated(bt, base, 0.5)[1]))
    fused = sgd.quantize_select_blocks(q, k, v, cu, G, 1.0, 1e-6, 1, 4, base, bt.lengths, **cal)
    check_status(sgd, fused[6])
    kc, vc, ks, vs, _ = sgd.quantize_kv(k, v, cu, base, bt.lengths, **cal)
    blk, cu_kb, _ = sgd.oam_select_blocks(q, k, v, cu, G, 1.0, 1e-6, 1, 4, bt.lengths)
    for a, b in zip(fused[:6], (kc, vc, ks, vs, blk, cu_kb)):
        assert torch.equal(a, b)
    _, _, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, G, 1.0, 1e-6, 1, 4)
    ref_blk, ref_cu, bscores = oracle.select_blocks(scores, bt.cu_seqlens, 2, 1, 4)
    check_selection(fused[4], fused[5].cpu(), ref_blk, ref_cu, bscores, bt.wl.B, 2)


def test_quantize_select_multi_rejects_too_many_columns(sgd):
    bt = make_multi((64, 300), 4, 8, seed=5)  # M * G = 32 > 16
    q, k, v, cu = dev(bt)
    with pytest.raises(sgd.SgdError):  # the workspace query already refuses 32 columns
        sgd.quantize_select_multi(q, k, v, cu, 8, 1.0, 1e-6, 1, 8, "A", bt.lengths)
