"""Pins of the fp64 oracle to things other than itself: closed forms, library routines,
invariants, hand-derived worked examples (tests/golden/) and brute force on tiny inputs.

Each group names the oracle function it pins.  tests/test_oracle_mutants.py plants plausible
mistakes into copies of the oracle and checks that these pins catch every one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.filterwarnings("ignore")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------------------
# attend: softmax attention of G heads over n tokens
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("G,D,n", [(1, 8, 1), (4, 8, 16), (3, 16, 37), (8, 64, 5)])
def test_attend_matches_torch_sdpa(G, D, n):
    q, k, v = _rand((G, D), 1), _rand((n, D), 2), _rand((n, D), 3)
    out, lse = oracle.attend(q, k, v)
    tq, tk, tv = (torch.from_numpy(a) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq[None], tk[None], tv[None])[0]
    ref_lse = torch.logsumexp(tq @ tk.T / math.sqrt(D), dim=-1)
    assert np.allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


def test_attend_identical_keys_gives_mean_of_v():
    # every logit equals z = q.k/sqrt(D): weights 1/n, out = mean(v), lse = z + ln n
    G, D, n = 4, 16, 23
    q, v = _rand((G, D), 4), _rand((n, D), 5)
    k1 = _rand((1, D), 6)
    out, lse = oracle.attend(q, np.repeat(k1, n, axis=0), v)
    assert np.allclose(out, np.broadcast_to(v.mean(axis=0), (G, D)), atol=1e-13)
    z = (q @ k1[0]) / math.sqrt(D)
    assert np.allclose(lse, z + math.log(n), atol=1e-13)


def test_attend_one_token_returns_its_value():
    G, D = 4, 32
    q, k, v = _rand((G, D), 7), _rand((1, D), 8), _rand((1, D), 9)
    out, lse = oracle.attend(q, k, v)
    assert np.array_equal(out, np.broadcast_to(v[0], (G, D)))
    assert np.allclose(lse, q @ k[0] / math.sqrt(D), atol=1e-14)


def test_attend_two_tokens_closed_form():
    # two tokens: weight of token 0 is the logistic function of the logit difference
    D = 4
    q = np.array([[1.0, 0.0, 0.0, 0.0]])
    k = np.array([[2.0, 0, 0, 0], [0.0, 0, 0, 0]])  # logits 1 and 0
    v = np.array([[1.0, 0, 0, 0], [0.0, 1, 0, 0]])
    out, lse = oracle.attend(q, k, v)
    w0 = math.e / (math.e + 1.0)
    assert np.allclose(out[0], [w0, 1 - w0, 0, 0], atol=1e-15)
    assert abs(lse[0] - math.log(math.e + 1.0)) < 1e-15


def test_attend_permutation_invariance_and_v_linearity():
    G, D, n = 2, 8, 19
    q, k, v = _rand((G, D), 10), _rand((n, D), 11), _rand((n, D), 12)
    out, lse = oracle.attend(q, k, v)
    p = np.random.default_rng(13).permutation(n)
    out_p, lse_p = oracle.attend(q, k[p], v[p])
    assert np.allclose(out, out_p, atol=1e-13) and np.allclose(lse, lse_p, atol=1e-13)
    out2, lse2 = oracle.attend(q, k, 3.0 * v)
    assert np.allclose(out2, 3.0 * out, atol=1e-13) and np.array_equal(lse, lse2)


def test_attend_rejects_empty():
    with pytest.raises(ValueError):
        oracle.attend(np.ones((1, 4)), np.ones((0, 4)), np.ones((0, 4)))


# ---------------------------------------------------------------------------------------------
# decode: GQA head mapping (query head h -> KV head h // G), G = 1 is MHA
# ---------------------------------------------------------------------------------------------
def _tiny_batch(G, D=16, lengths=(7, 30, 1), Hkv=2, seed=0, dtype="f32"):
    wl = workloads.Workload("tiny", B=len(lengths), Hkv=Hkv, G=G, D=D, kv_dtype=dtype,
                            dist="normal", lengths=tuple(lengths))
    return workloads.generate(wl, seed)


@pytest.mark.parametrize("G", [1, 4])
def test_decode_matches_sdpa_with_repeat_interleave(G):
    bt = _tiny_batch(G)
    out, lse = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, G)
    cu = bt.cu_seqlens.numpy()
    for b in range(bt.wl.B):
        s, e = int(cu[b]), int(cu[b + 1])
        kk = bt.k[:, s:e].double().repeat_interleave(G, dim=0)  # [Hq, L, D], [AO] GQA example
        vv = bt.v[:, s:e].double().repeat_interleave(G, dim=0)
        qq = bt.q[b].double()[:, None, :]  # [Hq, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, 0]
        assert np.allclose(out[b], ref.numpy(), atol=1e-12)
        ref_lse = torch.logsumexp((qq @ kk.transpose(1, 2))[:, 0] / math.sqrt(bt.wl.D), dim=-1)
        assert np.allclose(lse[b], ref_lse.numpy(), atol=1e-12)


def test_gqa_example_numbers(golden_dir):
    g = _load(golden_dir, "gqa_example.json")
    H, Hkv, D, L = g["num_heads"], g["num_kv_heads"], g["head_dim"], g["seq_len"]
    assert 2 * H * D * L == g["mha_cache_entries"]
    assert 2 * Hkv * D * L == g["gqa_cache_entries"]
    assert round(100 * (1 - g["gqa_cache_entries"] / g["mha_cache_entries"])) == g["saving_percent"]
    # our layout: k, v [Hkv, T, D] hold exactly the GQA cache entries
    bt = _tiny_batch(G=H // Hkv, D=D, lengths=(L,), Hkv=Hkv)
    assert bt.k.numel() + bt.v.numel() == g["gqa_cache_entries"]
    # and head h reads KV head h // G, as repeat_interleave does
    G = g["heads_per_group"]
    mapping = torch.arange(Hkv).repeat_interleave(G).tolist()
    assert mapping == g["kv_head_of_query_head"] == [h // G for h in range(H)]


# ---------------------------------------------------------------------------------------------
# merge: split = unsplit for every chunking
# ---------------------------------------------------------------------------------------------
def test_merge_single_chunk_is_identity():
    o, l = _rand((1, 3, 5), 20), _rand((1, 3), 21)
    out, lse = oracle.merge(o, l)
    assert np.allclose(out, o[0], atol=1e-15) and np.allclose(lse, l[0], atol=1e-15)


@pytest.mark.parametrize("n", [1, 2, 7, 13])
def test_merge_of_every_chunking_equals_unsplit(n):
    G, D = 3, 8
    q, k, v = _rand((G, D), 30 + n), _rand((n, D), 31 + n, 2.0), _rand((n, D), 32 + n)
    ref_out, ref_lse = oracle.attend(q, k, v)
    # every composition of n into contiguous chunks (2^(n-1) of them) for small n
    cuts_all = range(1, n)
    for r in range(0, n):
        for cuts in itertools.combinations(cuts_all, r):
            bounds = [0, *cuts, n]
            parts = [oracle.attend(q, k[a:b], v[a:b]) for a, b in zip(bounds[:-1], bounds[1:])]
            out, lse = oracle.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
            assert np.allclose(out, ref_out, atol=1e-12) and np.allclose(lse, ref_lse, atol=1e-12)


def test_merge_random_chunkings_long_row():
    G, D, n = 4, 16, 500
    q, k, v = _rand((G, D), 40), _rand((n, D), 41, 3.0), _rand((n, D), 42)
    ref_out, ref_lse = oracle.attend(q, k, v)
    rng = np.random.default_rng(43)
    for trial in range(20):
        cuts = np.sort(rng.choice(np.arange(1, n), size=rng.integers(1, 30), replace=False))
        bounds = [0, *cuts.tolist(), n]
        parts = [oracle.attend(q, k[a:b], v[a:b]) for a, b in zip(bounds[:-1], bounds[1:])]
        out, lse = oracle.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        assert np.allclose(out, ref_out, atol=1e-12) and np.allclose(lse, ref_lse, atol=1e-12)


def test_printed_merge_update_without_chunk_factor_is_not_exact():
    """The page's printed out-update lacks exp(m_chunk - m_new) on the chunk term; written out
    literally it disagrees with unsplit attention, which is why the oracle merges in LSE form."""
    G, D, n = 1, 8, 40
    q, k, v = _rand((G, D), 50), _rand((n, D), 51, 2.0), _rand((n, D), 52)
    ref_out, _ = oracle.attend(q, k, v)
    (o1, l1), (o2, l2) = oracle.attend(q, k[:20], v[:20]), oracle.attend(q, k[20:], v[20:])
    # per chunk: m = chunk max logit, exp_sum = sum exp(z - m) = exp(lse - m)
    z1 = (q @ k[:20].T)[0] / math.sqrt(D)
    z2 = (q @ k[20:].T)[0] / math.sqrt(D)
    m1, m2 = z1.max(), z2.max()
    s1, s2 = math.exp(l1[0] - m1), math.exp(l2[0] - m2)
    m_new = max(m1, m2)
    exp_sum = math.exp(m1 - m_new) * s1 + math.exp(m2 - m_new) * s2
    printed = (math.exp(m1 - m_new) * o1[0] * s1 + o2[0] * s2) / exp_sum
    restored = (math.exp(m1 - m_new) * o1[0] * s1 + math.exp(m2 - m_new) * o2[0] * s2) / exp_sum
    assert np.allclose(restored, ref_out[0], atol=1e-12)
    assert not np.allclose(printed, ref_out[0], atol=1e-6)


# ---------------------------------------------------------------------------------------------
# quantisation
# ---------------------------------------------------------------------------------------------
def test_quantize_worked_cases(golden_dir):
    for grp in _load(golden_dir, "quantize_worked_cases.json")["groups"]:
        x = np.array(grp["values"], np.float32)
        s = oracle.scale_from_amax(oracle.amax(x))
        assert s == np.float32(grp["scale"])
        assert oracle.quantize(x, s).tolist() == grp["codes"]


def test_quantize_clamps_to_127(golden_dir):
    c = _load(golden_dir, "quantize_worked_cases.json")["clamp"]
    assert oracle.quantize(np.array(c["values"], np.float32), c["scale"]).tolist() == c["codes"]


def test_quantize_matches_numpy_float32_route():
    # independent route: numpy's IEEE float32 division and round-half-even
    rng = np.random.default_rng(60)
    for trial in range(20):
        x = (rng.standard_normal(4096) * rng.lognormal(0, 2)).astype(np.float32)
        s = oracle.scale_from_amax(oracle.amax(x))
        assert s == np.float32(np.abs(x).max()) / np.float32(127.0)
        ref = np.clip(np.rint(x / s), -127, 127).astype(np.int8)
        assert np.array_equal(oracle.quantize(x, s), ref)


def test_quantize_amax_element_maps_to_127_and_bounds():
    rng = np.random.default_rng(61)
    for trial in range(50):
        x = (rng.standard_normal(257) * 10 ** rng.uniform(-30, 30)).astype(np.float32)
        s = oracle.scale_from_amax(oracle.amax(x))
        c = oracle.quantize(x, s)
        i = int(np.argmax(np.abs(x)))
        assert c[i] == (127 if x[i] > 0 else -127)
        assert c.min() >= -127 and c.max() <= 127
        err = np.abs(x.astype(np.float64) - c.astype(np.float64) * np.float64(s))
        assert (err <= np.float64(s) * 0.5 * (1 + 1e-5)).all()


def test_quantize_integers_reproduce_and_ties_go_to_even():
    x = np.arange(-127, 128, dtype=np.float32)
    s = oracle.scale_from_amax(oracle.amax(x))
    assert s == 1.0
    assert np.array_equal(oracle.quantize(x, s), x.astype(np.int8))
    halves = np.arange(-126.5, 127.0, 1.0, dtype=np.float32)
    halves = np.concatenate([halves, [127.0]]).astype(np.float32)
    c = oracle.quantize(halves, oracle.scale_from_amax(oracle.amax(halves)))
    assert (c[:-1] % 2 == 0).all()  # every .5 case rounds to the even neighbour


def test_quantize_zero_group_gives_zero_scale_and_codes():
    x = np.zeros(64, np.float32)
    s = oracle.scale_from_amax(oracle.amax(x))
    assert s == 0.0 and not oracle.quantize(x, s).any()


def test_query_quantisation_per_row_and_per_tensor():
    # row 0 reaches 127: scale 1, codes are the rounded values (ties to even); row 1 is row 0 times
    # 2^-3 (scale 2^-3, the same codes); per tensor, the one scale is 1 and row 1's codes shrink
    q = np.zeros((1, 2, 8), np.float32)
    q[0, 0] = [127.0, 2.5, -3.5, 0.5, -0.5, 1.49, 64.0, 0.0]
    q[0, 1] = q[0, 0] * 0.125
    codes, scales = oracle.quantize_q(q, "token")
    assert scales.tolist() == [[1.0, 0.125]]
    assert codes[0, 0].tolist() == [127, 2, -4, 0, 0, 1, 64, 0]
    assert codes[0, 1].tolist() == codes[0, 0].tolist()
    tcodes, ts = oracle.quantize_q(q, "tensor")
    assert ts.tolist() == [1.0] and tcodes[0, 0].tolist() == codes[0, 0].tolist()
    assert tcodes[0, 1].tolist() == [16, 0, 0, 0, 0, 0, 8, 0]  # 15.875 -> 16, 0.3125 -> 0, 8 -> 8
    assert np.array_equal(oracle.dequant_q(codes, scales)[0, 1], codes[0, 1] * 0.125)


def test_scheme_a_partitions_start_at_each_sequence():
    bt = _tiny_batch(G=2, D=8, lengths=(70, 64, 3, 129), Hkv=2, dtype="bf16")
    kc, vc, ks, vs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    cu = bt.cu_seqlens.numpy()
    assert ks.shape == (2, 2 + 1 + 1 + 3)
    col = 0
    for b in range(4):
        s0, e0 = int(cu[b]), int(cu[b + 1])
        for p in range(0, e0 - s0, 64):
            for h in range(2):
                block = bt.k[h, s0 + p:min(s0 + p + 64, e0)].float().numpy()
                assert ks[h, col] == np.float32(np.abs(block).max()) / np.float32(127)
                ref = np.clip(np.rint(block / ks[h, col]), -127, 127)
                assert np.array_equal(kc[h, s0 + p:min(s0 + p + 64, e0)], ref.astype(np.int8))
            col += 1
    assert vs[0] == np.float32(bt.v.float().abs().max().item()) / np.float32(127)


def test_scheme_b_equals_scheme_a_with_one_partition():
    bt = _tiny_batch(G=2, D=8, lengths=(100,), Hkv=1, dtype="bf16")
    kc_b, vc_b, ks_b, vs_b = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "B")
    kc_a, vc_a, ks_a, vs_a = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A", part=100)
    assert np.array_equal(kc_a, kc_b) and np.array_equal(vc_a, vc_b)
    assert ks_a.ravel()[0] == ks_b[0] and vs_a[0] == vs_b[0]


def test_calibrated_scales_hand_example(golden_dir):
    c = _load(golden_dir, "quantize_worked_cases.json")["calibrated"]
    k = np.array(c["k"], np.float32).reshape(1, 1, 8)
    v = np.array(c["v"], np.float32).reshape(1, 1, 8)
    cu = np.array([0, 1], np.int64)
    kc, vc, ks, vs = oracle.quantize_kv(k, v, cu, "A", v_scale=c["A"]["v_scale"])
    assert vc[0, 0].tolist() == c["A"]["v_codes"] and vs.tolist() == [c["A"]["v_scale"]]
    # the K partition scales and codes are scheme A's own (one 1-token partition: scale max|k|/127)
    assert ks.shape == (1, 1) and ks[0, 0] == np.float32(40.0) / np.float32(127.0)
    assert kc[0, 0, 2] == 127 and kc[0, 0, 5] == 0
    kc, vc, ks, vs = oracle.quantize_kv(k, v, cu, "B", k_scale=c["B"]["k_scale"], v_scale=c["B"]["v_scale"])
    assert kc[0, 0].tolist() == c["B"]["k_codes"] and vc[0, 0].tolist() == c["B"]["v_codes"]
    assert ks.tolist() == [c["B"]["k_scale"]] and vs.tolist() == [c["B"]["v_scale"]]


def test_calibrated_with_the_computed_scales_is_the_dynamic_quantisation():
    bt = _tiny_batch(G=2, D=8, lengths=(70, 64, 3, 129), Hkv=2, dtype="bf16")
    for scheme in ("A", "B"):
        kc, vc, ks, vs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme)
        kw = {"k_scale": ks[0]} if scheme == "B" else {}
        got = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, scheme, v_scale=vs[0], **kw)
        for a, b in zip(got, (kc, vc, ks, vs)):
            assert np.array_equal(a, b)
    # a calibrated V scale of a quarter of the computed one: codes are 4x (within the rounding) and
    # saturate where 4x leaves the range
    kc, vc, ks, vs = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    _, vc4, _, _ = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A", v_scale=vs[0] / 4)
    x = bt.v.float().numpy().astype(np.float64) / np.float64(np.float32(vs[0] / 4))
    inside = np.abs(x) < 126.5
    assert np.all(np.abs(vc4[inside].astype(np.int64) - np.rint(x[inside])) <= 1)
    assert np.all(vc4[x >= 127.5] == 127) and np.all(vc4[x <= -127.5] == -127)
    assert (np.abs(x) >= 127.5).any()


# ---------------------------------------------------------------------------------------------
# OAM scores and top-K
# ---------------------------------------------------------------------------------------------
def test_oam_hand_example(golden_dir):
    g = _load(golden_dir, "oam_hand_example.json")
    s = oracle.oam_scores(np.array(g["q"], float), np.array(g["k"], float), np.array(g["v"], float),
                          g["beta"], g["eps"])
    assert np.allclose(s, g["scores"], rtol=0, atol=1e-15)


def test_oam_scores_match_torch_route():
    G, D, n = 8, 64, 300
    q, k, v = _rand((G, D), 70), _rand((n, D), 71), _rand((n, D), 72)
    s = oracle.oam_scores(q, k, v, 0.7, 1e-6)
    tq, tk, tv = (torch.from_numpy(a) for a in (q, k, v))
    ref = (tk @ tq.T / math.sqrt(D)).max(dim=1).values + 0.7 * torch.log(torch.linalg.vector_norm(tv, dim=1) + 1e-6)
    assert np.allclose(s, ref.numpy(), rtol=0, atol=1e-12)


def test_topk_matches_brute_force_sort():
    rng = np.random.default_rng(80)
    for trial in range(30):
        n = int(rng.integers(1, 200))
        s = np.round(rng.standard_normal(n), 1)  # many exact ties
        K = int(rng.integers(1, n + 1))
        ref = sorted(sorted(range(n), key=lambda t: (-s[t], t))[:K])
        assert oracle.topk(s, K).tolist() == ref


def test_topk_all_equal_keeps_lowest_indices_and_keep_all():
    assert oracle.topk(np.zeros(50), 7).tolist() == list(range(7))
    s = _rand(33, 81)
    assert oracle.topk(s, 33).tolist() == list(range(33))


def test_kept_count():
    assert [oracle.kept_count(L, 1, 8) for L in (1, 7, 8, 9, 16, 17, 131072)] == [1, 1, 1, 2, 2, 3, 16384]
    assert oracle.kept_count(10, 1, 1) == 10 and oracle.kept_count(5, 0, 8) == 1


def test_beta_zero_is_classic_qk_ranking_and_q_zero_is_norm_ranking():
    G, D, n = 4, 16, 120
    q, k, v = _rand((G, D), 90), _rand((n, D), 91), _rand((n, D), 92)
    s0 = oracle.oam_scores(q, k, v, 0.0, 1e-6)
    qk = (k @ q.T).max(axis=1)  # classic Q x K score, group max
    assert np.array_equal(oracle.topk(s0, 15), np.sort(np.argsort(-qk, kind="stable")[:15]))
    sz = oracle.oam_scores(np.zeros((G, D)), k, v, 1.0, 1e-6)
    norms = np.linalg.norm(v, axis=1)
    assert np.array_equal(oracle.topk(sz, 15), np.sort(np.argsort(-norms, kind="stable")[:15]))
    # equal |v| for every token: OAM ranks exactly like Q x K
    vu = v / np.linalg.norm(v, axis=1, keepdims=True) * 2.0
    su = oracle.oam_scores(q, k, vu, 1.0, 1e-6)
    assert np.array_equal(oracle.topk(su, 15), np.sort(np.argsort(-qk, kind="stable")[:15]))


def test_value_norms_closed_form_and_library():
    v = np.zeros((2, 3, 8))
    v[0, 0, :2] = (3.0, 4.0)  # 5
    v[1, 2, :] = 1.0  # sqrt(8)
    n = oracle.value_norms(v)
    assert n[0, 0] == 5.0 and n[1, 2] == math.sqrt(8.0) and n[0, 1] == 0.0
    w = np.random.default_rng(3).standard_normal((4, 50, 64))
    assert np.allclose(oracle.value_norms(w), np.linalg.norm(w, axis=-1), rtol=1e-14, atol=0)


def test_int8_selection_with_exact_codes_is_the_plain_selection():
    # keys = integer codes * 2^e with every 64-token partition reaching |127| * 2^e: the partition
    # scale is exactly 2^e (a different e per partition and head) and the codes are the integers,
    # so the dequantised keys equal the keys and the INT8-cache selection must equal the plain one
    rng = np.random.default_rng(11)
    lengths = [70, 200, 5]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    Hkv, G, D = 2, 4, 64
    T = int(cu[-1])
    codes = rng.integers(-127, 128, size=(Hkv, T, D)).astype(np.float32)
    k = np.empty_like(codes)
    want_scales = []
    for h in range(Hkv):
        row = []
        for b in range(3):
            for p0 in range(0, lengths[b], 64):
                e = int(rng.integers(-3, 4))
                sl = slice(cu[b] + p0, cu[b] + min(p0 + 64, lengths[b]))
                codes[h, sl.start, 0] = 127.0
                k[h, sl] = codes[h, sl] * 2.0 ** e
                row.append(2.0 ** e)
        want_scales.append(row)
    v = rng.standard_normal((Hkv, T, D)).astype(np.float32)
    q = rng.standard_normal((3, Hkv * G, D)).astype(np.float32)
    kc, _, ks, _ = oracle.quantize_kv(k, v, cu, "A")
    assert np.array_equal(ks, np.array(want_scales, np.float32)) and np.array_equal(kc.astype(np.float32), codes)
    got = oracle.oam_select_int8(q, kc, ks, v, cu, "A", G, 1.0, 1e-6, 1, 4)
    want = oracle.oam_select(q, k, v, cu, G, 1.0, 1e-6, 1, 4)
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
    for key in want[2]:
        assert np.array_equal(got[2][key], want[2][key])


def test_keep_all_selection_equals_dense_decode():
    bt = _tiny_batch(G=4, D=16, lengths=(9, 40), Hkv=2, dtype="bf16")
    idx, cu_kept, _ = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, 4, 1.0, 1e-6, 1, 1)
    assert cu_kept.tolist() == [0, 9, 49]
    assert idx[:, :9].tolist() == [list(range(9))] * 2
    dense = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 4)
    sel = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 4, idx=idx, cu_kept=cu_kept)
    assert np.allclose(dense[0], sel[0], atol=1e-13) and np.allclose(dense[1], sel[1], atol=1e-13)


def test_indexed_decode_equals_attention_over_the_subset():
    bt = _tiny_batch(G=2, D=8, lengths=(50,), Hkv=1)
    idx, cu_kept, _ = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, 2, 1.0, 1e-6, 1, 8)
    out, lse = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 2, idx=idx, cu_kept=cu_kept)
    sel = idx[0]
    assert sel.size == 7 and (np.diff(sel) > 0).all()
    q = bt.q[0].double()
    kk, vv = bt.k[0, sel].double(), bt.v[0, sel].double()
    ref = torch.nn.functional.scaled_dot_product_attention(q[:, None], kk[None].expand(2, -1, -1),
                                                           vv[None].expand(2, -1, -1))[:, 0]
    assert np.allclose(out[0], ref.numpy(), atol=1e-12)


def test_int8_decode_is_attention_over_dequantised_cache():
    bt = _tiny_batch(G=2, D=8, lengths=(70, 5), Hkv=2, dtype="bf16")
    quant = oracle.quantize_kv(bt.k, bt.v, bt.cu_seqlens, "A")
    kc, vc, ks, vs = quant
    out, lse = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 2, quant=(*quant, "A"))
    # independent dequantisation: partition p of sequence 0 head 1 holds tokens 64p .. 64p+63
    k_hat = torch.from_numpy(kc[1, :70].astype(np.float64))
    k_hat[:64] *= float(ks[1, 0])
    k_hat[64:] *= float(ks[1, 1])
    v_hat = torch.from_numpy(vc[1, :70].astype(np.float64)) * float(vs[0])
    q = bt.q[0, 2:4].double()
    ref = torch.nn.functional.scaled_dot_product_attention(q[:, None], k_hat[None].expand(2, -1, -1),
                                                           v_hat[None].expand(2, -1, -1))[:, 0]
    assert np.allclose(out[0, 2:4], ref.numpy(), atol=1e-12)


# ---------------------------------------------------------------------------------------------
# partition
# ---------------------------------------------------------------------------------------------
def test_plan_hand_example(golden_dir):
    g = _load(golden_dir, "plan_hand_example.json")
    p = oracle.plan(g["row_lengths"], g["n_req"], g["granule"], g["min_chunk"], 0)
    segs = [list(map(int, t)) for t in zip(p["cta"], p["row"], p["start"], p["len"])]
    assert segs == g["segments"] and p["n_cta"] == g["n_cta"]
    c = g["row_cost_case"]
    p = oracle.plan(c["row_lengths"], c["n_req"], c["granule"], c["min_chunk"], 0, c["row_cost"])
    segs = [list(map(int, t)) for t in zip(p["cta"], p["row"], p["start"], p["len"])]
    assert segs == c["segments"] and p["n_cta"] == c["n_cta"]


@pytest.mark.parametrize("row_cost", [0, 256])
@pytest.mark.parametrize("seed", range(12))
def test_plan_covers_every_token_once_with_equal_work(seed, row_cost):
    plan_coverage(seed, row_cost)


def plan_coverage(seed, row_cost=0):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 40))
    lens = np.rint(np.exp(rng.uniform(0, 10, R))).astype(np.int64)
    n_req = int(rng.integers(1, 300))
    gran = 16
    p = oracle.plan(lens, n_req, gran, gran, 0, row_cost)
    assert p["n_cta"] <= n_req
    covered = [np.zeros(L, np.int32) for L in lens]
    for c, r, s, l in zip(p["cta"], p["row"], p["start"], p["len"]):
        assert l >= 1 and s % gran == 0
        covered[r][s:s + l] += 1
    assert all((cv == 1).all() for cv in covered)
    # segments come in stream order; a CTA's padded work is at most S
    order = list(zip(p["cta"], p["row"]))
    assert order == sorted(order)
    W = int(sum((L + gran - 1) // gran * gran + row_cost for L in lens))
    S = max(gran, -(-(-(-W // n_req)) // gran) * gran)
    work = np.zeros(p["n_cta"], np.int64)
    for c, l in zip(p["cta"], p["len"]):
        work[c] += (l + gran - 1) // gran * gran
    assert work.max() <= S
    # with a row charge, a CTA's tokens plus the charges of the rows starting in it stay within
    # S plus one charge (a row's charge follows its tokens and may spill into the next range)
    if row_cost:
        starts = np.zeros(p["n_cta"], np.int64)
        for c, s in zip(p["cta"], p["start"]):
            starts[c] += row_cost if s == 0 else 0
        assert (work + starts).max() <= S + row_cost
    one = oracle.plan(lens, 0, gran, gran, 1)
    assert one["n_cta"] == R and one["len"].tolist() == lens.tolist()


# ---------------------------------------------------------------------------------------------
# decode_multi: M query tokens per sequence, causal over the last M cache entries
# ---------------------------------------------------------------------------------------------
def _multi_batch(M, G=2, D=16, lengths=(9, 40, 3), Hkv=2, seed=3, dtype="f32"):
    wl = workloads.Workload("tiny-multi", B=len(lengths), Hkv=Hkv, G=G, D=D, kv_dtype=dtype,
                            dist="normal", lengths=tuple(lengths), M=M)
    return workloads.generate(wl, seed)


def test_multi_token_with_one_token_is_decode():
    bt = _multi_batch(1)
    q = bt.q[:, None]
    out, lse = oracle.decode_multi(q, bt.k, bt.v, bt.cu_seqlens, 2, 1)
    ref = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 2)
    assert np.array_equal(out[:, 0], ref[0]) and np.array_equal(lse[:, 0], ref[1])


@pytest.mark.parametrize("M", [2, 4])
def test_multi_token_query_m_is_decode_over_the_truncated_cache(M):
    # query m sees the first L - M + m + 1 tokens: the single-token decode of a repacked cache
    # holding only that prefix of every sequence must give the same numbers
    bt = _multi_batch(M)
    out, lse = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, 2, M)
    cu = bt.cu_seqlens.numpy().astype(np.int64)
    for m in range(M):
        keep = [max(0, int(cu[b + 1] - cu[b]) - M + m + 1) for b in range(bt.wl.B)]
        live = [b for b in range(bt.wl.B) if keep[b] > 0]
        k = torch.cat([bt.k[:, cu[b]:cu[b] + keep[b]] for b in live], dim=1)
        v = torch.cat([bt.v[:, cu[b]:cu[b] + keep[b]] for b in live], dim=1)
        cu2 = np.concatenate([[0], np.cumsum([keep[b] for b in live])])
        ref = oracle.decode(bt.q[live, m], k, v, cu2, 2)
        assert np.array_equal(out[live, m], ref[0]) and np.array_equal(lse[live, m], ref[1])
        for b in set(range(bt.wl.B)) - set(live):  # L < M: this query sees nothing
            assert (out[b, m] == 0).all() and np.isneginf(lse[b, m]).all()


def test_multi_token_matches_sdpa_with_a_causal_offset_mask():
    M, G, D = 3, 2, 16
    bt = _multi_batch(M, G=G, D=D, lengths=(11,), Hkv=1)
    out, lse = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, G, M)
    L = 11
    allowed = torch.arange(L)[None, :] <= (L - M + torch.arange(M))[:, None]  # [M, L]
    q = bt.q[0].double().permute(1, 0, 2)  # [G, M, D]
    kk, vv = bt.k[0].double(), bt.v[0].double()
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk[None].expand(G, -1, -1),
                                                           vv[None].expand(G, -1, -1), attn_mask=allowed)
    assert np.allclose(out[0], ref.permute(1, 0, 2).numpy(), atol=1e-12)
    z = (q @ kk.T) / math.sqrt(D)
    ref_lse = torch.logsumexp(z.masked_fill(~allowed, -math.inf), dim=-1)  # [G, M]
    assert np.allclose(lse[0], ref_lse.T.numpy(), atol=1e-12)
    assert allowed.sum().item() == 3 * (L - M) + 1 + 2 + 3


def test_multi_token_over_kept_tokens_masks_by_position():
    M = 2
    bt = _multi_batch(M, lengths=(30,), Hkv=1)
    idx = np.array([[0, 5, 28, 29]], np.int32)
    cu_kept = np.array([0, 4], np.int32)
    out, lse = oracle.decode_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, 2, M, idx=idx, cu_kept=cu_kept)
    # query 0 sees positions 0, 5, 28; query 1 all four
    for m, sel in ((0, [0, 5, 28]), (1, [0, 5, 28, 29])):
        ref = oracle.attend(bt.q[0, m, 0:2], bt.k[0, sel], bt.v[0, sel])
        assert np.array_equal(out[0, m], ref[0]) and np.array_equal(lse[0, m], ref[1])


# ---------------------------------------------------------------------------------------------
# block-granular selection: 64-token blocks scored by the max of their token scores
# ---------------------------------------------------------------------------------------------
def test_block_scores_brute_force_with_ragged_last_block():
    s = _rand(130, 5)
    bs = oracle.block_scores(s, 64)
    assert bs.size == 3
    assert bs[0] == max(s[:64]) and bs[1] == max(s[64:128]) and bs[2] == max(s[128], s[129])


def test_block_selection_with_one_token_blocks_is_token_selection():
    bt = _tiny_batch(G=2, D=16, lengths=(9, 40, 1), Hkv=2, dtype="bf16")
    idx, cu_kept, scores = oracle.oam_select(bt.q, bt.k, bt.v, bt.cu_seqlens, 2, 1.0, 1e-6, 3, 8)
    blk, cu_b, _ = oracle.select_blocks(scores, bt.cu_seqlens, 2, 3, 8, block=1)
    assert np.array_equal(blk, idx) and np.array_equal(cu_b, cu_kept)


def test_block_selection_hand_example_and_ties():
    # one sequence of 130 tokens: blocks of 64, 64 and 2 tokens; keep ceil(3 / 3) = 1 block
    s = np.zeros(130)
    s[10], s[100], s[129] = 1.0, 2.0, 3.0  # the ragged last block holds the best token
    blk, cu_b, bs = oracle.select_blocks({(0, 0): s}, [0, 130], 1, 1, 3)
    assert cu_b.tolist() == [0, 1] and blk.tolist() == [[2]] and bs[(0, 0)].tolist() == [1.0, 2.0, 3.0]
    # keep 2 of 3 with blocks 0 and 2 tied: the lower block index wins the tie, output ascending
    s = np.zeros(130)
    s[5], s[70], s[128] = 5.0, 7.0, 5.0
    blk, cu_b, _ = oracle.select_blocks({(0, 0): s}, [0, 130], 1, 2, 3)
    assert blk.tolist() == [[0, 1]]


def test_block_selection_brute_force_ranking():
    rng = np.random.default_rng(11)
    cu = [0, 300, 1000]
    scores = {(b, h): np.round(rng.standard_normal(cu[b + 1] - cu[b]), 1) for b in range(2) for h in range(2)}
    blk, cu_b, _ = oracle.select_blocks(scores, cu, 2, 1, 4)
    for (b, h), s in scores.items():
        nb = -(-s.size // 64)
        S = [max(s[64 * j:64 * j + 64]) for j in range(nb)]
        K = -(-nb // 4)
        want = sorted(sorted(range(nb), key=lambda j: (-S[j], j))[:K])
        assert blk[h, cu_b[b]:cu_b[b + 1]].tolist() == want


def test_decode_over_blocks_is_attention_over_their_tokens():
    bt = _tiny_batch(G=2, D=8, lengths=(150, 64), Hkv=2)
    blk = np.array([[0, 2, 0], [1, 2, 0]], np.int32)  # sequence 0 keeps 2 blocks, sequence 1 one
    cu_b = np.array([0, 2, 3], np.int32)
    out, lse = oracle.decode_blocks(bt.q, bt.k, bt.v, bt.cu_seqlens, 2, blk, cu_b)
    # head 1 of sequence 0: blocks 1 and 2 = tokens 64..127 and the ragged 128..149
    sel = list(range(64, 150))
    ref = oracle.attend(bt.q[0, 2:4], bt.k[1, sel], bt.v[1, sel])
    assert np.array_equal(out[0, 2:4], ref[0]) and np.array_equal(lse[0, 2:4], ref[1])
    # keeping every block is the dense decode
    dense = oracle.decode(bt.q, bt.k, bt.v, bt.cu_seqlens, 2)
    allb = np.array([[0, 1, 2, 0], [0, 1, 2, 0]], np.int32)
    o2, l2 = oracle.decode_blocks(bt.q, bt.k, bt.v, bt.cu_seqlens, 2, allb, np.array([0, 3, 4], np.int32))
    assert np.allclose(o2, dense[0], atol=1e-13) and np.allclose(l2, dense[1], atol=1e-13)


# ---------------------------------------------------------------------------------------------
# oam_select_multi: one kept set for the M query tokens of a speculative step
# ---------------------------------------------------------------------------------------------
def test_multi_token_scores_are_the_max_over_the_tokens_single_scores():
    M, G = 3, 2
    bt = _multi_batch(M, G=G, D=16, lengths=(40, 9), Hkv=2, seed=8)
    idx, cu_kept, scores = oracle.oam_select_multi(bt.q, bt.k, bt.v, bt.cu_seqlens, G, M, 1.0, 1e-6, 1, 4)
    singles = [oracle.oam_select(bt.q[:, m], bt.k, bt.v, bt.cu_seqlens, G, 1.0, 1e-6, 1, 4)[2] for m in range(M)]
    for key, s in scores.items():
        want = np.max(np.stack([sm[key] for sm in singles]), axis=0)  # beta * ln(|v| + eps) is common
        assert np.allclose(s, want, rtol=0, atol=1e-12)
        b, h = key
        ref = sorted(sorted(range(s.size), key=lambda t: (-want[t], t))[:cu_kept[b + 1] - cu_kept[b]])
        assert idx[h, cu_kept[b]:cu_kept[b + 1]].tolist() == ref
    one = oracle.oam_select_multi(bt.q[:, :1], bt.k, bt.v, bt.cu_seqlens, G, 1, 1.0, 1e-6, 1, 4)
    base = oracle.oam_select(bt.q[:, 0], bt.k, bt.v, bt.cu_seqlens, G, 1.0, 1e-6, 1, 4)
    assert np.array_equal(one[0], base[0]) and np.array_equal(one[1], base[1])
