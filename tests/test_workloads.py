"""The seeded input recipe (workloads/__init__.py docstring) restated and checked draw by draw,
so every input the parity tests and the bench use is reproducible from its description."""
import math

import numpy as np
import torch

import workloads


def _streams(seed, Hkv):
    return np.random.SeedSequence(seed).spawn(1 + 2 * Hkv)


def test_normal_recipe_draw_by_draw():
    wl = workloads.Workload("t", B=2, Hkv=2, G=4, D=64, kv_dtype="bf16", dist="normal", lengths=(5, 9))
    bt = workloads.generate(wl, 3)
    st = _streams(3, 2)
    r0 = np.random.default_rng(st[0])
    q = r0.standard_normal((2, 8, 64), dtype=np.float32)
    assert torch.equal(bt.q, torch.from_numpy(q).to(torch.bfloat16))
    for h in range(2):
        k = np.random.default_rng(st[1 + h]).standard_normal((14, 64), dtype=np.float32)
        v = np.random.default_rng(st[3 + h]).standard_normal((14, 64), dtype=np.float32)
        assert torch.equal(bt.k[h], torch.from_numpy(k).to(torch.bfloat16))
        assert torch.equal(bt.v[h], torch.from_numpy(v).to(torch.bfloat16))
    assert bt.cu_seqlens.tolist() == [0, 5, 14]


def test_outlier_recipe_and_ragged_lengths():
    wl = workloads.Workload("t", B=3, Hkv=1, G=2, D=32, kv_dtype="f32", dist="outlier", length_range=(16, 400))
    bt = workloads.generate(wl, 11)
    st = _streams(11, 1)
    r0 = np.random.default_rng(st[0])
    L = np.rint(np.exp(r0.uniform(math.log(16), math.log(400), size=3))).astype(np.int64)
    assert bt.lengths.tolist() == L.tolist() and (16 <= L).all() and (L <= 400).all()
    ch = np.sort(r0.choice(32, size=4, replace=False))
    assert bt.outlier_channels.tolist() == ch.tolist()
    T = int(L.sum())
    k = np.random.default_rng(st[1]).standard_normal((T, 32), dtype=np.float32)
    k[:, ch] *= np.float32(20.0)
    rv = np.random.default_rng(st[2])
    v = rv.standard_normal((T, 32), dtype=np.float32)
    v *= rv.lognormal(0.0, 1.0, size=T).astype(np.float32)[:, None]
    assert torch.equal(bt.k[0], torch.from_numpy(k)) and torch.equal(bt.v[0], torch.from_numpy(v))


def test_several_query_tokens_and_determinism():
    wl = workloads.Workload("t", B=2, Hkv=1, G=8, D=128, kv_dtype="bf16", dist="normal", lengths=(3, 4), M=2)
    a, b = workloads.generate(wl, 5), workloads.generate(wl, 5)
    assert a.q.shape == (2, 2, 8, 128)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    c = workloads.generate(wl, 6)
    assert not torch.equal(a.q, c.q)


def test_named_configurations_and_their_seeds():
    assert workloads.config(5).scheme == "A" and workloads.config(5).oam
    assert workloads.config(7).seed == 5 and workloads.config(9).seed == 6  # shared batches
    assert workloads.config(4, lengths=(64,) * 8).lengths == (64,) * 8


def test_ragged_int8_workload_shares_the_ragged_lengths():
    # workload 14 is workload 3's ragged batch (same seed, lengths drawn first) over workload 4's
    # INT8 cache distribution; one KV head is enough to see the lengths
    a = workloads.generate(workloads.config(3).with_(Hkv=1))
    b = workloads.generate(workloads.config(14).with_(Hkv=1))
    assert a.lengths.tolist() == b.lengths.tolist()
    assert b.outlier_channels is not None and workloads.config(14).scheme == "A"
    assert (512 <= b.lengths).all() and (b.lengths <= 131072).all()


def test_calibrated_workload_is_the_default_batch():
    # workload 15 draws workload 5's batch (its seed): the calibrated step quantises the same cache
    w5, w15 = workloads.config(5), workloads.config(15)
    assert w15.calibrated and not w5.calibrated
    assert w15.with_(name=w5.name, calibrated=False, seed=None) == w5
    small5 = w5.with_(length_range=(300, 900))
    small15 = w15.with_(length_range=(300, 900))
    a = workloads.generate(small5, seed=5)
    b = workloads.generate(small15, seed=small15.seed)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v), (a.cu_seqlens, b.cu_seqlens)):
        assert torch.equal(x, y)
