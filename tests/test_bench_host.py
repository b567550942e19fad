"""bench.py's host arithmetic without a GPU: the algorithmic bytes each stage and kernel must
move (restated here from the data layout, independently of bench.py's formulas), the naming of
the library's kernels in the per-launch timing, and the traffic record's staleness check."""
import importlib.util
import json
import os

import pytest

import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_kernel_roles_from_demangled_names(bench):
    r = bench.kernel_role
    assert r("void sgd::decode_mma_kernel<sgd::MmaCfg<128, 1, false, false, 2, false, false, false> >") == \
        "score_quantize"
    assert r("void sgd::decode_mma_kernel<sgd::MmaCfg<128, 2, true, true, 0, true, false, false> >") == "decode"
    assert r("void sgd::decode_mma_kernel<sgd::MmaCfg<128, 1, true, false, 1, false, false, false> >") == "score"
    assert r("void sgd::quant_global_kernel<__nv_bfloat16, false>") == "v_codes"
    assert r("void sgd::topk_cluster_kernel<512, 8, 2>") == "topk"
    assert r("sgd::plan_kernel") == "plan" and r("sgd::block_max_kernel") == "block_max"
    assert r("sgd::plan_fast_kernel(const int *, const int *, int, int)") == "plan"
    assert r("void sgd::decode_generic_kernel<128, float, true, 0>") == "decode"
    # without a demangler the mangled names give the same roles
    assert r("_ZN3sgd17decode_mma_kernelINS_6MmaCfgILi128ELi1ELb0ELb0ELi2ELb0ELb0ELb0EEEEEv14CUtensorMap_stS3_"
             "NS_10DecodeArgsE") == "score_quantize"
    assert r("_ZN3sgd17decode_mma_kernelINS_6MmaCfgILi128ELi1ELb1ELb1ELi0ELb0ELb0ELb0EEEEEv14CUtensorMap_stS3_"
             "NS_10DecodeArgsE") == "decode"


def test_demangle_reads_the_library_names(bench):
    out = bench.demangle(["_ZN3sgd11plan_kernelEPKiS1_iiiiiiNS_8PlanViewEPNS_8WsHeaderEiPfS5_iiPK13__nv_bfloat16liii"])
    assert out[0].startswith("sgd::plan_kernel(") or out[0].startswith("_ZN3sgd11plan_kernel")


def test_fused_pass_and_decode_bytes_from_the_layout(bench):
    # two sequences of 100 and 64 tokens, Hkv 2, G 4, D 128, scheme A, keep 1/8
    wl = workloads.Workload("t", B=2, Hkv=2, G=4, D=128, kv_dtype="bf16", dist="normal", lengths=(100, 64),
                            scheme="A", oam=True)
    lengths = [100, 64]
    T, Hkv, D = 164, 2, 128
    parts = 2 + 1  # ceil(100/64) + ceil(64/64)
    q = 2 * 8 * D * 2  # B * Hq * D bf16
    fused = 2 * Hkv * T * D * 2 + Hkv * T * D + Hkv * parts * 4 + Hkv * T * 4 + q
    assert bench.kernel_bytes(wl, lengths, "score_quantize") == fused
    assert bench.kernel_bytes(wl, lengths, "v_codes") == Hkv * T * D * 2 + Hkv * T * D + 4
    kept = 13 + 8  # ceil(100/8) + ceil(64/8)
    out = 2 * 8 * (D + 1) * 4
    decode = 2 * Hkv * kept * D + Hkv * kept * 4 + Hkv * parts * 4 + q + out
    assert bench.algorithmic_bytes(wl, lengths)["decode"] == decode
    assert bench.kernel_bytes(wl, lengths, "decode") == decode
    assert bench.kernel_bytes(wl, lengths, "topk") is None


def test_block_selection_counts_whole_blocks(bench):
    wl = workloads.Workload("t", B=2, Hkv=1, G=8, D=128, kv_dtype="bf16", dist="normal", lengths=(130, 1000),
                            scheme="A", oam=True, select_on_codes=True, blocks=True)
    nb = [3, 16]
    kept = 1 + 2  # ceil(3/8), ceil(16/8)
    st = bench.algorithmic_bytes(wl, [130, 1000])
    q, out = 2 * 8 * 128 * 2, 2 * 8 * 129 * 4
    assert st["decode"] == 2 * 64 * kept * 128 + kept * 4 + sum(nb) * 4 + q + out


def test_multi_token_decode_counts_every_query_token(bench):
    wl = workloads.Workload("t", B=1, Hkv=1, G=8, D=128, kv_dtype="bf16", dist="normal", lengths=(640,),
                            scheme="A", M=4)
    st = bench.algorithmic_bytes(wl, [640])
    assert st["decode"] == 2 * 640 * 128 + 10 * 4 + 4 * (8 * 128 * 2 + 8 * 129 * 4)


def test_traffic_record_is_ignored_once_a_source_changes(bench, tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("one")
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"w": {"kernels": {"decode": {"bytes_per_launch": 7, "sources": ["k.cu"],
                                        "source_hash": bench.source_hash([str(src)])}}}}
    (prof / "dram_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("decode", "w") == 7
    src.write_text("two")
    assert bench.load_traffic("decode", "w") is None
    assert bench.load_traffic("decode", "other") is None


def test_scheme_b_codes_both_tensors_in_one_launch(bench):
    wl = workloads.Workload("t", B=1, Hkv=2, G=4, D=128, kv_dtype="bf16", dist="normal", lengths=(100,),
                            scheme="B")
    T, Hkv, D = 100, 2, 128
    assert bench.kernel_bytes(wl, [100], "v_codes") == 2 * (Hkv * T * D * 2 + Hkv * T * D + 4)
    assert bench.kernel_bytes(wl, [100], "amax") == 2 * Hkv * T * D * 2
    sel = wl.with_(oam=True)  # the fused pass of scheme B writes no K codes
    assert bench.kernel_bytes(sel, [100], "score_quantize") == 2 * Hkv * T * D * 2 + Hkv * T * 4 + 1 * 8 * D * 2


@pytest.mark.parametrize("workload", [7, 9])
def test_reference_arm_prints_the_contract_line(workload):
    # the oracle arm runs on the host cores: one bounded step of the workload, one JSON line
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        str(workload), "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == workloads.config(workload).name


def test_rates_against_the_three_denominators(bench):
    f = bench.fractions(4000.0, 6400.0, 7000.0)
    assert f["frac_of_hbm"] == pytest.approx(0.625) and f["frac_of_nominal"] == pytest.approx(0.5)
    assert f["frac_of_read_only"] == pytest.approx(4000 / 7000, abs=1e-4)
    assert "frac_of_read_only" not in bench.fractions(1.0, 2.0, None)


def test_cpu_baseline_counts_the_same_rows_on_one_or_several_threads(bench):
    # a small copy of the default workload: every row fits the budget, so both runs cover all rows
    wl = workloads.config(5, B=2, Hkv=2, length_range=(200, 900))
    bt = workloads.generate(wl, 5)
    _, s1, _, t1 = bench.cpu_baseline_sample(bt, wl, budget_s=60.0, threads=1)
    _, s4, _, t4 = bench.cpu_baseline_sample(bt, wl, budget_s=60.0, threads=4)
    assert t1 == 1 and t4 == 4
    tokens = int(bt.lengths.sum()) * wl.Hkv
    for s in (s1, s4):
        assert s.startswith(f"4 (sequence, KV head) rows of the workload, shortest first, {tokens} tokens")


def test_kept_rows_are_the_cache_rows_of_the_kept_tokens(bench):
    # the rows the gather ceiling reads: kvh * T + cu_seqlens[b] + idx, against a plain loop
    import numpy as np
    import torch
    rng = np.random.default_rng(7)
    lengths = [5, 1, 17, 9]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    kept = [max(1, (L + 3) // 4) for L in lengths]
    cu_kept = np.concatenate([[0], np.cumsum(kept)]).astype(np.int32)
    Hkv, T, Kt = 3, int(cu[-1]), int(cu_kept[-1])
    idx = np.zeros((Hkv, Kt), np.int32)
    for h in range(Hkv):
        for b, L in enumerate(lengths):
            idx[h, cu_kept[b]:cu_kept[b + 1]] = np.sort(rng.choice(L, kept[b], replace=False))
    rows = bench.kept_rows(torch.from_numpy(idx), torch.from_numpy(cu_kept), torch.from_numpy(cu), T).numpy()
    ref = [h * T + cu[b] + idx[h, j] for h in range(Hkv) for b in range(len(lengths))
           for j in range(cu_kept[b], cu_kept[b + 1])]
    assert rows.dtype == np.int32 and rows.tolist() == ref
    assert rows.min() >= 0 and rows.max() < Hkv * T


def test_calibrated_fused_pass_counts_every_code(bench):
    # with calibrated scales the fused pass also writes the V codes (scheme B: the K codes too);
    # the step's algorithmic bytes are those of the computed-scale step
    lengths = [100, 64]
    T, Hkv, D, parts = 164, 2, 128, 3
    q = 2 * 8 * D * 2
    for scheme in ("A", "B"):
        wl = workloads.Workload("t", B=2, Hkv=2, G=4, D=128, kv_dtype="bf16", dist="normal", lengths=(100, 64),
                                scheme=scheme, oam=True)
        cal = wl.with_(calibrated=True)
        scales = Hkv * parts * 4 if scheme == "A" else 0
        want = 2 * Hkv * T * D * 2 + 2 * Hkv * T * D + scales + Hkv * T * 4 + q
        assert bench.kernel_bytes(cal, lengths, "score_quantize") == want
        assert bench.algorithmic_bytes(cal, lengths) == bench.algorithmic_bytes(wl, lengths)
