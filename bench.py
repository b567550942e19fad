#!/usr/bin/env python
"""Benchmark of the decode hot path: INT8 scheme-A quantisation -> OAM token selection ->
split-KV decode over the kept tokens (-> LSE merge), on seeded synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 5] [--impl reference]

One step = one pass of the whole path over one batch (the default workload: 4 sequences of
32K-128K tokens, 8 KV heads, G = 8, D = 128, beta = 1, eps = 1e-6, keep 1/8).  Prints one JSON
line.  `value` is algorithmic KV bytes moved per second by the whole job (GB/s); stage times,
sequences*heads/s, a roofline entry for the dominant stage and the fp64 oracle's CPU rate on a
bounded sample are included.  With N > 1 (torchrun), every rank runs its own copy of the
workload on its own GPU (independent rows: weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, "about 8 TB/s"
READ_ONLY_BYTES = 4 << 30  # the read-only ceiling streams 4 GiB (far above L2)
# the 128K INT8 split-KV decode stages timed beside the default workload: workload 4 (8 x 128K,
# INT8 scheme A, dense) and workload 14 (the ragged 512-128K batch over the same INT8 cache)
INT8_DECODE_WORKLOADS = (4, 14)
CALIBRATED_WORKLOAD = 15  # workload 5 with a calibrated V scale


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", type=int, default=5, choices=[2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15])
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra-records", action="store_true",
                   help="skip the records beside the step: the read-only ceiling, the workload 4 / 14 INT8 decode "
                        "stages, the calibrated-scale step and the gather ceiling")
    p.add_argument("--scale", type=float, default=1.0,
                   help="sequence lengths times this factor (a smaller case of the same shapes, for profiling)")
    return p.parse_args()


def scaled(wl, scale):
    """The workload with every sequence length times `scale` (at least one token)."""
    if scale == 1.0:
        return wl
    if wl.lengths is not None:
        return wl.with_(lengths=tuple(max(1, int(round(L * scale))) for L in wl.lengths))
    lo, hi = wl.length_range
    return wl.with_(length_range=(max(1, int(round(lo * scale))), max(1, int(round(hi * scale)))))


# ------------------------------------------------------------------------------------------------
# algorithmic bytes
# ------------------------------------------------------------------------------------------------
def kept_of(L, num, den):
    return max(1, min(int(L), -(-int(L) * num // den)))


def algorithmic_bytes(wl, lengths):
    """Bytes each stage must move at minimum (inputs read once, outputs written once)."""
    Hkv, D, G, B = wl.Hkv, wl.D, wl.G, wl.B
    T = int(sum(lengths))
    P = int(sum((int(L) + 63) // 64 for L in lengths))
    kv_bf16 = 2 * Hkv * T * D * 2
    q = B * Hkv * G * D * 2
    out = B * Hkv * G * (D + 1) * 4
    st = {}
    codes_out = 2 * Hkv * T * D + (Hkv * P * 4 if wl.scheme == "A" else 4) + 4
    if wl.oam:
        # kept tokens (block selection: kept blocks, each counted as the 64 tokens its tile reads)
        nb = [(int(L) + 63) // 64 for L in lengths]
        Kt = (sum(kept_of(n, wl.keep_num, wl.keep_den) for n in nb) if wl.blocks
              else sum(kept_of(L, wl.keep_num, wl.keep_den) for L in lengths))
        sel_out = q + Hkv * Kt * 4 + (B + 1) * 4
    if wl.select_on_codes:  # the cache is already INT8: the selection reads K codes and the norms
        st["select"] = Hkv * T * D + Hkv * T * 4 + (Hkv * P * 4 if wl.scheme == "A" else 4) + sel_out
    elif wl.scheme and wl.oam:  # one call reads K and V once for both
        st["quantize_select"] = kv_bf16 + codes_out + sel_out
    elif wl.scheme:
        st["quantize"] = kv_bf16 + codes_out
    elif wl.oam:
        st["select"] = kv_bf16 + sel_out
    if wl.oam:
        n_att = 64 * Kt if wl.blocks else Kt
        idx_bytes = Hkv * Kt * 4
    else:
        n_att = T
        idx_bytes = 0
    eb = 1 if wl.scheme else 2
    scales = (Hkv * P * 4 if wl.scheme == "A" else 8) if wl.scheme else 0
    st["decode"] = 2 * Hkv * n_att * D * eb + idx_bytes + scales + wl.M * (q + out)  # M query tokens
    return st


def kernel_role(name):
    """What a library kernel (demangled name) does in the step."""
    if "decode_mma_kernel" in name:
        m = re.search(r"MmaCfg<\d+, \d+, \w+, \w+, (\d+)", name)
        mode = m.group(1) if m else ""
        if not m and "MmaCfgI" in name:  # a mangled name: the fifth template argument is the mode
            args = re.findall(r"L[ib](\d+)E", name.split("MmaCfgI", 1)[1])
            mode = args[4] if len(args) > 4 else ""
        return {"0": "decode", "1": "score", "2": "score_quantize"}.get(mode, "decode")
    for key, role in (("quant_global_kernel", "v_codes"), ("topk_cluster_kernel", "topk"), ("plan_kernel", "plan"),
                      ("plan_fast_kernel", "plan"),
                      ("block_max_kernel", "block_max"), ("quant_k_partition_kernel", "k_codes"),
                      ("quant_amax_kernel", "amax"), ("quant_prep_kernel", "prep"), ("merge_kernel", "merge"),
                      ("decode_generic_kernel", "decode")):
        if key in name:
            return role
    return name


def kernel_bytes(wl, lengths, role):
    """Bytes the kernel of this role must move per launch (inputs read once, outputs written
    once), or None where no figure is stated."""
    Hkv, D, B = wl.Hkv, wl.D, wl.B
    T = int(sum(lengths))
    P = int(sum((int(L) + 63) // 64 for L in lengths))
    q = B * wl.M * Hkv * wl.G * D * 2
    scales = Hkv * P * 4 if wl.scheme == "A" else 4
    if role == "score_quantize":  # K and V (bf16) in; scores out; scheme A: K codes and scales out
        codes = Hkv * T * D + scales if wl.scheme == "A" else 0
        if wl.calibrated:  # and the V codes (scheme B: the K codes too)
            codes = Hkv * T * D + (Hkv * T * D + scales if wl.scheme == "A" else Hkv * T * D)
        return 2 * Hkv * T * D * 2 + codes + Hkv * T * 4 + q
    if role == "v_codes":  # V (bf16) in, V codes out; scheme B: K and V in one launch
        n = 2 if wl.scheme == "B" else 1
        return n * (Hkv * T * D * 2 + Hkv * T * D + 4)
    if role == "amax":  # scheme B: K and V in (their maxima)
        return 2 * Hkv * T * D * 2
    if role == "k_codes":  # K and V in (max|V| on the way), K codes and scales out
        return 2 * Hkv * T * D * 2 + Hkv * T * D + scales
    if role == "score":  # INT8 K codes, value norms and scales in; scores out
        return Hkv * T * D + Hkv * T * 4 + scales + q + Hkv * T * 4
    if role == "decode":
        return algorithmic_bytes(wl, lengths)["decode"]
    return None


def demangle(names):
    try:
        r = subprocess.run(["c++filt"], input="\n".join(names), capture_output=True, text=True, timeout=30)
        out = r.stdout.splitlines()
        if r.returncode == 0 and len(out) == len(names):
            return out
    except (OSError, subprocess.SubprocessError):
        pass
    return list(names)


# ------------------------------------------------------------------------------------------------
# clocks
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"sgd_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
class Pipeline:
    """Device buffers and the three C-ABI calls of one step (outputs and workspaces reused)."""

    def __init__(self, sgd, wl, bt, dev):
        self.sgd, self.wl, self.bt, self.dev = sgd, wl, bt, dev
        self.lengths = [int(x) for x in bt.lengths]
        self.q = bt.q.to(dev)
        self.k = bt.k.to(dev)
        self.v = bt.v.to(dev)
        self.cu = bt.cu_seqlens.to(dev)
        self.parts = sgd.n_parts(self.lengths)
        self.qout = self.kept = None
        self.ws_q = self.ws_s = self.ws_d = None
        self.sel_out = None
        self.dec_out = None
        self.stage_events = {}
        self.cal = {}
        if wl.calibrated:
            # per-tensor scales calibrated once, before the steps (untimed), from the same cache
            _, _, ks, vs, _ = sgd.quantize_kv(self.k, self.v, self.cu, wl.scheme, self.lengths)
            self.cal = {"v_scale_in": vs.clone()}
            if wl.scheme == "B":
                self.cal["k_scale_in"] = ks.clone()
            torch.cuda.synchronize(dev)
        if wl.select_on_codes:
            # a cache quantised once, before the steps (untimed), with its value norms
            self.vn = torch.empty(self.k.shape[:2], dtype=torch.float32, device=dev)
            self.kc, self.vc, self.ks, self.vs, _ = sgd.quantize_kv(self.k, self.v, self.cu, wl.scheme,
                                                                    self.lengths, v_norm=self.vn)
            torch.cuda.synchronize(dev)
            del self.k, self.v

    def inputs(self):
        """The device tensors a step reads (for the end-to-end copies)."""
        if self.wl.select_on_codes:
            return [self.q, self.kc, self.vc, self.ks, self.vs, self.vn, self.cu]
        return [self.q, self.k, self.v, self.cu]

    def run(self, record=None):
        """One step.  record: dict stage -> (start_event, end_event) to time each stage."""
        sgd, wl = self.sgd, self.wl

        def ev(name, i):
            if record is not None:
                record[name][i].record()

        idx = cu_kept = None
        Kt = 0
        if wl.select_on_codes:  # the cache is INT8 already: select on its codes
            kc, vc, ks, vs = self.kc, self.vc, self.ks, self.vs
            ev("select", 0)
            select = sgd.oam_select_blocks if wl.blocks else sgd.oam_select
            idx, cu_kept, self.ws_s = select(self.q, kc, vc, self.cu, wl.G, wl.beta, wl.eps, wl.keep_num,
                                             wl.keep_den, self.lengths, out=self.sel_out, workspace=self.ws_s,
                                             k_scale=ks, v_scale=vs, scheme=wl.scheme, n_parts_=self.parts,
                                             v_norm=self.vn)
            self.sel_out = (idx, cu_kept)
            Kt = idx.shape[1]
            ev("select", 1)
        elif wl.scheme and wl.oam:
            ev("quantize_select", 0)
            kc, vc, ks, vs, idx, cu_kept, self.ws_q = sgd.quantize_select(
                self.q, self.k, self.v, self.cu, wl.G, wl.beta, wl.eps, wl.keep_num, wl.keep_den, wl.scheme,
                self.lengths, out=self.qout, workspace=self.ws_q, **self.cal)
            self.qout = (kc, vc, ks, vs, idx, cu_kept)
            Kt = idx.shape[1]
            ev("quantize_select", 1)
        elif wl.scheme:
            ev("quantize", 0)
            kc, vc, ks, vs, self.ws_q = sgd.quantize_kv(self.k, self.v, self.cu, wl.scheme, self.lengths,
                                                        out=self.qout, workspace=self.ws_q)
            self.qout = (kc, vc, ks, vs)
            ev("quantize", 1)
        elif wl.oam:
            kc, vc, ks, vs = self.k, self.v, None, None
            ev("select", 0)
            idx, cu_kept, self.ws_s = sgd.oam_select(self.q, self.k, self.v, self.cu, wl.G, wl.beta, wl.eps,
                                                     wl.keep_num, wl.keep_den, self.lengths, out=self.sel_out,
                                                     workspace=self.ws_s)
            self.sel_out = (idx, cu_kept)
            Kt = idx.shape[1]
            ev("select", 1)
        else:
            kc, vc, ks, vs = self.k, self.v, None, None
        ev("decode", 0)
        if wl.blocks:
            o, lse, self.ws_d = sgd.decode_attn_blocks(self.q, wl.G, kc, vc, self.cu, idx, cu_kept, k_scale=ks,
                                                       v_scale=vs, scheme=wl.scheme, n_parts_=self.parts,
                                                       out=self.dec_out, workspace=self.ws_d)
            self.dec_out = (o, lse)
            ev("decode", 1)
            return o, lse
        decode = sgd.decode_attn if wl.M == 1 else sgd.decode_attn_multi
        o, lse, self.ws_d = decode(self.q, wl.G, kc, vc, self.cu, k_scale=ks, v_scale=vs,
                                            scheme=wl.scheme or "A", n_parts_=self.parts, idx=idx,
                                            cu_kept=cu_kept, kept_total_=Kt, out=self.dec_out,
                                            workspace=self.ws_d, q_quant=wl.q_quant or "none")
        self.dec_out = (o, lse)
        ev("decode", 1)
        return o, lse

    def launches_per_step(self):
        # decode: plan + the tensor-core decode, which merges each row itself (D = 128, bf16 q)
        if self.wl.select_on_codes:  # plan, INT8 score, (block max,) top-K; plan, decode
            return (4 if self.wl.blocks else 3) + 2
        if self.wl.scheme and self.wl.oam:
            return 4 + 2  # plan, score+quantize, V codes, top-K; plan, decode
        return (3 if self.wl.scheme else 0) + (3 if self.wl.oam else 0) + 2


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, torch copy)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (MEASURED_PEAKS.json absent)"


def load_traffic(key, wl_name, kind="kernels"):
    """DRAM bytes per launch of a kernel role (kind "kernels") or per call of a stage ("stages")
    from a committed ncu summary, if the sources it was taken from are unchanged."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        d = json.load(open(path))
    except (OSError, ValueError):
        return None
    ent = d.get(wl_name, {}).get(kind, {}).get(key)
    if not ent:
        return None
    srcs = [os.path.join(ROOT, p) for p in ent["sources"]]
    if source_hash(srcs) != ent["source_hash"]:
        return None
    return ent["bytes_per_launch"]


def oracle_row(bt, wl, b, h):
    """The whole path of one (sequence, KV head) row in the fp64 oracle, as the step runs it on the
    GPU; returns the row's algorithmic bytes."""
    import oracle
    cu = bt.cu_seqlens.numpy().astype(np.int64)
    s, e = int(cu[b]), int(cu[b + 1])
    L = e - s
    kk = bt.k[h:h + 1, s:e]
    vv = bt.v[h:h + 1, s:e]
    one = np.array([0, L], np.int64)
    qrow = bt.q[b:b + 1, ..., h * wl.G:(h + 1) * wl.G, :]  # [1, (M,) G, D]
    rowwl = wl.with_(B=1, Hkv=1, lengths=(L,), length_range=None)
    quant = None
    if wl.scheme:
        quant = oracle.quantize_kv(kk, vv, one, wl.scheme)
    idx = cu_kept = None
    if wl.oam and wl.select_on_codes:
        idx, cu_kept, sc = oracle.oam_select_int8(qrow, quant[0], quant[2], vv, one, wl.scheme, wl.G, wl.beta,
                                                  wl.eps, wl.keep_num, wl.keep_den)
        if wl.blocks:
            blk, cu_b, _ = oracle.select_blocks(sc, one, 1, wl.keep_num, wl.keep_den)
            oracle.decode_blocks(qrow, kk, vv, one, wl.G, blk, cu_b, quant=(*quant, wl.scheme))
            return sum(algorithmic_bytes(rowwl, [L]).values())
    elif wl.oam:
        idx, cu_kept, _ = oracle.oam_select(qrow, kk, vv, one, wl.G, wl.beta, wl.eps, wl.keep_num, wl.keep_den)
    if wl.q_quant:  # the attention sees the query's code * scale
        qrow = oracle.dequant_q(*oracle.quantize_q(qrow, wl.q_quant))
    if wl.M > 1:
        oracle.decode_multi(qrow, kk, vv, one, wl.G, wl.M, idx=idx, cu_kept=cu_kept,
                            quant=None if quant is None else (*quant, wl.scheme))
    else:
        oracle.decode(qrow, kk, vv, one, wl.G, idx=idx, cu_kept=cu_kept,
                      quant=None if quant is None else (*quant, wl.scheme))
    return sum(algorithmic_bytes(rowwl, [L]).values())


def cpu_baseline_sample(bt, wl, budget_s=20.0, max_rows=None, rows=None, threads=1):
    """The fp64 oracle on a bounded sample of the workload's rows, shortest rows first, one row per
    host thread at a time (the oracle's C loops run without the GIL); rows not started when the
    budget runs out are left out.  Returns (GB/s, sample text, seconds, threads used)."""
    import concurrent.futures
    import oracle
    oracle.lib()  # compiled and loaded before any thread starts
    cu = bt.cu_seqlens.numpy().astype(np.int64)
    order = rows or [(b, h) for h in range(wl.Hkv) for b in range(wl.B)]
    order = sorted(order, key=lambda r: int(cu[r[0] + 1] - cu[r[0]]))  # shortest rows first
    if max_rows is not None:
        order = order[:max_rows]
    threads = max(1, min(int(threads), len(order)))
    t0 = time.perf_counter()
    deadline = t0 + budget_s

    def job(r):
        if time.perf_counter() > deadline:
            return None
        return r, oracle_row(bt, wl, *r)

    done = []
    if threads == 1:
        for r in order:
            done.append(job(r))
            if time.perf_counter() > deadline:
                break
    else:
        with concurrent.futures.ThreadPoolExecutor(threads) as ex:
            done = list(ex.map(job, order))
    done = [d for d in done if d is not None]
    dt = time.perf_counter() - t0
    nbytes = sum(n for _, n in done)
    tokens = sum(int(cu[b + 1] - cu[b]) for (b, _), _ in done)
    sample = (f"{len(done)} (sequence, KV head) rows of the workload, shortest first, {tokens} tokens, the whole "
              f"path per row in the fp64 oracle on {threads} host thread(s) (one row per thread); {dt:.1f} s")
    return nbytes / dt / 1e9, sample, dt, threads


def reduce_max(x, dev, world):
    """The maximum of x over all ranks (x itself for one rank): every timing is the slowest rank's."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_gbs(step_bytes, steps, total_ms, world):
    """Whole-job GB/s: each of `world` ranks moves step_bytes per step over `steps` steps, in the
    slowest rank's total_ms (weak scaling: the per-rank work is fixed)."""
    return world * step_bytes * steps / (total_ms / 1e3) / 1e9


def fractions(gbs, peak, read_only):
    """A rate against the three denominators: the measured copy, the read-only stream, nominal."""
    d = {"frac_of_hbm": round(gbs / peak, 4), "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4)}
    if read_only:
        d["frac_of_read_only"] = round(gbs / read_only, 4)
    return d


def read_only_ceiling(sgd, dev, reps=10):
    """The read-only HBM rate of the library's streaming kernel (sgd_stream_read) over 4 GiB, both
    of its methods, best of `reps` launches each (CUDA events on the launching stream)."""
    buf = torch.randint(0, 256, (READ_ONLY_BYTES,), dtype=torch.uint8, device=dev)
    sink = torch.zeros(1, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    res = {}
    for method, name in ((0, "vector_loads"), (1, "bulk_copies")):
        for _ in range(3):
            sgd.stream_read(buf, method, sink, status)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            a.record()
            sgd.stream_read(buf, method, sink, status)
            b.record()
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b in ev]
        res[name] = {"GB_s": round(READ_ONLY_BYTES / (min(ms) / 1e3) / 1e9, 1),
                     "median_GB_s": round(READ_ONLY_BYTES / (statistics.median(ms) / 1e3) / 1e9, 1)}
    if int(status.item()) != 0:
        raise RuntimeError(f"stream read status {int(status.item()):#x}")
    del buf
    best = max(r["GB_s"] for r in res.values())
    return {"GB_s": best, "bytes": READ_ONLY_BYTES, **res,
            "how": "sgd_stream_read over 4 GiB of device memory, every byte read once and XOR-folded; best of "
                   f"{reps} launches per method (CUDA events)"}


def decode_stage_record(sgd, n, dev, K, W, flush_l2, peak, read_only, world):
    """The decode stage of workload n over its INT8 cache (quantised once, untimed): sgd_decode_attn
    timed as a call (plan + decode kernels) and per kernel, L2 flushed before each call."""
    wl = workloads.config(n)
    bt = workloads.generate(wl, seed=wl.seed if wl.seed is not None else n)
    lengths = [int(x) for x in bt.lengths]
    q, cu = bt.q.to(dev), bt.cu_seqlens.to(dev)
    k, v = bt.k.to(dev), bt.v.to(dev)
    del bt
    kc, vc, ks, vs, wsq = sgd.quantize_kv(k, v, cu, wl.scheme, lengths)
    if sgd.workspace_status(wsq):
        raise RuntimeError(f"quantize status on workload {n}")
    del k, v
    kw = dict(k_scale=ks, v_scale=vs, scheme=wl.scheme, n_parts_=sgd.n_parts(lengths))
    state = {"out": None, "ws": None}

    def call():
        o, l, state["ws"] = sgd.decode_attn(q, wl.G, kc, vc, cu, out=state["out"], workspace=state["ws"], **kw)
        state["out"] = (o, l)

    for _ in range(max(W, 3)):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i, (a, b) in enumerate(ev):
        flush_l2(i)
        a.record()
        call()
        b.record()
    torch.cuda.synchronize()
    call_ms = reduce_max(statistics.median([a.elapsed_time(b) for a, b in ev]), dev, world)
    kern = {}
    for i in range(K):
        flush_l2(i)
        sgd.kernel_timing_start(16)
        call()
        got = sgd.kernel_timing_stop()
        for (name, ms), dn in zip(got, demangle([x for x, _ in got])):
            kern.setdefault(kernel_role(dn), {"name": dn.split("(")[0], "ms": []})["ms"].append(ms)
    if sgd.workspace_status(state["ws"]):
        raise RuntimeError(f"decode status on workload {n}")
    nbytes = algorithmic_bytes(wl, lengths)["decode"]
    dk = kern.get("decode", {"name": "?", "ms": [float("nan")]})
    k_ms = reduce_max(statistics.mean(dk["ms"]), dev, world)
    k_gbs = nbytes / (k_ms / 1e3) / 1e9
    c_gbs = nbytes / (call_ms / 1e3) / 1e9
    rec = {"workload": wl.name, "B": wl.B, "Hkv": wl.Hkv, "G": wl.G, "D": wl.D, "T": int(sum(lengths)),
           "lengths": lengths, "scheme": wl.scheme,
           "step": "sgd_decode_attn over the INT8 scheme-A cache, equal-work split over all SMs (cache quantised "
                   "once, untimed; L2 flushed before each call)",
           "algorithmic_bytes": nbytes,
           "kernel": dk["name"], "kernel_ms": round(k_ms, 4), "kernel_GB_s": round(k_gbs, 1),
           **fractions(k_gbs, peak, read_only),
           # DRAM bytes per launch from the committed ncu record (None once the kernel's sources change)
           "traffic": load_traffic("decode", wl.name),
           "call_ms": round(call_ms, 4), "call_GB_s": round(c_gbs, 1),
           "call_frac_of_hbm": round(c_gbs / peak, 4),
           "other_kernels_ms": {r: round(statistics.mean(e["ms"]), 4) for r, e in kern.items() if r != "decode"},
           "seq_heads_per_s": round(wl.B * wl.Hq / (call_ms / 1e3), 1)}
    del q, cu, kc, vc, ks, vs, state
    torch.cuda.empty_cache()
    return rec


def capture_step(pipe, dev):
    """The step's C-ABI calls captured once in a CUDA graph (the library is stream-ordered,
    allocates nothing and never synchronises); the timed steps replay it.  Returns (graph or None,
    how the timed steps launch)."""
    graph, launch = None, "CUDA graph replay of the step's C-ABI calls"
    try:
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            pipe.run()
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            pipe.run()
        graph = g
    except RuntimeError as exc:
        launch = "eager C-ABI calls (graph capture failed: " + str(exc).splitlines()[0][:120] + ")"
    torch.cuda.synchronize()
    return graph, launch


def kept_rows(idx, cu_kept, cu_seqlens, T):
    """Cache row numbers (kvh * T + token) of every kept token: the rows a kept-set decode reads
    from the K codes and from the V codes.  idx [Hkv, Kt] (positions within their sequence),
    cu_kept / cu_seqlens [B+1]."""
    Hkv, Kt = idx.shape
    col = torch.arange(Kt, device=idx.device, dtype=torch.int64)
    seq = torch.searchsorted(cu_kept.to(torch.int64), col, right=True) - 1  # sequence of each kept column
    start = cu_seqlens.to(torch.int64)[seq]
    head = torch.arange(Hkv, device=idx.device, dtype=torch.int64)[:, None] * T
    return (head + start[None, :] + idx.to(torch.int64)).to(torch.int32).reshape(-1)


def gather_ceiling(sgd, pipe, flush_l2, reps=10):
    """The scattered-row read ceiling for the step's kept-set decode: sgd_gather_read over the same
    K and V code rows, L2 flushed before each call, best of `reps` (CUDA events)."""
    wl = pipe.wl
    if wl.select_on_codes:
        kc, vc, (idx, cu_kept) = pipe.kc, pipe.vc, pipe.sel_out
    else:
        kc, vc, idx, cu_kept = pipe.qout[0], pipe.qout[1], pipe.qout[4], pipe.qout[5]
    rows = kept_rows(idx, cu_kept, pipe.cu, kc.shape[1])
    dense = torch.arange(rows.numel(), dtype=torch.int32, device=rows.device)  # control: the same count, contiguous
    row_bytes = kc.shape[2] * kc.element_size()

    def best_ms(r):
        sgd.gather_read(kc, r, row_bytes, b=vc)  # checked once, untimed
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i, (a, b) in enumerate(ev):
            flush_l2(i)
            a.record()
            sgd.gather_read(kc, r, row_bytes, b=vc, check=False)
            b.record()
        torch.cuda.synchronize()
        return min(a.elapsed_time(b) for a, b in ev)

    ms, ms_dense = best_ms(rows), best_ms(dense)
    nbytes = 2 * rows.numel() * row_bytes
    # second control: the vector stream (sgd_stream_read, no indices) over as many bytes of the codes
    flat = kc.reshape(-1)[: nbytes // 16 * 16]
    sink = torch.zeros(1, dtype=torch.int64, device=kc.device)
    status = torch.zeros(1, dtype=torch.int32, device=kc.device)
    sgd.stream_read(flat, 0, sink, status)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for i, (a, b) in enumerate(ev):
        flush_l2(i)
        a.record()
        sgd.stream_read(flat, 0, sink, status)
        b.record()
    torch.cuda.synchronize()
    ms_stream = min(a.elapsed_time(b) for a, b in ev)
    return {"GB_s": round(nbytes / (ms / 1e3) / 1e9, 1), "bytes": nbytes, "rows": 2 * rows.numel(),
            "row_bytes": row_bytes, "ms": round(ms, 4),
            "dense_control_GB_s": round(nbytes / (ms_dense / 1e3) / 1e9, 1), "dense_control_ms": round(ms_dense, 4),
            "stream_control_GB_s": round(flat.numel() / (ms_stream / 1e3) / 1e9, 1),
            "stream_control_ms": round(ms_stream, 4),
            "how": "sgd_gather_read over the kept tokens' K and V code rows (16-byte loads, indices of each batch "
                   "first); controls: as many rows from the start of each tensor, contiguous, and the vector stream "
                   f"of sgd_stream_read over as many bytes; L2 flushed before each call, best of {reps}"}


def calibrated_record(sgd, dev, K, W, flush_l2, peak, read_only, world, ref=None):
    """The headline step with calibrated per-tensor scales (workload 15: workload 5's batch, its V
    scale calibrated once, untimed, from the same cache, so every code equals the computed-scale
    step's): one pass writes every code, so the select stage reads K and V once.  Timed like the
    headline step (graph replay, L2 flushed before each step), and per kernel."""
    wl = workloads.config(CALIBRATED_WORKLOAD)
    bt = workloads.generate(wl, seed=wl.seed)
    pipe = Pipeline(sgd, wl, bt, dev)
    step_bytes = sum(algorithmic_bytes(wl, pipe.lengths).values())
    del bt
    for _ in range(max(W, 3)):
        pipe.run()
    graph, launch = capture_step(pipe, dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i, (a, b) in enumerate(ev):
        flush_l2(i)
        a.record()
        if graph is not None:
            graph.replay()
        else:
            pipe.run()
        b.record()
    torch.cuda.synchronize()
    ms = reduce_max(sum(a.elapsed_time(b) for a, b in ev), dev, world) / K
    kern = {}
    for i in range(K):
        flush_l2(i)
        sgd.kernel_timing_start(64)
        pipe.run()
        got = sgd.kernel_timing_stop()
        for (name, kms), dn in zip(got, demangle([x for x, _ in got])):
            kern.setdefault(kernel_role(dn), {"name": dn.split("(")[0], "ms": []})["ms"].append(kms)
    for who in (pipe.ws_q, pipe.ws_d):
        if sgd.workspace_status(who):
            raise RuntimeError(f"device status {sgd.workspace_status(who):#x} in the calibrated step")
    kernels = {}
    for role, e in kern.items():
        kernels[role] = {"kernel": e["name"], "ms_per_launch": round(statistics.mean(e["ms"]), 4),
                         "launches_per_step": len(e["ms"]) // K}
        kb = kernel_bytes(wl, pipe.lengths, role) if len(e["ms"]) == K else None
        if kb is not None:
            gbs = kb / (statistics.mean(e["ms"]) / 1e3) / 1e9
            kernels[role].update({"algorithmic_bytes": kb, "GB_s": round(gbs, 1), **fractions(gbs, peak, read_only),
                                  "traffic": load_traffic(role, wl.name)})
    gbs = world * step_bytes / (ms / 1e3) / 1e9
    rec = {"workload": wl.name, "scheme": wl.scheme + " with the V scale calibrated",
           "step": "sgd_quantize_select with a calibrated V scale (one pass: score, K codes and scales, V codes) "
                   "-> sgd_decode_attn over the kept tokens; the scale calibrated once, untimed, from the same "
                   "cache", "launch": launch, "ms_per_step": round(ms, 4), "algorithmic_bytes": step_bytes,
           "GB_s": round(gbs, 1), **fractions(gbs, peak, read_only), "kernels": kernels}
    if ref is not None and ref.wl.name == workloads.config(5).name:
        rec["codes_equal_computed_scale_step"] = bool(all(torch.equal(a, b) for a, b in zip(pipe.qout, ref.qout)))
    del pipe
    torch.cuda.empty_cache()
    return rec


def run_ours(args, rank, world, local_rank):
    import sparse_gqa_decode_b200 as sgd

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = scaled(workloads.config(args.workload), args.scale)
    bt = workloads.generate(wl, seed=wl.seed if wl.seed is not None else args.workload)  # the same batch on every rank
    pipe = Pipeline(sgd, wl, bt, dev)
    stages = algorithmic_bytes(wl, pipe.lengths)
    step_bytes = sum(stages.values())
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2(i):
        """Evict the previous step's lines from L2 (untimed): a 256 MiB write, then a 256 MiB
        read, so that L2 holds clean lines and the timed step pays no write-back of the flush."""
        flush.fill_(i & 0xff)
        torch.sum(flush_r, dim=0, out=sink)

    for _ in range(max(args.warmup, 3)):
        pipe.run()
    torch.cuda.synchronize()
    st = sgd.workspace_status(pipe.ws_d)
    if st:
        raise RuntimeError(f"device status {st:#x} after warm-up")

    graph, launch = capture_step(pipe, dev)

    names = [n for n in ("quantize_select", "quantize", "select", "decode") if n in stages]
    K = args.steps
    rec = [{n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in names}
           for _ in range(K)]
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    eager_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for i in range(K):
        flush_l2(i)
        step_ev[i][0].record()
        if graph is not None:
            graph.replay()
        else:
            pipe.run()
        step_ev[i][1].record()
    for i in range(K):  # the same steps as eager calls, timed per stage
        flush_l2(i)
        eager_ev[i][0].record()
        pipe.run(rec[i])
        eager_ev[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    # per kernel: the same eager steps once more with every library launch bracketed by events
    # on its stream (outside the timed region above)
    per_kernel = {}
    for i in range(K):
        flush_l2(i)
        sgd.kernel_timing_start(64)
        pipe.run()
        got = sgd.kernel_timing_stop()
        for (name, ms), dn in zip(got, demangle([n for n, _ in got])):
            ent = per_kernel.setdefault(kernel_role(dn), {"name": dn.split("(")[0], "ms": [], "per_step": 0})
            ent["ms"].append(ms)
    for ent in per_kernel.values():
        ent["per_step"] = len(ent["ms"]) // K
    st = sgd.workspace_status(pipe.ws_d)
    if st:
        raise RuntimeError(f"device status {st:#x} after the timed steps")
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    stage_ms = {n: [r[n][0].elapsed_time(r[n][1]) for r in rec] for n in names}
    total_ms = reduce_max(sum(step_ms), dev, world)
    ms_per_step = total_ms / K
    value = job_gbs(step_bytes, K, total_ms, world)
    eager_ms = reduce_max(sum(a.elapsed_time(b) for a, b in eager_ev), dev, world) / K

    # e2e: host buffers through the same calls, copies inside the timed region
    dev_in = pipe.inputs()
    pin_in = [x.cpu().pin_memory() for x in dev_in]
    h_out = torch.empty(tuple(bt.q.shape), dtype=torch.float32).pin_memory()  # [B, (M,) Hq, D]
    h_lse = torch.empty(tuple(bt.q.shape[:-1]), dtype=torch.float32).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in pin_in)
    d2h = h_out.numel() * 4 + h_lse.numel() * 4
    e2e_steps = max(2, min(K, 5))
    for _ in range(2):
        for d_t, h_t in zip(dev_in, pin_in):
            d_t.copy_(h_t, non_blocking=True)
        o, lse = pipe.run()
        h_out.copy_(o, non_blocking=True)
        h_lse.copy_(lse, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        for d_t, h_t in zip(dev_in, pin_in):
            d_t.copy_(h_t, non_blocking=True)
        o, lse = pipe.run()
        h_out.copy_(o, non_blocking=True)
        h_lse.copy_(lse, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, dev, world)

    # the read-only ceiling and the INT8 decode stages (every rank takes the same steps)
    peak, peak_src = load_peaks()
    ro, north, calibrated = None, {}, None
    if not args.no_extra_records:
        ro = read_only_ceiling(sgd, dev)
        for n in INT8_DECODE_WORKLOADS:
            rec = decode_stage_record(sgd, n, dev, K, args.warmup, flush_l2, peak, ro["GB_s"], world)
            north[rec["workload"]] = rec
        if args.scale == 1.0 and not wl.calibrated:
            calibrated = calibrated_record(sgd, dev, K, args.warmup, flush_l2, peak, ro["GB_s"], world, ref=pipe)
    ro_gbs = ro["GB_s"] if ro else None
    # the scattered-row ceiling of the kept-set decode (INT8 codes of kept tokens)
    gather = None
    if wl.oam and wl.scheme and not wl.blocks and wl.M == 1 and args.scale == 1.0:
        gather = gather_ceiling(sgd, pipe, flush_l2)
        gather["GB_s"] = round(-reduce_max(-gather["GB_s"], dev, world), 1)  # the slowest rank's

    if rank != 0:
        return None
    med = {n: statistics.median(v) for n, v in stage_ms.items()}
    dom = max(med, key=lambda n: med[n])
    achieved = stages[dom] / (med[dom] / 1e3) / 1e9
    # the dominant kernel: the largest time per step among the library's kernels
    kern_report = {}
    for role, ent in per_kernel.items():
        kern_report[role] = {"kernel": ent["name"], "launches_per_step": ent["per_step"],
                             "ms_per_launch": round(statistics.mean(ent["ms"]), 4),
                             "ms_per_step": round(sum(ent["ms"]) / K, 4)}
        kb = kernel_bytes(wl, pipe.lengths, role) if ent["per_step"] == 1 else None
        if kb is not None:
            gbs = kb / (statistics.mean(ent["ms"]) / 1e3) / 1e9
            kern_report[role].update({"algorithmic_bytes": kb, "GB_s": round(gbs, 1), **fractions(gbs, peak, ro_gbs)})
    if gather and "GB_s" in kern_report.get("decode", {}):
        kern_report["decode"]["frac_of_gather_ceiling"] = round(kern_report["decode"]["GB_s"] / gather["GB_s"], 4)
    dom_k = max(kern_report, key=lambda r: kern_report[r]["ms_per_step"]) if kern_report else None
    kernels = {"quantize_select": "sgd_quantize_select (plan + fused OAM score/K quantise + V codes + top-K)",
               "quantize": "sgd_quantize_kv (prep + K-partition + V kernels)",
               "select": "sgd_oam_select (plan + OAM score + top-K kernels)",
               "decode": "sgd_decode_attn (plan + split decode + merge kernels)"}
    traffic = load_traffic(dom, wl.name, "stages")
    stage_report = {}
    for n in names:
        gbs = stages[n] / (med[n] / 1e3) / 1e9
        stage_report[n] = {"ms": round(med[n], 4), "algorithmic_bytes": stages[n], "GB_s": round(gbs, 1),
                           **fractions(gbs, peak, ro_gbs)}
    line = {
        "metric": "decode-attn KV GB/s & % of B200 HBM peak at 128K; seq·heads/s, INT8+OAM",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8" if wl.scheme else "bf16",
        "data": "synthetic",
        "config": {
            "workload": wl.name, "B": wl.B, "Hkv": wl.Hkv, "G": wl.G, "D": wl.D, "lengths": pipe.lengths,
            "T": int(sum(pipe.lengths)), "scheme": wl.scheme, "oam": wl.oam, "beta": wl.beta, "eps": wl.eps,
            "keep": f"{wl.keep_num}/{wl.keep_den}", "seed": wl.seed if wl.seed is not None else args.workload, "q_quant": wl.q_quant,
            "query_tokens": wl.M,
            "step": ("oam_select_blocks(int8 cache, stored norms) -> decode_attn_blocks(kept 64-token blocks); "
                     "cache quantised once, untimed" if wl.blocks else
                     "oam_select(int8 cache, stored norms) -> decode_attn(kept); cache quantised once, untimed"
                     if wl.select_on_codes else
                     "quantize_select -> decode_attn(kept)" if wl.oam else "quantize_kv -> decode_attn"),
            "l2": "flushed between steps (untimed 256 MiB write then 256 MiB read: L2 left clean); inputs > L2",
            "parallelism": f"dp{world} (independent copies, no collective)",
            "launch": launch,
            **({"length_scale": args.scale} if args.scale != 1.0 else {}),
        },
        "eager_ms_per_step": round(eager_ms, 4),
        "pct_hbm_peak": round(100 * value / world / peak, 2),
        "pct_nominal": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        # the decode over the kept (or all) tokens alone, beside the whole step's rate
        "decode_stage_GB_s": stage_report["decode"]["GB_s"],
        "decode_stage_frac_of_hbm": stage_report["decode"]["frac_of_hbm"],
        "seq_heads_per_s": round(world * wl.B * wl.Hq / (ms_per_step / 1e3), 1),
        "stages": stage_report,
        "kernels": kern_report,
        "roofline": ({"bound": "hbm", "kernel": kern_report[dom_k]["kernel"], "role": dom_k,
                      "achieved": kern_report[dom_k]["GB_s"], "peak": peak, "peak_source": peak_src, "unit": "GB/s",
                      "frac": kern_report[dom_k]["frac_of_hbm"],
                      "frac_of_nominal": kern_report[dom_k]["frac_of_nominal"],
                      "frac_of_read_only": kern_report[dom_k].get("frac_of_read_only"),
                      "traffic": load_traffic(dom_k, wl.name),
                      "algorithmic_bytes": kern_report[dom_k]["algorithmic_bytes"],
                      "launch_ms": kern_report[dom_k]["ms_per_launch"],
                      "timing": "CUDA events around each launch on its stream, eager steps, L2 flushed between steps"}
                     if dom_k is not None and "GB_s" in kern_report[dom_k] else
                     {"bound": "hbm", "kernel": kernels[dom], "achieved": round(achieved, 1), "peak": peak,
                      "peak_source": peak_src, "unit": "GB/s", "frac": round(achieved / peak, 4),
                      "traffic": traffic, "algorithmic_bytes": stages[dom]}),
        "stage_roofline": {"stage": dom, "calls": kernels[dom], "achieved": round(achieved, 1),
                           "frac": round(achieved / peak, 4), "traffic": traffic, "algorithmic_bytes": stages[dom]},
        "e2e": {"value": round(job_gbs(step_bytes, 1, e2e_ms, world), 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        # library launches per step as the per-launch timing counted them (the step's kernel list)
        "gpu_launches": (sum(e["per_step"] for e in per_kernel.values()) or pipe.launches_per_step()) * K,
        "clocks": clk,
        "read_only": ro,
        "gather_ceiling": gather,
        "nominal_hbm_GB_s": NOMINAL_HBM_GBS,
        # the 128K INT8 split-KV decode stages, dense (workload 4) and ragged (workload 14)
        "int8_decode_stages": north or None,
        "calibrated_scales": calibrated,
    }
    if world == 1 and not args.no_cpu_baseline:
        host = os.cpu_count() or 1
        v, sample, _, used = cpu_baseline_sample(bt, wl, budget_s=15.0, threads=host)
        v1, sample1, _, _ = cpu_baseline_sample(bt, wl, budget_s=10.0, threads=1)
        line["cpu_baseline"] = {"value": round(v, 4), "unit": "GB/s", "cores": used, "host_cpu_count": host,
                                "kind": "oracle", "sample": sample,
                                "one_thread": {"value": round(v1, 4), "unit": "GB/s", "cores": 1, "sample": sample1}}
    return line


# ------------------------------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores, one bounded sample of the workload per step
# ------------------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands on the host cores.  Each step runs the whole
    path for the min(host CPUs, rows) shortest (sequence, KV head) rows of the workload, one row per
    host thread (for the default workload's 32 rows and a host with at least 32 CPUs: the whole
    batch)."""
    if rank != 0:
        return None
    wl = scaled(workloads.config(args.workload), args.scale)
    bt = workloads.generate(wl, seed=wl.seed if wl.seed is not None else args.workload)
    cu = bt.cu_seqlens.numpy()
    rows = sorted(((b, h) for h in range(wl.Hkv) for b in range(wl.B)), key=lambda r: int(cu[r[0] + 1] - cu[r[0]]))
    host = os.cpu_count() or 1
    n = min(host, len(rows))
    for _ in range(args.warmup):
        cpu_baseline_sample(bt, wl, budget_s=1e9, rows=rows[:1], threads=1)
    total_b, total_t, sample, used = 0.0, 0.0, "", 1
    for _ in range(args.steps):
        gbs, sample, dt, used = cpu_baseline_sample(bt, wl, budget_s=1e9, rows=rows[:n], threads=n)
        total_b += gbs * dt
        total_t += dt
    v = total_b / total_t
    line = {
        "impl": "reference",
        "metric": "decode-attn KV GB/s & % of B200 HBM peak at 128K; seq·heads/s, INT8+OAM",
        "value": round(v, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total_t / args.steps, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "Hkv": wl.Hkv, "G": wl.G, "D": wl.D,
                   "lengths": [int(x) for x in bt.lengths],
                   "parallelism": f"host cores ({used} threads, one row each; {host} CPUs on the host)"},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": used, "host_cpu_count": host,
                         "kind": "oracle", "sample": f"per step: {sample}"},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":  # rank 0 alone times the oracle; other ranks exit without work
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
