#!/usr/bin/env python
"""Benchmark of the SAW-INT4 KV-cache write/read hot path on B200.

One step = one pass of the whole path over one batch: the fused BDR + INT4 append
of every token of the batch into the paged cache (one kv_append_quant launch),
then one paged GQA decode step per sequence (kv_decode_attn: split + merge
kernels).  Default workload: 16 sequences with lengths ~U[512, 4096] (seed 0),
8 KV heads, 32 query heads, head_dim 128, page size 16, shuffled page table,
K/V ~ N(0,1) with 4 outlier channels per head x20, BDR block 128 on keys.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on the
host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_paged_kv_append_b200 import kvq, synth  # noqa: E402

METRIC = "INT4+BDR KV append tokens/s; paged decode attn HBM GB/s (% of ~8 TB/s)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
VARIANTS = [("bf16", kvq.KV_BF16, 0, False), ("int4", kvq.KV_INT4, 0, False)] + [
    (f"bdr{b}_{'kv' if rv else 'k'}", kvq.KV_INT4_BDR, b, rv) for b in (16, 32, 64, 128) for rv in (False, True)]
HEADLINE = "bdr128_k"


def peak_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {"append_kernel": ["kvq_append.cu", "kvq_common.cuh", "kvq_internal.h"],
                  "decode_mma_kernel": ["kvq_decode_mma.cu", "kvq_decode.cuh", "kvq_common.cuh", "kvq_internal.h"]}


def src_hash(kernel: str):
    """Hash of the sources one kernel is built from (the ncu counters are void once they change)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_paged_kv_append_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel][workload]
        if rec.get("src_sha") == src_hash(kernel):
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# --------------------------------------------------------------------------- workload

class Workload:
    def __init__(self, name: str, seed: int, device):
        self.wl = synth.WORKLOADS[name]
        self.name = name
        self.lengths = synth.seq_lengths(name, seed=seed)
        self.T = sum(self.lengths)
        self.B = len(self.lengths)
        self.H, self.Hq, self.ps = self.wl.num_kv_heads, self.wl.num_q_heads, self.wl.page_size
        # inputs below 1 GB are drawn on the CPU (identical on every machine), larger ones on the device
        gen_dev = "cpu" if self.T * self.H * 128 * 2 * 2 < (1 << 30) or device.type == "cpu" else device
        self.k, self.v = (t.to(device) for t in synth.make_kv(self.T, self.wl, seed, device=gen_dev, chunk=8192))
        pt, self.num_pages = synth.make_page_table(self.lengths, self.ps, seed)
        self.page_table = pt.to(device)
        ts, tp = synth.append_positions(self.lengths)
        self.tok_seq, self.tok_pos = ts.to(device), tp.to(device)
        self.q = synth.make_q(self.B, self.Hq, 128, seed).to(device)
        self.seq_lens = torch.tensor(self.lengths, dtype=torch.int32, device=device)
        self.max_len = max(self.lengths)

    def append_bytes(self, mode):
        # read K and V rows (2 x 256 B per head); write bf16 rows (2 x 256 B) or INT4 codes + scale/zero (2 x 68 B)
        write = 2 * 256 if mode == kvq.KV_BF16 else 2 * 68
        return self.T * self.H * (2 * 256 + write)

    def decode_bytes(self, mode):
        per_tok = self.H * (2 * 256 if mode == kvq.KV_BF16 else 2 * 68)
        pages = sum(-(-L // self.ps) for L in self.lengths)
        return self.T * per_tok + self.B * self.Hq * 128 * 2 * 2 + pages * 4


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms while running."""

    FIELDS = "clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, index: int):
        self.index, self.samples, self.proc = index, [], None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.index), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 6:
                self.samples.append(parts)

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[2 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


def make_cache(w: Workload, mode, b, rv, device):
    return kvq.PagedKVCache(w.num_pages, w.ps, w.H, w.Hq, mode, b, rv, device=device, fill=0)


def run_variant(w: Workload, mode, b, rv, steps, warmup, device, clocks=False):
    """Device-timed steps; returns per-kernel and per-step mean times (ms)."""
    cache = make_cache(w, mode, b, rv, device)
    ws, _ = cache.workspace(w.B, w.max_len, device)
    out = torch.empty(w.B, w.Hq, 128, dtype=torch.bfloat16, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]

    def step(e=None):
        if e: e[0].record(stream)
        cache.append(w.k, w.v, w.tok_seq, w.tok_pos, w.page_table, stream)
        if e: e[1].record(stream)
        kvq.kv_decode_attn(cache.handle, w.q, w.seq_lens, w.page_table, w.page_table.shape[1], w.B, w.max_len,
                           out, 0, ws, ws.numel(), stream)
        if e: e[2].record(stream)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    status = cache.get_error()
    if status != kvq.KV_OK:
        raise RuntimeError(f"device error after warm-up: {kvq.status_string(status)}")
    sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
    if sampler:
        sampler.__enter__()
        time.sleep(0.3)
    _barrier()
    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    for i in range(steps):
        flush.zero_()  # write 256 MiB > 126 MB L2 between timed steps
        step(evs[i])
    torch.cuda.synchronize(device)
    wall = time.perf_counter() - t0
    _barrier()
    if sampler:
        sampler.__exit__()
    app = np.array([e[0].elapsed_time(e[1]) for e in evs])
    dec = np.array([e[1].elapsed_time(e[2]) for e in evs])
    status = cache.get_error()
    cache.close()
    return {"append_ms": float(app.mean()), "decode_ms": float(dec.mean()), "step_ms": float((app + dec).mean()),
            "append_ms_median": float(np.median(app)), "decode_ms_median": float(np.median(dec)),
            "wall_s": wall, "status": status, "clocks": sampler.summary() if sampler else None}


def run_e2e(w: Workload, mode, b, rv, steps, warmup, device):
    """Same step through the C ABI with pinned HOST inputs: H2D copies of the step's inputs and a
    D2H read of the attention output are inside the timed region."""
    cache = make_cache(w, mode, b, rv, device)
    ws, _ = cache.workspace(w.B, w.max_len, device)
    host = {n: getattr(w, n).cpu().pin_memory() for n in ("k", "v", "tok_seq", "tok_pos", "page_table", "q",
                                                          "seq_lens")}
    dev = {n: torch.empty_like(t, device=device) for n, t in host.items()}
    out = torch.empty(w.B, w.Hq, 128, dtype=torch.bfloat16, device=device)
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    stream = torch.cuda.current_stream(device)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()

    def step():
        for n, t in host.items():
            dev[n].copy_(t, non_blocking=True)
        kvq.kv_append_quant(cache.handle, dev["k"], dev["v"], w.T, dev["tok_seq"], dev["tok_pos"],
                            dev["page_table"], w.page_table.shape[1], w.B, stream)
        kvq.kv_decode_attn(cache.handle, dev["q"], dev["seq_lens"], dev["page_table"], w.page_table.shape[1],
                           w.B, w.max_len, out, 0, ws, ws.numel(), stream)
        out_h.copy_(out, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    _barrier()
    ms = e0.elapsed_time(e1) / steps
    cache.close()
    return ms, h2d, d2h


# --------------------------------------------------------------------------- oracle (CPU)

def oracle_inputs(w: Workload):
    bits = lambda t: t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return dict(k=bits(w.k), v=bits(w.v), q=bits(w.q), ts=w.tok_seq.cpu().numpy(), tp=w.tok_pos.cpu().numpy(),
                pt=w.page_table.cpu().numpy())


def oracle_step_estimate(w: Workload, inp, mode, b, rv, tok_budget: int, row_budget: int):
    """Run the oracle on a bounded sample (the first tok_budget tokens appended, row_budget
    decode rows) and return (seconds one full step would take, sample description)."""
    import oracle

    H, ps, P = w.H, w.ps, w.num_pages
    if mode == kvq.KV_BF16:
        kp = np.zeros((P, H, ps, 128), np.uint16)
        ks = np.zeros(1, np.uint16)
    else:
        kp = np.zeros((P, H, ps, 64), np.uint8)
        ks = np.zeros((P, H, ps, 2), np.uint16)
    vp, vs = kp.copy(), ks.copy()
    n = max(1, min(tok_budget, w.T))
    t0 = time.perf_counter()
    oracle.append(mode, b, rv, kp, vp, ks, vs, inp["k"][:n], inp["v"][:n], inp["ts"][:n], inp["tp"][:n], inp["pt"])
    t_app = time.perf_counter() - t0
    rows_all = [(s, j) for s in range(w.B) for j in range(w.Hq)]
    rng = np.random.default_rng(0)
    r = max(1, min(row_budget, len(rows_all)))
    pick = [rows_all[i] for i in sorted(rng.choice(len(rows_all), r, replace=False))]
    t0 = time.perf_counter()
    oracle.decode(mode, b, rv, kp, vp, ks, vs, inp["q"], np.array(w.lengths), inp["pt"], H, rows=pick)
    t_dec = time.perf_counter() - t0
    est = t_app * (w.T / n) + t_dec * (len(rows_all) / r)
    sample = f"oracle append of {n}/{w.T} tokens + decode of {r}/{len(rows_all)} (seq, q-head) rows, " \
             f"1 thread, scaled to one full step"
    return est, sample


# --------------------------------------------------------------------------- dist

_dist = None


def _init_dist():
    global _dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        _dist = dist
    return ws


def _barrier():
    if _dist is not None:
        _dist.barrier()


def max_over_ranks(x: float, device) -> float:
    if _dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    _dist.all_reduce(t, op=_dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device) -> float:
    if _dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    _dist.all_reduce(t, op=_dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default="batch16", choices=list(synth.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    if args.impl == "reference":
        # the CPU oracle: rank 0 alone runs it, other ranks exit without work
        if int(os.environ.get("RANK", "0")) != 0:
            return
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")))

    world = _init_dist()
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    w = Workload(args.workload, args.seed + rank, device)

    res = run_variant(w, kvq.KV_INT4_BDR, 128, False, args.steps, args.warmup, device, clocks=True)
    step_ms = max_over_ranks(res["step_ms"], device)
    tokens = sum_over_ranks(w.T, device)
    value = tokens / (step_ms / 1e3)

    sweep = {}
    if not args.no_sweep:
        n = max(50, min(args.steps // 4, 500))
        for name, mode, b, rv in VARIANTS:
            r = res if name == HEADLINE else run_variant(w, mode, b, rv, n, 3, device)
            sweep[name] = {"append_tok_per_s": w.T / (r["append_ms"] / 1e3),
                           "append_gbs": w.append_bytes(mode) / (r["append_ms"] / 1e3) / 1e9,
                           "decode_gbs": w.decode_bytes(mode) / (r["decode_ms"] / 1e3) / 1e9,
                           "append_us": r["append_ms"] * 1e3, "decode_us": r["decode_ms"] * 1e3}
        if "int4" in sweep:
            sweep["bdr128_k_over_int4_append"] = sweep[HEADLINE]["append_tok_per_s"] / sweep["int4"]["append_tok_per_s"]

    e2e_ms, h2d, d2h = run_e2e(w, kvq.KV_INT4_BDR, 128, False, max(20, args.steps // 20), args.warmup, device)
    e2e_ms = max_over_ranks(e2e_ms, device)

    peak, peak_kind = peak_hbm()
    app_b, dec_b = w.append_bytes(kvq.KV_INT4_BDR), w.decode_bytes(kvq.KV_INT4_BDR)
    app_gbs = app_b / (res["append_ms"] / 1e3) / 1e9
    dec_gbs = dec_b / (res["decode_ms"] / 1e3) / 1e9
    dominant = "append" if res["append_ms"] >= res["decode_ms"] else "decode"
    dom_gbs = app_gbs if dominant == "append" else dec_gbs
    traffic = profiled_traffic("append_kernel" if dominant == "append" else "decode_mma_kernel", args.workload)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, int4+fp16 scale/zero cache, fp32 math", "data": "synthetic",
        "config": {"workload": args.workload, "description": w.wl.description, "variant": "INT4+BDR-128, keys only",
                   "sequences": w.B, "tokens_appended_per_step": w.T, "cached_tokens_decoded_per_step": w.T,
                   "num_kv_heads": w.H, "num_q_heads": w.Hq, "head_dim": 128, "page_size": w.ps,
                   "l2": "256 MiB buffer written between timed steps (L2 is 126 MB)",
                   "parallelism": f"{world} independent replica(s), one per GPU, no collective on the data path",
                   "seed": args.seed},
        "components": {
            "append": {"us": res["append_ms"] * 1e3, "tokens_per_s": w.T / (res["append_ms"] / 1e3),
                       "algorithmic_bytes": app_b, "gbs": app_gbs, "frac_of_peak": app_gbs / peak,
                       "frac_of_8tbs": app_gbs / NOMINAL_HBM_GBS},
            "decode": {"us": res["decode_ms"] * 1e3, "algorithmic_bytes": dec_b, "gbs": dec_gbs,
                       "frac_of_peak": dec_gbs / peak, "frac_of_8tbs": dec_gbs / NOMINAL_HBM_GBS,
                       "note": "split + merge kernels; reads the pages the append of the same step wrote"}},
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": dom_gbs, "peak": peak, "unit": "GB/s",
                     "frac": dom_gbs / peak, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                     "traffic": traffic},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": 3 * args.steps,
        "clocks": res["clocks"],
        "device_status": kvq.status_string(res["status"]),
    }
    if sweep:
        line["sweep"] = sweep
    if rank == 0 and world == 1 and not args.no_cpu:
        inp = oracle_inputs(w)
        est, sample = oracle_step_estimate(w, inp, kvq.KV_INT4_BDR, 128, False, tok_budget=w.T, row_budget=96)
        line["cpu_baseline"] = {"value": w.T / est, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if _dist is not None:
        _dist.destroy_process_group()


def run_reference(args, world):
    """The CPU oracle as the reference arm, on a bounded sample per step (rank 0 only)."""
    w = Workload(args.workload, args.seed, torch.device("cpu"))
    inp = oracle_inputs(w)
    budget_s = 120.0
    per_step = budget_s / (args.steps + args.warmup)
    # calibrate: seconds per token (append) and per row (decode)
    est0, _ = oracle_step_estimate(w, inp, kvq.KV_INT4_BDR, 128, False, tok_budget=256, row_budget=2)
    frac = min(1.0, per_step / max(est0, 1e-9))
    tok = max(16, int(w.T * frac))
    rows = max(1, int(w.B * w.Hq * frac))
    times, sample = [], ""
    for i in range(args.warmup + args.steps):
        est, sample = oracle_step_estimate(w, inp, kvq.KV_INT4_BDR, 128, False, tok_budget=tok, row_budget=rows)
        if i >= args.warmup:
            times.append(est)
    step_s = float(np.mean(times))
    value = w.T / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 write path, f64 attention", "data": "synthetic",
            "config": {"workload": args.workload, "variant": "INT4+BDR-128, keys only", "sequences": w.B,
                       "tokens_appended_per_step": w.T},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
