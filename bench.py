#!/usr/bin/env python
"""Benchmark of the SAW-INT4 KV-cache write/read hot path on B200.

One step = one pass of the whole path over one batch of a serving workload:
the fused BDR + INT4 appends of the step's new tokens into the paged cache
(kv_append_quant), then one paged GQA decode step (kv_decode_attn: split +
merge kernels).  Workloads (synthetic, seeded; K/V ~ N(0,1) with outlier
channels, q ~ N(0,1)):

  single256    1 sequence x 256 tokens, page size 16: append it, decode it.
  batch16      16 sequences, lengths ~U[512, 4096], page size 16: a step appends
               every token of every sequence, then decodes all 16.
  decode64x8k  64 x 8192 cached tokens (prefilled, untimed): a step appends 1
               token per sequence at position 8192 and decodes 8193 tokens each.
  mixed256     (default) 256 sequences, lengths log-uniform [1024, 32768], 64
               query heads, K and V rotated (prefilled, untimed): a step appends
               a 2048-token chunk to 8 sequences and 1 token to each of the other
               248, then decodes those 248.  The largest single-GPU workload with
               both halves of the path.
  long1m       1 sequence x 1,048,576 tokens, page size 64: a step appends the
               context in 128 chunks of 8192 tokens, then decodes it (split-K).
Steps rewrite the same slots each time, so every step does the same work.

The headline line times exactly --steps steps of the chosen workload, with CUDA
events on the launching stream at the start of each step, between its appends and
its decode, and at its end.  ``value`` is the appended tokens per second of the
append kernel's own time (the metric's first half); the decode's HBM GB/s is the
second half.  Unless --no-configs, the line also carries a sub-record per workload
(all five) with the append and decode rates of INT4+BDR-128, naive INT4 and BF16
pages built the same way.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
the host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
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
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Before every timed step: write a 256 MiB buffer (L2 is 126 MB), then read a second one.
    The write evicts the step's inputs; the read evicts the write's dirty lines again, so the
    timed kernels start from a cold L2 with no write-back of someone else's data pending."""

    def __init__(self, device):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)
        self.sink = torch.zeros(1, dtype=torch.int32, device=device)

    def zero_(self):
        self.w.zero_()
        torch.amax(self.r, dim=0, keepdim=True, out=self.sink)
VARIANTS = [("bf16", kvq.KV_BF16, 0, False), ("int4", kvq.KV_INT4, 0, False)] + [
    (f"bdr{b}_{'kv' if rv else 'k'}", kvq.KV_INT4_BDR, b, rv) for b in (16, 32, 64, 128) for rv in (False, True)]
# the variant each workload is quoted on (the blog's section 4: block 128, keys only; K and V for mixed serving)
HEADLINE = {"batch16": ("bdr128_k", kvq.KV_INT4_BDR, 128, False),
            "single256": ("bdr128_k", kvq.KV_INT4_BDR, 128, False),
            "decode64x8k": ("bdr128_k", kvq.KV_INT4_BDR, 128, False),
            "mixed256": ("bdr128_kv", kvq.KV_INT4_BDR, 128, True),
            "long1m": ("bdr128_k", kvq.KV_INT4_BDR, 128, False)}
_DECODE_SOURCES = ["kvq_decode_mma.cu", "kvq_mma.cuh", "kvq_decode.cuh", "kvq_common.cuh", "kvq_internal.h"]
KERNEL_SOURCES = {"append_kernel": ["kvq_append.cu", "kvq_common.cuh", "kvq_internal.h"],
                  "decode_tok_kernel": _DECODE_SOURCES, "decode_mma_kernel": _DECODE_SOURCES,
                  "decode_bf16_kernel": ["kvq_decode_bf16.cu", "kvq_mma.cuh", "kvq_decode.cuh", "kvq_common.cuh",
                                         "kvq_internal.h"],
                  "extend_tc_kernel": ["kvq_extend_tc.cu", "kvq_mma.cuh", "kvq_decode.cuh", "kvq_common.cuh",
                                       "kvq_internal.h"]}


def peak_bf16_tflops():
    """Dense bf16 tensor peak, burst figure (a kernel timed alone)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def peak_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


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


# --------------------------------------------------------------------------- workloads

class Workload:
    """Device-resident inputs of one serving step, plus the untimed prefill that precedes it."""

    def __init__(self, name: str, seed: int, device):
        wl = synth.WORKLOADS[name]
        self.wl, self.name, self.seed, self.device = wl, name, seed, device
        self.H, self.Hq, self.ps = wl.num_kv_heads, wl.num_q_heads, wl.page_size
        lengths = synth.seq_lengths(name, seed=seed)
        self.lengths = lengths
        B = len(lengths)
        if name in ("batch16", "single256"):
            self.prefill = []  # (sequence lengths, starts) appended untimed
            step = [(lengths, [0] * B)]
            dec_seqs, dec_lens = list(range(B)), lengths
            caps = lengths
        elif name == "decode64x8k":
            self.prefill = [(lengths, [0] * B)]
            step = [([1] * B, lengths)]
            dec_seqs, dec_lens = list(range(B)), [L + 1 for L in lengths]
            caps = [L + 1 for L in lengths]
        elif name == "mixed256":
            rng = np.random.default_rng(seed + 7)
            prefilling = set(rng.choice(B, 8, replace=False).tolist())
            self.prefilling = sorted(prefilling)
            self.prefill = [(lengths, [0] * B)]
            step = [([2048 if s in prefilling else 1 for s in range(B)], lengths)]
            dec_seqs = [s for s in range(B) if s not in prefilling]
            dec_lens = [lengths[s] + 1 for s in dec_seqs]
            caps = [L + 2048 for L in lengths]
        elif name == "long1m":
            L = lengths[0]
            self.prefill = []
            step = [([8192], [c]) for c in range(0, L, 8192)]
            dec_seqs, dec_lens = [0], [L]
            caps = lengths
        else:
            raise KeyError(name)
        pt, self.num_pages = synth.make_page_table(caps, self.ps, seed)
        self.page_table = pt.to(device)
        self.pt_stride, self.num_seqs = pt.shape[1], pt.shape[0]
        # the step's appends: one call per entry, each with its own tokens
        self.appends = []
        for i, (ls, st) in enumerate(step):
            ts, tp = synth.append_positions(ls, st)
            k, v = self._rows(len(ts), 1000 + i)
            self.appends.append((k, v, ts.to(device), tp.to(device)))
        self.tokens_per_step = sum(int(a[2].numel()) for a in self.appends)
        self.dec_lens = dec_lens
        self.dec_B = len(dec_seqs)
        self.dec_pt = pt[dec_seqs].contiguous().to(device)
        self.q = synth.make_q(self.dec_B, self.Hq, 128, seed).to(device)
        self.seq_lens = torch.tensor(dec_lens, dtype=torch.int32, device=device)
        self.max_len = max(dec_lens)

    def _rows(self, n, salt):
        # inputs below 1 GB are drawn on the CPU (identical on every machine), larger ones on the device
        gen = "cpu" if n * self.H * 128 * 2 * 2 < (1 << 30) or self.device.type == "cpu" else self.device
        k, v = synth.make_kv(n, self.wl, self.seed * 7 + salt, device=gen, chunk=8192)
        return k.to(self.device), v.to(self.device)

    def run_prefill(self, cache):
        """Append the untimed prefill; its K/V rows are drawn once and kept for later caches."""
        if not hasattr(self, "_prefill_rows"):
            self._prefill_rows = []
            for i, (ls, st) in enumerate(self.prefill):
                ts, tp = synth.append_positions(ls, st)
                for c0 in range(0, len(ts), 1 << 20):
                    c1 = min(len(ts), c0 + (1 << 20))
                    k, v = self._rows(c1 - c0, 10_000 + i * 4096 + c0 // (1 << 20))
                    self._prefill_rows.append((k, v, ts[c0:c1].to(self.device), tp[c0:c1].to(self.device)))
        for k, v, ts, tp in self._prefill_rows:
            cache.append(k, v, ts, tp, self.page_table)

    def append_bytes(self, mode):
        # read K and V rows (2 x 256 B per head); write bf16 rows (2 x 256 B) or INT4 codes + scale/zero (2 x 68 B)
        write = 2 * 256 if mode == kvq.KV_BF16 else 2 * 68
        return self.tokens_per_step * self.H * (2 * 256 + write)

    def decode_bytes(self, mode):
        per_tok = self.H * (2 * 256 if mode == kvq.KV_BF16 else 2 * 68)
        pages = sum(-(-L // self.ps) for L in self.dec_lens)
        return sum(self.dec_lens) * per_tok + self.dec_B * self.Hq * 128 * 2 * 2 + pages * 4


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


def make_cache(w: Workload, mode, b, rv, device, rope=None, code_bits=4):
    cache = kvq.PagedKVCache(w.num_pages, w.ps, w.H, w.Hq, mode, b, rv, device=device, fill=0, rope=rope,
                             code_bits=code_bits)
    w.run_prefill(cache)
    return cache


def run_variant(w: Workload, mode, b, rv, steps, warmup, device, clocks=False, rope=None, code_bits=4):
    """Exactly `steps` device-timed steps after `warmup` untimed ones.  Each step is bracketed by
    CUDA events on the launching stream, with one more between its appends and its decode, so the
    per-kernel and per-step means (ms) all come from the same timed steps.  L2 is flushed (a
    256 MiB write) before every step, outside its events.  rope: optional (cos, sin) table for
    the fused rotary embedding; code_bits: 4 or 2."""
    cache = make_cache(w, mode, b, rv, device, rope, code_bits)
    ws, _ = cache.workspace(w.dec_B, w.max_len, device)
    out = torch.empty(w.dec_B, w.Hq, 128, dtype=torch.bfloat16, device=device)
    flush = L2Flush(device)
    stream = torch.cuda.current_stream(device)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]

    def step(e=None):
        if e: e[0].record(stream)
        for k, v, ts, tp in w.appends:
            kvq.kv_append_quant(cache.handle, k, v, k.shape[0], ts, tp, w.page_table, w.pt_stride, w.num_seqs,
                                stream)
        if e: e[1].record(stream)
        kvq.kv_decode_attn(cache.handle, w.q, w.seq_lens, w.dec_pt, w.pt_stride, w.dec_B, w.max_len, out, 0, ws,
                           ws.numel(), stream)
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
        flush.zero_()  # L2 flush: write one 256 MiB buffer, read another (L2 is 126 MB)
        step(evs[i])
    torch.cuda.synchronize(device)
    wall = time.perf_counter() - t0
    _barrier()
    if sampler:
        sampler.__exit__()
    stp = np.array([e[0].elapsed_time(e[2]) for e in evs])
    app = np.array([e[0].elapsed_time(e[1]) for e in evs])
    dec = np.array([e[1].elapsed_time(e[2]) for e in evs])
    status = cache.get_error()
    cache.close()
    return {"append_ms": float(app.mean()), "decode_ms": float(dec.mean()), "step_ms": float(stp.mean()),
            "append_ms_median": float(np.median(app)), "decode_ms_median": float(np.median(dec)),
            "wall_s": wall, "status": status, "clocks": sampler.summary() if sampler else None,
            "launches_per_step": len(w.appends) + 2}


def extend_setup(w: Workload):
    """The step's prefill attention: (sequences, their cached lengths after the step's append,
    new queries per sequence).  mixed256: the 8 sequences that append a 2048-token chunk attend
    over it; batch16 / single256: every sequence, appended from position 0, is one prefill."""
    if w.name == "mixed256":
        return w.prefilling, [w.lengths[s] + 2048 for s in w.prefilling], [2048] * len(w.prefilling)
    if w.name in ("batch16", "single256"):
        return list(range(len(w.lengths))), list(w.lengths), list(w.lengths)
    return None


def run_extend(w: Workload, mode, b, rv, reps, device):
    """kv_extend_attn over the step's prefill queries (after the step's append), CUDA events around
    each launch on the launching stream, L2 flushed between launches.  Work: 4 D flops per
    (query head, attended token) -- the q.K and P.V of bf16 attention, to compare with the dense
    bf16 tensor peak; bytes: each sequence's cached codes + scale/zero read once, q and out."""
    seqs, lens, qlens = extend_setup(w)
    cache = make_cache(w, mode, b, rv, device)
    for k, v, ts, tp in w.appends:
        cache.append(k, v, ts, tp, w.page_table)
    nq = sum(qlens)
    q = synth.make_q(nq, w.Hq, 128, w.seed + 99, device=device)
    qi = torch.tensor(np.concatenate([[0], np.cumsum(qlens)]), dtype=torch.int32, device=device)
    sl = torch.tensor(lens, dtype=torch.int32, device=device)
    pt = w.page_table[torch.tensor(seqs, device=device)].contiguous()
    out = torch.empty(nq, w.Hq, 128, dtype=torch.bfloat16, device=device)
    flush = L2Flush(device)
    stream = torch.cuda.current_stream(device)

    def launch():
        kvq.kv_extend_attn(cache.handle, q, qi, sl, pt, w.pt_stride, len(seqs), max(qlens), max(lens), out, 0, stream)

    for _ in range(3):
        flush.zero_()
        launch()
    torch.cuda.synchronize(device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        launch()
        e1.record(stream)
    torch.cuda.synchronize(device)
    ms = np.array([e0.elapsed_time(e1) for e0, e1 in evs])
    status = cache.get_error()
    cache.close()
    attended = sum(n * (L - n) + n * (n + 1) // 2 for L, n in zip(lens, qlens))  # sum over queries of position + 1
    flops = 4 * 128 * w.Hq * attended
    per_tok = w.H * (2 * 68 if mode != kvq.KV_BF16 else 2 * 256)
    nbytes = sum(lens) * per_tok + nq * w.Hq * 128 * 2 * 2
    peak, kind = peak_bf16_tflops()
    ekern = "extend_tc_kernel"
    t = float(ms.mean())
    return {"us": t * 1e3, "us_median": float(np.median(ms)) * 1e3, "launches": reps, "sequences": len(seqs),
            "queries": nq, "query_heads": w.Hq, "attended_tokens_per_query_head": attended,
            "flops": flops, "tflops": flops / (t / 1e3) / 1e12,
            "roofline": {"bound": "tensor", "kernel": ekern, "achieved": flops / (t / 1e3) / 1e12,
                         "peak": peak, "unit": "TFLOP/s", "frac": flops / (t / 1e3) / 1e12 / peak,
                         "peak_source": f"{kind} dense bf16 burst (MEASURED_PEAKS.json bf16_tflops); " + (
                             "the kernel runs fp16 tcgen05 MMAs (kind::f16, the same dense rate as bf16)"),
                         "traffic": profiled_traffic(ekern, w.name)},
            "algorithmic_bytes": nbytes, "gbs": nbytes / (t / 1e3) / 1e9,
            "device_status": kvq.status_string(status)}


def run_profile_case(case: str):
    """Small seeded cases for ncu captures with many passes (more than L2 on the device, well under
    1 GB): the cache is filled through the append, then the captured kernel runs 4 times."""
    device = torch.device("cuda")
    B, L, H, Hq, rv = (32, 4096, 8, 64, True) if case == "decode_g8" else (4, 4096, 8, 32, False)
    ps = 16
    num_pages = B * L // ps
    g = torch.Generator(device=device).manual_seed(0)
    pt = torch.randperm(num_pages, device=device, generator=g).to(torch.int32).view(B, L // ps).contiguous()
    cache = kvq.PagedKVCache(num_pages, ps, H, Hq, kvq.KV_INT4_BDR, 128, rv, device=device, fill=0)
    k = torch.randn(B * L, H, 128, device=device, generator=g).to(torch.bfloat16)
    v = torch.randn(B * L, H, 128, device=device, generator=g).to(torch.bfloat16)
    ts = torch.arange(B, device=device, dtype=torch.int32).repeat_interleave(L)
    tp = torch.arange(L, device=device, dtype=torch.int32).repeat(B)
    cache.append(k, v, ts, tp, pt)
    sl = torch.full((B,), L, device=device, dtype=torch.int32)
    if case == "decode_g8":
        q = torch.randn(B, Hq, 128, device=device, generator=g).to(torch.bfloat16)
        ws = cache.workspace(B, L, device)
        for _ in range(4):
            out = cache.decode(q, sl, pt, L, workspace=ws)
    else:
        q = torch.randn(B * L, Hq, 128, device=device, generator=g).to(torch.bfloat16)
        qi = torch.arange(0, B * L + 1, L, device=device, dtype=torch.int32)
        for _ in range(4):
            out = cache.extend(q, qi, sl, pt, L, L)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": case, "sequences": B, "tokens_per_sequence": L, "num_kv_heads": H,
                      "num_q_heads": Hq, "device_status": kvq.status_string(cache.get_error()),
                      "mean_abs_out": float(out.float().abs().mean())}))


def exact_attention(k, v, q, lengths, H, Hq):
    """float64 attention of q over the unquantised bf16 K/V rows (sequence-major, positions 0..L-1):
    the values the quantised caches approximate (no cache, no quantisation, no rotation)."""
    kf = k.float().cpu().numpy().astype(np.float64)
    vf = v.float().cpu().numpy().astype(np.float64)
    qf = q.float().cpu().numpy().astype(np.float64)
    G = Hq // H
    out = np.zeros((len(lengths), Hq, 128))
    off = 0
    for s, L in enumerate(lengths):
        Ks, Vs = kf[off:off + L], vf[off:off + L]
        off += L
        for j in range(Hq):
            sc = Ks[:, j // G] @ qf[s, j] / np.sqrt(128.0)
            p = np.exp(sc - sc.max())
            out[s, j] = (p @ Vs[:, j // G]) / p.sum()
    return out


def accuracy_study(w: Workload, device):
    """Attention-output error of every cache variant (append + decode through the library, fp32
    output) against exact float64 attention on the unquantised rows, per (sequence, query head)
    row: max |o - r| / max |r|.  Whole sequences appended from position 0 (batch16, single256)."""
    k, v, ts, tp = w.appends[0]
    ref = exact_attention(k, v, w.q, w.dec_lens, w.H, w.Hq)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-30)
    res = {}
    two_bit = [("int2", kvq.KV_INT4, 0, False, 2), ("bdr128_k_int2", kvq.KV_INT4_BDR, 128, False, 2),
               ("bdr128_kv_int2", kvq.KV_INT4_BDR, 128, True, 2)]
    for name, mode, b, rv, bits in [v + (4,) for v in VARIANTS] + two_bit:
        cache = kvq.PagedKVCache(w.num_pages, w.ps, w.H, w.Hq, mode, b, rv, device=device, fill=0, code_bits=bits)
        cache.append(k, v, ts, tp, w.page_table)
        out = cache.decode(w.q, w.seq_lens, w.dec_pt, w.max_len, out_fp32=True)
        status = cache.get_error()
        cache.close()
        if status != kvq.KV_OK:
            raise RuntimeError(f"device error in the accuracy study: {kvq.status_string(status)}")
        err = np.abs(out.cpu().numpy().astype(np.float64) - ref).max(axis=-1) / den
        res[name] = {"max_rel": float(err.max()), "mean_rel": float(err.mean())}
    return res


def run_e2e(w: Workload, mode, b, rv, steps, warmup, device):
    """Same step through the C ABI with pinned HOST inputs: H2D copies of the step's inputs and a
    D2H read of the attention output are inside the timed region (CUDA events, launching stream)."""
    cache = make_cache(w, mode, b, rv, device)
    ws, _ = cache.workspace(w.dec_B, w.max_len, device)
    host = [[t.cpu().pin_memory() for t in a] for a in w.appends]
    hdec = [t.cpu().pin_memory() for t in (w.q, w.seq_lens, w.dec_pt, w.page_table)]
    dev = [[torch.empty_like(t, device=device) for t in a] for a in host]
    ddec = [torch.empty_like(t, device=device) for t in hdec]
    out = torch.empty(w.dec_B, w.Hq, 128, dtype=torch.bfloat16, device=device)
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    stream = torch.cuda.current_stream(device)
    h2d = sum(t.numel() * t.element_size() for a in host for t in a) + sum(t.numel() * t.element_size() for t in hdec)
    d2h = out_h.numel() * out_h.element_size()

    def step():
        for hd, dd in zip(hdec, ddec):
            dd.copy_(hd, non_blocking=True)
        q, sl, dpt, pt = ddec
        for ha, da in zip(host, dev):
            for h_, d_ in zip(ha, da):
                d_.copy_(h_, non_blocking=True)
            k, v, ts, tp = da
            kvq.kv_append_quant(cache.handle, k, v, k.shape[0], ts, tp, pt, w.pt_stride, w.num_seqs, stream)
        kvq.kv_decode_attn(cache.handle, q, sl, dpt, w.pt_stride, w.dec_B, w.max_len, out, 0, ws, ws.numel(), stream)
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

def oracle_unit_costs(w: Workload, mode, b, rv, tok_budget: int, row_budget: int, seed=0, dec_seqs: int = 1,
                      reps: int = 1, threads: int = 1):
    """Seconds per appended token and per (cached token x query head) of the CPU oracle, measured
    on a bounded sample shaped like the workload: tok_budget appended tokens, and row_budget
    query-head rows of each of dec_seqs sequences of the workload's mean decoded length; the
    whole sample is run reps times (seeds seed .. seed + reps - 1) and the times summed.  With
    threads > 1 the appended tokens and the decoded rows are split into that many contiguous
    parts run concurrently (the C oracle keeps no global state and ctypes releases the GIL), and
    the wall time is what counts."""
    import concurrent.futures

    import oracle

    H, ps = w.H, w.ps
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    n = max(1, tok_budget)
    Ls = int(min(max(np.mean(w.dec_lens), 16), 32768))
    r = max(1, min(row_budget, w.Hq))
    nd = max(1, dec_seqs)
    t_app = t_dec = 0.0
    pool = concurrent.futures.ThreadPoolExecutor(max_workers=threads) if threads > 1 else None
    for rep in range(reps):
        sd = seed + rep
        k, v = synth.make_kv(n, w.wl, sd)
        pt, P = synth.make_page_table([max(n, Ls)] + [Ls] * (nd - 1), ps, sd)
        if mode == kvq.KV_BF16:
            kp = np.zeros((P, H, ps, 128), np.uint16)
            ks = np.zeros(1, np.uint16)
        else:
            kp = np.zeros((P, H, ps, 64), np.uint8)
            ks = np.zeros((P, H, ps, 2), np.uint16)
        vp, vs = kp.copy(), ks.copy()
        ts, tp = synth.append_positions([n])
        kb, vb, tsn, tpn, ptn = bits(k), bits(v), ts.numpy(), tp.numpy(), pt.numpy()
        cuts = np.linspace(0, n, max(1, threads) + 1).astype(int)

        def app(part):
            a, z = cuts[part], cuts[part + 1]
            oracle.append(mode, b, rv, kp, vp, ks, vs, kb[a:z], vb[a:z], tsn[a:z], tpn[a:z], ptn)

        t0 = time.perf_counter()
        if pool:
            list(pool.map(app, range(threads)))
        else:
            app(0)
        t_app += time.perf_counter() - t0
        qb = bits(synth.make_q(nd, w.Hq, 128, sd))
        rows = [(s, j) for s in range(nd) for j in range(r)]
        rcuts = np.linspace(0, len(rows), max(1, threads) + 1).astype(int)

        def dec(part):
            sub = rows[rcuts[part]:rcuts[part + 1]]
            if sub:
                oracle.decode(mode, b, rv, kp, vp, ks, vs, qb, np.array([Ls] * nd), ptn, H, rows=sub)

        t0 = time.perf_counter()
        if pool:
            list(pool.map(dec, range(threads)))
        else:
            dec(0)
        t_dec += time.perf_counter() - t0
    if pool:
        pool.shutdown()
    c_app = t_app / (n * reps)
    c_dec = t_dec / (r * nd * Ls * reps)
    sample = (f"{reps} x (oracle append of {n} tokens and decode of {r} query-head rows of {nd} sequence(s) "
              f"over {Ls} cached tokens), {threads} thread(s), {t_app + t_dec:.1f} s wall; per-unit costs scaled "
              f"to one step ({w.tokens_per_step} tokens appended, {sum(w.dec_lens) * w.Hq} (token x query head) "
              f"decoded)")
    return c_app, c_dec, sample


def host_cpu():
    """(usable cores, CPU model) of this host."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return cores, model


def oracle_step_seconds(w: Workload, c_app, c_dec):
    return c_app * w.tokens_per_step + c_dec * sum(w.dec_lens) * w.Hq


# --------------------------------------------------------------------------- dist

_dist = None


def _init_dist():
    global _dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        _dist = dist
    return ws


def _barrier():
    if _dist is not None:
        _dist.barrier()


def reduce_over_ranks(x: float, op: str, device) -> float:
    """MAX or SUM of one number over all ranks (the only collectives: timing bookkeeping)."""
    if _dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    _dist.all_reduce(t, op=_dist.ReduceOp.MAX if op == "max" else _dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------- main

# the comparators of every sub-record: naive INT4 and BF16 pages, built the same way
COMPARATORS = [("int4", kvq.KV_INT4, 0, False), ("bf16", kvq.KV_BF16, 0, False)]
CONFIG_STEPS = 50  # timed steps of each sub-record variant (after 3 warm-ups)


def _dec_kernel(w: Workload, mode):
    if mode == kvq.KV_BF16:
        return "decode_bf16_kernel + merge_kernel"
    # the INT4 decode runs the tokens-on-M tile for up to 4 query heads per KV head, else heads-on-M
    return ("decode_tok_kernel" if w.Hq // w.H <= 4 else "decode_mma_kernel") + " + merge_kernel"


def roofline_record(kernel, achieved, peak, peak_kind, traffic=None, **extra):
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
            "traffic": traffic, **extra}


def variant_record(w: Workload, mode, r, workload_name, peak, peak_kind, with_traffic=False):
    """Append and decode rates of one variant's timed steps, each against the HBM roofline."""
    app_b, dec_b = w.append_bytes(mode), w.decode_bytes(mode)
    app_gbs = app_b / (r["append_ms"] / 1e3) / 1e9
    dec_gbs = dec_b / (r["decode_ms"] / 1e3) / 1e9
    napp = len(w.appends)
    app_traffic = profiled_traffic("append_kernel", workload_name) if with_traffic else None
    dkern = _dec_kernel(w, mode)
    dec_traffic = (profiled_traffic(dkern.split()[0], workload_name)
                   if with_traffic and mode != kvq.KV_BF16 else None)
    return {
        "append": {"us": r["append_ms"] * 1e3, "launches_per_step": napp,
                   "tokens_per_s": w.tokens_per_step / (r["append_ms"] / 1e3),
                   "algorithmic_bytes": app_b, "algorithmic_bytes_per_launch": app_b / napp, "gbs": app_gbs,
                   "frac_of_8tbs": app_gbs / NOMINAL_HBM_GBS,
                   "roofline": roofline_record("append_kernel", app_gbs, peak, peak_kind, app_traffic,
                                               traffic_unit="DRAM bytes per launch (ncu)")},
        "decode": {"us": r["decode_ms"] * 1e3, "launches_per_step": 2, "algorithmic_bytes": dec_b, "gbs": dec_gbs,
                   "frac_of_8tbs": dec_gbs / NOMINAL_HBM_GBS,
                   "roofline": roofline_record(dkern, dec_gbs, peak, peak_kind, dec_traffic,
                                               traffic_unit="DRAM bytes of the split kernel per launch (ncu)")},
        "step_us": r["step_ms"] * 1e3, "steps": r.get("steps"),
    }


def measure_config(name, seed, device, peak, peak_kind, head=None, extend=True, accuracy=True):
    """Sub-record of one workload: the headline variant, naive INT4 and BF16 pages (batch16: every
    block size, K and K+V, fused RoPE and 2-bit codes too), the ratios the targets are stated in,
    and the extend attention where the workload has prefill queries.  head: the headline variant's
    measurement when it was already taken (the headline workload)."""
    w = Workload(name, seed, device)
    hname, hmode, hb, hrv = HEADLINE[name]
    variants = [(hname, hmode, hb, hrv)] + COMPARATORS
    if name == "batch16":
        variants = [(hname, hmode, hb, hrv)] + [v for v in VARIANTS if v[0] != hname]
    rec = {"description": w.wl.description, "headline_variant": hname, "tokens_appended_per_step": w.tokens_per_step,
           "append_launches_per_step": len(w.appends), "sequences_decoded_per_step": w.dec_B,
           "cached_tokens_decoded_per_step": sum(w.dec_lens), "num_q_heads": w.Hq, "page_size": w.ps,
           "variants": {}}
    for vname, mode, b, rv in variants:
        if head is not None and vname == hname:
            r = head
        else:
            r = run_variant(w, mode, b, rv, CONFIG_STEPS, 3, device)
            r["steps"] = CONFIG_STEPS
        rec["variants"][vname] = variant_record(w, mode, r, name, peak, peak_kind, with_traffic=(vname == hname))
    V = rec["variants"]
    rec["ratios"] = {
        f"{hname}_over_int4_append_tokens_per_s": V[hname]["append"]["tokens_per_s"] / V["int4"]["append"]["tokens_per_s"],
        f"{hname}_over_int4_decode_time": V["int4"]["decode"]["us"] / V[hname]["decode"]["us"],
        "bf16_over_int4_decode_time": V["bf16"]["decode"]["us"] / V["int4"]["decode"]["us"],
        "bf16_over_int4_step_time": V["bf16"]["step_us"] / V["int4"]["step_us"],
        f"bf16_over_{hname}_step_time": V["bf16"]["step_us"] / V[hname]["step_us"],
        "note": "time ratios > 1 mean the second variant is faster; targets: INT4+BDR-128 append and decode "
                ">= 0.70 of the HBM roofline each, BDR-128 append >= 0.95 of naive INT4"}
    if name == "batch16":
        n = CONFIG_STEPS
        tab = synth.rope_table(max(w.dec_lens) + 1).to(device)
        r = run_variant(w, kvq.KV_INT4_BDR, 128, False, n, 3, device, rope=tab)
        rec["bdr128_k_rope"] = {"append_us": r["append_ms"] * 1e3, "decode_us": r["decode_ms"] * 1e3,
                                "append_tok_per_s": w.tokens_per_step / (r["append_ms"] / 1e3),
                                "note": "fused rotary embedding; plus the table reads (512 B per appended token)"}
        r = run_variant(w, kvq.KV_INT4_BDR, 128, False, n, 3, device, code_bits=2)
        rec["bdr128_k_int2"] = {"append_us": r["append_ms"] * 1e3, "decode_us": r["decode_ms"] * 1e3,
                                "append_tok_per_s": w.tokens_per_step / (r["append_ms"] / 1e3),
                                "note": "2-bit codes; timed like the others, bytes not comparable"}
        if accuracy:
            rec["accuracy"] = {"vs": "exact float64 attention on the unquantised bf16 K/V",
                               "metric": "per (sequence, query head) row max|o-r|/max|r|", **accuracy_study(w, device)}
    if extend and extend_setup(w) is not None:
        rec["extend"] = {"what": "kv_extend_attn: causal attention of the step's prefill queries over the paged "
                                 "cache (one launch), outside the timed step", **run_extend(w, hmode, hb, hrv, 10, device)}
    del w
    torch.cuda.empty_cache()
    return rec


def config_dict(w: Workload, variant: str, world: int, seed: int):
    """The workload the line is quoted on (identical in the kernel and the reference arm)."""
    return {"workload": w.name, "description": w.wl.description, "variant": variant,
            "sequences": len(w.lengths), "tokens_appended_per_step": w.tokens_per_step,
            "append_launches_per_step": len(w.appends), "sequences_decoded_per_step": w.dec_B,
            "cached_tokens_decoded_per_step": sum(w.dec_lens), "num_kv_heads": w.H, "num_q_heads": w.Hq,
            "head_dim": 128, "page_size": w.ps, "l2": "before every timed step a 256 MiB buffer is written and a second one read (L2 is 126 MB): cold inputs, no dirty lines pending",
            "parallelism": f"{world} independent replica(s), one per GPU, no collective on the data path",
            "seed": seed}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default="mixed256", choices=list(synth.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload sub-records")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-accuracy", action="store_true")
    ap.add_argument("--no-extend", action="store_true")
    ap.add_argument("--profile-case", choices=["decode_g8", "extend_g4"],
                    help="a small case for multi-metric ncu captures: decode_g8 = 32 sequences x 4096 tokens, "
                         "64 query / 8 KV heads, BDR-128 keys and values, 4 decode launches; extend_g4 = 4 "
                         "sequences x 4096 tokens, 32 query / 8 KV heads, BDR-128 keys, full causal prefill, "
                         "4 extend launches")
    ap.add_argument("--extend-only", action="store_true",
                    help="only the extend attention of --workload (3 warm-up + 10 timed launches), one JSON line; "
                         "the entry point of its ncu captures")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    if args.profile_case:
        return run_profile_case(args.profile_case)

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
    w = Workload(args.workload, args.seed + rank, device)  # each rank: its own independent batch
    hname, hmode, hb, hrv = HEADLINE[args.workload]
    peak, peak_kind = peak_hbm()
    if args.extend_only:
        if extend_setup(w) is None:
            raise SystemExit(f"{args.workload} has no prefill queries")
        r = run_extend(w, hmode, hb, hrv, 10, device)
        if rank == 0:
            print(json.dumps({"workload": args.workload, "variant": hname, "extend": r}))
        if _dist is not None:
            _dist.destroy_process_group()
        return

    res = run_variant(w, hmode, hb, hrv, args.steps, args.warmup, device, clocks=True)
    res["steps"] = args.steps
    step_ms = reduce_over_ranks(res["step_ms"], "max", device)
    app_ms = reduce_over_ranks(res["append_ms"], "max", device)
    dec_ms = reduce_over_ranks(res["decode_ms"], "max", device)
    tokens = reduce_over_ranks(w.tokens_per_step, "sum", device)
    value = tokens / (app_ms / 1e3)  # appended tokens per second of the append kernel's own time

    e2e_ms, h2d, d2h = run_e2e(w, hmode, hb, hrv, max(20, min(200, args.steps)), args.warmup, device)
    e2e_ms = reduce_over_ranks(e2e_ms, "max", device)

    head = variant_record(w, hmode, res, args.workload, peak, peak_kind, with_traffic=True)
    dominant = "append" if res["append_ms"] >= res["decode_ms"] else "decode"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32",
        "dtype_detail": "bf16 rows in; fp32 rotation and quantiser; INT4 codes + fp16 scale/zero stored; attention on "
                        "int8 / fp16 tensor-core tiles with int32 / fp32 accumulation", "data": "synthetic",
        "value_detail": "appended tokens per second of the append kernel's own time (CUDA events around the step's "
                        "appends inside each timed step; all ranks' tokens / the slowest rank's mean append time); "
                        "ms_per_step is the whole step (appends + decode)",
        "config": config_dict(w, hname, world, args.seed),
        "components": {"append": head["append"], "decode": {**head["decode"], "note": "split + merge kernels"}},
        "decode_gbs": head["decode"]["gbs"], "decode_frac_of_peak": head["decode"]["roofline"]["frac"],
        "roofline": {**head[dominant]["roofline"], "component": dominant,
                     "note": "the dominant kernel of the step; both components carry their own roofline"},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "what": "the whole step through the C ABI from pinned host buffers: the step's inputs copied to the "
                        "device and the attention output read back inside the timed region"},
        "gpu_launches": res["launches_per_step"] * args.steps,
        "clocks": res["clocks"],
        "device_status": kvq.status_string(res["status"]),
    }
    if not args.no_configs:
        # every workload, each with the headline variant and the comparators built the same way
        del w
        torch.cuda.empty_cache()
        configs = {}
        for name in synth.WORKLOADS:
            configs[name] = measure_config(name, args.seed + rank, device, peak, peak_kind,
                                           head=res if name == args.workload else None,
                                           extend=not args.no_extend, accuracy=not args.no_accuracy)
        line["configs"] = configs
        w = Workload(args.workload, args.seed + rank, device)
    if rank == 0 and world == 1 and not args.no_cpu:
        kw = cpu_sample(w)
        c_app, c_dec, sample = oracle_unit_costs(w, hmode, hb, hrv, **kw)
        cores, model = host_cpu()
        line["cpu_baseline"] = {"value": w.tokens_per_step / oracle_step_seconds(w, c_app, c_dec),
                                "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample,
                                "cpu_model": model, "host_cores": cores}
        if cores > 1:
            p_app, p_dec, psample = oracle_unit_costs(w, hmode, hb, hrv, threads=cores, **kw)
            line["cpu_baseline"]["all_cores"] = {"value": w.tokens_per_step / oracle_step_seconds(w, p_app, p_dec),
                                                 "unit": "tokens/s", "cores": cores, "sample": psample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if _dist is not None:
        _dist.destroy_process_group()


def cpu_sample(w: Workload):
    """The bounded oracle sample of one step of w: up to 40960 appended tokens, and every query head of
    up to 16 sequences of the workload's mean decoded length (fewer for long sequences, about 1 M
    (token x query head) units), three repetitions."""
    Ls = int(min(max(np.mean(w.dec_lens), 16), 32768))
    nd = max(1, min(w.dec_B, 16, (1 << 20) // (w.Hq * Ls)))
    return dict(tok_budget=min(w.tokens_per_step, 40960), row_budget=w.Hq, dec_seqs=nd, reps=3)


def run_reference(args, world):
    """The CPU oracle as the reference arm (rank 0 only): each step runs the same bounded sample of
    the workload's step as the kernel arm's all-core cpu_baseline (its tokens and rows split over
    every host core), and scales its unit costs to the full step."""
    w = Workload(args.workload, args.seed, torch.device("cpu"))
    hname, hmode, hb, hrv = HEADLINE[args.workload]
    cores, model = host_cpu()
    kw = cpu_sample(w)
    times, sample = [], ""
    for i in range(args.warmup + args.steps):
        c_app, c_dec, sample = oracle_unit_costs(w, hmode, hb, hrv, seed=i, threads=cores, **kw)
        if i >= args.warmup:
            times.append(oracle_step_seconds(w, c_app, c_dec))
    step_s = float(np.mean(times))
    value = w.tokens_per_step / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "dtype_detail": "oracle: fp32 write path, float64 attention", "data": "synthetic",
            "config": config_dict(w, hname, world, args.seed),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
                             "cpu_model": model},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
