"""Host-side logic of bench.py (CPU only): the work and byte counts it reports for the extend
leg, and the all-cores oracle baseline, whose threads must compute exactly what one call does."""
import concurrent.futures

import numpy as np
import torch

import bench
import oracle
from bit_paged_kv_append_b200 import kvq, synth


def test_extend_work_counts_match_the_oracle_positions():
    """bench counts sum over queries of (position + 1) attended tokens per query head; the oracle's
    extend_lengths gives every query's position + 1 directly."""
    for name in ("batch16", "mixed256"):
        w = bench.Workload(name, 0, torch.device("cpu"))
        seqs, lens, qlens = bench.extend_setup(w)
        assert len(seqs) == len(lens) == len(qlens)
        qi = np.concatenate([[0], np.cumsum(qlens)])
        _, per_query = oracle.extend_lengths(qi, lens)
        counted = sum(n * (L - n) + n * (n + 1) // 2 for L, n in zip(lens, qlens))
        assert counted == int(per_query.sum())
        assert per_query.min() >= 1  # every query has at least itself to attend to
        if name == "mixed256":
            assert qlens == [2048] * 8 and all(L >= 2048 + 1024 for L in lens)
        else:
            assert qlens == lens  # a full causal prefill of every sequence


def test_threaded_oracle_append_equals_one_call():
    """The all-cores baseline splits the appended tokens over threads: the pools must come out
    bit for bit as one call writes them (the oracle keeps no global state)."""
    wl = synth.WORKLOADS["batch16"]
    n, H, ps = 3000, wl.num_kv_heads, wl.page_size
    k, v = synth.make_kv(n, wl, 5)
    pt, P = synth.make_page_table([n], ps, 5)
    ts, tp = synth.append_positions([n])
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    kb, vb = bits(k), bits(v)

    def pools():
        kp = np.zeros((P, H, ps, 64), np.uint8)
        ks = np.zeros((P, H, ps, 2), np.uint16)
        return kp, kp.copy(), ks, ks.copy()

    one = pools()
    oracle.append(oracle.MODE_INT4_BDR, 128, True, *one, kb, vb, ts.numpy(), tp.numpy(), pt.numpy())
    split = pools()
    cuts = np.linspace(0, n, 9).astype(int)

    def part(i):
        a, z = cuts[i], cuts[i + 1]
        oracle.append(oracle.MODE_INT4_BDR, 128, True, *split, kb[a:z], vb[a:z], ts.numpy()[a:z], tp.numpy()[a:z],
                      pt.numpy())

    with concurrent.futures.ThreadPoolExecutor(max_workers=8) as ex:
        list(ex.map(part, range(8)))
    for x, y in zip(one, split):
        assert np.array_equal(x, y)


def test_oracle_unit_costs_threads_and_host_cpu():
    w = bench.Workload("single256", 0, torch.device("cpu"))
    for threads in (1, 4):
        c_app, c_dec, sample = bench.oracle_unit_costs(w, kvq.KV_INT4_BDR, 128, False, tok_budget=256, row_budget=8,
                                                       threads=threads)
        assert c_app > 0 and c_dec > 0 and f"{threads} thread(s)" in sample
    cores, model = bench.host_cpu()
    assert cores >= 1 and isinstance(model, str) and model


def test_variant_record_rates_and_fractions():
    """A sub-record's rates are its algorithmic bytes over the measured times, its fractions
    those rates over the peak, per component."""
    w = bench.Workload("batch16", 0, torch.device("cpu"))
    r = {"append_ms": 0.05, "decode_ms": 0.025, "step_ms": 0.08}
    rec = bench.variant_record(w, kvq.KV_INT4_BDR, r, "batch16", 6544.0, "measured")
    app_b = w.tokens_per_step * 8 * (2 * 256 + 2 * 68)
    assert rec["append"]["algorithmic_bytes"] == app_b
    assert abs(rec["append"]["gbs"] - app_b / 0.05e-3 / 1e9) < 1e-6
    assert abs(rec["append"]["roofline"]["frac"] - rec["append"]["gbs"] / 6544.0) < 1e-12
    assert abs(rec["append"]["tokens_per_s"] - w.tokens_per_step / 0.05e-3) < 1e-3
    dec_b = w.decode_bytes(kvq.KV_INT4_BDR)
    assert sum(w.dec_lens) * 8 * 136 < dec_b < sum(w.dec_lens) * 8 * 136 * 1.01
    assert abs(rec["decode"]["roofline"]["frac"] - dec_b / 0.025e-3 / 1e9 / 6544.0) < 1e-12
    assert rec["decode"]["roofline"]["kernel"].startswith("decode_tok_kernel")
    w8 = bench.Workload("mixed256", 0, torch.device("cpu"))
    assert bench._dec_kernel(w8, kvq.KV_INT4_BDR).startswith("decode_mma_kernel")


def test_reference_arm_prints_the_kernel_arms_config(capsys):
    """The reference arm quotes the same workload, variant, metric and unit as the kernel arm, and
    its sample has the shape of the kernel arm's all-core baseline."""
    import argparse
    import json

    args = argparse.Namespace(workload="single256", seed=0, steps=1, warmup=1)
    bench.run_reference(args, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    w = bench.Workload("single256", 0, torch.device("cpu"))
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["config"] == bench.config_dict(w, bench.HEADLINE["single256"][0], 1, 0)
    kw = bench.cpu_sample(w)
    assert kw["row_budget"] == w.Hq and kw["reps"] >= 3
    assert f"decode of {w.Hq} query-head rows" in line["cpu_baseline"]["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_kernel_source_lists_and_profiled_traffic_are_consistent():
    """Every source a benched kernel's counters are keyed on exists; every profiled-traffic entry
    names a benched kernel, and its hash is what src_hash gives now (or the bench reports null)."""
    import json
    import os

    csrc = os.path.join(bench.ROOT, "bit_paged_kv_append_b200", "csrc")
    for kernel, files in bench.KERNEL_SOURCES.items():
        for name in files:
            assert os.path.isfile(os.path.join(csrc, name)), (kernel, name)
        assert len(bench.src_hash(kernel)) == 16
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        traffic = json.load(f)
    for kernel, recs in traffic.items():
        assert kernel in bench.KERNEL_SOURCES, kernel
        for workload, rec in recs.items():
            assert workload in synth.WORKLOADS, workload
            assert rec["dram_bytes_per_launch"] == rec["dram_read"] + rec["dram_write"]
            expect = float(rec["dram_bytes_per_launch"]) if rec["src_sha"] == bench.src_hash(kernel) else None
            assert bench.profiled_traffic(kernel, workload) == expect
