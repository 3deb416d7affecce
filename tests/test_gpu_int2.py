"""GPU parity of the 2-bit variant (kv_desc.code_bits = 2; the pages leave 2-bit open) against
the oracle: appended pools bit for bit, decode attention within ATTN_RTOL, for the plain and
rotated modes, both decode tiles (G = 4, 8), the gather path (page size not a multiple of 16)
and RoPE."""
import dataclasses

import numpy as np
import pytest
import torch

from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import (ATTN_RTOL, assert_pools_equal, attn_rel_err, gpu_append, gpu_decode, make_case,
                         oracle_append, oracle_decode)

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["batch16"]
VARIANTS = [("int2", kvq.KV_INT4, 0, False), ("bdr128k", kvq.KV_INT4_BDR, 128, False),
            ("bdr64kv", kvq.KV_INT4_BDR, 64, True), ("bdr16kv", kvq.KV_INT4_BDR, 16, True)]


def _run(c, lengths, hq):
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    q = synth.make_q(len(lengths), hq, 128, seed=21)
    out, st = gpu_decode(c, q, lengths)
    assert st == kvq.KV_OK
    ref, skipped = oracle_decode(c, q, lengths)
    assert skipped == 0
    err = attn_rel_err(out.cpu().numpy(), ref)
    assert err <= ATTN_RTOL, err
    out16, _ = gpu_decode(c, q, lengths, out_fp32=False)
    assert torch.equal(out16, out.to(torch.bfloat16))


@pytest.mark.parametrize("name,mode,b,rv", VARIANTS, ids=[v[0] for v in VARIANTS])
@pytest.mark.parametrize("hq", [32, 64])
def test_int2_append_and_decode(name, mode, b, rv, hq):
    lengths = [900, 2049, 37]
    c = make_case(mode, b, rv, lengths, dataclasses.replace(WL, num_q_heads=hq), seed=20, code_bits=2)
    _run(c, lengths, hq)


@pytest.mark.parametrize("ps", [7, 24])
def test_int2_gather_path(ps):
    lengths = [301, 95]
    wl = dataclasses.replace(synth.WORKLOADS["single256"], page_size=ps)
    c = make_case(kvq.KV_INT4_BDR, 128, False, lengths, wl, seed=22, code_bits=2)
    _run(c, lengths, wl.num_q_heads)


def test_int2_with_rope():
    lengths = [500, 129]
    tab = synth.rope_table(600)
    c = make_case(kvq.KV_INT4_BDR, 64, True, lengths, WL, seed=23, rope=tab, code_bits=2)
    _run(c, lengths, WL.num_q_heads)


def test_int2_nan_rows():
    k, v = synth.make_kv(40, synth.WORKLOADS["single256"], 24)
    k[3, 2, 0] = float("nan")
    k[9, 5, 77] = float("nan")
    c = make_case(kvq.KV_INT4_BDR, 128, False, [40], synth.WORKLOADS["single256"], seed=24, code_bits=2)
    assert gpu_append(c, k=k, v=v) == kvq.KV_OK
    oracle_append(c, k=k, v=v)
    assert_pools_equal(c)
