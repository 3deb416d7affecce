"""GPU parity of the fused rotary embedding (keys turned at their position before the block
rotation in kv_append_quant; q turned at position seq_len - 1 in kv_decode_attn) against the
oracle: appended pools bit for bit, attention within ATTN_RTOL; positions outside the table
skipped and flagged."""
import dataclasses

import numpy as np
import pytest
import torch

from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import (ATTN_RTOL, assert_pools_equal, attn_rel_err, gpu_append, gpu_decode, make_case,
                         oracle_append, oracle_decode)

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["batch16"]
VARIANTS = [("bf16", kvq.KV_BF16, 0, False), ("int4", kvq.KV_INT4, 0, False), ("bdr128k", kvq.KV_INT4_BDR, 128, False),
            ("bdr64kv", kvq.KV_INT4_BDR, 64, True), ("bdr16kv", kvq.KV_INT4_BDR, 16, True)]


@pytest.mark.parametrize("name,mode,b,rv", VARIANTS, ids=[v[0] for v in VARIANTS])
@pytest.mark.parametrize("hq", [32, 64])
def test_rope_append_and_decode(name, mode, b, rv, hq):
    """Append with RoPE bit-exact, decode with q turned at its position within tolerance, for the
    tokens-on-M (G = 4), heads-on-M (G = 8) and BF16 decode kernels."""
    lengths = [700, 1301, 64]
    wl = dataclasses.replace(WL, num_q_heads=hq)
    tab = synth.rope_table(max(lengths) + 5)
    c = make_case(mode, b, rv, lengths, wl, seed=11, rope=tab)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    q = synth.make_q(len(lengths), hq, 128, seed=12)
    out, st = gpu_decode(c, q, lengths)
    assert st == kvq.KV_OK
    ref, skipped = oracle_decode(c, q, lengths)
    assert skipped == 0
    assert attn_rel_err(out.cpu().numpy(), ref) <= ATTN_RTOL


def test_rope_positions_outside_the_table_are_skipped_and_flagged():
    lengths = [40, 20]
    tab = synth.rope_table(32)  # tokens 32..39 of the first sequence have no table row
    c = make_case(kvq.KV_INT4_BDR, 128, False, lengths, synth.WORKLOADS["single256"], seed=13, rope=tab)
    assert gpu_append(c) == kvq.KV_ERR_OOB
    skipped = oracle_append(c)
    assert skipped == 8
    assert_pools_equal(c)
    # decode: the first sequence's query position 39 has no table row -> zero output, flagged
    q = synth.make_q(2, 32, 128, seed=14)
    out, st = gpu_decode(c, q, [40, 20])
    assert st == kvq.KV_ERR_OOB
    ref, _ = oracle_decode(c, q, [40, 20])
    assert not out[0].any()
    assert attn_rel_err(out[1].cpu().numpy(), ref[1]) <= ATTN_RTOL


def test_rope_identity_table_equals_no_rope():
    lengths = [300, 77]
    ident = torch.zeros(400, 64, 2)
    ident[..., 0] = 1.0
    a = make_case(kvq.KV_INT4_BDR, 128, False, lengths, WL, seed=15)
    b = make_case(kvq.KV_INT4_BDR, 128, False, lengths, WL, seed=15, rope=ident)
    assert gpu_append(a) == kvq.KV_OK and gpu_append(b) == kvq.KV_OK
    for x, y in ((a.cache.k_pool, b.cache.k_pool), (a.cache.k_sz, b.cache.k_sz), (a.cache.v_pool, b.cache.v_pool)):
        assert torch.equal(x, y)
    q = synth.make_q(2, 32, 128, seed=16)
    oa, _ = gpu_decode(a, q, lengths)
    ob, _ = gpu_decode(b, q, lengths)
    assert torch.equal(oa, ob)
