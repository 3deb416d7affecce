"""GPU parity of the extend (chunked-prefill) attention kernel (kv_extend_attn) with the
oracle's float64 extend: every (query, head) row within ATTN_RTOL, the bf16 output the fp32
one rounded to nearest even bit for bit; pools built by kv_append_quant and checked bit for
bit against the oracle's first.  Sizes span several 64 / G-query blocks per sequence, ragged
block and chunk tails, both page-copy paths, every G, 4- and 2-bit codes; then the edge
cases and the full-size chunked-prefill step of the mixed serving workload."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import (ATTN_RTOL, FILL, assert_pools_equal, attn_rel_err, bits16, gpu_append, make_case,
                         oracle_append)

pytestmark = pytest.mark.gpu

BASE = synth.WORKLOADS["batch16"]


def _wl(H, Hq, ps):
    return dataclasses.replace(BASE, num_kv_heads=H, num_q_heads=Hq, page_size=ps)


def _indptr(qlens):
    return np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)


def gpu_extend(c, q, qlens, seq_lens, max_q_len=None, out_fp32=True, out=None):
    qi = torch.as_tensor(_indptr(qlens), dtype=torch.int32).cuda()
    sl = torch.as_tensor(seq_lens, dtype=torch.int32).cuda()
    mq = max(qlens) if max_q_len is None else max_q_len
    o = c.cache.extend(q.cuda(), qi, sl, c.page_table.cuda(), mq, max(seq_lens), out=out, out_fp32=out_fp32)
    return o, c.cache.get_error()


def oracle_extend(c, q, qlens, seq_lens, rows=None, page_table=None):
    kp, vp, ks, vs = c.ref_pools
    pt = (c.page_table if page_table is None else page_table).numpy()
    return oracle.extend(c.mode, c.bdr, c.rotate_v, kp, vp, ks, vs, bits16(q), _indptr(qlens),
                         np.asarray(seq_lens), pt, c.wl.num_kv_heads, rows=rows,
                         rope=None if c.rope is None else c.rope.numpy(), code_bits=c.code_bits)


def _built(mode, b, rv, lengths, wl, seed, rope=None, code_bits=4):
    c = make_case(mode, b, rv, lengths, wl, seed=seed, rope=rope, code_bits=code_bits)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    return c


CASES = [  # (id, H, Hq, page size, mode, block, rotate_v, code bits)
    ("g4_bdr128k", 2, 8, 16, kvq.KV_INT4_BDR, 128, False, 4),
    ("g8_bdr128kv", 2, 16, 16, kvq.KV_INT4_BDR, 128, True, 4),
    ("g4_int4_ps7", 2, 8, 7, kvq.KV_INT4, 0, False, 4),
    ("g1_bdr64kv", 4, 4, 16, kvq.KV_INT4_BDR, 64, True, 4),
    ("g2_bdr128kv_ps32", 4, 8, 32, kvq.KV_INT4_BDR, 128, True, 4),
    ("g2_bdr32k_int2", 2, 4, 16, kvq.KV_INT4_BDR, 32, False, 2),
    ("g8_bdr16kv_int2_ps12", 1, 8, 12, kvq.KV_INT4_BDR, 16, True, 2),
]


@pytest.mark.parametrize("name,H,Hq,ps,mode,b,rv,bits", CASES, ids=[c[0] for c in CASES])
def test_extend_matches_oracle(name, H, Hq, ps, mode, b, rv, bits):
    """A full prefill from position 0 (300 queries), a 13-query chunk after 64 cached tokens and a
    129-query chunk after 511: every row of both outputs against the oracle."""
    lengths, qlens = [300, 77, 640], [300, 13, 129]
    c = _built(mode, b, rv, lengths, _wl(H, Hq, ps), seed=21, code_bits=bits)
    q = synth.make_q(sum(qlens), Hq, 128, seed=22)
    out, st = gpu_extend(c, q, qlens, lengths)
    assert st == kvq.KV_OK
    out16, st16 = gpu_extend(c, q, qlens, lengths, out_fp32=False)
    assert st16 == kvq.KV_OK
    assert torch.equal(out16, out.to(torch.bfloat16))
    ref, skipped = oracle_extend(c, q, qlens, lengths)
    assert skipped == 0
    assert attn_rel_err(out.cpu().numpy(), ref) <= ATTN_RTOL


def test_extend_with_rotary_table_and_rows_outside_it():
    """q turned at each query's own position; the queries whose position has no table row give
    zero rows and KV_ERR_OOB, the rest match the oracle."""
    lengths, qlens = [90, 150], [90, 40]
    tab = synth.rope_table(140)  # positions 140..149 of the second sequence have no row
    c = make_case(kvq.KV_INT4_BDR, 128, False, lengths, _wl(2, 8, 16), seed=23, rope=synth.rope_table(160))
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    q = synth.make_q(sum(qlens), 8, 128, seed=24)
    # a second handle over the same pools with the shorter table
    c2 = dataclasses.replace(c)
    c2.rope = tab
    c2.cache = kvq.PagedKVCache(c.num_pages, 16, 2, 8, kvq.KV_INT4_BDR, 128, False,
                                pools=(c.cache.k_pool, c.cache.v_pool, c.cache.k_sz, c.cache.v_sz),
                                rope=tab.cuda())
    out, st = gpu_extend(c2, q, qlens, lengths)
    assert st == kvq.KV_ERR_OOB
    ref, _ = oracle_extend(c2, q, qlens, lengths)
    o = out.cpu().numpy()
    assert not o[-10:].any()
    assert attn_rel_err(o, ref) <= ATTN_RTOL
    out_full, st_full = gpu_extend(c, q, qlens, lengths)
    assert st_full == kvq.KV_OK
    ref_full, skipped = oracle_extend(c, q, qlens, lengths)
    assert skipped == 0
    assert attn_rel_err(out_full.cpu().numpy(), ref_full) <= ATTN_RTOL


def test_extend_edge_cases():
    lengths = [40, 17, 33]
    c = _built(kvq.KV_INT4_BDR, 64, True, lengths, _wl(2, 8, 16), seed=25)
    # more queries than cached tokens: the first ones have no tokens -> zero rows, flagged
    qlens = [45, 0, 33]
    q = synth.make_q(sum(qlens), 8, 128, seed=26)
    out, st = gpu_extend(c, q, qlens, lengths)
    assert st == kvq.KV_ERR_OOB
    ref, _ = oracle_extend(c, q, qlens, lengths)
    o = out.cpu().numpy()
    assert not o[:5].any()
    assert attn_rel_err(o, ref) <= ATTN_RTOL
    # max_q_len below a sequence's query count: only its last max_q_len queries are written
    qlens = [20, 17, 33]
    q = synth.make_q(sum(qlens), 8, 128, seed=27)
    sentinel = torch.full((sum(qlens), 8, 128), 7.0, dtype=torch.float32, device="cuda")
    out, st = gpu_extend(c, q, qlens, lengths, max_q_len=16, out=sentinel)
    assert st == kvq.KV_ERR_OOB
    ref, _ = oracle_extend(c, q, qlens, lengths)
    o = out.cpu().numpy()
    written = np.r_[4:20, 20 + 1:37, 37 + 17:70]
    untouched = np.r_[0:4, 20:21, 37:54]
    assert np.all(o[untouched] == 7.0)
    assert attn_rel_err(o[written], ref[written]) <= ATTN_RTOL
    # a page id outside the pool: its tokens are skipped (and flagged), as in the oracle
    pt = c.page_table.clone()
    pt[0, 1] = c.num_pages + 5
    qlens = [40, 1, 1]
    q = synth.make_q(sum(qlens), 8, 128, seed=28)
    qi = torch.as_tensor(_indptr(qlens)).cuda()
    out = c.cache.extend(q.cuda(), qi, torch.as_tensor(lengths, dtype=torch.int32).cuda(), pt.cuda(), 40, 40,
                         out_fp32=True)
    assert c.cache.get_error() == kvq.KV_ERR_OOB
    ref, skipped = oracle_extend(c, q, qlens, lengths, page_table=pt)
    assert skipped > 0
    assert attn_rel_err(out.cpu().numpy(), ref) <= ATTN_RTOL
    # empty calls are no-ops
    kvq.kv_extend_attn(c.cache.handle, q.cuda(), qi, qi, pt.cuda(), pt.shape[1], 0, 1, 1, out, 1)
    kvq.kv_extend_attn(c.cache.handle, q.cuda(), qi, qi, pt.cuda(), pt.shape[1], 3, 0, 1, out, 1)
    assert c.cache.get_error() == kvq.KV_OK


def test_extend_rejects_bf16_pages():
    c = make_case(kvq.KV_BF16, 0, False, [16], _wl(2, 8, 16), seed=29)
    q = torch.zeros(1, 8, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        gpu_extend(c, q, [1], [16])
    assert e.value.status == kvq.KV_ERR_UNSUPPORTED


def test_mixed256_prefill_chunks():
    """Full size: the 8 prefilling sequences of the mixed serving workload (64 query heads over
    8 KV heads, BDR-128 on K and V, cached lengths log-uniform in [1024, 32768] plus the
    2048-token chunk), extend over the chunk in the launch configuration bench.py times; pools
    bit-exact, sampled rows against the oracle."""
    wl = synth.WORKLOADS["mixed256"]
    all_lengths = synth.seq_lengths("mixed256", seed=0)
    rng = np.random.default_rng(7)
    pick = sorted(rng.choice(len(all_lengths), 8, replace=False).tolist())
    lengths = [all_lengths[s] + 2048 for s in pick]
    c = make_case(kvq.KV_INT4_BDR, 128, True, lengths, wl, seed=31)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    qlens = [2048] * 8
    q = synth.make_q(sum(qlens), wl.num_q_heads, 128, seed=32)
    out, st = gpu_extend(c, q, qlens, lengths)
    assert st == kvq.KV_OK
    rr = np.random.default_rng(33)
    rows = []
    for s in range(8):
        for i in (0, 1, 2047, *rr.choice(2048, 3).tolist()):
            rows.append((2048 * s + int(i), int(rr.integers(wl.num_q_heads))))
    ref, skipped = oracle_extend(c, q, qlens, lengths, rows=rows)
    assert skipped == 0
    got = np.stack([out[r, j].cpu().numpy() for r, j in rows])
    assert attn_rel_err(got, ref) <= ATTN_RTOL
