"""GPU parity of paged GQA decode attention (C ABI kv_decode_attn) against the float64 oracle
over the same (oracle-verified) cache: fp32 output within ATTN_RTOL per row, bf16 output equal
to the fp32 output rounded to nearest even."""
import numpy as np
import pytest
import torch

from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import (ATTN_RTOL, assert_pools_equal, attn_rel_err, gpu_append, gpu_decode, make_case,
                         oracle_append, oracle_decode)

pytestmark = pytest.mark.gpu

WL0 = synth.WORKLOADS["single256"]
SWEEP = [("bf16", kvq.KV_BF16, 0, False), ("int4", kvq.KV_INT4, 0, False)] + [
    (f"bdr{b}{'kv' if rv else 'k'}", kvq.KV_INT4_BDR, b, rv) for b in (16, 32, 64, 128) for rv in (False, True)]


def _run(c, lengths, q_seed=1, max_len=None):
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    q = synth.make_q(len(lengths), c.wl.num_q_heads, 128, seed=q_seed)
    out32, st = gpu_decode(c, q, lengths, max_len=max_len, out_fp32=True)
    assert st == kvq.KV_OK
    out16, st = gpu_decode(c, q, lengths, max_len=max_len, out_fp32=False)
    assert st == kvq.KV_OK
    ref, skipped = oracle_decode(c, q, lengths)
    assert skipped == 0
    err = attn_rel_err(out32.cpu().numpy(), ref)
    assert err <= ATTN_RTOL, err
    assert torch.equal(out16, out32.to(torch.bfloat16))
    return err


@pytest.mark.parametrize("name,mode,b,rv", SWEEP, ids=[v[0] for v in SWEEP])
def test_decode_single_sequence(name, mode, b, rv):
    c = make_case(mode, b, rv, [256], WL0, seed=0)
    _run(c, [256])


@pytest.mark.parametrize("name,mode,b,rv", SWEEP, ids=[v[0] for v in SWEEP])
def test_decode_batch16_sweep(name, mode, b, rv):
    """16 sequences, lengths ~U[512, 4096], every variant of the block-size / K-vs-KV sweep."""
    wl = synth.WORKLOADS["batch16"]
    lengths = synth.seq_lengths("batch16", seed=0)
    c = make_case(mode, b, rv, lengths, wl, seed=0)
    _run(c, lengths)


def test_decode_gqa8_mixed_lengths():
    """64 query heads over 8 KV heads (G = 8), K+V rotated, lengths from 1 to a few thousand."""
    wl = synth.WORKLOADS["mixed256"]
    lengths = [1, 2, 15, 16, 17, 33, 500, 1024, 3001]
    c = make_case(kvq.KV_INT4_BDR, 128, True, lengths, wl, seed=4)
    _run(c, lengths)


@pytest.mark.parametrize("G", [1, 2, 8])
def test_decode_group_sizes(G):
    wl = synth.Workload("t", 4, 4 * G, 128, 16, synth.OUTLIERS_X20, "test")
    lengths = [70, 300]
    c = make_case(kvq.KV_INT4_BDR, 64, False, lengths, wl, seed=G)
    _run(c, lengths)


@pytest.mark.parametrize("mode,b", [(kvq.KV_INT4_BDR, 128), (kvq.KV_BF16, 0)], ids=["bdr128k", "bf16"])
def test_decode_long_sequence_many_splits(mode, b):
    """One 40k-token sequence, page size 64: split-K across the context, then the merge."""
    wl = synth.Workload("t", 8, 32, 128, 64, synth.OUTLIERS_1PCT, "test")
    lengths = [40_000]
    c = make_case(mode, b, False, lengths, wl, seed=2)
    _run(c, lengths)


def test_decode_long_rows_shared_by_merge_warps():
    """More than 32 splits per row and few rows: the merge CTA's four warps share each row (the
    40k-token row has three passes of 32 splits, so one warp holds none) and warp 0 combines
    them; values rotated, so the merged output is turned back; an empty and a short sequence in
    the same batch."""
    wl = synth.Workload("t", 8, 32, 128, 64, synth.OUTLIERS_1PCT, "test")
    c = make_case(kvq.KV_INT4_BDR, 64, True, [40_000, 1, 3000], wl, seed=4)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    lengths = [40_000, 0, 3000]
    q = synth.make_q(3, 32, 128, seed=9)
    ref, skipped = oracle_decode(c, q, lengths)
    assert skipped == 0
    out32, st = gpu_decode(c, q, lengths, out_fp32=True)
    assert st == kvq.KV_OK
    o = out32.cpu().numpy()
    assert not o[1].any()
    assert attn_rel_err(o, ref) <= ATTN_RTOL
    out16, st = gpu_decode(c, q, lengths, out_fp32=False)
    assert st == kvq.KV_OK
    assert torch.equal(out16, out32.to(torch.bfloat16))


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_bf16_group_sizes_nan_filled_pool(G):
    """BF16 pages, every group size.  The pools hold NaN bits before the append, so the slots
    past each sequence's end, which its last 16-token chunk copies too, are NaN; a page id
    outside the pool is skipped.  Masked rows must never reach the P.V product."""
    wl = synth.Workload("t", 4, 4 * G, 128, 16, synth.OUTLIERS_X20, "test")
    lengths = [1, 17, 333, 2100]
    c = make_case(kvq.KV_BF16, 0, False, lengths, wl, seed=10 + G)
    for t in (c.cache.k_pool, c.cache.v_pool):
        t.view(torch.uint8).fill_(0xFF)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    q = synth.make_q(len(lengths), 4 * G, 128, seed=3)
    ref, _ = oracle_decode(c, q, lengths)
    out, st = gpu_decode(c, q, lengths)
    assert st == kvq.KV_OK
    assert torch.isfinite(out).all()
    assert attn_rel_err(out.cpu().numpy(), ref) <= ATTN_RTOL
    pt = c.page_table.clone()
    pt[3, 5] = -7
    out, st = gpu_decode(c, q, lengths, page_table=pt)
    assert st == kvq.KV_ERR_OOB
    ref, skipped = oracle_decode(c, q, lengths, page_table=pt)
    assert skipped == 16 * 4 * G
    assert torch.isfinite(out).all()
    assert attn_rel_err(out.cpu().numpy(), ref) <= ATTN_RTOL


def test_decode_empty_and_loose_bound():
    """seq_len 0 gives a zero row; a max_seq_len bound above the real lengths changes only the plan."""
    lengths = [0, 5, 64]
    c = make_case(kvq.KV_INT4_BDR, 32, True, [1, 5, 64], WL0, seed=6)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    q = synth.make_q(3, 32, 128, seed=3)
    ref, _ = oracle_decode(c, q, lengths)
    for max_len in (64, 5000):
        out, st = gpu_decode(c, q, lengths, max_len=max_len)
        assert st == kvq.KV_OK
        o = out.cpu().numpy()
        assert not o[0].any()
        assert attn_rel_err(o, ref) <= ATTN_RTOL


def test_decode_out_of_range_is_flagged():
    """A length beyond the page table and a page id outside the pool are skipped and reported."""
    c = make_case(kvq.KV_INT4, 0, False, [48], WL0, seed=8)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    q = synth.make_q(1, 32, 128, seed=5)
    pt = c.page_table.clone()
    pt[0, 1] = -7
    out, st = gpu_decode(c, q, [48], page_table=pt)
    assert st == kvq.KV_ERR_OOB
    ref, skipped = oracle_decode(c, q, [48], page_table=pt)
    assert skipped == 16 * 32  # one page of 16 tokens, for each of the 32 query heads
    assert attn_rel_err(out.cpu().numpy(), ref) <= ATTN_RTOL
    big = c.page_table.shape[1] * 16 + 5
    out, st = gpu_decode(c, q, [big], max_len=big)
    assert st == kvq.KV_ERR_OOB


@pytest.mark.parametrize("ps", [1, 7, 24, 32, 48, 1024])
def test_decode_page_sizes(ps):
    """Page sizes that are not a multiple of 16 take the per-token gather; 32 and 48 the bulk copies."""
    wl = synth.Workload("t", 8, 32, 128, ps, synth.OUTLIERS_X20, "test")
    lengths = [5, 100, 333]
    for mode, b, rv in ((kvq.KV_INT4_BDR, 128, True), (kvq.KV_INT4, 0, False), (kvq.KV_BF16, 0, False)):
        c = make_case(mode, b, rv, lengths, wl, seed=ps)
        _run(c, lengths)


def test_stale_workspace_and_graph_replay():
    """The split-K scratch needs no initial contents: a workspace full of stale bytes of any
    kind, repeated calls, and replays of a captured CUDA graph of the decode (split and merge
    kernels, programmatic dependent launch) all give the same rows as a fresh call."""
    lengths = [700, 0, 1301, 64, 4100]
    c = make_case(kvq.KV_INT4_BDR, 128, True, lengths, synth.WORKLOADS["batch16"], seed=41)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    q = synth.make_q(len(lengths), 32, 128, seed=42).cuda()
    sl = torch.as_tensor(lengths, dtype=torch.int32).cuda()
    pt = c.page_table.cuda()
    ws, n = c.cache.workspace(len(lengths), max(lengths))
    ref, _ = oracle_decode(c, q.cpu(), lengths)
    outs = []
    for fill in (0xFF, 0x00, 0x5A):  # NaN, zero and arbitrary scratch words
        ws.fill_(fill)
        outs.append(c.cache.decode(q, sl, pt, max(lengths), out_fp32=True, workspace=(ws, n)))
        assert c.cache.get_error() == kvq.KV_OK
    for o in outs:
        assert torch.equal(o, outs[0])
    assert attn_rel_err(outs[0].cpu().numpy(), ref) <= ATTN_RTOL
    assert not outs[0][1].any()  # the empty sequence
    # capture one decode call in a graph and replay it (its call tag is baked in)
    out = torch.full_like(outs[0], 3.0)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        kvq.kv_decode_attn(c.cache.handle, q, sl, pt, pt.shape[1], len(lengths), max(lengths), out, 1, ws, n, stream)
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        kvq.kv_decode_attn(c.cache.handle, q, sl, pt, pt.shape[1], len(lengths), max(lengths), out, 1, ws, n,
                           torch.cuda.current_stream())
    for _ in range(3):
        out.fill_(3.0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, outs[0])
    del g
    assert c.cache.get_error() == kvq.KV_OK
