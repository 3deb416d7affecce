"""GPU parity of the fused append kernel (C ABI kv_append_quant) against the CPU oracle:
whole pools (codes and scale/zero words, untouched slots included) must match bit for bit."""
import numpy as np
import pytest
import torch

from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import (FILL, assert_pools_equal, gpu_append, make_case, np_pool, oracle_append)

pytestmark = pytest.mark.gpu

WL0 = synth.WORKLOADS["single256"]
VARIANTS = [("bf16", kvq.KV_BF16, 0, False), ("int4", kvq.KV_INT4, 0, False)] + [
    (f"bdr{b}{'kv' if rv else 'k'}", kvq.KV_INT4_BDR, b, rv) for b in (16, 32, 64, 128) for rv in (False, True)]


@pytest.mark.parametrize("name,mode,b,rv", VARIANTS, ids=[v[0] for v in VARIANTS])
def test_append_single_sequence(name, mode, b, rv):
    """1 sequence x 256 tokens, page size 16, 16 shuffled pages (+3 spare pages left untouched)."""
    c = make_case(mode, b, rv, [256], WL0, seed=0)
    pt_before = c.page_table.clone()
    assert gpu_append(c) == kvq.KV_OK
    assert oracle_append(c) == 0
    assert_pools_equal(c)
    assert torch.equal(c.page_table, pt_before)


@pytest.mark.parametrize("name,mode,b,rv", [v for v in VARIANTS if v[0] in ("bf16", "int4", "bdr128k",
                                                                             "bdr128kv", "bdr16k")],
                         ids=["bf16", "int4", "bdr16k", "bdr128k", "bdr128kv"])
def test_append_batch16(name, mode, b, rv):
    """16 sequences, lengths ~U[512, 4096], page size 16, shuffled global page table."""
    wl = synth.WORKLOADS["batch16"]
    lengths = synth.seq_lengths("batch16", seed=0)
    c = make_case(mode, b, rv, lengths, wl, seed=0)
    assert gpu_append(c) == kvq.KV_OK
    assert oracle_append(c) == 0
    assert_pools_equal(c)


@pytest.mark.parametrize("H,ps,lengths", [
    (8, 16, [1]), (8, 16, [3, 1, 2]), (8, 1, [5, 9]), (8, 7, [33, 1, 70]), (8, 64, [300]),
    (2, 16, [129, 77]), (1, 16, [600]), (16, 16, [17, 40]), (4, 32, [511]), (32, 8, [9, 10]),
    (8, 1024, [1500, 3]),
])
def test_append_ragged_shapes(H, ps, lengths):
    """Ragged tails (rows not a multiple of the 224-row tile), tiny, odd and the largest page sizes,
    other head counts."""
    wl = synth.Workload("t", H, 4 * H if H <= 32 else H, 128, ps, synth.OUTLIERS_X20, "test")
    for mode, b, rv in ((kvq.KV_INT4_BDR, 128, True), (kvq.KV_INT4_BDR, 32, False), (kvq.KV_BF16, 0, False)):
        c = make_case(mode, b, rv, lengths, wl, seed=sum(lengths) + H)
        assert gpu_append(c) == kvq.KV_OK
        assert oracle_append(c) == 0
        assert_pools_equal(c)


def _chunk_case_tokens(S, TT, whole, short, last):
    """Token count whose per-CTA chunks are `whole` tiles + `short` tokens on S SMs, the last chunk
    `last` tokens."""
    Tc = whole * TT + short
    N = (S - 1) * Tc + last
    assert 1 <= last <= Tc and -(-N // S) == Tc
    return N


# (H, whole tiles per chunk, short tokens, last chunk's tokens): the last chunk's remainder above
# the short box (it takes the whole-tile box) or within it, chunks of one short tile, other H
CHUNK_CASES = [(8, 1, 1, 21), (8, 2, 19, 42), (8, 0, 5, 5), (2, 1, 30, 10), (32, 3, 2, 6)]


@pytest.mark.parametrize("H,whole,short,last", CHUNK_CASES, ids=[f"H{c[0]}_w{c[1]}_s{c[2]}_l{c[3]}" for c in CHUNK_CASES])
def test_append_chunk_schedule(H, whole, short, last):
    """Each CTA appends a contiguous chunk of ceil(T / SMs) tokens: a short first tile (its own
    small TMA box) when the chunk is not whole tiles, then whole tiles of 224 / H tokens."""
    S = torch.cuda.get_device_properties(0).multi_processor_count
    N = _chunk_case_tokens(S, 224 // H, whole, short, last)
    lengths = [N // 3, N // 3, N - 2 * (N // 3)]
    wl = synth.Workload("t", H, 4 * H if H <= 32 else H, 128, 16, synth.OUTLIERS_X20, "test")
    for mode, b, rv in ((kvq.KV_INT4_BDR, 128, True), (kvq.KV_BF16, 0, False)):
        c = make_case(mode, b, rv, lengths, wl, seed=N + H)
        assert gpu_append(c) == kvq.KV_OK
        assert oracle_append(c) == 0
        assert_pools_equal(c)


def test_append_fewer_tokens_than_sms():
    """Fewer tokens than SMs: one token per CTA, each a short tile of H rows."""
    S = torch.cuda.get_device_properties(0).multi_processor_count
    wl = synth.Workload("t", 8, 32, 128, 16, synth.OUTLIERS_X20, "test")
    for mode, b, rv in ((kvq.KV_INT4_BDR, 64, False), (kvq.KV_INT4, 0, False)):
        c = make_case(mode, b, rv, [S // 2, S // 3], wl, seed=5)
        assert gpu_append(c) == kvq.KV_OK
        assert oracle_append(c) == 0
        assert_pools_equal(c)


def test_append_empty_is_noop():
    c = make_case(kvq.KV_INT4_BDR, 128, False, [4], WL0)
    e = torch.empty(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    i = torch.empty(0, dtype=torch.int32, device="cuda")
    kvq.kv_append_quant(c.cache.handle, e, e, 0, i, i, c.page_table.cuda(), c.page_table.shape[1], 1)
    assert c.cache.get_error() == kvq.KV_OK
    assert np.all(np_pool(c.cache.k_pool) == FILL) and np.all(np_pool(c.cache.k_sz).view(np.uint8) == FILL)


def test_append_out_of_range_is_skipped_and_flagged():
    """Bad sequence ids, negative / too-large positions and out-of-pool page ids are skipped
    (never dereferenced) and reported as KV_ERR_OOB; every valid token is still written."""
    c = make_case(kvq.KV_INT4_BDR, 64, True, [40], WL0, seed=3)
    pt = c.page_table.clone()
    pt[0, 1] = c.num_pages + 5  # positions 16..31 point outside the pool
    c.page_table = pt
    ts = c.tok_seq.clone()
    tp = c.tok_pos.clone()
    ts[3] = 7  # no such sequence
    tp[5] = -2
    tp[6] = 10_000  # beyond the page table
    assert gpu_append(c, ts=ts, tp=tp) == kvq.KV_ERR_OOB
    assert oracle_append(c, ts=ts, tp=tp) == 3 + 16
    assert_pools_equal(c)
    assert c.cache.get_error() == kvq.KV_OK  # reading the error word clears it


def _special_rows(H):
    rows = []
    rows.append(torch.full((128,), 1.75))  # constant: scale 0
    rows.append(torch.zeros(128))
    z = torch.zeros(128)
    z[::2] = -0.0  # signed zeros
    rows.append(z)
    rows.append(torch.linspace(-3, 3, 128))
    rows.append(torch.randn(128, generator=torch.Generator().manual_seed(1)) * 1e4)
    rows.append(torch.randn(128, generator=torch.Generator().manual_seed(6)) * 3e5)  # scale and zero overflow fp16
    rows.append(torch.randn(128, generator=torch.Generator().manual_seed(2)) * 1e-6)  # subnormal fp16 scale
    big = torch.randn(128, generator=torch.Generator().manual_seed(3))
    big[7] = -9e4  # zero = fp16(min) overflows to -inf
    rows.append(big)
    off = torch.randn(128, generator=torch.Generator().manual_seed(4)) * 1e-3 + 300.0  # |min|/range large
    rows.append(off)
    levels = (torch.arange(128) % 16).float() * 0.5
    rows.append(levels)
    for where in (0, 77):  # a NaN anywhere: every code 0, scale = zero = fp16 NaN
        nan_row = torch.linspace(-2, 3, 128)
        nan_row[where] = float("nan")
        rows.append(nan_row)
    x = torch.stack(rows)  # [R, 128]
    reps = -(-(H * 40) // x.shape[0])
    return x.repeat(reps, 1)[: H * 40].reshape(40, H, 128).to(torch.bfloat16)


@pytest.mark.parametrize("b,rv", [(0, False), (16, True), (128, True)])
def test_append_special_values(b, rv):
    """Constant rows, signed zeros, fp16 overflow of scale or zero, subnormal fp16 scales,
    rows far from zero, exact 16-level rows and rows holding a NaN take the same decisions
    as the oracle."""
    mode = kvq.KV_INT4 if b == 0 else kvq.KV_INT4_BDR
    c = make_case(mode, b, rv, [40], WL0, seed=5)
    k = _special_rows(8)
    v = k.flip(0).contiguous()
    assert gpu_append(c, k=k, v=v) == kvq.KV_OK
    oracle_append(c, k=k, v=v)
    assert_pools_equal(c)


def test_append_incremental_equals_bulk():
    """Decode-style appends (one token per sequence per call) give the same pools as one bulk append."""
    wl = synth.WORKLOADS["single256"]
    lengths = [20, 35, 7]
    bulk = make_case(kvq.KV_INT4_BDR, 128, False, lengths, wl, seed=9)
    assert gpu_append(bulk) == kvq.KV_OK
    inc = make_case(kvq.KV_INT4_BDR, 128, False, lengths, wl, seed=9)
    order = torch.argsort(inc.tok_pos * 16 + inc.tok_seq, stable=True)  # position-major interleave
    for chunk in torch.split(order, 3):
        assert gpu_append(inc, k=inc.k[chunk], v=inc.v[chunk], ts=inc.tok_seq[chunk], tp=inc.tok_pos[chunk]) \
            == kvq.KV_OK
    for a, b in zip((bulk.cache.k_pool, bulk.cache.v_pool, bulk.cache.k_sz, bulk.cache.v_sz),
                    (inc.cache.k_pool, inc.cache.v_pool, inc.cache.k_sz, inc.cache.v_sz)):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
