"""Parity at the full sizes of the serving workloads, in the launch configuration bench.py
times: the whole cache is built with kv_append_quant on the GPU, then a serving step (new
tokens appended, decode attention) runs; sampled appended rows are compared bit for bit
with the oracle's quantiser, and every query head of at least two whole sequences (the
longest among them where lengths differ; the one sequence of long1m) with the oracle's
float64 decode over the same pages."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import ATTN_RTOL, attn_rel_err, bits16, oracle_decode_rows

pytestmark = pytest.mark.gpu


def _pool_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _check_rows(cache, k, v, ts, tp, pt, mode, b, rv, n_samples, seed):
    """Sampled appended tokens: codes and scale/zero of every KV head bit-exact vs the oracle."""
    rng = np.random.default_rng(seed)
    idx = np.sort(rng.choice(k.shape[0], size=min(n_samples, k.shape[0]), replace=False))
    it = torch.as_tensor(idx, device=k.device)
    kb, vb = bits16(k[it]), bits16(v[it])
    seqs, poss = ts[it].cpu().numpy(), tp[it].cpu().numpy()
    ptn = pt.cpu().numpy()
    ps = cache.page_size
    pages = ptn[seqs, poss // ps]
    slots = poss % ps
    pg_t, sl_t = torch.as_tensor(pages, device=k.device), torch.as_tensor(slots, device=k.device)
    gk = cache.k_pool[pg_t, :, sl_t].cpu().numpy()
    gv = cache.v_pool[pg_t, :, sl_t].cpu().numpy()
    gks = _pool_bits(cache.k_sz[pg_t, :, sl_t])
    gvs = _pool_bits(cache.v_sz[pg_t, :, sl_t])
    bk = b if mode == kvq.KV_INT4_BDR else 0
    bv = b if (mode == kvq.KV_INT4_BDR and rv) else 0
    ck, sk = oracle.quant_rows(kb, bk)
    cv, sv = oracle.quant_rows(vb, bv)
    assert np.array_equal(gk, ck) and np.array_equal(gks, sk)
    assert np.array_equal(gv, cv) and np.array_equal(gvs, sv)


def _check_decode(cache, q, seq_lens, pt, max_len, mode, b, rv, rows):
    out = cache.decode(q, torch.as_tensor(seq_lens, dtype=torch.int32, device="cuda"), pt, max_len, out_fp32=True)
    out16 = cache.decode(q, torch.as_tensor(seq_lens, dtype=torch.int32, device="cuda"), pt, max_len)
    assert cache.get_error() == kvq.KV_OK
    assert torch.equal(out16, out.to(torch.bfloat16))
    pools = (cache.k_pool.cpu().numpy(), cache.v_pool.cpu().numpy(), _pool_bits(cache.k_sz), _pool_bits(cache.v_sz))
    ref, skipped = oracle_decode_rows(mode, b, rv, pools, bits16(q), seq_lens, pt.cpu().numpy(), cache.num_kv_heads,
                                      rows)
    assert skipped == 0
    got = np.stack([out[s, j].cpu().numpy() for s, j in rows])
    err = attn_rel_err(got, ref)
    assert err <= ATTN_RTOL, err


def test_decode64x8k_step():
    """64 sequences x 8192 cached tokens (page size 16), BDR-128 on keys; one serving step
    appends 1 token per sequence and decodes all 64."""
    wl = synth.WORKLOADS["decode64x8k"]
    lengths = synth.seq_lengths("decode64x8k", seed=0)
    B, H, Hq, ps = len(lengths), wl.num_kv_heads, wl.num_q_heads, wl.page_size
    mode, b, rv = kvq.KV_INT4_BDR, 128, False
    pt, P = synth.make_page_table([L + 100 for L in lengths], ps, seed=0)
    cache = kvq.PagedKVCache(P, ps, H, Hq, mode, b, rv, fill=0)
    ptd = pt.cuda()
    k, v = synth.make_kv(sum(lengths), wl, seed=0, device="cuda", chunk=8192)
    ts, tp = synth.append_positions(lengths)
    ts, tp = ts.cuda(), tp.cuda()
    cache.append(k, v, ts, tp, ptd)
    _check_rows(cache, k, v, ts, tp, pt, mode, b, rv, 512, seed=1)
    del k, v
    # the step: one new token per sequence at position L, then decode L + 1 tokens
    k1, v1 = synth.make_kv(B, wl, seed=1, device="cuda")
    ts1, tp1 = synth.append_positions([1] * B, lengths)
    cache.append(k1, v1, ts1.cuda(), tp1.cuda(), ptd)
    _check_rows(cache, k1, v1, ts1.cuda(), tp1.cuda(), pt, mode, b, rv, B, seed=2)
    new_lens = [L + 1 for L in lengths]
    q = synth.make_q(B, Hq, 128, seed=3).cuda()
    # every query head of two whole sequences (all lengths are equal here)
    seqs = [0, int(np.random.default_rng(4).integers(1, B))]
    rows = [(s, j) for s in seqs for j in range(Hq)]
    _check_decode(cache, q, new_lens, ptd, max(new_lens), mode, b, rv, rows)


def test_mixed256_step():
    """256 sequences, lengths log-uniform in [1024, 32768], 64 query heads over 8 KV heads,
    BDR-128 on keys and values; one step appends a 2048-token chunk to 8 sequences and one
    token to each of the other 248, then decodes those 248."""
    wl = synth.WORKLOADS["mixed256"]
    lengths = synth.seq_lengths("mixed256", seed=0)
    B, H, Hq, ps = len(lengths), wl.num_kv_heads, wl.num_q_heads, wl.page_size
    mode, b, rv = kvq.KV_INT4_BDR, 128, True
    pt, P = synth.make_page_table([L + 2048 for L in lengths], ps, seed=0)
    cache = kvq.PagedKVCache(P, ps, H, Hq, mode, b, rv, fill=0)
    ptd = pt.cuda()
    T = sum(lengths)
    ts, tp = synth.append_positions(lengths)
    for c0 in range(0, T, 1 << 20):  # build the cache in pieces of 1 Mi tokens
        c1 = min(T, c0 + (1 << 20))
        k, v = synth.make_kv(c1 - c0, wl, seed=10 + c0, device="cuda")
        cache.append(k, v, ts[c0:c1].cuda(), tp[c0:c1].cuda(), ptd)
        if c0 == 0:
            _check_rows(cache, k, v, ts[c0:c1].cuda(), tp[c0:c1].cuda(), pt, mode, b, rv, 256, seed=1)
        del k, v
    rng = np.random.default_rng(7)
    prefill = sorted(rng.choice(B, 8, replace=False).tolist())
    decoding = [s for s in range(B) if s not in prefill]
    step_lens = [2048 if s in prefill else 1 for s in range(B)]
    k1, v1 = synth.make_kv(sum(step_lens), wl, seed=2, device="cuda")
    ts1, tp1 = synth.append_positions(step_lens, lengths)
    cache.append(k1, v1, ts1.cuda(), tp1.cuda(), ptd)
    _check_rows(cache, k1, v1, ts1.cuda(), tp1.cuda(), pt, mode, b, rv, 512, seed=3)
    assert cache.get_error() == kvq.KV_OK
    # decode the 248 decoding sequences (their own page-table rows, in order)
    dl = [lengths[s] + 1 for s in decoding]
    ptdec = pt[decoding].contiguous()
    q = synth.make_q(len(decoding), Hq, 128, seed=4).cuda()
    # every query head of the longest decoding sequence and of one other
    longest = int(np.argmax(dl))
    other = int(np.random.default_rng(8).choice([i for i in range(len(decoding)) if i != longest]))
    rows = [(s, j) for s in (longest, other) for j in range(Hq)]
    _check_decode(cache, q, dl, ptdec.cuda(), max(dl), mode, b, rv, rows)


def test_long1m_chunked_append_and_decode():
    """One sequence of 1,048,576 tokens, page size 64, appended in 8192-token chunks, then
    split-K decode over the whole context; BDR-128 on keys."""
    wl = synth.WORKLOADS["long1m"]
    L = synth.seq_lengths("long1m", seed=0)[0]
    H, Hq, ps = wl.num_kv_heads, wl.num_q_heads, wl.page_size
    mode, b, rv = kvq.KV_INT4_BDR, 128, False
    pt, P = synth.make_page_table([L], ps, seed=0)
    cache = kvq.PagedKVCache(P, ps, H, Hq, mode, b, rv, fill=0)
    ptd = pt.cuda()
    k, v = synth.make_kv(L, wl, seed=0, device="cuda", chunk=8192)
    ts, tp = synth.append_positions([L])
    ts, tp = ts.cuda(), tp.cuda()
    for c0 in range(0, L, 8192):
        cache.append(k[c0:c0 + 8192], v[c0:c0 + 8192], ts[c0:c0 + 8192], tp[c0:c0 + 8192], ptd)
    _check_rows(cache, k, v, ts, tp, pt, mode, b, rv, 1024, seed=1)
    del k, v
    q = synth.make_q(1, Hq, 128, seed=3).cuda()
    _check_decode(cache, q, [L], ptd, L, mode, b, rv, [(0, j) for j in range(Hq)])  # every query head
