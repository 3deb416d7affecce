"""Pins of the oracle's extend (chunked-prefill) attention: the newest n_s tokens of each
sequence attend causally to the paged cache, query i at position seq_len - n_s + i (the
SAW-INT4 abstract keeps attention over the paged quantised cache a serving constraint;
the wispaper.ai blog, section 3, rotates the query in step).  The oracle states it as one
decode row per query; these tests hold it against a dense masked-matrix formulation of
causal attention built from the dequantised pools, against the one-query case (decode),
and against the invariants chunked prefill relies on.  CPU only."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_append_b200 import synth

D = 128
WL = synth.Workload("tiny", 2, 8, 128, 16, synth.OUTLIERS_X20, "2 KV heads, 8 query heads, page size 16")


def _case(mode, bdr, rotate_v, lengths, seed=0, rope=None, code_bits=4, wl=WL):
    """Oracle pools holding `lengths` tokens per sequence (one append from position 0)."""
    H, ps = wl.num_kv_heads, wl.page_size
    T = sum(lengths)
    k, v = synth.make_kv(T, wl, seed)
    pt, P = synth.make_page_table(lengths, ps, seed, spare_pages=2)
    ts, tp = synth.append_positions(lengths, None)
    if mode == oracle.MODE_BF16:
        kp = np.zeros((P, H, ps, D), np.uint16)
        ks = vs = np.zeros(1, np.uint16)
        vp = kp.copy()
    else:
        kp = np.zeros((P, H, ps, 16 * code_bits), np.uint8)
        vp = kp.copy()
        ks = np.zeros((P, H, ps, 2), np.uint16)
        vs = ks.copy()

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    skipped = oracle.append(mode, bdr, rotate_v, kp, vp, ks, vs, bits(k), bits(v), ts.numpy(), tp.numpy(),
                            pt.numpy(), rope=rope, code_bits=code_bits)
    assert skipped == 0
    return (kp, vp, ks, vs), pt.numpy()


def _queries(total_q, seed, wl=WL):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(total_q, wl.num_q_heads, D, generator=g).to(torch.bfloat16)
    return q.view(torch.int16).numpy().view(np.uint16)


def _dequant(mode, pool, sz, rows, code_bits):
    """float64 [len(rows), D] of the cached rows (value = code * scale + zero)."""
    if mode == oracle.MODE_BF16:
        b = pool.reshape(-1, D)[rows].astype(np.uint32) << 16
        return b.view(np.float32).astype(np.float64)
    codes = oracle.unpack_codes(pool.reshape(-1, pool.shape[-1])[rows], code_bits).astype(np.float64)
    s = sz.reshape(-1, 2)[rows].view(np.float16).astype(np.float64)
    return codes * s[:, :1] + s[:, 1:]


def _dense_extend(mode, bdr, rotate_v, pools, q_bits, q_indptr, seq_lens, pt, rope=None, code_bits=4, wl=WL):
    """Causal attention as masked matrices: S = Q K^T / sqrt(D) with S[i, j] = -inf for
    j > position of query i, softmax along j, O = P V (float64, dequantised pools)."""
    kp, vp, ks, vs = pools
    H, ps = wl.num_kv_heads, wl.page_size
    Hq = q_bits.shape[1]
    G = Hq // H
    out = np.zeros((q_bits.shape[0], Hq, D))
    for s in range(len(seq_lens)):
        a, b = q_indptr[s], q_indptr[s + 1]
        n, L = b - a, int(seq_lens[s])
        pos = L - n + np.arange(n)
        Q = (q_bits[a:b].astype(np.uint32) << 16).view(np.float32).astype(np.float64)  # [n, Hq, D]
        if rope is not None:
            c = rope[np.maximum(pos, 0), :, 0].astype(np.float64)[:, None, :]
            sn = rope[np.maximum(pos, 0), :, 1].astype(np.float64)[:, None, :]
            x, y = Q[..., :64].copy(), Q[..., 64:].copy()
            Q = np.concatenate([x * c - y * sn, y * c + x * sn], axis=-1)
        if mode == oracle.MODE_INT4_BDR:
            Q = oracle.rotate_f64(Q.reshape(-1, D), bdr).reshape(Q.shape)
        t = np.arange(L)
        mask = t[None, :] > pos[:, None]  # [n, L]
        for h in range(H):
            rows = (pt[s, t // ps].astype(np.int64) * H + h) * ps + t % ps
            K = _dequant(mode, kp, ks, rows, code_bits)
            V = _dequant(mode, vp, vs, rows, code_bits)
            for g in range(G):
                S = Q[:, h * G + g, :] @ K.T / np.sqrt(D)
                S[mask] = -np.inf
                live = pos >= 0
                S = S[live]
                P = np.exp(S - S.max(axis=1, keepdims=True))
                P /= P.sum(axis=1, keepdims=True)
                O = P @ V
                if mode == oracle.MODE_INT4_BDR and rotate_v:
                    O = oracle.rotate_f64(O, bdr)
                out[a:b][live, h * G + g, :] = O
    return out


def _run(mode, bdr, rotate_v, lengths, qlens, seed, rope=None, code_bits=4):
    pools, pt = _case(mode, bdr, rotate_v, lengths, seed, rope=rope, code_bits=code_bits)
    q_indptr = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = _queries(int(q_indptr[-1]), seed + 100)
    got, skipped = oracle.extend(mode, bdr, rotate_v, *pools, q, q_indptr, np.asarray(lengths, np.int32), pt,
                                 WL.num_kv_heads, rope=rope, code_bits=code_bits)
    ref = _dense_extend(mode, bdr, rotate_v, pools, q, q_indptr, lengths, pt, rope=rope, code_bits=code_bits)
    return got, ref, skipped, pools, pt, q, q_indptr


@pytest.mark.parametrize("mode,bdr,rotate_v,code_bits", [
    (oracle.MODE_INT4_BDR, 128, False, 4),
    (oracle.MODE_INT4_BDR, 32, True, 4),
    (oracle.MODE_INT4, 0, False, 4),
    (oracle.MODE_BF16, 0, False, 4),
    (oracle.MODE_INT4_BDR, 64, True, 2),
])
def test_extend_is_dense_causal_attention(mode, bdr, rotate_v, code_bits):
    got, ref, skipped, *_ = _run(mode, bdr, rotate_v, [37, 70, 9], [5, 70, 1], seed=3, code_bits=code_bits)
    assert skipped == 0
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_extend_with_rotary_table_is_dense_causal_attention():
    tab = synth.rope_table(256).numpy()
    got, ref, skipped, *_ = _run(oracle.MODE_INT4_BDR, 128, False, [40, 19], [12, 19], seed=4, rope=tab)
    assert skipped == 0
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_one_query_per_sequence_is_decode():
    lengths = [33, 1, 64]
    pools, pt = _case(oracle.MODE_INT4_BDR, 128, True, lengths, seed=5)
    q = _queries(3, 6)
    ext, _ = oracle.extend(oracle.MODE_INT4_BDR, 128, True, *pools, q, np.array([0, 1, 2, 3], np.int32),
                           np.asarray(lengths, np.int32), pt, WL.num_kv_heads)
    dec, _ = oracle.decode(oracle.MODE_INT4_BDR, 128, True, *pools, q, np.asarray(lengths, np.int32), pt,
                           WL.num_kv_heads)
    assert np.array_equal(ext, dec)


def test_query_ignores_tokens_after_its_position():
    """Rewriting the cache after position p changes no output row of a query at or before p."""
    lengths = [50]
    pools, pt = _case(oracle.MODE_INT4_BDR, 64, False, lengths, seed=7)
    q = _queries(20, 8)
    qi = np.array([0, 20], np.int32)
    sl = np.asarray(lengths, np.int32)
    before, _ = oracle.extend(oracle.MODE_INT4_BDR, 64, False, *pools, q, qi, sl, pt, WL.num_kv_heads)
    kp, vp, ks, vs = (x.copy() for x in pools)
    p_cut = 41  # queries 0..20 sit at positions 30..49; rewrite tokens 42..49
    H, ps = WL.num_kv_heads, WL.page_size
    for t in range(p_cut + 1, 50):
        for h in range(H):
            r = (int(pt[0, t // ps]) * H + h) * ps + t % ps
            kp.reshape(-1, 64)[r] ^= 0x5A
            vp.reshape(-1, 64)[r] ^= 0xA5
    after, _ = oracle.extend(oracle.MODE_INT4_BDR, 64, False, kp, vp, ks, vs, q, qi, sl, pt, WL.num_kv_heads)
    pos = 30 + np.arange(20)
    keep = pos <= p_cut
    assert np.array_equal(before[keep], after[keep])
    assert np.all(np.max(np.abs(before[~keep] - after[~keep]), axis=(1, 2)) > 0)


def test_two_chunks_equal_one_call():
    """Chunked prefill: the last 24 tokens as one extend call, or as 10 then 14 (the first call
    seeing the sequence 14 tokens shorter), give the same rows."""
    lengths = [61]
    pools, pt = _case(oracle.MODE_INT4_BDR, 128, True, lengths, seed=9)
    q = _queries(24, 10)
    args = (oracle.MODE_INT4_BDR, 128, True, *pools)
    one, _ = oracle.extend(*args, q, np.array([0, 24], np.int32), np.array([61], np.int32), pt, WL.num_kv_heads)
    a, _ = oracle.extend(*args, q[:10], np.array([0, 10], np.int32), np.array([47], np.int32), pt, WL.num_kv_heads)
    b, _ = oracle.extend(*args, q[10:], np.array([0, 14], np.int32), np.array([61], np.int32), pt, WL.num_kv_heads)
    assert np.array_equal(one, np.concatenate([a, b]))


def test_queries_before_position_zero_are_zero_rows():
    """More new queries than cached tokens: the first n_s - seq_len rows have no tokens."""
    lengths = [6]
    pools, pt = _case(oracle.MODE_INT4, 0, False, lengths, seed=11)
    q = _queries(9, 12)
    out, _ = oracle.extend(oracle.MODE_INT4, 0, False, *pools, q, np.array([0, 9], np.int32),
                           np.array([6], np.int32), pt, WL.num_kv_heads)
    assert not np.any(out[:3])
    assert np.all(np.max(np.abs(out[3:]), axis=-1) > 0)
    seq_of, lens = oracle.extend_lengths([0, 9], [6])
    assert list(lens) == [-2, -1, 0, 1, 2, 3, 4, 5, 6]


def test_first_query_of_a_fresh_sequence_copies_its_value_row():
    """Position 0 attends to token 0 alone: the output is that token's dequantised value."""
    lengths = [16]
    pools, pt = _case(oracle.MODE_INT4, 0, False, lengths, seed=13)
    q = _queries(16, 14)
    out, _ = oracle.extend(oracle.MODE_INT4, 0, False, *pools, q, np.array([0, 16], np.int32),
                           np.array([16], np.int32), pt, WL.num_kv_heads)
    H, ps = WL.num_kv_heads, WL.page_size
    for h in range(H):
        r = (int(pt[0, 0]) * H + h) * ps
        v0 = _dequant(oracle.MODE_INT4, pools[1], pools[3], np.array([r]), 4)[0]
        for g in range(WL.num_q_heads // H):
            assert np.allclose(out[0, h * 4 + g], v0, rtol=0, atol=1e-12 * np.max(np.abs(v0)))
