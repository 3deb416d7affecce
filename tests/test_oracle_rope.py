"""Pins of the oracle's fused rotary embedding (rotate-half pairs (i, i + 64), a caller-given
(cos, sin) table; keys turned before the block rotation, the query at position seq_len - 1).
The pages keep RoPE outside the cache write; fusing it is the next step the blog's
"no separate kernel" principle (section 3) points to.  CPU only."""
import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle
from bit_paged_kv_append_b200 import synth

D = 128


def bf16_bits(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def test_rope_identity_table_changes_nothing():
    x = np.random.default_rng(0).standard_normal((4, D)).astype(np.float32)
    cs = np.zeros((D // 2, 2), np.float32)
    cs[:, 0] = 1.0
    assert np.array_equal(oracle.rope_f32(x, cs), x)


def test_rope_sign_convention_closed_form():
    """e_0 turns to (cos t) e_0 + (sin t) e_64; e_64 to -(sin t) e_0 + (cos t) e_64."""
    t = 0.7
    cs = np.zeros((D // 2, 2), np.float32)
    cs[:, 0] = 1.0
    cs[0] = (np.float32(np.cos(t)), np.float32(np.sin(t)))
    e0 = np.zeros((1, D), np.float32)
    e0[0, 0] = 1.0
    e64 = np.zeros((1, D), np.float32)
    e64[0, 64] = 1.0
    a, b = oracle.rope_f32(e0, cs)[0], oracle.rope_f32(e64, cs)[0]
    assert a[0] == cs[0, 0] and a[64] == cs[0, 1] and np.count_nonzero(a) == 2
    assert b[0] == -cs[0, 1] and b[64] == cs[0, 0] and np.count_nonzero(b) == 2


def test_rope_is_the_float64_rotation_to_fp32_rounding():
    tab = synth.rope_table(1000).numpy()
    x = np.random.default_rng(1).standard_normal((6, D)).astype(np.float32) * 3
    for pos in (0, 1, 17, 999):
        got = oracle.rope_f32(x, tab[pos]).astype(np.float64)
        c, s = tab[pos, :, 0].astype(np.float64), tab[pos, :, 1].astype(np.float64)
        a, b = x[:, :64].astype(np.float64), x[:, 64:].astype(np.float64)
        ref = np.concatenate([a * c - b * s, b * c + a * s], axis=1)
        assert np.max(np.abs(got - ref)) <= 4e-7 * np.max(np.abs(x))


def test_rope_keeps_norms_and_scores_depend_on_relative_position():
    tab = synth.rope_table(4096).numpy()
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, D)).astype(np.float32)
    k = rng.standard_normal((1, D)).astype(np.float32)
    qm = oracle.rope_f32(q, tab[100])[0].astype(np.float64)
    assert abs(np.linalg.norm(qm) - np.linalg.norm(q)) < 1e-5 * np.linalg.norm(q)
    for m, n, d in ((100, 40, 7), (2000, 1990, 1000), (5, 5, 3000)):
        s1 = oracle.rope_f32(q, tab[m])[0].astype(np.float64) @ oracle.rope_f32(k, tab[n])[0].astype(np.float64)
        s2 = oracle.rope_f32(q, tab[m + d])[0].astype(np.float64) @ oracle.rope_f32(k, tab[n + d])[0].astype(np.float64)
        assert abs(s1 - s2) < 2e-4 * np.linalg.norm(q) * np.linalg.norm(k), (m, n, d)


def _pools(P, H, ps, mode):
    if mode == 0:
        kp = np.zeros((P, H, ps, D), np.uint16)
        return kp, kp.copy(), np.zeros(1, np.uint16), np.zeros(1, np.uint16)
    kp = np.zeros((P, H, ps, D // 2), np.uint8)
    ks = np.zeros((P, H, ps, 2), np.uint16)
    return kp, kp.copy(), ks, ks.copy()


def test_append_with_identity_table_equals_plain_append():
    wl = synth.WORKLOADS["single256"]
    k, v = synth.make_kv(40, wl, 3)
    pt, P = synth.make_page_table([40], 16, 3)
    ts, tp = synth.append_positions([40])
    ident = np.zeros((64, D // 2, 2), np.float32)
    ident[..., 0] = 1.0
    for mode, b in ((1, 0), (2, 128), (0, 0)):
        a = _pools(P, 8, 16, mode)
        c = _pools(P, 8, 16, mode)
        kb, vb = bf16_bits(k.float()), bf16_bits(v.float())
        oracle.append(mode, b, False, *a, kb, vb, ts.numpy(), tp.numpy(), pt.numpy())
        oracle.append(mode, b, False, *c, kb, vb, ts.numpy(), tp.numpy(), pt.numpy(), rope=ident)
        for x, y in zip(a, c):
            assert np.array_equal(x, y)


def test_append_rope_turns_keys_only_and_skips_positions_outside_the_table():
    wl = synth.WORKLOADS["single256"]
    n = 30
    k, v = synth.make_kv(n, wl, 4)
    pt, P = synth.make_page_table([n], 16, 4)
    ts, tp = synth.append_positions([n])
    tab = synth.rope_table(24).numpy()  # positions 24..29 are outside the table
    kb, vb = bf16_bits(k.float()), bf16_bits(v.float())
    kp, vp, ks, vs = _pools(P, 8, 16, 1)
    skipped = oracle.append(1, 0, False, kp, vp, ks, vs, kb, vb, ts.numpy(), tp.numpy(), pt.numpy(), rope=tab)
    assert skipped == 6
    for t in range(n):
        page, slot = pt.numpy()[0, t // 16], t % 16
        if t >= 24:
            assert not kp[page, :, slot].any() and not vp[page, :, slot].any()
            continue
        yk = oracle.rope_f32(bits_to_f32(kb[t]), tab[t])  # [H, D]
        for h in range(8):
            c1, s1 = oracle.quant_row(yk[h])
            assert np.array_equal(kp[page, h, slot], c1) and np.array_equal(ks[page, h, slot], s1)
            c2, s2 = oracle.quant_row(bits_to_f32(vb[t, h]))
            assert np.array_equal(vp[page, h, slot], c2) and np.array_equal(vs[page, h, slot], s2)


def test_bf16_pages_store_the_turned_row_rounded_to_nearest_even():
    wl = synth.WORKLOADS["single256"]
    k, v = synth.make_kv(16, wl, 5)
    pt, P = synth.make_page_table([16], 16, 5)
    ts, tp = synth.append_positions([16])
    tab = synth.rope_table(16).numpy()
    kb, vb = bf16_bits(k.float()), bf16_bits(v.float())
    kp, vp, ks, vs = _pools(P, 8, 16, 0)
    oracle.append(0, 0, False, kp, vp, ks, vs, kb, vb, ts.numpy(), tp.numpy(), pt.numpy(), rope=tab)
    for t in (0, 5, 15):
        page, slot = pt.numpy()[0, 0], t
        y = oracle.rope_f32(bits_to_f32(kb[t]), tab[t])
        u = y.view(np.uint32).astype(np.uint64)
        rn = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)  # round to nearest even
        assert np.array_equal(kp[page, :, slot], rn)
        assert np.array_equal(vp[page, :, slot], vb[t])


def test_decode_rope_brute_force_and_out_of_table_query():
    wl = synth.WORKLOADS["single256"]
    lengths = [37, 20]
    k, v = synth.make_kv(sum(lengths), wl, 6)
    pt, P = synth.make_page_table(lengths, 16, 6)
    ts, tp = synth.append_positions(lengths)
    tab = synth.rope_table(64).numpy()
    kb, vb = bf16_bits(k.float()), bf16_bits(v.float())
    kp, vp, ks, vs = _pools(P, 8, 16, 2)
    oracle.append(2, 128, False, kp, vp, ks, vs, kb, vb, ts.numpy(), tp.numpy(), pt.numpy(), rope=tab)
    q = synth.make_q(2, 32, D, 7)
    qb = q.view(torch.int16).numpy().view(np.uint16)
    out, sk = oracle.decode(2, 128, False, kp, vp, ks, vs, qb, np.array(lengths), pt.numpy(), 8, rope=tab)
    assert sk == 0
    from scipy.linalg import hadamard
    Hm = hadamard(128) / np.sqrt(128)
    f16 = lambda u: u.view(np.float16).astype(np.float64)
    for s, L in enumerate(lengths):
        c, sn = tab[L - 1, :, 0].astype(np.float64), tab[L - 1, :, 1].astype(np.float64)
        for j in (0, 13, 31):
            x = bits_to_f32(qb[s, j]).astype(np.float64)
            xr = np.concatenate([x[:64] * c - x[64:] * sn, x[64:] * c + x[:64] * sn]) @ Hm
            h = j // 4
            rowsK, rowsV = [], []
            for t in range(L):
                page, slot = pt.numpy()[s, t // 16], t % 16
                for pool, sz, acc in ((kp, ks, rowsK), (vp, vs, rowsV)):
                    codes = oracle.unpack_codes(pool[page, h, slot][None])[0].astype(np.float64)
                    acc.append(codes * f16(sz[page, h, slot, 0]) + f16(sz[page, h, slot, 1]))
            p = softmax(np.array(rowsK) @ xr / np.sqrt(128.0))
            assert np.allclose(out[s, j], p @ np.array(rowsV), rtol=1e-9, atol=1e-12)
    # a query position outside the table: the sequence is skipped (zeros)
    out2, sk2 = oracle.decode(2, 128, False, kp, vp, ks, vs, qb, np.array(lengths), pt.numpy(), 8,
                              rope=tab[:30])
    assert sk2 == 32 * 37 and not out2[0].any() and np.array_equal(out2[1], out[1])  # counted per query-head row
