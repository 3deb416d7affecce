"""Pins of the oracle's 2-bit variant (the pages leave 2-bit open; reading: the same token-wise
asymmetric quantiser with range/3, codes 0..3, four per byte, code k of a byte in bits 2k and
2k + 1).  CPU only."""
import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle
from bit_paged_kv_append_b200 import synth

D = 128


def bf16_bits(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f16(b):
    return np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float64)


def test_int2_worked_row_four_levels():
    """y = (e mod 4) / 2: range 1.5, scale fl(1.5 / 3) = 0.5 exactly (fp16 0x3800), zero 0, codes
    e mod 4, so every byte is 0 | 1 << 2 | 2 << 4 | 3 << 6 = 0xE4."""
    y = (np.arange(D) % 4).astype(np.float32) * 0.5
    codes, sz = oracle.quant_row(y, bits=2)
    assert codes.shape == (32,) and np.all(codes == 0xE4)
    assert sz[0] == 0x3800 and sz[1] == 0


def test_int2_ties_round_to_even():
    """With scale 1 (range 3) and zero 0, quotients 0.5, 1.5, 2.5 round to 0, 2, 2."""
    y = np.zeros(D, np.float32)
    y[1] = 3.0  # max: range 3, scale 1
    y[2], y[3], y[4] = 0.5, 1.5, 2.5
    codes, sz = oracle.quant_row(y, bits=2)
    c = oracle.unpack_codes(codes, bits=2)
    assert f16(sz[0]) == 1.0 and f16(sz[1]) == 0.0
    assert list(c[:5]) == [0, 3, 0, 2, 2]


def test_int2_pack_unpack_all_bytes():
    b = np.arange(256, dtype=np.uint8)
    c = oracle.unpack_codes(b[None], bits=2)[0].reshape(256, 4)
    assert np.array_equal((c[:, 0] | (c[:, 1] << 2) | (c[:, 2] << 4) | (c[:, 3] << 6)).astype(np.uint8), b)


def test_int2_error_bound_and_monotone_codes():
    rng = np.random.default_rng(3)
    for _ in range(50):
        y = (rng.standard_normal(D) * rng.uniform(0.01, 50)).astype(np.float32)
        codes, sz = oracle.quant_row(y, bits=2)
        c = oracle.unpack_codes(codes, bits=2).astype(np.float64)
        scale, zero = f16(sz[0]), f16(sz[1])
        mn, mx = float(y.min()), float(y.max())
        s32 = float(np.float32(np.float32(mx - mn) / np.float32(3.0)))
        bound = scale / 2 + 3 * abs(s32 - scale) + abs(mn - zero) + 4 * np.spacing(np.float32(np.abs(y).max()))
        assert np.all(np.abs(c * scale + zero - y.astype(np.float64)) <= bound)
        order = np.argsort(y, kind="stable")
        assert np.all(np.diff(c[order]) >= 0)
        assert c.min() >= 0 and c.max() <= 3


def test_four_bit_wrapper_unchanged():
    y = np.random.default_rng(4).standard_normal(D).astype(np.float32) * 5
    a = oracle.quant_row(y)
    b = oracle.quant_row(y, bits=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_int2_append_and_decode_brute_force():
    wl = synth.WORKLOADS["single256"]
    lengths = [45, 16]
    k, v = synth.make_kv(sum(lengths), wl, 8)
    pt, P = synth.make_page_table(lengths, 16, 8)
    ts, tp = synth.append_positions(lengths)
    kp = np.zeros((P, 8, 16, 32), np.uint8)
    vp = kp.copy()
    ks = np.zeros((P, 8, 16, 2), np.uint16)
    vs = ks.copy()
    kb, vb = bf16_bits(k.float()), bf16_bits(v.float())
    assert oracle.append(2, 64, True, kp, vp, ks, vs, kb, vb, ts.numpy(), tp.numpy(), pt.numpy(), code_bits=2) == 0
    ck, sk = oracle.quant_rows(kb, 64, bits=2)
    cv, sv = oracle.quant_rows(vb, 64, bits=2)
    ptn = pt.numpy()
    off = 0
    for s, L in enumerate(lengths):
        for t in range(L):
            page, slot = ptn[s, t // 16], t % 16
            assert np.array_equal(kp[page, :, slot], ck[off + t]) and np.array_equal(ks[page, :, slot], sk[off + t])
            assert np.array_equal(vp[page, :, slot], cv[off + t]) and np.array_equal(vs[page, :, slot], sv[off + t])
        off += L
    q = synth.make_q(2, 32, D, 9)
    qb = q.view(torch.int16).numpy().view(np.uint16)
    out, skipped = oracle.decode(2, 64, True, kp, vp, ks, vs, qb, np.array(lengths), ptn, 8, code_bits=2)
    assert skipped == 0
    from scipy.linalg import hadamard
    Hm = np.kron(np.eye(2), hadamard(64) / 8.0)
    for s, L in enumerate(lengths):
        for j in (0, 9, 31):
            h = j // 4
            x = (np.asarray(qb[s, j], np.uint32) << 16).view(np.float32).astype(np.float64) @ Hm
            K, V = [], []
            for t in range(L):
                page, slot = ptn[s, t // 16], t % 16
                for pool, sz, acc in ((kp, ks, K), (vp, vs, V)):
                    c = oracle.unpack_codes(pool[page, h, slot], bits=2).astype(np.float64)
                    acc.append(c * f16(sz[page, h, slot, 0]) + f16(sz[page, h, slot, 1]))
            p = softmax(np.array(K) @ x / np.sqrt(128.0))
            assert np.allclose(out[s, j], (p @ np.array(V)) @ Hm, rtol=1e-9, atol=1e-12)


def test_int2_rotation_lowers_error_on_outliers():
    wl = synth.WORKLOADS["decode64x8k"]
    k, _ = synth.make_kv(64, wl, 10)
    kb = bf16_bits(k.float())
    x = (np.asarray(kb, np.uint32) << 16).view(np.float32).astype(np.float64)  # [T, H, D]
    errs = {}
    for b in (0, 128):
        codes, sz = oracle.quant_rows(kb, b, bits=2)
        xr = x if b == 0 else x @ (np.kron(np.eye(1), __import__("scipy.linalg").linalg.hadamard(128) / np.sqrt(128.0)))
        deq = oracle.unpack_codes(codes, bits=2) * f16(sz[..., :1]) + f16(sz[..., 1:])
        errs[b] = np.sqrt(np.mean((deq - xr) ** 2))
    assert errs[128] < 0.7 * errs[0], errs
