"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests retypes the oracle's code: each checks it against a closed
form (Sylvester's Hadamard matrix), an invariant (orthonormality, q.k
invariance, permutation invariance of the page table), a hand-derived worked
example (tests/golden/quant_levels.txt), an error bound, a library routine
(numpy's fp16 conversion, scipy's softmax) or a special case that reduces to a
known answer.  Sources: the SAW-INT4 abstract (token-wise INT4 + block-diagonal
Hadamard rotation, paged layout) and the wispaper.ai blog, sections 2-3
(blocks of 16..128; K~ = quant(K H_blk); query rotated in step).
"""
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from bit_paged_kv_append_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BLOCKS = [2, 4, 8, 16, 32, 64, 128]


# ---------------------------------------------------------------- helpers ---

def sylvester(b):
    """Closed form H[i][j] = (-1)^popcount(i & j), as int64."""
    i = np.arange(b)[:, None]
    j = np.arange(b)[None, :]
    x = i & j
    pc = np.zeros_like(x)
    while x.any():
        pc += x & 1
        x >>= 1
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


def blockdiag(D, b):
    H = np.zeros((D, D), dtype=np.int64)
    for s in range(0, D, b):
        H[s:s + b, s:s + b] = sylvester(b)
    return H


def bf16_bits(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


def bits_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def dequant(codes, sz):
    c = oracle.unpack_codes(codes).astype(np.float64)
    return c * f16(sz[..., 0])[..., None] + f16(sz[..., 1])[..., None]


# ------------------------------------------------------------- rotation -----

@pytest.mark.parametrize("b", BLOCKS)
def test_fwht_equals_sylvester_on_integers(b):
    """Unnormalised fp32 FWHT on small integers is exact and must equal H_blk x."""
    rng = np.random.default_rng(b)
    x = rng.integers(-8, 9, size=(5, 128)).astype(np.float32)
    got = oracle.rotate_f32(x, b, normalise=False)
    want = (x.astype(np.int64) @ blockdiag(128, b)).astype(np.float32)  # H symmetric: x H = H x
    assert np.array_equal(got, want)


@pytest.mark.parametrize("b", BLOCKS)
def test_fwht_normalisation(b):
    """Normalised result = the exact integer transform times fl32(1/sqrt(b)), one rounding."""
    rng = np.random.default_rng(100 + b)
    x = rng.integers(-8, 9, size=(3, 128)).astype(np.float32)
    got = oracle.rotate_f32(x, b)
    exact = (x.astype(np.int64) @ blockdiag(128, b)).astype(np.float64) / np.sqrt(b)
    # one fp32 rounding of an exactly-representable integer times fl32(1/sqrt b)
    assert np.all(np.abs(got - exact) <= np.abs(exact) * 2.0 ** -22 + 1e-30)
    if b in (4, 16, 64):  # 1/sqrt(b) is a power of two: exact
        assert np.array_equal(got.astype(np.float64), exact)


@pytest.mark.parametrize("b", BLOCKS)
def test_rotate_f64_is_normalised_sylvester(b):
    """Rotating the identity gives H_blk / sqrt(b); it is orthonormal and self-inverse."""
    D = 128
    M = oracle.rotate_f64(np.eye(D), b)
    Hn = blockdiag(D, b) / np.sqrt(b)
    assert np.max(np.abs(M - Hn)) < 1e-15
    assert np.max(np.abs(M @ M.T - np.eye(D))) < 1e-14
    assert np.max(np.abs(M @ M - np.eye(D))) < 1e-14


@pytest.mark.parametrize("b", BLOCKS)
def test_rotate_roundtrip_f32(b):
    rng = np.random.default_rng(7 + b)
    x = (rng.standard_normal((64, 128)) * np.where(rng.random(128) < 0.03, 20, 1)).astype(np.float32)
    back = oracle.rotate_f32(oracle.rotate_f32(x, b), b)
    assert np.max(np.abs(back - x)) <= 1e-6 * np.max(np.abs(x))


@pytest.mark.parametrize("b", BLOCKS)
def test_qk_invariance_f64(b):
    """(q H)(k H)^T = q k^T: the query rotated in step preserves the dot product."""
    rng = np.random.default_rng(11 + b)
    q = rng.standard_normal((16, 128))
    k = rng.standard_normal((16, 128)) * 10
    lhs = oracle.rotate_f64(q, b) @ oracle.rotate_f64(k, b).T
    rhs = q @ k.T
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))


def test_rotation_spreads_outlier_energy():
    """A single outlier channel is spread over its whole block with equal magnitude."""
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 5] = 20.0
    y = oracle.rotate_f32(x, 128)
    assert np.allclose(np.abs(y), 20.0 / np.sqrt(128), rtol=1e-6)


# ------------------------------------------------------------ fp16 ----------

def test_f32_to_f16_matches_numpy():
    """Round-to-nearest-even binary16 against numpy's conversion, over every upper-16-bit
    pattern (all signs, exponents and top mantissa bits) crossed with the low-bit patterns
    that decide rounding, plus random bit patterns."""
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x0FFF, 0x1000, 0x1001, 0x1FFF, 0x2000, 0x3000, 0x7FFF, 0x8000, 0x8001, 0xFFFF,
                     0xEFFF, 0xF000, 0xF001, 0x0800, 0x17FF, 0x1800], dtype=np.uint32)
    bits = (hi[:, None] | lows[None, :]).ravel()
    rng = np.random.default_rng(0)
    bits = np.concatenate([bits, rng.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)])
    x = bits.view(np.float32)
    got = oracle.f32_to_f16_bits(x)
    with np.errstate(over="ignore", invalid="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.all(np.isnan(got[nan].view(np.float16)))


# -------------------------------------------------------- quantiser ---------

def _golden():
    out = {}
    with open(os.path.join(GOLDEN, "quant_levels.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, val = line.split(None, 1)
            out[key] = val.split()
    return out


def _row_d():
    y = np.zeros(128)
    y[0], y[1], y[2] = -9.375, 28.125, 1.875
    return y


def _row_e():
    y = np.zeros(128)
    y[1], y[2], y[3], y[4] = 1.5, 15934463 / 2 ** 24, 7371 / 2 ** 14, 23751 / 2 ** 14
    return y


def _worked_row(row):
    i = np.arange(128)
    return {"A": 0.5 * (i % 16), "B": -3 + 0.25 * (i % 16), "C": np.full(128, 1.75), "D": _row_d(),
            "E": _row_e()}[row].astype(np.float32)


@pytest.mark.parametrize("row", ["A", "B", "C", "D", "E"])
def test_quant_worked_examples(row):
    g = _golden()
    codes, sz = oracle.quant_row(_worked_row(row))
    assert sz[0] == int(g[f"{row}.scale"][0], 16)
    assert sz[1] == int(g[f"{row}.zero"][0], 16)
    want = bytes.fromhex("".join(g[f"{row}.bytes"]))
    assert codes.tobytes() == want


# The rounding step of the oracle's quantiser, as written in kvq_oracle.c, and the two
# other readings of "round to nearest" that the worked rows D and E tell apart: the
# product rounded to fp32 before the rounding to an integer, and the exact quotient.
_R4_LINE = "double v = (double)t * (double)inv;"
_R4_MUTANTS = {"fp32_product": "double v = (double)(float)(t * inv);",
               "exact_quotient": "double v = (scale > 0.0f) ? (double)t / (double)scale : 0.0;"}


def _mutant_quant_row(tmp_path, name):
    """oracle_quant_row from a copy of the oracle whose rounding step is replaced by another
    reading (a planted mistake, built and run on the CPU only)."""
    import ctypes
    import subprocess

    src = open(os.path.join(ROOT, "oracle", "kvq_oracle.c")).read()
    assert src.count(_R4_LINE) == 1, "the oracle's rounding step moved; update the mutants"
    path = tmp_path / f"oracle_{name}.c"
    path.write_text(src.replace(_R4_LINE, _R4_MUTANTS[name]))
    lib_path = tmp_path / f"liboracle_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=gnu11", "-shared", "-fPIC",
                           "-o", str(lib_path), str(path), "-lm"])
    lib = ctypes.CDLL(str(lib_path))
    P = ctypes.c_void_p
    lib.oracle_quant_row.argtypes = [P, ctypes.c_int, P, P]

    def quant_row(y):
        y = np.ascontiguousarray(y, dtype=np.float32)
        codes = np.zeros(64, np.uint8)
        sz = np.zeros(2, np.uint16)
        lib.oracle_quant_row(y.ctypes.data_as(P), 128, codes.ctypes.data_as(P), sz.ctypes.data_as(P))
        return codes, sz

    return quant_row


@pytest.mark.parametrize("name", sorted(_R4_MUTANTS))
def test_worked_rows_reject_the_other_rounding_readings(tmp_path, name):
    """Rows D and E pin the rounding reading: an oracle built with either other reading
    computes different bytes for both rows (and row E's bytes are the ones derived by hand
    for that reading in the golden file)."""
    g = _golden()
    quant_row = _mutant_quant_row(tmp_path, name)
    for row in ("D", "E"):
        codes, sz = quant_row(_worked_row(row))
        assert sz[0] == int(g[f"{row}.scale"][0], 16) and sz[1] == int(g[f"{row}.zero"][0], 16)
        assert codes.tobytes() != bytes.fromhex("".join(g[f"{row}.bytes"])), row
    codes, _ = quant_row(_worked_row("E"))
    key = {"fp32_product": "E.bytes_if_fp32_product", "exact_quotient": "E.bytes_if_exact_quotient"}[name]
    assert codes.tobytes() == bytes.fromhex("".join(g[key]))


def test_pack_unpack_all_byte_values():
    """Every (even, odd) code pair lands in the byte as even | odd << 4 and unpacks back."""
    pairs = [(a, b) for b in range(16) for a in range(16)]  # 256 pairs, 64 per row
    for r in range(4):
        chunk = pairs[64 * r: 64 * (r + 1)]
        y = np.array([v for p in chunk for v in p], dtype=np.float32) * 0.5  # levels 0..15, scale 0.5
        codes, sz = oracle.quant_row(y)
        assert sz[0] == 0x3800 and sz[1] == 0
        assert list(codes) == [a | (b << 4) for a, b in chunk]
        assert np.array_equal(oracle.unpack_codes(codes), (y / 0.5).astype(np.uint8))


@pytest.mark.parametrize("mag", [1e-3, 1.0, 30.0, 500.0])
def test_quant_error_bound_and_monotone(mag):
    """|x^ - y| <= scale/2 + 15|range/15 - scale| + |min - zero| (+ fp32 rounding); codes in
    0..15 and non-decreasing in y."""
    rng = np.random.default_rng(int(mag * 1000) + 3)
    for _ in range(200):
        y = (rng.standard_normal(128) * mag * np.where(rng.random(128) < 0.05, 20, 1)).astype(np.float32)
        codes, sz = oracle.quant_row(y)
        c = oracle.unpack_codes(codes)
        assert c.max() <= 15
        xh = dequant(codes[None], sz[None])[0]
        mn, mx = float(y.min()), float(y.max())
        scale, zero = f16(sz[0]), f16(sz[1])
        bound = scale / 2 + 15 * abs((mx - mn) / 15 - scale) + abs(mn - zero) + 1e-6 * max(abs(mn), abs(mx))
        assert np.max(np.abs(xh - y)) <= bound
        order = np.argsort(y, kind="stable")
        assert np.all(np.diff(c[order].astype(int)) >= 0)


def test_quant_cross_check_exact_product_on_random_rows():
    """Cross-check, not a pin: it restates the oracle's rounding step (rint, ties to even, of
    the exact product fl(y - zero) * fl(1/scale)) with rational arithmetic on random rows, so
    it only confirms that the C code computes what it says.  The pins of that step are the
    hand-derived rows D and E above."""
    from fractions import Fraction

    rng = np.random.default_rng(17)
    for _ in range(50):
        y = (rng.standard_normal(128) * rng.choice([0.01, 1.0, 40.0])).astype(np.float32)
        codes, sz = oracle.quant_row(y)
        c = oracle.unpack_codes(codes)
        scale = np.uint16(sz[0]).view(np.float16).astype(np.float32)
        zero = np.uint16(sz[1]).view(np.float16).astype(np.float32)
        inv = np.float32(1) / scale if scale > 0 else np.float32(0)
        for e in range(128):
            q = Fraction(float(np.float32(y[e]) - zero)) * Fraction(float(inv))
            r = round(q)  # Fraction rounding: nearest, ties to even
            assert c[e] == (0 if r <= 0 else min(15, r))


def test_quant_signed_zero_row_is_canonical():
    y = np.full(128, -0.0, dtype=np.float32)
    codes, sz = oracle.quant_row(y)
    assert sz[0] == 0 and sz[1] == 0 and not codes.any()


@pytest.mark.parametrize("where", [0, 77, 127])
def test_quant_nan_row_is_all_zero_codes_with_nan_scale(where):
    """A NaN anywhere in the row (reading: min and max are then NaN): every code 0, scale
    and zero the fp16 quiet NaN 0x7E00; the position of the NaN does not matter."""
    y = np.linspace(-2, 3, 128).astype(np.float32)
    y[where] = np.nan
    codes, sz = oracle.quant_row(y)
    assert not codes.any() and sz[0] == 0x7E00 and sz[1] == 0x7E00


def test_quant_rows_matches_rotate_then_quant():
    """quant_rows(x, b) == quant_row(rotate_f32(x)) row by row; b = 0 means no rotation."""
    rng = np.random.default_rng(5)
    x = bf16_bits(rng.standard_normal((6, 128)) * 3)
    for b in (0, 16, 128):
        codes, sz = oracle.quant_rows(x, b)
        for r in range(6):
            y = bits_to_f32(x[r])
            if b:
                y = oracle.rotate_f32(y[None], b)[0]
            c1, s1 = oracle.quant_row(y)
            assert np.array_equal(codes[r], c1) and np.array_equal(sz[r], s1)


def test_bdr_reduces_error_on_outliers():
    """The method's premise (blog section 2): rotation spreads outlier energy, so the
    dequantisation error of rotated INT4 is far below naive INT4 on outlier data."""
    wl = synth.WORKLOADS["single256"]
    k, _ = synth.make_kv(256, wl, seed=0)
    kb = k.view(torch.int16).numpy().view(np.uint16)
    x = bits_to_f32(kb).astype(np.float64)
    c0, s0 = oracle.quant_rows(kb, 0)
    err_naive = np.mean((dequant(c0, s0) - x) ** 2)
    c1, s1 = oracle.quant_rows(kb, 128)
    xr = oracle.rotate_f64(x, 128)
    err_bdr = np.mean((dequant(c1, s1) - xr) ** 2)  # orthonormal: same error in the original space
    assert err_bdr < 0.25 * err_naive


# ------------------------------------------------------------ append --------

def _setup_cache(num_pages, H, ps, D, mode, fill=0xA5):
    if mode == oracle.MODE_BF16:
        kp = np.full((num_pages, H, ps, D), fill * 257, dtype=np.uint16)
        vp = kp.copy()
        ks = vs = np.zeros((1,), dtype=np.uint16)
    else:
        kp = np.full((num_pages, H, ps, D // 2), fill, dtype=np.uint8)
        vp = kp.copy()
        ks = np.full((num_pages, H, ps, 2), fill * 257, dtype=np.uint16)
        vs = ks.copy()
    return kp, vp, ks, vs


def _append_case(mode, b, rotate_v, lengths, ps=4, H=2, D=128, seed=0, spare=2):
    wl = synth.Workload("t", H, 2 * H, D, ps, synth.OUTLIERS_X20, "test")
    T = sum(lengths)
    k, v = synth.make_kv(T, wl, seed)
    kb = k.view(torch.int16).numpy().view(np.uint16)
    vb = v.view(torch.int16).numpy().view(np.uint16)
    pt, P = synth.make_page_table(lengths, ps, seed, spare_pages=spare)
    ts, tp = synth.append_positions(lengths)
    kp, vp, ks, vs = _setup_cache(P, H, ps, D, mode)
    skipped = oracle.append(mode, b, rotate_v, kp, vp, ks, vs, kb, vb, ts.numpy(), tp.numpy(), pt.numpy())
    return dict(kb=kb, vb=vb, pt=pt.numpy(), ts=ts.numpy(), tp=tp.numpy(), kp=kp, vp=vp, ks=ks, vs=vs,
                skipped=skipped, P=P, H=H, ps=ps)


@pytest.mark.parametrize("mode,b,rv", [(oracle.MODE_INT4, 0, False), (oracle.MODE_INT4_BDR, 16, False),
                                       (oracle.MODE_INT4_BDR, 128, True)])
def test_append_places_rows_through_page_table(mode, b, rv):
    c = _append_case(mode, b, rv, [7, 1, 10])
    assert c["skipped"] == 0
    touched = np.zeros(c["kp"].shape[:3], dtype=bool)
    for i, (s, p) in enumerate(zip(c["ts"], c["tp"])):
        page, slot = c["pt"][s, p // c["ps"]], p % c["ps"]
        touched[page, :, slot] = True
        bk = b if mode == oracle.MODE_INT4_BDR else 0
        bv = b if (mode == oracle.MODE_INT4_BDR and rv) else 0
        ck, sk = oracle.quant_rows(c["kb"][i], bk)
        cv, sv = oracle.quant_rows(c["vb"][i], bv)
        assert np.array_equal(c["kp"][page, :, slot], ck) and np.array_equal(c["ks"][page, :, slot], sk)
        assert np.array_equal(c["vp"][page, :, slot], cv) and np.array_equal(c["vs"][page, :, slot], sv)
    assert np.all(c["kp"][~touched] == 0xA5) and np.all(c["ks"][~touched] == 0xA5A5)


def test_append_bf16_copies_bits():
    c = _append_case(oracle.MODE_BF16, 0, False, [5, 9])
    for i, (s, p) in enumerate(zip(c["ts"], c["tp"])):
        page, slot = c["pt"][s, p // c["ps"]], p % c["ps"]
        assert np.array_equal(c["kp"][page, :, slot], c["kb"][i])
        assert np.array_equal(c["vp"][page, :, slot], c["vb"][i])


def test_append_skips_out_of_range():
    H, ps, D = 2, 4, 128
    kp, vp, ks, vs = _setup_cache(3, H, ps, D, oracle.MODE_INT4)
    pt = np.array([[0, 7], [2, -1]], dtype=np.int32)  # page 7 and -1 are outside the 3-page pool
    kb = bf16_bits(np.ones((5, H, D)))
    ts = np.array([0, 0, 1, 5, 1], dtype=np.int32)  # seq 5 does not exist
    tp = np.array([1, 4, 4, 0, -1], dtype=np.int32)  # pos 4 of seq 0 -> page 7; pos 4 of seq 1 -> -1
    n = oracle.append(oracle.MODE_INT4, 0, False, kp, vp, ks, vs, kb, kb, ts, tp, pt)
    assert n == 4
    assert not np.all(kp[0, :, 1] == 0xA5)  # the one valid token was written
    kp[0, :, 1] = 0xA5
    assert np.all(kp == 0xA5)


# ------------------------------------------------------------ decode --------

def _np_attention(q, K, V):
    """Softmax attention of one query row over rows of K, V, with scipy's softmax."""
    z = K @ q / np.sqrt(q.shape[0])
    return scipy.special.softmax(z) @ V


def _dequant_seq(c, which, s, h, L, mode):
    pool, sz = (c["kp"], c["ks"]) if which == "k" else (c["vp"], c["vs"])
    rows = []
    for t in range(L):
        page, slot = c["pt"][s, t // c["ps"]], t % c["ps"]
        if mode == oracle.MODE_BF16:
            rows.append(bits_to_f32(pool[page, h, slot]).astype(np.float64))
        else:
            rows.append(dequant(pool[page, h, slot][None], sz[page, h, slot][None])[0])
    return np.array(rows)


@pytest.mark.parametrize("mode,b,rv", [(oracle.MODE_BF16, 0, False), (oracle.MODE_INT4, 0, False),
                                       (oracle.MODE_INT4_BDR, 32, False), (oracle.MODE_INT4_BDR, 128, True)])
def test_decode_brute_force(mode, b, rv):
    """Against scipy-softmax attention over the dequantised cache, with the query rotated
    by the explicit normalised block-diagonal Sylvester matrix and, for rotated V, the
    output rotated back by the same matrix."""
    lengths = [7, 1, 10]
    c = _append_case(mode, b, rv, lengths)
    H, Hq, D = c["H"], 2 * c["H"], 128
    q = synth.make_q(len(lengths), Hq, D, seed=3)
    qb = q.view(torch.int16).numpy().view(np.uint16)
    out, skipped = oracle.decode(mode, b, rv, c["kp"], c["vp"], c["ks"], c["vs"], qb, np.array(lengths),
                                 c["pt"], H)
    assert skipped == 0
    Hn = blockdiag(D, b) / np.sqrt(b) if b else np.eye(D)
    for s, L in enumerate(lengths):
        for j in range(Hq):
            h = j // (Hq // H)
            qq = bits_to_f32(qb[s, j]).astype(np.float64)
            if mode == oracle.MODE_INT4_BDR:
                qq = qq @ Hn
            o = _np_attention(qq, _dequant_seq(c, "k", s, h, L, mode), _dequant_seq(c, "v", s, h, L, mode))
            if mode == oracle.MODE_INT4_BDR and rv:
                o = o @ Hn
            assert np.max(np.abs(out[s, j] - o)) <= 1e-12 * max(1.0, np.max(np.abs(o)))


def test_decode_special_cases():
    """L = 1 gives v^_0; identical keys give the mean of the values; an empty sequence
    gives zeros; each query head reads its own KV head (group j // G)."""
    H, Hq, D, ps = 2, 4, 128, 4
    kp, vp, ks, vs = _setup_cache(4, H, ps, D, oracle.MODE_BF16)
    pt = np.array([[0, 1], [2, 3], [3, -1]], dtype=np.int32)
    rng = np.random.default_rng(1)
    vals = bf16_bits(rng.standard_normal((4, H, ps, D)))
    vp[:] = vals
    kp[:] = bf16_bits(np.ones((4, H, ps, D)))  # every key identical
    q = bf16_bits(rng.standard_normal((3, Hq, D)))
    out, _ = oracle.decode(oracle.MODE_BF16, 0, False, kp, vp, ks, vs, q, np.array([1, 6, 0]), pt, H)
    v = bits_to_f32(vals).astype(np.float64)
    for j in range(Hq):
        h = j // 2
        assert np.allclose(out[0, j], v[0, h, 0], rtol=0, atol=0)
        mean6 = (v[2, h, 0:4].sum(0) + v[3, h, 0:2].sum(0)) / 6
        assert np.allclose(out[1, j], mean6, rtol=1e-14, atol=1e-14)
        assert not out[2, j].any()


def test_decode_dominant_score_selects_value():
    H, Hq, D, ps = 1, 1, 128, 4
    kp, vp, ks, vs = _setup_cache(2, H, ps, D, oracle.MODE_BF16)
    kp[:] = 0
    kp[1, 0, 2] = bf16_bits(np.full(D, 8.0))  # token 6 (page 1 slot 2) gets a huge score
    vp[:] = bf16_bits(np.arange(2 * ps * D).reshape(2, 1, ps, D) % 7)
    q = bf16_bits(np.full((1, 1, D), 8.0))
    out, _ = oracle.decode(oracle.MODE_BF16, 0, False, kp, vp, ks, vs, q, np.array([8]), np.array([[0, 1]]), H)
    assert np.allclose(out[0, 0], bits_to_f32(vp[1, 0, 2]), atol=1e-12)


def test_decode_page_table_permutation_invariance():
    """The same tokens placed through two different page tables give identical outputs."""
    lengths = [9, 13]
    res = []
    for seed in (0, 1):
        wl = synth.Workload("t", 2, 8, 128, 4, synth.OUTLIERS_X20, "test")
        k, v = synth.make_kv(sum(lengths), wl, 0)
        kb = k.view(torch.int16).numpy().view(np.uint16)
        vb = v.view(torch.int16).numpy().view(np.uint16)
        pt, P = synth.make_page_table(lengths, 4, seed=seed + 10, spare_pages=3)
        ts, tp = synth.append_positions(lengths)
        kp, vp, ks, vs = _setup_cache(P, 2, 4, 128, oracle.MODE_INT4_BDR)
        oracle.append(oracle.MODE_INT4_BDR, 64, True, kp, vp, ks, vs, kb, vb, ts.numpy(), tp.numpy(), pt.numpy())
        q = synth.make_q(2, 8, 128, seed=4).view(torch.int16).numpy().view(np.uint16)
        out, _ = oracle.decode(oracle.MODE_INT4_BDR, 64, True, kp, vp, ks, vs, q, np.array(lengths),
                               pt.numpy(), 2)
        res.append(out)
    assert np.array_equal(res[0], res[1])


def test_decode_rows_subset_matches_full():
    c = _append_case(oracle.MODE_INT4_BDR, 128, False, [5, 11])
    q = synth.make_q(2, 4, 128, seed=9).view(torch.int16).numpy().view(np.uint16)
    full, _ = oracle.decode(oracle.MODE_INT4_BDR, 128, False, c["kp"], c["vp"], c["ks"], c["vs"], q,
                            np.array([5, 11]), c["pt"], 2)
    rows = [(1, 3), (0, 0), (1, 1)]
    sub, _ = oracle.decode(oracle.MODE_INT4_BDR, 128, False, c["kp"], c["vp"], c["ks"], c["vs"], q,
                           np.array([5, 11]), c["pt"], 2, rows=rows)
    for r, (s, j) in enumerate(rows):
        assert np.array_equal(sub[r], full[s, j])


def test_decode_counts_bad_pages():
    H, Hq, D, ps = 1, 1, 128, 4
    kp, vp, ks, vs = _setup_cache(2, H, ps, D, oracle.MODE_INT4)
    pt = np.array([[0, 9]], dtype=np.int32)
    q = bf16_bits(np.ones((1, 1, D)))
    _, skipped = oracle.decode(oracle.MODE_INT4, 0, False, kp, vp, ks, vs, q, np.array([12]), pt, H)
    assert skipped == 4 + 4  # 4 tokens on page 9, 4 beyond the page table
