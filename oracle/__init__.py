"""CPU oracle for the SAW-INT4 KV-cache write/read path -- TEST INFRASTRUCTURE.

This package is the plain, slow, obviously-correct restatement that the CUDA
library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; the product path
(``bit_paged_kv_append_b200``) never does, and the two share no code.  The
arithmetic lives in ``kvq_oracle.c`` (plain C, built here with gcc and loaded
through ctypes); this module only marshals numpy arrays.

Every function cites the passage it follows (see ``kvq_oracle.c``):
the paper's abstract (token-wise INT4 with block-diagonal Hadamard rotation,
fused into paged KV-cache layouts) and the wispaper.ai blog's sections 2-3
(blocks of 16..128 along head_dim; K~ = quant(K H_blk), V~ = quant(V H_blk);
query rotated in step at decode).

Parity status: every exported function is pinned by ``tests/test_oracle_pins.py``
(and ``extend`` by ``tests/test_oracle_extend.py``) against closed forms,
invariants, special cases or brute force on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")

MODE_BF16, MODE_INT4, MODE_INT4_BDR = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FP contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=gnu11", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        lib.oracle_version.restype = ctypes.c_int
        lib.oracle_f32_to_f16.argtypes = [P, P, i64]
        lib.oracle_rotate_f32.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.oracle_rotate_f64.argtypes = [P, ctypes.c_int, ctypes.c_int]
        lib.oracle_quant_row.argtypes = [P, ctypes.c_int, P, P]
        lib.oracle_quant_rows.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P, P]
        lib.oracle_quant_row_bits.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P]
        lib.oracle_quant_rows_bits.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        lib.oracle_append.restype = i64
        lib.oracle_append.argtypes = [ctypes.c_int] * 7 + [P] * 6 + [ctypes.c_int, P, P, P, ctypes.c_int,
                                                                     ctypes.c_int, P, ctypes.c_int, ctypes.c_int]
        lib.oracle_decode.restype = i64
        lib.oracle_decode.argtypes = [ctypes.c_int] * 8 + [P] * 7 + [ctypes.c_int, ctypes.c_int, P,
                                                                     ctypes.c_int, P, P, ctypes.c_int, ctypes.c_int]
        lib.oracle_rope_f32.argtypes = [P, ctypes.c_int, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """IEEE binary32 -> binary16 bits, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f32_to_f16(_ptr(x), _ptr(out), x.size)
    return out


def rotate_f32(x: np.ndarray, b: int, normalise: bool = True) -> np.ndarray:
    """Block-diagonal fp32 FWHT of each row of x (last axis = head_dim)."""
    x = np.array(x, dtype=np.float32, order="C", copy=True)
    D = x.shape[-1]
    rows = x.reshape(-1, D)
    lib = _load()
    for r in range(rows.shape[0]):
        lib.oracle_rotate_f32(rows[r].ctypes.data_as(ctypes.c_void_p), D, b, int(normalise))
    return x


def rotate_f64(x: np.ndarray, b: int) -> np.ndarray:
    """Block-diagonal normalised Hadamard rotation of each row, float64."""
    x = np.array(x, dtype=np.float64, order="C", copy=True)
    D = x.shape[-1]
    rows = x.reshape(-1, D)
    lib = _load()
    for r in range(rows.shape[0]):
        lib.oracle_rotate_f64(rows[r].ctypes.data_as(ctypes.c_void_p), D, b)
    return x


def quant_row(y: np.ndarray, bits: int = 4):
    """Token-wise asymmetric INT4 (bits = 4) or INT2 (bits = 2) of one fp32 row -> (packed codes
    uint8[D * bits / 8], (scale, zero) fp16 bits)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    D = y.shape[0]
    codes = np.empty(D * bits // 8, dtype=np.uint8)
    sz = np.empty(2, dtype=np.uint16)
    _load().oracle_quant_row_bits(_ptr(y), D, bits, _ptr(codes), _ptr(sz))
    return codes, sz


def quant_rows(x_bf16_bits: np.ndarray, b: int, bits: int = 4):
    """Rotate (block b; b == 0: none) and quantise bf16 rows [..., D] -> (codes [..., D*bits/8], sz [..., 2])."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    D = x.shape[-1]
    n = x.size // D
    codes = np.empty(x.shape[:-1] + (D * bits // 8,), dtype=np.uint8)
    sz = np.empty(x.shape[:-1] + (2,), dtype=np.uint16)
    _load().oracle_quant_rows_bits(_ptr(x), n, D, b, bits, _ptr(codes), _ptr(sz))
    return codes, sz


def unpack_codes(codes: np.ndarray, bits: int = 4) -> np.ndarray:
    """Packed bytes [..., D*bits/8] -> codes [..., D] (code k of a byte in bits k*bits ..)."""
    per = 8 // bits
    parts = [(codes >> (bits * k)) & ((1 << bits) - 1) for k in range(per)]
    return np.stack(parts, axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * per,))


def _rope_args(rope):
    if rope is None:
        return None, None, 0
    r = np.ascontiguousarray(rope, dtype=np.float32)
    return r, _ptr(r), r.shape[0]


def rope_f32(x: np.ndarray, cs: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE of rows x (float32 [n, D]) with one table row cs (float32 [D/2, 2] = (cos, sin))."""
    x = np.ascontiguousarray(x, dtype=np.float32).copy()
    c = np.ascontiguousarray(cs, dtype=np.float32)
    for r in range(x.shape[0]):
        _load().oracle_rope_f32(_ptr(x[r]), x.shape[1], _ptr(c))
    return x


def append(mode: int, bdr_block: int, rotate_v: bool, k_pool, v_pool, k_sz, v_sz, k_bits, v_bits,
           tok_seq, tok_pos, page_table, rope=None, code_bits: int = 4) -> int:
    """Append tokens into the pools in place (numpy arrays); returns the skipped-token count.

    Pools: INT4 uint8 [P, H, ps, D/2] (+ sz uint16 [P, H, ps, 2]); BF16 uint16 [P, H, ps, D].
    k_bits/v_bits: bf16 bits uint16 [T, H, D]; page_table int32 [num_seqs, pt_stride].
    rope: optional float32 [positions, D/2, 2] (cos, sin) table that turns the keys first.
    """
    P, H, ps = k_pool.shape[:3]
    D = k_bits.shape[-1]
    T = k_bits.shape[0]
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    ts = np.ascontiguousarray(tok_seq, dtype=np.int32)
    tp = np.ascontiguousarray(tok_pos, dtype=np.int32)
    keep, rp, rn = _rope_args(rope)
    return int(_load().oracle_append(mode, bdr_block, int(rotate_v), P, ps, H, D, _ptr(k_pool), _ptr(v_pool),
                                     _ptr(k_sz), _ptr(v_sz), _ptr(np.ascontiguousarray(k_bits)),
                                     _ptr(np.ascontiguousarray(v_bits)), T, _ptr(ts), _ptr(tp), _ptr(pt),
                                     pt.shape[1], pt.shape[0], rp, rn, int(code_bits)))


def decode(mode: int, bdr_block: int, rotate_v: bool, k_pool, v_pool, k_sz, v_sz, q_bits, seq_lens,
           page_table, num_kv_heads: int, rows=None, rope=None, code_bits: int = 4):
    """Paged GQA decode attention in float64.

    q_bits: bf16 bits uint16 [B, Hq, D].  rows: optional int array [(seq, qhead), ...]; when None all
    B*Hq rows are computed.  rope: optional float32 [positions, D/2, 2] table turning q at position
    seq_len - 1.  Returns (out float64 [n, D] or [B, Hq, D], skipped-token count).
    """
    P = k_pool.shape[0]
    ps = k_pool.shape[2]
    B, Hq, D = q_bits.shape
    pt = np.ascontiguousarray(page_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    if rows is not None:
        rws = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 2))
        n = rws.shape[0]
    else:
        rws = None
        n = B * Hq
    out = np.empty((n, D), dtype=np.float64)
    keep, rp, rn = _rope_args(rope)
    skipped = _load().oracle_decode(mode, bdr_block, int(rotate_v), P, ps, num_kv_heads, Hq, D, _ptr(k_pool),
                                    _ptr(v_pool), _ptr(k_sz), _ptr(v_sz), _ptr(np.ascontiguousarray(q_bits)),
                                    _ptr(sl), _ptr(pt), pt.shape[1], B, _ptr(rws), n, _ptr(out), rp, rn,
                                    int(code_bits))
    if rows is None:
        out = out.reshape(B, Hq, D)
    return out, int(skipped)


def extend_lengths(q_indptr, seq_lens) -> tuple[np.ndarray, np.ndarray]:
    """Per query row of an extend call: (its sequence, its decode length = position + 1).

    Query i (0-based) of the n_s = q_indptr[s+1] - q_indptr[s] newest tokens of sequence s
    sits at position seq_lens[s] - n_s + i: the new tokens are the last n_s of the
    sequence, in order."""
    qi = np.asarray(q_indptr, dtype=np.int64)
    n = np.diff(qi)
    seq_of = np.repeat(np.arange(len(n)), n)
    i_in = np.arange(int(qi[-1])) - qi[seq_of]
    lens = np.asarray(seq_lens, dtype=np.int64)[seq_of] - n[seq_of] + i_in + 1
    return seq_of, lens


def extend(mode: int, bdr_block: int, rotate_v: bool, k_pool, v_pool, k_sz, v_sz, q_bits, q_indptr, seq_lens,
           page_table, num_kv_heads: int, rows=None, rope=None, code_bits: int = 4):
    """Extend (chunked-prefill) attention in float64: causal attention of each sequence's
    newest tokens over the paged cache (the SAW-INT4 abstract: attention executed over the
    paged quantised cache; the wispaper.ai blog, section 3: the query rotated in step).

    The query at position p attends to tokens 0 .. p, which is the decode attention of a
    sequence of length p + 1 (query turned by the rotary table at p): this function is that
    definition, one decode row per (query, head).  q_bits: bf16 bits uint16 [total_q, Hq, D];
    rows: optional [(query row, query head), ...].  Returns (out float64 [n, D] or
    [total_q, Hq, D], skipped-token count)."""
    seq_of, lens = extend_lengths(q_indptr, seq_lens)
    lens = np.clip(lens, -1, np.iinfo(np.int32).max).astype(np.int32)  # <= 0: no tokens (zero row)
    pt = np.ascontiguousarray(np.asarray(page_table, dtype=np.int32)[seq_of])
    return decode(mode, bdr_block, rotate_v, k_pool, v_pool, k_sz, v_sz, q_bits, lens, pt, num_kv_heads,
                  rows=rows, rope=rope, code_bits=code_bits)
