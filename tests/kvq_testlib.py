"""Shared helpers for the parity tests: build one seeded case, run it through the
CUDA library (C ABI) and through the CPU oracle, and compare.

Tolerances (stated once, used everywhere):
  * pools, packed INT4 codes, scale/zero words, page tables: bit-exact;
  * attention: fp32 output of the kernel vs the float64 oracle, per (sequence,
    query head) row, max_i |o_i - r_i| / max_i |r_i| <= ATTN_RTOL; the bf16
    output must equal the fp32 output rounded to nearest even, bit for bit.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
from bit_paged_kv_append_b200 import kvq, synth

ATTN_RTOL = 2e-3
FILL = 0xA5
MODES = {"bf16": kvq.KV_BF16, "int4": kvq.KV_INT4, "bdr": kvq.KV_INT4_BDR}


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def np_pool(t: torch.Tensor | None) -> np.ndarray | None:
    if t is None:
        return None
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.uint8:
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


@dataclasses.dataclass
class Case:
    mode: int
    bdr: int
    rotate_v: bool
    wl: synth.Workload
    lengths: list
    k: torch.Tensor
    v: torch.Tensor
    tok_seq: torch.Tensor
    tok_pos: torch.Tensor
    page_table: torch.Tensor
    num_pages: int
    cache: kvq.PagedKVCache = None
    ref_pools: tuple = None
    rope: torch.Tensor = None  # optional (cos, sin) table, float32 [positions, 64, 2] on the CPU
    code_bits: int = 4


def make_case(mode, bdr, rotate_v, lengths, wl: synth.Workload, seed=0, spare_pages=3, device="cuda",
              starts=None, capacities=None, rope=None, code_bits=4):
    T = sum(lengths)
    k, v = synth.make_kv(T, wl, seed)
    caps = capacities or [st + n for st, n in zip(starts or [0] * len(lengths), lengths)]
    pt, P = synth.make_page_table(caps, wl.page_size, seed, spare_pages=spare_pages)
    ts, tp = synth.append_positions(lengths, starts)
    c = Case(mode, bdr, rotate_v, wl, lengths, k, v, ts, tp, pt, P)
    c.rope = rope
    c.code_bits = code_bits
    c.cache = kvq.PagedKVCache(P, wl.page_size, wl.num_kv_heads, wl.num_q_heads, mode, bdr, rotate_v,
                               device=device, fill=FILL, rope=None if rope is None else rope.to(device),
                               code_bits=code_bits)
    return c


def gpu_append(c: Case, k=None, v=None, ts=None, tp=None):
    k = (c.k if k is None else k).cuda()
    v = (c.v if v is None else v).cuda()
    ts = (c.tok_seq if ts is None else ts).cuda()
    tp = (c.tok_pos if tp is None else tp).cuda()
    c.cache.append(k, v, ts, tp, c.page_table.cuda())
    return c.cache.get_error()


def oracle_pools(c: Case):
    H, ps, P = c.wl.num_kv_heads, c.wl.page_size, c.num_pages
    if c.mode == kvq.KV_BF16:
        kp = np.full((P, H, ps, 128), FILL * 257, dtype=np.uint16)
        vp = kp.copy()
        ks = vs = np.zeros(1, dtype=np.uint16)
    else:
        kp = np.full((P, H, ps, 16 * c.code_bits), FILL, dtype=np.uint8)
        vp = kp.copy()
        ks = np.full((P, H, ps, 2), FILL * 257, dtype=np.uint16)
        vs = ks.copy()
    return kp, vp, ks, vs


def oracle_append(c: Case, pools=None, k=None, v=None, ts=None, tp=None):
    pools = pools or oracle_pools(c)
    kp, vp, ks, vs = pools
    skipped = oracle.append(c.mode, c.bdr, c.rotate_v, kp, vp, ks, vs, bits16(c.k if k is None else k),
                            bits16(c.v if v is None else v), (c.tok_seq if ts is None else ts).numpy(),
                            (c.tok_pos if tp is None else tp).numpy(), c.page_table.numpy(),
                            rope=None if c.rope is None else c.rope.numpy(), code_bits=c.code_bits)
    c.ref_pools = pools
    return skipped


def assert_pools_equal(c: Case):
    kp, vp, ks, vs = c.ref_pools
    gk, gv = np_pool(c.cache.k_pool), np_pool(c.cache.v_pool)
    assert np.array_equal(gk, kp), _first_diff(gk, kp, "k_pool")
    assert np.array_equal(gv, vp), _first_diff(gv, vp, "v_pool")
    if c.mode != kvq.KV_BF16:
        gks, gvs = np_pool(c.cache.k_sz), np_pool(c.cache.v_sz)
        assert np.array_equal(gks, ks), _first_diff(gks, ks, "k_sz")
        assert np.array_equal(gvs, vs), _first_diff(gvs, vs, "v_sz")


def _first_diff(a, b, name):
    idx = np.argwhere(a != b)
    if idx.size == 0:
        return f"{name}: shapes {a.shape} vs {b.shape}"
    i = tuple(idx[0])
    return f"{name}: {len(idx)} mismatches, first at {i}: gpu {a[i]} vs oracle {b[i]}"


def gpu_decode(c: Case, q, seq_lens, max_len=None, page_table=None, out_fp32=True):
    pt = (c.page_table if page_table is None else page_table).cuda()
    sl = torch.as_tensor(seq_lens, dtype=torch.int32).cuda()
    max_len = max(seq_lens) if max_len is None else max_len
    out = c.cache.decode(q.cuda(), sl, pt, max_len, out_fp32=out_fp32)
    return out, c.cache.get_error()


def oracle_decode(c: Case, q, seq_lens, rows=None, page_table=None):
    kp, vp, ks, vs = c.ref_pools
    pt = (c.page_table if page_table is None else page_table).numpy()
    return oracle.decode(c.mode, c.bdr, c.rotate_v, kp, vp, ks, vs, bits16(q), np.asarray(seq_lens), pt,
                         c.wl.num_kv_heads, rows=rows, rope=None if c.rope is None else c.rope.numpy(),
                         code_bits=c.code_bits)


def oracle_decode_rows(mode, bdr, rotate_v, pools, q_bits, seq_lens, page_table, num_kv_heads, rows, threads=None,
                       rope=None, code_bits=4):
    """oracle.decode over the given (sequence, query head) rows, split into contiguous parts run
    on concurrent threads (the C oracle keeps no global state and ctypes releases the GIL); the
    rows come back in the order given.  Returns (out float64 [n, D], skipped-token count)."""
    import concurrent.futures
    import os

    kp, vp, ks, vs = pools
    rows = [tuple(map(int, r)) for r in rows]
    n = len(rows)
    threads = max(1, min(threads or (os.cpu_count() or 1), n))
    cuts = np.linspace(0, n, threads + 1).astype(int)

    def part(i):
        sub = rows[cuts[i]:cuts[i + 1]]
        if not sub:
            return np.zeros((0, 128)), 0
        return oracle.decode(mode, bdr, rotate_v, kp, vp, ks, vs, q_bits, np.asarray(seq_lens), page_table,
                             num_kv_heads, rows=sub, rope=rope, code_bits=code_bits)

    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(part, range(threads)))
    return np.concatenate([p[0] for p in parts]), sum(p[1] for p in parts)


def attn_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of max_i |got - ref| / max_i |ref| (rows with ref == 0 compare absolutely)."""
    got = got.reshape(-1, got.shape[-1]).astype(np.float64)
    ref = ref.reshape(-1, ref.shape[-1]).astype(np.float64)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    num = np.abs(got - ref).max(axis=1)
    zero = np.abs(ref).max(axis=1) == 0
    rel = np.where(zero, num, num / den)
    return float(rel.max()) if rel.size else 0.0
