"""Crafted inputs for the paths that seeded random data rarely reaches.

Both attention kernels keep the online softmax's reference maximum lazily: it moves only when a
later block's scores pass it by 2^8, and then the accumulated output and sums are rescaled (the
decode in registers; the tcgen05 extend in tensor memory and in its fp32 fold copy).  The extend
also scales P by a power of two chosen from the value scales seen so far and raises it when a
later block's values are larger.  With N(0,1) rows the first blocks already hold nearly the
largest scores and scales, so these moves almost never happen after the first block.  Here a few
key rows are multiplied by 30 (their scores jump far above everything before them) and a few
value rows by 200 (their scales jump), at positions in different 128-token blocks, including a
block where the extend also folds its accumulator.  Every (query, head) row of the decode and of a
full causal prefill is compared with the float64 oracle; pools are checked bit for bit first."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import (ATTN_RTOL, assert_pools_equal, attn_rel_err, bits16, gpu_append, gpu_decode, make_case,
                         oracle_append, oracle_decode)

pytestmark = pytest.mark.gpu


def _crafted(mode, b, rv, H, Hq, lengths, key_jumps, value_jumps, seed):
    wl = dataclasses.replace(synth.WORKLOADS["batch16"], num_kv_heads=H, num_q_heads=Hq, page_size=16)
    c = make_case(mode, b, rv, lengths, wl, seed=seed)
    k, v = c.k.float(), c.v.float()
    for t0, t1, f in key_jumps:  # rows t0 .. t1 - 1 of the sequence-major token list
        k[t0:t1] *= f
    for t0, t1, f in value_jumps:
        v[t0:t1] *= f
    c.k, c.v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    return c


def _extend_all_rows(c, lengths, q):
    qi = torch.as_tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)).cuda()
    sl = torch.as_tensor(lengths, dtype=torch.int32).cuda()
    out = c.cache.extend(q.cuda(), qi, sl, c.page_table.cuda(), max(lengths), max(lengths), out_fp32=True)
    assert c.cache.get_error() == kvq.KV_OK
    kp, vp, ks, vs = c.ref_pools
    ref, skipped = oracle.extend(c.mode, c.bdr, c.rotate_v, kp, vp, ks, vs, bits16(q), qi.cpu().numpy(),
                                 np.asarray(lengths), c.page_table.numpy(), c.wl.num_kv_heads)
    assert skipped == 0
    return out.cpu().numpy(), ref


# (id, mode, block, rotate_v, H_kv, H_q): G = 4 and G = 8, keys only and keys + values rotated, naive
# INT4, and BF16 pages (decode only: the extend serves the INT4 modes)
CASES = [("g4_bdr128k", kvq.KV_INT4_BDR, 128, False, 2, 8),
         ("g8_bdr64kv", kvq.KV_INT4_BDR, 64, True, 2, 16),
         ("g4_int4", kvq.KV_INT4, 0, False, 2, 8),
         ("g8_bf16", kvq.KV_BF16, 0, False, 2, 16)]


@pytest.mark.parametrize("name,mode,b,rv,H,Hq", CASES, ids=[c[0] for c in CASES])
def test_reference_and_scale_moves(name, mode, b, rv, H, Hq):
    lengths = [1200, 700]
    # sequence 0: key jumps in blocks 2 and 7 (positions 300.., 900..), a value jump in block 3 and
    # one in block 4 (a fold block of the extend); sequence 1 (rows 1200..): a key jump in block 1
    # and a value jump in block 4
    key_jumps = [(300, 304, 30.0), (900, 903, 30.0), (1200 + 130, 1200 + 133, 30.0)]
    value_jumps = [(450, 455, 200.0), (520, 522, 200.0), (1200 + 530, 1200 + 540, 200.0)]
    c = _crafted(mode, b, rv, H, Hq, lengths, key_jumps, value_jumps, seed=41)
    q = synth.make_q(sum(lengths), Hq, 128, seed=42)

    # decode: the newest token of each sequence attends to all of it
    qd = q[np.cumsum(lengths) - 1]
    out, st = gpu_decode(c, qd, lengths)
    assert st == kvq.KV_OK
    ref, skipped = oracle_decode(c, qd, lengths)
    assert skipped == 0
    assert attn_rel_err(out.cpu().numpy(), ref) <= ATTN_RTOL

    if mode == kvq.KV_BF16:
        return
    # extend: a full causal prefill, so rows end before, inside and after every jump
    o, ref = _extend_all_rows(c, lengths, q)
    assert np.isfinite(o).all()
    assert attn_rel_err(o, ref) <= ATTN_RTOL
