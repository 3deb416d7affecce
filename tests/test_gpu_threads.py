"""Host threads sharing one process: two threads each create a cache handle, append into it
and run decode and extend attention on their own CUDA streams at the same time.  The first
launch of a kernel raises its shared-memory limit for the device; two threads may reach it
together, so the check runs in a fresh process where no kernel has been launched yet.  Each
thread's pools must equal the oracle's bit for bit and its attention rows must be within
the tolerance of the oracle's float64 decode."""
import os
import subprocess
import sys
import threading

import numpy as np
import pytest
import torch

from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import (ATTN_RTOL, assert_pools_equal, attn_rel_err, make_case, oracle_append, oracle_decode,
                         oracle_pools)
import oracle

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _worker(mode, b, rv, seed, results, idx):
    try:
        wl = synth.WORKLOADS["batch16"]
        lengths = [int(x) for x in np.random.default_rng(seed).integers(300, 1500, size=4)]
        c = make_case(mode, b, rv, lengths, wl, seed=seed)
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            pt = c.page_table.cuda()
            c.cache.append(c.k.cuda(), c.v.cuda(), c.tok_seq.cuda(), c.tok_pos.cuda(), pt, stream=stream)
            q = synth.make_q(len(lengths), wl.num_q_heads, 128, seed=seed + 1).cuda()
            sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
            out = c.cache.decode(q, sl, pt, max(lengths), out_fp32=True, stream=stream)
            n_new = 64
            qe = synth.make_q(n_new * len(lengths), wl.num_q_heads, 128, seed=seed + 2).cuda()
            qi = torch.arange(0, n_new * len(lengths) + 1, n_new, dtype=torch.int32, device="cuda")
            oute = c.cache.extend(qe, qi, sl, pt, n_new, max(lengths), out_fp32=True, stream=stream)
        status = c.cache.get_error(stream)
        results[idx] = (c, q.cpu(), out.cpu(), qe.cpu(), qi.cpu(), oute.cpu(), status)
    except Exception as e:  # reported by the main thread
        results[idx] = e


def _two_threads():
    torch.cuda.init()
    results = [None, None]
    cfgs = [(kvq.KV_INT4_BDR, 128, False, 3), (kvq.KV_INT4_BDR, 128, False, 4)]
    ths = [threading.Thread(target=_worker, args=(*cfg, results, i)) for i, cfg in enumerate(cfgs)]
    for t in ths:
        t.start()
    for t in ths:
        t.join()
    torch.cuda.synchronize()
    for r in results:
        if isinstance(r, Exception):
            raise r
        c, q, out, qe, qi, oute, status = r
        assert status == kvq.KV_OK
        oracle_append(c)
        assert_pools_equal(c)
        want, skipped = oracle_decode(c, q, c.lengths)
        assert skipped == 0
        assert attn_rel_err(out.numpy(), want) <= ATTN_RTOL
        kp, vp, ks, vs = c.ref_pools
        from kvq_testlib import bits16
        rows = [(i, j) for i in range(0, qe.shape[0], 37) for j in (0, 31)]
        ref, sk = oracle.extend(c.mode, c.bdr, c.rotate_v, kp, vp, ks, vs, bits16(qe), qi.numpy(), c.lengths,
                                c.page_table.numpy(), c.wl.num_kv_heads, rows=rows)
        assert sk == 0
        got = np.stack([oute[i, j].numpy() for i, j in rows])
        assert attn_rel_err(got, ref) <= ATTN_RTOL
    print("two-thread check passed")


def test_two_host_threads_fresh_process():
    code = f"import sys; sys.path[:0] = [{ROOT!r}, {HERE!r}]; import test_gpu_threads as t; t._two_threads()"
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "two-thread check passed" in r.stdout
