"""kv_decode_attn_noalloc: decode for callers that cannot allocate device memory at decode time
(code inside an allocator or memory pool, fixed-budget runtimes, hosts without a device
allocator).  It must give the same attention output as kv_decode_attn with a caller-allocated
workspace, call after call, while its split-K scratch is the library's fixed device array.

This file is named to be collected last, so a run that stops at the first failure has already
run every other test; it also passes when run alone in a fresh process."""
import numpy as np
import pytest
import torch

from bit_paged_kv_append_b200 import kvq, synth
from kvq_testlib import ATTN_RTOL, assert_pools_equal, attn_rel_err, gpu_append, make_case, oracle_append, oracle_decode

pytestmark = pytest.mark.gpu


def _decode_noalloc(c, q, lens, max_len, out_fp32=True):
    out = torch.empty(q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16, device="cuda")
    pt = c.page_table.cuda()
    kvq.kv_decode_attn_noalloc(c.cache.handle, q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"), pt,
                               pt.shape[1], q.shape[0], max_len, out, out_fp32)
    return out


def _decode_ws(c, q, lens, max_len, out_fp32=True):
    return c.cache.decode(q.cuda(), torch.tensor(lens, dtype=torch.int32, device="cuda"), c.page_table.cuda(),
                          max_len, out_fp32=out_fp32)


def test_noalloc_matches_workspace_decode_on_consecutive_calls():
    wl = synth.WORKLOADS["batch16"]
    lengths = synth.seq_lengths("batch16", seed=0)
    c = make_case(kvq.KV_INT4_BDR, 128, True, lengths, wl, seed=0)
    assert gpu_append(c) == kvq.KV_OK
    oracle_append(c)
    assert_pools_equal(c)
    # two calls in a row with different queries and batch shapes: the second must not see the first's scratch
    calls = [(synth.make_q(16, 32, 128, seed=11), lengths, max(lengths)),
             (synth.make_q(16, 32, 128, seed=12), [L // 3 for L in lengths], 5000)]
    for q, lens, max_len in calls:
        got = _decode_noalloc(c, q, lens, max_len)
        torch.cuda.synchronize()
        ref = _decode_ws(c, q, lens, max_len)
        assert c.cache.get_error() == kvq.KV_OK
        # the same plan and kernels as kv_decode_attn: the same bits
        assert torch.equal(got, ref)
        # and within the attention tolerance of the float64 oracle
        want, skipped = oracle_decode(c, q, lens)
        assert skipped == 0
        assert attn_rel_err(got.cpu().numpy(), want) <= ATTN_RTOL
        got16 = _decode_noalloc(c, q, lens, max_len, out_fp32=False)
        assert torch.equal(got16, got.to(torch.bfloat16))


def test_noalloc_rejects_requests_beyond_its_scratch():
    wl = synth.WORKLOADS["single256"]
    c = make_case(kvq.KV_INT4_BDR, 128, False, [256], wl, seed=0)
    assert gpu_append(c) == kvq.KV_OK
    batch = 4096  # 4096 x 32 heads x (512 + 8) B per split > 8 MiB
    assert kvq.kv_decode_workspace_bytes(c.cache.handle, batch, 256) > kvq.KV_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(batch, 32, 128, dtype=torch.bfloat16, device="cuda")
    lens = torch.full((batch,), 256, dtype=torch.int32, device="cuda")
    pt = c.page_table.cuda().expand(batch, -1).contiguous()
    out = torch.empty(batch, 32, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KVQError) as ei:
        kvq.kv_decode_attn_noalloc(c.cache.handle, q, lens, pt, pt.shape[1], batch, 256, out, False)
    assert ei.value.status == kvq.KV_ERR_SCRATCH_TOO_SMALL
    assert c.cache.get_error() == kvq.KV_OK
