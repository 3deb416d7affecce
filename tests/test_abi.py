"""CPU-side checks of the C ABI: the library builds/loads, exports every entry point
include/kvq.h declares, and host validation rejects bad arguments before touching
the GPU (none of these calls launches a kernel)."""
import ctypes
import os
import re

import pytest

from bit_paged_kv_append_b200 import kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for hdr in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if hdr.endswith(".h"):
            text = open(os.path.join(ROOT, "include", hdr)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(kv_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("kv_create_paged", "kv_append_quant", "kv_decode_attn", "kv_free"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = kvq.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(kvq.EXPORTS) <= set(declared_functions())


def test_status_strings():
    assert kvq.status_string(kvq.KV_OK) == "KV_OK"
    assert kvq.status_string(kvq.KV_ERR_OOB) == "KV_ERR_OOB"
    assert kvq.status_string(12345) == "KV_ERR_UNKNOWN"


def _desc(**kw):
    base = dict(num_pages=4, page_size=16, num_kv_heads=8, num_q_heads=32, head_dim=128, mode=kvq.KV_INT4_BDR,
                bdr_block=128, rotate_v=0, k_pool=0x1000, v_pool=0x2000, k_sz=0x3000, v_sz=0x4000)
    base.update(kw)
    return kvq.kv_desc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(num_pages=0), kvq.KV_ERR_INVALID),
    (dict(page_size=0), kvq.KV_ERR_INVALID),
    (dict(page_size=2048), kvq.KV_ERR_INVALID),
    (dict(num_q_heads=30), kvq.KV_ERR_INVALID),
    (dict(head_dim=64), kvq.KV_ERR_UNSUPPORTED),
    (dict(num_kv_heads=3, num_q_heads=12), kvq.KV_ERR_UNSUPPORTED),
    (dict(num_kv_heads=64, num_q_heads=64), kvq.KV_ERR_UNSUPPORTED),
    (dict(num_q_heads=8 * 16), kvq.KV_ERR_UNSUPPORTED),
    (dict(mode=7), kvq.KV_ERR_INVALID),
    (dict(bdr_block=8), kvq.KV_ERR_UNSUPPORTED),
    (dict(bdr_block=256), kvq.KV_ERR_UNSUPPORTED),
    (dict(k_pool=0), kvq.KV_ERR_INVALID),
    (dict(v_pool=0x2010), kvq.KV_ERR_INVALID),  # not 32-byte aligned
    (dict(k_sz=0), kvq.KV_ERR_INVALID),
    (dict(rope=0x5000, rope_positions=0), kvq.KV_ERR_INVALID),  # a table needs >= 1 row
    (dict(rope=0x5004, rope_positions=8), kvq.KV_ERR_INVALID),  # not 16-byte aligned
    (dict(code_bits=3), kvq.KV_ERR_UNSUPPORTED),
    (dict(code_bits=2, mode=kvq.KV_BF16), kvq.KV_ERR_INVALID),
])
def test_create_rejects_bad_descriptors(kw, status):
    lib = kvq.load()
    d = _desc(**kw)
    h = ctypes.c_void_p()
    assert lib.kv_create_paged(ctypes.byref(d), ctypes.byref(h)) == status
    assert h.value is None


def test_null_arguments_are_rejected():
    lib = kvq.load()
    assert lib.kv_create_paged(None, None) == kvq.KV_ERR_INVALID
    assert lib.kv_append_quant(None, None, None, 1, None, None, None, 1, 1, None) == kvq.KV_ERR_INVALID
    assert lib.kv_decode_attn(None, None, None, None, 1, 1, 1, None, 0, None, 0, None) == kvq.KV_ERR_INVALID
    assert lib.kv_extend_attn(None, None, None, None, None, 1, 1, 1, 1, None, 0, None) == kvq.KV_ERR_INVALID
    assert lib.kv_get_error(None, None) == kvq.KV_ERR_INVALID
    assert lib.kv_decode_workspace_bytes(None, 1, 1) == 0
    lib.kv_free(None)
