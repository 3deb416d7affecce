"""ctypes binding of libkvq.so (``include/kvq.h``), same entry-point names.

This module only marshals arguments: torch tensors become raw device pointers,
``stream=None`` becomes torch's current CUDA stream, and a non-OK status raises
:class:`KVQError`.  Every step of the write and read path runs in the CUDA
kernels behind the C ABI; there is no fallback of any kind, and loading fails
loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

KV_OK, KV_ERR_INVALID, KV_ERR_UNSUPPORTED, KV_ERR_CUDA, KV_ERR_OOB, KV_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
KV_ERR_SCRATCH_TOO_SMALL = -6
KV_NOALLOC_SCRATCH_BYTES = 8 << 20  # size of the fixed scratch behind kv_decode_attn_noalloc
KV_BF16, KV_INT4, KV_INT4_BDR = 0, 1, 2
HEAD_DIM = 128

EXPORTS = ("kv_create_paged", "kv_append_quant", "kv_decode_workspace_bytes", "kv_decode_attn", "kv_get_error",
           "kv_free", "kv_status_string", "kv_decode_attn_noalloc", "kv_extend_attn")


class KVQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class kv_desc(ctypes.Structure):
    _fields_ = [("num_pages", ctypes.c_int), ("page_size", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("num_q_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("mode", ctypes.c_int),
                ("bdr_block", ctypes.c_int), ("rotate_v", ctypes.c_int), ("k_pool", ctypes.c_void_p),
                ("v_pool", ctypes.c_void_p), ("k_sz", ctypes.c_void_p), ("v_sz", ctypes.c_void_p),
                ("rope", ctypes.c_void_p), ("rope_positions", ctypes.c_int), ("code_bits", ctypes.c_int)]


_lib = None


def load(path: str | None = None, build_if_missing: bool = True):
    """Load libkvq.so (building it in-tree with nvcc first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or _build.LIB
    if build_if_missing and _build.stale():
        _build.build()
    if not os.path.exists(path):
        raise OSError(f"libkvq.so not found at {path}; build it with `python -m bit_paged_kv_append_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.kv_create_paged.argtypes = [ctypes.POINTER(kv_desc), ctypes.POINTER(P)]
    lib.kv_create_paged.restype = I
    lib.kv_append_quant.argtypes = [P, P, P, I, P, P, P, I, I, P]
    lib.kv_append_quant.restype = I
    lib.kv_decode_workspace_bytes.argtypes = [P, I, I]
    lib.kv_decode_workspace_bytes.restype = Z
    lib.kv_decode_attn.argtypes = [P, P, P, P, I, I, I, P, I, P, Z, P]
    lib.kv_decode_attn.restype = I
    lib.kv_decode_attn_noalloc.argtypes = [P, P, P, P, I, I, I, P, I, P]
    lib.kv_decode_attn_noalloc.restype = I
    lib.kv_extend_attn.argtypes = [P, P, P, P, P, I, I, I, I, P, I, P]
    lib.kv_extend_attn.restype = I
    lib.kv_get_error.argtypes = [P, P]
    lib.kv_get_error.restype = I
    lib.kv_free.argtypes = [P]
    lib.kv_free.restype = None
    lib.kv_status_string.argtypes = [I]
    lib.kv_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().kv_status_string(int(status)).decode()


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    return int(x)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, what: str):
    if status != KV_OK:
        raise KVQError(status, what)


def kv_create_paged(num_pages, page_size, num_kv_heads, num_q_heads, head_dim, mode, bdr_block, rotate_v,
                    k_pool, v_pool, k_sz=None, v_sz=None, rope=None, code_bits=4) -> int:
    """Returns the opaque handle (an integer address); release it with kv_free.  rope: optional
    device float32 [positions, head_dim/2, 2] (cos, sin) table (fused rotary embedding);
    code_bits: 4 or 2 for the INT4 modes."""
    d = kv_desc(num_pages, page_size, num_kv_heads, num_q_heads, head_dim, mode, bdr_block, int(bool(rotate_v)),
                _ptr(k_pool), _ptr(v_pool), _ptr(k_sz), _ptr(v_sz), _ptr(rope),
                int(rope.shape[0]) if rope is not None else 0, int(code_bits))
    h = ctypes.c_void_p()
    _check(load().kv_create_paged(ctypes.byref(d), ctypes.byref(h)), "kv_create_paged")
    return h.value


def kv_append_quant(cache, k, v, num_tokens, tok_seq, tok_pos, page_table, pt_stride, num_seqs, stream=None):
    _check(load().kv_append_quant(cache, _ptr(k), _ptr(v), int(num_tokens), _ptr(tok_seq), _ptr(tok_pos),
                                  _ptr(page_table), int(pt_stride), int(num_seqs), _stream(stream)),
           "kv_append_quant")


def kv_decode_workspace_bytes(cache, batch, max_seq_len) -> int:
    return int(load().kv_decode_workspace_bytes(cache, int(batch), int(max_seq_len)))


def kv_decode_attn(cache, q, seq_lens, page_table, pt_stride, batch, max_seq_len, out, out_fp32, workspace,
                   workspace_bytes, stream=None):
    _check(load().kv_decode_attn(cache, _ptr(q), _ptr(seq_lens), _ptr(page_table), int(pt_stride), int(batch),
                                 int(max_seq_len), _ptr(out), int(bool(out_fp32)), _ptr(workspace),
                                 int(workspace_bytes), _stream(stream)), "kv_decode_attn")


def kv_decode_attn_noalloc(cache, q, seq_lens, page_table, pt_stride, batch, max_seq_len, out, out_fp32,
                           stream=None):
    """kv_decode_attn for callers that cannot allocate device memory when they decode (code inside an
    allocator or memory pool, fixed-budget runtimes, hosts without a device allocator): the split-K scratch
    is the library's fixed KV_NOALLOC_SCRATCH_BYTES device array, so no workspace is passed.  Calls that
    need more scratch raise KVQError(KV_ERR_SCRATCH_TOO_SMALL); calls overlapping on the GPU share the
    array and race, so keep them on one stream."""
    _check(load().kv_decode_attn_noalloc(cache, _ptr(q), _ptr(seq_lens), _ptr(page_table), int(pt_stride),
                                         int(batch), int(max_seq_len), _ptr(out), int(bool(out_fp32)),
                                         _stream(stream)), "kv_decode_attn_noalloc")


def kv_extend_attn(cache, q, q_indptr, seq_lens, page_table, pt_stride, batch, max_q_len, max_seq_len, out,
                   out_fp32, stream=None):
    _check(load().kv_extend_attn(cache, _ptr(q), _ptr(q_indptr), _ptr(seq_lens), _ptr(page_table), int(pt_stride),
                                 int(batch), int(max_q_len), int(max_seq_len), _ptr(out), int(bool(out_fp32)),
                                 _stream(stream)), "kv_extend_attn")


def kv_get_error(cache, stream=None) -> int:
    """Synchronises the stream; returns (does not raise) KV_OK, KV_ERR_OOB or KV_ERR_TIMEOUT."""
    return int(load().kv_get_error(cache, _stream(stream)))


def kv_free(cache):
    if cache:
        load().kv_free(cache)


# ---- device-memory plumbing (torch allocations in the documented layouts) ----

def alloc_pools(num_pages, page_size, num_kv_heads, mode, device="cuda", fill: int | None = None, code_bits=4):
    """Caller-owned pools for a cache: (k_pool, v_pool, k_sz, v_sz); sz is None in BF16 mode."""
    if mode == KV_BF16:
        shape = (num_pages, num_kv_heads, page_size, HEAD_DIM)
        k = torch.empty(shape, dtype=torch.bfloat16, device=device)
        v = torch.empty(shape, dtype=torch.bfloat16, device=device)
        ks = vs = None
    else:
        shape = (num_pages, num_kv_heads, page_size, HEAD_DIM * code_bits // 8)
        k = torch.empty(shape, dtype=torch.uint8, device=device)
        v = torch.empty(shape, dtype=torch.uint8, device=device)
        ks = torch.empty((num_pages, num_kv_heads, page_size, 2), dtype=torch.float16, device=device)
        vs = torch.empty_like(ks)
    if fill is not None:
        for t in (k, v, ks, vs):
            if t is not None:
                t.view(torch.uint8).fill_(fill)
    return k, v, ks, vs


class PagedKVCache:
    """Owns one handle over caller-provided (or freshly allocated) pools."""

    def __init__(self, num_pages, page_size, num_kv_heads, num_q_heads, mode, bdr_block=128, rotate_v=False,
                 pools=None, device="cuda", fill=None, rope=None, code_bits=4):
        self.mode, self.bdr_block, self.rotate_v = mode, bdr_block, bool(rotate_v)
        self.rope = rope  # kept alive with the handle
        self.code_bits = code_bits
        self.num_pages, self.page_size = num_pages, page_size
        self.num_kv_heads, self.num_q_heads = num_kv_heads, num_q_heads
        self.k_pool, self.v_pool, self.k_sz, self.v_sz = pools or alloc_pools(num_pages, page_size, num_kv_heads,
                                                                               mode, device, fill, code_bits)
        self.handle = kv_create_paged(num_pages, page_size, num_kv_heads, num_q_heads, HEAD_DIM, mode, bdr_block,
                                      rotate_v, self.k_pool, self.v_pool, self.k_sz, self.v_sz, rope, code_bits)

    def append(self, k, v, tok_seq, tok_pos, page_table, stream=None):
        kv_append_quant(self.handle, k, v, k.shape[0], tok_seq, tok_pos, page_table, page_table.shape[1],
                        page_table.shape[0], stream)

    def workspace(self, batch, max_seq_len, device="cuda"):
        n = kv_decode_workspace_bytes(self.handle, batch, max_seq_len)
        return torch.empty(max(n, 16), dtype=torch.uint8, device=device), n

    def decode(self, q, seq_lens, page_table, max_seq_len, out=None, out_fp32=False, workspace=None,
               stream=None):
        B = q.shape[0]
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
        if workspace is None:
            workspace = self.workspace(B, max_seq_len, q.device)
        ws, n = workspace
        kv_decode_attn(self.handle, q, seq_lens, page_table, page_table.shape[1], B, max_seq_len, out, out_fp32,
                       ws, ws.numel(), stream)
        return out

    def extend(self, q, q_indptr, seq_lens, page_table, max_q_len, max_seq_len, out=None, out_fp32=False,
               stream=None):
        """Causal attention of each sequence's newest q_indptr[s+1] - q_indptr[s] tokens (rows of q)."""
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
        kv_extend_attn(self.handle, q, q_indptr, seq_lens, page_table, page_table.shape[1], seq_lens.shape[0],
                       max_q_len, max_seq_len, out, out_fp32, stream)
        return out

    def get_error(self, stream=None) -> int:
        return kv_get_error(self.handle, stream)

    def close(self):
        if self.handle:
            kv_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
