"""Seeded synthetic inputs for the KV-cache write/read path.

This module only draws random numbers and lays out page tables; it holds none
of the method's arithmetic (no rotation, no quantisation, no attention), so
both the CUDA path and the CPU oracle may consume what it produces.

Distributions follow the workloads of the SAW-INT4 pages (keys and values with
a few outlier channels per head, which is what the blog's section 2 says
wrecks naive INT4): K, V ~ N(0, 1) in fp32, a seeded set of channels per KV
head multiplied by a factor, then rounded to bf16; queries ~ N(0, 1) in bf16.
Outlier channels are fixed per head across tokens and drawn independently for
K and V.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Outliers:
    """n_channels seeded channels per KV head scaled by a factor ~ U[lo, hi]."""

    n_channels: int
    lo: float
    hi: float


OUTLIERS_X20 = Outliers(4, 20.0, 20.0)  # 4 channels per head, x20
OUTLIERS_1PCT = Outliers(max(1, round(0.01 * 128)), 10.0, 30.0)  # 1 % of 128 channels, x10..x30


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes of one synthetic serving workload (single layer)."""

    name: str
    num_kv_heads: int
    num_q_heads: int
    head_dim: int
    page_size: int
    outliers: Outliers
    description: str


# The five workloads, in the order the build's measurement plan lists them.
WORKLOADS = {
    "single256": Workload("single256", 8, 32, 128, 16, OUTLIERS_X20,
                          "1 sequence x 256 tokens, page size 16 (16 shuffled pages), then 1 decode step"),
    "batch16": Workload("batch16", 8, 32, 128, 16, OUTLIERS_X20,
                        "16 sequences, lengths ~U[512, 4096], page size 16, shuffled pages; append all, "
                        "then 1 decode step per sequence"),
    "decode64x8k": Workload("decode64x8k", 8, 32, 128, 16, OUTLIERS_1PCT,
                            "Qwen3-8B-like decode: 64 sequences x 8192 cached tokens, page size 16; "
                            "per step append 1 token per sequence then decode"),
    "mixed256": Workload("mixed256", 8, 64, 128, 16, OUTLIERS_1PCT,
                         "Qwen3-32B-like mixed serving: 256 sequences, lengths log-uniform [1024, 32768], "
                         "page size 16; 8 sequences append a 2048-token prefill chunk, the rest decode"),
    "long1m": Workload("long1m", 8, 32, 128, 64, OUTLIERS_1PCT,
                       "1 sequence x 1,048,576 tokens, page size 64, appended in 8192-token chunks, "
                       "then split-K decode"),
}


def outlier_multipliers(num_kv_heads: int, head_dim: int, spec: Outliers, seed: int) -> torch.Tensor:
    """fp32 [H, D] per-channel multipliers: 1 except spec.n_channels seeded channels per head."""
    g = torch.Generator().manual_seed(seed)
    mult = torch.ones(num_kv_heads, head_dim, dtype=torch.float32)
    for h in range(num_kv_heads):
        ch = torch.randperm(head_dim, generator=g)[: spec.n_channels]
        f = spec.lo + (spec.hi - spec.lo) * torch.rand(spec.n_channels, generator=g)
        mult[h, ch] = f
    return mult


def make_rows(num_tokens: int, mult: torch.Tensor, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [T, H, D]: N(0,1) fp32 times the per-channel multipliers, rounded to bf16."""
    H, D = mult.shape
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(num_tokens, H, D, generator=g, device=device, dtype=torch.float32)
    x.mul_(mult.to(device))
    return x.to(torch.bfloat16)


def make_kv(num_tokens: int, wl: Workload, seed: int, device="cpu", chunk: int | None = None):
    """Seeded K and V rows (bf16 [T, H, D]) with the workload's outlier channels.

    With ``chunk`` set, tokens are drawn chunk by chunk from seeds derived from
    (seed, chunk index) so that very long inputs can be produced piecewise.
    """
    mk = outlier_multipliers(wl.num_kv_heads, wl.head_dim, wl.outliers, seed * 7919 + 1)
    mv = outlier_multipliers(wl.num_kv_heads, wl.head_dim, wl.outliers, seed * 7919 + 2)
    if chunk is None:
        return make_rows(num_tokens, mk, seed * 2 + 101, device), make_rows(num_tokens, mv, seed * 2 + 102, device)
    ks, vs = [], []
    for c, start in enumerate(range(0, num_tokens, chunk)):
        n = min(chunk, num_tokens - start)
        ks.append(make_rows(n, mk, (seed * 1_000_003 + c) * 2 + 101, device))
        vs.append(make_rows(n, mv, (seed * 1_000_003 + c) * 2 + 102, device))
    return torch.cat(ks), torch.cat(vs)


def make_q(batch: int, num_q_heads: int, head_dim: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [B, Hq, D] ~ N(0, 1)."""
    g = torch.Generator(device=device).manual_seed(seed * 2 + 1_000_001)
    return torch.randn(batch, num_q_heads, head_dim, generator=g, device=device).to(torch.bfloat16)


def seq_lengths(wl_name: str, seed: int, num_seqs: int | None = None) -> list[int]:
    """Cached lengths per sequence for each named workload."""
    g = torch.Generator().manual_seed(seed * 31 + 7)
    if wl_name == "single256":
        return [256]
    if wl_name == "batch16":
        n = num_seqs or 16
        return [int(x) for x in torch.randint(512, 4097, (n,), generator=g)]
    if wl_name == "decode64x8k":
        return [8192] * (num_seqs or 64)
    if wl_name == "mixed256":
        n = num_seqs or 256
        u = torch.rand(n, generator=g, dtype=torch.float64)
        lo, hi = math.log(1024), math.log(32768)
        return [int(round(math.exp(lo + (hi - lo) * float(x)))) for x in u]
    if wl_name == "long1m":
        return [1 << 20]
    raise KeyError(wl_name)


def make_page_table(capacities: list[int], page_size: int, seed: int, spare_pages: int = 0):
    """Assign pages to sequences from a seeded global permutation of the pool.

    Sequence s gets ceil(capacities[s] / page_size) pages, taken in order from
    the permutation; unused page-table entries are -1.  Returns
    (page_table int32 [num_seqs, pt_stride], num_pages).
    """
    need = [max(1, -(-c // page_size)) for c in capacities]
    num_pages = sum(need) + spare_pages
    g = torch.Generator().manual_seed(seed * 131 + 17)
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    stride = max(need)
    pt = torch.full((len(capacities), stride), -1, dtype=torch.int32)
    off = 0
    for s, n in enumerate(need):
        pt[s, :n] = perm[off: off + n]
        off += n
    return pt, num_pages


def rope_table(positions: int, head_dim: int = 128, base: float = 1_000_000.0) -> torch.Tensor:
    """A rotary-embedding input table, float32 [positions, head_dim/2, 2] = (cos, sin) of angle
    pos * base^(-2i/head_dim) (the usual frequencies; computed in float64, rounded once)."""
    i = torch.arange(head_dim // 2, dtype=torch.float64)
    theta = base ** (-2.0 * i / head_dim)
    ang = torch.arange(positions, dtype=torch.float64)[:, None] * theta[None, :]
    return torch.stack([torch.cos(ang), torch.sin(ang)], dim=-1).to(torch.float32).contiguous()


def append_positions(lengths: list[int], starts: list[int] | None = None):
    """Flattened (tok_seq, tok_pos) int32 for appending lengths[s] tokens to sequence s at starts[s]."""
    starts = starts or [0] * len(lengths)
    seq = torch.cat([torch.full((n,), s, dtype=torch.int32) for s, n in enumerate(lengths)]) if lengths else \
        torch.empty(0, dtype=torch.int32)
    pos = torch.cat([torch.arange(st, st + n, dtype=torch.int32) for st, n in zip(starts, lengths)]) if lengths \
        else torch.empty(0, dtype=torch.int32)
    return seq, pos
