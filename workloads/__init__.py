"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle checks.

This module holds only workload *data*: shapes, seeds, value distributions and the
per-layer (anchor, d, b) tables.  It contains none of the method's arithmetic (no
quantiser, no attention, no cost model).  The tables in ``tables.json`` were written by
``oracle/make_tables.py``, which uses the oracle's cost function only.

The five workloads follow the serving shapes of the KV-Kaizen pages (Qwen2.5-7B / -14B
shapes, 32 sequences x 8k tokens, the 1/8 eviction keep ratio, the budget sweep):

* ``tiny``      1 seq, 4 layers (anchors L0, L2), 8 heads, r=64, d_R=16, 256 tokens, fp32
* ``7b_4x``     28 layers, 28 heads, r=512, d_R=64, batch 8, 8192 tokens, bf16, 4x budget
* ``14b_4x``    48 layers, 40 heads, r=512, d_R=64, batch 32, 8192 tokens, bf16, 4x budget,
                latent channel j scaled by std_j ~ U(0.5, 2) (per layer)
* ``14b_evict`` as 14b with batch 16, 32768 tokens, sorted keep list of 4096 per sequence
* ``14b_sweep`` as 14b with batch 8, 8192-token prefill, budgets 1x..16x, Student-t(3) latents

Two fixed plans of the 14B shape (batch 32, 8192 tokens, latents as ``14b_4x``) bracket them:

* ``14b_bf16``  every layer an uncompressed bf16 anchor with the full rank (d = 512): the MLA
                cache the compression is measured against (C_0 / bits = 3.56)
* ``14b_g32``   the composition of the M3 Ultra benchmark: 12 anchors (one per 4 layers) of
                rank 128 at 4 bits with one fp16 scale per 32 elements (C_0 / bits = 151.7)
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
TABLES_PATH = os.path.join(_HERE, "tables.json")


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_heads: int
    r: int
    d_rope: int
    batch: int
    tokens: int
    dtype: str                 # "f32" or "bf16" (input / query dtype)
    latent_dist: str           # "normal" | "channel_std" | "student_t3"
    n_kv: int = 0              # non-MLA KV heads (for C_0); 0 = not applicable
    d_h: int = 0               # non-MLA head dim (for C_0)
    keep: int = 0              # tokens kept per sequence (0 = no eviction)
    budgets: tuple = ()        # compression targets rho* (C_0 / budget bits)
    d_set: tuple = ()
    b_set: tuple = ()
    seed: int = 0
    prefill: bool = False
    scale_group: int = 0       # elements per fp16 scale (0: one scale per token)
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny": Workload("tiny", 4, 8, 64, 16, 1, 256, "f32", "normal", seed=11),
    "7b_4x": Workload("7b_4x", 28, 28, 512, 64, 8, 8192, "bf16", "normal", n_kv=4, d_h=128,
                      budgets=(4,), d_set=(128, 256, 384, 512), b_set=(4, 8, 16), seed=7),
    "14b_4x": Workload("14b_4x", 48, 40, 512, 64, 32, 8192, "bf16", "channel_std", n_kv=8,
                       d_h=128, budgets=(4,), d_set=(128, 256, 384, 512), b_set=(4, 8, 16),
                       seed=14),
    "14b_evict": Workload("14b_evict", 48, 40, 512, 64, 16, 32768, "bf16", "normal", n_kv=8,
                          d_h=128, keep=4096, budgets=(4,), d_set=(128, 256, 384, 512),
                          b_set=(4, 8, 16), seed=32),
    "14b_bf16": Workload("14b_bf16", 48, 40, 512, 64, 32, 8192, "bf16", "channel_std", n_kv=8,
                         d_h=128, seed=14),
    "14b_g32": Workload("14b_g32", 48, 40, 512, 64, 32, 8192, "bf16", "channel_std", n_kv=8,
                        d_h=128, seed=14, scale_group=32),
    "14b_sweep": Workload("14b_sweep", 48, 40, 512, 64, 8, 8192, "bf16", "student_t3", n_kv=8,
                          d_h=128, budgets=(1, 2, 4, 8, 16), d_set=(128, 256, 384, 512),
                          b_set=(2, 4, 8, 16), seed=16, prefill=True),
}

# The tiny workload's table is fixed: L0 anchor (d=32, b=8), L1 -> L0, L2 anchor
# (d=64, b=4), L3 -> L2; "tiny_swap" exchanges the two anchors' (d, b).
TINY_TABLES = {
    "tiny": {"anchor": [0, 0, 2, 2], "d": [32, 0, 64, 0], "b": [8, 0, 4, 0]},
    "tiny_swap": {"anchor": [0, 0, 2, 2], "d": [64, 0, 32, 0], "b": [4, 0, 8, 0]},
}


# Fixed plans of the 14B shape (b = 0: an uncompressed bf16 anchor).
FIXED_TABLES = {
    "14b_bf16": {"anchor": list(range(48)), "d": [512] * 48, "b": [0] * 48},
    "14b_g32": {"anchor": [4 * (l // 4) for l in range(48)],
                "d": [128 if l % 4 == 0 else 0 for l in range(48)],
                "b": [4 if l % 4 == 0 else 0 for l in range(48)]},
}


def load_tables() -> dict:
    with open(TABLES_PATH) as f:
        t = json.load(f)
    t.update({k: dict(v) for k, v in TINY_TABLES.items()})
    t.update({k: dict(v) for k, v in FIXED_TABLES.items()})
    return t


def table(name: str, budget: int | None = None) -> dict:
    """Per-layer table {anchor, d, b, ...} of a workload (``budget`` selects a sweep point)."""
    tabs = load_tables()
    key = name if budget is None else f"{name}@{budget}x"
    if key not in tabs:
        key = f"{name}@{WORKLOADS[name].budgets[0]}x"
    return tabs[key]


# --------------------------------------------------------------------------
# seeded tensors
# --------------------------------------------------------------------------

_KIND = {"c_kv": 1, "k_rope": 2, "q_lat": 3, "q_rope": 4, "std": 5, "keep": 6, "append": 7}


def _gen(w: Workload, layer: int, kind: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((w.seed * 1_000_003 + layer * 1009 + _KIND[kind] * 7919) & 0x7FFFFFFFFFFF)
    return g


def torch_dtype(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def latent(w: Workload, layer: int, batch: int, tokens: int, device="cpu", kind="c_kv"):
    """Latent c^KV [batch, tokens, r] for an anchor layer, in the workload's dtype."""
    g = _gen(w, layer, kind, device)
    x = torch.randn(batch, tokens, w.r, generator=g, device=device, dtype=torch.float32)
    if w.latent_dist == "channel_std":
        gs = _gen(w, layer, "std", device)
        std = torch.empty(w.r, device=device, dtype=torch.float32).uniform_(0.5, 2.0, generator=gs)
        x.mul_(std)
    elif w.latent_dist == "student_t3":
        chi = torch.zeros_like(x)
        for _ in range(3):
            chi.add_(torch.randn(x.shape, generator=g, device=device, dtype=torch.float32).square_())
        x.div_(chi.div_(3.0).sqrt_())
    return x.to(torch_dtype(w))


def rope_key(w: Workload, layer: int, batch: int, tokens: int, device="cpu", kind="k_rope"):
    """Decoupled RoPE key k^R [batch, tokens, d_R], N(0, 1), in the workload's dtype."""
    g = _gen(w, layer, kind, device)
    x = torch.randn(batch, tokens, w.d_rope, generator=g, device=device, dtype=torch.float32)
    return x.to(torch_dtype(w))


def queries(w: Workload, layer: int, batch: int, device="cpu"):
    """(q_lat [batch, H, r], q_rope [batch, H, d_R]), N(0, 1), in the workload's dtype."""
    g = _gen(w, layer, "q_lat", device)
    ql = torch.randn(batch, w.n_heads, w.r, generator=g, device=device, dtype=torch.float32)
    g = _gen(w, layer, "q_rope", device)
    qr = torch.randn(batch, w.n_heads, w.d_rope, generator=g, device=device, dtype=torch.float32)
    return ql.to(torch_dtype(w)), qr.to(torch_dtype(w))


def keep_lists(w: Workload, batch: int, tokens: int, keep: int, device="cpu"):
    """Sorted keep indices [batch, keep] int32: uniform without replacement per sequence."""
    g = _gen(w, 0, "keep", device)
    out = torch.empty(batch, keep, dtype=torch.int32, device=device)
    for s in range(batch):
        perm = torch.randperm(tokens, generator=g, device=device)[:keep]
        out[s] = torch.sort(perm).values.to(torch.int32)
    return out


def softmax_scale(d: int, d_rope: int) -> float:
    """Per-layer softmax scale 1/sqrt(d + d_R) of the anchor's row width."""
    return 1.0 / float(d + d_rope) ** 0.5
