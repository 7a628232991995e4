"""Helpers for the GPU parity tests: build caches through the C ABI from seeded inputs and
compare against the CPU oracle run on the very same inputs (copied to the host)."""
from __future__ import annotations

import numpy as np
import torch

TOL_REL = 2e-3      # per (sequence, head): max|o - o_ref| <= TOL_REL * max|o_ref|
TOL_LSE = 2e-3      # absolute, natural-log units


def bf16_or_f32_to_np(t: torch.Tensor) -> np.ndarray:
    """Exact host copy as float32 (bf16 widening is exact)."""
    return t.detach().cpu().float().numpy()


def check_outputs(out, lse, o_ref, l_ref, what=""):
    """out [H, d] vs o_ref [H, d]: per-head relative max error; lse absolute."""
    out = np.asarray(out, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    err = np.abs(out - o_ref).max(axis=1)
    ref = np.abs(o_ref).max(axis=1)
    bad = err > TOL_REL * ref
    assert not bad.any(), (f"{what}: heads {np.nonzero(bad)[0][:8]} rel err "
                           f"{(err / np.maximum(ref, 1e-300)).max():.3e}")
    if lse is not None:
        lse = np.asarray(lse, dtype=np.float64)
        fin = np.isfinite(l_ref)
        assert np.array_equal(np.isfinite(lse), fin), what
        if fin.any():
            e = np.abs(lse[fin] - l_ref[fin]).max()
            assert e <= TOL_LSE, f"{what}: lse err {e:.3e}"
    return (err / np.maximum(ref, 1e-300)).max() if len(err) else 0.0


def rel_err(out, o_ref):
    out = np.asarray(out, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    return (np.abs(out - o_ref).max(axis=1) / np.maximum(np.abs(o_ref).max(axis=1), 1e-300)).max()


class Case:
    """One layer configuration: a 2-layer plan (anchor + inheriting layer) with given d, b."""

    def __init__(self, pkg, d, b, r, d_rope, batch, max_tokens, device="cuda"):
        self.d, self.b, self.r, self.d_rope = d, b, r, d_rope
        self.batch, self.max_tokens = batch, max_tokens
        self.lay = pkg.Layout([0, 0], [d, 0], [b, 0], r, d_rope, batch, max_tokens,
                              device=device)

    def write(self, c, kr, start=None):
        B = c.shape[0]
        if start is None:
            start = torch.zeros(B, dtype=torch.int32)
        self.lay.quant_write(0, c.cuda(), kr.cuda(), start.to(torch.int32).cuda())

    def close(self):
        self.lay.close()


def oracle_cache(oracle, c, kr, d, b):
    """Oracle quantisation of [B, T, r] / [B, T, dR] host tensors -> (codes, scales, rows)."""
    cn, kn = bf16_or_f32_to_np(c), bf16_or_f32_to_np(kr)
    out = []
    for i in range(cn.shape[0]):
        rows, s, k = oracle.quantize_rows(cn[i], kn[i], d, b)
        out.append((k, s, rows))
    return out


def oracle_decode(oracle, cache_i, ql, qr, d, sigma, tok=None):
    k, s, _ = cache_i
    return oracle.decode_sequence(np.asarray(ql, dtype=np.float64), np.asarray(qr, np.float64),
                                  k, s, d, sigma, tok)
