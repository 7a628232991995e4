"""GPU test of kvk_mla_decode_noalloc, the decode entry point for callers that cannot
allocate device memory (for instance a host application that owns the whole device memory
budget and gives a plugin only its input and output buffers).

The entry point takes its scratch space from an array built into the library instead of a
caller-provided workspace.  These tests call it through the C ABI twice in a row, with
different queries (and keep lists), and check each result against the regular
kvk_mla_decode (which uses a workspace tensor) within the tolerance the other decode tests
use.  The second call runs on scratch that still holds the first call's contents.  The
file is named so that pytest collects it last; it builds everything it needs, so it also
passes alone in a fresh process.
"""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import rel_err

pytestmark = pytest.mark.gpu


def _pkg():
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as pkg
    assert torch.cuda.is_available()
    return pkg


@pytest.mark.parametrize("qdtype,d,b,H,B,lens", [
    (torch.bfloat16, 512, 16, 40, 4, [2048, 1500, 1, 777]),
    (torch.float32, 64, 4, 8, 2, [256, 100]),
    # one layer of the 14B benchmark shape: the tensor-core kernel's workspace (~15 MB) fits
    # the built-in scratch, although the size that covers both kernels does not
    (torch.bfloat16, 512, 16, 40, 32, [8192] * 32),
], ids=["d512", "f32", "bench_shape"])
def test_noalloc_decode_matches_workspace_decode(qdtype, d, b, H, B, lens):
    pkg = _pkg()
    r, dR, T = max(d, 64), 64 if d >= 128 else 16, max(lens)
    lay = pkg.Layout([0, 0], [d, 0], [b, 0], r, dR, B, T)
    try:
        g = torch.Generator(device="cuda").manual_seed(1234 + d + B)
        c = torch.randn(B, T, r, generator=g, device="cuda").to(torch.bfloat16)
        kr = torch.randn(B, T, dR, generator=g, device="cuda").to(torch.bfloat16)
        lay.quant_write(0, c, kr, torch.zeros(B, dtype=torch.int32, device="cuda"))
        del c, kr
        seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
        sigma = 1 / math.sqrt(d + dR)
        for call in range(2):                      # two calls in a row on the shared scratch
            ql = torch.randn(B, H, r, generator=g, device="cuda").to(qdtype)
            qr = torch.randn(B, H, dR, generator=g, device="cuda").to(qdtype)
            lse_ref = torch.empty(B, H, device="cuda")
            ref = lay.mla_decode(1, ql, qr, seq_lens, sigma, lse=lse_ref)
            out = torch.full((B, H, d), float("nan"), device="cuda")
            lse = torch.full((B, H), float("nan"), device="cuda")
            pkg.kvk_mla_decode_noalloc(lay.handle, 1, ql, qr, seq_lens, sigma, out, lse=lse)
            torch.cuda.synchronize()
            o, o_ref = out.cpu().numpy(), ref.cpu().numpy()
            for i in range(B):
                assert rel_err(o[i], o_ref[i]) <= 2e-3, (call, i)
            assert np.abs(lse.cpu().numpy() - lse_ref.cpu().numpy()).max() <= 2e-3
        assert lay.read_status() == 0
    finally:
        lay.close()


def test_noalloc_keep_lists_two_calls():
    """Keep lists through the built-in scratch: two calls in a row with lists of different
    lengths (some entries invalid, fewer valid entries than the row stride), each compared
    with kvk_mla_decode on a workspace of the size that lets the tensor-core kernel gather
    the kept rows.  The second call reads scratch holding the first call's dense copy."""
    pkg = _pkg()
    d, b, r, dR, H, B, T, K = 512, 8, 512, 64, 40, 6, 3000, 700
    lay = pkg.Layout([0], [d], [b], r, dR, B, T)
    try:
        keep_ws = lay.workspace_bytes(0, B, H, keep_stride=K)
        # this shape's dense copy fits the scratch, so the call takes the tensor-core kernel
        assert keep_ws <= pkg.kvk.KVK_NOALLOC_SCRATCH_BYTES
        assert lay.decode_path_for(0, torch.bfloat16, H, has_keep=True) == pkg.KVK_PATH_TENSOR
        g = torch.Generator().manual_seed(77)
        c = torch.randn(B, T, r, generator=g).to(torch.bfloat16).cuda()
        kr = torch.randn(B, T, dR, generator=g).to(torch.bfloat16).cuda()
        lay.quant_write(0, c, kr, torch.zeros(B, dtype=torch.int32, device="cuda"))
        lens = torch.tensor([3000, 2500, 100, 3000, 1, 640], dtype=torch.int32)
        rng = np.random.default_rng(3)
        sigma = 1 / math.sqrt(d + dR)
        for call, klen in enumerate(([700, 300, 100, 650, 1, 9], [40, 700, 64, 0, 1, 333])):
            keep = np.zeros((B, K), dtype=np.int32)
            for i in range(B):
                n = min(klen[i], int(lens[i]))
                keep[i, :n] = np.sort(rng.choice(int(lens[i]), n, replace=False))
            keep[0, 3] = 3001        # beyond seq_len: skipped and flagged
            keep[1, 10] = -5         # negative: skipped and flagged
            keep_t = torch.from_numpy(keep).cuda()
            klen_t = torch.tensor(klen, dtype=torch.int32, device="cuda")
            ql = torch.randn(B, H, r, generator=g).to(torch.bfloat16).cuda()
            qr = torch.randn(B, H, dR, generator=g).to(torch.bfloat16).cuda()
            ws = torch.empty(keep_ws, dtype=torch.uint8, device="cuda")
            lse_ref = torch.empty(B, H, device="cuda")
            ref = lay.mla_decode(0, ql, qr, lens.cuda(), sigma, lse=lse_ref, workspace=ws,
                                 keep_idx=keep_t, keep_len=klen_t)
            out = torch.full((B, H, d), float("nan"), device="cuda")
            lse = torch.full((B, H), float("nan"), device="cuda")
            pkg.kvk_mla_decode_noalloc(lay.handle, 0, ql, qr, lens.cuda(), sigma, out, lse=lse,
                                       keep_idx=keep_t, keep_len=klen_t)
            torch.cuda.synchronize()
            o, o_ref = out.cpu().numpy(), ref.cpu().numpy()
            for i in range(B):
                if klen[i] == 0:
                    assert not o[i].any() and np.all(np.isneginf(lse[i].cpu().numpy()))
                else:
                    assert rel_err(o[i], o_ref[i]) <= 2e-3, (call, i)
            fin = np.isfinite(lse_ref.cpu().numpy())
            assert np.array_equal(np.isfinite(lse.cpu().numpy()), fin)
            assert np.abs(lse.cpu().numpy()[fin] - lse_ref.cpu().numpy()[fin]).max() <= 2e-3
            assert lay.read_status(clear=True) == pkg.KVK_FLAG_KEEP_INDEX
    finally:
        lay.close()


def test_noalloc_rejects_workspace_beyond_scratch():
    pkg = _pkg()
    # 256 sequences x 64 heads x d = 512 needs more than the built-in scratch on either kernel
    lay = pkg.Layout([0], [512], [16], 512, 64, 256, 64)
    try:
        B, H = 256, 64
        assert lay.workspace_bytes(0, B, H) > pkg.kvk.KVK_NOALLOC_SCRATCH_BYTES
        ql = torch.zeros(B, H, 512, dtype=torch.bfloat16, device="cuda")
        qr = torch.zeros(B, H, 64, dtype=torch.bfloat16, device="cuda")
        out = torch.zeros(B, H, 512, device="cuda")
        with pytest.raises(pkg.KvkError) as e:
            pkg.kvk_mla_decode_noalloc(lay.handle, 0, ql, qr,
                                       torch.ones(B, dtype=torch.int32, device="cuda"), 1.0, out)
        assert e.value.status == 5
    finally:
        lay.close()


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs two GPUs")
def test_calls_with_another_device_current_are_refused():
    pkg = _pkg()
    lay = pkg.Layout([0], [64], [8], 64, 16, 2, 64, device="cuda:0")
    try:
        ql = torch.zeros(2, 4, 64, dtype=torch.bfloat16, device="cuda:0")
        qr = torch.zeros(2, 4, 16, dtype=torch.bfloat16, device="cuda:0")
        out = torch.zeros(2, 4, 64, device="cuda:0")
        lens = torch.ones(2, dtype=torch.int32, device="cuda:0")
        with torch.cuda.device(1):
            with pytest.raises(pkg.KvkError) as e:
                pkg.kvk_mla_decode_noalloc(lay.handle, 0, ql, qr, lens, 1.0, out)
            assert e.value.status == 1
            with pytest.raises(pkg.KvkError) as e:
                pkg.kvk_mla_decode(lay.handle, 0, ql, qr, lens, 1.0, out,
                                   torch.empty(1 << 20, dtype=torch.uint8, device="cuda:0"))
            assert e.value.status == 1
    finally:
        lay.close()
