"""GPU test of kvk_mla_decode_noalloc, the decode entry point for callers that cannot
allocate device memory (for instance a host application that owns the whole device memory
budget and gives a plugin only its input and output buffers).

The entry point takes its scratch space from an array built into the library instead of a
caller-provided workspace.  This test calls it through the C ABI twice in a row, with
different queries, and checks each result against the regular kvk_mla_decode (which uses
a workspace tensor) within the tolerance the other decode tests use.  The second call runs
on scratch that still holds the first call's contents.  The file is named so that pytest
collects it last; it builds everything it needs, so it also passes alone in a fresh process.
"""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("qdtype,d,b,H,B,lens", [
    (torch.bfloat16, 512, 16, 40, 4, [2048, 1500, 1, 777]),
    (torch.float32, 64, 4, 8, 2, [256, 100]),
])
def test_noalloc_decode_matches_workspace_decode(qdtype, d, b, H, B, lens):
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as pkg

    assert torch.cuda.is_available()
    r, dR, T = max(d, 64), 64 if d >= 128 else 16, max(lens)
    lay = pkg.Layout([0, 0], [d, 0], [b, 0], r, dR, B, T)
    try:
        g = torch.Generator().manual_seed(1234 + d)
        c = torch.randn(B, T, r, generator=g).to(torch.bfloat16).cuda()
        kr = torch.randn(B, T, dR, generator=g).to(torch.bfloat16).cuda()
        lay.quant_write(0, c, kr, torch.zeros(B, dtype=torch.int32, device="cuda"))
        seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
        sigma = 1 / math.sqrt(d + dR)
        assert lay.workspace_bytes(1, B, H) <= pkg.kvk.KVK_NOALLOC_SCRATCH_BYTES
        for call in range(2):                      # two calls in a row on the shared scratch
            ql = torch.randn(B, H, r, generator=g).to(qdtype).cuda()
            qr = torch.randn(B, H, dR, generator=g).to(qdtype).cuda()
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


def test_noalloc_rejects_workspace_beyond_scratch():
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as pkg

    # 256 sequences x 64 heads x d = 512 needs more than the built-in scratch
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
