"""Failure detection of the tensor-core decode, exercised without faulting the GPU: every wait
inside the kernel gives up after a time limit (kvk_set_wait_limit).  A limit of a few hundred
nanoseconds makes the first slow wait (the query staging, the first tiles' loads) run out, so
the kernel takes its stopping path: it records KVK_FLAG_TIMEOUT, lets its own loads and MMAs
finish, frees its tensor memory and returns.  The context stays usable: with the default
limit restored, the next decode on the same stream matches the oracle again."""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import bf16_or_f32_to_np, check_outputs, oracle_cache, oracle_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkg():
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as p
    assert torch.cuda.is_available()
    return p


@pytest.mark.parametrize("b", [16, 8])
def test_wait_limit_expiry_sets_flag_and_recovers(pkg, oracle_mod, b):
    d, r, dR, H, B, T = 512, 512, 64, 40, 4, 4096
    g = torch.Generator().manual_seed(90 + b)
    c = torch.randn(B, T, r, generator=g).to(torch.bfloat16)
    kr = torch.randn(B, T, dR, generator=g).to(torch.bfloat16)
    ql = torch.randn(B, H, r, generator=g).to(torch.bfloat16)
    qr = torch.randn(B, H, dR, generator=g).to(torch.bfloat16)
    sigma = 1 / math.sqrt(d + dR)
    lay = pkg.Layout([0], [d], [b], r, dR, B, T)
    try:
        lay.quant_write(0, c.cuda(), kr.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
        lay.set_decode_path(pkg.KVK_PATH_TENSOR)
        lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
        assert lay.read_status(clear=True) == 0
        lay.set_wait_limit(200)          # 200 ns: some wait is bound to run out
        for _ in range(2):
            lay.mla_decode(0, ql.cuda(), qr.cuda(), lens, sigma)
            torch.cuda.synchronize()     # the kernel returned
            assert lay.read_status(clear=True) & pkg.kvk.KVK_FLAG_TIMEOUT
        lay.set_wait_limit(0)            # the default limit again
        lse = torch.empty(B, H, device="cuda")
        out = lay.mla_decode(0, ql.cuda(), qr.cuda(), lens, sigma, lse=lse)
        torch.cuda.synchronize()
        assert lay.read_status() == 0
        ref = oracle_cache(oracle_mod, c, kr, d, b)
        for i in (0, B - 1):
            o_ref, l_ref = oracle_decode(oracle_mod, ref[i], bf16_or_f32_to_np(ql[i]),
                                         bf16_or_f32_to_np(qr[i]), d, sigma)
            check_outputs(out[i].cpu().numpy(), lse[i].cpu().numpy(), o_ref, l_ref,
                          f"after a timed-out call, b={b} seq {i}")
    finally:
        lay.close()
