"""The absorbed MLA projections on the tensor cores (kvk_absorb) against the oracle's binary64
product: the query side (bf16 q_nope, W_UK truncated to the layer's first d latent columns,
bf16 q_lat) and the output side (fp32 decode output, W_UV truncated to the first d rows, fp32
values), at the 14B shape and at small ragged shapes.

Tolerance from the arithmetic: bf16 inputs give exact products and fp32 accumulation
(relative error about K * 2^-24); a bf16 result adds its rounding (2^-9 relative); an fp32 x
enters as two bf16 parts (about 2^-17 relative per element).  So per (b, h):
max|y - y_ref| <= 2^-8 * max|y_ref| for bf16 results and 1e-4 * max|y_ref| for fp32 ones."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkg():
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as p
    assert torch.cuda.is_available()
    return p


def _check(y, y_ref, tol, what):
    y = y.double().cpu().numpy()
    err = np.abs(y - y_ref).max(axis=2)
    ref = np.abs(y_ref).max(axis=2)
    bad = err > tol * ref
    assert not bad.any(), f"{what}: rel err {(err / np.maximum(ref, 1e-300)).max():.3e}"
    return (err / np.maximum(ref, 1e-300)).max()


@pytest.mark.parametrize("B,H,dh,d,r", [(32, 40, 128, 512, 512), (32, 40, 128, 384, 512),
                                         (8, 28, 128, 128, 512), (3, 5, 64, 48, 64),
                                         (45, 2, 128, 256, 512)])
def test_query_absorption(pkg, oracle_mod, B, H, dh, d, r):
    g = torch.Generator().manual_seed(B + H + d)
    q_nope = torch.randn(B, H, dh, generator=g).to(torch.bfloat16)
    w_uk = (torch.randn(H, dh, r, generator=g) / dh ** 0.5).to(torch.bfloat16)
    q_lat = torch.full((B, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    # only the first d latent columns the layer keeps: w viewed [H, dh, d] with row stride r
    pkg.kvk_absorb(q_nope.cuda(), w_uk.cuda()[:, :, :d], q_lat)
    torch.cuda.synchronize()
    ref = oracle_mod.absorb(q_nope.float().numpy(), w_uk.float().numpy()[:, :, :d])
    _check(q_lat, ref, 2.0 ** -8, f"q_lat B={B} H={H} d={d}")


@pytest.mark.parametrize("B,H,d,dv", [(32, 40, 512, 128), (32, 40, 384, 128), (8, 28, 128, 128),
                                       (33, 3, 64, 16)])
def test_output_absorption(pkg, oracle_mod, B, H, d, dv):
    g = torch.Generator().manual_seed(7 * B + H + d)
    out_lat = torch.randn(B, H, d, generator=g)                 # fp32, as the decode writes it
    out_lat[:, :, 1::7] *= 1e-3                                  # mixed magnitudes
    w_uv = (torch.randn(H, 512, dv, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    y = torch.full((B, H, dv), float("nan"), device="cuda")
    pkg.kvk_absorb(out_lat.cuda(), w_uv.cuda()[:, :d, :], y)    # the first d rows of W_UV
    torch.cuda.synchronize()
    ref = oracle_mod.absorb(out_lat.numpy(), w_uv.float().numpy()[:, :d, :])
    _check(y, ref, 1e-4, f"values B={B} H={H} d={d}")


def test_absorption_argument_errors(pkg):
    x = torch.zeros(2, 3, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(3, 64, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(2, 3, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pkg.KvkError) as e:        # K not a multiple of 64
        pkg.kvk_absorb(x[:, :, :48], w, y)
    assert e.value.status == 1
    with pytest.raises(pkg.KvkError) as e:        # misaligned y
        buf = torch.zeros(2 * 3 * 64 + 8, dtype=torch.bfloat16, device="cuda")
        pkg.kvk_absorb(x, w, buf[1:1 + 2 * 3 * 64].view(2, 3, 64))
    assert e.value.status == 6
