"""Quantise-on-write on the GPU vs the oracle: codes, scales and packed bytes bit-exact."""
import numpy as np
import pytest
import torch

from gpu_helpers import bf16_or_f32_to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkg():
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as p
    assert torch.cuda.is_available()
    return p


def _inputs(B, T, r, dR, dtype, seed, kind="mixed"):
    g = torch.Generator().manual_seed(seed)
    c = torch.randn(B, T, r, generator=g)
    kr = torch.randn(B, T, dR, generator=g)
    if kind == "mixed":
        c[:, 1::7] *= 1e-3
        c[:, 2::7] *= 300.0
        c[:, 3::7] = 0.0
        kr[:, 3::7] = 0.0                                  # all-zero token
        c[:, 4::7, 5] = 40.0                               # one dominant latent value
        kr[:, 5::7, 1] = -55.0                             # dominant rope value
        t3 = torch.randn(B, T, r, generator=g) / torch.sqrt(
            sum(torch.randn(B, T, r, generator=g) ** 2 for _ in range(3)) / 3)
        c[:, 6::7] = t3[:, 6::7]
    return c.to(dtype), kr.to(dtype)


def _check_against_oracle(oracle, lay, layer, c, kr, starts, n_new, d, b):
    codes, scales = lay.cache_views(layer)
    codes = codes.cpu().numpy()
    scales = scales.cpu().view(torch.int16).numpy().view(np.uint16)
    cn, kn = bf16_or_f32_to_np(c), bf16_or_f32_to_np(kr)
    for i in range(c.shape[0]):
        rows, s, _ = oracle.quantize_rows(cn[i, :n_new], kn[i, :n_new], d, b)
        p0 = int(starts[i])
        assert np.array_equal(scales[i, p0:p0 + n_new], s), f"seq {i} scales"
        got = codes[i, p0:p0 + n_new]
        if not np.array_equal(got, rows):
            bad = np.argwhere(got != rows)[:5]
            raise AssertionError(f"seq {i} codes differ at {bad.tolist()}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("b", [2, 4, 8, 16])
@pytest.mark.parametrize("d,r,dR", [(16, 64, 16), (32, 64, 16), (64, 64, 16), (128, 512, 64),
                                    (384, 512, 64), (512, 512, 64), (512, 1024, 0)])
def test_quant_write_bit_exact(pkg, oracle_mod, dtype, b, d, r, dR):
    B, T, n_new = 3, 80, 67
    lay = pkg.Layout([0, 0], [d, 0], [b, 0], r, dR, B, T)
    try:
        c, kr = _inputs(B, n_new, r, max(dR, 8), dtype, seed=d * 131 + b)
        kr = kr[:, :, :dR].contiguous() if dR else torch.zeros(B, n_new, 8, dtype=dtype)
        starts = torch.tensor([0, 5, 13], dtype=torch.int32)
        lay.quant_write(0, c.cuda(), kr.cuda(), starts.cuda())
        torch.cuda.synchronize()
        assert lay.read_status() == 0
        _check_against_oracle(oracle_mod, lay, 0, c, kr[:, :, :dR], starts, n_new, d, b)
    finally:
        lay.close()


def test_quant_write_strided_inputs_and_append(pkg, oracle_mod):
    B, T, r, dR, d, b = 2, 64, 128, 32, 96, 8
    lay = pkg.Layout([0], [d], [b], r, dR, B, T)
    try:
        big_c = torch.randn(B, 40, 2 * r).to(torch.bfloat16)          # strided view
        big_k = torch.randn(B, 40, 2 * dR).to(torch.bfloat16)
        c = big_c.cuda()[:, :, :r]
        kr = big_k.cuda()[:, :, dR:]
        lay.quant_write(0, c, kr, torch.zeros(B, dtype=torch.int32, device="cuda"))
        # append one token at position 40 for each sequence
        a_c = torch.randn(B, 1, r).to(torch.bfloat16)
        a_k = torch.randn(B, 1, dR).to(torch.bfloat16)
        lay.quant_write(0, a_c.cuda(), a_k.cuda(), torch.full((B,), 40, dtype=torch.int32,
                                                                device="cuda"))
        torch.cuda.synchronize()
        full_c = torch.cat([big_c[:, :, :r], a_c], 1)
        full_k = torch.cat([big_k[:, :, dR:], a_k], 1)
        _check_against_oracle(oracle_mod, lay, 0, full_c, full_k, [0, 0], 41, d, b)
    finally:
        lay.close()


def test_quant_write_exact_ties(pkg, oracle_mod):
    # s = 0.125 exactly at b = 8 (absmax 15.875); values on k + 1/2 go to the even code
    v = torch.zeros(1, 1, 64)
    v[0, 0, 0] = 15.875
    v[0, 0, 1:40] = (torch.arange(-20, 19).float() + 0.5) * 0.125
    lay = pkg.Layout([0], [48], [8], 64, 16, 1, 4)
    try:
        kr = torch.zeros(1, 1, 16)
        lay.quant_write(0, v.cuda(), kr.cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        _check_against_oracle(oracle_mod, lay, 0, v, kr, [0], 1, 48, 8)
        codes, scales = lay.cache_views(0)
        assert float(scales[0, 0].item()) == 0.125
    finally:
        lay.close()


def test_quant_write_flags(pkg):
    lay = pkg.Layout([0, 0], [32, 0], [8, 0], 64, 16, 2, 16)
    try:
        codes, scales = lay.cache_views(0)
        codes.fill_(0xAB)
        c = torch.randn(2, 3, 64, device="cuda")
        kr = torch.randn(2, 3, 16, device="cuda")
        # positions 14, 15, 16 for seq 0 (16 is out of range); -1.. for seq 1
        lay.quant_write(0, c, kr, torch.tensor([14, -1], dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        assert lay.read_status() & pkg.KVK_FLAG_WRITE_RANGE
        assert (codes[1, 2:] == 0xAB).all() and not (codes[1, 0:2] == 0xAB).all()
        assert (codes[0, :14] == 0xAB).all()
        lay.read_status(clear=True)
        assert lay.read_status() == 0
        c[0, 0, 0] = float("nan")
        lay.quant_write(0, c, kr, torch.zeros(2, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        assert lay.read_status() & pkg.KVK_FLAG_NONFINITE
        lay.read_status(clear=True)
        c[0, 0, 0] = 1e30                                   # scale beyond the fp16 range
        lay.quant_write(0, c, kr, torch.zeros(2, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        assert lay.read_status() & pkg.KVK_FLAG_NONFINITE
        with pytest.raises(pkg.KvkError) as e:
            lay.quant_write(1, c, kr, torch.zeros(2, dtype=torch.int32, device="cuda"))
        assert e.value.status == 4
    finally:
        lay.close()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quant_write_layers_matches_oracle(pkg, oracle_mod, dtype):
    """One launch over several anchor layers (different d, b, strided inputs) writes exactly
    what the oracle gives per layer, and leaves the other layers untouched."""
    B, T, n_new, r, dR = 4, 96, 3, 512, 64
    anchor = [0, 0, 2, 3, 3, 5]
    dd = [512, 0, 384, 128, 0, 256]
    bb = [16, 0, 8, 2, 0, 4]
    lay = pkg.Layout(anchor, dd, bb, r, dR, B, T)
    try:
        starts = torch.tensor([0, 17, 90, 45], dtype=torch.int32)
        layers = [5, 0, 3]      # any order, a subset of the anchors
        cs, ks = [], []
        for li, layer in enumerate(layers):
            c, kr = _inputs(B, n_new + 2, r, dR, dtype, seed=1000 + layer)
            cs.append(c.cuda()[:, 1:1 + n_new])          # strided: skips a token per sequence
            ks.append(kr.cuda()[:, 1:1 + n_new])
        codes2, scales2 = lay.cache_views(2)
        before = (codes2.clone(), scales2.clone())
        pkg.kvk.kvk_quant_write_layers(lay.handle, layers, cs, ks, starts.cuda())
        torch.cuda.synchronize()
        for layer, c, kr in zip(layers, cs, ks):
            _check_against_oracle(oracle_mod, lay, layer, c.cpu(), kr.cpu(), starts, n_new,
                                  dd[layer], bb[layer])
        # anchor 2 is not in the list: its planes are unchanged
        assert torch.equal(codes2, before[0]) and torch.equal(scales2.view(torch.int16),
                                                               before[1].view(torch.int16))
        assert lay.read_status() == 0
    finally:
        lay.close()


def test_quant_write_layers_arguments(pkg):
    lay = pkg.Layout([0, 0, 2], [64, 0, 64], [8, 0, 4], 64, 16, 2, 32)
    try:
        c = torch.zeros(2, 1, 64, dtype=torch.bfloat16, device="cuda")
        kr = torch.zeros(2, 1, 16, dtype=torch.bfloat16, device="cuda")
        pos = torch.zeros(2, dtype=torch.int32, device="cuda")
        for layers, status in (([0, 0], 1), ([1], 4), ([0, 7], 1)):
            with pytest.raises(pkg.kvk.KvkError) as e:
                pkg.kvk.kvk_quant_write_layers(lay.handle, layers, [c] * len(layers),
                                               [kr] * len(layers), pos)
            assert e.value.status == status, (layers, e.value.status)
    finally:
        lay.close()
