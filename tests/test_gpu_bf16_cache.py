"""The uncompressed bf16 anchor (b = KVK_BITS_BF16): the MLA cache the compressed choices are
measured against, written and decoded through the same layout, kernels and entry points.

Writes are bit-exact against the oracle's round-to-nearest-even bfloat16 rows (scale plane
1.0); decode matches the oracle's attention over those rows within the north-star
tolerance, on both decode kernels, including long sequences on few CTAs, keep lists and a
layer that inherits the uncompressed anchor."""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import bf16_or_f32_to_np, check_outputs

pytestmark = pytest.mark.gpu

BF16 = 0   # KVK_BITS_BF16


@pytest.fixture(scope="module")
def pkg():
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as p
    assert torch.cuda.is_available()
    return p


def _paths(pkg, lay, dtype, H, has_keep=False):
    ps = [pkg.KVK_PATH_CUDA_CORE]
    lay.set_decode_path(pkg.KVK_PATH_TENSOR)
    try:
        if lay.decode_path_for(0, dtype, H, has_keep) == pkg.KVK_PATH_TENSOR:
            # the token-scale tensor-core kernel, and the general one forced
            ps += [pkg.KVK_PATH_TENSOR, pkg.KVK_PATH_TENSOR_GENERAL]
    except pkg.KvkError:
        pass
    finally:
        lay.set_decode_path(pkg.KVK_PATH_AUTO)
    return ps


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d,r,dR", [(32, 64, 16), (128, 512, 64), (512, 512, 64)])
def test_bf16_anchor_write_bit_exact(pkg, oracle_mod, dtype, d, r, dR):
    B, T, n_new = 3, 70, 61
    lay = pkg.Layout([0, 0], [d, 0], [BF16, 0], r, dR, B, T)
    try:
        assert lay.bits_per_token == (d + dR) * 16
        g = torch.Generator().manual_seed(d + dR)
        c = (torch.randn(B, n_new, r, generator=g) * 3).to(dtype)
        kr = torch.randn(B, n_new, dR, generator=g).to(dtype)
        c[:, 5::9] *= 1e-30                     # tiny values stay exact in bf16
        starts = torch.tensor([0, 4, 9], dtype=torch.int32)
        lay.quant_write(0, c.cuda(), kr.cuda(), starts.cuda())
        torch.cuda.synchronize()
        assert lay.read_status() == 0
        codes, scales = lay.cache_views(0)
        codes = codes.cpu().numpy()
        scales = scales.cpu().view(torch.int16).numpy().view(np.uint16)
        info = lay.layer_info(0)
        assert info["row_bytes"] == ((d + dR) * 2 + 15) // 16 * 16
        for i in range(B):
            bits, _ = oracle_mod.bf16_rows(bf16_or_f32_to_np(c[i]), bf16_or_f32_to_np(kr[i]), d)
            want = np.zeros((n_new, info["row_bytes"]), dtype=np.uint8)
            want[:, :2 * (d + dR)] = bits.view(np.uint8).reshape(n_new, -1)
            p0 = int(starts[i])
            assert np.array_equal(codes[i, p0:p0 + n_new], want), f"seq {i}"
            assert np.all(scales[i, p0:p0 + n_new] == 0x3C00)
    finally:
        lay.close()


SHAPES = [  # d, r, dR, H, lens, max_tokens
    (64, 64, 16, 8, [256, 1, 97], 260),
    (128, 512, 64, 28, [300, 64, 129], 300),
    (512, 512, 64, 40, [1000, 777], 1000),
    (512, 512, 64, 40, [8192, 4133, 4100], 8192),   # many tiles per CTA with few CTAs
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"d{s[0]}H{s[3]}T{max(s[4])}")
def test_bf16_anchor_decode_matches_oracle(pkg, oracle_mod, shape):
    d, r, dR, H, lens, T = shape
    B = len(lens)
    g = torch.Generator().manual_seed(d * 3 + H + T)
    c = torch.randn(B, T, r, generator=g).to(torch.bfloat16)
    kr = torch.randn(B, T, dR, generator=g).to(torch.bfloat16)
    ql = torch.randn(B, H, r, generator=g).to(torch.bfloat16)
    qr = torch.randn(B, H, dR, generator=g).to(torch.bfloat16)
    sigma = 1 / math.sqrt(d + dR)
    refs = []
    for i in range(B):
        _, vals = oracle_mod.bf16_rows(bf16_or_f32_to_np(c[i, :lens[i]]),
                                       bf16_or_f32_to_np(kr[i, :lens[i]]), d)
        refs.append(oracle_mod.decode_sequence_bf16(bf16_or_f32_to_np(ql[i]),
                                                    bf16_or_f32_to_np(qr[i]), vals, d, sigma))
    lay = pkg.Layout([0, 0], [d, 0], [BF16, 0], r, dR, B, T)
    try:
        lay.quant_write(0, c.cuda(), kr.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
        lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
        for path in _paths(pkg, lay, torch.bfloat16, H):
            lay.set_decode_path(path)
            for ctas in ((0,) if path == pkg.KVK_PATH_CUDA_CORE else (0, 1, 7)):
                lay.set_decode_ctas(ctas)
                lse = torch.empty(B, H, device="cuda")
                out = lay.mla_decode(1, ql.cuda(), qr.cuda(), lens_t, sigma, lse=lse)
                torch.cuda.synchronize()
                for i in range(B):
                    check_outputs(out[i].cpu().numpy(), lse[i].cpu().numpy(), refs[i][0],
                                  refs[i][1], f"path {path} ctas {ctas} seq {i}")
        lay.set_decode_ctas(0)
        assert lay.read_status() == 0
    finally:
        lay.close()


def test_bf16_anchor_keep_list(pkg, oracle_mod):
    d, r, dR, H, B, T, K = 512, 512, 64, 40, 3, 2000, 300
    g = torch.Generator().manual_seed(5)
    c = torch.randn(B, T, r, generator=g).to(torch.bfloat16)
    kr = torch.randn(B, T, dR, generator=g).to(torch.bfloat16)
    ql = torch.randn(B, H, r, generator=g).to(torch.bfloat16)
    qr = torch.randn(B, H, dR, generator=g).to(torch.bfloat16)
    lens = [2000, 1500, 200]
    klen = [300, 123, 200]
    rng = np.random.default_rng(8)
    keep = np.zeros((B, K), dtype=np.int32)
    for i in range(B):
        keep[i, :klen[i]] = np.sort(rng.choice(lens[i], klen[i], replace=False))
    sigma = 1 / math.sqrt(d + dR)
    lay = pkg.Layout([0], [d], [BF16], r, dR, B, T)
    try:
        lay.quant_write(0, c.cuda(), kr.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
        for path in _paths(pkg, lay, torch.bfloat16, H, has_keep=True):
            lay.set_decode_path(path)
            lse = torch.empty(B, H, device="cuda")
            out = lay.mla_decode(0, ql.cuda(), qr.cuda(),
                                 torch.tensor(lens, dtype=torch.int32, device="cuda"), sigma,
                                 lse=lse, keep_idx=torch.from_numpy(keep).cuda(),
                                 keep_len=torch.tensor(klen, dtype=torch.int32, device="cuda"))
            torch.cuda.synchronize()
            for i in range(B):
                _, vals = oracle_mod.bf16_rows(bf16_or_f32_to_np(c[i]), bf16_or_f32_to_np(kr[i]), d)
                o_ref, l_ref = oracle_mod.decode_sequence_bf16(
                    bf16_or_f32_to_np(ql[i]), bf16_or_f32_to_np(qr[i]), vals, d, sigma,
                    tok=keep[i, :klen[i]])
                check_outputs(out[i].cpu().numpy(), lse[i].cpu().numpy(), o_ref, l_ref,
                              f"keep path {path} seq {i}")
        assert lay.read_status() == 0
    finally:
        lay.close()
