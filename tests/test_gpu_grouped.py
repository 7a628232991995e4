"""Group-scaled caches (kvk_create_layout_grouped): one fp16 scale per G consecutive elements
of [c[:d] || k^R] instead of one per token -- the 4.5-bit cache (b = 4, G = 32) behind the
152x composition of the M3 Ultra benchmark, and a KIVI-style comparison point.

Inputs follow the workloads' latent distributions (per-channel std U(0.5, 2), Student-t(3)).
Writes are bit-exact against the oracle's grouped quantiser (codes, every group scale, row
bytes); decode matches the oracle's attention over the group-dequantised rows on both
kernels (the tensor-core kernel applies the scales while unpacking b <= 8 codes; 16-bit
codes take the CUDA-core kernel), over many tiles per CTA, with keep lists and with the
fused append."""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import bf16_or_f32_to_np, check_outputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkg():
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as p
    assert torch.cuda.is_available()
    return p


def _paths(pkg, lay, H, has_keep=False):
    ps = [pkg.KVK_PATH_CUDA_CORE]
    lay.set_decode_path(pkg.KVK_PATH_TENSOR)
    try:
        if lay.decode_path_for(0, torch.bfloat16, H, has_keep) == pkg.KVK_PATH_TENSOR:
            ps.append(pkg.KVK_PATH_TENSOR)
    except pkg.KvkError:
        pass
    finally:
        lay.set_decode_path(pkg.KVK_PATH_AUTO)
    return ps


def _heavy(B, T, r, g):
    """Latents drawn as the workloads draw them, so that groups differ in scale: per-channel
    std U(0.5, 2) (the 14B workloads) for half the tokens, Student-t(3) (the budget sweep) for
    the other half."""
    std = torch.empty(r).uniform_(0.5, 2.0, generator=g)
    c = torch.randn(B, T, r, generator=g) * std
    t3 = torch.randn(B, T, r, generator=g) / torch.sqrt(
        sum(torch.randn(B, T, r, generator=g) ** 2 for _ in range(3)) / 3)
    c[:, 1::2] = t3[:, 1::2]
    return c


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("b", [2, 4, 8, 16])
@pytest.mark.parametrize("d,r,dR,G", [(32, 64, 16, 16), (128, 512, 64, 32), (512, 512, 64, 32),
                                      (512, 512, 64, 64)])
def test_grouped_write_bit_exact(pkg, oracle_mod, dtype, b, d, r, dR, G):
    B, T, n_new = 3, 70, 61
    lay = pkg.Layout([0, 0], [d, 0], [b, 0], r, dR, B, T, scale_group=G)
    try:
        n = d + dR
        assert lay.bits_per_token == n * b + 16 * (n // G)
        assert lay.bits_per_token == oracle_mod.bits_per_token_grouped([0, 0], [d, 0], [b, 0],
                                                                       dR, G)
        g = torch.Generator().manual_seed(b * 7 + d + G)
        c = _heavy(B, n_new, r, g).to(dtype)
        kr = torch.randn(B, n_new, dR, generator=g).to(dtype)
        c[:, 3, :] = 0.0
        kr[:, 3, :] = 0.0                   # an all-zero token: every group scale 0
        starts = torch.tensor([0, 4, 9], dtype=torch.int32)
        lay.quant_write(0, c.cuda(), kr.cuda(), starts.cuda())
        torch.cuda.synchronize()
        assert lay.read_status() == 0
        codes, scales = lay.cache_views(0)
        codes = codes.cpu().numpy()
        scales = scales.cpu().view(torch.int16).numpy().view(np.uint16)
        assert scales.shape[-1] == n // G
        for i in range(B):
            rows, s, _ = oracle_mod.quantize_rows_grouped(bf16_or_f32_to_np(c[i]),
                                                          bf16_or_f32_to_np(kr[i]), d, b, G)
            p0 = int(starts[i])
            assert np.array_equal(scales[i, p0:p0 + n_new], s), f"seq {i} scales"
            assert np.array_equal(codes[i, p0:p0 + n_new], rows), f"seq {i} codes"
    finally:
        lay.close()


CASES = [  # d, r, dR, H, G, lens, max_tokens
    (32, 64, 16, 8, 16, [256, 1, 97], 260),
    (128, 512, 64, 28, 32, [300, 64, 129], 300),
    (512, 512, 64, 40, 32, [1000, 777], 1000),
    (512, 512, 64, 40, 64, [8192, 4133, 4100], 8192),   # many tiles per CTA with few CTAs
]


@pytest.mark.parametrize("b", [2, 4, 8, 16])
@pytest.mark.parametrize("case", CASES, ids=lambda s: f"d{s[0]}G{s[4]}T{max(s[5])}")
def test_grouped_decode_matches_oracle(pkg, oracle_mod, b, case):
    d, r, dR, H, G, lens, T = case
    B = len(lens)
    g = torch.Generator().manual_seed(d + b + G + T)
    c = _heavy(B, T, r, g).to(torch.bfloat16)
    kr = torch.randn(B, T, dR, generator=g).to(torch.bfloat16)
    ql = torch.randn(B, H, r, generator=g).to(torch.bfloat16)
    qr = torch.randn(B, H, dR, generator=g).to(torch.bfloat16)
    sigma = 1 / math.sqrt(d + dR)
    refs = []
    for i in range(B):
        _, s, k = oracle_mod.quantize_rows_grouped(bf16_or_f32_to_np(c[i, :lens[i]]),
                                                   bf16_or_f32_to_np(kr[i, :lens[i]]), d, b, G)
        refs.append(oracle_mod.decode_sequence_grouped(bf16_or_f32_to_np(ql[i]),
                                                       bf16_or_f32_to_np(qr[i]), k, s, d, sigma))
    lay = pkg.Layout([0, 0], [d, 0], [b, 0], r, dR, B, T, scale_group=G)
    try:
        lay.quant_write(0, c.cuda(), kr.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
        lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
        paths = _paths(pkg, lay, H)
        if b < 16 and d >= 128:
            assert pkg.KVK_PATH_TENSOR in paths   # the tensor-core kernel takes b <= 8 groups
        for path in paths:
            lay.set_decode_path(path)
            for ctas in ((0,) if path == pkg.KVK_PATH_CUDA_CORE else (0, 3)):
                lay.set_decode_ctas(ctas)
                lse = torch.empty(B, H, device="cuda")
                out = lay.mla_decode(1, ql.cuda(), qr.cuda(), lens_t, sigma, lse=lse)
                torch.cuda.synchronize()
                for i in range(B):
                    check_outputs(out[i].cpu().numpy(), lse[i].cpu().numpy(), refs[i][0],
                                  refs[i][1], f"b={b} G={G} path {path} ctas {ctas} seq {i}")
        lay.set_decode_ctas(0)
        assert lay.read_status() == 0
    finally:
        lay.close()


def test_grouped_keep_list_and_append(pkg, oracle_mod):
    d, r, dR, H, G, b, B, T, K = 512, 512, 64, 40, 32, 4, 3, 2000, 300
    g = torch.Generator().manual_seed(17)
    c = _heavy(B, T, r, g).to(torch.bfloat16)
    kr = torch.randn(B, T, dR, generator=g).to(torch.bfloat16)
    ql = torch.randn(B, H, r, generator=g).to(torch.bfloat16)
    qr = torch.randn(B, H, dR, generator=g).to(torch.bfloat16)
    c_new = torch.randn(B, r, generator=g).to(torch.bfloat16)
    kr_new = torch.randn(B, dR, generator=g).to(torch.bfloat16)
    lens = [2000, 1500, 200]
    klen = [300, 123, 200]
    rng = np.random.default_rng(9)
    keep = np.zeros((B, K), dtype=np.int32)
    for i in range(B):
        keep[i, :klen[i]] = np.sort(rng.choice(lens[i], klen[i], replace=False))
    sigma = 1 / math.sqrt(d + dR)
    lay = pkg.Layout([0], [d], [b], r, dR, B, T, scale_group=G)
    try:
        lay.quant_write(0, c.cuda(), kr.cuda(), torch.zeros(B, dtype=torch.int32, device="cuda"))
        lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
        # keep lists: the tensor-core kernel copies the kept rows and their group scales
        for path in _paths(pkg, lay, H, has_keep=True):
            lay.set_decode_path(path)
            lse = torch.empty(B, H, device="cuda")
            out = lay.mla_decode(0, ql.cuda(), qr.cuda(), lens_t, sigma, lse=lse,
                                 keep_idx=torch.from_numpy(keep).cuda(),
                                 keep_len=torch.tensor(klen, dtype=torch.int32, device="cuda"))
            torch.cuda.synchronize()
            for i in range(B):
                _, s, k = oracle_mod.quantize_rows_grouped(bf16_or_f32_to_np(c[i]),
                                                           bf16_or_f32_to_np(kr[i]), d, b, G)
                o_ref, l_ref = oracle_mod.decode_sequence_grouped(
                    bf16_or_f32_to_np(ql[i]), bf16_or_f32_to_np(qr[i]), k, s, d, sigma,
                    tok=keep[i, :klen[i]])
                check_outputs(out[i].cpu().numpy(), lse[i].cpu().numpy(), o_ref, l_ref,
                              f"keep path {path} seq {i}")
        # fused append: the new token's groups written at len - 1, then decoded
        lay.set_decode_path(pkg.KVK_PATH_AUTO)
        lse = torch.empty(B, H, device="cuda")
        out = lay.mla_decode_append(0, c_new.cuda(), kr_new.cuda(), ql.cuda(), qr.cuda(), lens_t,
                                    sigma, lse=lse)
        torch.cuda.synchronize()
        codes, scales = lay.cache_views(0)
        codes, scales = codes.cpu().numpy(), scales.cpu().view(torch.int16).numpy().view(np.uint16)
        for i, n in enumerate(lens):
            full_c, full_k = c[i, :n].clone(), kr[i, :n].clone()
            full_c[n - 1], full_k[n - 1] = c_new[i], kr_new[i]
            rows, s, k = oracle_mod.quantize_rows_grouped(bf16_or_f32_to_np(full_c),
                                                          bf16_or_f32_to_np(full_k), d, b, G)
            assert np.array_equal(codes[i, n - 1], rows[n - 1])
            assert np.array_equal(scales[i, n - 1], s[n - 1])
            o_ref, l_ref = oracle_mod.decode_sequence_grouped(
                bf16_or_f32_to_np(ql[i]), bf16_or_f32_to_np(qr[i]), k, s, d, sigma)
            check_outputs(out[i].cpu().numpy(), lse[i].cpu().numpy(), o_ref, l_ref,
                          f"append seq {i}")
        assert lay.read_status() == 0
    finally:
        lay.close()
