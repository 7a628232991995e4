"""Fused append + decode (kvk_mla_decode_append): the new token of each sequence is quantised
and stored at position seq_len - 1, and the decode attends over the cache that includes it,
in one launch on the tensor-core kernel.

Checks: the appended rows and scales are bit-exact against the oracle's quantisation of the
new tokens; the outputs are bit-identical to a separate kvk_quant_write followed by
kvk_mla_decode (the same cache bytes through the same kernel); and they match the oracle's
decode of the whole sequence within the benchmark spec's tolerance.  Both decode kernels, every
bit width and the uncompressed anchor, ragged lengths including 0 (nothing appended) and 1
(the new token alone)."""
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


def _oracle_rows(oracle, c, kr, d, b):
    """(row bytes [T, row_bytes], scale bits [T], dequantised rows float64 [T, n])."""
    if b == 0:
        bits, vals = oracle.bf16_rows(c, kr, d)
        return bits.view(np.uint8).reshape(bits.shape[0], -1), \
            np.full(bits.shape[0], 0x3C00, dtype=np.uint16), vals
    rows, s, k = oracle.quantize_rows(c, kr, d, b)
    return rows, s, oracle.dequant(k, s)


@pytest.mark.parametrize("b", [16, 8, 4, 2, 0])
@pytest.mark.parametrize("qdtype", [torch.bfloat16, torch.float32])
def test_append_decode(pkg, oracle_mod, b, qdtype):
    d, r, dR, H, T = 512, 512, 64, 40, 1200
    lens = [1200, 777, 1, 0, 65]
    B = len(lens)
    g = torch.Generator().manual_seed(300 + b)
    c = torch.randn(B, T, r, generator=g).to(torch.bfloat16)
    kr = torch.randn(B, T, dR, generator=g).to(torch.bfloat16)
    c_new = torch.randn(B, r, generator=g).to(torch.bfloat16)
    kr_new = torch.randn(B, dR, generator=g).to(torch.bfloat16)
    ql = torch.randn(B, H, r, generator=g).to(qdtype)
    qr = torch.randn(B, H, dR, generator=g).to(qdtype)
    sigma = 1 / math.sqrt(d + dR)
    # the sequence as the oracle sees it: its first len-1 tokens, then the new one
    full_c, full_k = c.clone(), kr.clone()
    for i, n in enumerate(lens):
        if n:
            full_c[i, n - 1] = c_new[i]
            full_k[i, n - 1] = kr_new[i]
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    outs = {}
    for fused in (True, False):
        lay = pkg.Layout([0, 0], [d, 0], [b, 0], r, dR, B, T)
        try:
            # prefill every position; the append then overwrites position len - 1
            lay.quant_write(0, c.cuda(), kr.cuda(), torch.zeros(B, dtype=torch.int32,
                                                                 device="cuda"))
            lse = torch.empty(B, H, device="cuda")
            if fused:
                out = lay.mla_decode_append(0, c_new.cuda(), kr_new.cuda(), ql.cuda(), qr.cuda(),
                                            lens_t, sigma, lse=lse)
            else:
                # the two-call form: write the new tokens at len - 1 (an empty sequence gets an
                # out-of-range position: skipped and flagged), then decode
                start = torch.tensor([n - 1 if n else 10 ** 6 for n in lens], dtype=torch.int32,
                                     device="cuda")
                lay.quant_write(0, c_new[:, None].cuda(), kr_new[:, None].cuda(), start)
                flags = lay.read_status(clear=True)
                assert flags == (pkg.KVK_FLAG_WRITE_RANGE if 0 in lens else 0)
                out = lay.mla_decode(0, ql.cuda(), qr.cuda(), lens_t, sigma, lse=lse)
            torch.cuda.synchronize()
            codes, scales = lay.cache_views(0)
            outs[fused] = (out.cpu().numpy(), lse.cpu().numpy(), codes.cpu().numpy(),
                           scales.cpu().view(torch.int16).numpy().view(np.uint16))
            if fused:
                assert lay.read_status() == 0
        finally:
            lay.close()
    o, l_, codes, scales = outs[True]
    # bit-identical to the two-call form, cache and outputs
    assert np.array_equal(codes, outs[False][2])
    assert np.array_equal(scales, outs[False][3])
    assert np.array_equal(o, outs[False][0]) and np.array_equal(l_, outs[False][1])
    for i, n in enumerate(lens):
        if n == 0:
            assert not o[i].any() and np.all(np.isneginf(l_[i]))
            continue
        rows, s, vals = _oracle_rows(oracle_mod, bf16_or_f32_to_np(full_c[i, :n]),
                                     bf16_or_f32_to_np(full_k[i, :n]), d, b)
        # the appended row and scale, bit for bit
        assert np.array_equal(codes[i, n - 1, :rows.shape[1]], rows[n - 1]), f"seq {i} row"
        assert scales[i, n - 1] == s[n - 1], f"seq {i} scale"
        o_ref, l_ref = oracle_mod.attend(bf16_or_f32_to_np(ql[i])[:, :d].astype(np.float64),
                                         bf16_or_f32_to_np(qr[i]), vals, np.arange(n), sigma)
        check_outputs(o[i], l_[i], o_ref, l_ref, f"b={b} {qdtype} seq {i}")


def test_append_refuses_inheriting_layer_and_keeps_arguments_checked(pkg):
    lay = pkg.Layout([0, 0], [64, 0], [8, 0], 64, 16, 2, 32)
    try:
        B, H = 2, 4
        ql = torch.zeros(B, H, 64, dtype=torch.bfloat16, device="cuda")
        qr = torch.zeros(B, H, 16, dtype=torch.bfloat16, device="cuda")
        c_new = torch.zeros(B, 64, dtype=torch.bfloat16, device="cuda")
        k_new = torch.zeros(B, 16, dtype=torch.bfloat16, device="cuda")
        lens = torch.ones(B, dtype=torch.int32, device="cuda")
        with pytest.raises(pkg.KvkError) as e:
            lay.mla_decode_append(1, c_new, k_new, ql, qr, lens, 1.0)
        assert e.value.status == 4
        with pytest.raises(pkg.KvkError) as e:   # new token misaligned
            buf = torch.zeros(B * 64 + 8, dtype=torch.bfloat16, device="cuda")
            lay.mla_decode_append(0, buf[1:1 + B * 64].view(B, 64), k_new, ql, qr, lens, 1.0)
        assert e.value.status == 6
    finally:
        lay.close()
