"""Compressed decode attention on the GPU vs the oracle (per-head tolerance), plus the
invariants: inheriting layer == anchor (bit-identical), split-count invariance, keep list ==
compacted cache, both decode kernels, edge cases (empty / one-token / ragged sequences)."""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import (Case, bf16_or_f32_to_np, check_outputs, oracle_cache, oracle_decode,
                         rel_err)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkg():
    import __graft_entry__
    __graft_entry__.build()
    import compressed_decode_attention_kvk_b200 as p
    assert torch.cuda.is_available()
    return p


def _rand(shape, seed, dtype, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(dtype)


def _decode(case, layer, ql, qr, lens, sigma, path, ctas=0, keep=None, keep_len=None):
    lay = case.lay
    lay.set_decode_path(path)
    lay.set_decode_ctas(ctas)
    B, H = ql.shape[0], ql.shape[1]
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    out = lay.mla_decode(layer, ql.cuda(), qr.cuda(), lens.cuda(), sigma, lse=lse,
                         keep_idx=None if keep is None else keep.cuda(),
                         keep_len=None if keep_len is None else keep_len.cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def _paths(pkg, case, dtype, H, has_keep=False):
    """Decode kernels that run this shape: always the CUDA-core one, plus the tensor one."""
    ps = [2]
    case.lay.set_decode_path(1)
    try:
        if case.lay.decode_path_for(0, dtype, H, has_keep) == 1:
            ps.append(1)
    except pkg.KvkError:
        pass
    finally:
        case.lay.set_decode_path(0)
    return ps


# ---------------------------------------------------------------------------
# tiny workload (fp32, the pages' small case)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("table_name", ["tiny", "tiny_swap"])
def test_tiny_workload_all_layers(pkg, oracle_mod, table_name):
    import workloads
    w = workloads.WORKLOADS["tiny"]
    t = workloads.table(table_name)
    lay = pkg.Layout(t["anchor"], t["d"], t["b"], w.r, w.d_rope, w.batch, w.tokens)
    try:
        host = {}
        for l in range(w.n_layers):
            if t["anchor"][l] == l:
                c = workloads.latent(w, l, w.batch, w.tokens)
                kr = workloads.rope_key(w, l, w.batch, w.tokens)
                host[l] = (c, kr)
                lay.quant_write(l, c.cuda(), kr.cuda(),
                                torch.zeros(w.batch, dtype=torch.int32, device="cuda"))
        lens = torch.full((w.batch,), w.tokens, dtype=torch.int32, device="cuda")
        outs = {}
        for l in range(w.n_layers):
            a = t["anchor"][l]
            d = t["d"][a]
            ql, qr = workloads.queries(w, l, w.batch)
            sigma = workloads.softmax_scale(d, w.d_rope)
            lse = torch.empty(w.batch, w.n_heads, device="cuda")
            out = lay.mla_decode(l, ql.cuda(), qr.cuda(), lens, sigma, lse=lse)
            torch.cuda.synchronize()
            c, kr = host[a]
            ref = oracle_cache(oracle_mod, c, kr, d, t["b"][a])
            o_ref, l_ref = oracle_decode(oracle_mod, ref[0], ql[0].double().numpy(),
                                         qr[0].double().numpy(), d, sigma)
            check_outputs(out[0].cpu().numpy(), lse[0].cpu().numpy(), o_ref, l_ref, f"layer {l}")
            outs[l] = (ql, qr, out.cpu())
        # inheriting layer with its anchor's query reproduces the anchor's output bit for bit
        for l in range(w.n_layers):
            a = t["anchor"][l]
            if a != l:
                ql, qr, o_a = outs[a]
                d = t["d"][a]
                o_l = lay.mla_decode(l, ql.cuda(), qr.cuda(), lens,
                                     workloads.softmax_scale(d, w.d_rope))
                assert torch.equal(o_l.cpu(), o_a)
        assert lay.read_status() == 0
    finally:
        lay.close()


# ---------------------------------------------------------------------------
# shapes x bit widths x kernels, ragged lengths
# ---------------------------------------------------------------------------

SHAPES = [  # d, r, dR, H, B, lens
    (64, 64, 16, 8, 3, [256, 1, 97]),
    (128, 512, 64, 28, 3, [300, 64, 129]),
    (512, 512, 64, 40, 2, [1000, 777]),
    (384, 512, 64, 40, 3, [0, 512, 65]),
    (256, 512, 64, 16, 4, [200, 63, 1, 128]),
]


@pytest.mark.parametrize("b", [2, 4, 8, 16])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"d{s[0]}H{s[3]}")
@pytest.mark.parametrize("qdtype", [torch.bfloat16, torch.float32])
def test_decode_matches_oracle(pkg, oracle_mod, b, shape, qdtype):
    d, r, dR, H, B, lens = shape
    T = max(lens) + 5
    case = Case(pkg, d, b, r, dR, B, T)
    try:
        seed = d * 7 + b * 3 + H
        c = _rand((B, T, r), seed, torch.bfloat16)
        kr = _rand((B, T, dR), seed + 1, torch.bfloat16)
        case.write(c, kr)
        ql = _rand((B, H, r), seed + 2, qdtype)
        qr = _rand((B, H, dR), seed + 3, qdtype)
        sigma = 1 / math.sqrt(d + dR)
        ref_cache = oracle_cache(oracle_mod, c, kr, d, b)
        lens_t = torch.tensor(lens, dtype=torch.int32)
        refs = []
        for i in range(B):
            k, s, rows = ref_cache[i]
            refs.append(oracle_decode(oracle_mod, (k[:lens[i]], s[:lens[i]], None),
                                      bf16_or_f32_to_np(ql[i]), bf16_or_f32_to_np(qr[i]), d,
                                      sigma))
        for path in _paths(pkg, case, qdtype, H):
            out, lse = _decode(case, 1, ql, qr, lens_t, sigma, path)   # layer 1 inherits 0
            for i in range(B):
                check_outputs(out[i], lse[i], refs[i][0], refs[i][1], f"path {path} seq {i}")
        assert case.lay.read_status() == 0
    finally:
        case.close()


def test_split_count_invariance_and_paths_agree(pkg, oracle_mod):
    d, r, dR, H, B = 512, 512, 64, 40, 3
    lens = [2000, 1500, 37]
    case = Case(pkg, d, 16, r, dR, B, 2048)
    try:
        c = _rand((B, 2048, r), 1, torch.bfloat16)
        kr = _rand((B, 2048, dR), 2, torch.bfloat16)
        case.write(c, kr)
        ql, qr = _rand((B, H, r), 3, torch.bfloat16), _rand((B, H, dR), 4, torch.bfloat16)
        lens_t = torch.tensor(lens, dtype=torch.int32)
        sigma = 1 / math.sqrt(d + dR)
        base, _ = _decode(case, 0, ql, qr, lens_t, sigma, 2, ctas=1)
        for path in _paths(pkg, case, torch.bfloat16, H):
            for ctas in (1, 2, 7, 64, 148, 300):
                out, _ = _decode(case, 0, ql, qr, lens_t, sigma, path, ctas=ctas)
                for i in range(B):
                    assert rel_err(out[i], base[i]) <= 2e-3, (path, ctas, i)
    finally:
        case.close()


def test_short_sequences_many_ctas_poisoned_workspace(pkg, oracle_mod):
    """Far fewer tokens than CTAs (CTAs that own nothing write no partials) with a workspace
    full of NaN bytes: the merge takes exactly the CTAs that hold a piece of each sequence,
    on both kernels and for several CTA counts."""
    d, r, dR, H, B, T = 512, 512, 64, 40, 4, 4096
    case = Case(pkg, d, 16, r, dR, B, T)
    try:
        c = _rand((B, T, r), 41, torch.bfloat16)
        kr = _rand((B, T, dR), 42, torch.bfloat16)
        case.write(c, kr)
        ql, qr = _rand((B, H, r), 43, torch.bfloat16), _rand((B, H, dR), 44, torch.bfloat16)
        lens = [3, 0, 70, 1]
        lens_t = torch.tensor(lens, dtype=torch.int32)
        sigma = 1 / math.sqrt(d + dR)
        ref_cache = oracle_cache(oracle_mod, c, kr, d, 16)
        refs = {}
        for i in range(B):
            if lens[i]:
                k, s_, _ = ref_cache[i]
                refs[i] = oracle_decode(oracle_mod, (k[:lens[i]], s_[:lens[i]], None),
                                        bf16_or_f32_to_np(ql[i]), bf16_or_f32_to_np(qr[i]), d,
                                        sigma)
        lay = case.lay
        for path in _paths(pkg, case, torch.bfloat16, H):
            for ctas in (0, 37, 1000):
                lay.set_decode_path(path)
                lay.set_decode_ctas(ctas)
                ws = torch.full((lay.workspace_bytes(0, B, H),), 255, dtype=torch.uint8,
                                device="cuda")
                lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
                out = lay.mla_decode(0, ql.cuda(), qr.cuda(), lens_t.cuda(), sigma, lse=lse,
                                     workspace=ws)
                torch.cuda.synchronize()
                out, lse = out.cpu().numpy(), lse.cpu().numpy()
                assert not out[1].any() and np.all(np.isneginf(lse[1])), (path, ctas)
                for i, (o_ref, l_ref) in refs.items():
                    check_outputs(out[i], lse[i], o_ref, l_ref, f"path {path} ctas {ctas} seq {i}")
        lay.set_decode_ctas(0)
        lay.set_decode_path(0)
        assert lay.read_status() == 0
    finally:
        case.close()


def test_keep_list_equals_compacted_cache(pkg, oracle_mod):
    d, r, dR, H, B, T = 256, 512, 64, 40, 3, 3000
    case = Case(pkg, d, 8, r, dR, B, T)
    try:
        c = _rand((B, T, r), 11, torch.bfloat16)
        kr = _rand((B, T, dR), 12, torch.bfloat16)
        case.write(c, kr)
        ql, qr = _rand((B, H, r), 13, torch.bfloat16), _rand((B, H, dR), 14, torch.bfloat16)
        lens = [3000, 2500, 40]
        K = 400
        g = np.random.default_rng(0)
        keep = np.zeros((B, K), dtype=np.int32)
        klen = [400, 312, 40]
        for i in range(B):
            keep[i, :klen[i]] = np.sort(g.choice(lens[i], klen[i], replace=False))
        sigma = 1 / math.sqrt(d + dR)
        ref_cache = oracle_cache(oracle_mod, c, kr, d, 8)
        keep_t = torch.from_numpy(keep)
        for path in _paths(pkg, case, torch.bfloat16, H, has_keep=True):
            out, lse = _decode(case, 0, ql, qr, torch.tensor(lens, dtype=torch.int32), sigma,
                               path, keep=keep_t, keep_len=torch.tensor(klen, dtype=torch.int32))
            for i in range(B):
                o_ref, l_ref = oracle_decode(oracle_mod, ref_cache[i], bf16_or_f32_to_np(ql[i]),
                                             bf16_or_f32_to_np(qr[i]), d, sigma,
                                             tok=keep[i, :klen[i]])
                check_outputs(out[i], lse[i], o_ref, l_ref, f"keep path {path} seq {i}")
        # keep-all list == dense decode
        allk = torch.arange(T, dtype=torch.int32).repeat(B, 1)
        dense, _ = _decode(case, 0, ql, qr, torch.tensor(lens, dtype=torch.int32), sigma, 0)
        kept, _ = _decode(case, 0, ql, qr, torch.tensor(lens, dtype=torch.int32), sigma, 0,
                          keep=allk, keep_len=torch.tensor(lens, dtype=torch.int32))
        for i in range(B):
            assert rel_err(kept[i], dense[i]) <= 2e-3
        assert case.lay.read_status() == 0
        # an index beyond seq_len is skipped and flagged, by both kernels (the tensor-core one
        # through the dense copy of the kept rows)
        bad = keep_t.clone()
        bad[2, 0] = 39
        bad[2, 1] = 45   # >= seq_len 40
        bad[0, 5] = -3   # negative, in the middle of a list
        for path in _paths(pkg, case, torch.bfloat16, H, has_keep=True):
            out, _ = _decode(case, 0, ql, qr, torch.tensor(lens, dtype=torch.int32), sigma, path,
                             keep=bad, keep_len=torch.tensor([400, 312, 2], dtype=torch.int32))
            assert case.lay.read_status(clear=True) & pkg.KVK_FLAG_KEEP_INDEX
            o_ref, _ = oracle_decode(oracle_mod, ref_cache[2], bf16_or_f32_to_np(ql[2]),
                                     bf16_or_f32_to_np(qr[2]), d, sigma, tok=[39])
            check_outputs(out[2], None, o_ref, None, f"bad keep entry skipped, path {path}")
            tok0 = np.delete(keep[0, :400], 5)
            o_ref, _ = oracle_decode(oracle_mod, ref_cache[0], bf16_or_f32_to_np(ql[0]),
                                     bf16_or_f32_to_np(qr[0]), d, sigma, tok=tok0)
            check_outputs(out[0], None, o_ref, None, f"negative keep entry skipped, path {path}")
    finally:
        case.close()


def test_keep_list_tensor_core_workspace(pkg, oracle_mod):
    """A keep list on the tensor-core kernel: with the keep workspace (NaN-filled) the kept
    rows are copied densely and decoded there; with only the plain workspace the automatic
    choice falls back to the CUDA-core kernel, and a forced tensor-core call is refused."""
    d, r, dR, H, B, T = 512, 512, 64, 40, 3, 2500
    case = Case(pkg, d, 16, r, dR, B, T)
    try:
        c = _rand((B, T, r), 51, torch.bfloat16)
        kr = _rand((B, T, dR), 52, torch.bfloat16)
        case.write(c, kr)
        ql, qr = _rand((B, H, r), 53, torch.bfloat16), _rand((B, H, dR), 54, torch.bfloat16)
        lens = [2500, 1800, 90]
        K = 333   # not a multiple of the 64-row tile
        klen = [333, 200, 90]
        g = np.random.default_rng(5)
        keep = np.zeros((B, K), dtype=np.int32)
        for i in range(B):
            keep[i, :klen[i]] = np.sort(g.choice(lens[i], klen[i], replace=False))
        sigma = 1 / math.sqrt(d + dR)
        ref_cache = oracle_cache(oracle_mod, c, kr, d, 16)
        refs = [oracle_decode(oracle_mod, ref_cache[i], bf16_or_f32_to_np(ql[i]),
                              bf16_or_f32_to_np(qr[i]), d, sigma, tok=keep[i, :klen[i]])
                for i in range(B)]
        lay = case.lay
        args = (ql.cuda(), qr.cuda(), torch.tensor(lens, dtype=torch.int32).cuda(), sigma)
        kw = dict(keep_idx=torch.from_numpy(keep).cuda(),
                  keep_len=torch.tensor(klen, dtype=torch.int32).cuda())
        big = lay.workspace_bytes(0, B, H, keep_stride=K)
        small = lay.workspace_bytes(0, B, H)
        assert big > small
        for mode, nbytes in ((1, big), (0, big), (0, small)):
            lay.set_decode_path(mode)
            ws = torch.full((nbytes,), 255, dtype=torch.uint8, device="cuda")
            lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
            out = lay.mla_decode(0, *args, lse=lse, workspace=ws, **kw)
            torch.cuda.synchronize()
            out, lse = out.cpu().numpy(), lse.cpu().numpy()
            for i in range(B):
                check_outputs(out[i], lse[i], refs[i][0], refs[i][1],
                              f"mode {mode} workspace {nbytes} seq {i}")
        lay.set_decode_path(1)
        with pytest.raises(pkg.KvkError):
            lay.mla_decode(0, *args, workspace=torch.empty(small, dtype=torch.uint8,
                                                           device="cuda"), **kw)
        lay.set_decode_path(0)
        assert lay.read_status() == 0
    finally:
        case.close()


def test_full_width_16_bit_cache_close_to_unquantised(pkg, oracle_mod):
    """b = 16, d = r: the GPU result equals plain MLA attention on the unquantised inputs
    within the output tolerance."""
    r, dR, H, B, T = 512, 64, 40, 2, 1024
    case = Case(pkg, r, 16, r, dR, B, T)
    try:
        c = _rand((B, T, r), 21, torch.bfloat16)
        kr = _rand((B, T, dR), 22, torch.bfloat16)
        case.write(c, kr)
        ql, qr = _rand((B, H, r), 23, torch.bfloat16), _rand((B, H, dR), 24, torch.bfloat16)
        sigma = 1 / math.sqrt(r + dR)
        out, lse = _decode(case, 0, ql, qr, torch.full((B,), T, dtype=torch.int32), sigma, 0)
        for i in range(B):
            rows = np.concatenate([bf16_or_f32_to_np(c[i]), bf16_or_f32_to_np(kr[i])], 1)
            o_ref, l_ref = oracle_mod.attend(bf16_or_f32_to_np(ql[i]), bf16_or_f32_to_np(qr[i]),
                                             rows.astype(np.float64), np.arange(T), sigma)
            check_outputs(out[i], lse[i], o_ref, l_ref, f"seq {i}")
    finally:
        case.close()


def test_edge_lengths_and_flags(pkg, oracle_mod):
    d, r, dR, H, B, T = 128, 128, 16, 8, 4, 50
    case = Case(pkg, d, 4, r, dR, B, T)
    try:
        c = _rand((B, T, r), 31, torch.bfloat16)
        kr = _rand((B, T, dR), 32, torch.bfloat16)
        case.write(c, kr)
        ql, qr = _rand((B, H, r), 33, torch.bfloat16), _rand((B, H, dR), 34, torch.bfloat16)
        sigma = 0.1
        ref_cache = oracle_cache(oracle_mod, c, kr, d, 4)
        # empty sequence -> zeros and -inf; one token -> c_hat; over-long -> clamped + flag
        for path in _paths(pkg, case, torch.bfloat16, H):
            out, lse = _decode(case, 0, ql, qr, torch.tensor([0, 1, 50, 70], dtype=torch.int32),
                               sigma, path)
            assert not out[0].any() and np.all(np.isneginf(lse[0]))
            k, s, _ = ref_cache[1]
            chat = oracle_mod.dequant(k[:1], s[:1])[0, :d]
            np.testing.assert_allclose(out[1], np.tile(chat, (H, 1)), rtol=1e-3, atol=1e-6)
            for i in (2, 3):
                o_ref, l_ref = oracle_decode(oracle_mod, ref_cache[i], bf16_or_f32_to_np(ql[i]),
                                             bf16_or_f32_to_np(qr[i]), d, sigma)
                check_outputs(out[i], lse[i], o_ref, l_ref, f"path {path} seq {i}")
            assert case.lay.read_status(clear=True) & pkg.KVK_FLAG_SEQ_LEN
    finally:
        case.close()


def test_argument_errors(pkg):
    case = Case(pkg, 64, 8, 64, 16, 2, 32)
    try:
        lay = case.lay
        q = torch.zeros(2, 4, 64, dtype=torch.bfloat16, device="cuda")
        qr = torch.zeros(2, 4, 16, dtype=torch.bfloat16, device="cuda")
        lens = torch.ones(2, dtype=torch.int32, device="cuda")
        ws = lay.new_workspace(0, 2, 4)
        out = torch.empty(2, 4, 64, device="cuda")
        with pytest.raises(pkg.KvkError) as e:   # workspace too small
            pkg.kvk_mla_decode(lay.handle, 0, q, qr, lens, 1.0, out, ws[:16])
        assert e.value.status == 5
        buf = torch.empty(2 * 4 * 64 + 4, device="cuda")
        with pytest.raises(pkg.KvkError) as e:   # output not 16-byte aligned
            pkg.kvk_mla_decode(lay.handle, 0, q, qr, lens, 1.0, buf[1:1 + 512].view(2, 4, 64), ws)
        assert e.value.status == 6
        with pytest.raises(pkg.KvkError) as e:   # layer out of range
            pkg.kvk_mla_decode(lay.handle, 5, q, qr, lens, 1.0, out, ws)
        assert e.value.status == 1
    finally:
        case.close()
