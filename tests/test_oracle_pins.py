"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against something it does not share code with: the pages'
printed numbers (tests/golden/), exhaustive enumeration of binary16 values, brute-force
search over all codes, an independent bit reader (numpy.unpackbits), closed forms of
softmax attention, a library attention routine (torch scaled_dot_product_attention in
float64), and a 50-digit mpmath evaluation.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# all finite binary16 values in increasing order (+inf appended), from numpy's own decoder
_ALL16 = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
_VALS16 = _ALL16.view(np.float16).astype(np.float64)
_FIN = np.isfinite(_VALS16)
_ORDER = np.argsort(_VALS16[_FIN], kind="stable")
_SORTED_VALS = _VALS16[_FIN][_ORDER]
_SORTED_BITS = _ALL16[_FIN][_ORDER]


def _smallest_f16_at_least(x: float):
    """Brute force over every binary16 value: the smallest one >= x (value, bits)."""
    i = np.searchsorted(_SORTED_VALS, x, side="left")
    if i == len(_SORTED_VALS):
        return math.inf, 0x7C00
    return _SORTED_VALS[i], int(_SORTED_BITS[i])


def _read_examples(path):
    ex, cur = [], None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("example"):
            cur = {"name": line.split()[1]}
            ex.append(cur)
            continue
        k, v = [s.strip() for s in line.split("=", 1)]
        cur[k] = v
    return ex


def _read_kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = [s.strip() for s in line.split("=", 1)]
            out[k] = int(v)
    return out


# --------------------------------------------------------------------------
# binary16 helpers
# --------------------------------------------------------------------------

def test_f16_decode_matches_numpy(oracle_mod):
    for h in list(range(0, 0x7C00, 97)) + [0, 1, 0x3FF, 0x400, 0x3C00, 0x7BFF, 0x8001, 0xBC00]:
        ref = np.array([h], dtype=np.uint16).view(np.float16).astype(np.float64)[0]
        assert oracle_mod.f16_bits_to_f64(h) == ref


def test_f16_round_up_is_smallest_value_at_least(oracle_mod):
    rng = np.random.default_rng(0)
    xs = []
    # exact binary16 values, their float32 neighbours and midpoints, across all binades
    for h in range(1, 0x7C00, 37):
        v = np.float32(_VALS16[h])
        xs += [v, np.nextafter(v, np.float32(np.inf)), np.nextafter(v, np.float32(0))]
        if h + 1 < 0x7C00:
            xs.append(np.float32((_VALS16[h] + _VALS16[h + 1]) / 2))
    xs += list(rng.uniform(0, 70000, 2000).astype(np.float32))
    xs += list((10.0 ** rng.uniform(-12, -4, 2000)).astype(np.float32))   # subnormal range
    xs += [np.float32(65504.0), np.float32(65504.5), np.float32(65520.0), np.float32(1e-30)]
    xs += list(-rng.uniform(0, 70000, 500).astype(np.float32))             # negatives
    for x in xs:
        want_val, want_bits = _smallest_f16_at_least(float(x))
        got = oracle_mod.f32_to_f16_ru(float(x))
        if float(x) == 0.0:
            assert oracle_mod.f16_bits_to_f64(got) == 0.0
            continue
        assert oracle_mod.f16_bits_to_f64(got) == want_val, (x, hex(got), want_val)


# --------------------------------------------------------------------------
# quantiser
# --------------------------------------------------------------------------

def test_golden_worked_examples(oracle_mod):
    for ex in _read_examples(os.path.join(GOLDEN, "quant_worked_examples.txt")):
        b = int(ex["b"])
        v = np.array([float(x) for x in ex["v"].split()], dtype=np.float32)[None, :]
        scales, codes = oracle_mod.quantize(v, b)
        assert int(scales[0]) == int(ex["scale_bits"], 16), ex["name"]
        assert codes[0].tolist() == [int(x) for x in ex["codes"].split()], ex["name"]
        rows = oracle_mod.pack(codes, b)
        want = bytes(int(x, 16) for x in ex["row"].split())
        assert rows[0].tobytes() == want, ex["name"]
        assert oracle_mod.unpack(rows, v.shape[1], b).tolist() == codes.tolist()


def _brute_codes(v, s, q):
    """Argmin over every integer code in [-q, q] of |fp32(v/s) - code|, ties to even."""
    out = np.zeros(v.shape, dtype=np.int64)
    cand = np.arange(-q, q + 1, dtype=np.int64)
    for i, x in enumerate(v):
        t = np.float32(x) / np.float32(s)        # one IEEE binary32 division
        if q > 1000:                              # b = 16: search a window around t
            c0 = int(np.floor(np.float64(t)))
            cc = np.arange(max(-q, c0 - 2), min(q, c0 + 3), dtype=np.int64)
        else:
            cc = cand
        dist = np.abs(np.float64(t) - cc.astype(np.float64))
        best = dist.min()
        ties = cc[dist == best]
        even = ties[ties % 2 == 0]
        out[i] = even[0] if len(even) else ties[0]
    return out


@pytest.mark.parametrize("b", [2, 4, 8, 16])
def test_quantizer_against_brute_force_and_bounds(oracle_mod, b):
    rng = np.random.default_rng(b)
    q = 2 ** (b - 1) - 1
    T, n = 24, 80
    v = rng.standard_normal((T, n)).astype(np.float32)
    v[3] *= 1e-3
    v[4] *= 1e4
    v[5, :] = 0.0
    v[6, 7] = 5.0                       # one dominant value
    v[7] = rng.standard_t(3, n).astype(np.float32)
    scales, codes = oracle_mod.quantize(v, b)
    for t in range(T):
        A = float(np.max(np.abs(v[t])))
        s = oracle_mod.f16_bits_to_f64(int(scales[t]))
        if A == 0.0:
            assert s == 0.0 and not codes[t].any()
            continue
        # scale: smallest binary16 value not below the binary32 quotient A/q
        quot = float(np.float32(A) / np.float32(q))
        want_s, _ = _smallest_f16_at_least(quot)
        assert s == want_s
        # codes: brute force over all codes
        assert np.array_equal(codes[t], _brute_codes(v[t], s, q)), t
        assert np.abs(codes[t]).max() <= q
        # dequantisation error <= s/2, up to the binary32 rounding of the quotient v/s
        err = np.abs(v[t].astype(np.float64) - codes[t] * s)
        bound = s / 2 + np.abs(v[t].astype(np.float64)) * 2.0 ** -23
        assert np.all(err <= bound), (t, (err - bound).max())


def test_quantizer_ties_round_to_even(oracle_mod):
    # s = 0.125 exactly: A = 127 * 0.125 at b = 8
    s = 0.125
    ks = np.arange(-120, 120)
    v = np.concatenate([[127 * s], (ks + 0.5) * s]).astype(np.float32)
    scales, codes = oracle_mod.quantize(v[None, :], 8)
    assert oracle_mod.f16_bits_to_f64(int(scales[0])) == s
    c = codes[0][1:]
    lo, hi = ks, ks + 1
    want = np.where(lo % 2 == 0, lo, hi)
    assert np.array_equal(c, want)


def test_quantizer_scale_is_shared_by_latent_and_rope(oracle_mod):
    # one scale per token over [c[:d] || k^R]: a large rope value sets the scale for the latent
    c = np.zeros((1, 64), dtype=np.float32)
    c[0, :32] = 0.01
    kr = np.zeros((1, 16), dtype=np.float32)
    kr[0, 3] = 100.0
    rows, scales, codes = oracle_mod.quantize_rows(c, kr, 32, 8)
    s = oracle_mod.f16_bits_to_f64(int(scales[0]))
    assert s >= 100.0 / 127
    assert codes.shape == (1, 48)
    assert codes[0, 32 + 3] == 127 and np.all(codes[0, :32] == 0)


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------

@pytest.mark.parametrize("b", [2, 4, 8, 16])
@pytest.mark.parametrize("n", [48, 80, 192, 576])
def test_pack_against_numpy_bit_reader(oracle_mod, b, n):
    rng = np.random.default_rng(n * 31 + b)
    q = 2 ** (b - 1) - 1
    codes = rng.integers(-q, q + 1, size=(5, n)).astype(np.int32)
    rows = oracle_mod.pack(codes, b)
    rb = rows.shape[1]
    assert rb % 16 == 0 and rb * 8 >= n * b and (rb - 16) * 8 < n * b
    bits = np.unpackbits(rows, axis=1, bitorder="little")           # independent reader
    fields = bits[:, : n * b].reshape(5, n, b).astype(np.int64)
    u = (fields << np.arange(b, dtype=np.int64)).sum(axis=2)
    assert np.array_equal(u - 2 ** (b - 1), codes)
    assert not bits[:, n * b:].any()                                  # zero padding


def test_row_bytes_of_the_configured_shapes(oracle_mod):
    # tiny: d=32,b=8 -> 48 B; d=64,b=4 -> 40 B padded to 48 B; 14B shapes need no padding
    assert oracle_mod.row_bytes(32 + 16, 8) == 48
    assert oracle_mod.row_bytes(64 + 16, 4) == 48
    for d in (128, 256, 384, 512):
        for b in (2, 4, 8, 16):
            assert oracle_mod.row_bytes(d + 64, b) == (d + 64) * b // 8


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _sdpa(q_lat, q_rope, rows, d, sigma):
    """torch's attention routine in float64: keys [c || kR], values c[:d]."""
    Q = torch.from_numpy(np.concatenate([q_lat, q_rope], axis=1))[None, None]
    K = torch.from_numpy(rows)[None, None]
    V = torch.from_numpy(rows[:, :d])[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=sigma)[0, 0].numpy()
    lse = torch.logsumexp(sigma * (Q[0, 0] @ K[0, 0].T), dim=-1).numpy()
    return out, lse


def test_attention_matches_library_routine(oracle_mod):
    rng = np.random.default_rng(5)
    H, d, dR, T = 6, 32, 16, 77
    q_lat = rng.standard_normal((H, d))
    q_rope = rng.standard_normal((H, dR))
    rows = rng.standard_normal((T, d + dR)) * 1.5
    sigma = 1 / math.sqrt(d + dR)
    out, lse = oracle_mod.attend(q_lat, q_rope, rows, np.arange(T), sigma)
    ref, ref_lse = _sdpa(q_lat, q_rope, rows, d, sigma)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_closed_forms(oracle_mod):
    rng = np.random.default_rng(6)
    H, d, dR, T = 3, 16, 8, 10
    rows = rng.standard_normal((T, d + dR))
    q_lat = rng.standard_normal((H, d))
    q_rope = rng.standard_normal((H, dR))
    # single token: out = c_hat[:d], lse = its score
    out, lse = oracle_mod.attend(q_lat, q_rope, rows, [4], 0.3)
    for h in range(H):
        np.testing.assert_allclose(out[h], rows[4, :d], rtol=0, atol=1e-15)
        z = 0.3 * (q_lat[h] @ rows[4, :d] + q_rope[h] @ rows[4, d:])
        assert abs(lse[h] - z) < 1e-12
    # zero query: uniform weights, out = mean, lse = log T
    out, lse = oracle_mod.attend(np.zeros((H, d)), np.zeros((H, dR)), rows, np.arange(T), 1.0)
    np.testing.assert_allclose(out, np.tile(rows[:, :d].mean(0), (H, 1)), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(T), atol=1e-14)
    # two tokens: logistic weights
    out, _ = oracle_mod.attend(q_lat, q_rope, rows, [1, 7], 0.5)
    for h in range(H):
        z1 = 0.5 * (q_lat[h] @ rows[1, :d] + q_rope[h] @ rows[1, d:])
        z7 = 0.5 * (q_lat[h] @ rows[7, :d] + q_rope[h] @ rows[7, d:])
        w1 = 1 / (1 + math.exp(z7 - z1))
        np.testing.assert_allclose(out[h], w1 * rows[1, :d] + (1 - w1) * rows[7, :d], atol=1e-13)
    # empty token set (reading R5)
    out, lse = oracle_mod.attend(q_lat, q_rope, rows, [], 1.0)
    assert not out.any() and np.all(np.isneginf(lse))


def test_attention_invariances(oracle_mod):
    rng = np.random.default_rng(7)
    H, d, dR, T = 4, 32, 16, 50
    rows = rng.standard_normal((T, d + dR))
    q_lat, q_rope = rng.standard_normal((H, d)), rng.standard_normal((H, dR))
    out, lse = oracle_mod.attend(q_lat, q_rope, rows, np.arange(T), 0.2)
    perm = rng.permutation(T)
    out2, lse2 = oracle_mod.attend(q_lat, q_rope, rows[perm], np.arange(T), 0.2)
    np.testing.assert_allclose(out2, out, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)
    # keep list == attention over the host-compacted rows
    keep = np.sort(rng.choice(T, 13, replace=False)).astype(np.int32)
    o_k, l_k = oracle_mod.attend(q_lat, q_rope, rows, keep, 0.2)
    o_c, l_c = oracle_mod.attend(q_lat, q_rope, rows[keep], np.arange(13), 0.2)
    np.testing.assert_allclose(o_k, o_c, atol=0)
    np.testing.assert_allclose(l_k, l_c, atol=0)


def test_attention_high_precision_brute_force(oracle_mod):
    mp = pytest.importorskip("mpmath")
    mp.mp.dps = 50
    rng = np.random.default_rng(8)
    H, d, dR, T = 2, 4, 2, 3
    rows = rng.standard_normal((T, d + dR)) * 3
    q_lat, q_rope = rng.standard_normal((H, d)) * 2, rng.standard_normal((H, dR))
    sigma = 0.7
    out, lse = oracle_mod.attend(q_lat, q_rope, rows, np.arange(T), sigma)
    for h in range(H):
        z = [mp.mpf(sigma) * (mp.fsum(mp.mpf(q_lat[h, j]) * mp.mpf(rows[t, j]) for j in range(d))
                              + mp.fsum(mp.mpf(q_rope[h, j]) * mp.mpf(rows[t, d + j]) for j in range(dR)))
             for t in range(T)]
        e = [mp.e ** zt for zt in z]
        Z = mp.fsum(e)
        for j in range(d):
            o = mp.fsum(e[t] * mp.mpf(rows[t, j]) for t in range(T)) / Z
            assert abs(float(o) - out[h, j]) <= 1e-13 * max(1.0, abs(float(o)))
        assert abs(float(mp.log(Z)) - lse[h]) <= 1e-13


def test_full_width_16_bit_cache_matches_unquantised_attention(oracle_mod):
    """b = 16, d = r: attention over the quantised cache equals plain MLA attention on the
    original inputs, up to the quantisation error (|v - v_hat| <= s/2 with s ~ A/32767)."""
    rng = np.random.default_rng(9)
    H, r, dR, T = 8, 64, 16, 200
    c = rng.standard_normal((T, r)).astype(np.float32)
    kr = rng.standard_normal((T, dR)).astype(np.float32)
    q_lat = rng.standard_normal((H, r))
    q_rope = rng.standard_normal((H, dR))
    sigma = 1 / math.sqrt(r + dR)
    _, scales, codes = oracle_mod.quantize_rows(c, kr, r, 16)
    out, lse = oracle_mod.decode_sequence(q_lat, q_rope, codes, scales, r, sigma)
    exact = np.concatenate([c, kr], axis=1).astype(np.float64)
    ref, ref_lse = _sdpa(q_lat, q_rope, exact, r, sigma)
    # per-element error <= A/32767/2 ~ 7e-5 here; the output moves by about as much
    for h in range(H):
        assert np.abs(out[h] - ref[h]).max() <= 2e-3 * np.abs(ref[h]).max()
        assert np.abs(out[h] - ref[h]).max() <= 1e-3
    np.testing.assert_allclose(lse, ref_lse, atol=1e-3)


# --------------------------------------------------------------------------
# cost model
# --------------------------------------------------------------------------

def test_cost_model_closed_forms(oracle_mod):
    g = _read_kv(os.path.join(GOLDEN, "cost_model_closed_forms.txt"))
    c0 = oracle_mod.c0_bits(48, 8, 128)
    assert c0 == g["c0_bits_14b"]
    assert c0 // 8 == g["c0_bytes_14b"] == 192 * 1024
    assert 32 * 8192 * (c0 // 8) == g["cache_32x8k_bytes_14b"] == 48 * 2 ** 30
    D, B = (64, 128, 256, 512), (2, 4, 8, 16)
    assert 1 + len(D) * len(B) == g["n_actions"]
    # M3 Ultra composition: 12 anchors of rank 128 (+ d_R = 64) at 4 bits, scale-free cost,
    # plus the 0.5 bit / element of a grouped scale -> 151.7 ~ 152x
    anchor = [4 * (l // 4) for l in range(48)]
    d = [128 if l % 4 == 0 else 0 for l in range(48)]
    b = [4 if l % 4 == 0 else 0 for l in range(48)]
    bits4 = oracle_mod.bits_per_token(anchor, d, b, 64, with_scale=False)
    assert bits4 == 12 * 192 * 4
    assert round(c0 / (bits4 * 4.5 / 4)) == g["m3_ultra_ratio_rounded"]
    assert 4 * 8 == g["composed_eviction_ratio"]


def test_cost_model_counts_anchors_only(oracle_mod):
    anchor, d, b = [0, 0, 2, 2], [32, 0, 64, 0], [8, 0, 4, 0]
    assert oracle_mod.bits_per_token(anchor, d, b, 16) == (48 * 8 + 16) + (80 * 4 + 16)
    assert oracle_mod.bits_per_token(anchor, d, b, 16, with_scale=False) == 48 * 8 + 80 * 4


def test_workload_tables_meet_their_budgets(oracle_mod):
    import workloads
    tabs = workloads.load_tables()
    for key, t in tabs.items():
        a = t["anchor"]
        assert a[0] == 0
        last = 0
        for l in range(len(a)):
            if a[l] == l:
                last = l
                assert t["d"][l] > 0 and t["b"][l] in (0, 2, 4, 8, 16)
            assert a[l] == last
        if "budget_bits" in t:
            bits = oracle_mod.bits_per_token(a, t["d"], t["b"], 64)
            assert bits == t["bits_per_token"]
            full = len(a) * ((512 + 64) * 16 + 16)
            assert bits <= t["budget_bits"] or (bits == full and t["budget_bits"] >= full)


# --------------------------------------------------------------------------
# the uncompressed (bfloat16) cache the compressed one is measured against
# --------------------------------------------------------------------------

def _bf16_value(h):
    return float(np.array([int(h) << 16], dtype=np.uint32).view(np.float32)[0])


def test_bf16_rounding_is_nearest_even_by_search(oracle_mod):
    """binary32 -> bfloat16: no other bfloat16 value of the same sign is nearer to x (exact
    binary64 arithmetic over the neighbouring patterns), and exact ties go to an even last
    fraction bit.  Includes constructed ties, subnormals, and values next to the largest."""
    rng = np.random.default_rng(21)
    xs = list(rng.standard_normal(2000).astype(np.float32))
    xs += list((rng.standard_normal(500) * 2.0 ** rng.integers(-140, 120, 500)).astype(np.float32))
    for h in (0x3F80, 0x3F81, 0x0001, 0x0080, 0x7F7E, 0x7F7F, 0x4049):
        lo, hi = _bf16_value(h), _bf16_value(h + 1)
        xs.append(np.float32((lo + hi) / 2))         # exact tie
        xs.append(np.nextafter(np.float32((lo + hi) / 2), np.float32(np.inf)))
        xs.append(np.nextafter(np.float32((lo + hi) / 2), np.float32(-np.inf)))
        xs.append(-np.float32((lo + hi) / 2))
    for x in xs:
        x = np.float32(x)
        if not np.isfinite(x):
            continue
        h = oracle_mod.f32_to_bf16_rne(float(x))
        y = _bf16_value(h)
        if np.isinf(y):          # overflow: x is at least half an ulp beyond the largest
            assert abs(float(x)) >= _bf16_value(0x7F7F) + 2.0 ** (127 - 8)
            continue
        e = abs(float(x) - y)
        sign = h & 0x8000
        for k in (-2, -1, 1, 2):
            hk = ((h & 0x7FFF) + k)
            if 0 <= hk < 0x7F80:
                ek = abs(float(x) - _bf16_value(sign | hk))
                assert e <= ek, (float(x), hex(h), k)
                if e == ek:
                    assert (h & 1) == 0, (float(x), hex(h))


def test_bf16_rounding_matches_torch(oracle_mod):
    """The same conversion as torch's round-to-nearest-even bfloat16 cast (an implementation
    the oracle does not call) on a million values of mixed magnitude."""
    rng = np.random.default_rng(22)
    x = (rng.standard_normal(1 << 20) * 2.0 ** rng.integers(-130, 127, 1 << 20)).astype(np.float32)
    x[:4] = [0.0, -0.0, 1.0, -3.0]
    bits = np.zeros(x.shape, dtype=np.uint16)
    oracle_mod.lib().kvko_bf16_round(x.ctypes.data, x.size, bits.ctypes.data)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


def test_bf16_cache_attention_equals_attention_on_the_rounded_rows(oracle_mod):
    """For bfloat16 inputs the uncompressed cache holds them exactly, so its attention is
    plain MLA attention on the inputs (torch SDPA in float64)."""
    rng = np.random.default_rng(23)
    T, r, dR, H = 300, 64, 16, 6
    c = torch.from_numpy(rng.standard_normal((T, r)).astype(np.float32)).to(torch.bfloat16)
    kr = torch.from_numpy(rng.standard_normal((T, dR)).astype(np.float32)).to(torch.bfloat16)
    ql, qr = rng.standard_normal((H, r)), rng.standard_normal((H, dR))
    bits, vals = oracle_mod.bf16_rows(c.float().numpy(), kr.float().numpy(), r)
    exact = np.concatenate([c.float().numpy(), kr.float().numpy()], 1).astype(np.float64)
    assert np.array_equal(vals, exact)
    out, lse = oracle_mod.decode_sequence_bf16(ql, qr, vals, r, 0.125)
    ref, ref_lse = _sdpa(ql, qr, exact, r, 0.125)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# group scales: one fp16 scale per G consecutive elements instead of per token
# --------------------------------------------------------------------------

def test_grouped_cost_reproduces_the_m3_ultra_ratio(oracle_mod):
    """"Hardware Benchmarking (M3 Ultra)": a 4-bit cache, MLA rank 128 and 12 groups of 4
    layers compose to 152x.  With one fp16 scale per 32 elements the 4-bit cache costs 4.5
    bits per element, and the grouped cost function gives C_0 / bits = 151.7 -> 152."""
    g = _read_kv(os.path.join(GOLDEN, "cost_model_closed_forms.txt"))
    anchor = [4 * (l // 4) for l in range(48)]
    d = [128 if l % 4 == 0 else 0 for l in range(48)]
    b = [4 if l % 4 == 0 else 0 for l in range(48)]
    bits = oracle_mod.bits_per_token_grouped(anchor, d, b, 64, 32)
    assert bits == 12 * (128 + 64) * 4 + 12 * 16 * (128 + 64) // 32
    c0 = oracle_mod.c0_bits(48, 8, 128)
    assert round(c0 / bits) == g["m3_ultra_ratio_rounded"]
    # one group per row is the per-token cost
    assert oracle_mod.bits_per_token_grouped([0], [128], [4], 64, 192) == \
        oracle_mod.bits_per_token([0], [128], [4], 64)


def test_grouped_quantiser_with_one_group_is_the_per_token_quantiser(oracle_mod):
    rng = np.random.default_rng(31)
    c = rng.standard_normal((40, 64)).astype(np.float32)
    kr = rng.standard_normal((40, 16)).astype(np.float32)
    for b in (2, 4, 8, 16):
        rows, s, k = oracle_mod.quantize_rows(c, kr, 64, b)
        rows_g, s_g, k_g = oracle_mod.quantize_rows_grouped(c, kr, 64, b, 80)
        assert np.array_equal(rows, rows_g) and np.array_equal(k, k_g)
        assert np.array_equal(s, s_g[:, 0])


@pytest.mark.parametrize("b", [2, 4, 8])
@pytest.mark.parametrize("G", [16, 32])
def test_grouped_quantiser_against_brute_force_and_bounds(oracle_mod, b, G):
    """Each group's scale is the smallest binary16 value not below max|v_group| / q, its codes
    the brute-force nearest (ties to even) under that scale, and the dequantised error at
    most half the group's scale (up to the binary32 rounding of v / s)."""
    rng = np.random.default_rng(40 + b + G)
    q = 2 ** (b - 1) - 1
    T, d, dR = 12, 64, 32
    c = rng.standard_normal((T, d)).astype(np.float32)
    kr = rng.standard_normal((T, dR)).astype(np.float32)
    c[2, :G] *= 1e3                   # one loud group: the others keep their own scale
    c[3, G:2 * G] = 0.0               # an all-zero group
    _, scales, codes = oracle_mod.quantize_rows_grouped(c, kr, d, b, G)
    v = np.concatenate([c, kr], axis=1)
    for t in range(T):
        for j in range(v.shape[1] // G):
            vg = v[t, j * G:(j + 1) * G]
            A = float(np.max(np.abs(vg)))
            s = oracle_mod.f16_bits_to_f64(int(scales[t, j]))
            cg = codes[t, j * G:(j + 1) * G]
            if A == 0.0:
                assert s == 0.0 and not cg.any()
                continue
            want_s, _ = _smallest_f16_at_least(float(np.float32(A) / np.float32(q)))
            assert s == want_s, (t, j)
            assert np.array_equal(cg, _brute_codes(vg, s, q)), (t, j)
            err = np.abs(vg.astype(np.float64) - cg * s)
            assert np.all(err <= s / 2 + np.abs(vg.astype(np.float64)) * 2.0 ** -23)
    # the loud group does not coarsen its neighbours
    assert scales[2, 1] < scales[2, 0]
    rows_hat = oracle_mod.dequant_grouped(codes, scales)
    assert np.array_equal(rows_hat[:, :G], codes[:, :G] * np.array(
        [oracle_mod.f16_bits_to_f64(int(x)) for x in scales[:, 0]])[:, None])


# --------------------------------------------------------------------------
# absorbed projections
# --------------------------------------------------------------------------

def test_absorb_against_brute_force_and_identity(oracle_mod):
    """y[b, h, j] = sum_k x[b, h, k] w[h, k, j]: a brute-force loop on a tiny case, the
    identity weight (y = x's first n coordinates), and a per-head weight that picks one head."""
    rng = np.random.default_rng(51)
    B, H, K, n = 2, 3, 5, 4
    x = rng.standard_normal((B, H, K))
    w = rng.standard_normal((H, K, n))
    y = oracle_mod.absorb(x, w)
    for b in range(B):
        for h in range(H):
            for j in range(n):
                s = 0.0
                for k in range(K):
                    s += x[b, h, k] * w[h, k, j]
                assert abs(y[b, h, j] - s) <= 1e-12 * max(1.0, abs(s))
    eye = np.broadcast_to(np.eye(K, 3), (H, K, 3))
    assert np.array_equal(oracle_mod.absorb(x, eye), x[:, :, :3])
    sel = np.zeros((H, K, n))
    sel[1, 2, :] = 1.0
    y2 = oracle_mod.absorb(x, sel)
    assert not y2[:, 0].any() and not y2[:, 2].any()
    assert np.array_equal(y2[:, 1], np.repeat(x[:, 1, 2:3], n, axis=1))
