"""CPU oracle for the KV-Kaizen compressed MLA cache -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` /
``--impl reference`` legs may import this module.  It shares nothing with the
CUDA library (``compressed_decode_attention_kvk_b200``) and never imports it.

The arithmetic lives in ``kvk_oracle.c`` (plain C, IEEE binary32 steps for the
quantiser, binary64 for attention); this module only marshals numpy arrays.
What each function follows is cited in ``kvk_oracle.c``'s header
(KV-Kaizen whiteboard summary: "Three Non-Eviction Compression Axes",
"Action Space and Cost Model", "Background: The KV Cache Bottleneck").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvk_oracle.c")
_LIB = os.path.join(_HERE, "libkvk_oracle.so")

# gcc flags: no contraction into FMA, no fast-math, so every float operation in
# the C source is one IEEE operation.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fopenmp"]


def build(force: bool = False) -> str:
    """Compile ``kvk_oracle.c`` into ``libkvk_oracle.so`` (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.kvko_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.kvko_f16_to_f64.restype = f64
        L.kvko_f32_to_f16_ru.argtypes = [ctypes.c_float]
        L.kvko_f32_to_f16_ru.restype = ctypes.c_uint16
        L.kvko_quantize.argtypes = [P, i64, i32, i32, P, P]
        L.kvko_row_bytes.argtypes = [i32, i32]
        L.kvko_row_bytes.restype = i32
        L.kvko_pack.argtypes = [P, i64, i32, i32, i32, P]
        L.kvko_unpack.argtypes = [P, i64, i32, i32, i32, P]
        L.kvko_dequant.argtypes = [P, P, i64, i32, P]
        L.kvko_attend.argtypes = [P, P, P, P, i32, i32, i32, i32, f64, P, P]
        L.kvko_bits_per_token.argtypes = [i32, P, P, P, i32, i32]
        L.kvko_bits_per_token.restype = i64
        L.kvko_c0_bits.argtypes = [i32, i32, i32]
        L.kvko_c0_bits.restype = i64
        L.kvko_num_threads.restype = i32
        L.kvko_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.kvko_bf16_to_f64.restype = f64
        L.kvko_f32_to_bf16_rne.argtypes = [ctypes.c_float]
        L.kvko_f32_to_bf16_rne.restype = ctypes.c_uint16
        L.kvko_bf16_round.argtypes = [P, i64, P]
        L.kvko_bits_per_token_grouped.argtypes = [i32, P, P, P, i32, i32]
        L.kvko_bits_per_token_grouped.restype = i64
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# scalar helpers
# --------------------------------------------------------------------------

def f16_bits_to_f64(h: int) -> float:
    return lib().kvko_f16_to_f64(int(h))


def f32_to_f16_ru(x: float) -> int:
    """binary32 -> binary16 bit pattern, rounded toward +inf (reading R2)."""
    return int(lib().kvko_f32_to_f16_ru(float(np.float32(x))))


def num_threads() -> int:
    return int(lib().kvko_num_threads())


# --------------------------------------------------------------------------
# quantiser / packing
# --------------------------------------------------------------------------

def row_bytes(n: int, b: int) -> int:
    return int(lib().kvko_row_bytes(n, b))


def quantize(v: np.ndarray, b: int):
    """v: [T, n] float32 -> (scales uint16 bits [T], codes int32 [T, n])."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    T, n = v.shape
    scales = np.zeros(T, dtype=np.uint16)
    codes = np.zeros((T, n), dtype=np.int32)
    lib().kvko_quantize(_p(v), T, n, b, _p(scales), _p(codes))
    return scales, codes


def pack(codes: np.ndarray, b: int, rb: int | None = None) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    T, n = codes.shape
    rb = row_bytes(n, b) if rb is None else rb
    rows = np.zeros((T, rb), dtype=np.uint8)
    lib().kvko_pack(_p(codes), T, n, b, rb, _p(rows))
    return rows


def unpack(rows: np.ndarray, n: int, b: int) -> np.ndarray:
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    T, rb = rows.shape
    codes = np.zeros((T, n), dtype=np.int32)
    lib().kvko_unpack(_p(rows), T, n, b, rb, _p(codes))
    return codes


def dequant(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    T, n = codes.shape
    out = np.zeros((T, n), dtype=np.float64)
    lib().kvko_dequant(_p(codes), _p(scales), T, n, _p(out))
    return out


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def attend(q_lat: np.ndarray, q_rope: np.ndarray, rows_hat: np.ndarray, tok, sigma: float):
    """Decode attention for one sequence over dequantised rows (binary64).

    q_lat [H, d], q_rope [H, d_R], rows_hat [T, d+d_R]; tok: indices attended.
    Returns (out [H, d] float64, lse [H] float64).
    """
    q_lat = np.ascontiguousarray(q_lat, dtype=np.float64)
    q_rope = np.ascontiguousarray(q_rope, dtype=np.float64)
    rows_hat = np.ascontiguousarray(rows_hat, dtype=np.float64)
    tok = np.ascontiguousarray(np.asarray(tok, dtype=np.int32))
    H, d = q_lat.shape
    d_R = q_rope.shape[1]
    assert rows_hat.shape[1] == d + d_R
    if tok.size:
        assert 0 <= tok.min() and tok.max() < rows_hat.shape[0]
    out = np.zeros((H, d), dtype=np.float64)
    lse = np.zeros(H, dtype=np.float64)
    lib().kvko_attend(_p(q_lat), _p(q_rope), _p(rows_hat), _p(tok), int(tok.size), H, d, d_R,
                      float(sigma), _p(out), _p(lse))
    return out, lse


# --------------------------------------------------------------------------
# cost model
# --------------------------------------------------------------------------

def bits_per_token(anchor, d, b, d_R: int, with_scale: bool = True) -> int:
    a = np.ascontiguousarray(np.asarray(anchor, dtype=np.int32))
    dd = np.ascontiguousarray(np.asarray(d, dtype=np.int32))
    bb = np.ascontiguousarray(np.asarray(b, dtype=np.int32))
    return int(lib().kvko_bits_per_token(len(a), _p(a), _p(dd), _p(bb), d_R, 1 if with_scale else 0))


def bits_per_token_grouped(anchor, d, b, d_R: int, G: int) -> int:
    """Bits per token with one fp16 scale per G elements of each anchor's row."""
    a = np.ascontiguousarray(np.asarray(anchor, dtype=np.int32))
    dd = np.ascontiguousarray(np.asarray(d, dtype=np.int32))
    bb = np.ascontiguousarray(np.asarray(b, dtype=np.int32))
    return int(lib().kvko_bits_per_token_grouped(len(a), _p(a), _p(dd), _p(bb), d_R, G))


def c0_bits(n_layers: int, n_kv: int, d_h: int) -> int:
    return int(lib().kvko_c0_bits(n_layers, n_kv, d_h))


# --------------------------------------------------------------------------
# whole-layer helpers built from the functions above
# --------------------------------------------------------------------------

def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact bf16 -> binary32 widening (a bf16 is the top half of a binary32)."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def token_vectors(c_kv: np.ndarray, k_rope: np.ndarray, d: int) -> np.ndarray:
    """[T, r] latent + [T, d_R] rope -> [T, d + d_R] float32 vectors [c[:d] || k^R]."""
    return np.ascontiguousarray(np.concatenate([c_kv[:, :d], k_rope], axis=1), dtype=np.float32)


def quantize_rows(c_kv: np.ndarray, k_rope: np.ndarray, d: int, b: int):
    """Quantise one sequence's tokens for an anchor with (d, b).

    Returns (packed rows uint8 [T, row_bytes], scales uint16 [T], codes int32 [T, n]).
    """
    v = token_vectors(c_kv, k_rope, d)
    scales, codes = quantize(v, b)
    return pack(codes, b), scales, codes


def f32_to_bf16_rne(x: float) -> int:
    """binary32 -> bfloat16 bit pattern, round to nearest, ties to even."""
    return int(lib().kvko_f32_to_bf16_rne(float(np.float32(x))))


def bf16_bits_to_f64(h: int) -> float:
    return lib().kvko_bf16_to_f64(int(h))


def bf16_rows(c_kv: np.ndarray, k_rope: np.ndarray, d: int):
    """The uncompressed cache of one sequence: the token vectors [c[:d] || k^R] stored as
    bfloat16 (round to nearest even).  Returns (bits uint16 [T, n], values float64 [T, n])."""
    v = token_vectors(c_kv, k_rope, d)
    bits = np.zeros(v.shape, dtype=np.uint16)
    lib().kvko_bf16_round(_p(v), v.size, _p(bits))
    return bits, bf16_bits_to_f32(bits).astype(np.float64)


def decode_sequence_bf16(q_lat, q_rope, values, d: int, sigma: float, tok=None):
    """Attention of one sequence over its uncompressed (bf16) cache rows `values` [T, n]."""
    T = values.shape[0]
    if tok is None:
        tok = np.arange(T, dtype=np.int32)
    return attend(np.asarray(q_lat, dtype=np.float64)[:, :d], q_rope, values, tok, sigma)


def quantize_rows_grouped(c_kv: np.ndarray, k_rope: np.ndarray, d: int, b: int, G: int):
    """Quantise one sequence's tokens with one scale per group of G consecutive elements of
    [c[:d] || k^R]: the per-token quantiser applied to every group as if it were a token.

    Returns (packed rows uint8 [T, row_bytes], scales uint16 [T, n / G], codes int32 [T, n]).
    """
    v = token_vectors(c_kv, k_rope, d)
    T, n = v.shape
    assert n % G == 0
    scales, codes = quantize(v.reshape(T * (n // G), G), b)
    codes = codes.reshape(T, n)
    return pack(codes, b), scales.reshape(T, n // G), codes


def dequant_grouped(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """c_hat = code * s of its group, exact in binary64; scales [T, n / G]."""
    T, n = codes.shape
    ng = scales.shape[1]
    return dequant(codes.reshape(T * ng, n // ng), scales.reshape(T * ng)).reshape(T, n)


def decode_sequence_grouped(q_lat, q_rope, codes, scales, d: int, sigma: float, tok=None):
    """Attention of one sequence over a group-scaled cache (codes [T, n], scales [T, n/G])."""
    rows_hat = dequant_grouped(codes, scales)
    T = rows_hat.shape[0]
    if tok is None:
        tok = np.arange(T, dtype=np.int32)
    return attend(np.asarray(q_lat, dtype=np.float64)[:, :d], q_rope, rows_hat, tok, sigma)


def absorb(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """The absorbed MLA projection (the query into the latent space with W_UK, the output out
    of it with W_UV; "Three Non-Eviction Compression Axes", item 2): y[b, h, j] =
    sum_k x[b, h, k] w[h, k, j], in binary64 (a matrix product per head)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    return np.einsum("bhk,hkj->bhj", x, w)


def decode_sequence(q_lat, q_rope, codes, scales, d: int, sigma: float, tok=None):
    """Attention of one sequence over its anchor's quantised cache.

    q_lat [H, >=d] (only the first d columns are used), q_rope [H, d_R],
    codes [T, d + d_R] int32, scales [T] fp16 bits; tok: keep list or None (all).
    """
    rows_hat = dequant(codes, scales)
    T = rows_hat.shape[0]
    if tok is None:
        tok = np.arange(T, dtype=np.int32)
    return attend(np.asarray(q_lat, dtype=np.float64)[:, :d], q_rope, rows_hat, tok, sigma)
