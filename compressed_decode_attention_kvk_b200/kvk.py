"""Python binding of libkvk (include/kvk.h): argument marshalling only.

Every computation runs in the CUDA library; this module checks tensor devices / dtypes,
turns torch tensors into pointers and strides, and raises ``KvkError`` on a non-OK status.
There is no fallback: if ``libkvk.so`` is missing or a call fails, an exception is raised.

Low-level functions carry the C names (``kvk_create_layout``, ``kvk_quant_write``,
``kvk_mla_decode``, ...); ``Layout`` wraps them for convenience.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvk.so")

KVK_OK = 0
STATUS_NAMES = {0: "KVK_OK", 1: "KVK_ERR_INVALID_ARG", 2: "KVK_ERR_BAD_TABLE",
                3: "KVK_ERR_BUDGET", 4: "KVK_ERR_INHERITING_LAYER", 5: "KVK_ERR_WORKSPACE",
                6: "KVK_ERR_ALIGNMENT", 7: "KVK_ERR_CUDA", 8: "KVK_ERR_UNSUPPORTED"}
KVK_F32, KVK_BF16, KVK_F16 = 0, 1, 2
KVK_PATH_AUTO, KVK_PATH_TENSOR, KVK_PATH_CUDA_CORE, KVK_PATH_TENSOR_GENERAL = 0, 1, 2, 3
KVK_FLAG_NONFINITE, KVK_FLAG_WRITE_RANGE, KVK_FLAG_SEQ_LEN, KVK_FLAG_KEEP_INDEX = 1, 2, 4, 8
KVK_FLAG_TIMEOUT = 16

_DTYPE = {torch.float32: KVK_F32, torch.bfloat16: KVK_BF16, torch.float16: KVK_F16}

# every symbol the header declares
EXPORTED = ("kvk_create_layout", "kvk_destroy", "kvk_get_layer_info", "kvk_quant_write",
            "kvk_decode_workspace_bytes", "kvk_mla_decode", "kvk_read_status",
            "kvk_set_decode_path", "kvk_set_decode_ctas", "kvk_decode_path_for",
            "kvk_status_string", "kvk_mla_decode_noalloc", "kvk_quant_write_layers",
            "kvk_decode_workspace_bytes_keep", "kvk_set_wait_limit", "kvk_mla_decode_append",
            "kvk_create_layout_grouped", "kvk_absorb")

# size of the library's built-in scratch array used by kvk_mla_decode_noalloc
KVK_NOALLOC_SCRATCH_BYTES = 32 << 20


class KvkError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = _lib_handle().kvk_status_string(status).decode() if _LIB else ""
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)} ({msg})")


class LayerInfo(ctypes.Structure):
    _fields_ = [("anchor", ctypes.c_int32), ("d", ctypes.c_int32), ("b", ctypes.c_int32),
                ("row_bytes", ctypes.c_int32), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("codes_offset", ctypes.c_int64),
                ("scales_offset", ctypes.c_int64), ("max_batch", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("r", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("scales_per_token", ctypes.c_int32), ("scale_group", ctypes.c_int32)]


_LIB = None


def _lib_handle():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.kvk_create_layout.argtypes = [i32, P, P, P, i32, i32, i32, i32, i64, P, sz, P, P, P]
        L.kvk_create_layout_grouped.argtypes = [i32, P, P, P, i32, i32, i32, i32, i32, i64, P,
                                                sz, P, P, P]
        L.kvk_absorb.argtypes = [P, i32, i64, i64, P, i64, i64, P, i32, i64, i64, i32, i32, i32,
                                 i32, P]
        L.kvk_destroy.argtypes = [P]
        L.kvk_destroy.restype = None
        L.kvk_get_layer_info.argtypes = [P, i32, P]
        L.kvk_quant_write.argtypes = [P, i32, P, i32, i64, i64, P, i64, i64, i32, P, i32, P]
        L.kvk_quant_write_layers.argtypes = [P, i32, P, P, i32, P, P, P, P, P, i32, P, i32, P]
        L.kvk_decode_workspace_bytes.argtypes = [P, i32, i32, i32, P]
        L.kvk_decode_workspace_bytes_keep.argtypes = [P, i32, i32, i32, i32, P]
        L.kvk_mla_decode.argtypes = [P, i32, P, P, i32, i64, i64, i64, i64, i32, i32, P, P, P,
                                     i32, ctypes.c_float, P, P, P, sz, P]
        L.kvk_mla_decode_append.argtypes = [P, i32, P, P, i32, i64, i64, P, P, i32, i64, i64, i64,
                                            i64, i32, i32, P, ctypes.c_float, P, P, P, sz, P]
        L.kvk_mla_decode_noalloc.argtypes = [P, i32, P, P, i32, i64, i64, i64, i64, i32, i32,
                                             P, P, P, i32, ctypes.c_float, P, P, P]
        L.kvk_read_status.argtypes = [P, P, i32, P]
        L.kvk_set_decode_path.argtypes = [P, i32]
        L.kvk_set_decode_ctas.argtypes = [P, i32]
        L.kvk_set_wait_limit.argtypes = [P, ctypes.c_uint64]
        L.kvk_decode_path_for.argtypes = [P, i32, i32, i32, i32, P]
        L.kvk_status_string.argtypes = [i32]
        L.kvk_status_string.restype = ctypes.c_char_p
        for name in EXPORTED:
            if name not in ("kvk_destroy", "kvk_status_string"):
                getattr(L, name).restype = i32
        _LIB = L
    return _LIB


def _check(fn, status):
    if status != KVK_OK:
        raise KvkError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _i32_array(xs):
    return (ctypes.c_int32 * len(xs))(*[int(x) for x in xs])


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(t, name, dtypes=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")


# ---------------------------------------------------------------------------
# C-named functions
# ---------------------------------------------------------------------------

def kvk_create_layout(anchor, d, b, r, d_rope, max_batch, max_tokens, budget_bits_per_token=0,
                      arena=None, query_only=False, scale_group=0):
    """Returns (handle or None, arena_bytes_needed, bits_per_token).  scale_group > 0 calls
    kvk_create_layout_grouped (one fp16 scale per scale_group elements)."""
    L = _lib_handle()
    n = len(anchor)
    need = ctypes.c_size_t(0)
    bits = ctypes.c_int64(0)
    handle = ctypes.c_void_p()
    if arena is not None:
        _need_cuda(arena, "arena")
    common = (_ptr(arena), 0 if arena is None else arena.numel() * arena.element_size(),
              None if query_only else ctypes.byref(handle), ctypes.byref(need), ctypes.byref(bits))
    if scale_group:
        st = L.kvk_create_layout_grouped(n, _i32_array(anchor), _i32_array(d), _i32_array(b), r,
                                         d_rope, scale_group, max_batch, max_tokens,
                                         int(budget_bits_per_token), *common)
        _check("kvk_create_layout_grouped", st)
    else:
        st = L.kvk_create_layout(n, _i32_array(anchor), _i32_array(d), _i32_array(b), r, d_rope,
                                 max_batch, max_tokens, int(budget_bits_per_token), *common)
        _check("kvk_create_layout", st)
    return (None if query_only else handle), need.value, bits.value


def kvk_destroy(handle):
    if handle:
        _lib_handle().kvk_destroy(handle)


def kvk_get_layer_info(handle, layer) -> dict:
    info = LayerInfo()
    _check("kvk_get_layer_info", _lib_handle().kvk_get_layer_info(handle, layer, ctypes.byref(info)))
    return {f: getattr(info, f) for f, _ in LayerInfo._fields_}


def kvk_quant_write(handle, layer, c_kv, k_rope, start_pos, stream=None):
    """c_kv [B, n_new, >=d], k_rope [B, n_new, d_rope] (fp32 or bf16, CUDA, last dim
    contiguous); start_pos int32 [B] on the device."""
    _need_cuda(c_kv, "c_kv", (torch.float32, torch.bfloat16))
    _need_cuda(k_rope, "k_rope", (c_kv.dtype,))
    _need_cuda(start_pos, "start_pos", (torch.int32,))
    if c_kv.dim() != 3 or k_rope.dim() != 3 or c_kv.stride(2) != 1 or k_rope.stride(2) != 1:
        raise ValueError("c_kv / k_rope must be [batch, n_new, width] with contiguous width")
    B, n_new = c_kv.shape[0], c_kv.shape[1]
    st = _lib_handle().kvk_quant_write(handle, layer, _ptr(c_kv), _DTYPE[c_kv.dtype],
                                       c_kv.stride(0), c_kv.stride(1), _ptr(k_rope),
                                       k_rope.stride(0), k_rope.stride(1), B, _ptr(start_pos),
                                       n_new, _stream(stream))
    _check("kvk_quant_write", st)


def kvk_quant_write_layers(handle, layers, c_kvs, k_ropes, start_pos, stream=None):
    """kvk_quant_write for several anchor layers in one launch: layers[k] takes c_kvs[k]
    [B, n_new, >=d] and k_ropes[k] [B, n_new, d_rope] (same dtype, batch and n_new for all)."""
    n = len(layers)
    if not (len(c_kvs) == len(k_ropes) == n) or n == 0:
        raise ValueError("layers, c_kvs and k_ropes must have the same non-zero length")
    for c_kv, k_rope in zip(c_kvs, k_ropes):
        _need_cuda(c_kv, "c_kv", (torch.float32, torch.bfloat16))
        _need_cuda(k_rope, "k_rope", (c_kvs[0].dtype,))
        if c_kv.dim() != 3 or k_rope.dim() != 3 or c_kv.stride(2) != 1 or k_rope.stride(2) != 1:
            raise ValueError("c_kv / k_rope must be [batch, n_new, width] with contiguous width")
        if c_kv.dtype != c_kvs[0].dtype or c_kv.shape[:2] != c_kvs[0].shape[:2]:
            raise ValueError("every layer needs the same dtype, batch and n_new")
    B, n_new = c_kvs[0].shape[0], c_kvs[0].shape[1]
    _need_cuda(start_pos, "start_pos", (torch.int32,))
    I32 = ctypes.c_int32 * n
    I64 = ctypes.c_int64 * n
    VP = ctypes.c_void_p * n
    st = _lib_handle().kvk_quant_write_layers(
        handle, n, I32(*layers), VP(*[_ptr(t) for t in c_kvs]), _DTYPE[c_kvs[0].dtype],
        I64(*[t.stride(0) for t in c_kvs]), I64(*[t.stride(1) for t in c_kvs]),
        VP(*[_ptr(t) for t in k_ropes]), I64(*[t.stride(0) for t in k_ropes]),
        I64(*[t.stride(1) for t in k_ropes]), B, _ptr(start_pos), n_new, _stream(stream))
    _check("kvk_quant_write_layers", st)


def kvk_decode_workspace_bytes(handle, layer, batch, n_heads) -> int:
    out = ctypes.c_size_t(0)
    _check("kvk_decode_workspace_bytes",
           _lib_handle().kvk_decode_workspace_bytes(handle, layer, batch, n_heads,
                                                    ctypes.byref(out)))
    return out.value


def kvk_decode_workspace_bytes_keep(handle, layer, batch, n_heads, keep_stride) -> int:
    out = ctypes.c_size_t(0)
    _check("kvk_decode_workspace_bytes_keep",
           _lib_handle().kvk_decode_workspace_bytes_keep(handle, layer, batch, n_heads,
                                                         keep_stride, ctypes.byref(out)))
    return out.value


def kvk_mla_decode(handle, layer, q_lat, q_rope, seq_lens, softmax_scale, out, workspace,
                   lse=None, keep_idx=None, keep_len=None, stream=None):
    """q_lat [B, H, >=d], q_rope [B, H, d_rope] (same dtype, CUDA, last dim contiguous);
    seq_lens int32 [B]; keep_idx int32 [B, K] + keep_len int32 [B] (optional);
    out fp32 [B, H, d]; lse fp32 [B, H] (optional); workspace uint8 CUDA tensor."""
    _need_cuda(q_lat, "q_lat", tuple(_DTYPE))
    _need_cuda(q_rope, "q_rope", (q_lat.dtype,))
    _need_cuda(seq_lens, "seq_lens", (torch.int32,))
    _need_cuda(out, "out", (torch.float32,))
    _need_cuda(lse, "lse", (torch.float32,))
    _need_cuda(keep_idx, "keep_idx", (torch.int32,))
    _need_cuda(keep_len, "keep_len", (torch.int32,))
    _need_cuda(workspace, "workspace")
    if q_lat.stride(2) != 1 or q_rope.stride(2) != 1:
        raise ValueError("q_lat / q_rope last dim must be contiguous")
    if not out.is_contiguous() or (lse is not None and not lse.is_contiguous()):
        raise ValueError("out / lse must be contiguous")
    if keep_idx is not None and keep_idx.stride(1) != 1:
        raise ValueError("keep_idx rows must be contiguous")
    B, H = q_lat.shape[0], q_lat.shape[1]
    st = _lib_handle().kvk_mla_decode(
        handle, layer, _ptr(q_lat), _ptr(q_rope), _DTYPE[q_lat.dtype], q_lat.stride(0),
        q_lat.stride(1), q_rope.stride(0), q_rope.stride(1), B, H, _ptr(seq_lens),
        _ptr(keep_idx), _ptr(keep_len), 0 if keep_idx is None else keep_idx.stride(0),
        float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("kvk_mla_decode", st)


def kvk_mla_decode_append(handle, layer, c_new, k_rope_new, q_lat, q_rope, seq_lens,
                          softmax_scale, out, workspace, lse=None, stream=None):
    """Append each sequence's new token (c_new [B, >=d], k_rope_new [B, d_rope], fp32 or bf16)
    at position seq_lens[i] - 1 of the anchor layer's cache and decode over the cache that
    includes it (one launch on the tensor-core kernel).  Other arguments as kvk_mla_decode."""
    _need_cuda(c_new, "c_new", (torch.float32, torch.bfloat16))
    _need_cuda(k_rope_new, "k_rope_new", (c_new.dtype,))
    _need_cuda(q_lat, "q_lat", tuple(_DTYPE))
    _need_cuda(q_rope, "q_rope", (q_lat.dtype,))
    _need_cuda(seq_lens, "seq_lens", (torch.int32,))
    _need_cuda(out, "out", (torch.float32,))
    _need_cuda(lse, "lse", (torch.float32,))
    _need_cuda(workspace, "workspace")
    if c_new.dim() != 2 or k_rope_new.dim() != 2 or c_new.stride(1) != 1 or \
            k_rope_new.stride(1) != 1:
        raise ValueError("c_new / k_rope_new must be [batch, width] with contiguous width")
    if q_lat.stride(2) != 1 or q_rope.stride(2) != 1:
        raise ValueError("q_lat / q_rope last dim must be contiguous")
    if not out.is_contiguous() or (lse is not None and not lse.is_contiguous()):
        raise ValueError("out / lse must be contiguous")
    B, H = q_lat.shape[0], q_lat.shape[1]
    st = _lib_handle().kvk_mla_decode_append(
        handle, layer, _ptr(c_new), _ptr(k_rope_new), _DTYPE[c_new.dtype], c_new.stride(0),
        k_rope_new.stride(0), _ptr(q_lat), _ptr(q_rope), _DTYPE[q_lat.dtype], q_lat.stride(0),
        q_lat.stride(1), q_rope.stride(0), q_rope.stride(1), B, H, _ptr(seq_lens),
        float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("kvk_mla_decode_append", st)


def kvk_mla_decode_noalloc(handle, layer, q_lat, q_rope, seq_lens, softmax_scale, out,
                           lse=None, keep_idx=None, keep_len=None, stream=None):
    """kvk_mla_decode with the library's built-in scratch instead of a workspace tensor,
    for callers that cannot allocate device memory (see include/kvk.h).  Same tensor rules
    as kvk_mla_decode."""
    _need_cuda(q_lat, "q_lat", tuple(_DTYPE))
    _need_cuda(q_rope, "q_rope", (q_lat.dtype,))
    _need_cuda(seq_lens, "seq_lens", (torch.int32,))
    _need_cuda(out, "out", (torch.float32,))
    _need_cuda(lse, "lse", (torch.float32,))
    _need_cuda(keep_idx, "keep_idx", (torch.int32,))
    _need_cuda(keep_len, "keep_len", (torch.int32,))
    if q_lat.stride(2) != 1 or q_rope.stride(2) != 1:
        raise ValueError("q_lat / q_rope last dim must be contiguous")
    if not out.is_contiguous() or (lse is not None and not lse.is_contiguous()):
        raise ValueError("out / lse must be contiguous")
    B, H = q_lat.shape[0], q_lat.shape[1]
    st = _lib_handle().kvk_mla_decode_noalloc(
        handle, layer, _ptr(q_lat), _ptr(q_rope), _DTYPE[q_lat.dtype], q_lat.stride(0),
        q_lat.stride(1), q_rope.stride(0), q_rope.stride(1), B, H, _ptr(seq_lens),
        _ptr(keep_idx), _ptr(keep_len), 0 if keep_idx is None else keep_idx.stride(0),
        float(softmax_scale), _ptr(out), _ptr(lse), _stream(stream))
    _check("kvk_mla_decode_noalloc", st)


def kvk_absorb(x, w, y, stream=None):
    """y[b, h, j] = sum_k x[b, h, k] * w[h, k, j] on the tensor cores.  x [B, H, K] (bf16 or
    fp32, last dim contiguous), w [H, K, >= n] bf16 (rows contiguous), y [B, H, n] (bf16 or
    fp32, last dim contiguous); n = y.shape[2]."""
    _need_cuda(x, "x", (torch.bfloat16, torch.float32))
    _need_cuda(w, "w", (torch.bfloat16,))
    _need_cuda(y, "y", (torch.bfloat16, torch.float32))
    if x.stride(2) != 1 or w.stride(2) != 1 or y.stride(2) != 1:
        raise ValueError("x, w and y need a contiguous last dim")
    B, H, K = x.shape
    n = y.shape[2]
    if tuple(y.shape[:2]) != (B, H) or w.shape[0] != H or w.shape[1] < K or w.shape[2] < n:
        raise ValueError("shapes of x [B, H, K], w [H, >=K, >=n] and y [B, H, n] do not match")
    st = _lib_handle().kvk_absorb(_ptr(x), _DTYPE[x.dtype], x.stride(0), x.stride(1), _ptr(w),
                                  w.stride(1), w.stride(0), _ptr(y), _DTYPE[y.dtype], y.stride(0),
                                  y.stride(1), B, H, K, n, _stream(stream))
    _check("kvk_absorb", st)
    return y


def kvk_read_status(handle, clear=False, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check("kvk_read_status", _lib_handle().kvk_read_status(handle, ctypes.byref(v),
                                                            1 if clear else 0, _stream(stream)))
    return v.value


def kvk_set_decode_path(handle, path):
    _check("kvk_set_decode_path", _lib_handle().kvk_set_decode_path(handle, path))


def kvk_set_decode_ctas(handle, ctas):
    _check("kvk_set_decode_ctas", _lib_handle().kvk_set_decode_ctas(handle, ctas))


def kvk_set_wait_limit(handle, ns):
    _check("kvk_set_wait_limit", _lib_handle().kvk_set_wait_limit(handle, int(ns)))


def kvk_decode_path_for(handle, layer, dtype, n_heads, has_keep=False) -> int:
    p = ctypes.c_int(0)
    _check("kvk_decode_path_for", _lib_handle().kvk_decode_path_for(
        handle, layer, _DTYPE.get(dtype, dtype), n_heads, 1 if has_keep else 0, ctypes.byref(p)))
    return p.value


def kvk_status_string(status) -> str:
    return _lib_handle().kvk_status_string(status).decode()


# ---------------------------------------------------------------------------
# convenience wrapper
# ---------------------------------------------------------------------------

class Layout:
    """A per-layer plan plus its arena (a CUDA uint8 tensor owned by this object unless
    one is passed in)."""

    def __init__(self, anchor, d, b, r, d_rope, max_batch, max_tokens, budget_bits_per_token=0,
                 arena=None, device="cuda", scale_group=0):
        self.anchor, self.d, self.b = list(anchor), list(d), list(b)
        self.r, self.d_rope = r, d_rope
        self.max_batch, self.max_tokens = max_batch, max_tokens
        self.scale_group = scale_group
        _, need, bits = kvk_create_layout(anchor, d, b, r, d_rope, max_batch, max_tokens,
                                          budget_bits_per_token, query_only=True,
                                          scale_group=scale_group)
        self.arena_bytes, self.bits_per_token = need, bits
        if arena is None:
            arena = torch.empty(need, dtype=torch.uint8, device=device)
        self.arena = arena
        self.handle, _, _ = kvk_create_layout(anchor, d, b, r, d_rope, max_batch, max_tokens,
                                              budget_bits_per_token, arena=arena,
                                              scale_group=scale_group)

    @staticmethod
    def query(anchor, d, b, r, d_rope, max_batch, max_tokens, budget_bits_per_token=0,
              scale_group=0):
        _, need, bits = kvk_create_layout(anchor, d, b, r, d_rope, max_batch, max_tokens,
                                          budget_bits_per_token, query_only=True,
                                          scale_group=scale_group)
        return need, bits

    @property
    def n_layers(self):
        return len(self.anchor)

    def layer_info(self, layer):
        return kvk_get_layer_info(self.handle, layer)

    def cache_views(self, layer):
        """(codes uint8 [max_batch, max_tokens, row_bytes], scales fp16 [max_batch, max_tokens]
        -- [max_batch, max_tokens, scales_per_token] for a group-scaled anchor) views of the
        arena for the layer's anchor."""
        info = self.layer_info(layer)
        T = self.max_batch * self.max_tokens
        co, so, sg = info["codes_offset"], info["scales_offset"], info["scales_per_token"]
        codes = self.arena[co:co + T * info["row_bytes"]].view(self.max_batch, self.max_tokens,
                                                               info["row_bytes"])
        scales = self.arena[so:so + 2 * T * sg].view(torch.float16)
        if sg == 1:
            scales = scales.view(self.max_batch, self.max_tokens)
        else:
            scales = scales.view(self.max_batch, self.max_tokens, sg)
        return codes, scales

    def quant_write(self, layer, c_kv, k_rope, start_pos, stream=None):
        kvk_quant_write(self.handle, layer, c_kv, k_rope, start_pos, stream)

    def quant_write_layers(self, layers, c_kvs, k_ropes, start_pos, stream=None):
        kvk_quant_write_layers(self.handle, layers, c_kvs, k_ropes, start_pos, stream)

    def workspace_bytes(self, layer, batch, n_heads, keep_stride=None):
        """keep_stride: the row stride of a keep list the calls will pass (None: no keep
        list), so that such calls can take the tensor-core kernel."""
        if keep_stride is None:
            return kvk_decode_workspace_bytes(self.handle, layer, batch, n_heads)
        return kvk_decode_workspace_bytes_keep(self.handle, layer, batch, n_heads, keep_stride)

    def new_workspace(self, layer, batch, n_heads, keep_stride=None):
        return torch.empty(self.workspace_bytes(layer, batch, n_heads, keep_stride),
                           dtype=torch.uint8, device=self.arena.device)

    def mla_decode(self, layer, q_lat, q_rope, seq_lens, softmax_scale, out=None, lse=None,
                   workspace=None, keep_idx=None, keep_len=None, stream=None):
        B, H = q_lat.shape[0], q_lat.shape[1]
        d = self.layer_info(layer)["d"]
        if out is None:
            out = torch.empty(B, H, d, dtype=torch.float32, device=q_lat.device)
        if workspace is None:
            workspace = self.new_workspace(
                layer, B, H, None if keep_idx is None else keep_idx.stride(0))
        kvk_mla_decode(self.handle, layer, q_lat, q_rope, seq_lens, softmax_scale, out,
                       workspace, lse=lse, keep_idx=keep_idx, keep_len=keep_len, stream=stream)
        return out

    def mla_decode_append(self, layer, c_new, k_rope_new, q_lat, q_rope, seq_lens, softmax_scale,
                          out=None, lse=None, workspace=None, stream=None):
        B, H = q_lat.shape[0], q_lat.shape[1]
        d = self.layer_info(layer)["d"]
        if out is None:
            out = torch.empty(B, H, d, dtype=torch.float32, device=q_lat.device)
        if workspace is None:
            workspace = self.new_workspace(layer, B, H)
        kvk_mla_decode_append(self.handle, layer, c_new, k_rope_new, q_lat, q_rope, seq_lens,
                              softmax_scale, out, workspace, lse=lse, stream=stream)
        return out

    def read_status(self, clear=False, stream=None):
        return kvk_read_status(self.handle, clear, stream)

    def set_decode_path(self, path):
        kvk_set_decode_path(self.handle, path)

    def set_decode_ctas(self, ctas):
        kvk_set_decode_ctas(self.handle, ctas)

    def set_wait_limit(self, ns):
        kvk_set_wait_limit(self.handle, ns)

    def decode_path_for(self, layer, dtype, n_heads, has_keep=False):
        return kvk_decode_path_for(self.handle, layer, dtype, n_heads, has_keep)

    def close(self):
        if getattr(self, "handle", None):
            kvk_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
