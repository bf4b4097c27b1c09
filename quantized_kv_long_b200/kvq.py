"""Thin ctypes binding of ``libkvq.so`` (the C ABI in ``include/kvq.h``).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Functions keep the C names; tensors are passed as their data
pointers (``torch.Tensor`` or a raw integer address), streams as
``torch.cuda.Stream`` (default: torch's current stream).  A non-OK status
raises :class:`KvqError` with the library's message.

The library is loaded when this module is imported; if ``libkvq.so`` has not
been built, the import fails loudly -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libkvq.so is not built ({LIB_PATH}); run __graft_entry__.build() or "
                      "python -m quantized_kv_long_b200.build")

_lib = ctypes.CDLL(LIB_PATH)

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = 1
KVQ_ERR_ALIGNMENT = 2
KVQ_ERR_UNSUPPORTED = 3
KVQ_ERR_CUDA = 4
KVQ_ERR_TIMEOUT = 5
KVQ_ERR_COPY = 6
KVQ_ERR_WORKSPACE = 7
KVQ_OP_DECODE = 1
KVQ_OP_PREFILL = 2
KVQ_OP_DECODE_STEP = 3
KVQ_MAX_LAYERS = 64
KVQ_MAX_DECODE_T = 4
KVQ_STATIC_SCRATCH_BYTES = 8 << 20

QK, Q8_0_BYTES, Q4_0_BYTES = 32, 34, 18
QK_OSCAR2, OSCAR2_BYTES = 128, 36
KVQ_TYPE_DEFAULT, KVQ_TYPE_Q8_0, KVQ_TYPE_Q4_0, KVQ_TYPE_OSCAR2 = 0, 1, 2, 3


def _resolve(kvq_type: int, tensor: str) -> int:
    if kvq_type == KVQ_TYPE_DEFAULT:
        return KVQ_TYPE_Q8_0 if tensor == "k" else KVQ_TYPE_Q4_0
    return kvq_type


def block_bytes(kvq_type: int, tensor: str) -> int:
    """Bytes per block of a cache tensor ('k' or 'v') in ``kvq_type``."""
    return {KVQ_TYPE_Q8_0: Q8_0_BYTES, KVQ_TYPE_Q4_0: Q4_0_BYTES,
            KVQ_TYPE_OSCAR2: OSCAR2_BYTES}[_resolve(kvq_type, tensor)]


def block_elems(kvq_type: int, tensor: str) -> int:
    """Elements per block of a cache tensor ('k' or 'v') in ``kvq_type``."""
    return QK_OSCAR2 if _resolve(kvq_type, tensor) == KVQ_TYPE_OSCAR2 else QK


def row_bytes(kvq_type: int, tensor: str, head_dim: int) -> int:
    """Bytes of one head-row of a cache tensor ('k' or 'v') in ``kvq_type``."""
    return head_dim // block_elems(kvq_type, tensor) * block_bytes(kvq_type, tensor)


class kvq_layer(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("capacity", ctypes.c_int64),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("k_type", ctypes.c_int32), ("v_type", ctypes.c_int32)]


class kvq_test_hooks(ctypes.Structure):
    _fields_ = [("decode_general", ctypes.c_int32), ("decode_timeout", ctypes.c_int32),
                ("prefill_timeout", ctypes.c_int32), ("stream_fail_layer", ctypes.c_int32)]


class KvqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} [{status}: {kvq_status_string(status)}]")
        self.status = status


_P, _I32, _I64, _F32, _SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
_LP = ctypes.POINTER(kvq_layer)
_SIGS = {
    "kvq_quantize_q8_0": ([_P, _P, _I64, _P], _I32),
    "kvq_quantize_q4_0": ([_P, _P, _I64, _P], _I32),
    "kvq_quantize_oscar2": ([_P, _P, _I64, _P], _I32),
    "kvq_append": ([_LP, _I32, _P, _P, _I64, _I32, _P], _I32),
    "kvq_decode_attn": ([_LP, _I32, _P, _I32, _I32, _I64, _I32, _F32, _P, _P, _P], _I32),
    "kvq_merge_lse": ([_P, _P, _I64, _I32, _I32, _P, _P, _P], _I32),
    "kvq_decode_attn_shard": ([_LP, _I32, _P, _I32, _I32, _I64, _I64, _I64, _I32, _F32, _P, _P,
                               _P], _I32),
    "kvq_merge_lse_parts": ([_P, _P, _I32, _I64, _I32, _P, _P, _P], _I32),
    "kvq_decode_step": ([_LP, _I32, _P, _P, _P, _I32, _I32, _I64, _I32, _F32, _P, _P, _P, _P, _P,
                         _SZ, _P], _I32),
    "kvq_decode_step_host": ([_LP, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I64, _I32,
                              _F32, _P, _P, _P, _P, _P], _I32),
    "kvq_prefill_attn": ([_LP, _I32, _P, _I32, _I32, _I64, _I32, _F32, _P, _P, _P, _P, _P, _SZ,
                          _P], _I32),
    "kvq_stream_decode": ([_LP, _I32, _LP, _P, _I32, _I32, _I64, _I32, _F32, _P, _P, _P, _P, _P,
                           _P], _I32),
    "kvq_decode_merged_static": ([_LP, _I32, _P, _I32, _I32, _I64, _I32, _F32, _P, _P, _P],
                                 _I32),
    "kvq_resident_layers": ([_SZ, _I32, _I64, _I32, _I32, _I32, _I32], _I32),
    "kvq_prefill_workspace_bytes": ([_I32, _I32, _I32, _I64], _SZ),
    "kvq_workspace_bytes": ([_I32, _I32, _I32, _I32, _I32, _I32], _SZ),
    "kvq_check": ([_P], _I32),
    "kvq_status_string": ([_I32], ctypes.c_char_p),
    "kvq_last_error": ([], ctypes.c_char_p),
    "kvq_version": ([], _I32),
    "kvq_test_set_hooks": ([ctypes.POINTER(kvq_test_hooks)], _I32),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _layers(layers) -> tuple[ctypes.Array, int]:
    if isinstance(layers, QuantizedKVCache):
        layers = layers.layers()
    if isinstance(layers, kvq_layer):
        layers = [layers]
    arr = (kvq_layer * len(layers))(*layers)
    return arr, len(layers)


def _check(status: int) -> None:
    if status != KVQ_OK:
        raise KvqError(status, kvq_last_error())


def kvq_status_string(status: int) -> str:
    return _lib.kvq_status_string(status).decode()


def kvq_last_error() -> str:
    return _lib.kvq_last_error().decode()


def kvq_version() -> int:
    return _lib.kvq_version()


def kvq_quantize_q8_0(x, blocks, n: int | None = None, stream=None) -> None:
    n = x.numel() if n is None else n
    _check(_lib.kvq_quantize_q8_0(_ptr(x), _ptr(blocks), n, _stream(stream)))


def kvq_quantize_q4_0(x, blocks, n: int | None = None, stream=None) -> None:
    n = x.numel() if n is None else n
    _check(_lib.kvq_quantize_q4_0(_ptr(x), _ptr(blocks), n, _stream(stream)))


def kvq_quantize_oscar2(x, blocks, n: int | None = None, stream=None) -> None:
    n = x.numel() if n is None else n
    _check(_lib.kvq_quantize_oscar2(_ptr(x), _ptr(blocks), n, _stream(stream)))


def kvq_append(layers, k_new, v_new, pos: int, n_tok: int, stream=None) -> None:
    arr, n = _layers(layers)
    _check(_lib.kvq_append(arr, n, _ptr(k_new), _ptr(v_new), pos, n_tok, _stream(stream)))


def kvq_decode_attn(layers, q, n_q_heads: int, T: int, n_kv: int, chunk: int, scale: float,
                    out_part, lse_part, stream=None) -> None:
    arr, n = _layers(layers)
    _check(_lib.kvq_decode_attn(arr, n, _ptr(q), n_q_heads, T, n_kv, chunk, scale,
                                _ptr(out_part), _ptr(lse_part), _stream(stream)))


def kvq_merge_lse(out_part, lse_part, rows: int, n_chunks: int, head_dim: int, out, lse,
                  stream=None) -> None:
    _check(_lib.kvq_merge_lse(_ptr(out_part), _ptr(lse_part), rows, n_chunks, head_dim,
                              _ptr(out), _ptr(lse), _stream(stream)))


def kvq_decode_attn_shard(layers, q, n_q_heads: int, T: int, n_keys: int, key0: int, n_kv: int,
                          chunk: int, scale: float, out_part, lse_part, stream=None) -> None:
    """Decode over keys [key0, key0 + n_keys) of an n_kv-key context (see include/kvq.h)."""
    arr, n = _layers(layers)
    _check(_lib.kvq_decode_attn_shard(arr, n, _ptr(q), n_q_heads, T, n_keys, key0, n_kv, chunk,
                                      scale, _ptr(out_part), _ptr(lse_part), _stream(stream)))


def kvq_merge_lse_parts(out_parts, lse_parts, n_parts: int, rows: int, head_dim: int, out, lse,
                        stream=None) -> None:
    """Merge part-major partials [n_parts][rows][head_dim] (see include/kvq.h)."""
    _check(_lib.kvq_merge_lse_parts(_ptr(out_parts), _ptr(lse_parts), n_parts, rows, head_dim,
                                    _ptr(out), _ptr(lse), _stream(stream)))


def kvq_decode_step(layers, k_new, v_new, q, n_q_heads: int, T: int, n_kv: int, chunk: int,
                    scale: float, out_part, lse_part, out, lse, workspace=None, ws_bytes: int = 0,
                    stream=None) -> None:
    """Append + decode + merge as three launches on ``stream`` (see include/kvq.h);
    ``workspace`` is reserved and not read."""
    arr, n = _layers(layers)
    _check(_lib.kvq_decode_step(arr, n, _ptr(k_new), _ptr(v_new), _ptr(q), n_q_heads, T, n_kv,
                                chunk, scale, _ptr(out_part), _ptr(lse_part), _ptr(out), _ptr(lse),
                                _ptr(workspace), ws_bytes, _stream(stream)))


def kvq_decode_step_host(layers, k_host, v_host, q_host, out_host, lse_host, k_new, v_new, q,
                         n_q_heads: int, T: int, n_kv: int, chunk: int, scale: float, out_part,
                         lse_part, out, lse, stream=None) -> None:
    """kvq_decode_step with inputs and results in (pinned) host tensors; the device
    tensors k_new, v_new, q, out_part, lse_part, out, lse are the copies' targets and
    the step's buffers (see include/kvq.h)."""
    arr, n = _layers(layers)
    _check(_lib.kvq_decode_step_host(arr, n, _ptr(k_host), _ptr(v_host), _ptr(q_host),
                                     _ptr(out_host), _ptr(lse_host), _ptr(k_new), _ptr(v_new),
                                     _ptr(q), n_q_heads, T, n_kv, chunk, scale, _ptr(out_part),
                                     _ptr(lse_part), _ptr(out), _ptr(lse), _stream(stream)))


def kvq_prefill_attn(layers, q, n_q_heads: int, T: int, n_cached: int, page: int, scale: float,
                     out, lse, page_out=None, page_lse=None, workspace=None, ws_bytes: int = 0,
                     stream=None) -> None:
    arr, n = _layers(layers)
    if workspace is not None and not ws_bytes and isinstance(workspace, torch.Tensor):
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.kvq_prefill_attn(arr, n, _ptr(q), n_q_heads, T, n_cached, page, scale,
                                 _ptr(out), _ptr(lse), _ptr(page_out), _ptr(page_lse),
                                 _ptr(workspace), ws_bytes, _stream(stream)))


def kvq_stream_decode(host_layers, dev_slots, q, n_q_heads: int, T: int, n_kv: int, chunk: int,
                      scale: float, out_part, lse_part, out, lse, compute=None,
                      copy=None) -> None:
    harr, n = _layers(host_layers)
    if dev_slots is None:
        sarr = None
    else:
        sarr, ns = _layers(dev_slots)
        if ns != 2:
            raise ValueError("dev_slots must hold exactly 2 layers")
    _check(_lib.kvq_stream_decode(harr, n, sarr, _ptr(q), n_q_heads, T, n_kv, chunk, scale,
                                  _ptr(out_part), _ptr(lse_part), _ptr(out), _ptr(lse),
                                  _stream(compute), _stream(copy)))


def kvq_decode_merged_static(layers, q, n_q_heads: int, T: int, n_kv: int, chunk: int,
                             scale: float, out, lse, stream=None) -> None:
    """Decode + merge with the chunk partials in the library's own static device
    array (for callers that cannot allocate); see include/kvq.h for the limit."""
    arr, n = _layers(layers)
    _check(_lib.kvq_decode_merged_static(arr, n, _ptr(q), n_q_heads, T, n_kv, chunk, scale,
                                         _ptr(out), _ptr(lse), _stream(stream)))


def kvq_resident_layers(budget_bytes: int, n_layers: int, capacity: int, n_kv_heads: int,
                        head_dim: int, k_type: int = 0, v_type: int = 0) -> int:
    return _lib.kvq_resident_layers(budget_bytes, n_layers, capacity, n_kv_heads, head_dim,
                                    k_type, v_type)


def kvq_prefill_workspace_bytes(n_layers: int, n_kv_heads: int, head_dim: int,
                                n_keys: int) -> int:
    return _lib.kvq_prefill_workspace_bytes(n_layers, n_kv_heads, head_dim, n_keys)


def kvq_workspace_bytes(op: int, n_layers: int, n_q_heads: int, n_kv_heads: int, T: int,
                        head_dim: int) -> int:
    return _lib.kvq_workspace_bytes(op, n_layers, n_q_heads, n_kv_heads, T, head_dim)


def kvq_test_set_hooks(decode_general: bool = False, decode_timeout: bool = False,
                       prefill_timeout: bool = False, stream_fail_layer: int = -1) -> None:
    """Set the library's process-wide test hooks (all off by default)."""
    h = kvq_test_hooks(int(decode_general), int(decode_timeout), int(prefill_timeout),
                       stream_fail_layer)
    _check(_lib.kvq_test_set_hooks(ctypes.byref(h)))


class test_hooks:
    """Context manager: the given test hooks on inside the block, all off after it."""

    def __init__(self, **kw):
        self.kw = kw

    def __enter__(self):
        kvq_test_set_hooks(**self.kw)
        return self

    def __exit__(self, *exc):
        _check(_lib.kvq_test_set_hooks(None))
        return False


def kvq_check(stream=None) -> None:
    _check(_lib.kvq_check(_stream(stream)))


class QuantizedKVCache:
    """Caller-owned cache memory in the library's layout (torch allocates it).

    K of layer ``l``: uint8 ``[n_kv_heads, capacity, head_dim // 32 * 34]``;
    V: ``[n_kv_heads, capacity, head_dim // 32 * 18]`` (the default Q8_0 K /
    Q4_0 V; ``k_type`` / ``v_type`` select another block format per tensor:
    Q8_0, Q4_0 or OSCAR2, ``head_dim // 128 * 36`` bytes per head-row).
    ``device="cpu"`` with ``pin=True`` gives pinned host memory for
    :func:`kvq_stream_decode`.
    """

    def __init__(self, n_layers: int, n_kv_heads: int, head_dim: int, capacity: int,
                 device="cuda", pin: bool = False, k_type: int = KVQ_TYPE_DEFAULT,
                 v_type: int = KVQ_TYPE_DEFAULT):
        if capacity % 8:
            raise ValueError("capacity must be a multiple of 8")
        self.n_layers, self.n_kv_heads, self.head_dim, self.capacity = (
            n_layers, n_kv_heads, head_dim, capacity)
        self.k_type, self.v_type = k_type, v_type
        kb = row_bytes(k_type, "k", head_dim)
        vb = row_bytes(v_type, "v", head_dim)
        kw = dict(dtype=torch.uint8, device=device)
        if pin:
            kw["pin_memory"] = True
        self.k = [torch.empty((n_kv_heads, capacity, kb), **kw) for _ in range(n_layers)]
        self.v = [torch.empty((n_kv_heads, capacity, vb), **kw) for _ in range(n_layers)]

    def layer(self, l: int) -> kvq_layer:
        return kvq_layer(self.k[l].data_ptr(), self.v[l].data_ptr(), self.capacity,
                         self.n_kv_heads, self.head_dim, self.k_type, self.v_type)

    def layers(self, start: int = 0, stop: int | None = None) -> list[kvq_layer]:
        stop = self.n_layers if stop is None else stop
        return [self.layer(l) for l in range(start, stop)]

    @property
    def nbytes(self) -> int:
        return sum(t.numel() for t in self.k) + sum(t.numel() for t in self.v)


def make_layers(ks: Sequence[torch.Tensor], vs: Sequence[torch.Tensor], capacity: int,
                n_kv_heads: int, head_dim: int, k_type: int = KVQ_TYPE_DEFAULT,
                v_type: int = KVQ_TYPE_DEFAULT) -> list[kvq_layer]:
    return [kvq_layer(k.data_ptr(), v.data_ptr(), capacity, n_kv_heads, head_dim, k_type, v_type)
            for k, v in zip(ks, vs)]
