"""CPU oracle for attention over a Q8_0-K / Q4_0-V cache -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference legs may import this package.  It wraps ``kvq_oracle.c`` (plain
C, fp32 quantizers, fp64 attention) through ctypes; it never imports the CUDA
library and the CUDA library never imports it.  The definitions it implements,
and the readings taken where the quantized-KV pages are silent, are listed in
the header of ``kvq_oracle.c``.

Every function here takes and returns numpy arrays.  Caches use the layout of
one layer: K ``[n_kv_heads, capacity, head_dim // 32 * 34]`` uint8 and V
``[n_kv_heads, capacity, head_dim // 32 * 18]`` uint8 in the main (Q8_0 K /
Q4_0 V) configuration; either tensor may use another block format
(``empty_cache(..., k_fmt=, v_fmt=)``: Q8_0, Q4_0 or the INT2 OSCAR2 block of
36 bytes per 128 elements), and the functions read each tensor's format from
its head-row length and the head_dim of their other inputs (at a given
head_dim the three formats give three different row lengths).

Parity pins: every function below is pinned by the CPU tests (golden blocks,
closed forms, library cross-checks, invariants); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, library_path

QK = 32
Q8_0_BYTES = 34
Q4_0_BYTES = 18
QK_OSCAR2 = 128
OSCAR2_BYTES = 36
FMT_Q8_0, FMT_Q4_0, FMT_OSCAR2 = 1, 2, 3
_BLOCK_BYTES = {FMT_Q8_0: Q8_0_BYTES, FMT_Q4_0: Q4_0_BYTES, FMT_OSCAR2: OSCAR2_BYTES}
_BLOCK_ELEMS = {FMT_Q8_0: QK, FMT_Q4_0: QK, FMT_OSCAR2: QK_OSCAR2}

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(
            os.path.join(os.path.dirname(__file__), "kvq_oracle.c")):
        build_oracle()
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    sigs = {
        "orc_num_threads": ([], i32),
        "orc_f32_to_f16": ([P, P, i64], None),
        "orc_f16_to_f64": ([P, P, i64], None),
        "orc_quantize_q8_0": ([P, P, i64], None),
        "orc_quantize_q4_0": ([P, P, i64], None),
        "orc_dequant_q8_0": ([P, P, i64], None),
        "orc_dequant_q4_0": ([P, P, i64], None),
        "orc_quantize_oscar2": ([P, P, i64], None),
        "orc_dequant_oscar2": ([P, P, i64], None),
        "orc_append": ([P, P, i32, i32, i64, P, P, i64, i64, i32, i32], None),
        "orc_decode_attn": ([P, P, i32, i32, i64, P, i32, i32, i64, i64, f64, P, P, i32, i32],
                            None),
        "orc_merge_lse": ([P, P, i64, i32, i32, P, P], None),
        "orc_attn_rows": ([P, P, i32, i32, i64, P, P, i32, P, P, i64, f64, P, P, i32, i32],
                          None),
        "orc_prefill_attn": ([P, P, i32, i32, i64, P, i32, i32, i64, i64, f64, P, P, P, P, i32,
                              i32], None),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags.c_contiguous
    return a.ctypes.data


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return _load().orc_num_threads()


# ---- fp16 -----------------------------------------------------------------

def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().orc_f32_to_f16(_ptr(x), _ptr(out), x.size)
    return out


def f16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float64)
    _load().orc_f16_to_f64(_ptr(h), _ptr(out), h.size)
    return out


# ---- quantizers -------------------------------------------------------------

def _quant(fn, nbytes, x, elems=QK):
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.size % elems:
        raise ValueError(f"element count must be a multiple of {elems}")
    out = np.empty(x.size // elems * nbytes, dtype=np.uint8)
    fn(_ptr(x), _ptr(out), x.size)
    return out


def quantize_q8_0(x: np.ndarray) -> np.ndarray:
    """Q8_0 blocks (34 B per 32 elements) of ``x`` in memory order."""
    return _quant(_load().orc_quantize_q8_0, Q8_0_BYTES, x)


def quantize_q4_0(x: np.ndarray) -> np.ndarray:
    """Q4_0 blocks (18 B per 32 elements) of ``x`` in memory order."""
    return _quant(_load().orc_quantize_q4_0, Q4_0_BYTES, x)


def quantize_oscar2(x: np.ndarray) -> np.ndarray:
    """OSCAR2 INT2 blocks (36 B per 128 elements) of ``x`` in memory order."""
    return _quant(_load().orc_quantize_oscar2, OSCAR2_BYTES, x, QK_OSCAR2)


def _dequant(fn, nbytes, b, elems=QK):
    b = np.ascontiguousarray(b, dtype=np.uint8).reshape(-1)
    if b.size % nbytes:
        raise ValueError("byte count must be a multiple of the block size")
    out = np.empty(b.size // nbytes * elems, dtype=np.float64)
    fn(_ptr(b), _ptr(out), out.size)
    return out


def dequant_q8_0(b: np.ndarray) -> np.ndarray:
    return _dequant(_load().orc_dequant_q8_0, Q8_0_BYTES, b)


def dequant_q4_0(b: np.ndarray) -> np.ndarray:
    return _dequant(_load().orc_dequant_q4_0, Q4_0_BYTES, b)


def dequant_oscar2(b: np.ndarray) -> np.ndarray:
    return _dequant(_load().orc_dequant_oscar2, OSCAR2_BYTES, b, QK_OSCAR2)


# ---- cache ------------------------------------------------------------------

def empty_cache(n_kv_heads: int, head_dim: int, capacity: int, k_fmt: int = FMT_Q8_0,
                v_fmt: int = FMT_Q4_0):
    """Zeroed K and V byte arrays of one layer (K blocks in ``k_fmt``, V in ``v_fmt``)."""
    for f in (k_fmt, v_fmt):
        if head_dim % _BLOCK_ELEMS[f]:
            raise ValueError(f"head_dim {head_dim} is not a multiple of the block size")
    k = np.zeros((n_kv_heads, capacity, head_dim // _BLOCK_ELEMS[k_fmt] * _BLOCK_BYTES[k_fmt]),
                 dtype=np.uint8)
    v = np.zeros((n_kv_heads, capacity, head_dim // _BLOCK_ELEMS[v_fmt] * _BLOCK_BYTES[v_fmt]),
                 dtype=np.uint8)
    return k, v


def _fmt_of(row_bytes: int, head_dim: int) -> int:
    """Block format of a head-row of ``row_bytes`` at ``head_dim``: at one head_dim the
    formats' row lengths (34, 18 and 9 bytes per 32 elements) all differ."""
    fits = [f for f in _BLOCK_BYTES
            if head_dim % _BLOCK_ELEMS[f] == 0
            and head_dim // _BLOCK_ELEMS[f] * _BLOCK_BYTES[f] == row_bytes]
    if len(fits) != 1:
        raise ValueError(f"no block format has {row_bytes}-byte head-rows at head_dim {head_dim}")
    return fits[0]


def _cache_dims(k_cache, v_cache, head_dim: int):
    """(n_kv_heads, capacity, k_fmt, v_fmt) of one layer's caches read at ``head_dim``."""
    H, cap, kb = k_cache.shape
    assert v_cache.shape[:2] == (H, cap)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    return H, cap, _fmt_of(kb, head_dim), _fmt_of(v_cache.shape[2], head_dim)


def append(k_cache, v_cache, k_new, v_new, pos: int) -> None:
    """Quantize rows ``k_new``/``v_new`` ``[n_tok, n_kv_heads, head_dim]`` into rows
    ``[pos, pos + n_tok)`` of the caches, in place."""
    k_new = np.ascontiguousarray(k_new, dtype=np.float32)
    v_new = np.ascontiguousarray(v_new, dtype=np.float32)
    n_tok, h2, D = k_new.shape
    H, cap, k_fmt, v_fmt = _cache_dims(k_cache, v_cache, D)
    if h2 != H or v_new.shape != k_new.shape or pos < 0 or pos + n_tok > cap:
        raise ValueError("bad append shape")
    _load().orc_append(_ptr(k_cache), _ptr(v_cache), H, D, cap, _ptr(k_new), _ptr(v_new),
                       pos, n_tok, k_fmt, v_fmt)


# ---- attention --------------------------------------------------------------

def decode_attn(k_cache, v_cache, q: np.ndarray, n_kv: int, chunk: int, scale: float):
    """Per-chunk partials.  ``q`` fp16 ``[T, n_q_heads, head_dim]``.

    Returns ``(out_part [T, Hq, n_chunks, D] f64, lse_part [T, Hq, n_chunks] f64)``.
    """
    q = np.ascontiguousarray(q, dtype=np.float16)
    T, Hq, D = q.shape
    H, cap, k_fmt, v_fmt = _cache_dims(k_cache, v_cache, D)
    assert Hq % H == 0 and 1 <= T <= n_kv <= cap and chunk >= 1
    n_chunks = -(-n_kv // chunk)
    out = np.empty((T, Hq, n_chunks, D), dtype=np.float64)
    lse = np.empty((T, Hq, n_chunks), dtype=np.float64)
    _load().orc_decode_attn(_ptr(k_cache), _ptr(v_cache), H, D, cap, _ptr(q.view(np.uint16)),
                            Hq, T, n_kv, chunk, scale, _ptr(out), _ptr(lse), k_fmt, v_fmt)
    return out, lse


def merge_lse(out_part: np.ndarray, lse_part: np.ndarray):
    """Merge ``[..., n_chunks, D]`` partials over the chunk axis."""
    out_part = np.ascontiguousarray(out_part, dtype=np.float64)
    lse_part = np.ascontiguousarray(lse_part, dtype=np.float64)
    *lead, C, D = out_part.shape
    assert tuple(lse_part.shape) == (*lead, C)
    rows = int(np.prod(lead)) if lead else 1
    out = np.empty((*lead, D), dtype=np.float64)
    lse = np.empty(tuple(lead), dtype=np.float64)
    _load().orc_merge_lse(_ptr(out_part), _ptr(lse_part), rows, C, D, _ptr(out), _ptr(lse))
    return out, lse


def attn_rows(k_cache, v_cache, q_rows: np.ndarray, q_head: np.ndarray, n_q_heads: int,
              key_begin: np.ndarray, key_end: np.ndarray, scale: float):
    """One-pass attention of arbitrary rows (fp16 ``q_rows [n, D]``)."""
    q_rows = np.ascontiguousarray(q_rows, dtype=np.float16)
    n, D = q_rows.shape
    H, cap, k_fmt, v_fmt = _cache_dims(k_cache, v_cache, D)
    q_head = np.ascontiguousarray(q_head, dtype=np.int32)
    kb = np.ascontiguousarray(key_begin, dtype=np.int64)
    ke = np.ascontiguousarray(key_end, dtype=np.int64)
    assert q_rows.shape == (n, D) and q_head.shape == kb.shape == ke.shape == (n,)
    assert (kb >= 0).all() and (ke <= cap).all()
    out = np.empty((n, D), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    _load().orc_attn_rows(_ptr(k_cache), _ptr(v_cache), H, D, cap,
                          _ptr(q_rows.view(np.uint16)), _ptr(q_head), n_q_heads, _ptr(kb),
                          _ptr(ke), n, scale, _ptr(out), _ptr(lse), k_fmt, v_fmt)
    return out, lse


def prefill_attn(k_cache, v_cache, q: np.ndarray, n_cached: int, page: int, scale: float,
                 pages: bool = False):
    """Prefill of ``T`` new tokens over ``n_cached + T`` keys (causal tail).

    Returns ``(out [T, Hq, D], lse [T, Hq])`` and, with ``pages=True``, also
    ``(page_out [T, Hq, n_pages, D], page_lse [T, Hq, n_pages])``.
    """
    q = np.ascontiguousarray(q, dtype=np.float16)
    T, Hq, D = q.shape
    H, cap, k_fmt, v_fmt = _cache_dims(k_cache, v_cache, D)
    assert n_cached + T <= cap and Hq % H == 0
    n_pages = -(-(n_cached + T) // page)
    out = np.empty((T, Hq, D), dtype=np.float64)
    lse = np.empty((T, Hq), dtype=np.float64)
    po = np.empty((T, Hq, n_pages, D), dtype=np.float64) if pages else None
    pl = np.empty((T, Hq, n_pages), dtype=np.float64) if pages else None
    _load().orc_prefill_attn(_ptr(k_cache), _ptr(v_cache), H, D, cap,
                             _ptr(q.view(np.uint16)), Hq, T, n_cached, page, scale, _ptr(out),
                             _ptr(lse), _ptr(po), _ptr(pl), k_fmt, v_fmt)
    return (out, lse, po, pl) if pages else (out, lse)
