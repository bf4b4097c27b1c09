"""Seeded synthetic inputs for quantized-KV long-context attention.

This module only draws numbers: it holds none of the method's arithmetic
(no quantization, no attention, no merge).  Both the CUDA library's tests and
the CPU oracle's tests take their inputs from here, so the two sides see the
same fp32 K/V rows and the same fp16 queries.

Shapes follow the workloads of the quantized-KV pages: a hybrid model whose
16 full-attention layers each hold 4 KV heads of dimension 256 (the "Why it
matters" section of "Adaptive KV streaming lands on ROCm ...": 26,624 bytes per
token for Q8_0 K + Q4_0 V), 24 query heads sharing them in groups of 6 (GQA, as
the KV-cache guide's "why GQA made long context cheap" section describes), and
contexts up to 262,144 tokens.

Recipe (one reading, stated once):

* K and V rows of layer ``l`` are standard normal fp32.  Rows are drawn in
  token blocks of ``TOKEN_BLOCK`` rows; block ``b`` of tensor ``t`` (0 = K,
  1 = V) comes from ``default_rng(SeedSequence([seed, l, t, b]))``, shape
  ``[rows, n_kv_heads, head_dim]``.  Blocks are independent so that a
  262,144-token layer can be drawn by many threads at once.
* Four outlier channels: ``default_rng([seed, 99]).choice(head_dim, 4,
  replace=False)``; those head-dim indices are multiplied by 8 in every
  layer, head and token, for K and V alike.
* Queries of layer ``l``: ``default_rng(SeedSequence([seed, l, 2]))``
  standard normal fp32 of shape ``[T, n_q_heads, head_dim]``, cast to fp16.
* The step's new rows are the last ``T`` rows of each layer's stream, so a
  cache filled with rows ``[0, n_kv)`` already holds them; appending them
  again rewrites the same bytes.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

TOKEN_BLOCK = 16384
N_OUTLIERS = 4
OUTLIER_GAIN = np.float32(8.0)


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: sizes, seed and which step of the path it runs."""

    name: str
    mode: str              # "decode", "prefill" or "stream"
    n_layers: int
    T: int                 # query tokens per layer in one step (appended rows)
    n_kv: int              # decode: keys after the T rows are appended
    n_cached: int = 0      # prefill: keys already cached before the T new rows
    chunk: int = 4096      # split-KV chunk (decode)
    page: int = 16384      # prefill page
    seed: int = 0
    n_q_heads: int = 24
    n_kv_heads: int = 4
    head_dim: int = 256
    scale: float = 1.0 / 16.0
    note: str = field(default="", compare=False)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_keys(self) -> int:
        """Keys visible to the last query token of the step."""
        return self.n_kv if self.mode != "prefill" else self.n_cached + self.T

    @property
    def capacity(self) -> int:
        return self.n_keys

    @property
    def n_chunks(self) -> int:
        return -(-self.n_kv // self.chunk)


# The five workloads of the quantized-KV pages, restated with sizes.
WORKLOADS = {
    "tiny": Workload("tiny", "decode", n_layers=1, T=1, n_kv=1024, chunk=4096, seed=0,
                     note="1 layer, 1 query token, 1,024 context"),
    "decode65k": Workload("decode65k", "decode", n_layers=16, T=1, n_kv=65536, chunk=4096,
                          seed=1, note="16 layers, 1 query token, 65,536 context"),
    "verify262k": Workload("verify262k", "decode", n_layers=16, T=4, n_kv=262144, chunk=4096,
                           seed=2, note="16 layers, 4-token verify batch, 262,144 context"),
    "prefill262k": Workload("prefill262k", "prefill", n_layers=16, T=2048, n_kv=0,
                            n_cached=262144, page=16384, seed=3,
                            note="16 layers, 2,048 new tokens over 262,144 cached"),
    "stream262k": Workload("stream262k", "stream", n_layers=16, T=1, n_kv=262144, chunk=4096,
                           seed=4, note="16 layers host-resident, 262,144 context"),
}


def outlier_channels(seed: int, head_dim: int) -> np.ndarray:
    """Head-dim indices that carry the x8 outliers (sorted for readability)."""
    rng = np.random.default_rng([seed, 99])
    return np.sort(rng.choice(head_dim, N_OUTLIERS, replace=False))


def _kv_block(seed: int, layer: int, tensor: int, block: int, rows: int,
              n_kv_heads: int, head_dim: int, outliers: np.ndarray) -> np.ndarray:
    rng = np.random.default_rng(np.random.SeedSequence([seed, layer, tensor, block]))
    x = rng.standard_normal((rows, n_kv_heads, head_dim), dtype=np.float32)
    x[:, :, outliers] *= OUTLIER_GAIN
    return x


def kv_rows(w: Workload, layer: int, tensor: int, start: int, stop: int,
            threads: int | None = None) -> np.ndarray:
    """fp32 rows ``[start, stop)`` of K (tensor=0) or V (tensor=1) of ``layer``.

    Returns a C-contiguous array ``[stop-start, n_kv_heads, head_dim]``.
    """
    if not (0 <= start <= stop):
        raise ValueError("bad row range")
    outliers = outlier_channels(w.seed, w.head_dim)
    out = np.empty((stop - start, w.n_kv_heads, w.head_dim), dtype=np.float32)
    b0, b1 = start // TOKEN_BLOCK, -(-stop // TOKEN_BLOCK)

    def fill(b: int) -> None:
        lo, hi = b * TOKEN_BLOCK, (b + 1) * TOKEN_BLOCK
        blk = _kv_block(w.seed, layer, tensor, b, TOKEN_BLOCK, w.n_kv_heads, w.head_dim,
                        outliers)
        s, e = max(lo, start), min(hi, stop)
        out[s - start:e - start] = blk[s - lo:e - lo]

    blocks = range(b0, b1)
    if threads is None:
        threads = min(len(blocks), os.cpu_count() or 1)
    if threads <= 1 or len(blocks) <= 1:
        for b in blocks:
            fill(b)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, blocks))
    return out


def q_rows(w: Workload, layer: int, T: int | None = None) -> np.ndarray:
    """fp16 queries ``[T, n_q_heads, head_dim]`` of ``layer``."""
    T = w.T if T is None else T
    rng = np.random.default_rng(np.random.SeedSequence([w.seed, layer, 2]))
    return rng.standard_normal((T, w.n_q_heads, w.head_dim), dtype=np.float32).astype(np.float16)


def small(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some sizes replaced (for reduced parity cases)."""
    d = {f: getattr(w, f) for f in w.__dataclass_fields__}
    d.update(kw)
    return Workload(**d)
