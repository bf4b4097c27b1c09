"""Helpers shared by the GPU parity tests: caches built on both sides from
the same seeded inputs, and the tolerance checks.

Tolerances (written here once, used by every attention parity test):
  * out: max |gpu - oracle| <= 2e-3 (absolute, fp32 output vs fp64 oracle);
  * lse: |gpu - oracle| <= 1e-4 * max(|oracle|, 1) (relative, natural log);
  * quantized blocks: bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_kv_long_b200 import workload as wl

OUT_ATOL = 2e-3
LSE_RTOL = 1e-4


def assert_attn_close(out, lse, ref_out, ref_lse, what=""):
    out = np.asarray(out, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    ref_out = np.asarray(ref_out)
    ref_lse = np.asarray(ref_lse)
    masked = ref_lse == -np.inf
    assert (lse[masked] == -np.inf).all(), f"{what}: masked partials must have lse = -inf"
    assert (out[masked] == 0).all(), f"{what}: masked partials must be 0"
    live = ~masked
    if live.any():
        err = np.abs(out[live] - ref_out[live]).max()
        assert err <= OUT_ATOL, f"{what}: out max-abs error {err:.3e} > {OUT_ATOL}"
        den = np.maximum(np.abs(ref_lse[live]), 1.0)
        lerr = (np.abs(lse[live] - ref_lse[live]) / den).max()
        assert lerr <= LSE_RTOL, f"{what}: lse relative error {lerr:.3e} > {LSE_RTOL}"


def oracle_fmt(kvq, kvq_type: int, tensor: str) -> int:
    """The oracle's block format for a kvq_type of a cache tensor ('k' or 'v')."""
    if kvq_type == kvq.KVQ_TYPE_DEFAULT:
        return oracle.FMT_Q8_0 if tensor == "k" else oracle.FMT_Q4_0
    return {kvq.KVQ_TYPE_Q8_0: oracle.FMT_Q8_0, kvq.KVQ_TYPE_Q4_0: oracle.FMT_Q4_0,
            kvq.KVQ_TYPE_OSCAR2: oracle.FMT_OSCAR2}[kvq_type]


def fill_both(w: wl.Workload, layers, n_rows: int, capacity: int, device="cuda", k_type=0,
              v_type=0):
    """Quantize rows [0, n_rows) of the given layers on the GPU (through
    kvq_append) and on the CPU (oracle), K and V in the given block formats
    (0 = the default Q8_0 K / Q4_0 V).  Returns (gpu cache, oracle caches)."""
    from quantized_kv_long_b200 import kvq
    cache = kvq.QuantizedKVCache(len(layers), w.n_kv_heads, w.head_dim, capacity, device=device,
                                 k_type=k_type, v_type=v_type)
    orc = []
    for i, l in enumerate(layers):
        k = wl.kv_rows(w, l, 0, 0, n_rows)
        v = wl.kv_rows(w, l, 1, 0, n_rows)
        kt = torch.from_numpy(k).to(device)
        vt = torch.from_numpy(v).to(device)
        kvq.kvq_append(cache.layer(i), kt, vt, 0, n_rows)
        kc, vc = oracle.empty_cache(w.n_kv_heads, w.head_dim, capacity,
                                    k_fmt=oracle_fmt(kvq, k_type, "k"),
                                    v_fmt=oracle_fmt(kvq, v_type, "v"))
        oracle.append(kc, vc, k, v, 0)
        orc.append((kc, vc))
    torch.cuda.synchronize()
    return cache, orc


def q_all(w: wl.Workload, layers, T: int | None = None) -> np.ndarray:
    return np.stack([wl.q_rows(w, l, T) for l in layers])
