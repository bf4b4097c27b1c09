"""Parity at the full workload sizes, in the launch configuration bench.py
times: all 16 layers filled from the seeded generator, one append + one
16-layer decode + one merge call.  The oracle quantizes two sampled layers
itself (bit-exact against the GPU cache) and computes sampled rows and sampled
chunk partials one by one over the full context."""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_long_b200 import workload as wl

from helpers import assert_attn_close

pytestmark = pytest.mark.gpu

SAMPLED_LAYERS = (0, 11)


def _run_step(kvq, w):
    import bench
    device = torch.device("cuda", 0)
    cache = bench.fill_cache(kvq, torch, w, device)
    L, T, Hq, D, n_kv, C = w.n_layers, w.T, w.n_q_heads, w.head_dim, w.n_kv, w.n_chunks
    q = np.stack([wl.q_rows(w, l) for l in range(L)])
    k_new = np.stack([wl.kv_rows(w, l, 0, n_kv - T, n_kv) for l in range(L)])
    v_new = np.stack([wl.kv_rows(w, l, 1, n_kv - T, n_kv) for l in range(L)])
    layers = cache.layers()
    op = torch.full((L, T, Hq, C, D), float("nan"), device=device)
    lp = torch.full((L, T, Hq, C), float("nan"), device=device)
    out = torch.full((L, T, Hq, D), float("nan"), device=device)
    lse = torch.full((L, T, Hq), float("nan"), device=device)
    kvq.kvq_append(layers, torch.from_numpy(k_new).cuda(), torch.from_numpy(v_new).cuda(),
                   n_kv - T, T)
    kvq.kvq_decode_attn(layers, torch.from_numpy(q).cuda(), Hq, T, n_kv, w.chunk, w.scale, op, lp)
    kvq.kvq_merge_lse(op, lp, L * T * Hq, C, D, out, lse)
    kvq.kvq_check()
    return cache, q, op, lp, out, lse


@pytest.mark.parametrize("name", ["verify262k", "decode65k"])
def test_full_size_sampled(name):
    from quantized_kv_long_b200 import kvq
    w = wl.WORKLOADS[name]
    cache, q, op, lp, out, lse = _run_step(kvq, w)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    assert torch.isfinite(op).all() and not torch.isnan(lp).any()
    T, Hq, n_kv, chunk = w.T, w.n_q_heads, w.n_kv, w.chunk
    rng = np.random.default_rng(123)
    for l in SAMPLED_LAYERS:
        kc, vc = oracle.empty_cache(w.n_kv_heads, w.head_dim, w.capacity)
        oracle.append(kc, vc, wl.kv_rows(w, l, 0, 0, n_kv), wl.kv_rows(w, l, 1, 0, n_kv), 0)
        assert np.array_equal(cache.k[l].cpu().numpy(), kc), f"K cache layer {l}"
        assert np.array_equal(cache.v[l].cpu().numpy(), vc), f"V cache layer {l}"
        # merged rows over the whole context
        ts = rng.integers(0, T, 12)
        hs = rng.integers(0, Hq, 12)
        ro, rl = oracle.attn_rows(kc, vc, q[l, ts, hs], hs, Hq, np.zeros(12),
                                  n_kv - T + ts + 1, w.scale)
        assert_attn_close(out[l, ts, hs].cpu().numpy(), lse[l, ts, hs].cpu().numpy(), ro, rl,
                          f"{name} merged rows layer {l}")
        # chunk partials, including the last (causal) chunk
        cs = np.concatenate([rng.integers(0, w.n_chunks, 10), [w.n_chunks - 1] * 2])
        kb = cs * chunk
        ke = np.minimum((cs + 1) * chunk, n_kv - T + ts + 1)
        po, pl = oracle.attn_rows(kc, vc, q[l, ts, hs], hs, Hq, kb, ke, w.scale)
        assert_attn_close(op[l, ts, hs, cs].cpu().numpy(), lp[l, ts, hs, cs].cpu().numpy(), po,
                          pl, f"{name} chunk partials layer {l}")
