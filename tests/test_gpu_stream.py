"""Layer-pipelined host streaming: bit-identical to the resident path (same
kernels, same data), within tolerance of the oracle, and a copy failure
injected on the host (no device fault) returns KVQ_ERR_COPY."""
import os

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_long_b200 import workload as wl

from helpers import assert_attn_close, fill_both, q_all

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from quantized_kv_long_b200 import kvq as m
    return m


def _setup(kvq, n_layers=5, n_kv=5000, cap=5008, T=1):
    w = wl.small(wl.WORKLOADS["stream262k"], n_kv=n_kv, n_layers=n_layers, T=T)
    layers = list(range(n_layers))
    dev, orc = fill_both(w, layers, n_kv, cap)
    host = kvq.QuantizedKVCache(n_layers, w.n_kv_heads, w.head_dim, cap, device="cpu", pin=True)
    for l in layers:
        host.k[l].copy_(dev.k[l].cpu())
        host.v[l].copy_(dev.v[l].cpu())
    slots = kvq.QuantizedKVCache(2, w.n_kv_heads, w.head_dim, n_kv + (-n_kv) % 8)
    q = torch.from_numpy(q_all(w, layers, T)).cuda()
    return w, dev, orc, host, slots, q


def _resident(kvq, w, dev, q, n_kv, chunk, T):
    L, Hq, D = len(dev.k), w.n_q_heads, w.head_dim
    C = -(-n_kv // chunk)
    op = torch.empty((L, T, Hq, C, D), device="cuda")
    lp = torch.empty((L, T, Hq, C), device="cuda")
    out = torch.empty((L, T, Hq, D), device="cuda")
    lse = torch.empty((L, T, Hq), device="cuda")
    for l in range(L):  # the same per-layer calls the streamed path makes
        kvq.kvq_decode_attn(dev.layer(l), q[l], Hq, T, n_kv, chunk, w.scale, op[l], lp[l])
        kvq.kvq_merge_lse(op[l], lp[l], T * Hq, C, D, out[l], lse[l])
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def _streamed(kvq, w, host, slots, q, n_kv, chunk, T):
    L, Hq, D = host.n_layers, w.n_q_heads, w.head_dim
    C = -(-n_kv // chunk)
    op = torch.empty((T, Hq, C, D), device="cuda")
    lp = torch.empty((T, Hq, C), device="cuda")
    out = torch.full((L, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((L, T, Hq), float("nan"), device="cuda")
    copy = torch.cuda.Stream()
    kvq.kvq_stream_decode(host, slots, q, Hq, T, n_kv, chunk, w.scale, op, lp, out, lse,
                          compute=torch.cuda.current_stream(), copy=copy)
    kvq.kvq_check()
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("T", [1, 4])
def test_streamed_equals_resident_and_oracle(kvq, T):
    n_kv, chunk = 5000, 1024
    w, dev, orc, host, slots, q = _setup(kvq, T=T)
    so, sl = _streamed(kvq, w, host, slots, q, n_kv, chunk, T)
    ro, rl = _resident(kvq, w, dev, q, n_kv, chunk, T)
    assert np.array_equal(so, ro) and np.array_equal(sl, rl)
    qn = q.cpu().numpy()
    for l in range(host.n_layers):
        p, pl = oracle.decode_attn(orc[l][0], orc[l][1], qn[l], n_kv, chunk, w.scale)
        mo, ml = oracle.merge_lse(p, pl)
        assert_attn_close(so[l], sl[l], mo, ml, f"streamed layer {l}")


def test_injected_copy_failure(kvq):
    n_kv, chunk = 5000, 1024
    w, dev, orc, host, slots, q = _setup(kvq, n_layers=4)
    Hq, D = w.n_q_heads, w.head_dim
    C = -(-n_kv // chunk)
    op = torch.empty((1, Hq, C, D), device="cuda")
    lp = torch.empty((1, Hq, C), device="cuda")
    out = torch.full((4, 1, Hq, D), float("nan"), device="cuda")
    lse = torch.full((4, 1, Hq), float("nan"), device="cuda")
    with kvq.test_hooks(stream_fail_layer=2), pytest.raises(kvq.KvqError) as e:
        kvq.kvq_stream_decode(host, slots, q, Hq, 1, n_kv, chunk, w.scale, op, lp, out, lse,
                              compute=torch.cuda.current_stream(), copy=torch.cuda.Stream())
    assert e.value.status == kvq.KVQ_ERR_COPY
    kvq.kvq_check()  # the work already enqueued completes; the context stays usable
    o = out.cpu().numpy()
    assert np.isfinite(o[:2]).all() and np.isnan(o[2:]).all()
    so, sl = _streamed(kvq, w, host, slots, q, n_kv, chunk, 1)
    assert np.isfinite(so).all()


def test_pageable_host_memory_rejected(kvq):
    w, dev, orc, host, slots, q = _setup(kvq, n_layers=1, n_kv=64, cap=64)
    pageable = kvq.QuantizedKVCache(1, w.n_kv_heads, w.head_dim, 64, device="cpu")
    Hq, D = w.n_q_heads, w.head_dim
    op = torch.empty((1, Hq, 1, D), device="cuda")
    lp = torch.empty((1, Hq, 1), device="cuda")
    out = torch.empty((1, 1, Hq, D), device="cuda")
    lse = torch.empty((1, 1, Hq), device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_stream_decode(pageable, slots, q, Hq, 1, 64, 64, w.scale, op, lp, out, lse,
                              compute=torch.cuda.current_stream(), copy=torch.cuda.Stream())
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG


def _mixed(kvq, dev, host, pattern):
    """Layer l from device memory where pattern[l] == 'D', from pinned host memory where 'H'."""
    return [dev.layer(l) if c == "D" else host.layer(l) for l, c in enumerate(pattern)]


@pytest.mark.parametrize("pattern", ["DDHHH", "HDHDH", "DDDDH"])
def test_resident_layers_mixed_with_streamed(kvq, pattern):
    """A resident prefix (the plan kvq_resident_layers makes), an interleaving and a
    single streamed layer: bit-identical to the all-resident path."""
    n_kv, chunk, T = 5000, 1024, 4
    w, dev, orc, host, slots, q = _setup(kvq, T=T)
    Hq, D = w.n_q_heads, w.head_dim
    C = -(-n_kv // chunk)
    op = torch.empty((T, Hq, C, D), device="cuda")
    lp = torch.empty((T, Hq, C), device="cuda")
    out = torch.full((5, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((5, T, Hq), float("nan"), device="cuda")
    kvq.kvq_stream_decode(_mixed(kvq, dev, host, pattern), slots, q, Hq, T, n_kv, chunk, w.scale,
                          op, lp, out, lse, compute=torch.cuda.current_stream(),
                          copy=torch.cuda.Stream())
    kvq.kvq_check()
    ro, rl = _resident(kvq, w, dev, q, n_kv, chunk, T)
    assert np.array_equal(out.cpu().numpy(), ro) and np.array_equal(lse.cpu().numpy(), rl)


def test_all_resident_needs_no_slots(kvq):
    n_kv, chunk = 5000, 1024
    w, dev, orc, host, slots, q = _setup(kvq, n_layers=3)
    Hq, D = w.n_q_heads, w.head_dim
    C = -(-n_kv // chunk)
    op = torch.empty((1, Hq, C, D), device="cuda")
    lp = torch.empty((1, Hq, C), device="cuda")
    out = torch.full((3, 1, Hq, D), float("nan"), device="cuda")
    lse = torch.full((3, 1, Hq), float("nan"), device="cuda")
    kvq.kvq_stream_decode(dev.layers(), None, q, Hq, 1, n_kv, chunk, w.scale, op, lp, out, lse,
                          compute=torch.cuda.current_stream(), copy=torch.cuda.Stream())
    kvq.kvq_check()
    ro, rl = _resident(kvq, w, dev, q, n_kv, chunk, 1)
    assert np.array_equal(out.cpu().numpy(), ro) and np.array_equal(lse.cpu().numpy(), rl)
    # a streamed layer without slots is refused before anything is enqueued
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_stream_decode(_mixed(kvq, dev, host, "DHD"), None, q, Hq, 1, n_kv, chunk,
                              w.scale, op, lp, out, lse, compute=torch.cuda.current_stream(),
                              copy=torch.cuda.Stream())
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG


def test_split_placement_rejected(kvq):
    """K on the device and V in host memory (or the reverse) is not a valid layer."""
    n_kv, chunk = 64, 64
    w, dev, orc, host, slots, q = _setup(kvq, n_layers=1, n_kv=n_kv, cap=64)
    Hq, D = w.n_q_heads, w.head_dim
    bad = [kvq.kvq_layer(dev.k[0].data_ptr(), host.v[0].data_ptr(), 64, w.n_kv_heads, D)]
    op = torch.empty((1, Hq, 1, D), device="cuda")
    lp = torch.empty((1, Hq, 1), device="cuda")
    out = torch.empty((1, 1, Hq, D), device="cuda")
    lse = torch.empty((1, 1, Hq), device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_stream_decode(bad, slots, q, Hq, 1, n_kv, chunk, w.scale, op, lp, out, lse,
                              compute=torch.cuda.current_stream(), copy=torch.cuda.Stream())
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
