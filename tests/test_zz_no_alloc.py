"""kvq_decode_merged_static: decode attention + LSE merge for callers that
cannot allocate device memory for the chunk partials (a plug-in inside a host
program that owns all device memory, or a step loop where cudaMalloc is not
allowed).  The partials live in the library's own 8 MiB device array, so the
call takes only inputs and outputs.

Its results must equal those of kvq_decode_attn + kvq_merge_lse (partials in
caller-provided memory) bit for bit -- the same two kernels run in both -- on
two calls in a row with different shapes and data (the array keeps the last
call's contents).  Arguments are checked before the scratch size is worked
out from them.  The file sorts last so that a run that stops at the first
failure has run every other test before it; it also passes on its own.
"""
import numpy as np
import pytest
import torch

from quantized_kv_long_b200 import workload as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from quantized_kv_long_b200 import kvq as m
    return m


def _cache(kvq, w, n_layers, n_kv):
    cap = -(-n_kv // 8) * 8
    cache = kvq.QuantizedKVCache(n_layers, w.n_kv_heads, w.head_dim, cap)
    for l in range(n_layers):
        k = torch.from_numpy(wl.kv_rows(w, l, 0, 0, n_kv)).cuda()
        v = torch.from_numpy(wl.kv_rows(w, l, 1, 0, n_kv)).cuda()
        kvq.kvq_append(cache.layer(l), k, v, 0, n_kv)
    return cache


def _both(kvq, w, n_layers, T, n_kv, chunk):
    cache = _cache(kvq, w, n_layers, n_kv)
    Hq, D = w.n_q_heads, w.head_dim
    q = torch.from_numpy(np.stack([wl.q_rows(w, l, T) for l in range(n_layers)])).cuda()
    C = -(-n_kv // chunk)
    # the existing path: partials in memory the caller allocates
    op = torch.empty((n_layers, T, Hq, C, D), device="cuda")
    lp = torch.empty((n_layers, T, Hq, C), device="cuda")
    ref_out = torch.empty((n_layers, T, Hq, D), device="cuda")
    ref_lse = torch.empty((n_layers, T, Hq), device="cuda")
    kvq.kvq_decode_attn(cache, q, Hq, T, n_kv, chunk, w.scale, op, lp)
    kvq.kvq_merge_lse(op, lp, n_layers * T * Hq, C, D, ref_out, ref_lse)
    # the static-scratch path: only inputs and outputs
    out = torch.full((n_layers, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((n_layers, T, Hq), float("nan"), device="cuda")
    kvq.kvq_decode_merged_static(cache, q, Hq, T, n_kv, chunk, w.scale, out, lse)
    kvq.kvq_check()
    return out, lse, ref_out, ref_lse


def _equal(out, lse, ro, rl, what):
    assert torch.equal(out, ro) and torch.equal(lse, rl), what


def test_static_scratch_matches_caller_scratch_two_calls(kvq):
    # call 1: a 4-token verify batch over 2 layers (ragged last chunk)
    w1 = wl.small(wl.WORKLOADS["verify262k"], n_kv=9001)
    out, lse, ro, rl = _both(kvq, w1, 2, 4, 9001, 1024)
    _equal(out, lse, ro, rl, "static scratch, call 1")
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    # call 2: a different shape and different data in the same array
    w2 = wl.small(wl.WORKLOADS["decode65k"], n_kv=20000)
    out, lse, ro, rl = _both(kvq, w2, 3, 1, 20000, 4096)
    _equal(out, lse, ro, rl, "static scratch, call 2")


def test_static_scratch_refuses_oversize(kvq):
    """16 layers of the 262,144-key verify batch need ~100 MB of partials."""
    w = wl.WORKLOADS["verify262k"]
    A = 1 << 20  # never dereferenced: the size check comes first
    layers = [kvq.kvq_layer(A, A, 262144, 4, 256)] * 16
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_merged_static(layers, A, 24, 4, 262144, 4096, w.scale, A, A)
    assert e.value.status == kvq.KVQ_ERR_UNSUPPORTED
    assert "static scratch" in kvq.kvq_last_error()


def test_static_scratch_validates_before_sizing(kvq):
    """A bad argument is reported as such even where the sizes it implies would not
    fit the scratch: n_kv beyond the layers' capacity (invalid), and a head_dim of 0
    (an unsupported shape, not a scratch overflow)."""
    w = wl.WORKLOADS["verify262k"]
    A = 1 << 20
    over = [kvq.kvq_layer(A, A, 1024, 4, 256)] * 16
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_merged_static(over, A, 24, 4, (1 << 62), 64, w.scale, A, A)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    assert "capacity" in kvq.kvq_last_error()
    bad_dim = [kvq.kvq_layer(A, A, 262144, 4, 0)] * 16
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_merged_static(bad_dim, A, 24, 4, 262144, 64, w.scale, A, A)
    assert e.value.status == kvq.KVQ_ERR_UNSUPPORTED
    assert "head_dim" in kvq.kvq_last_error() and "scratch" not in kvq.kvq_last_error()
