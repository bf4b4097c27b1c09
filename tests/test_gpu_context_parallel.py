"""The context-parallel split's kernels on one GPU: kvq_decode_attn_shard over
shards of a context (each in a cache of its own, as on separate GPUs), each
shard merged over its chunks with kvq_merge_lse, the shards' rows stacked as an
all-gather lays them out, and merged with kvq_merge_lse_parts.

Checked against the oracle's decode + merge of the whole context, on both
decode kernels (the persistent tensor-core kernel and the general one), with
shard boundaries inside the verify batch's causal tail (rows that see part of
a shard, and rows of the first tokens that see none of the last one).  A shard
that is the whole context is bit-identical to kvq_decode_attn.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_long_b200 import workload as wl

from helpers import assert_attn_close, q_all

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from quantized_kv_long_b200 import kvq as m
    return m


def _shard_cache(kvq, w, layers, key0, n_keys):
    """A cache holding keys [key0, key0 + n_keys) of the given layers at rows [0, n_keys)."""
    cache = kvq.QuantizedKVCache(len(layers), w.n_kv_heads, w.head_dim, -(-n_keys // 8) * 8)
    for i, l in enumerate(layers):
        k = torch.from_numpy(wl.kv_rows(w, l, 0, key0, key0 + n_keys)).cuda()
        v = torch.from_numpy(wl.kv_rows(w, l, 1, key0, key0 + n_keys)).cuda()
        kvq.kvq_append(cache.layer(i), k, v, 0, n_keys)
    return cache


def _split(kvq, w, layers, q, T, n_kv, chunk, bounds):
    """Decode + local merge per shard, then the merge over the shards."""
    L, Hq, D = len(layers), w.n_q_heads, w.head_dim
    rows = L * T * Hq
    parts_out = torch.full((len(bounds) - 1, rows, D), float("nan"), device="cuda")
    parts_lse = torch.full((len(bounds) - 1, rows), float("nan"), device="cuda")
    qd = torch.from_numpy(q).cuda()
    for p in range(len(bounds) - 1):
        key0, n_keys = bounds[p], bounds[p + 1] - bounds[p]
        cache = _shard_cache(kvq, w, layers, key0, n_keys)
        C = -(-n_keys // chunk)
        op = torch.empty((rows, C, D), device="cuda")
        lp = torch.empty((rows, C), device="cuda")
        kvq.kvq_decode_attn_shard(cache, qd, Hq, T, n_keys, key0, n_kv, chunk, w.scale, op, lp)
        kvq.kvq_merge_lse(op, lp, rows, C, D, parts_out[p], parts_lse[p])
    out = torch.empty((rows, D), device="cuda")
    lse = torch.empty((rows,), device="cuda")
    kvq.kvq_merge_lse_parts(parts_out, parts_lse, len(bounds) - 1, rows, D, out, lse)
    kvq.kvq_check()
    return out.view(L, T, Hq, D).cpu().numpy(), lse.view(L, T, Hq).cpu().numpy()


@pytest.mark.parametrize("general", [False, True])
@pytest.mark.parametrize("bounds", [
    [0, 4096, 8192, 9001],      # chunk-aligned shards, ragged last chunk
    [0, 3000, 8998, 9001],      # the last shard is the causal tail's last 3 keys:
                                # token 0 sees none of it, token 3 all of it
    [0, 129, 5000, 9001],       # unaligned shards of 129 and 4,871 keys
])
def test_shards_match_oracle(kvq, general, bounds):
    n_kv, T, chunk, layers = 9001, 4, 1024, [0, 1]
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=n_kv)
    q = q_all(w, layers, T)
    with kvq.test_hooks(decode_general=general):
        out, lse = _split(kvq, w, layers, q, T, n_kv, chunk, bounds)
    for i, l in enumerate(layers):
        kc, vc = oracle.empty_cache(w.n_kv_heads, w.head_dim, n_kv)
        oracle.append(kc, vc, wl.kv_rows(w, l, 0, 0, n_kv), wl.kv_rows(w, l, 1, 0, n_kv), 0)
        rp, rl = oracle.decode_attn(kc, vc, q[i], n_kv, chunk, w.scale)
        ro, rlse = oracle.merge_lse(rp, rl)
        assert_attn_close(out[i], lse[i], ro, rlse, f"layer {l}, shards {bounds}")


def test_whole_context_shard_is_decode_attn(kvq):
    """key0 = 0, n_keys = n_kv: the same launch as kvq_decode_attn, bit for bit."""
    n_kv, T, chunk = 5000, 4, 1024
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=n_kv)
    cache = _shard_cache(kvq, w, [0], 0, n_kv)
    q = torch.from_numpy(q_all(w, [0], T)).cuda()
    C, rows, D = -(-n_kv // chunk), T * w.n_q_heads, w.head_dim
    a = [torch.empty((rows, C, D), device="cuda"), torch.empty((rows, C), device="cuda")]
    b = [torch.empty((rows, C, D), device="cuda"), torch.empty((rows, C), device="cuda")]
    kvq.kvq_decode_attn(cache, q, w.n_q_heads, T, n_kv, chunk, w.scale, *a)
    kvq.kvq_decode_attn_shard(cache, q, w.n_q_heads, T, n_kv, 0, n_kv, chunk, w.scale, *b)
    kvq.kvq_check()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_merge_parts_equals_merge_of_transposed(kvq):
    """kvq_merge_lse_parts on [P][rows][D] gives the bits of kvq_merge_lse on the
    same partials laid out [rows][P][D] (the same order of operations)."""
    P, rows, D = 5, 300, 256
    g = torch.Generator().manual_seed(11)
    po = torch.randn((P, rows, D), generator=g)
    pl = torch.randn((P, rows), generator=g) * 4
    pl[1, :50] = float("-inf")   # a masked part
    pl[:, 7] = float("-inf")     # a row with every part masked
    out_a = torch.empty((rows, D), device="cuda")
    lse_a = torch.empty((rows,), device="cuda")
    kvq.kvq_merge_lse_parts(po.cuda(), pl.cuda(), P, rows, D, out_a, lse_a)
    out_b = torch.empty_like(out_a)
    lse_b = torch.empty_like(lse_a)
    kvq.kvq_merge_lse(po.transpose(0, 1).contiguous().cuda(), pl.T.contiguous().cuda(), rows, P,
                      D, out_b, lse_b)
    kvq.kvq_check()
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)
    assert lse_a[7].item() == float("-inf") and (out_a[7] == 0).all()
