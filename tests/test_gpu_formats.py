"""Other block formats of the cache (Q8_0 or Q4_0 for each of K and V, the
choices of the KV-cache guide's levers section, and the OSCAR2 page's INT2
block) on the GPU, against the oracle.

The default pair (Q8_0 K / Q4_0 V) is covered by the other GPU tests; here
five other pairs go through append (bit-exact cache bytes), the general
decode kernel and the merge (tolerances of helpers.py), the decode step
(bit-identical to the separate calls), the streamed decode (bit-identical to
the resident one) and prefill (the exact kernel, which serves every pair).
"""
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


# (k_type, v_type): q8_0/q8_0, q4_0/q4_0, q4_0/q8_0, oscar2/oscar2 (the OSCAR2 page's
# cache), q8_0/oscar2
PAIRS = [(1, 1), (2, 2), (2, 1), (3, 3), (1, 3)]


@pytest.mark.parametrize("k_type,v_type", PAIRS)
def test_append_and_decode(kvq, k_type, v_type):
    n_kv, chunk, T = 3001, 1024, 4
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=n_kv)
    layers = [0, 1]
    cap = -(-n_kv // 8) * 8
    cache, orc = fill_both(w, layers, n_kv, cap, k_type=k_type, v_type=v_type)
    for i in range(len(layers)):  # quantized bytes of the written rows: bit-exact
        assert np.array_equal(cache.k[i].cpu().numpy()[:, :n_kv], orc[i][0][:, :n_kv])
        assert np.array_equal(cache.v[i].cpu().numpy()[:, :n_kv], orc[i][1][:, :n_kv])
    q = q_all(w, layers, T)
    Hq, D = w.n_q_heads, w.head_dim
    C = -(-n_kv // chunk)
    op = torch.full((2, T, Hq, C, D), float("nan"), device="cuda")
    lp = torch.full((2, T, Hq, C), float("nan"), device="cuda")
    out = torch.full((2, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((2, T, Hq), float("nan"), device="cuda")
    kvq.kvq_decode_attn(cache, torch.from_numpy(q).cuda(), Hq, T, n_kv, chunk, w.scale, op, lp)
    kvq.kvq_merge_lse(op, lp, 2 * T * Hq, C, D, out, lse)
    kvq.kvq_check()
    for i in range(len(layers)):
        rp, rl = oracle.decode_attn(orc[i][0], orc[i][1], q[i], n_kv, chunk, w.scale)
        assert_attn_close(op[i].cpu().numpy(), lp[i].cpu().numpy(), rp, rl, f"partials {i}")
        ro, rlse = oracle.merge_lse(rp, rl)
        assert_attn_close(out[i].cpu().numpy(), lse[i].cpu().numpy(), ro, rlse, f"merged {i}")


@pytest.mark.parametrize("k_type,v_type", PAIRS)
def test_decode_step_three_launches(kvq, k_type, v_type):
    """kvq_decode_step on these formats appends, decodes and merges in three launches."""
    n_kv, chunk, T = 2050, 512, 4
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=n_kv)
    n0, cap = n_kv - T, -(-n_kv // 8) * 8
    Hq, H, D = w.n_q_heads, w.n_kv_heads, w.head_dim
    C = -(-n_kv // chunk)
    ca, _ = fill_both(w, [0], n0, cap, k_type=k_type, v_type=v_type)
    cb, _ = fill_both(w, [0], n0, cap, k_type=k_type, v_type=v_type)
    k_new = torch.from_numpy(wl.kv_rows(w, 0, 0, n0, n_kv)[None]).cuda()
    v_new = torch.from_numpy(wl.kv_rows(w, 0, 1, n0, n_kv)[None]).cuda()
    q = torch.from_numpy(q_all(w, [0], T)).cuda()
    outs = []
    for one_call, c in ((False, ca), (True, cb)):
        op = torch.full((1, T, Hq, C, D), float("nan"), device="cuda")
        lp = torch.full((1, T, Hq, C), float("nan"), device="cuda")
        out = torch.full((1, T, Hq, D), float("nan"), device="cuda")
        lse = torch.full((1, T, Hq), float("nan"), device="cuda")
        if one_call:
            kvq.kvq_decode_step(c, k_new, v_new, q, Hq, T, n_kv, chunk, w.scale, op, lp, out,
                                lse)
        else:
            kvq.kvq_append(c, k_new, v_new, n0, T)
            kvq.kvq_decode_attn(c, q, Hq, T, n_kv, chunk, w.scale, op, lp)
            kvq.kvq_merge_lse(op, lp, T * Hq, C, D, out, lse)
        kvq.kvq_check()
        outs.append((c.k[0][:, :n_kv].clone(), c.v[0][:, :n_kv].clone(), op, lp, out, lse))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_streamed_q8_0_values(kvq):
    """q8_0/q8_0 cache in pinned host memory, one layer resident: bit-identical to resident."""
    n_kv, chunk, T = 2000, 512, 1
    w = wl.small(wl.WORKLOADS["stream262k"], n_kv=n_kv, n_layers=3, T=T)
    cap = 2000
    dev, _ = fill_both(w, [0, 1, 2], n_kv, cap, k_type=1, v_type=1)
    host = kvq.QuantizedKVCache(3, w.n_kv_heads, w.head_dim, cap, device="cpu", pin=True,
                                k_type=1, v_type=1)
    for l in range(3):
        host.k[l].copy_(dev.k[l].cpu())
        host.v[l].copy_(dev.v[l].cpu())
    slots = kvq.QuantizedKVCache(2, w.n_kv_heads, w.head_dim, cap, k_type=1, v_type=1)
    Hq, D = w.n_q_heads, w.head_dim
    C = -(-n_kv // chunk)
    q = torch.from_numpy(q_all(w, [0, 1, 2], T)).cuda()
    op = torch.empty((T, Hq, C, D), device="cuda")
    lp = torch.empty((T, Hq, C), device="cuda")
    out = torch.full((3, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((3, T, Hq), float("nan"), device="cuda")
    layers = [dev.layer(0), host.layer(1), host.layer(2)]
    kvq.kvq_stream_decode(layers, slots, q, Hq, T, n_kv, chunk, w.scale, op, lp, out, lse,
                          compute=torch.cuda.current_stream(), copy=torch.cuda.Stream())
    kvq.kvq_check()
    for l in range(3):
        op2 = torch.empty((T, Hq, C, D), device="cuda")
        lp2 = torch.empty((T, Hq, C), device="cuda")
        o2 = torch.empty((T, Hq, D), device="cuda")
        l2 = torch.empty((T, Hq), device="cuda")
        kvq.kvq_decode_attn(dev.layer(l), q[l], Hq, T, n_kv, chunk, w.scale, op2, lp2)
        kvq.kvq_merge_lse(op2, lp2, T * Hq, C, D, o2, l2)
        kvq.kvq_check()
        assert torch.equal(out[l], o2) and torch.equal(lse[l], l2)


@pytest.mark.parametrize("k_type,v_type", PAIRS)
def test_prefill_formats(kvq, k_type, v_type):
    """Prefill on these formats: every row on the exact kernel (the tensor-core path
    is built for Q8_0 K / Q4_0 V), 2 layers, rows seeing 16,100 to 16,139 keys."""
    n_cached, T, L = 16100, 40, 2
    n = n_cached + T
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=n_cached, T=T)
    cache, orc = fill_both(w, list(range(L)), n, -(-n // 8) * 8, k_type=k_type, v_type=v_type)
    q = q_all(w, list(range(L)), T)
    Hq, D = w.n_q_heads, w.head_dim
    out = torch.full((L, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((L, T, Hq), float("nan"), device="cuda")
    kvq.kvq_prefill_attn(cache.layers(), torch.from_numpy(q).cuda(), Hq, T, n_cached, 4096,
                         w.scale, out, lse)
    kvq.kvq_check()
    for l in range(L):
        ro, rl = oracle.prefill_attn(orc[l][0], orc[l][1], q[l], n_cached, 4096, w.scale)
        assert_attn_close(out[l].cpu().numpy(), lse[l].cpu().numpy(), ro, rl, f"layer {l}")
