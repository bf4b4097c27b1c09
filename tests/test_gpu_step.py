"""kvq_decode_step (append, decode and merge issued by one call) on the GPU.

The step must give exactly what the three separate calls give: the same
cache bytes, the same chunk partials and the same merged rows, bit for bit,
on cases that put the new rows in one chunk, across a chunk boundary, and
make up the whole cache; one case is also checked against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_long_b200 import workload as wl

from helpers import assert_attn_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from quantized_kv_long_b200 import kvq as m
    return m


def _cache(kvq, w, n_layers, n0, cap):
    cache = kvq.QuantizedKVCache(n_layers, w.n_kv_heads, w.head_dim, cap)
    for l in range(n_layers):
        cache.k[l].zero_()
        cache.v[l].zero_()
        if n0 > 0:
            k = torch.from_numpy(wl.kv_rows(w, l, 0, 0, n0)).cuda()
            v = torch.from_numpy(wl.kv_rows(w, l, 1, 0, n0)).cuda()
            kvq.kvq_append(cache.layer(l), k, v, 0, n0)
    return cache


def _outputs(L, T, Hq, C, D):
    nan = float("nan")
    return (torch.full((L, T, Hq, C, D), nan, device="cuda"),
            torch.full((L, T, Hq, C), nan, device="cuda"),
            torch.full((L, T, Hq, D), nan, device="cuda"),
            torch.full((L, T, Hq), nan, device="cuda"))


def run_both(kvq, w, n_layers, T, n_kv, chunk):
    """The three-call step on one cache and kvq_decode_step on an identical one."""
    cap = -(-n_kv // 8) * 8
    n0 = n_kv - T
    Hq, H, D = w.n_q_heads, w.n_kv_heads, w.head_dim
    C = -(-n_kv // chunk)
    ca = _cache(kvq, w, n_layers, n0, cap)
    cb = _cache(kvq, w, n_layers, n0, cap)
    k_new = torch.from_numpy(np.stack([wl.kv_rows(w, l, 0, n0, n_kv) for l in range(n_layers)])).cuda()
    v_new = torch.from_numpy(np.stack([wl.kv_rows(w, l, 1, n0, n_kv) for l in range(n_layers)])).cuda()
    q = torch.from_numpy(np.stack([wl.q_rows(w, l, T) for l in range(n_layers)])).cuda()
    # three calls
    op_a, lp_a, out_a, lse_a = _outputs(n_layers, T, Hq, C, D)
    kvq.kvq_append(ca, k_new, v_new, n0, T)
    kvq.kvq_decode_attn(ca, q, Hq, T, n_kv, chunk, w.scale, op_a, lp_a)
    kvq.kvq_merge_lse(op_a, lp_a, n_layers * T * Hq, C, D, out_a, lse_a)
    # one call (no workspace)
    op_b, lp_b, out_b, lse_b = _outputs(n_layers, T, Hq, C, D)
    assert kvq.kvq_workspace_bytes(kvq.KVQ_OP_DECODE_STEP, n_layers, Hq, H, T, D) == 0
    kvq.kvq_decode_step(cb, k_new, v_new, q, Hq, T, n_kv, chunk, w.scale, op_b, lp_b, out_b,
                        lse_b)
    kvq.kvq_check()
    for l in range(n_layers):
        assert torch.equal(ca.k[l], cb.k[l]), f"K cache bytes, layer {l}"
        assert torch.equal(ca.v[l], cb.v[l]), f"V cache bytes, layer {l}"
    assert torch.equal(op_a, op_b) and torch.equal(lp_a, lp_b), "chunk partials"
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b), "merged rows"
    return ca, q.cpu().numpy(), out_b.cpu().numpy(), lse_b.cpu().numpy()


def test_step_verify_batch_matches_three_calls(kvq):
    """4 new tokens x 6 heads per KV head, 2 layers, ragged last chunk."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=9001)
    run_both(kvq, w, 2, 4, 9001, 1024)


def test_step_single_token(kvq):
    w = wl.small(wl.WORKLOADS["decode65k"], n_kv=20000)
    run_both(kvq, w, 3, 1, 20000, 4096)


def test_step_new_rows_straddle_chunks(kvq):
    """Rows 4,094..4,097 are new: two in chunk 0 and two in chunk 1."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=4098)
    run_both(kvq, w, 1, 4, 4098, 4096)


def test_step_all_rows_new(kvq):
    """n_kv = T: the whole cache is appended by the step itself (small chunk)."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=4)
    run_both(kvq, w, 2, 4, 4, 64)


def test_step_many_chunks_against_oracle(kvq):
    """chunk 64: 157 partials per row; checked against the oracle too."""
    n_kv, T, chunk = 10000, 4, 64
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=n_kv)
    cache, q, out, lse = run_both(kvq, w, 1, T, n_kv, chunk)
    kc, vc = oracle.empty_cache(w.n_kv_heads, w.head_dim, n_kv)
    oracle.append(kc, vc, wl.kv_rows(w, 0, 0, 0, n_kv), wl.kv_rows(w, 0, 1, 0, n_kv), 0)
    rp, rl = oracle.decode_attn(kc, vc, q[0], n_kv, chunk, w.scale)
    ro, rlse = oracle.merge_lse(rp, rl)
    assert_attn_close(out[0], lse[0], ro, rlse, "decode step vs oracle")


def test_step_general_kernel_path(kvq):
    """The general decode kernel (forced here): the same bit-identity."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=3001)
    with kvq.test_hooks(decode_general=True):
        run_both(kvq, w, 1, 4, 3001, 512)


def test_step_with_host_buffers_matches_device_step(kvq):
    """kvq_decode_step_host: inputs copied from pinned host memory, results copied
    back; the cache bytes and the host results equal the device-buffer step, bit
    for bit, and the device buffers hold the copied inputs."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=5000)
    L, T, n_kv, chunk = 2, 4, 5000, 1024
    cap, n0 = -(-n_kv // 8) * 8, n_kv - T
    Hq, H, D = w.n_q_heads, w.n_kv_heads, w.head_dim
    C = -(-n_kv // chunk)
    ca = _cache(kvq, w, L, n0, cap)
    cb = _cache(kvq, w, L, n0, cap)
    k_h = torch.from_numpy(np.stack([wl.kv_rows(w, l, 0, n0, n_kv) for l in range(L)]))
    v_h = torch.from_numpy(np.stack([wl.kv_rows(w, l, 1, n0, n_kv) for l in range(L)]))
    q_h = torch.from_numpy(np.stack([wl.q_rows(w, l, T) for l in range(L)]))
    op_a, lp_a, out_a, lse_a = _outputs(L, T, Hq, C, D)
    kvq.kvq_decode_step(ca, k_h.cuda(), v_h.cuda(), q_h.cuda(), Hq, T, n_kv, chunk, w.scale,
                        op_a, lp_a, out_a, lse_a)
    k_pin, v_pin, q_pin = k_h.pin_memory(), v_h.pin_memory(), q_h.pin_memory()
    out_pin = torch.full(out_a.shape, float("nan")).pin_memory()
    lse_pin = torch.full(lse_a.shape, float("nan")).pin_memory()
    k_d = torch.empty_like(k_h, device="cuda")
    v_d = torch.empty_like(v_h, device="cuda")
    q_d = torch.empty_like(q_h, device="cuda")
    op_b, lp_b, out_b, lse_b = _outputs(L, T, Hq, C, D)
    kvq.kvq_decode_step_host(cb, k_pin, v_pin, q_pin, out_pin, lse_pin, k_d, v_d, q_d, Hq, T,
                             n_kv, chunk, w.scale, op_b, lp_b, out_b, lse_b)
    kvq.kvq_check()
    torch.cuda.synchronize()
    for l in range(L):
        assert torch.equal(ca.k[l], cb.k[l]) and torch.equal(ca.v[l], cb.v[l])
    assert torch.equal(k_d.cpu(), k_h) and torch.equal(q_d.cpu(), q_h)
    assert torch.equal(out_pin, out_a.cpu()) and torch.equal(lse_pin, lse_a.cpu())
