"""Split-KV decode attention and the LSE merge on the GPU against the oracle.

Both sides quantize the same seeded fp32 rows (bit-exact, checked in
test_gpu_quant); the oracle then dequantizes and computes fp64 attention.
Per-chunk partials and merged results are compared with the tolerances of
helpers.py (out max-abs 2e-3, lse relative 1e-4).
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


@pytest.fixture(params=["tc", "simple"])
def kernel(request, kvq):
    """Run a case on the tiled tensor-core kernel and on the general kernel."""
    with kvq.test_hooks(decode_general=request.param == "simple"):
        yield request.param


def run_decode(kvq, cache, q, Hq, T, n_kv, chunk, scale, layers=None):
    n_layers = q.shape[0]
    D = q.shape[-1]
    C = -(-n_kv // chunk)
    qt = torch.from_numpy(q).cuda()
    op = torch.full((n_layers, T, Hq, C, D), float("nan"), device="cuda")
    lp = torch.full((n_layers, T, Hq, C), float("nan"), device="cuda")
    kvq.kvq_decode_attn(cache.layers() if layers is None else layers, qt, Hq, T, n_kv, chunk,
                        scale, op, lp)
    out = torch.full((n_layers, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((n_layers, T, Hq), float("nan"), device="cuda")
    kvq.kvq_merge_lse(op, lp, n_layers * T * Hq, C, D, out, lse)
    kvq.kvq_check()
    return op.cpu().numpy(), lp.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


def check_case(kvq, w, n_layers, T, n_kv, chunk, cap=None):
    cap = cap or -(-n_kv // 8) * 8
    layers = list(range(n_layers))
    cache, orc = fill_both(w, layers, n_kv, cap)
    q = q_all(w, layers, T)
    op, lp, out, lse = run_decode(kvq, cache, q, w.n_q_heads, T, n_kv, chunk, w.scale)
    for l in layers:
        rp, rl = oracle.decode_attn(orc[l][0], orc[l][1], q[l], n_kv, chunk, w.scale)
        assert_attn_close(op[l], lp[l], rp, rl, f"partials layer {l}")
        mo, ml = oracle.merge_lse(rp, rl)
        assert_attn_close(out[l], lse[l], mo, ml, f"merged layer {l}")


def test_tiny_workload(kvq, kernel):
    """1 layer, 1 token, 1,024 context, seed 0: chunk 4,096 (one chunk) and 256."""
    w = wl.WORKLOADS["tiny"]
    check_case(kvq, w, 1, 1, 1024, 4096)
    check_case(kvq, w, 1, 1, 1024, 256)


@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("chunk", [256, 4096])
def test_verify_batch_ragged_context(kvq, T, chunk, kernel):
    """4,097 keys: a ragged last chunk; causal within the T new tokens."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=4097)
    check_case(kvq, w, 2, T, 4097, chunk)


@pytest.mark.parametrize("T", [1, 4])
def test_fully_masked_last_chunk(kvq, T, kernel):
    """n_kv = 3*64 + 1: the last 64-key chunk holds one key, which only the
    last token sees; for the others that chunk must be (0, -inf)."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=193)
    check_case(kvq, w, 1, T, 193, 64)


@pytest.mark.parametrize("D,H,Hq,T", [(64, 2, 16, 2), (128, 8, 32, 1), (512, 1, 8, 4),
                                      (256, 4, 4, 4), (32, 1, 1, 1), (256, 2, 16, 4),
                                      (256, 2, 10, 4), (256, 1, 8, 3), (256, 3, 12, 4)])
def test_other_shapes(kvq, D, H, Hq, T):
    """Other head sizes and GQA groups; at head_dim 256, 20 and 24 rows (group 5 x 4
    tokens, 8 x 3) take the role-split kernel and 16 rows (4 x 4) the pair kernel."""
    w = wl.small(wl.WORKLOADS["tiny"], head_dim=D, n_kv_heads=H, n_q_heads=Hq,
                 scale=float(D) ** -0.5)
    check_case(kvq, w, 2, T, 700, 128)


def test_minimal_context(kvq, kernel):
    """n_kv == T: the first token sees exactly one key."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=4)
    check_case(kvq, w, 1, 4, 4, 64, cap=8)


def test_sixteen_layers_one_call(kvq, kernel):
    w = wl.small(wl.WORKLOADS["decode65k"], n_kv=2000)
    check_case(kvq, w, 16, 1, 2000, 512)


def test_merge_kernel_against_oracle(kvq):
    rng = np.random.default_rng(3)
    rows, C, D = 300, 37, 256
    op = rng.standard_normal((rows, C, D)).astype(np.float32)
    lp = (rng.standard_normal((rows, C)) * 5 + 10).astype(np.float32)
    lp[rng.random((rows, C)) < 0.2] = -np.inf
    lp[5] = -np.inf  # a row with nothing visible
    op[lp == -np.inf] = 0
    out = torch.empty((rows, D), device="cuda")
    lse = torch.empty(rows, device="cuda")
    kvq.kvq_merge_lse(torch.from_numpy(op).cuda(), torch.from_numpy(lp).cuda(), rows, C, D, out,
                      lse)
    ro, rl = oracle.merge_lse(op.astype(np.float64), lp.astype(np.float64))
    assert_attn_close(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, "merge")
    assert (out.cpu().numpy()[5] == 0).all() and lse.cpu().numpy()[5] == -np.inf


def test_deterministic(kvq, kernel):
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=3000)
    cache, _ = fill_both(w, [0], 3000, 3000)
    q = q_all(w, [0], 4)
    a = run_decode(kvq, cache, q, 24, 4, 3000, 1024, w.scale)
    b = run_decode(kvq, cache, q, 24, 4, 3000, 1024, w.scale)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("n_kv,chunk", [(64, 64), (130, 64), (5000, 4096), (8192, 128)])
def test_tc_stage_edges(kvq, n_kv, chunk):
    """Chunks of one stage, a partial second stage (pairs without tokens),
    chunks longer than the 4-stage ring, and many short chunks."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=n_kv)
    check_case(kvq, w, 1, 4, n_kv, chunk)
    check_case(kvq, w, 1, 1, n_kv, chunk)


@pytest.mark.parametrize("T", [1, 4])
def test_bounded_wait_times_out_and_context_survives(kvq, T):
    """A wait on a barrier that nothing completes runs out after about a
    second: the kernel ends, kvq_check reports KVQ_ERR_TIMEOUT once, and the
    next call on the same context is correct again (the persistent kernel, one
    and three n-tiles of rows)."""
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=512)
    cache, orc = fill_both(w, [0], 512, 512)
    q = q_all(w, [0], T)
    qt = torch.from_numpy(q).cuda()
    op = torch.empty((1, T, 24, 1, 256), device="cuda")
    lp = torch.empty((1, T, 24, 1), device="cuda")
    with kvq.test_hooks(decode_timeout=True):
        kvq.kvq_decode_attn(cache.layers(), qt, 24, T, 512, 512, w.scale, op, lp)
        with pytest.raises(kvq.KvqError) as e:
            kvq.kvq_check()
    assert e.value.status == kvq.KVQ_ERR_TIMEOUT
    kvq.kvq_check()  # the status word was cleared
    op2, lp2, out, lse = run_decode(kvq, cache, q, 24, T, 512, 512, w.scale)
    rp, rl = oracle.decode_attn(orc[0][0], orc[0][1], q[0], 512, 512, w.scale)
    assert_attn_close(op2[0], lp2[0], rp, rl, "after timeout")
