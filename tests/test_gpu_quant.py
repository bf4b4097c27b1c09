"""Quantize-on-append on the GPU is bit-exact against the oracle."""
import os

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_long_b200 import workload as wl

from helpers import fill_both
from test_oracle_quant import _golden_blocks, _oscar2_blocks, _random_blocks

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from quantized_kv_long_b200 import kvq as m
    return m


def _gpu_quant(kvq, x, q8):
    """Blocks of x on the GPU: Q8_0 if q8 is True, Q4_0 if False, OSCAR2 if "oscar2"."""
    xt = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    if q8 == "oscar2":
        out = torch.empty(x.size // 128 * 36, dtype=torch.uint8, device="cuda")
        kvq.kvq_quantize_oscar2(xt, out)
    else:
        nb = x.size // 32
        out = torch.empty(nb * (34 if q8 else 18), dtype=torch.uint8, device="cuda")
        (kvq.kvq_quantize_q8_0 if q8 else kvq.kvq_quantize_q4_0)(xt, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("q8", [True, False], ids=["q8_0", "q4_0"])
def test_random_blocks_bit_exact(kvq, q8):
    x = _random_blocks(10, 200000)
    ref = (oracle.quantize_q8_0 if q8 else oracle.quantize_q4_0)(x)
    assert np.array_equal(_gpu_quant(kvq, x, q8), ref)


def test_golden_and_edge_blocks_bit_exact(kvq):
    cases = [c for c in _golden_blocks()]
    edge = [
        np.zeros(32, np.float32),
        -np.zeros(32, np.float32),                        # -0.0 everywhere: m stays +0
        np.full(32, 3.0, np.float32),                     # all ties at the max
        np.array([-5.0] + [5.0] * 31, np.float32),        # first max negative, rest clamp
        np.array([1e-30] * 32, np.float32),               # d underflows fp16
        np.array([60000.0 * 127 / 128] + [1.0] * 31, np.float32),  # large amax
        (np.arange(32, dtype=np.float32) - 15.5) / 2,     # exact .25 / .75 products
        np.array([0.5 * (i % 2 * 2 - 1) for i in range(32)], np.float32),
    ]
    for fmt, x, expected in cases:
        got = _gpu_quant(kvq, x, "oscar2" if fmt == "oscar2" else fmt == "q8_0")
        assert bytes(got) == expected, fmt
    for x in edge:
        assert np.array_equal(_gpu_quant(kvq, x, True), oracle.quantize_q8_0(x))
        assert np.array_equal(_gpu_quant(kvq, x, False), oracle.quantize_q4_0(x))


def test_ties_at_half_bit_exact(kvq):
    """Products that land exactly on .5 after the scale: Q8_0 rounds them away
    from zero, Q4_0 rounds them up (floor(x + 8.5))."""
    rng = np.random.default_rng(5)
    n = 4096
    q = rng.integers(-126, 127, size=(n, 31)).astype(np.float32) + 0.5
    x = np.concatenate([np.full((n, 1), 127.0, np.float32), q], axis=1)  # d = 1 exactly
    scale = (2.0 ** rng.integers(-6, 6, size=(n, 1))).astype(np.float32)
    x = (x * scale).astype(np.float32)
    assert np.array_equal(_gpu_quant(kvq, x, True), oracle.quantize_q8_0(x))
    y = np.concatenate([np.full((n, 1), -8.0, np.float32),
                        rng.integers(-7, 8, size=(n, 31)).astype(np.float32) + 0.5], axis=1)
    y = (y * scale).astype(np.float32)
    assert np.array_equal(_gpu_quant(kvq, y, False), oracle.quantize_q4_0(y))


def test_oscar2_blocks_bit_exact(kvq):
    """OSCAR2 on the GPU against the oracle: random blocks, grid blocks with exact
    ties at .5 after the scale, and edge blocks (signed zeros, constants, a minimum
    or maximum that occurs twice, values near the fp16 limits)."""
    x = _oscar2_blocks(11, 100000)
    assert np.array_equal(_gpu_quant(kvq, x, "oscar2"), oracle.quantize_oscar2(x))
    rng = np.random.default_rng(12)
    n = 4096
    u2 = rng.integers(0, 7, size=(n, 128)).astype(np.float32) / 2  # codes and half-codes
    u2[:, 5], u2[:, 77] = 0.0, 3.0
    scale = (2.0 ** rng.integers(-8, 8, size=(n, 1))).astype(np.float32)
    y = (u2 * scale + rng.integers(-4, 4, size=(n, 1)).astype(np.float32) * scale)
    y = y.astype(np.float32)
    assert np.array_equal(_gpu_quant(kvq, y, "oscar2"), oracle.quantize_oscar2(y))
    z = np.zeros(128, np.float32)
    mixed = z.copy()
    mixed[::3] = -0.0                                     # -0 and +0: the first one wins
    edge = [z, -z, mixed, -mixed, np.full(128, -7.25, np.float32),
            np.concatenate([[2.0], np.zeros(126), [2.0]]).astype(np.float32),
            np.concatenate([[-1.0], np.ones(126), [-1.0]]).astype(np.float32),
            np.linspace(-60000, 60000, 128, dtype=np.float32),
            np.full(128, 1e-30, np.float32),
            (np.arange(128, dtype=np.float32) - 64) * np.float32(2.0 ** -20)]
    for e in edge:
        assert np.array_equal(_gpu_quant(kvq, e, "oscar2"), oracle.quantize_oscar2(e))


@pytest.mark.parametrize("D,H,n_rows,cap", [(256, 4, 1024, 1024), (128, 2, 77, 80),
                                            (512, 1, 40, 48), (32, 3, 9, 16)])
def test_append_matches_oracle(kvq, D, H, n_rows, cap):
    w = wl.small(wl.WORKLOADS["tiny"], head_dim=D, n_kv_heads=H, n_q_heads=H)
    cache, orc = fill_both(w, [0, 1], n_rows, cap)
    for i in range(2):
        k = cache.k[i].cpu().numpy()[:, :n_rows]
        v = cache.v[i].cpu().numpy()[:, :n_rows]
        assert np.array_equal(k, orc[i][0][:, :n_rows])
        assert np.array_equal(v, orc[i][1][:, :n_rows])


def test_append_multi_layer_offsets(kvq):
    """Append at an offset into several layers in one call leaves the other
    rows untouched and writes each layer's own rows."""
    w = wl.small(wl.WORKLOADS["tiny"])
    L, cap, pos, n = 3, 64, 17, 5
    cache = kvq.QuantizedKVCache(L, 4, 256, cap)
    for t in cache.k + cache.v:
        t.fill_(0xA5)
    k = np.stack([wl.kv_rows(w, l, 0, pos, pos + n) for l in range(L)])
    v = np.stack([wl.kv_rows(w, l, 1, pos, pos + n) for l in range(L)])
    kvq.kvq_append(cache, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), pos, n)
    torch.cuda.synchronize()
    for l in range(L):
        kc, vc = oracle.empty_cache(4, 256, cap)
        kc[:] = 0xA5
        vc[:] = 0xA5
        oracle.append(kc, vc, k[l], v[l], pos)
        assert np.array_equal(cache.k[l].cpu().numpy(), kc)
        assert np.array_equal(cache.v[l].cpu().numpy(), vc)


def test_full_65k_layer_bit_exact(kvq):
    """A whole 65,536-token layer of the 65k decode workload (seed 1)."""
    w = wl.WORKLOADS["decode65k"]
    cache, orc = fill_both(w, [3], 65536, 65536)
    assert np.array_equal(cache.k[0].cpu().numpy(), orc[0][0])
    assert np.array_equal(cache.v[0].cpu().numpy(), orc[0][1])
