"""Pins of the CPU oracle's fp16 conversion and Q8_0 / Q4_0 / OSCAR2 quantizers.

Every expected value here comes from the pages (byte sizes), from a hand
derivation of the quantizer definitions (golden blocks), from a library
routine (torch / numpy fp16 casts) or from a property the definitions imply
(round-trip bounds, idempotence).  None comes from the CUDA library.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _expand(spec: str):
    vals = []
    for tok in spec.split(","):
        tok = tok.strip()
        if "*" in tok:
            k, v = tok.split("*")
            vals += [float(v)] * int(k)
        else:
            vals.append(float(tok))
    return np.array(vals, dtype=np.float32)


def _golden_blocks():
    cases = []
    with open(os.path.join(GOLDEN, "quant_blocks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, xs, hexs = [p.strip() for p in line.split("|")]
            cases.append((fmt, _expand(xs), bytes.fromhex(hexs.replace(" ", ""))))
    return cases


def _sizes():
    out = {}
    with open(os.path.join(GOLDEN, "kv_sizes.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, v = line.split("=")
                out[k.strip()] = int(v)
    return out


# ---------------------------------------------------------------- sizes

def test_block_sizes_match_pages():
    s = _sizes()
    x = np.zeros(128, np.float32)
    assert oracle.quantize_q8_0(x).size == s["q8_0_bytes_per_128"]
    assert np.zeros(128, np.float16).nbytes == s["f16_bytes_per_128"]
    assert oracle.quantize_oscar2(x).size == s["oscar2_bytes_per_128"]
    assert oracle.quantize_oscar2(x).size * 8 * 100 // 128 == s["oscar2_bits_per_elem_x100"]
    # 16 attention layers x 4 KV heads x 256: K as Q8_0 plus V as Q4_0
    row = np.zeros(4 * 256, np.float32)
    per_layer = oracle.quantize_q8_0(row).size + oracle.quantize_q4_0(row).size
    assert 16 * per_layer == s["q8k_q4v_bytes_per_token_16x4x256"]
    assert round(262144 * 16 * per_layer / 1e7) == s["q8k_q4v_bytes_262144_tokens_gb_x100"]
    # the one-layer cache helper uses the same sizes
    k, v = oracle.empty_cache(4, 256, 3)
    assert (k.nbytes + v.nbytes) // 3 == per_layer
    # KV-size formula of the KV-cache guide with fp16 (2 bytes per element)
    assert 2 * 32 * 8 * 128 * np.dtype(np.float16).itemsize == s["f16_bytes_per_token_32x8x128"]


# ---------------------------------------------------------------- fp16

def test_f32_to_f16_all_relevant_patterns_match_library():
    """Every fp32 bit pattern whose exponent lies in [98, 146] (both signs) --
    all values that do not trivially flush to zero or overflow -- against the
    hardware RNE conversion torch uses; a spread sample of the rest."""
    mant = np.arange(1 << 23, dtype=np.uint32)
    for sign in (0, 1):
        for exp in range(98, 147):
            bits = (np.uint32(sign << 31) | np.uint32(exp << 23) | mant)
            x = bits.view(np.float32)
            ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
            got = oracle.f32_to_f16_bits(x)
            bad = np.nonzero(ref != got)[0]
            assert bad.size == 0, (sign, exp, hex(int(bits[bad[0]])))
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    finite = np.isfinite(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    got = oracle.f32_to_f16_bits(x)
    assert (ref[finite] == got[finite]).all()
    assert np.isnan(got[~np.isfinite(x) & np.isnan(x)].view(np.float16)).all()


def test_f16_to_f64_all_patterns_match_library():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    got = oracle.f16_bits_to_f64(h)
    same = (ref == got) | (np.isnan(ref) & np.isnan(got))
    assert same.all()


# ---------------------------------------------------------------- golden blocks

@pytest.mark.parametrize("case", _golden_blocks(), ids=lambda c: c[0])
def test_golden_blocks(case):
    fmt, x, expected = case
    assert x.size == (128 if fmt == "oscar2" else 32)
    got = {"q8_0": oracle.quantize_q8_0, "q4_0": oracle.quantize_q4_0,
           "oscar2": oracle.quantize_oscar2}[fmt](x)
    assert bytes(got) == expected


def test_golden_dequant():
    # q8a: d = 1.0 -> dequant equals the int8 values
    b = np.frombuffer(bytes.fromhex("003c7f81" + "0102fffd03" + "00" * 25), np.uint8)
    y = oracle.dequant_q8_0(b)
    assert y[:9].tolist() == [127, -127, 1, 2, -1, -3, 3, 0, 0]
    # q4a: d = -1 -> x^ = -(u - 8); byte 0x50 -> u0 = 0 (x^ = 8), u16 = 5 (x^ = 3)
    b = np.frombuffer(bytes.fromhex("00bc50bf" + "88" * 14), np.uint8)
    y = oracle.dequant_q4_0(b)
    assert y[0] == 8 and y[16] == 3 and y[1] == -7 and y[17] == -3 and y[2] == 0
    # OSCAR2: d = 0.5 (0x3800), m = -1.25 (0xBD00); byte 0 = 0b11_10_01_00 holds codes
    # 0, 1, 2, 3 of elements 0, 32, 64, 96; byte 5 = 0b00_00_00_11: element 5 -> u = 3
    b = np.frombuffer(bytes.fromhex("0038 00bd e4 00 00 00 00 03".replace(" ", "") + "00" * 26),
                      np.uint8)
    y = oracle.dequant_oscar2(b)
    assert y.size == 128
    assert [y[0], y[32], y[64], y[96]] == [-1.25, -0.75, -0.25, 0.25]
    assert y[5] == 0.25 and y[37] == -1.25 and y[1] == -1.25


# ---------------------------------------------------------------- properties

def _random_blocks(seed, n_blocks):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n_blocks, 32)).astype(np.float32)
    x[:, rng.choice(32, 4, replace=False)] *= 8
    scale = np.exp(rng.uniform(-8, 8, size=(n_blocks, 1))).astype(np.float32)
    return (x * scale).astype(np.float32)


def _d(blocks, nbytes):
    b = blocks.reshape(-1, nbytes)
    return b[:, :2].copy().view(np.float16).astype(np.float64)[:, 0]


def test_q8_0_round_trip_bound():
    x = _random_blocks(1, 20000)
    b = oracle.quantize_q8_0(x)
    xh = oracle.dequant_q8_0(b).reshape(x.shape)
    d16 = np.abs(_d(b, 34))[:, None]
    d32 = (np.abs(x).max(axis=1).astype(np.float32) / np.float32(127)).astype(np.float64)[:, None]
    bound = d16 / 2 + 127 * np.abs(d32 - d16) + 1e-6 * np.abs(x).max(axis=1, keepdims=True)
    assert (np.abs(x - xh) <= bound).all()
    # the max element is reproduced as +-127 d16
    q = b.reshape(-1, 34)[:, 2:].view(np.int8)
    assert (np.abs(q).max(axis=1) == 127).all()


def test_q4_0_round_trip_bound_and_clamp():
    x = _random_blocks(2, 20000)
    b = oracle.quantize_q4_0(x)
    xh = oracle.dequant_q4_0(b).reshape(x.shape)
    d16 = _d(b, 18)[:, None]
    first = np.argmax(np.abs(x), axis=1)
    m = x[np.arange(x.shape[0]), first].astype(np.float64)[:, None]
    d32 = (m.astype(np.float32) / np.float32(-8)).astype(np.float64)
    # elements whose x/d reaches the clamp (x*id + 8.5 >= 16) carry error up to |d|
    clamped = (x / d32) >= 7.5 - 1e-6
    slack = 8 * np.abs(d32 - d16) + 1e-6 * np.abs(m)
    err = np.abs(x - xh)
    assert (err[~clamped] <= (np.abs(d16) / 2 + slack).repeat(32, 1)[~clamped]).all()
    assert (err[clamped] <= (np.abs(d16) + slack).repeat(32, 1)[clamped]).all()
    assert clamped.any()  # the clamp case occurs in N(0,1) data with outliers
    # the first max element dequantizes to m16 = -8 d16 exactly
    assert np.allclose(xh[np.arange(x.shape[0]), first], -8 * d16[:, 0], rtol=0, atol=0)


def _oscar2_blocks(seed, n_blocks):
    """128-element blocks: N(0,1) with 4 outlier elements x 8, block scales e^U(-8, 6)
    (the minimum is stored as fp16, so every value stays well inside its range)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n_blocks, 128)).astype(np.float32)
    x[:, rng.choice(128, 4, replace=False)] *= 8
    scale = np.exp(rng.uniform(-8, 6, size=(n_blocks, 1))).astype(np.float32)
    return (x * scale).astype(np.float32)


def _dm(blocks):
    b = blocks.reshape(-1, 36)
    dm = b[:, :4].copy().view(np.float16).astype(np.float64)
    return dm[:, 0:1], dm[:, 1:2]


def test_oscar2_round_trip_bound():
    """|x - x^| <= d/2 for the fp32 d and minimum the codes were chosen with, plus the
    fp16 rounding of d (up to 3 steps) and of the minimum, plus fp32 rounding slack."""
    x = _oscar2_blocks(4, 20000)
    b = oracle.quantize_oscar2(x)
    xh = oracle.dequant_oscar2(b).reshape(x.shape)
    d16, m16 = _dm(b)
    mn = x.min(axis=1, keepdims=True)
    mx = x.max(axis=1, keepdims=True)
    d32 = (((mx - mn).astype(np.float32)) / np.float32(3)).astype(np.float64)
    slack = 3 * np.abs(d32 - d16) + np.abs(mn - m16) + 1e-6 * (np.abs(mx) + np.abs(mn))
    assert (np.abs(x - xh) <= d32 / 2 + slack).all()
    # the stored scale and zero-point are the fp16 roundings of d and of the minimum
    assert (np.abs(d16 - d32) <= 2.0 ** -11 * d32 + 2.0 ** -25).all()
    assert (np.abs(m16 - mn) <= 2.0 ** -11 * np.abs(mn) + 2.0 ** -25).all()
    # the minimum decodes from code 0 and the maximum from code 3
    codes = np.unpackbits(b.reshape(-1, 36)[:, 4:, None], axis=2, bitorder="little")
    assert codes.shape == (x.shape[0], 32, 8)
    u = (codes[:, :, 0::2] + 2 * codes[:, :, 1::2]).transpose(0, 2, 1).reshape(x.shape)
    r = np.arange(x.shape[0])
    assert (u[r, np.argmin(x, axis=1)] == 0).all() and (u[r, np.argmax(x, axis=1)] == 3).all()


def test_oscar2_grid_values_round_trip_exactly():
    """Blocks whose values lie on an fp16 grid m + d u with codes 0 and 3 present come
    back exactly, and their codes are the grid indices."""
    rng = np.random.default_rng(5)
    n = 3000
    d = np.float16(2.0) ** rng.integers(-12, 6, size=(n, 1)).astype(np.float16)
    d = (d * rng.integers(1024, 2048, size=(n, 1)) / 1024).astype(np.float16)
    m = (rng.integers(-64, 64, size=(n, 1)) * d.astype(np.float64)).astype(np.float16)
    m = m.astype(np.float64)  # an fp16 zero-point within 64 steps of 0
    u = rng.integers(0, 4, size=(n, 128))
    u[:, 0], u[:, 127] = 0, 3
    x = (m + d.astype(np.float64) * u).astype(np.float32)
    assert np.array_equal(x.astype(np.float64), m + d.astype(np.float64) * u)  # exact inputs
    b = oracle.quantize_oscar2(x)
    assert np.array_equal(oracle.dequant_oscar2(b).reshape(x.shape), x.astype(np.float64))


@pytest.mark.parametrize("fmt", ["q8_0", "q4_0", "oscar2"])
def test_quantize_dequant_idempotent(fmt):
    x = _oscar2_blocks(3, 2000) if fmt == "oscar2" else _random_blocks(3, 5000)
    q, dq, nb = {"q8_0": (oracle.quantize_q8_0, oracle.dequant_q8_0, 34),
                 "q4_0": (oracle.quantize_q4_0, oracle.dequant_q4_0, 18),
                 "oscar2": (oracle.quantize_oscar2, oracle.dequant_oscar2, 36)}[fmt]
    b = q(x)
    d16 = np.abs(_d(b, nb))
    normal = d16 >= 2.0 ** -14  # fp16 normal scale: dequantized values re-quantize exactly
    xh = dq(b).astype(np.float32)
    b2 = q(xh)
    same = (b.reshape(-1, nb) == b2.reshape(-1, nb)).all(axis=1)
    assert same[normal].all()
    assert normal.mean() > 0.9


def test_zero_scale_block_dequantizes_to_zero():
    x = np.zeros(64, np.float32)
    assert (oracle.dequant_q8_0(oracle.quantize_q8_0(x)) == 0).all()
    assert (oracle.dequant_q4_0(oracle.quantize_q4_0(x)) == 0).all()
    assert (oracle.dequant_oscar2(oracle.quantize_oscar2(np.zeros(256, np.float32))) == 0).all()
