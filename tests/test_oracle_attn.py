"""Pins of the CPU oracle's attention, LSE merge and prefill.

Expected values come from closed forms (one key, identical keys, zero query),
from a library routine (torch's fp64 scaled_dot_product_attention and
logsumexp on CPU over the oracle's pinned dequantization), or from invariants
of the method (chunked merge = one pass, merge associativity, fully masked
chunk is a no-op, a uniform logit shift moves only the lse, prefill row =
decode of that token).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_long_b200 import workload as wl

SCALE = 1.0 / 16.0


def _cache(H, D, cap, seed, same_key=False):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((cap, H, D)).astype(np.float32)
    v = rng.standard_normal((cap, H, D)).astype(np.float32)
    k[:, :, :4] *= 8
    if same_key:
        k[:] = k[0]
    kc, vc = oracle.empty_cache(H, D, cap)
    oracle.append(kc, vc, k, v, 0)
    return kc, vc


def _deq(kc, vc):
    H, cap, _ = kc.shape
    D = kc.shape[2] // 34 * 32
    K = oracle.dequant_q8_0(kc).reshape(H, cap, D)
    V = oracle.dequant_q4_0(vc).reshape(H, cap, D)
    return K, V


def _q(T, Hq, D, seed, zero=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, Hq, D)).astype(np.float16)
    return np.zeros_like(q) if zero else q


# ------------------------------------------------------------- closed forms

def test_single_key_returns_its_value_row():
    kc, vc = _cache(2, 64, 1, 0)
    K, V = _deq(kc, vc)
    q = _q(1, 4, 64, 1)
    out, lse = oracle.decode_attn(kc, vc, q, n_kv=1, chunk=64, scale=SCALE)
    for g in range(4):
        h = g // 2
        assert np.array_equal(out[0, g, 0], V[h, 0])
        s = SCALE * float(np.dot(q[0, g].astype(np.float64), K[h, 0]))
        assert abs(lse[0, g, 0] - s) < 1e-12


def test_identical_keys_give_mean_value_and_log_count():
    n = 37
    kc, vc = _cache(1, 32, n, 2, same_key=True)
    K, V = _deq(kc, vc)
    q = _q(1, 3, 32, 3)
    out, lse = oracle.decode_attn(kc, vc, q, n_kv=n, chunk=n, scale=SCALE)
    for g in range(3):
        assert np.allclose(out[0, g, 0], V[0, :n].mean(axis=0), rtol=0, atol=1e-12)
        s = SCALE * float(np.dot(q[0, g].astype(np.float64), K[0, 0]))
        assert abs(lse[0, g, 0] - (s + math.log(n))) < 1e-12


@pytest.mark.parametrize("T", [1, 4])
def test_uniform_logit_shift_moves_lse_only(T):
    """Softmax invariance: adding the same constant to every logit of a row leaves
    its output unchanged and adds the constant to its lse.  Every key gets the same
    first 32-element block (so the same dequantized values there); a query that
    differs only in that block shifts all of a row's logits by
    scale * dq . k_block0, computed here in fp64 from the pinned dequantization."""
    H, D, n = 2, 64, 150
    rng = np.random.default_rng(7)
    k = rng.standard_normal((n, H, D)).astype(np.float32)
    v = rng.standard_normal((n, H, D)).astype(np.float32)
    k[:, :, 32:36] *= 8
    k[:, :, :32] = k[0, :, :32]
    kc, vc = oracle.empty_cache(H, D, n)
    oracle.append(kc, vc, k, v, 0)
    K, _ = _deq(kc, vc)
    assert np.array_equal(K[:, 0, :32], K[:, n - 1, :32])
    q = _q(T, 4, D, 8)
    q2 = q.copy()
    dq = (np.random.default_rng(9).standard_normal((T, 4, 32)) * 2).astype(np.float16)
    q2[:, :, :32] = dq
    o1, l1 = oracle.decode_attn(kc, vc, q, n_kv=n, chunk=n, scale=SCALE)
    o2, l2 = oracle.decode_attn(kc, vc, q2, n_kv=n, chunk=n, scale=SCALE)
    for t in range(T):
        for g in range(4):
            h = g // 2
            shift = SCALE * float(np.dot(q2[t, g, :32].astype(np.float64) -
                                         q[t, g, :32].astype(np.float64), K[h, 0, :32]))
            assert np.allclose(o2[t, g, 0], o1[t, g, 0], rtol=0, atol=1e-12)
            assert abs(l2[t, g, 0] - (l1[t, g, 0] + shift)) < 1e-10


@pytest.mark.parametrize("T", [1, 4])
def test_zero_query_gives_mean_over_visible_keys(T):
    """With q = 0 every visible key has weight 1: out is the mean of the
    visible V rows and lse = ln(count).  This pins the causal mask: token t
    of a T-token step sees n_kv - T + t + 1 keys."""
    n_kv, chunk = 50, 16
    kc, vc = _cache(1, 64, n_kv, 4)
    _, V = _deq(kc, vc)
    q = _q(T, 2, 64, 5, zero=True)
    out, lse = oracle.decode_attn(kc, vc, q, n_kv=n_kv, chunk=chunk, scale=SCALE)
    mo, ml = oracle.merge_lse(out, lse)
    for t in range(T):
        vis = n_kv - T + t + 1
        for c in range(out.shape[2]):
            lo, hi = c * chunk, min((c + 1) * chunk, vis)
            if hi <= lo:
                assert lse[t, 0, c] == -np.inf and (out[t, 0, c] == 0).all()
            else:
                assert abs(lse[t, 0, c] - math.log(hi - lo)) < 1e-12
                assert np.allclose(out[t, 0, c], V[0, lo:hi].mean(axis=0), atol=1e-12, rtol=0)
        assert abs(ml[t, 1] - math.log(vis)) < 1e-12
        assert np.allclose(mo[t, 1], V[0, :vis].mean(axis=0), atol=1e-12, rtol=0)


# ------------------------------------------------------------- library routine

def _torch_ref(K, V, q, n_kv, T, Hq, H, first_visible_last):
    """fp64 attention through torch's SDPA with GQA by repeat_interleave
    (query head g reads KV head g // (Hq // H)) and a boolean causal mask."""
    G = Hq // H
    Kt = torch.from_numpy(K[:, :n_kv]).repeat_interleave(G, dim=0)      # [Hq, n, D]
    Vt = torch.from_numpy(V[:, :n_kv]).repeat_interleave(G, dim=0)
    Q = torch.from_numpy(q.astype(np.float64)).permute(1, 0, 2)          # [Hq, T, D]
    last = torch.tensor([first_visible_last + t for t in range(T)])
    mask = torch.arange(n_kv)[None, :] <= last[:, None]                  # [T, n]
    o = torch.nn.functional.scaled_dot_product_attention(Q, Kt, Vt, attn_mask=mask,
                                                         scale=SCALE)
    s = torch.einsum("htd,hnd->htn", Q, Kt) * SCALE
    s = s.masked_fill(~mask, -math.inf)
    lse = torch.logsumexp(s, dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.permute(1, 0).numpy()


@pytest.mark.parametrize("n_kv,D,T,H,Hq", [(1, 32, 1, 1, 1), (2, 64, 1, 2, 4), (3, 256, 1, 4, 24),
                                           (33, 64, 2, 2, 6), (100, 256, 4, 4, 24),
                                           (257, 32, 3, 1, 3)])
def test_matches_torch_sdpa_fp64(n_kv, D, T, H, Hq):
    if n_kv < T:
        pytest.skip("needs n_kv >= T")
    kc, vc = _cache(H, D, n_kv, n_kv + D)
    K, V = _deq(kc, vc)
    q = _q(T, Hq, D, 11)
    part, plse = oracle.decode_attn(kc, vc, q, n_kv=n_kv, chunk=7, scale=SCALE)
    out, lse = oracle.merge_lse(part, plse)
    ro, rl = _torch_ref(K, V, q, n_kv, T, Hq, H, n_kv - T)
    assert np.allclose(out, ro, rtol=0, atol=1e-12)
    assert np.allclose(lse, rl, rtol=0, atol=1e-12)


# ------------------------------------------------------------- invariants

@pytest.mark.parametrize("chunk", [1, 7, 32, 4096])
def test_chunked_merge_equals_one_pass(chunk):
    n_kv, T = 300, 4
    kc, vc = _cache(2, 64, n_kv, 21)
    q = _q(T, 6, 64, 22)
    p, l = oracle.decode_attn(kc, vc, q, n_kv=n_kv, chunk=chunk, scale=SCALE)
    out, lse = oracle.merge_lse(p, l)
    p1, l1 = oracle.decode_attn(kc, vc, q, n_kv=n_kv, chunk=n_kv, scale=SCALE)
    assert np.allclose(out, p1[:, :, 0], rtol=0, atol=1e-12)
    assert np.allclose(lse, l1[:, :, 0], rtol=0, atol=1e-12)
    # and the one-pass row function agrees
    G = 3
    rows = [(t, g) for t in range(T) for g in range(6)]
    ro, rl = oracle.attn_rows(kc, vc, np.stack([q[t, g] for t, g in rows]),
                              np.array([g for _, g in rows]), 6,
                              np.zeros(len(rows)), np.array([n_kv - T + t + 1 for t, _ in rows]),
                              SCALE)
    assert np.allclose(ro.reshape(T, 6, 64), out, rtol=0, atol=1e-12)
    assert np.allclose(rl.reshape(T, 6), lse, rtol=0, atol=1e-12)
    assert G * 2 == 6


def test_merge_is_associative():
    n_kv = 200
    kc, vc = _cache(1, 32, n_kv, 31)
    q = _q(1, 2, 32, 32)
    p, l = oracle.decode_attn(kc, vc, q, n_kv=n_kv, chunk=9, scale=SCALE)
    flat_o, flat_l = oracle.merge_lse(p, l)
    C = p.shape[2]
    groups = [list(range(i, min(i + 5, C))) for i in range(0, C, 5)]
    go = np.stack([oracle.merge_lse(p[:, :, g], l[:, :, g])[0] for g in groups], axis=2)
    gl = np.stack([oracle.merge_lse(p[:, :, g], l[:, :, g])[1] for g in groups], axis=2)
    tree_o, tree_l = oracle.merge_lse(go, gl)
    assert np.allclose(tree_o, flat_o, rtol=0, atol=1e-12)
    assert np.allclose(tree_l, flat_l, rtol=0, atol=1e-12)


def test_fully_masked_chunk_is_a_no_op():
    T, chunk = 4, 16
    n_kv = 3 * chunk + 1           # the last chunk holds one key, seen only by t = 3
    kc, vc = _cache(1, 64, n_kv, 41)
    q = _q(T, 2, 64, 42)
    p, l = oracle.decode_attn(kc, vc, q, n_kv=n_kv, chunk=chunk, scale=SCALE)
    assert (l[:3, :, 3] == -np.inf).all() and (p[:3, :, 3] == 0).all()
    assert np.isfinite(l[3, :, 3]).all()
    out, lse = oracle.merge_lse(p, l)
    o3, l3 = oracle.merge_lse(p[:, :, :3], l[:, :, :3])
    assert np.array_equal(out[:3], o3[:3]) and np.array_equal(lse[:3], l3[:3])


def test_merge_of_nothing_is_empty():
    p = np.zeros((2, 3, 8))
    l = np.full((2, 3), -np.inf)
    o, ls = oracle.merge_lse(p, l)
    assert (o == 0).all() and (ls == -np.inf).all()


def test_prefill_rows_equal_decode_of_each_token_and_pages_merge():
    H, Hq, D, n_cached, T, page = 2, 6, 64, 70, 9, 32
    kc, vc = _cache(H, D, n_cached + T, 51)
    q = _q(T, Hq, D, 52)
    out, lse, po, pl = oracle.prefill_attn(kc, vc, q, n_cached, page, SCALE, pages=True)
    for t in range(T):
        d, dl = oracle.decode_attn(kc, vc, q[t:t + 1], n_kv=n_cached + t + 1, chunk=1 << 20,
                                   scale=SCALE)
        assert np.allclose(out[t], d[0, :, 0], rtol=0, atol=1e-12)
        assert np.allclose(lse[t], dl[0, :, 0], rtol=0, atol=1e-12)
    mo, ml = oracle.merge_lse(po, pl)
    assert np.allclose(mo, out, rtol=0, atol=1e-12)
    assert np.allclose(ml, lse, rtol=0, atol=1e-12)
    K, V = _deq(kc, vc)
    ro, rl = _torch_ref(K, V, q, n_cached + T, T, Hq, H, n_cached)
    assert np.allclose(out, ro, rtol=0, atol=1e-12)
    assert np.allclose(lse, rl, rtol=0, atol=1e-12)


# ------------------------------------------------------------- workload inputs

def test_workload_generator_is_seeded_and_blockwise():
    w = wl.small(wl.WORKLOADS["tiny"], n_kv=40000)
    a = wl.kv_rows(w, 0, 0, 0, 40000)
    b = wl.kv_rows(w, 0, 0, 16000, 33000, threads=1)
    assert np.array_equal(a[16000:33000], b)
    ch = wl.outlier_channels(w.seed, w.head_dim)
    assert len(ch) == 4 and np.abs(a[:, :, ch]).mean() > 6 * np.abs(np.delete(a, ch, 2)).mean()
    q = wl.q_rows(w, 0)
    assert q.dtype == np.float16 and q.shape == (1, 24, 256)
    assert not np.array_equal(wl.kv_rows(w, 0, 1, 0, 10), a[:10])


# ------------------------------------------------------- other block formats
# The KV-cache guide's levers section lists q8_0 and q4_0 caches for both
# tensors.  The format plumbing (which block format each tensor's rows are
# written and read in) is pinned against the separately pinned block
# quantizers and dequantizers.

O2 = oracle.FMT_OSCAR2
FORMATS = [(oracle.FMT_Q8_0, oracle.FMT_Q8_0), (oracle.FMT_Q4_0, oracle.FMT_Q4_0),
           (oracle.FMT_Q4_0, oracle.FMT_Q8_0), (O2, O2), (oracle.FMT_Q8_0, O2),
           (O2, oracle.FMT_Q4_0)]
_QUANT = {oracle.FMT_Q8_0: oracle.quantize_q8_0, oracle.FMT_Q4_0: oracle.quantize_q4_0,
          O2: oracle.quantize_oscar2}
_DEQ = {oracle.FMT_Q8_0: oracle.dequant_q8_0, oracle.FMT_Q4_0: oracle.dequant_q4_0,
        O2: oracle.dequant_oscar2}


def _dim(k_fmt, v_fmt):
    """head_dim of the format tests: 64, or 128 where an OSCAR2 tensor needs whole blocks."""
    return 128 if O2 in (k_fmt, v_fmt) else 64


def _fmt_cache(H, D, cap, k_fmt, v_fmt, seed):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((cap, H, D)).astype(np.float32)
    v = rng.standard_normal((cap, H, D)).astype(np.float32)
    k[:, :, :4] *= 8
    kc, vc = oracle.empty_cache(H, D, cap, k_fmt=k_fmt, v_fmt=v_fmt)
    oracle.append(kc, vc, k, v, 0)
    return k, v, kc, vc


@pytest.mark.parametrize("k_fmt,v_fmt", FORMATS)
def test_format_append_writes_each_tensors_blocks(k_fmt, v_fmt):
    H, D, cap = 2, _dim(k_fmt, v_fmt), 5
    k, v, kc, vc = _fmt_cache(H, D, cap, k_fmt, v_fmt, 11)
    for h in range(H):
        assert np.array_equal(kc[h].reshape(-1), _QUANT[k_fmt](k[:, h].reshape(-1)))
        assert np.array_equal(vc[h].reshape(-1), _QUANT[v_fmt](v[:, h].reshape(-1)))


@pytest.mark.parametrize("k_fmt,v_fmt", FORMATS)
def test_format_single_key_and_brute_force(k_fmt, v_fmt):
    H, D, Hq, T = 2, _dim(k_fmt, v_fmt), 4, 2
    n_kv = 9
    k, v, kc, vc = _fmt_cache(H, D, n_kv, k_fmt, v_fmt, 12)
    K = _DEQ[k_fmt](kc).reshape(H, n_kv, D)
    V = _DEQ[v_fmt](vc).reshape(H, n_kv, D)
    q = _q(T, Hq, D, 13)
    # one key: its V row and its own score
    out, lse = oracle.decode_attn(kc, vc, q[:1], n_kv=1, chunk=64, scale=SCALE)
    for g in range(Hq):
        h = g // (Hq // H)
        assert np.array_equal(out[0, g, 0], V[h, 0])
        assert abs(lse[0, g, 0] - SCALE * float(np.dot(q[0, g].astype(np.float64), K[h, 0]))) < 1e-12
    # brute force over the dequantized rows, causal verify batch, one chunk
    out, lse = oracle.decode_attn(kc, vc, q, n_kv=n_kv, chunk=64, scale=SCALE)
    for t in range(T):
        for g in range(Hq):
            h = g // (Hq // H)
            n = n_kv - T + t + 1
            s = SCALE * (K[h, :n] @ q[t, g].astype(np.float64))
            w = np.exp(s - s.max())
            ref = (w / w.sum()) @ V[h, :n]
            assert np.allclose(out[t, g, 0], ref, rtol=0, atol=1e-12)
            assert abs(lse[t, g, 0] - (s.max() + math.log(w.sum()))) < 1e-12


@pytest.mark.parametrize("k_fmt,v_fmt", [(O2, O2), (oracle.FMT_Q8_0, O2)])
def test_format_prefill_equals_decode_and_brute_force(k_fmt, v_fmt):
    """Prefill over OSCAR2 caches: each token's row equals a decode over the keys it
    sees, the page partials merge to the one-pass rows, and both equal softmax
    attention over the dequantized rows."""
    H, Hq, D, n_cached, T, page = 2, 4, 128, 37, 5, 16
    k, v, kc, vc = _fmt_cache(H, D, n_cached + T, k_fmt, v_fmt, 53)
    K = _DEQ[k_fmt](kc).reshape(H, n_cached + T, D)
    V = _DEQ[v_fmt](vc).reshape(H, n_cached + T, D)
    q = _q(T, Hq, D, 54)
    out, lse, po, pl = oracle.prefill_attn(kc, vc, q, n_cached, page, SCALE, pages=True)
    mo, ml = oracle.merge_lse(po, pl)
    assert np.allclose(mo, out, rtol=0, atol=1e-12) and np.allclose(ml, lse, rtol=0, atol=1e-12)
    for t in range(T):
        d, dl = oracle.decode_attn(kc, vc, q[t:t + 1], n_kv=n_cached + t + 1, chunk=1 << 20,
                                   scale=SCALE)
        assert np.allclose(out[t], d[0, :, 0], rtol=0, atol=1e-12)
        for g in range(Hq):
            h = g // (Hq // H)
            n = n_cached + t + 1
            s = SCALE * (K[h, :n] @ q[t, g].astype(np.float64))
            w = np.exp(s - s.max())
            assert np.allclose(out[t, g], (w / w.sum()) @ V[h, :n], rtol=0, atol=1e-12)
            assert abs(lse[t, g] - (s.max() + math.log(w.sum()))) < 1e-12
