"""Chunked prefill on the GPU against the oracle.

Cases cover the tensor-core path (every row sees >= 4,096 keys), the exact
path (short prompts), a run that splits between them, ragged row tiles, several
layers per call, and the full prefill262k workload (2,048 new tokens over
262,144 cached, 16 layers in one call) on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_long_b200 import workload as wl

from helpers import assert_attn_close, fill_both

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from quantized_kv_long_b200 import kvq as m
    return m


def run_prefill(kvq, cache, q, Hq, T, n_cached, scale, page=1024, expand=False):
    """expand: pass a workspace, so that the key tiles are expanded once per call."""
    L, D = q.shape[0], q.shape[-1]
    out = torch.full((L, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((L, T, Hq), float("nan"), device="cuda")
    ws = None
    if expand:
        nb = kvq.kvq_prefill_workspace_bytes(L, cache.n_kv_heads, D, n_cached + T)
        ws = torch.full((max(nb, 1),), 0x7F, dtype=torch.uint8, device="cuda")  # garbage
    kvq.kvq_prefill_attn(cache.layers(), torch.from_numpy(q).cuda(), Hq, T, n_cached, page, scale,
                         out, lse, workspace=ws)
    kvq.kvq_check()
    return out.cpu().numpy(), lse.cpu().numpy()


def check(kvq, w, n_layers, T, n_cached):
    n = n_cached + T
    cap = -(-n // 8) * 8
    layers = list(range(n_layers))
    cache, orc = fill_both(w, layers, n, cap)
    q = np.stack([wl.q_rows(w, l, T) for l in layers])
    out, lse = run_prefill(kvq, cache, q, w.n_q_heads, T, n_cached, w.scale)
    for l in layers:
        ro, rl = oracle.prefill_attn(orc[l][0], orc[l][1], q[l], n_cached, 1024, w.scale)
        assert_attn_close(out[l], lse[l], ro, rl, f"prefill layer {l}")
    # the expanded-tile path (workspace) gives the same bits
    eo, el = run_prefill(kvq, cache, q, w.n_q_heads, T, n_cached, w.scale, expand=True)
    assert np.array_equal(eo, out) and np.array_equal(el, lse), "workspace path differs"


def test_tensor_core_path(kvq):
    """Every row sees >= 16,448 keys; 128 tokens x 6 heads = 6 full 128-row tiles per head."""
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=16448, T=128)
    check(kvq, w, 1, 128, 16448)


def test_split_exact_and_tensor_core_ragged(kvq):
    """Tokens 0..85 see < 16,384 keys (exact kernel), 86..299 take the tensor
    cores; 214 x 6 rows of the tensor-core part leave a ragged last tile."""
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=16298, T=300)
    check(kvq, w, 2, 300, 16298)


def test_short_prompt_exact(kvq):
    """No cached keys: token 0 sees exactly one key (the exact kernel)."""
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=0, T=70)
    check(kvq, w, 1, 70, 0)


def test_exact_kernel_layers(kvq):
    """Mid-length context on the exact kernel, three layers in one call."""
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=9000, T=40)
    check(kvq, w, 3, 40, 9000)


def test_prefill262k_full_size_sampled(kvq):
    """The full workload in the launch configuration the benchmark times:
    16 layers, 2,048 new tokens appended after 262,144 cached keys."""
    import bench
    w = wl.WORKLOADS["prefill262k"]
    T, nc, Hq = w.T, w.n_cached, w.n_q_heads
    device = torch.device("cuda", 0)
    cache = bench.fill_cache(kvq, torch, wl.small(w, n_kv=nc + T), device)
    q = np.stack([wl.q_rows(w, l) for l in range(w.n_layers)])
    out = torch.full((w.n_layers, T, Hq, 256), float("nan"), device=device)
    lse = torch.full((w.n_layers, T, Hq), float("nan"), device=device)
    qd = torch.from_numpy(q).cuda()
    kvq.kvq_prefill_attn(cache.layers(), qd, Hq, T, nc, w.page, w.scale, out, lse)
    kvq.kvq_check()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    # the launch the benchmark times: a 2 GiB workspace (four of the 64 slabs, two
    # pairs per chunk), same bits
    slab = kvq.kvq_prefill_workspace_bytes(1, 1, 256, nc + T)
    ws = torch.empty(((2 << 30) // slab * slab,), dtype=torch.uint8, device=device)
    out2 = torch.full_like(out, float("nan"))
    lse2 = torch.full_like(lse, float("nan"))
    kvq.kvq_prefill_attn(cache.layers(), qd, Hq, T, nc, w.page, w.scale, out2, lse2, workspace=ws)
    kvq.kvq_check()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    del ws, out2, lse2
    rng = np.random.default_rng(7)
    for l in (0, 9):
        kc, vc = oracle.empty_cache(w.n_kv_heads, w.head_dim, nc + T)
        oracle.append(kc, vc, wl.kv_rows(w, l, 0, 0, nc + T), wl.kv_rows(w, l, 1, 0, nc + T), 0)
        ts = np.concatenate([[0, 1, T - 1], rng.integers(0, T, 9)])
        hs = rng.integers(0, Hq, len(ts))
        ro, rl = oracle.attn_rows(kc, vc, q[l, ts, hs], hs, Hq, np.zeros(len(ts)), nc + ts + 1,
                                  w.scale)
        assert_attn_close(out[l, ts, hs].cpu().numpy(), lse[l, ts, hs].cpu().numpy(), ro, rl,
                          f"prefill262k layer {l}")


@pytest.mark.parametrize("slabs", [1, 2, 3, 5, 7])
def test_bounded_workspace_chunks_bit_identical(kvq, slabs):
    """A workspace of fewer slabs than (layer, KV head) pairs (2 layers x 4 heads = 8):
    one slab runs the pairs one at a time; more alternate chunks of slabs // 2 pairs
    between two streams.  Every size gives the bits of the full workspace."""
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=16448, T=64)
    T, nc, L = 64, 16448, 2
    n = nc + T
    cache, _ = fill_both(w, list(range(L)), n, -(-n // 8) * 8)
    q = torch.from_numpy(np.stack([wl.q_rows(w, l, T) for l in range(L)])).cuda()
    Hq, D = w.n_q_heads, w.head_dim
    slab = kvq.kvq_prefill_workspace_bytes(1, 1, D, n)
    assert kvq.kvq_prefill_workspace_bytes(L, w.n_kv_heads, D, n) == 8 * slab

    def run(nbytes):
        out = torch.full((L, T, Hq, D), float("nan"), device="cuda")
        lse = torch.full((L, T, Hq), float("nan"), device="cuda")
        ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
        kvq.kvq_prefill_attn(cache.layers(), q, Hq, T, nc, 1024, w.scale, out, lse, workspace=ws)
        kvq.kvq_check()
        return out, lse

    ref_out, ref_lse = run(8 * slab)
    out, lse = run(slabs * slab + 256)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    with pytest.raises(kvq.KvqError) as e:
        run(slab - 256)
    assert e.value.status == kvq.KVQ_ERR_WORKSPACE


@pytest.mark.parametrize("Hq,H,n_cached,T,page", [
    (6, 1, 16300, 300, 256),    # exact + tensor-core rows; later pages fully masked for early rows
    (6, 1, 16384, 512, 256),    # tensor-core CTAs whose keys end before the last page
    (24, 4, 16448, 128, 4096),  # the default heads, five pages
])
def test_page_partials(kvq, Hq, H, n_cached, T, page):
    """The optional per-page partials [T][Hq][n_pages][D] and lse, element by element
    against the oracle's pages (a page a row sees nothing of is out = 0, lse = -inf),
    and out / lse as their merge against the oracle's one-pass result."""
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=n_cached, T=T, n_q_heads=Hq, n_kv_heads=H)
    n = n_cached + T
    cache, orc = fill_both(w, [0], n, -(-n // 8) * 8)
    q = np.stack([wl.q_rows(w, 0, T)])
    D, n_pages = w.head_dim, -(-n // page)
    out = torch.full((1, T, Hq, D), float("nan"), device="cuda")
    lse = torch.full((1, T, Hq), float("nan"), device="cuda")
    po = torch.full((1, T, Hq, n_pages, D), float("nan"), device="cuda")
    pl = torch.full((1, T, Hq, n_pages), float("nan"), device="cuda")
    kvq.kvq_prefill_attn(cache.layers(), torch.from_numpy(q).cuda(), Hq, T, n_cached, page,
                         w.scale, out, lse, page_out=po, page_lse=pl)
    kvq.kvq_check()
    ro, rl, rpo, rpl = oracle.prefill_attn(orc[0][0], orc[0][1], q[0], n_cached, page, w.scale,
                                           pages=True)
    gpo, gpl = po.cpu().numpy()[0], pl.cpu().numpy()[0]
    assert_attn_close(gpo, gpl, rpo, rpl, "page partials")
    masked = np.isneginf(rpl)
    assert np.isneginf(gpl[masked]).all() and (gpo[masked] == 0).all()
    assert_attn_close(out.cpu().numpy()[0], lse.cpu().numpy()[0], ro, rl, "merged pages")


@pytest.mark.parametrize("expand", [False, True])
def test_prefill_bounded_wait_times_out_and_context_survives(kvq, expand):
    """The prefill test hook makes one bounded wait of the first CTA of each
    tensor-core launch (the tile expansion and the attention kernel) run out after
    about a second: kvq_check reports KVQ_ERR_TIMEOUT, the CTAs free their tensor
    memory, and the next call on the same context matches the oracle."""
    n_cached, T = 16448, 128
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=n_cached, T=T)
    n = n_cached + T
    cache, orc = fill_both(w, [0], n, -(-n // 8) * 8)
    q = np.stack([wl.q_rows(w, 0, T)])
    with kvq.test_hooks(prefill_timeout=True):
        with pytest.raises(kvq.KvqError) as e:
            run_prefill(kvq, cache, q, w.n_q_heads, T, n_cached, w.scale, expand=expand)
    assert e.value.status == kvq.KVQ_ERR_TIMEOUT
    kvq.kvq_check()  # cleared
    out, lse = run_prefill(kvq, cache, q, w.n_q_heads, T, n_cached, w.scale, expand=expand)
    ro, rl = oracle.prefill_attn(orc[0][0], orc[0][1], q[0], n_cached, 1024, w.scale)
    assert_attn_close(out[0], lse[0], ro, rl, "after timeout")


@pytest.mark.parametrize("Hq,H,D,n_cached,T", [
    (8, 2, 512, 3000, 24),       # head_dim 512: the exact kernel (tensor cores need 256)
    (4, 4, 256, 16400, 160),     # G = 1: 160 rows per head, tensor cores, ragged tile
    (16, 2, 256, 16350, 48),     # G = 8: exact rows (t < 34) then tensor-core rows
    (32, 1, 256, 16448, 8),      # G = 32: one 256-row head, two row tiles
    (32, 1, 128, 500, 6),        # G = 32 at head_dim 128 on the exact kernel
])
def test_head_dims_and_group_sizes(kvq, Hq, H, D, n_cached, T):
    """Other head_dims and GQA ratios against the oracle, with the workspace path
    bit-identical to the in-CTA dequantization where the tensor cores run."""
    w = wl.small(wl.WORKLOADS["prefill262k"], n_cached=n_cached, T=T, n_q_heads=Hq,
                 n_kv_heads=H, head_dim=D)
    check(kvq, w, 1, T, n_cached)
