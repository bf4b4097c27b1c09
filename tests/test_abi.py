"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments with the documented status before launching anything
(these calls make no CUDA compute call, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvq():
    from quantized_kv_long_b200 import build
    build.build()
    from quantized_kv_long_b200 import kvq as m
    return m


def _declared():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(kvq):
    names = _declared()
    assert len(names) >= 12
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(kvq.EXPORTED)


def test_status_strings(kvq):
    for s in range(8):
        assert kvq.kvq_status_string(s) not in ("", "unknown status")
    assert kvq.kvq_status_string(99) == "unknown status"
    assert kvq.kvq_version() >= 100


def _raises(kvq, status, fn, *a, **k):
    with pytest.raises(kvq.KvqError) as e:
        fn(*a, **k)
    assert e.value.status == status, str(e.value)
    assert kvq.kvq_last_error()


A = 1 << 20  # a 16-byte aligned fake device address: never dereferenced here


def _layer(kvq, **kw):
    d = dict(k=A, v=A, capacity=1024, n_kv_heads=4, head_dim=256, k_type=0, v_type=0)
    d.update(kw)
    return kvq.kvq_layer(d["k"], d["v"], d["capacity"], d["n_kv_heads"], d["head_dim"],
                         d["k_type"], d["v_type"])


def test_quantize_validation(kvq):
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_quantize_q8_0, A, A, 33, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_quantize_q4_0, A, A, -32, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_quantize_q8_0, None, A, 64, 0)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, kvq.kvq_quantize_q4_0, A + 2, A, 64, 0)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, kvq.kvq_quantize_q8_0, A, A + 1, 64, 0)
    kvq.kvq_quantize_q8_0(None, None, 0, 0)  # n == 0 launches nothing
    # OSCAR2: whole 128-element blocks, 4-byte aligned blocks (two fp16 words)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_quantize_oscar2, A, A, 96, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_quantize_oscar2, None, A, 128, 0)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, kvq.kvq_quantize_oscar2, A, A + 2, 128, 0)
    kvq.kvq_quantize_oscar2(None, None, 0, 0)


def test_append_validation(kvq):
    L = _layer(kvq)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, L, None, A, 0, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, kvq.kvq_append, L, A + 4, A, 0, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, L, A, A, 1020, 5, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, L, A, A, -1, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, L, A, A, 0, 0, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, _layer(kvq, capacity=1020), A, A, 0, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, kvq.kvq_append, _layer(kvq, k=A + 8), A, A, 0, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_UNSUPPORTED, kvq.kvq_append, _layer(kvq, head_dim=48), A, A, 0, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_UNSUPPORTED, kvq.kvq_append, _layer(kvq, head_dim=1024), A, A, 0, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, [L, _layer(kvq, n_kv_heads=2)], A, A, 0,
            1, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, [L] * 65, A, A, 0, 1, 0)


def test_decode_validation(kvq):
    L = _layer(kvq)
    ok = dict(q=A, n_q_heads=24, T=1, n_kv=1024, chunk=256, scale=1 / 16, out_part=A,
              lse_part=A, stream=0)

    def call(**kw):
        d = dict(ok)
        d.update(kw)
        kvq.kvq_decode_attn(L, **d)

    def bad(status, **kw):
        _raises(kvq, status, call, **kw)

    bad(kvq.KVQ_ERR_INVALID_ARG, q=None)
    bad(kvq.KVQ_ERR_ALIGNMENT, q=A + 2)
    bad(kvq.KVQ_ERR_ALIGNMENT, out_part=A + 4)
    bad(kvq.KVQ_ERR_INVALID_ARG, n_q_heads=25)
    bad(kvq.KVQ_ERR_INVALID_ARG, T=0)
    bad(kvq.KVQ_ERR_UNSUPPORTED, T=5)
    bad(kvq.KVQ_ERR_UNSUPPORTED, n_q_heads=48, T=3)
    bad(kvq.KVQ_ERR_INVALID_ARG, chunk=100)
    bad(kvq.KVQ_ERR_INVALID_ARG, chunk=0)
    bad(kvq.KVQ_ERR_INVALID_ARG, n_kv=1025)
    bad(kvq.KVQ_ERR_INVALID_ARG, n_kv=3, T=4)
    bad(kvq.KVQ_ERR_INVALID_ARG, scale=float("nan"))


def test_merge_validation(kvq):
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_merge_lse, None, A, 4, 2, 256, A, A, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_merge_lse, A, A, 4, 0, 256, A, A, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_merge_lse, A, A, -1, 2, 256, A, A, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_merge_lse, A, A, 4, 2, 30, A, A, 0)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, kvq.kvq_merge_lse, A, A, 4, 2, 256, A + 4, A, 0)


def test_decode_step_validation(kvq):
    """kvq_decode_step: the decode and merge checks plus k_new / v_new, all before the
    first launch; the workspace is reserved (0 bytes, not read)."""
    L = [_layer(kvq)] * 16
    assert kvq.kvq_workspace_bytes(kvq.KVQ_OP_DECODE_STEP, 16, 24, 4, 4, 256) == 0
    ok = dict(k_new=A, v_new=A, q=A, n_q_heads=24, T=4, n_kv=1024, chunk=256, scale=1 / 16,
              out_part=A, lse_part=A, out=A, lse=A, workspace=None, ws_bytes=0, stream=0)

    def call(**kw):
        d = dict(ok)
        d.update(kw)
        kvq.kvq_decode_step(L, **d)

    def bad(status, **kw):
        _raises(kvq, status, call, **kw)

    bad(kvq.KVQ_ERR_INVALID_ARG, k_new=None)
    bad(kvq.KVQ_ERR_ALIGNMENT, v_new=A + 4)
    bad(kvq.KVQ_ERR_INVALID_ARG, q=None)
    bad(kvq.KVQ_ERR_UNSUPPORTED, T=5)
    bad(kvq.KVQ_ERR_INVALID_ARG, n_kv=3)
    bad(kvq.KVQ_ERR_INVALID_ARG, n_kv=1025)
    bad(kvq.KVQ_ERR_ALIGNMENT, out=A + 4)
    bad(kvq.KVQ_ERR_INVALID_ARG, lse=None)


def test_prefill_validation(kvq):
    L = _layer(kvq, capacity=4096)
    ok = dict(q=A, n_q_heads=24, T=128, n_cached=1024, page=1024, scale=1 / 16, out=A, lse=A,
              stream=0)

    def call(**kw):
        d = dict(ok)
        d.update(kw)
        kvq.kvq_prefill_attn(L, **d)

    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, call, page=100)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, call, n_cached=4000)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, call, page_out=A)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, call, page_out=A + 4, page_lse=A)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, call, page_out=A, page_lse=A + 2)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, call, T=0)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, call, out=A + 4)


def test_stream_validation(kvq):
    L = _layer(kvq)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_stream_decode, [L], [L, _layer(kvq, head_dim=128)],
            A, 24, 1, 1024, 256, 1 / 16, A, A, A, A, 0, 0)
    with pytest.raises(ValueError):
        kvq.kvq_stream_decode([L], [L], A, 24, 1, 1024, 256, 1 / 16, A, A, A, A, 0, 0)


def test_workspace_query(kvq):
    assert kvq.kvq_workspace_bytes(kvq.KVQ_OP_DECODE, 16, 24, 4, 4, 256) == 0
    # prefill requires no workspace; its optional one is kvq_prefill_workspace_bytes
    assert kvq.kvq_workspace_bytes(kvq.KVQ_OP_PREFILL, 16, 24, 4, 2048, 256) == 0
    assert kvq.kvq_prefill_workspace_bytes(16, 4, 256, 264192) > 0
    assert kvq.kvq_workspace_bytes(kvq.KVQ_OP_DECODE_STEP, 16, 24, 4, 4, 256) == 0
    assert kvq.kvq_workspace_bytes(99, 1, 1, 1, 1, 32) == ctypes.c_size_t(-1).value


def test_test_hooks_set_and_clear(kvq):
    """The hooks are plain process-wide switches: set, then cleared by the context
    manager (host only; no kernel runs)."""
    with kvq.test_hooks(decode_general=True, stream_fail_layer=3):
        pass
    kvq.kvq_test_set_hooks()  # all off
    assert kvq._lib.kvq_test_set_hooks(None) == kvq.KVQ_OK


def test_resident_layers_plan(kvq):
    """Host arithmetic of the residency plan: 16 layers x 4 heads x 262,144 tokens
    x (272 + 144) B = 436,207,616 B per layer."""
    lb = 4 * 262144 * (272 + 144)
    plan = lambda budget, n=16: kvq.kvq_resident_layers(budget, n, 262144, 4, 256)
    assert plan(16 * lb) == 16          # everything fits: no slots
    assert plan(16 * lb - 1) == 13      # 13 resident + 2 slots = 15 layers of memory
    assert plan(3 * lb) == 1
    assert plan(2 * lb) == 0            # only the two slots
    assert plan(2 * lb - 1) == -1       # not even the slots
    assert plan(2100 << 20) == 3        # the ~2,100 MiB decode working set of the pages
    assert plan(10**15, 1) == 1
    assert kvq.kvq_resident_layers(1 << 40, 0, 1024, 4, 256) == -1
    assert kvq.kvq_resident_layers(1 << 40, 4, 1024, 4, 48) == -1


def test_block_format_validation(kvq):
    """Block formats: unknown types and layers that differ are refused (prefill
    included); the residency plan sizes layers by format."""
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, _layer(kvq, k_type=4), A, A, 0, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, _layer(kvq, v_type=-1), A, A, 0, 1, 0)
    # explicit Q8_0 K / Q4_0 V equals the default pair, so these two layers agree
    mixed_ok = [_layer(kvq), _layer(kvq, k_type=kvq.KVQ_TYPE_Q8_0, v_type=kvq.KVQ_TYPE_Q4_0)]
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_append, mixed_ok + [_layer(kvq, v_type=1)],
            A, A, 0, 1, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_decode_attn,
            [_layer(kvq, k_type=2), _layer(kvq)], A, 24, 1, 1024, 256, 1 / 16, A, A, 0)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_prefill_attn,
            [_layer(kvq, v_type=1, capacity=4096), _layer(kvq, capacity=4096)],
            A, 24, 128, 1024, 1024, 1 / 16, A, A)
    # an OSCAR2 tensor needs whole 128-element blocks in a head-row
    O2 = kvq.KVQ_TYPE_OSCAR2
    for call in (lambda L: kvq.kvq_append(L, A, A, 0, 1, 0),
                 lambda L: kvq.kvq_decode_attn(L, A, 4, 1, 1024, 256, 1 / 16, A, A, 0),
                 lambda L: kvq.kvq_prefill_attn(L, A, 4, 128, 512, 1024, 1 / 16, A, A)):
        _raises(kvq, kvq.KVQ_ERR_UNSUPPORTED, call, _layer(kvq, head_dim=96, v_type=O2))
        _raises(kvq, kvq.KVQ_ERR_UNSUPPORTED, call, _layer(kvq, head_dim=320, k_type=O2))
    q8 = 4 * 262144 * (272 + 272)
    assert kvq.kvq_resident_layers(5 * q8, 16, 262144, 4, 256, 1, 1) == 3
    assert kvq.kvq_resident_layers(5 * q8, 16, 262144, 4, 256, 0, 0) == 4
    assert kvq.kvq_resident_layers(5 * q8, 16, 262144, 4, 256, 7, 0) == -1
    # OSCAR2 K and V head-rows of 72 B each: the bytes of 3 Q8_0/Q8_0 layers hold 11.3
    # OSCAR2 layers, 9 of them beside the 2 streaming slots; 5 hold all 16
    assert kvq.kvq_resident_layers(3 * q8, 16, 262144, 4, 256, O2, O2) == 9
    assert kvq.kvq_resident_layers(5 * q8, 16, 262144, 4, 256, O2, O2) == 16
    assert kvq.kvq_resident_layers(5 * q8, 16, 262144, 4, 96, O2, O2) == -1


def test_prefill_workspace_validation(kvq):
    """The optional prefill workspace: its size for the expanded f16 key tiles (one
    slab per (layer, KV head) pair), and one smaller than a slab or misaligned
    refused before anything is launched."""
    nb = kvq.kvq_prefill_workspace_bytes(16, 4, 256, 264192)
    assert nb == 16 * 4 * 8256 * 49152
    assert kvq.kvq_prefill_workspace_bytes(1, 1, 256, 264192) == 8256 * 49152  # one slab
    assert kvq.kvq_prefill_workspace_bytes(1, 4, 128, 1000) == 0  # no tensor-core path
    L = _layer(kvq, capacity=4096)
    need = kvq.kvq_prefill_workspace_bytes(1, 1, 256, 1024 + 128)
    args = (L, A, 24, 128, 1024, 1024, 1 / 16, A, A)
    _raises(kvq, kvq.KVQ_ERR_WORKSPACE, kvq.kvq_prefill_attn, *args, workspace=A,
            ws_bytes=need - 1)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, kvq.kvq_prefill_attn, *args, workspace=A + 16,
            ws_bytes=need)


def test_decode_step_host_validation(kvq):
    """kvq_decode_step_host refuses NULL host buffers and bad device arguments before
    the first copy (nothing runs on a device here)."""
    L = [_layer(kvq)]
    d = dict(n_q_heads=24, T=4, n_kv=1000, chunk=1024, scale=1 / 16, out_part=A, lse_part=A,
             out=A, lse=A)
    host = (A, A, A, A, A)
    dev = (A, A, A)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_decode_step_host, L, None, *host[1:], *dev,
            **d)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_decode_step_host, L, *host[:4], None, *dev,
            **d)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_decode_step_host, L, *host, A, A, None, **d)
    _raises(kvq, kvq.KVQ_ERR_ALIGNMENT, kvq.kvq_decode_step_host, L, *host, A + 4, A, A, **d)
    _raises(kvq, kvq.KVQ_ERR_INVALID_ARG, kvq.kvq_decode_step_host, L, *host, *dev,
            **dict(d, n_kv=2000))  # beyond the capacity


def test_cache_row_sizes_per_format(kvq):
    """Head-row bytes of each block format, as the cache helper allocates them (host
    memory here): 34, 18 and 9 bytes per 32 elements; OSCAR2 needs whole 128-element
    blocks."""
    assert kvq.row_bytes(kvq.KVQ_TYPE_DEFAULT, "k", 256) == 272
    assert kvq.row_bytes(kvq.KVQ_TYPE_DEFAULT, "v", 256) == 144
    assert kvq.row_bytes(kvq.KVQ_TYPE_OSCAR2, "k", 256) == 72
    assert kvq.row_bytes(kvq.KVQ_TYPE_OSCAR2, "v", 512) == 144
    c = kvq.QuantizedKVCache(2, 4, 256, 16, device="cpu", k_type=kvq.KVQ_TYPE_Q8_0,
                             v_type=kvq.KVQ_TYPE_OSCAR2)
    assert tuple(c.k[0].shape) == (4, 16, 272) and tuple(c.v[1].shape) == (4, 16, 72)
    assert c.nbytes == 2 * 4 * 16 * (272 + 72)
    assert (c.layer(1).k_type, c.layer(1).v_type) == (1, 3)
