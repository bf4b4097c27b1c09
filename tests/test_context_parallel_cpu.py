"""The context-parallel split on CPU: two (and three) gloo ranks, no GPU.

Each rank takes its shard of the context (``context_parallel.shard_range``),
computes the shard's merged rows with the oracle (one-pass attention over the
shard's keys that each row sees, which is what decode + merge over the shard's
chunks computes), and the ranks exchange and merge them with
``context_parallel.gather_merge`` over gloo, the merge done by the oracle.  The
result on every rank must match the oracle's one-pass attention over the whole
context.  The verify batch's causal tail lies in the last shard, whose rows
see different numbers of its keys.  (Shards that some rows do not see at all
are covered by the GPU tests of kvq_decode_attn_shard.)
"""
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from quantized_kv_long_b200 import context_parallel as cp
from quantized_kv_long_b200 import workload as wl

from helpers import assert_attn_close

N_KV, CHUNK, T = 1283, 128, 4  # 11 chunks; the causal tail is keys 1,279..1,282


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _caches(w):
    kc, vc = oracle.empty_cache(w.n_kv_heads, w.head_dim, N_KV)
    oracle.append(kc, vc, wl.kv_rows(w, 0, 0, 0, N_KV), wl.kv_rows(w, 0, 1, 0, N_KV), 0)
    return kc, vc


def _rows(w, q):
    """Every (token, query head) row: q rows, head index, token index."""
    Hq = w.n_q_heads
    t = np.repeat(np.arange(T), Hq)
    h = np.tile(np.arange(Hq), T)
    return q.reshape(T * Hq, -1), h, t


def _oracle_merge_parts(parts_out, parts_lse, out, lse):
    """[W, rows, D] / [W, rows] -> out [rows, D], lse [rows] with the oracle's merge."""
    po = parts_out.numpy().astype(np.float64).transpose(1, 0, 2)
    pl = parts_lse.numpy().astype(np.float64).T
    o, l = oracle.merge_lse(po, pl)
    out.copy_(torch.from_numpy(o))
    lse.copy_(torch.from_numpy(l))


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = wl.small(wl.WORKLOADS["verify262k"], n_kv=N_KV, n_layers=1)
        kc, vc = _caches(w)
        q = wl.q_rows(w, 0, T)
        qr, h, t = _rows(w, q)
        key0, n_keys = cp.shard_range(N_KV, world, rank, CHUNK, T)
        # this shard's keys that each row sees: [key0, min(key0 + n_keys, N_KV - T + t + 1))
        end = np.minimum(key0 + n_keys, N_KV - T + t + 1)
        begin = np.minimum(np.full_like(end, key0), end)
        o, l = oracle.attn_rows(kc, vc, qr, h, w.n_q_heads, begin, end, w.scale)
        out_r = torch.from_numpy(o.astype(np.float32))
        lse_r = torch.from_numpy(l.astype(np.float32))
        out = torch.empty_like(out_r)
        lse = torch.empty_like(lse_r)
        cp.gather_merge(out_r, lse_r, out, lse, _oracle_merge_parts)
        np.save(os.path.join(out_dir, f"out{rank}.npy"), out.numpy())
        np.save(os.path.join(out_dir, f"lse{rank}.npy"), lse.numpy())
        with open(os.path.join(out_dir, f"shard{rank}.json"), "w") as f:
            json.dump([key0, n_keys, int((end > begin).sum())], f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_match_one_pass(tmp_path, world):
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    w = wl.small(wl.WORKLOADS["verify262k"], n_kv=N_KV, n_layers=1)
    kc, vc = _caches(w)
    qr, h, t = _rows(w, wl.q_rows(w, 0, T))
    ro, rl = oracle.attn_rows(kc, vc, qr, h, w.n_q_heads, np.zeros_like(t), N_KV - T + t + 1,
                              w.scale)
    shards = [json.load(open(tmp_path / f"shard{r}.json")) for r in range(world)]
    # the shards tile the context in order
    assert shards[0][0] == 0 and sum(s[1] for s in shards) == N_KV
    assert all(shards[r][0] + shards[r][1] == shards[r + 1][0] for r in range(world - 1))
    assert all(s[2] > 0 for s in shards)  # every shard is seen by some row
    for r in range(world):
        out = np.load(tmp_path / f"out{r}.npy")
        lse = np.load(tmp_path / f"lse{r}.npy")
        assert_attn_close(out, lse, ro, rl, f"rank {r} of {world}")


def test_shard_range_edges():
    # 11 chunks over 4 ranks: 2, 3, 3, 3 chunks; the last shard ends at n_kv
    got = [cp.shard_range(1283, 4, r, 128, 4) for r in range(4)]
    assert got == [(0, 256), (256, 384), (640, 384), (1024, 259)]
    with pytest.raises(ValueError):
        cp.shard_range(300, 4, 0, 128)  # 3 chunks, 4 ranks
    assert cp.shard_range(258, 2, 1, 128, T=4) == (128, 130)  # chunks 1..2
    with pytest.raises(ValueError):
        cp.shard_range(130, 2, 1, 128, T=4)  # the last shard holds 2 keys < T
