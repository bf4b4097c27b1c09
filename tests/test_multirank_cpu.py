"""The N > 1 host path of bench.py on CPU: two gloo ranks (no GPU).

bench.py runs one independent replica per rank (weak scaling, no data-path
collective).  The ranks meet only at the timing barriers and in the max-over-
ranks reduction of the step time; the whole-job value is world x bytes per
rank / the slowest rank's time, and only rank 0 prints.  The reference arm
(the oracle) runs on rank 0 alone; the other ranks exit 0 without work.
"""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # a slower rank 1: the step time is the max over ranks, on every rank
        ms = [2.5, 4.0][rank]
        bench.barrier()
        ms_max = bench.reduce_max(ms)
        bench.barrier()
        gbs = bench.weak_gbs(world, 6_979_321_856, ms_max)
        rec = {"rank": rank, "dist_env": list(bench.dist_env()), "ms_max": ms_max, "gbs": gbs}
        # reference arm: rank 1 must do no work and print nothing
        if rank == 1:
            import contextlib
            import io
            buf = io.StringIO()
            with contextlib.redirect_stdout(buf):
                rc = bench.main(["--impl", "reference", "--config", "tiny", "--steps", "1",
                                 "--warmup", "3"])
            rec["ref_rc"] = rc
            rec["ref_stdout"] = buf.getvalue()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(rec, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    recs = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, rec in enumerate(recs):
        assert rec["dist_env"] == [r, world, r]
        assert rec["ms_max"] == pytest.approx(4.0)  # the slowest rank's time, on every rank
        # 2 replicas x 6.98 GB in 4 ms
        assert rec["gbs"] == pytest.approx(2 * 6_979_321_856 / 4e-3 / 1e9)
    assert recs[1]["ref_rc"] == 0 and recs[1]["ref_stdout"] == ""


def test_weak_gbs_single_rank():
    assert bench.weak_gbs(1, 1_000_000_000, 1000.0) == pytest.approx(1.0)
