"""Benchmark of the quantized-KV decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config verify262k|decode65k|stream262k|tiny]

One step (default workload ``verify262k``: 16 attention layers, 24 query heads
over 4 Q8_0/Q4_0 KV heads of 256, a 4-token speculative-verify batch against
262,144 keys) is the whole decode hot path of one batch:

  1. quantize-append the 4 new K/V rows of every layer (kvq_append, 1 launch),
  2. split-KV GQA decode attention of all 16 layers, chunk 4,096
     (kvq_decode_attn, 1 launch, per-chunk out + lse),
  3. LSE merge of the 64 chunk partials of every row (kvq_merge_lse, 1 launch).

``value`` is KV GB/s of the whole job: quantized KV bytes the step attends
over (16 x 262,144 x 1,664 B = 6.98 GB) times steps, over the max-over-ranks
device time.  Inputs are resident in HBM (the 7 GB cache is far larger than
the 126 MB L2, so no flush is needed).  ``e2e`` is the same metric through the
C-ABI with host buffers (``kvq_decode_step_host``): every step copies q and the
new rows from pinned host memory and copies out + lse back, inside the timed
region.

With --gpus N > 1 (torchrun, one rank per GPU, NCCL) every rank runs its own
independent sequence (weak scaling, no data-path collective); ranks meet only
at the timing barriers and the max-over-ranks reduction.

``--impl reference`` times the CPU oracle (fp64, OpenMP) on a bounded sample of
the same workload per step; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from quantized_kv_long_b200 import context_parallel as cp  # noqa: E402
from quantized_kv_long_b200 import workload as wl  # noqa: E402

METRIC = "q8_0/q4_0 decode attn: KV GB/s (% of HBM peak), query-tok/s at 262k ctx"
FALLBACK_HBM_GBS = 6650.0
KV_BYTES_PER_TOKEN_LAYER = lambda w: w.n_kv_heads * (w.head_dim // 32) * (34 + 18)  # noqa: E731
# --kv-formats: (K block type, V block type) of the C ABI and the bytes per 32 elements of
# each (OSCAR2: 36 B per 128 elements = 9 B per 32)
KV_FORMATS = {"q8_0/q4_0": (1, 2, 34, 18), "q8_0/q8_0": (1, 1, 34, 34),
              "q4_0/q4_0": (2, 2, 18, 18), "q4_0/q8_0": (2, 1, 18, 34),
              "oscar2/oscar2": (3, 3, 9, 9), "q8_0/oscar2": (1, 3, 34, 9)}


# --------------------------------------------------------------------------- helpers

def peaks() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def reduce_max(x: float, device=None) -> float:
    """Max over ranks (identity when torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_gbs(world: int, bytes_per_rank: int, ms_max: float) -> float:
    """Whole-job GB/s of a weak-scaling run: every rank moves `bytes_per_rank`
    per step, and the step time is the slowest rank's (`ms_max`)."""
    return world * bytes_per_rank / (ms_max * 1e-3) / 1e9


def barrier(device=None) -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except FileNotFoundError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9 and p[1].replace(".", "").isdigit():
                    rows.append(p)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


def gpu_id(torch, device) -> str:
    """nvidia-smi -i argument for this device (its UUID when torch knows it)."""
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        return str(device.index)


def source_hash(*names: str) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "quantized_kv_long_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel_files: tuple[str, ...], record: str = "decode_traffic.json"):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the kernel source as it is now (else None)."""
    p = os.path.join(ROOT, "profiles", record)
    try:
        rec = json.load(open(p))
    except Exception:
        return None
    if rec.get("source_hash") != source_hash(*kernel_files):
        return None
    return rec


# --------------------------------------------------------------------------- our arm

def fill_cache(kvq, torch, w: wl.Workload, device, k_type: int = 0, v_type: int = 0,
               key0: int = 0, n_keys: int | None = None):
    """Quantize the context of every layer into a device cache (setup, untimed):
    keys [key0, key0 + n_keys) (default: all n_kv) drawn per layer by the seeded
    generator, at cache rows [0, n_keys)."""
    n_keys = w.n_kv if n_keys is None else n_keys
    cap = w.capacity if (key0, n_keys) == (0, w.n_kv) else -(-n_keys // 8) * 8
    cache = kvq.QuantizedKVCache(w.n_layers, w.n_kv_heads, w.head_dim, cap, device=device,
                                 k_type=k_type, v_type=v_type)
    for l in range(w.n_layers):
        for start in range(key0, key0 + n_keys, 131072):
            stop = min(key0 + n_keys, start + 131072)
            k = torch.from_numpy(wl.kv_rows(w, l, 0, start, stop)).to(device)
            v = torch.from_numpy(wl.kv_rows(w, l, 1, start, stop)).to(device)
            kvq.kvq_append(cache.layer(l), k, v, start - key0, stop - start)
    torch.cuda.synchronize(device)
    return cache


def run_ours(args, w: wl.Workload) -> dict | None:
    import torch
    import torch.distributed as dist
    from quantized_kv_long_b200 import kvq

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)

    L, T, Hq, D, n_kv, chunk = w.n_layers, w.T, w.n_q_heads, w.head_dim, w.n_kv, w.chunk
    rows = L * T * Hq
    k_type, v_type, k_blk, v_blk = KV_FORMATS[args.kv_formats]
    # --split context: this rank holds keys [key0, key0 + n_keys) of every layer and the
    # ranks exchange their merged rows; replicas: every rank holds the whole context
    split = args.split == "context"
    key0, n_keys = cp.shard_range(n_kv, world, rank, chunk) if split else (0, n_kv)
    C = -(-n_keys // chunk)
    cache = fill_cache(kvq, torch, w, device, k_type, v_type, key0, n_keys)
    layers = cache.layers()
    # the new rows [n_kv - T, n_kv) that fall in this rank's keys
    a0, a1 = max(n_kv - T, key0), min(n_kv, key0 + n_keys)
    # the step's inputs: q and the T new rows of every layer (rows n_kv-T .. n_kv-1)
    q_h = np.stack([wl.q_rows(w, l) for l in range(L)])
    k_h = np.stack([wl.kv_rows(w, l, 0, n_kv - T, n_kv) for l in range(L)])
    v_h = np.stack([wl.kv_rows(w, l, 1, n_kv - T, n_kv) for l in range(L)])
    q = torch.from_numpy(q_h).to(device)
    k_new = torch.from_numpy(k_h).to(device)
    v_new = torch.from_numpy(v_h).to(device)
    op = torch.empty((L, T, Hq, C, D), device=device)
    lp = torch.empty((L, T, Hq, C), device=device)
    out = torch.empty((L, T, Hq, D), device=device)
    lse = torch.empty((L, T, Hq), device=device)
    exchange = split and world > 1
    if exchange:
        out_r = torch.empty((rows, D), device=device)
        lse_r = torch.empty((rows,), device=device)

        def merge_parts(po, pl, o, l):
            kvq.kvq_merge_lse_parts(po, pl, world, rows, D, o, l, stream)

    # this rank's part of the new rows (a view when it is all of them; the e2e copies
    # below refresh k_new / v_new, so a partial part is a view too: rows a0.. of dim 1)
    k_app = k_new[:, a0 - (n_kv - T):a1 - (n_kv - T)]
    v_app = v_new[:, a0 - (n_kv - T):a1 - (n_kv - T)]
    if a1 > a0 and (a0, a1) != (n_kv - T, n_kv):
        k_app, v_app = k_app.contiguous(), v_app.contiguous()  # [L][a1 - a0][H][D]
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]

    def step(i=None):
        # append, decode, merge: the three launches of kvq_decode_step, issued one by one
        # so that the decode launch can be timed on its own (a context split decodes this
        # rank's shard, merges it, all-gathers the merged rows and merges the ranks')
        if a1 > a0:
            kvq.kvq_append(layers, k_app, v_app, a0 - key0, a1 - a0, stream)
        if i is not None:
            ev_dec[i][0].record(stream)
        kvq.kvq_decode_attn_shard(layers, q, Hq, T, n_keys, key0, n_kv, chunk, w.scale, op, lp,
                                  stream)
        if i is not None:
            ev_dec[i][1].record(stream)
        if not exchange:
            kvq.kvq_merge_lse(op, lp, rows, C, D, out, lse, stream)
            return
        kvq.kvq_merge_lse(op, lp, rows, C, D, out_r, lse_r, stream)
        cp.gather_merge(out_r, lse_r, out.view(rows, D), lse.view(rows), merge_parts)

    for _ in range(args.warmup):
        step()
    kvq.kvq_check(stream)

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id(torch, device)) as clocks:
        barrier(device)
        torch.cuda.synchronize(device)
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
    kvq.kvq_check(stream)
    ms_local = t0.elapsed_time(t1) / args.steps
    dec_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_dec)
    ms = reduce_max(ms_local, device)
    dec_ms_max = reduce_max(dec_ms, device)

    # ---- e2e: the same step through the C ABI with host buffers
    q_pin = torch.from_numpy(q_h).pin_memory()
    k_pin = torch.from_numpy(k_h).pin_memory()
    v_pin = torch.from_numpy(v_h).pin_memory()
    out_pin = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_pin = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

    def e2e_step():
        if not split:
            # one library call: host inputs in, append + decode + merge, host results out
            kvq.kvq_decode_step_host(layers, k_pin, v_pin, q_pin, out_pin, lse_pin, k_new, v_new,
                                     q, Hq, T, n_kv, chunk, w.scale, op, lp, out, lse, stream)
            return
        q.copy_(q_pin, non_blocking=True)
        k_new.copy_(k_pin, non_blocking=True)
        v_new.copy_(v_pin, non_blocking=True)
        step()
        out_pin.copy_(out, non_blocking=True)
        lse_pin.copy_(lse, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, args.steps // 2)
    barrier(device)
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, device)
    h2d = q_pin.numel() * 2 + k_pin.numel() * 4 + v_pin.numel() * 4
    d2h = out_pin.numel() * 4 + lse_pin.numel() * 4

    # sanity: outputs are finite (the parity tests check them against the oracle)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()

    tok_bytes = L * w.n_kv_heads * (D // 32) * (k_blk + v_blk)  # one key of every layer
    kv_bytes = n_kv * tok_bytes    # the context of one replica, or of all ranks when split
    # a replica reads its whole context; a context split divides one context over the ranks
    per_rank = weak_gbs(world, kv_bytes, ms) if not split else kv_bytes / (ms * 1e-3) / 1e9
    e2e_gbs = weak_gbs(world, kv_bytes, e2e_ms) if not split else kv_bytes / (e2e_ms * 1e-3) / 1e9
    peak, peak_kind = peaks()
    cl = clocks.summary()
    res = None
    if rank == 0:
        gbs = per_rank
        # the decode launch of rank 0 against its own keys (the slowest rank's time)
        achieved = n_keys * tok_bytes / (dec_ms_max * 1e-3) / 1e9
        tr = (traffic_record(DECODE_SOURCES)
              if args.kv_formats == "q8_0/q4_0" and (key0, n_keys) == (0, n_kv) else None)
        kf, vf = args.kv_formats.split("/")
        res = {
            "metric": METRIC, "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "strong" if split else "weak",
            "vs_baseline": None,
            "dtype": f"{kf} K / {vf} V x f16 q, f32 accumulate", "data": "synthetic",
            "config": {"workload": w.name, "layers": L, "q_heads": Hq, "kv_heads": w.n_kv_heads,
                       "head_dim": D, "context": n_kv, "query_tokens": T, "chunk": chunk,
                       "seed": w.seed, "kv_bytes_per_step": kv_bytes,
                       "kv_formats": args.kv_formats,
                       "l2": "inputs larger than L2 (7 GB cache vs 126 MB)",
                       "step": ("append, decode, merge: 3 launches" if not exchange else
                                "append, decode of the shard, merge, all-gather (NCCL), merge "
                                "of the ranks' rows"),
                       "parallelism": (f"context{world}" if split and world > 1 else
                                       f"replicas{world}" if world > 1 else "single-gpu")},
            # query tokens per step (each attends all L layers) / step time
            "query_tok_per_s": round((1 if split else world) * T / (ms * 1e-3), 1),
            "layer_query_tok_per_s": round((1 if split else world) * L * T / (ms * 1e-3), 1),
            "pct_hbm_peak": round(100 * gbs / world / peak, 2),
            "e2e": {"value": round(e2e_gbs, 1), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 4),
                    "call": ("kvq_decode_step_host" if not split else
                             "host copies around the split step")},
            "roofline": {"bound": "hbm",
                         "kernel": (f"kvq_decode_attn ({L} layers, 1 launch)" if not split else
                                    f"kvq_decode_attn_shard ({L} layers x {n_keys} keys, "
                                    f"1 launch)"),
                         "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": tr["dram_bytes_per_launch"] if tr else None,
                         "launch_ms": round(dec_ms_max, 4)},
            "gpu_launches": ((a1 > a0) + 2 + exchange) * args.steps,
            "clocks": {"sm_mhz": cl["sm_mhz"], "sm_max_mhz": cl["sm_max_mhz"],
                       "reasons": cl["reasons"], "samples": cl["samples"]},
        }
    del cache
    if world > 1:
        dist.destroy_process_group()
    return res


DECODE_SOURCES = ("decode.cu", "decode_tmem.cu", "decode_frag.cuh", "ptx.cuh", "common.cuh",
                  "merge.cuh", "quant.cuh")
PREFILL_SOURCES = ("prefill.cu", "ptx.cuh", "common.cuh")
STREAM_METRIC = "q8_0/q4_0 host-streamed decode: H2D GB/s (% of measured H2D), query-tok/s at 262k ctx"


def h2d_peak(torch, device, nbytes: int) -> float:
    """Best-of-5 pinned host -> device copy bandwidth (GB/s) of an nbytes buffer."""
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    best = 0.0
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        torch.cuda.synchronize(device)
        best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    return best


def run_stream(args, w: wl.Workload) -> dict | None:
    """The stream262k step: the 16-layer cache lives in pinned host memory; every
    layer is copied into one of two device slots while the previous layer's
    decode attention + merge run on the other (kvq_stream_decode).  With
    --budget-mib, the layers that fit in that much device memory next to the two
    slots (kvq_resident_layers) stay resident and only the rest are streamed."""
    import torch
    import torch.distributed as dist
    from quantized_kv_long_b200 import kvq

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    compute = torch.cuda.current_stream(device)
    copy = torch.cuda.Stream(device)
    L, T, Hq, D, n_kv, chunk = w.n_layers, w.T, w.n_q_heads, w.head_dim, w.n_kv, w.chunk
    C = w.n_chunks
    host = kvq.QuantizedKVCache(L, w.n_kv_heads, D, w.capacity, device="cpu", pin=True)
    tmp = kvq.QuantizedKVCache(1, w.n_kv_heads, D, w.capacity, device=device)
    for l in range(L):  # quantize on the GPU, keep the cache on the host
        for start in range(0, n_kv, 131072):
            stop = min(n_kv, start + 131072)
            k = torch.from_numpy(wl.kv_rows(w, l, 0, start, stop)).to(device)
            v = torch.from_numpy(wl.kv_rows(w, l, 1, start, stop)).to(device)
            kvq.kvq_append(tmp.layer(0), k, v, start, stop - start)
        host.k[l].copy_(tmp.k[0])
        host.v[l].copy_(tmp.v[0])
    del tmp
    layer_bytes = w.capacity * KV_BYTES_PER_TOKEN_LAYER(w)  # one layer, all KV heads
    R = 0
    if args.budget_mib is not None:
        R = kvq.kvq_resident_layers(args.budget_mib << 20, L, w.capacity, w.n_kv_heads, D)
        if R < 0:
            raise SystemExit(f"--budget-mib {args.budget_mib}: not even the two slots fit")
    resident = kvq.QuantizedKVCache(R, w.n_kv_heads, D, w.capacity, device=device) if R else None
    for l in range(R):  # a resident prefix: the plan's layers live on the device
        resident.k[l].copy_(host.k[l])
        resident.v[l].copy_(host.v[l])
    layers = [resident.layer(l) if l < R else host.layer(l) for l in range(L)]
    slots = (kvq.QuantizedKVCache(2, w.n_kv_heads, D, w.capacity, device=device)
             if R < L else None)
    q = torch.from_numpy(np.stack([wl.q_rows(w, l) for l in range(L)])).to(device)
    op = torch.empty((T, Hq, C, D), device=device)
    lp = torch.empty((T, Hq, C), device=device)
    out = torch.empty((L, T, Hq, D), device=device)
    lse = torch.empty((L, T, Hq), device=device)

    def step():
        kvq.kvq_stream_decode(layers, slots, q, Hq, T, n_kv, chunk, w.scale, op, lp, out, lse,
                              compute=compute, copy=copy)

    for _ in range(args.warmup):
        step()
    kvq.kvq_check(compute)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id(torch, device)) as clocks:
        barrier(device)
        torch.cuda.synchronize(device)
        t0.record(compute)
        for _ in range(args.steps):
            step()
        t1.record(compute)
        torch.cuda.synchronize(device)
        barrier(device)
    kvq.kvq_check(compute)
    ms = reduce_max(t0.elapsed_time(t1) / args.steps, device)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    kv_bytes = L * n_kv * KV_BYTES_PER_TOKEN_LAYER(w)
    peak = h2d_peak(torch, device, kv_bytes // L)
    cl = clocks.summary()
    res = None
    streamed = (L - R) * kv_bytes // L
    if rank == 0:
        gbs = world * kv_bytes / (ms * 1e-3) / 1e9
        link = streamed / (ms * 1e-3) / 1e9  # bytes that crossed the link, per GPU
        res = {
            "metric": STREAM_METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "q8_0 K / q4_0 V x f16 q, f32 accumulate", "data": "synthetic",
            "config": {"workload": w.name, "layers": L, "q_heads": Hq, "kv_heads": w.n_kv_heads,
                       "head_dim": D, "context": n_kv, "query_tokens": T, "chunk": chunk,
                       "seed": w.seed, "host_cache_bytes": kv_bytes,
                       "slots": 2 if R < L else 0, "resident_layers": R,
                       "device_budget_mib": args.budget_mib,
                       "device_cache_bytes": (R + (2 if R < L else 0)) * layer_bytes},
            "query_tok_per_s": round(world * T / (ms * 1e-3), 2),
            "layer_query_tok_per_s": round(world * L * T / (ms * 1e-3), 2),
            "roofline": {"bound": "h2d", "kernel": "kvq_stream_decode (copy stream)",
                         "achieved": round(link, 2), "peak": round(peak, 2),
                         "peak_kind": "measured pinned H2D, best of 5, one layer's bytes",
                         "unit": "GB/s", "frac": round(link / peak, 4),
                         "streamed_bytes_per_step": streamed, "traffic": None},
            "gpu_launches": 2 * L * args.steps,
            "clocks": {"sm_mhz": cl["sm_mhz"], "sm_max_mhz": cl["sm_max_mhz"],
                       "reasons": cl["reasons"], "samples": cl["samples"]},
        }
    del host, slots, resident
    if world > 1:
        dist.destroy_process_group()
    return res


PREFILL_METRIC = "q8_0/q4_0 chunked prefill attn: TFLOP/s (% of tensor peak), query-tok/s at 262k ctx"


def prefill_flops(w: wl.Workload) -> float:
    """QK^T and PV multiply-adds of every visible (query row, key) pair, x2 flop."""
    visible = sum(w.n_cached + t + 1 for t in range(w.T))
    return 2.0 * 2.0 * w.head_dim * w.n_q_heads * visible * w.n_layers


def tensor_peak() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (bf16 sustained)"
    except Exception:
        return 1400.0, "fallback (sustained)"


def run_prefill(args, w: wl.Workload) -> dict | None:
    """The prefill262k step: append the 2,048 new rows of every layer, then
    prefill attention of all 16 layers (one launch each)."""
    import torch
    import torch.distributed as dist
    from quantized_kv_long_b200 import kvq

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    L, T, Hq, D, nc = w.n_layers, w.T, w.n_q_heads, w.head_dim, w.n_cached
    cache = fill_cache(kvq, torch, wl.small(w, n_kv=nc + T), device)
    layers = cache.layers()
    q = torch.from_numpy(np.stack([wl.q_rows(w, l) for l in range(L)])).to(device)
    k_new = torch.from_numpy(np.stack([wl.kv_rows(w, l, 0, nc, nc + T) for l in range(L)])).to(device)
    v_new = torch.from_numpy(np.stack([wl.kv_rows(w, l, 1, nc, nc + T) for l in range(L)])).to(device)
    out = torch.empty((L, T, Hq, D), device=device)
    lse = torch.empty((L, T, Hq), device=device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    # the f16 key tiles expanded once per call (the timed region includes the expansion)
    # into a workspace of whole slabs (one slab per (layer, KV head) pair) within
    # --ws-mib; 0 = a slab for every pair
    full = kvq.kvq_prefill_workspace_bytes(L, w.n_kv_heads, D, nc + T)
    slab = kvq.kvq_prefill_workspace_bytes(1, 1, D, nc + T)
    ws_bytes = full if args.ws_mib == 0 else min(full, (args.ws_mib << 20) // slab * slab)
    if args.no_expand:
        ws_bytes = 0
    elif ws_bytes < slab:
        raise SystemExit(f"--ws-mib {args.ws_mib} holds no slab of {slab} bytes")
    n_pairs = L * w.n_kv_heads
    slabs = ws_bytes // slab if ws_bytes else 0
    if 2 <= slabs < n_pairs:  # chunks alternate between two halves: an odd slab is unused
        slabs -= slabs % 2
        ws_bytes = slabs * slab
    chunk = n_pairs if slabs >= n_pairs else max(1, slabs // 2)
    n_chunks = -(-n_pairs // chunk) if ws_bytes else 0
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=device) if ws_bytes else None

    def step(i=None):
        kvq.kvq_append(layers, k_new, v_new, nc, T, stream)
        if i is not None:
            ev[i][0].record(stream)
        kvq.kvq_prefill_attn(layers, q, Hq, T, nc, w.page, w.scale, out, lse, workspace=ws,
                             stream=stream)
        if i is not None:
            ev[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    kvq.kvq_check(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id(torch, device)) as clocks:
        barrier(device)
        torch.cuda.synchronize(device)
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
    kvq.kvq_check(stream)
    ms = reduce_max(t0.elapsed_time(t1) / args.steps, device)
    k_ms = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in ev), device)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    fl = prefill_flops(w)
    peak, kind = tensor_peak()
    tr = traffic_record(PREFILL_SOURCES, "prefill_traffic.json")
    cl = clocks.summary()
    res = None
    if rank == 0:
        res = {
            "metric": PREFILL_METRIC, "value": round(world * fl / (ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16 (K, V, P dequantized on chip), f32 accumulate",
            "data": "synthetic",
            "config": {"workload": w.name, "layers": L, "q_heads": Hq, "kv_heads": w.n_kv_heads,
                       "head_dim": D, "cached": nc, "new_tokens": T, "seed": w.seed,
                       "flop_per_step": fl, "workspace_bytes": ws_bytes,
                       "key_tiles": (f"expanded once per call into {slabs} workspace slabs, "
                                     f"{n_chunks} chunk(s) of {chunk} (layer, KV head) pairs"
                                     if ws_bytes else "dequantized in each CTA")},
            "query_tok_per_s": round(world * T / (ms * 1e-3), 1),
            "layer_query_tok_per_s": round(world * L * T / (ms * 1e-3), 1),
            "roofline": {"bound": "tensor",
                         "kernel": (f"kvq_prefill_attn ({L} layers): tile expansion + prefill, "
                                    f"{2 * n_chunks} launches" if ws_bytes else
                                    f"kvq_prefill_attn ({L} layers, 1 launch)"),
                         "achieved": round(fl / (k_ms * 1e-3) / 1e12, 2), "peak": peak,
                         "peak_kind": kind, "unit": "TFLOP/s",
                         "frac": round(fl / (k_ms * 1e-3) / 1e12 / peak, 4),
                         "traffic": tr["dram_bytes_per_layer"] * L if tr else None,
                         "launch_ms": round(k_ms, 3)},
            "gpu_launches": (1 + (2 * n_chunks if ws_bytes else 1)) * args.steps,
            "clocks": {"sm_mhz": cl["sm_mhz"], "sm_max_mhz": cl["sm_max_mhz"],
                       "reasons": cl["reasons"], "samples": cl["samples"]},
        }
    del cache
    if world > 1:
        dist.destroy_process_group()
    return res


# --------------------------------------------------------------------------- oracle

def oracle_sample(w: wl.Workload, layers: list[int], n_keys: int, threads_note: bool = True):
    """Oracle decode of the given layers over their first n_keys keys (the
    per-chunk partials plus the merge).  Returns (seconds, kv bytes)."""
    import oracle
    caches = []
    for l in layers:
        kc, vc = oracle.empty_cache(w.n_kv_heads, w.head_dim, w.capacity)
        k = wl.kv_rows(w, l, 0, 0, n_keys)
        v = wl.kv_rows(w, l, 1, 0, n_keys)
        oracle.append(kc, vc, k, v, 0)
        caches.append((kc, vc))
    t = time.perf_counter()
    for (kc, vc), l in zip(caches, layers):
        p, pl = oracle.decode_attn(kc, vc, wl.q_rows(w, l), n_keys, w.chunk, w.scale)
        oracle.merge_lse(p, pl)
    dt = time.perf_counter() - t
    return dt, len(layers) * n_keys * KV_BYTES_PER_TOKEN_LAYER(w)


def cpu_baseline(w: wl.Workload, budget_s: float = 12.0) -> dict:
    """The oracle as it stands, on this host's cores, over whole layers of the
    workload until about budget_s of CPU time is spent."""
    import oracle
    tot_t, tot_b, done = 0.0, 0, []
    for l in range(w.n_layers):
        dt, b = oracle_sample(w, [l], w.n_kv)
        tot_t += dt
        tot_b += b
        done.append(l)
        if tot_t >= budget_s:
            break
    return {"value": round(tot_b / tot_t / 1e9, 3), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{len(done)} of {w.n_layers} layers, full {w.n_kv}-key context, "
                      f"T={w.T}, {w.n_q_heads} q heads: fp64 decode partials + merge",
            "seconds": round(tot_t, 2)}


def run_reference(args, w: wl.Workload) -> dict | None:
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    # per step: one layer's first 16 chunks (65,536 keys), layers in turn
    n_keys = min(w.n_kv, 16 * w.chunk)
    for i in range(args.warmup):
        oracle_sample(w, [i % w.n_layers], n_keys)
    tot_t, tot_b = 0.0, 0
    for i in range(args.steps):
        dt, b = oracle_sample(w, [i % w.n_layers], n_keys)
        tot_t += dt
        tot_b += b
    gbs = tot_b / tot_t / 1e9
    ms = 1e3 * tot_t / args.steps
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 3), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "layers": w.n_layers, "q_heads": w.n_q_heads,
                   "kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "context": w.n_kv,
                   "query_tokens": w.T, "chunk": w.chunk, "seed": w.seed},
        "cpu_baseline": {"value": round(gbs, 3), "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"per step one layer's first {n_keys} keys (all heads, "
                                   f"T={w.T}): fp64 decode partials + merge"},
        "e2e": {"value": round(gbs, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="verify262k",
                    choices=["verify262k", "decode65k", "tiny", "prefill262k", "stream262k"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", choices=["replicas", "context"], default="replicas",
                    help="decode configs with N > 1: one replica per GPU (default), or one "
                         "context split over the GPUs (each decodes its shard of the keys; the "
                         "merged rows are all-gathered over NCCL and merged)")
    ap.add_argument("--kv-formats", choices=sorted(KV_FORMATS), default="q8_0/q4_0",
                    help="decode configs: block formats of K and V (the other pairs run the "
                         "general decode kernel)")
    ap.add_argument("--ws-mib", type=int, default=2048,
                    help="prefill262k: workspace for the expanded key tiles, MiB (whole slabs "
                         "of one (layer, KV head) each; 0 = one slab per pair, 26 GB)")
    ap.add_argument("--no-expand", action="store_true",
                    help="prefill262k: no workspace; every CTA dequantizes its key tiles")
    ap.add_argument("--budget-mib", type=int, default=None,
                    help="stream262k: device memory for the cache; the layers that fit next to "
                         "the two streaming slots stay resident (default: all streamed)")
    ap.add_argument("--layers", type=int, default=None,
                    help="profile a smaller case of the same kernel: only this many layers")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = wl.WORKLOADS[args.config]
    if args.layers is not None:
        w = wl.small(w, n_layers=args.layers)
    rank, world, _ = dist_env()
    if args.impl == "reference":
        res = run_reference(args, w)
    elif w.mode == "prefill":
        res = run_prefill(args, w)
    elif w.mode == "stream":
        res = run_stream(args, w)
    else:
        res = run_ours(args, w)
        if res is not None and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(w)
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
