"""Benchmark of one POEM prefill attention layer (score -> select -> block-sparse
attention) on B200.

Default workload: the Llama-3.1-8B-shaped layer at 128K tokens (32 query heads,
8 KV heads, head dim 128, 128x128 blocks, RoPE base 500000, heavy-block
synthetic Q/K/V from seed 0, tau = 0.05).  One step = poem_score + poem_select
+ bsa_fwd over that layer with the inputs resident in HBM (inputs are larger
than L2, so no flush is needed between steps).  Prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--selector exact|practical [--w W --gamma G --rho R]]

--selector practical times the practical selector instead (poem_score_pooled +
poem_select_practical + bsa_fwd; pooled estimates, mass shortlist rho, rerank
log m~ + w log d~, pooled-mass threshold gamma).

With N > 1 (torchrun, one rank per GPU) every rank runs an independent replica
of the layer (the path needs no exchange step); the reported ms/layer is the
whole job's: max-over-ranks time / (N * K).

--impl reference times the fp64 CPU oracle (test infrastructure; the reference
arm of this benchmark) on a bounded sample of the same layer's (head, tile)
units on the host cores -- tile pairs (i, T-1-i), the last tile included, run in
parallel over the host threads -- and extrapolates to ms/layer by visible blocks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import poem_synth  # noqa: E402

METRIC = "128K-token prefill attention ms/layer; retained-block TFLOP/s vs BF16 tensor peak"

WORKLOADS = {
    # name: (n_tokens, Hq, Hkv, d, block, rope_base, tau)
    "llama3.1-8b-layer-128k": (131072, 32, 8, 128, 128, 500000.0, 0.05),
    "llama3.1-8b-layer-32k": (32768, 32, 8, 128, 128, 500000.0, 0.05),
    "llama3.1-8b-layer-64k": (65536, 32, 8, 128, 128, 500000.0, 0.05),
    "qwen3-14b-layer-64k": (65536, 40, 8, 128, 128, 1000000.0, 0.05),
}
# Roofline denominators measured on B200 (a STREAM-style copy and a bf16 GEMM;
# MEASURED_PEAKS.json, when present, takes precedence).
FALLBACK_PEAKS = {"bf16_tflops": 1667.9, "bf16_tflops_sustained": 1378.8, "hbm_gbs": 6452.5}
# DRAM bytes per bsa_fwd launch on the 128K layer: the ncu capture of the 64K layer
# (dram__bytes_read.sum + dram__bytes_write.sum = 842.4 + 502.8 = 1345.2 MB per launch)
# scaled by rows processed (x2); the 32K capture (642.4 MB, x2.09 to 64K) confirms the
# scaling.  Valid only for the kernel source it was taken on.
BSA_FWD_TRAFFIC = {"bytes": 2.690e9, "source_sha256_prefix": "090feeb3d9772452",
                   "note": "ncu dram bytes of the 64K layer launch x2 rows (32K capture x4: 2.57 GB)"}


def bsa_fwd_traffic():
    import hashlib

    path = os.path.join(ROOT, "block_sparse_attention_poem_b200", "csrc", "bsa_fwd.cu")
    with open(path, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    if digest != BSA_FWD_TRAFFIC["source_sha256_prefix"]:
        return None, "kernel changed since the ncu capture"
    return BSA_FWD_TRAFFIC["bytes"], BSA_FWD_TRAFFIC["note"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "measured on B200 (values copied into the benchmark)"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," \
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)), "reasons": sorted(reasons),
                "samples": len(sm)}


def retained_flops(row_ptr: np.ndarray, col_idx: np.ndarray, n_tiles: int, d: int, B: int, q_tile0: int = 0) -> float:
    """4 d (kept query-key pairs): full blocks B^2 pairs, the diagonal block B(B+1)/2.
    Row r is query tile r % n_tiles, global tile q_tile0 + r % n_tiles."""
    rows = len(row_ptr) - 1
    counts = np.diff(row_ptr).astype(np.int64)
    tiles = np.arange(rows) % n_tiles + q_tile0
    # diagonal present? (lists are ascending: last entry == tile)
    last = np.where(counts > 0, col_idx[np.maximum(row_ptr[1:] - 1, 0)], -1)
    diag = (last == tiles).astype(np.int64)
    pairs = (counts - diag) * B * B + diag * (B * (B + 1) // 2)
    return float(4 * d * pairs.sum())


def dense_flops(n: int, hq: int, d: int) -> float:
    return float(2 * d * hq * n * (n + 1))


def reduce_max(value: float) -> float:
    """Max of a per-rank value over the process group (identity without one).
    Works with any backend: the tensor lives on the GPU for NCCL, on the CPU else."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_ms_per_layer(max_rank_ms: float, steps: int, world: int, sharded: bool = False) -> float:
    """Replicas: every rank runs `steps` whole layers, so the job's ms per layer is the
    slowest rank's time over all steps * world layers.  Head-sharded: the ranks
    together run one layer per step, so it is the slowest rank's time per step."""
    return max_rank_ms / (steps if sharded else steps * world)


def shard_heads(n_q_heads: int, n_kv_heads: int, world: int, rank: int):
    """Head sharding of one layer (as in tensor-parallel attention): rank r owns KV
    heads [r Hkv/N, (r+1) Hkv/N) and the query heads that read them.  Every
    (head, tile) unit is independent, so no collective is needed.  Returns
    ((q_head_lo, q_head_hi), (kv_head_lo, kv_head_hi))."""
    if n_kv_heads % world:
        raise ValueError(f"{n_kv_heads} KV heads do not split over {world} ranks")
    per = n_kv_heads // world
    group = n_q_heads // n_kv_heads
    return (rank * per * group, (rank + 1) * per * group), (rank * per, (rank + 1) * per)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def run_ours(args):
    import block_sparse_attention_poem_b200 as poem

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    n, hq, hkv, d, B, base, tau = WORKLOADS[args.workload]
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, rope_base=base, seed=args.seed)
    sharded = args.shard == "heads" and world > 1
    hq_all, hkv_all = hq, hkv
    if sharded:  # this rank's heads only, as a tensor-parallel attention layer holds them
        (qa, qb), (ka, kb) = shard_heads(hq, hkv, world, rank)
        x = {"q": x["q"][:, qa:qb].contiguous(), "k": x["k"][:, ka:kb].contiguous(),
             "v": x["v"][:, ka:kb].contiguous()}
        hq, hkv = qb - qa, kb - ka
    q, k, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    practical = args.selector == "practical"
    layer = poem.alloc_layer(q, k, block=B, practical=practical)
    stream = torch.cuda.current_stream(dev)
    ws_first = layer.ws_pooled if practical else layer.ws_score

    def run_layer(qb, kb, vb, lay, ev=None, st=None):
        """One step -- score, select, bsa_fwd -- on the current stream (events on st)."""
        st = st or torch.cuda.current_stream(dev)
        if ev:
            ev[0].record(st)
        if practical:
            poem.poem_score_pooled(qb, kb, vb, lay.m_pool, lay.d_pool, lay.ws_pooled, shape=lay.shape)
        else:
            poem.poem_score(qb, kb, vb, lay.I_hat, lay.m_hat, lay.ws_score, shape=lay.shape)
        if ev:
            ev[1].record(st)
        if practical:
            poem.poem_select_practical(lay.shape, lay.m_pool, lay.d_pool, args.w, args.gamma, args.rho,
                                       lay.row_ptr, lay.col_idx, lay.ws_select, order=lay.order)
        else:
            poem.poem_select(lay.shape, lay.I_hat, lay.m_hat, tau, lay.row_ptr, lay.col_idx, lay.ws_select,
                             order=lay.order)
        if ev:
            ev[2].record(st)
        poem.bsa_fwd(qb, kb, vb, lay.row_ptr, lay.col_idx, lay.o, lay.ws_fwd, order=lay.order, shape=lay.shape)
        if ev:
            ev[3].record(st)

    def step(ev=None):
        run_layer(q, k, v, layer, ev, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for ws in (ws_first, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = t_start.elapsed_time(t_end)
    score_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    select_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    fwd_ms = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))
    total_ms = reduce_max(total_ms)
    ms_per_step = total_ms / args.steps
    ms_per_layer = whole_job_ms_per_layer(total_ms, args.steps, world, sharded)

    for ws in (ws_first, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)
    rp = layer.row_ptr.cpu().numpy()
    ci = layer.col_idx[: int(rp[-1])].cpu().numpy()
    kept = int(rp[-1])
    visible = hq * T * (T + 1) // 2
    if practical:  # exact masses (untimed) for the heavy-mass figure and the mass-only comparison
        poem.poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape)
        poem.poem_check(layer.ws_score)
    # realised heavy-mass fraction: visible (head, tile, block) with m_hat > 10 / (i + 1)
    mh = layer.m_hat.cpu().numpy()
    tile_of = np.tile(np.repeat(np.arange(T), np.arange(1, T + 1)), hq)
    heavy_frac = float(np.mean(mh > 10.0 / (tile_of + 1)))
    rflops = retained_flops(rp, ci, T, d, B)
    dflops = dense_flops(n, hq, d)
    peaks, peak_src = load_peaks()
    fwd_tflops = rflops / (fwd_ms * 1e-3) / 1e12
    if args.workload == "llama3.1-8b-layer-128k" and not practical:
        traffic, traffic_note = bsa_fwd_traffic()
    else:
        traffic, traffic_note = None, "no ncu capture of bsa_fwd on these lists"

    # end-to-end through the public API with host buffers: H2D of Q/K/V from pinned
    # memory, the three calls, D2H of O, every step.
    # End to end through the public API with host buffers: every step copies its Q/K/V
    # from pinned host memory to the device and its O back, inside the timed region.
    # Pipelined (how a caller runs consecutive layers): step s+1's upload (copy stream)
    # and step s-1's download (another copy stream) overlap step s's kernels, with
    # double-buffered device inputs and outputs.  The serial form (copy, compute, copy
    # on one stream) is reported beside it.
    e2e = None
    e2e_serial = None
    if not args.no_e2e:
        hq_h = x["q"].pin_memory()
        hk_h = x["k"].pin_memory()
        hv_h = x["v"].pin_memory()
        ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        h2d_bytes = int(hq_h.numel() * 2 + hk_h.numel() * 2 + hv_h.numel() * 2)
        d2h_bytes = int(ho.numel() * 2)
        bufs = [(q, k, v, layer), (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                                   poem.alloc_layer(q, k, block=B, practical=practical))]
        up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]

        def upload(b):
            with torch.cuda.stream(up_s):
                qb, kb, vb, _ = bufs[b]
                qb.copy_(hq_h, non_blocking=True)
                kb.copy_(hk_h, non_blocking=True)
                vb.copy_(hv_h, non_blocking=True)
                ev_up[b].record(up_s)

        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(up_s)
        upload(0)
        for st_i in range(args.e2e_steps):
            b = st_i % 2
            if st_i + 1 < args.e2e_steps:
                if st_i >= 1:
                    up_s.wait_event(ev_done[1 - b])  # step st_i-1 has read those inputs
                upload(1 - b)
            stream.wait_event(ev_up[b])
            if st_i >= 2:
                stream.wait_event(ev_down[b])  # step st_i-2's output has left that buffer
            run_layer(*bufs[b], st=stream)
            ev_done[b].record(stream)
            down_s.wait_event(ev_done[b])
            with torch.cuda.stream(down_s):
                ho.copy_(bufs[b][3].o, non_blocking=True)
                ev_down[b].record(down_s)
        e1.record(down_s)
        torch.cuda.synchronize()
        for ws in (bufs[1][3].ws_pooled if practical else bufs[1][3].ws_score, bufs[1][3].ws_select,
                   bufs[1][3].ws_fwd):
            poem.poem_check(ws)
        e2e_ms = reduce_max(e0.elapsed_time(e1))
        e2e = {"value": whole_job_ms_per_layer(e2e_ms, args.e2e_steps, world, sharded), "unit": "ms/layer",
               "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes, "steps": args.e2e_steps,
               "mode": "pipelined: next step's upload and previous step's download overlap this step's kernels"}
        del bufs
        torch.cuda.empty_cache()
        # serial form
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            q.copy_(hq_h, non_blocking=True)
            k.copy_(hk_h, non_blocking=True)
            v.copy_(hv_h, non_blocking=True)
            step()
            ho.copy_(layer.o, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = reduce_max(e0.elapsed_time(e1))
        e2e_serial = {"value": whole_job_ms_per_layer(e2e_ms, args.e2e_steps, world, sharded), "unit": "ms/layer",
                      "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                      "mode": "serial: copy in, compute, copy out on one stream"}

    # The practical selector on the same inputs (a nested record; the headline value
    # stays the exact selector's).
    prac, prac_o, prac_layer = None, None, None
    if not practical and not args.no_practical:
        prac, prac_o, prac_layer = practical_record(poem, q, k, v, args, n, hq, d, B, peaks, peak_src)
        prac["gpu_launches"] = 7 * args.steps

    extra = {}
    if not args.no_quality and rank == 0:
        extra = quality_report(poem, q, k, v, layer, tau, n, hq, T, B, dev,
                               extra_outputs={"practical": prac_o} if prac_o is not None else None)
        if practical:
            extra["err_vs_dense"]["practical"] = extra["err_vs_dense"].pop("poem")
        if prac is not None and "practical" in extra.get("err_vs_dense", {}):
            prac["err_vs_dense"] = extra["err_vs_dense"].pop("practical")
    del prac_o, prac_layer

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = (cpu_baseline_practical(x, n, hq, hkv, d, B, args.w, args.gamma, args.rho, args.cpu_budget_s)
               if practical else cpu_baseline(x, n, hq, hkv, d, B, tau, args.cpu_budget_s,
                                              gpu_rows=gpu_rows_fn(layer, T, B)))
    sel_cfg = ({"selector": "practical", "w": args.w, "gamma": args.gamma, "rho": args.rho} if practical
               else {"selector": "exact", "tau": tau})
    names = (("poem_score_pooled", "poem_select_practical") if practical else ("poem_score", "poem_select"))

    launches_per_step = 2 + 3 + 1 + 1  # score(2 passes | pool + pooled scores) + select(3 + order) + bsa_fwd
    line = {
        "metric": METRIC,
        "value": round(ms_per_layer, 4),
        "unit": "ms/layer",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": False,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded heavy-block generator; no model weights or datasets)",
        "config": {"workload": args.workload, "n_tokens": n, "n_q_heads": hq_all, "n_kv_heads": hkv_all,
                   "head_dim": d, "block": B, "n_sample": 16, **sel_cfg, "seed": args.seed,
                   "parallelism": (f"head-sharded x{world} ({hq} query / {hkv} KV heads per rank)" if sharded
                                   else f"replicas x{world}" if world > 1 else "single GPU"),
                   "l2": "inputs larger than L2 (no flush needed)"},
        "breakdown_ms": {names[0]: round(score_ms, 4), names[1]: round(select_ms, 4),
                         "bsa_fwd": round(fwd_ms, 4)},
        "density": round(kept / visible, 5),
        "heavy_mass_block_fraction": round(heavy_frac, 4),
        "dense_equiv_tflops": round(dflops / (ms_per_step * 1e-3) / 1e12, 2),
        "retained_tflops": round(rflops / (ms_per_step * 1e-3) / 1e12, 2),
        "score_select_over_fwd": round((score_ms + select_ms) / fwd_ms, 4),
        "roofline": {"bound": "tensor", "kernel": "bsa_fwd", "achieved": round(fwd_tflops, 2),
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": round(fwd_tflops / peaks["bf16_tflops_sustained"], 4),
                     "frac_of_burst_peak": round(fwd_tflops / peaks["bf16_tflops"], 4),
                     "peak_source": peak_src + ", sustained bf16 (kernel timed inside a long step)",
                     "algorithmic_flops_per_launch": rflops, "traffic": traffic,
                     "traffic_note": traffic_note},
        "clocks": clk,
        "e2e": e2e,
        "e2e_serial": e2e_serial,
        "gpu_launches": launches_per_step * args.steps,
        "cpu_baseline": cpu,
    }
    if cpu and "parity" in cpu:
        line["oracle_parity"] = cpu.pop("parity")
    if prac is not None:
        line["practical"] = prac
    line.update(extra)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def practical_record(poem, q, k, v, args, n, hq, d, B, peaks, peak_src):
    """The practical selector (pooled estimates, mass shortlist rho, rerank
    log m~ + w log d~, pooled-mass threshold gamma) timed on the same inputs with the
    same loop as the headline line: W warm-up steps, K steps with CUDA events around
    each call.  Returns (record, output, layer)."""
    T = n // B
    lay = poem.alloc_layer(q, k, block=B, practical=True)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        poem.poem_score_pooled(q, k, v, lay.m_pool, lay.d_pool, lay.ws_pooled, shape=lay.shape)
        if ev:
            ev[1].record(stream)
        poem.poem_select_practical(lay.shape, lay.m_pool, lay.d_pool, args.w, args.gamma, args.rho, lay.row_ptr,
                                   lay.col_idx, lay.ws_select, order=lay.order)
        if ev:
            ev[2].record(stream)
        poem.bsa_fwd(q, k, v, lay.row_ptr, lay.col_idx, lay.o, lay.ws_fwd, order=lay.order, shape=lay.shape)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s_ in range(args.steps):
        step(evs[s_])
    t1.record(stream)
    torch.cuda.synchronize()
    for ws in (lay.ws_pooled, lay.ws_select, lay.ws_fwd):
        poem.poem_check(ws)
    ms = t0.elapsed_time(t1) / args.steps
    pool_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    sel_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    fwd_ms = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))
    rp = lay.row_ptr.cpu().numpy()
    ci = lay.col_idx[: int(rp[-1])].cpu().numpy()
    rflops = retained_flops(rp, ci, T, d, B)
    tf = rflops / (fwd_ms * 1e-3) / 1e12
    rec = {"selector": "practical", "w": args.w, "gamma": args.gamma, "rho": args.rho,
           "ms_per_layer": round(ms, 4), "steps": args.steps, "warmup": args.warmup,
           "breakdown_ms": {"poem_score_pooled": round(pool_ms, 4), "poem_select_practical": round(sel_ms, 4),
                            "bsa_fwd": round(fwd_ms, 4)},
           "density": round(int(rp[-1]) / (hq * T * (T + 1) // 2), 5),
           "score_select_over_fwd": round((pool_ms + sel_ms) / fwd_ms, 4),
           "roofline": {"bound": "tensor", "kernel": "bsa_fwd", "achieved": round(tf, 2),
                        "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                        "frac": round(tf / peaks["bf16_tflops_sustained"], 4),
                        "frac_of_burst_peak": round(tf / peaks["bf16_tflops"], 4),
                        "peak_source": peak_src + ", sustained bf16 (kernel timed inside a long step)",
                        "algorithmic_flops_per_launch": rflops, "traffic": None,
                        "traffic_note": "no ncu capture of bsa_fwd on these lists"}}
    return rec, lay.o, lay


def quality_report(poem, q, k, v, layer, tau, n, hq, T, B, dev, extra_outputs=None):
    """Output error of the POEM lists and of mass-only lists at the same budget,
    both against dense attention (bsa_fwd over every causal block); extra_outputs
    (name -> O) are compared with the same dense output."""
    rp_all, ci_all = poem_synth.random_block_lists(1, T, 1.0, seed=0)
    counts = np.diff(rp_all)
    rp_dense = np.concatenate([[0], np.cumsum(np.tile(counts, hq))]).astype(np.int32)
    ci_dense = np.tile(ci_all, hq).astype(np.int32)
    rpd = torch.from_numpy(rp_dense).to(dev)
    cid = torch.from_numpy(ci_dense).to(dev)
    o_dense = torch.empty_like(q)
    poem.bsa_fwd(q, k, v, rpd, cid, o_dense, layer.ws_fwd, shape=layer.shape)
    # mass-only at matched per-row budget
    rp_m = torch.empty_like(layer.row_ptr)
    ci_m = torch.empty_like(layer.col_idx)
    poem.poem_select_mass_only(layer.shape, layer.m_hat, layer.row_ptr, rp_m, ci_m, layer.ws_select)
    o_mass = torch.empty_like(q)
    poem.bsa_fwd(q, k, v, rp_m, ci_m, o_mass, layer.ws_fwd, shape=layer.shape)
    torch.cuda.synchronize()
    poem.poem_check(layer.ws_fwd)
    poem.poem_check(layer.ws_select)

    def err(o):
        diff = (o.float() - o_dense.float())
        return {"max_abs": float(diff.abs().max()), "mean_abs": float(diff.abs().mean()),
                "rel_fro": float(diff.norm() / o_dense.float().norm()),
                "max_row_l2": float(diff.norm(dim=-1).max())}

    out = {"poem": err(layer.o), "mass_only_same_budget": err(o_mass)}
    for name, o in (extra_outputs or {}).items():
        out[name] = err(o)
    return {"err_vs_dense": out}


def gpu_rows_fn(layer, T, B):
    """Host copies of one (head, tile) row of a whole-prefill layer: Î and m̂ of the
    row, its block list and its output rows."""
    def rows(h, i):
        off = h * T * (T + 1) // 2 + i * (i + 1) // 2
        r = h * T + i
        a, b = (int(t) for t in layer.row_ptr[r:r + 2].cpu())
        return (layer.I_hat[off:off + i + 1].cpu().numpy().astype(np.float64),
                layer.m_hat[off:off + i + 1].cpu().numpy().astype(np.float64),
                layer.col_idx[a:b].cpu().numpy(),
                layer.o[i * B:(i + 1) * B, h].float().cpu().numpy())
    return rows


def oracle_sample_units(hq, T, n_pairs, salt=0):
    """(head, tile) units for the oracle baseline: n_pairs pairs of tiles (i, T-1-i)
    with i spread over [0, T/2) from i = 0, so that every pair holds T + 1 visible
    blocks (the pairs balance across the host threads) and the sample holds the last
    tile T-1."""
    units = []
    for p_ in range(n_pairs):
        i = min(T // 2, int(p_ * (T / 2) / n_pairs)) if T > 1 else 0
        h = (p_ * 7 + salt) % hq
        units.append((h, T - 1 - i))
        if T - 1 - i != i or T == 1:
            units.append(((h + 1) % hq, i))
    return sorted(set(units), key=lambda u: -u[1])  # largest first (dynamic schedule)


def cpu_baseline(x, n, hq, hkv, d, B, tau, budget_s, gpu_rows=None, n_pairs=None, salt=0):
    """Oracle (fp64, host cores) on a sample of (head, tile) units -- scores, selection
    and masked attention over the kept blocks -- run as one batch over all host
    threads (units in parallel), scaled to the whole layer by visible blocks (score
    ~ i+1 blocks, masked attention ~ kept blocks; selection is negligible).  With
    `gpu_rows` the same units also cross-check the CUDA path (outside the timed work):
    the worst Î or m̂ error as a fraction of its tolerance (Î: 1e-3 relative + 1e-5
    m_b R; m̂: 1e-3 relative + 1e-9), how many lists equal the oracle's, and the
    largest output error against the oracle's attention over the GPU's list."""
    import oracle

    oracle.build()
    T = n // B
    prob = oracle.Problem(q=poem_synth.bf16_bits(x["q"]), k=poem_synth.bf16_bits(x["k"]),
                          v=poem_synth.bf16_bits(x["v"]), block=B, n_sample=16)
    cores = oracle.num_threads()
    units = oracle_sample_units(hq, T, n_pairs or max(2, cores), salt)
    R = float(x["v"].float().norm(dim=-1).max())

    t0 = time.perf_counter()
    Ih, mh = prob.score_units(units)
    rows = [(h, i) for h, i in units]
    ref_rp, ref_ci, _ = oracle.select_all(hq, T, Ih, mh, tau, rows=rows)
    # the kept lists as a layer-wide CSR (rows not sampled are empty)
    counts = np.zeros(hq * T, dtype=np.int32)
    lists = {}
    for u, (h, i) in enumerate(units):
        lists[h * T + i] = ref_ci[ref_rp[u]:ref_rp[u + 1]]
        counts[h * T + i] = len(lists[h * T + i])
    rp = np.zeros(hq * T + 1, dtype=np.int32)
    rp[1:] = np.cumsum(counts)
    ci = np.concatenate([lists[r] for r in sorted(lists)]).astype(np.int32)
    prob.masked_units(units, rp, ci)
    t_total = time.perf_counter() - t0

    sampled_blocks = sum(i + 1 for _, i in units)
    total_blocks = hq * T * (T + 1) / 2
    est_ms = t_total * total_blocks / sampled_blocks * 1e3
    out = {"value": round(est_ms, 1), "unit": "ms/layer", "cores": min(cores, len(units)), "kind": "oracle",
           "sample": f"{len(units)} (head, tile) units, tile pairs (i, T-1-i) spread over the causal range "
                     f"(tiles {min(u[1] for u in units)}..{max(u[1] for u in units)} of {T}), score + select + "
                     f"masked attention in one batch over the host threads, {t_total:.1f} s, scaled by visible "
                     f"blocks to the whole layer",
           "extrapolated": True}
    if gpu_rows is not None:
        par = {"units": 0, "score_tol_ratio_max": 0.0, "lists_equal": 0, "o_max_abs": 0.0}
        g_counts = np.zeros(hq * T, dtype=np.int32)
        g_lists = {}
        for h, i in units:
            gI, gm, glist, go = gpu_rows(h, i)
            off = oracle.tri_offset(T, h, i)
            rI, rm = Ih[off:off + i + 1], mh[off:off + i + 1]
            tol_I = 1e-3 * rI + 1e-5 * rm * R + 1e-30
            tol_m = 1e-3 * rm + 1e-9
            par["units"] += 1
            par["score_tol_ratio_max"] = max(par["score_tol_ratio_max"], float(np.max(np.abs(gI - rI) / tol_I)),
                                             float(np.max(np.abs(gm - rm) / tol_m)))
            par["lists_equal"] += int(np.array_equal(glist, lists[h * T + i]))
            g_lists[h * T + i] = (np.asarray(glist, dtype=np.int32), go)
            g_counts[h * T + i] = len(glist)
        g_rp = np.zeros(hq * T + 1, dtype=np.int32)
        g_rp[1:] = np.cumsum(g_counts)
        g_ci = np.concatenate([g_lists[r][0] for r in sorted(g_lists)]).astype(np.int32)
        Og, _ = prob.masked_units(units, g_rp, g_ci)
        for u, (h, i) in enumerate(units):
            go = g_lists[h * T + i][1]
            par["o_max_abs"] = max(par["o_max_abs"], float(np.max(np.abs(go - np.asarray(Og[u])[:B]))))
        out["parity"] = par
    return out


def cpu_baseline_practical(x, n, hq, hkv, d, B, w, gamma, rho, budget_s):
    """Oracle (fp64, host cores) of the practical path on a bounded sample of
    (head, tile) units -- pooled estimates, practical selection, masked attention
    -- scaled to a whole layer by visible blocks per unit."""
    import oracle

    oracle.build()
    T = n // B
    prob = oracle.Problem(q=poem_synth.bf16_bits(x["q"]), k=poem_synth.bf16_bits(x["k"]),
                          v=poem_synth.bf16_bits(x["v"]), block=B, n_sample=16)
    units, per_unit, t_total, h = [], [], 0.0, 0
    for f in (1 / 16, 1 / 8, 1 / 4, 1 / 2, 1.0):
        if t_total > budget_s:
            break
        i = max(0, int(T * f) - 1)
        t0 = time.perf_counter()
        mp, dp = prob.pooled_units([(h, i)])
        off = oracle.tri_offset(T, h, i)
        keep, _ = oracle.select_practical_row(i, mp[off:off + i + 1], dp[off:off + i + 1], w, gamma, rho)
        rp = np.zeros(hq * T + 1, dtype=np.int32)
        rp[h * T + i + 1:] = len(keep)
        prob.masked_units([(h, i)], rp, np.asarray(keep, dtype=np.int32))
        dt = time.perf_counter() - t0
        t_total += dt
        units.append((h, i))
        per_unit.append(dt / (i + 1))
        h = (h + 1) % hq
    est_ms = float(np.mean(per_unit)) * hq * T * (T + 1) / 2 * 1e3
    return {"value": round(est_ms, 1), "unit": "ms/layer", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(units)} (head, tile) units at tiles {[u[1] for u in units]} (pooled estimates + "
                      f"practical selection + masked attention), {t_total:.1f} s, scaled by visible blocks per "
                      f"unit to the whole layer", "extrapolated": True}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    n, hq, hkv, d, B, base, tau = WORKLOADS[args.workload]
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, rope_base=base, seed=args.seed)
    budget = max(2.0, args.ref_step_budget_s)
    vals = []
    cb = None
    practical = args.selector == "practical"
    for s in range(args.warmup + args.steps):
        cb = (cpu_baseline_practical(x, n, hq, hkv, d, B, args.w, args.gamma, args.rho, budget) if practical
              else cpu_baseline(x, n, hq, hkv, d, B, tau, budget, n_pairs=args.ref_pairs, salt=s))
        if s >= args.warmup:
            vals.append(cb["value"])
    v = float(np.mean(vals))
    line = {
        "metric": METRIC, "value": round(v, 1), "unit": "ms/layer", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(v, 1), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded heavy-block generator)",
        "config": {"workload": args.workload, "n_tokens": n, "n_q_heads": hq, "n_kv_heads": hkv, "head_dim": d,
                   "block": B, "n_sample": 16,
                   **({"selector": "practical", "w": args.w, "gamma": args.gamma, "rho": args.rho} if practical
                      else {"selector": "exact", "tau": tau}), "seed": args.seed},
        "impl": "reference",
        "cpu_baseline": {"value": round(v, 1), "unit": "ms/layer", "cores": cb["cores"], "kind": "oracle",
                         "sample": cb["sample"]},
        "e2e": {"value": round(v, 1), "unit": "ms/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# --report: one JSON record per configuration (measurement table)
# --------------------------------------------------------------------------

REPORT_LAYERS = [
    # (name, generator kwargs, taus, run mass-only comparison)
    ("single-head-1k-d64-b64", None, [0.05], False),
    ("llama3.1-8b-layer-32k", "llama3.1-8b-layer-32k", [0.02, 0.05, 0.1], False),
    ("llama3.1-8b-layer-128k", "llama3.1-8b-layer-128k", [0.05], True),
    ("qwen3-14b-layer-64k", "qwen3-14b-layer-64k", [0.05], False),
]
SWEEP_TOKENS = [8192, 16384, 32768, 65536, 131072]
SWEEP_DENSITY = [0.05, 0.1, 0.25, 0.5, 1.0]


def _events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def _report_layer(poem, name, wl, tau, steps, warmup, mass_only, cpu_budget_s):
    if wl is None:
        xs = poem_synth.single_head(1024, 64, seed=0)
        x = {k: t.to(torch.bfloat16) for k, t in xs.items()}
        n, hq, hkv, d, B = 1024, 1, 1, 64, 64
    else:
        n, hq, hkv, d, B, base, _ = WORKLOADS[wl]
        x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, rope_base=base, seed=0)
    T = n // B
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    layer = poem.alloc_layer(q, k, block=B)
    ph = {"poem_score": [], "poem_select": [], "bsa_fwd": []}
    for it in range(warmup + steps):
        ev = _events(4)
        ev[0].record()
        poem.poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape)
        ev[1].record()
        poem.poem_select(layer.shape, layer.I_hat, layer.m_hat, tau, layer.row_ptr, layer.col_idx, layer.ws_select,
                         order=layer.order)
        ev[2].record()
        poem.bsa_fwd(q, k, v, layer.row_ptr, layer.col_idx, layer.o, layer.ws_fwd, order=layer.order,
                     shape=layer.shape)
        ev[3].record()
        torch.cuda.synchronize()
        if it >= warmup:
            for j, key in enumerate(ph):
                ph[key].append(ev[j].elapsed_time(ev[j + 1]))
    for ws in (layer.ws_score, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)
    ms = {key: float(np.median(val)) for key, val in ph.items()}
    total = sum(ms.values())
    rp = layer.row_ptr.cpu().numpy()
    ci = layer.col_idx[: int(rp[-1])].cpu().numpy()
    kept = int(rp[-1])
    visible = hq * T * (T + 1) // 2
    rfl = retained_flops(rp, ci, T, d, B)
    peaks, _ = load_peaks()
    fwd_tf = rfl / (ms["bsa_fwd"] * 1e-3) / 1e12
    sel_bytes = 8.0 * visible + 4.0 * kept + 4.0 * (hq * T + 1)
    sel_gbs = sel_bytes / (ms["poem_select"] * 1e-3) / 1e9
    rec = {
        "config": name, "tau": tau, "n_tokens": n, "n_q_heads": hq, "n_kv_heads": hkv, "head_dim": d, "block": B,
        "ms": {key: round(val, 4) for key, val in ms.items()}, "ms_per_layer": round(total, 4),
        "density": round(kept / visible, 5),
        "dense_equiv_tflops": round(dense_flops(n, hq, d) / (total * 1e-3) / 1e12, 2),
        "bsa_fwd_retained_tflops": round(fwd_tf, 2),
        "bsa_fwd_frac_burst": round(fwd_tf / peaks["bf16_tflops"], 4),
        "bsa_fwd_frac_sustained": round(fwd_tf / peaks["bf16_tflops_sustained"], 4),
        "select_gbs": round(sel_gbs, 1), "select_frac_hbm": round(sel_gbs / peaks["hbm_gbs"], 4),
        "score_select_over_fwd": round((ms["poem_score"] + ms["poem_select"]) / ms["bsa_fwd"], 4),
    }
    q_, k_, v_ = q, k, v
    rec["err_vs_dense"] = quality_report(poem, q_, k_, v_, layer, tau, n, hq, T, B, q.device)["err_vs_dense"]
    if not mass_only:
        rec["err_vs_dense"].pop("mass_only_same_budget", None)
    if cpu_budget_s > 0:
        cb = cpu_baseline(x, n, hq, hkv, d, B, tau, cpu_budget_s, gpu_rows=gpu_rows_fn(layer, T, B))
        rec["oracle_parity"] = cb.pop("parity")
        rec["oracle_ms_per_layer"] = cb["value"]
        rec["oracle_cores"] = cb["cores"]
        rec["oracle_note"] = cb["sample"]
    del layer, q, k, v
    torch.cuda.empty_cache()
    return rec


def _report_sweep(poem, steps, warmup):
    out = []
    peaks, _ = load_peaks()
    hq, hkv, d, B = 32, 8, 128, 128
    for n in SWEEP_TOKENS:
        x = poem_synth.iid_layer(n, hq, hkv, d, seed=0)
        q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
        T = n // B
        o = torch.empty_like(q)
        ws = poem.alloc_workspace(256)
        # up to 16K tokens the working set is close to L2's size: write 256 MiB between launches
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if n <= 16384 else None
        for dens in SWEEP_DENSITY:
            rp, ci = poem_synth.random_block_lists(hq, T, dens, seed=0)
            rpd, cid = torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()
            times = []
            for it in range(warmup + steps):
                if flush is not None:
                    flush.zero_()  # evict this layer's inputs from L2 before the timed launch
                ev = _events(2)
                ev[0].record()
                poem.bsa_fwd(q, k, v, rpd, cid, o, ws, block=B)
                ev[1].record()
                torch.cuda.synchronize()
                if it >= warmup:
                    times.append(ev[0].elapsed_time(ev[1]))
            poem.poem_check(ws)
            t = float(np.median(times))
            rfl = retained_flops(rp, ci, T, d, B)
            tf = rfl / (t * 1e-3) / 1e12
            out.append({"config": "bsa_fwd-sweep", "n_tokens": n, "density_target": dens,
                        "density": round(int(rp[-1]) / (hq * T * (T + 1) / 2), 5), "ms": round(t, 4),
                        "ms_min": round(float(np.min(times)), 4),
                        "l2": "256 MiB written between launches" if flush is not None else "inputs larger than L2",
                        "retained_tflops": round(tf, 2), "frac_burst": round(tf / peaks["bf16_tflops"], 4),
                        "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                        "dense_equiv_tflops": round(dense_flops(n, hq, d) / (t * 1e-3) / 1e12, 2)})
        del q, k, v, o, flush
        torch.cuda.empty_cache()
    return out


PRACTICAL_REPORT = [
    # (workload, [(w, gamma, rho), ...])
    ("llama3.1-8b-layer-32k", [(1.0, 0.9, 0.5), (1.0, 0.95, 0.5), (1.0, 0.99, 0.5), (0.0, 0.95, 0.5)]),
    ("llama3.1-8b-layer-128k", [(1.0, 0.9, 0.5), (1.0, 0.95, 0.5), (1.0, 0.99, 0.5), (0.0, 0.95, 0.5)]),
]


def _stage_diagnostics(m_pool, I_hat, row_ptr, col_idx, rho, hq, T, heads):
    """For the rows of `heads`: the candidates POEM's exact ranking keeps at the
    practical list's budget but the practical list drops, split into those the
    stage-1 mass shortlist excluded and those stage 2 ranked below the cut."""
    mp = m_pool.cpu().numpy()
    Ih = I_hat.cpu().numpy()
    rp = row_ptr.cpu().numpy()
    ci = col_idx[: int(rp[-1])].cpu().numpy()
    excl = misrank = kept_free = 0
    for h in heads:
        for i in range(3, T):
            r = h * T + i
            keep = set(ci[rp[r]:rp[r + 1]].tolist())
            off = h * (T * (T + 1) // 2) + i * (i + 1) // 2
            cand = np.arange(1, i - 1)
            free = len(keep) - 3
            kept_free += free
            if free <= 0:
                continue
            top_I = cand[np.lexsort((cand, -Ih[off + cand]))][:free]
            n1 = min(cand.size, int(math.ceil(rho * cand.size)))
            short = set(cand[np.lexsort((cand, -mp[off + cand]))][:n1].tolist())
            for b in top_I.tolist():
                if b not in keep:
                    if b in short:
                        misrank += 1
                    else:
                        excl += 1
    return {"rows": len(heads) * max(T - 3, 0), "free_blocks_kept": kept_free,
            "exact_topk_missed_stage1_excluded": excl, "exact_topk_missed_stage2_misranked": misrank}


def _report_practical(poem, wl, params, steps, warmup):
    n, hq, hkv, d, B, base, _ = WORKLOADS[wl]
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, rope_base=base, seed=0)
    T = n // B
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    layer = poem.alloc_layer(q, k, block=B, practical=True)
    poem.poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape)  # exact, for comparisons
    poem.poem_check(layer.ws_score)
    peaks, _ = load_peaks()
    visible = hq * T * (T + 1) // 2
    out = []
    for w, gamma, rho in params:
        ph = {"poem_score_pooled": [], "poem_select_practical": [], "bsa_fwd": []}
        for it in range(warmup + steps):
            ev = _events(4)
            ev[0].record()
            poem.poem_score_pooled(q, k, v, layer.m_pool, layer.d_pool, layer.ws_pooled, shape=layer.shape)
            ev[1].record()
            poem.poem_select_practical(layer.shape, layer.m_pool, layer.d_pool, w, gamma, rho, layer.row_ptr,
                                       layer.col_idx, layer.ws_select, order=layer.order)
            ev[2].record()
            poem.bsa_fwd(q, k, v, layer.row_ptr, layer.col_idx, layer.o, layer.ws_fwd, order=layer.order,
                         shape=layer.shape)
            ev[3].record()
            torch.cuda.synchronize()
            if it >= warmup:
                for j, key in enumerate(ph):
                    ph[key].append(ev[j].elapsed_time(ev[j + 1]))
        for ws in (layer.ws_pooled, layer.ws_select, layer.ws_fwd):
            poem.poem_check(ws)
        ms = {key: float(np.median(val)) for key, val in ph.items()}
        rp = layer.row_ptr.cpu().numpy()
        ci = layer.col_idx[: int(rp[-1])].cpu().numpy()
        rfl = retained_flops(rp, ci, T, d, B)
        fwd_tf = rfl / (ms["bsa_fwd"] * 1e-3) / 1e12
        # pooled scoring reads Q, K, V once (bf16) and writes m~, d~ (fp32)
        pooled_bytes = 2.0 * n * (hq + 2 * hkv) * d + 8.0 * visible
        rec = {"config": f"practical-{wl}", "w": w, "gamma": gamma, "rho": rho, "n_tokens": n,
               "ms": {key: round(val, 4) for key, val in ms.items()}, "ms_per_layer": round(sum(ms.values()), 4),
               "density": round(int(rp[-1]) / visible, 5),
               "bsa_fwd_retained_tflops": round(fwd_tf, 2),
               "bsa_fwd_frac_sustained": round(fwd_tf / peaks["bf16_tflops_sustained"], 4),
               "pooled_gbs": round(pooled_bytes / (ms["poem_score_pooled"] * 1e-3) / 1e9, 1)}
        q_err = quality_report(poem, q, k, v, layer, 0.0, n, hq, T, B, q.device)["err_vs_dense"]
        rec["err_vs_dense"] = {"practical": q_err["poem"], "mass_only_same_budget": q_err["mass_only_same_budget"]}
        # exact-score ranking at the same per-row budget
        rp_i = torch.empty_like(layer.row_ptr)
        ci_i = torch.empty_like(layer.col_idx)
        poem.poem_select_ranked_budget(layer.shape, layer.I_hat, layer.row_ptr, rp_i, ci_i, layer.ws_select)
        o_i = torch.empty_like(q)
        poem.bsa_fwd(q, k, v, rp_i, ci_i, o_i, layer.ws_fwd, shape=layer.shape)
        torch.cuda.synchronize()
        poem.poem_check(layer.ws_select)
        o_dense = _dense_output(poem, q, k, v, layer, hq, T)
        diff = o_i.float() - o_dense.float()
        rec["err_vs_dense"]["exact_I_same_budget"] = {
            "max_abs": float(diff.abs().max()), "mean_abs": float(diff.abs().mean()),
            "rel_fro": float(diff.norm() / o_dense.float().norm()), "max_row_l2": float(diff.norm(dim=-1).max())}
        del o_i, o_dense, diff
        rec["stage_diagnostics"] = _stage_diagnostics(layer.m_pool, layer.I_hat, layer.row_ptr, layer.col_idx, rho,
                                                      hq, T, heads=[0, hq // 2])
        out.append(rec)
    del layer, q, k, v
    torch.cuda.empty_cache()
    return out


def _dense_output(poem, q, k, v, layer, hq, T):
    rp_all, ci_all = poem_synth.random_block_lists(1, T, 1.0, seed=0)
    counts = np.diff(rp_all)
    rpd = torch.from_numpy(np.concatenate([[0], np.cumsum(np.tile(counts, hq))]).astype(np.int32)).to(q.device)
    cid = torch.from_numpy(np.tile(ci_all, hq).astype(np.int32)).to(q.device)
    o = torch.empty_like(q)
    poem.bsa_fwd(q, k, v, rpd, cid, o, layer.ws_fwd, shape=layer.shape)
    torch.cuda.synchronize()
    poem.poem_check(layer.ws_fwd)
    return o


CHUNK_REPORT = [
    # (context tokens, query-chunk tokens): the last chunk of a long prefill
    (131072, 16384),
    (131072, 32768),
    (65536, 16384),
]


def _report_chunked(poem, steps, warmup):
    """The last query chunk of a long prefill (queries are the final Nq of N
    tokens): exact POEM (tau = 0.05) and the practical selector (w = 1,
    gamma = 0.95, rho = 0.5) on the Llama-shaped heavy-block layer."""
    out = []
    peaks, _ = load_peaks()
    hq, hkv, d, B = 32, 8, 128, 128
    for n, nq in CHUNK_REPORT:
        x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, rope_base=500000.0, seed=0)
        q = x["q"][n - nq:].cuda()
        k, v = x["k"].cuda(), x["v"].cuda()
        T, t0 = n // B, (n - nq) // B
        Tq = T - t0
        visible = hq * (Tq * t0 + Tq * (Tq + 1) // 2)
        for selector in ("exact", "practical"):
            layer = poem.alloc_layer(q, k, block=B, practical=(selector == "practical"))
            ph = {"score": [], "select": [], "bsa_fwd": []}
            for it in range(warmup + steps):
                ev = _events(4)
                ev[0].record()
                if selector == "exact":
                    poem.poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape)
                else:
                    poem.poem_score_pooled(q, k, v, layer.m_pool, layer.d_pool, layer.ws_pooled, shape=layer.shape)
                ev[1].record()
                if selector == "exact":
                    poem.poem_select(layer.shape, layer.I_hat, layer.m_hat, 0.05, layer.row_ptr, layer.col_idx,
                                     layer.ws_select, order=layer.order)
                else:
                    poem.poem_select_practical(layer.shape, layer.m_pool, layer.d_pool, 1.0, 0.95, 0.5,
                                               layer.row_ptr, layer.col_idx, layer.ws_select, order=layer.order)
                ev[2].record()
                poem.bsa_fwd(q, k, v, layer.row_ptr, layer.col_idx, layer.o, layer.ws_fwd, order=layer.order,
                             shape=layer.shape)
                ev[3].record()
                torch.cuda.synchronize()
                if it >= warmup:
                    for j, key in enumerate(ph):
                        ph[key].append(ev[j].elapsed_time(ev[j + 1]))
            for ws in (layer.ws_pooled if selector == "practical" else layer.ws_score, layer.ws_select, layer.ws_fwd):
                poem.poem_check(ws)
            ms = {key: float(np.median(val)) for key, val in ph.items()}
            rp = layer.row_ptr.cpu().numpy()
            ci = layer.col_idx[: int(rp[-1])].cpu().numpy()
            rfl = retained_flops(rp, ci, Tq, d, B, q_tile0=t0)
            fwd_tf = rfl / (ms["bsa_fwd"] * 1e-3) / 1e12
            dense_fl = 2.0 * d * hq * nq * (2 * (n - nq) + nq + 1)
            out.append({"config": "chunked-prefill", "context_tokens": n, "query_tokens": nq, "q_offset": n - nq,
                        "selector": selector, "ms": {key: round(val, 4) for key, val in ms.items()},
                        "ms_per_chunk": round(sum(ms.values()), 4), "density": round(int(rp[-1]) / visible, 5),
                        "bsa_fwd_retained_tflops": round(fwd_tf, 2),
                        "bsa_fwd_frac_sustained": round(fwd_tf / peaks["bf16_tflops_sustained"], 4),
                        "dense_equiv_tflops": round(dense_fl / (sum(ms.values()) * 1e-3) / 1e12, 2)})
            del layer
            torch.cuda.empty_cache()
        del q, k, v
        torch.cuda.empty_cache()
    return out


def _report_dense_context(poem, steps, warmup, sizes=(32768, 131072)):
    """Context only (not the product path): dense causal GQA attention from the
    framework's own library kernel (torch scaled_dot_product_attention on the
    device) next to bsa_fwd with every causal block listed, on i.i.d. inputs."""
    import torch.nn.functional as F

    out = []
    hq, hkv, d, B = 32, 8, 128, 128
    for n in sizes:
        x = poem_synth.iid_layer(n, hq, hkv, d, seed=0)
        q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
        qt, kt, vt = q.permute(1, 0, 2).unsqueeze(0), k.permute(1, 0, 2).unsqueeze(0), v.permute(1, 0, 2).unsqueeze(0)
        qt, kt, vt = qt.contiguous(), kt.contiguous(), vt.contiguous()
        times = []
        for it in range(warmup + steps):
            ev = _events(2)
            ev[0].record()
            o_ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, enable_gqa=True)
            ev[1].record()
            torch.cuda.synchronize()
            if it >= warmup:
                times.append(ev[0].elapsed_time(ev[1]))
        t_sdpa = float(np.median(times))
        T = n // B
        layer = poem.alloc_layer(q, k, block=B)
        o_all = _dense_output(poem, q, k, v, layer, hq, T)
        rp_all, ci_all = poem_synth.random_block_lists(1, T, 1.0, seed=0)
        counts = np.diff(rp_all)
        rpd = torch.from_numpy(np.concatenate([[0], np.cumsum(np.tile(counts, hq))]).astype(np.int32)).cuda()
        cid = torch.from_numpy(np.tile(ci_all, hq).astype(np.int32)).cuda()
        times = []
        for it in range(warmup + steps):
            ev = _events(2)
            ev[0].record()
            poem.bsa_fwd(q, k, v, rpd, cid, layer.o, layer.ws_fwd, shape=layer.shape)
            ev[1].record()
            torch.cuda.synchronize()
            if it >= warmup:
                times.append(ev[0].elapsed_time(ev[1]))
        poem.poem_check(layer.ws_fwd)
        t_all = float(np.median(times))
        diff = (o_all.float() - o_ref[0].permute(1, 0, 2).float()).abs()
        dfl = dense_flops(n, hq, d)
        out.append({"config": "dense-context", "n_tokens": n, "sdpa_ms": round(t_sdpa, 4),
                    "sdpa_tflops": round(dfl / (t_sdpa * 1e-3) / 1e12, 1), "bsa_fwd_all_blocks_ms": round(t_all, 4),
                    "bsa_fwd_all_blocks_tflops": round(dfl / (t_all * 1e-3) / 1e12, 1),
                    "max_abs_diff_vs_sdpa": float(diff.max())})
        del q, k, v, qt, kt, vt, o_ref, o_all, layer
        torch.cuda.empty_cache()
    return out


EVAL_LAYERS = [
    ("heavy-block-32k", "heavy"),
    ("contrast-32k", "contrast"),
]


def _report_grouped(poem, steps, warmup, n_tokens=131072):
    """bsa_fwd against bsa_fwd_grouped (two query heads of a KV group sharing K/V tiles
    over the union of their lists) on the 128K Llama-shaped layer's exact (tau = 0.05)
    and practical (gamma = 0.95) lists; the outputs must be bit-identical."""
    _, hq, hkv, d, B, base, _ = WORKLOADS["llama3.1-8b-layer-128k"]
    n = n_tokens
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, rope_base=base, seed=0)
    T = n // B
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    layer = poem.alloc_layer(q, k, block=B, practical=True)
    o2 = torch.empty_like(layer.o)
    ws2 = poem.alloc_workspace(256)
    out = []
    for sel in ("exact", "practical"):
        if sel == "exact":
            poem.prefill_layer(q, k, v, 0.05, layer=layer, block=B)
        else:
            poem.prefill_layer_practical(q, k, v, 1.0, 0.95, 0.5, layer=layer, block=B)
        torch.cuda.synchronize()
        rp = layer.row_ptr.cpu().numpy()
        rfl = retained_flops(rp, layer.col_idx[: int(rp[-1])].cpu().numpy(), T, d, B)
        times = {"bsa_fwd": [], "bsa_fwd_grouped": []}
        for it in range(warmup + steps):
            for key in times:  # interleaved, one launch each per iteration
                ev = _events(2)
                ev[0].record()
                if key == "bsa_fwd":
                    poem.bsa_fwd(q, k, v, layer.row_ptr, layer.col_idx, layer.o, layer.ws_fwd, order=layer.order,
                                 shape=layer.shape)
                else:
                    poem.bsa_fwd_grouped(q, k, v, layer.row_ptr, layer.col_idx, o2, ws2, shape=layer.shape)
                ev[1].record()
                torch.cuda.synchronize()
                if it >= warmup:
                    times[key].append(ev[0].elapsed_time(ev[1]))
        poem.poem_check(layer.ws_fwd)
        poem.poem_check(ws2)
        ms = {key: float(np.median(val)) for key, val in times.items()}
        out.append({"config": f"grouped-llama3.1-8b-layer-{n // 1024}k", "selector": sel,
                    "density": round(int(rp[-1]) / (hq * T * (T + 1) // 2), 5),
                    "ms": {key: round(val, 4) for key, val in ms.items()},
                    "retained_tflops": {key: round(rfl / (val * 1e-3) / 1e12, 1) for key, val in ms.items()},
                    "bit_identical": bool(torch.equal(o2.view(torch.int16), layer.o.view(torch.int16)))})
    return out


def _err_vs(o, o_dense):
    diff = o.float() - o_dense.float()
    return {"rel_fro": round(float(diff.norm() / o_dense.float().norm()), 5),
            "mean_abs": round(float(diff.abs().mean()), 6), "max_row_l2": round(float(diff.norm(dim=-1).max()), 4)}


def _report_evaluation(poem):
    """Selectors compared on output error against dense attention (the evaluation
    the reading note proposes): POEM's threshold rule with mass-only at the same
    block count; exact-I order vs exact-mass order at the same retained mass
    (keep blocks in that order until the max-aggregated mass reaches gamma); the
    practical selector.  Heavy-block layer and the mass/deviation contrast layer
    (cancelling heavy pairs, flat heavy blocks, deviant light blocks), 32K tokens."""
    n, hq, hkv, d, B, base, _ = WORKLOADS["llama3.1-8b-layer-32k"]
    T = n // B
    visible = hq * T * (T + 1) // 2
    out = []
    for name, kind in EVAL_LAYERS:
        gen = poem_synth.contrast_layer if kind == "contrast" else poem_synth.heavy_block_layer
        x = gen(n, hq, hkv, d, block=B, rope_base=base, seed=0)
        q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
        layer = poem.alloc_layer(q, k, block=B, practical=True)
        poem.poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape)
        poem.poem_check(layer.ws_score)
        o_dense = _dense_output(poem, q, k, v, layer, hq, T)
        rp2 = torch.empty_like(layer.row_ptr)
        ci2 = torch.empty_like(layer.col_idx)
        o2 = torch.empty_like(q)

        def run(rp, ci):
            poem.bsa_fwd(q, k, v, rp, ci, o2, layer.ws_fwd, shape=layer.shape)
            torch.cuda.synchronize()
            poem.poem_check(layer.ws_fwd)
            return {"density": round(int(rp[-1]) / visible, 5), "err": _err_vs(o2, o_dense)}

        for tau in (0.05, 0.2, 0.5):
            poem.poem_select(layer.shape, layer.I_hat, layer.m_hat, tau, layer.row_ptr, layer.col_idx,
                             layer.ws_select)
            rec = {"config": "evaluation", "layer": name, "rule": "poem-threshold", "tau": tau,
                   **run(layer.row_ptr, layer.col_idx)}
            poem.poem_select_mass_only(layer.shape, layer.m_hat, layer.row_ptr, rp2, ci2, layer.ws_select)
            rec["mass_only_same_count"] = run(rp2, ci2)
            out.append(rec)
        d_ex = layer.I_hat / layer.m_hat.clamp_min(1e-30)  # harness-side: Î / m̂ turns the rerank key into log Î
        for gamma in (0.9, 0.95, 0.99):
            rec = {"config": "evaluation", "layer": name, "rule": "same-retained-mass", "gamma": gamma}
            for label, w in (("exact_I_order", 1.0), ("mass_order", 0.0)):
                poem.poem_select_practical(layer.shape, layer.m_hat, d_ex, w, gamma, 1.0, rp2, ci2, layer.ws_select)
                rec[label] = run(rp2, ci2)
            poem.poem_score_pooled(q, k, v, layer.m_pool, layer.d_pool, layer.ws_pooled, shape=layer.shape)
            poem.poem_select_practical(layer.shape, layer.m_pool, layer.d_pool, 1.0, gamma, 0.5, rp2, ci2,
                                       layer.ws_select)
            rec["practical_w1_rho0.5"] = run(rp2, ci2)
            out.append(rec)
        del layer, q, k, v, o_dense, o2, d_ex
        torch.cuda.empty_cache()
    return out


def run_report(args):
    import block_sparse_attention_poem_b200 as poem

    torch.cuda.set_device(0)
    clocks = ClockSampler(0)
    clocks.start()
    part = args.report_only
    if part in (None, "exact"):
        for name, wl, taus, mass_only in REPORT_LAYERS:
            for tau in taus:
                rec = _report_layer(poem, name, wl, tau, args.steps, args.warmup, mass_only, args.cpu_budget_s)
                print(json.dumps(rec), flush=True)
    if part in (None, "practical"):
        for wl, params in PRACTICAL_REPORT:
            for rec in _report_practical(poem, wl, params, args.steps, args.warmup):
                print(json.dumps(rec), flush=True)
    if part in (None, "evaluation"):
        for rec in _report_evaluation(poem):
            print(json.dumps(rec), flush=True)
    if part in (None, "chunked"):
        for rec in _report_chunked(poem, args.steps, args.warmup):
            print(json.dumps(rec), flush=True)
    if part in (None, "grouped"):
        for rec in _report_grouped(poem, args.steps, args.warmup, args.grouped_n):
            print(json.dumps(rec), flush=True)
    if part in (None, "dense"):
        for rec in _report_dense_context(poem, args.steps, args.warmup, tuple(args.dense_n)):
            print(json.dumps(rec), flush=True)
    if part in (None, "sweep"):
        for rec in _report_sweep(poem, args.steps, args.warmup):
            print(json.dumps(rec), flush=True)
    print(json.dumps({"config": "clocks", "clocks": clocks.stop()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama3.1-8b-layer-128k")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-quality", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-practical", action="store_true",
                    help="skip the nested practical-selector record of the default (exact) run")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--ref-step-budget-s", type=float, default=8.0)
    ap.add_argument("--ref-pairs", type=int, default=4,
                    help="reference arm: tile pairs (i, T-1-i) per step (the sample rotates over heads)")
    ap.add_argument("--selector", choices=["exact", "practical"], default="exact")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: independent whole-layer replicas (weak scaling) or one layer split by KV-head "
                         "groups across the ranks (strong scaling)")
    ap.add_argument("--w", type=float, default=1.0, help="practical: weight of log d~ in the rerank key")
    ap.add_argument("--gamma", type=float, default=0.95, help="practical: pooled-mass retention threshold")
    ap.add_argument("--rho", type=float, default=0.5, help="practical: stage-1 shortlist fraction")
    ap.add_argument("--report", action="store_true",
                    help="measure every configuration (one JSON record each) instead of the benchmark line")
    ap.add_argument("--grouped-n", type=int, default=131072,
                    help="token count of the grouped-attention report (a multiple of 128)")
    ap.add_argument("--dense-n", type=int, nargs="+", default=[32768, 131072],
                    help="token counts of the dense-context report (multiples of 128)")
    ap.add_argument("--report-only", choices=["exact", "practical", "evaluation", "chunked", "dense", "grouped",
                                                   "sweep"],
                    default=None,
                    help="with --report: only this part")
    args = ap.parse_args()
    if args.report:
        run_report(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
