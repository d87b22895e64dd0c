#!/usr/bin/env python
"""Benchmark of the lightning-indexer hot path on B200.

One step = one call of the library's hot path over one batch of synthetic
input resident in HBM: for a prefill workload the fused tcgen05 score +
streaming Top-k kernel and the final exact selection (dsa_index_prefill);
for the decode workload the planner, the same fused kernel and the
selection (dsa_index_decode).  The metric is causally visible (query, key)
pairs per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle, same metric

Under torchrun each rank runs its own replica of the workload (different
seed) on its own GPU by default; there is no collective in the data path
("scaling": "weak"): value = all ranks' pairs / the slowest rank's time.
With --shard rows the ranks split ONE workload instead ("scaling": "strong"):
contiguous query-row blocks balanced by visible pairs (decode: sequence
blocks), keys replicated, still no collective in the data path.
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
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from synth import WORKLOADS, make_decode, make_prefill, make_prefill_fp8  # noqa: E402

DEFAULT_WORKLOAD = "causal_16k_h64"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--path", choices=["dense", "pruned"], default="dense",
                    help="prefill path: dense fused scoring, or DoSA certified pruning")
    ap.add_argument("--paged", type=int, default=0,
                    help="decode: keys in a shuffled page pool of this page size (a multiple of 64)")
    ap.add_argument("--dtype", choices=["bf16", "fp8"], default="bf16",
                    help="dense prefill inputs: bf16, or FP8 E4M3 codes with per-row scales")
    ap.add_argument("--shard", choices=["replicas", "rows"], default="replicas",
                    help="N>1: independent replicas per rank (weak) or one workload split by rows (strong)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# the sources that decide the fused score kernel's code and its launches (the
# DRAM traffic recorded for it does not depend on the other kernels' files)
SCORE_KERNEL_SOURCES = ("dsa_score.cu", "dsa_kernels.cuh", "dsa_ptx.cuh", "dsa_api.cu")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in SCORE_KERNEL_SOURCES:
        f = ROOT / "sparse_attention_token_03_b200" / "csrc" / name
        h.update(f.name.encode())
        h.update(f.read_bytes())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel
    sources have not changed since the capture (else None)."""
    f = ROOT / "profiles" / "ncu_traffic.txt"
    if not f.exists():
        return None
    cur = kernel_source_hash()
    for line in f.read_text().splitlines():
        parts = line.split("#", 1)[0].split()
        if len(parts) >= 4 and parts[0] == workload and parts[1] == kernel and parts[2] == cur:
            return float(parts[3])
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", gpu_id, "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# CPU oracle timings (the reference arm and the cpu_baseline leg)
# ----------------------------------------------------------------------------

def oracle_sample_rate(wl, x, target_s: float, rows_cap: int | None = None):
    """Time the oracle on evenly spaced rows; returns (pairs/s, rows, pairs, secs, cores)."""
    import oracle
    cores = oracle.threads()
    if wl.kind == "decode":
        def run(n):
            pick = np.unique(np.linspace(0, wl.B - 1, n).round().astype(int))
            t0 = time.perf_counter()
            oracle.decode_topk(x["q"][pick], x["w"][pick], x["k"][pick], x["seq_len"][pick], wl.topk)
            dt = time.perf_counter() - t0
            return dt, int(x["seq_len"][pick].sum()), len(pick)
        total_rows = wl.B
    else:
        def run(n):
            rows = np.unique(np.linspace(0, wl.T_q - 1, n).round().astype(np.int64))
            t0 = time.perf_counter()
            if "q8" in x:  # FP8 inputs: the FP8 oracle
                oracle.prefill_topk_fp8(x["q8"], x["q_scale"], x["w"], x["k8"], x["k_scale"], x["q_offset"],
                                        wl.topk, rows=rows)
            else:
                oracle.prefill_topk(x["q"], x["w"], x["k"], x["q_offset"], wl.topk, rows=rows)
            dt = time.perf_counter() - t0
            return dt, int((x["q_offset"] + rows + 1).sum()), len(rows)
        total_rows = wl.T_q
    n = min(total_rows, max(cores, 4))
    dt, pairs, got = run(n)
    want = n * target_s / max(dt, 1e-3)
    n2 = int(min(total_rows, max(n, want)))
    if rows_cap:
        n2 = min(n2, rows_cap)
    if n2 > n:
        dt, pairs, got = run(n2)
    return pairs / dt, got, pairs, dt, cores


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = make_prefill(wl) if wl.kind == "prefill" else make_decode(wl)
    budget = 150.0
    per_step = budget / max(args.steps + args.warmup, 1)
    rate, rows, pairs, dt, cores = oracle_sample_rate(wl, x, per_step)
    # calibrated sample; now the timed steps on that sample size
    import oracle
    if wl.kind == "decode":
        pick = np.unique(np.linspace(0, wl.B - 1, rows).round().astype(int))
        step = lambda: oracle.decode_topk(x["q"][pick], x["w"][pick], x["k"][pick],
                                          x["seq_len"][pick], wl.topk)
        step_pairs = int(x["seq_len"][pick].sum())
        sample = f"{len(pick)} of {wl.B} sequences per step"
    else:
        rws = np.unique(np.linspace(0, wl.T_q - 1, rows).round().astype(np.int64))
        step = lambda: oracle.prefill_topk(x["q"], x["w"], x["k"], x["q_offset"], wl.topk, rows=rws)
        step_pairs = int((x["q_offset"] + rws + 1).sum())
        sample = f"{len(rws)} evenly spaced rows of {wl.T_q} per step ({step_pairs} pairs)"
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = step_pairs * args.steps / dt
    line = {
        "impl": "reference", "metric": "indexer causal q.k pairs/s", "value": value,
        "unit": "pairs/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": "pairs/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "pairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl):
    c = {"workload": wl.name, "H": wl.H, "d": wl.d, "topk": wl.topk, "keys": wl.keys}
    if wl.kind == "prefill":
        c.update(T_q=wl.T_q, T_k=wl.T_k, q_offset=wl.q_offset)
    else:
        c.update(B=wl.B, t_cap=wl.t_cap)
    c["pairs_per_step"] = wl.visible_pairs
    return c


# ----------------------------------------------------------------------------
# CUDA arm
# ----------------------------------------------------------------------------

def main():
    args = parse_args()
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return

    import torch
    import torch.distributed as dist

    import sparse_attention_token_03_b200 as dsa
    from sparse_attention_token_03_b200.shard import (max_over_ranks, row_shards, sequence_shards,
                                                      shard_pairs, sum_over_ranks)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    sharded = args.shard == "rows" and world > 1
    seed = wl.seed + (0 if sharded else 7919 * rank)
    pruned = args.path == "pruned"
    if pruned and (wl.kind != "prefill" or wl.n_seed == 0):
        raise SystemExit(f"--path pruned needs a chunked prefill workload with a seed set, not {wl.name}")
    fp8 = args.dtype == "fp8"
    if fp8 and (wl.kind != "prefill" or pruned):
        raise SystemExit("--dtype fp8 runs the dense prefill")
    if fp8:
        x = make_prefill_fp8(wl, seed=seed)
    elif wl.kind == "prefill":
        x = make_prefill(wl, seed=seed, with_anchor=pruned)
    else:
        x = make_decode(wl, seed=seed)
    q_off = wl.q_offset
    if sharded:
        # this rank's block of query rows (decode: sequences) of the one workload
        if wl.kind == "prefill":
            b, e = row_shards(wl.T_q, wl.q_offset, world)[rank]
            pairs = shard_pairs(wl.T_q, wl.q_offset, (b, e))
            q_off = wl.q_offset + b
        else:
            b, e = sequence_shards(x["seq_len"], world)[rank]
            x["k"] = x["k"][b:e]
            x["seq_len"] = x["seq_len"][b:e]
            pairs = int(x["seq_len"].sum())
        if e <= b:
            raise SystemExit(f"--shard rows: rank {rank} has no rows of {wl.name}")
        x["q"], x["w"] = x["q"][b:e], x["w"][b:e]
        if fp8:
            x["q8"], x["q_scale"] = x["q8"][b:e], x["q_scale"][b:e]
    else:
        pairs = wl.visible_pairs
    total_pairs = sum_over_ranks(pairs, dev) if world > 1 else pairs

    def to_dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    q, k = to_dev_bf16(x["q"]), to_dev_bf16(x["k"])
    w = torch.from_numpy(x["w"]).to(dev)
    rows = x["q"].shape[0]
    out_idx = torch.empty((rows, wl.topk), dtype=torch.int32, device=dev)
    out_score = torch.empty((rows, wl.topk), dtype=torch.float32, device=dev)
    filter_stats = None
    if wl.kind == "prefill" and pruned:
        # seed set: the anchor query's Top-k (the query just before the chunk,
        # selected by this library's own decode call) plus random keys
        qa = to_dev_bf16(x["q_anchor"][None])
        wa = torch.from_numpy(x["w_anchor"][None]).to(dev)
        ka = k[:wl.q_offset].unsqueeze(0)
        la = torch.tensor([wl.q_offset], dtype=torch.int32, device=dev)
        aidx, _ = dsa.dsa_index_decode(qa, wa, ka.contiguous(), la, wl.n_anchor)
        anchor = aidx[0].cpu().numpy()
        from synth import random_distinct_keys
        rnd = random_distinct_keys(seed + 1, 0, wl.q_offset, wl.n_seed - wl.n_anchor, exclude=anchor)
        seeds = torch.from_numpy(np.concatenate([anchor, rnd]).astype(np.int32)).to(dev)
        del ka
        ws = torch.empty(dsa.dsa_index_prefill_pruned_workspace_bytes(rows, wl.T_k, wl.H, wl.d, wl.topk,
                                                                      wl.n_seed),
                         dtype=torch.uint8, device=dev)
        _, _, filter_stats = dsa.dsa_index_prefill_pruned(q, w, k, q_off, wl.topk, seeds,
                                                          out_idx=out_idx, out_score=out_score,
                                                          workspace=ws, stats=True)
        # pairs of the query groups the dense pass computed (groups of 256/H
        # rows holding a row the pruned path did not finish)
        _, _, state = dsa.dsa_index_prefill_pruned_survivors(ws, rows, wl.T_k, q_off, wl.H, wl.d, wl.topk,
                                                             wl.n_seed)
        st_np = state.cpu().numpy()
        G = 256 // wl.H
        grp = np.zeros((rows + G - 1) // G, bool)
        np.logical_or.at(grp, np.arange(rows) // G, st_np != 0)
        dense_rows = np.flatnonzero(np.repeat(grp, G)[:rows])
        dense_group_pairs = int((q_off + dense_rows + 1).sum())
        filter_stats["dense_pass_pairs"] = dense_group_pairs

        def step(qq=q, ww=w, kk=k, oi=out_idx, osc=out_score):
            dsa.dsa_index_prefill_pruned(qq, ww, kk, q_off, wl.topk, seeds, out_idx=oi,
                                         out_score=osc, workspace=ws)
        n_kernels = 20  # launches of one pruned call (probe and rest of the chunk)
    elif fp8:
        ws = torch.empty(dsa.dsa_index_prefill_workspace_bytes(rows, wl.T_k, wl.H, wl.d, wl.topk),
                         dtype=torch.uint8, device=dev)
        q8 = torch.from_numpy(np.ascontiguousarray(x["q8"])).to(dev)
        k8 = torch.from_numpy(np.ascontiguousarray(x["k8"])).to(dev)
        qs = torch.from_numpy(x["q_scale"]).to(dev)
        ks = torch.from_numpy(x["k_scale"]).to(dev)
        del q, k

        def step(qq=q8, ww=w, kk=k8, oi=out_idx, osc=out_score, qsc=qs, ksc=ks):
            dsa.dsa_index_prefill_fp8(qq, qsc, ww, kk, ksc, q_off, wl.topk, out_idx=oi, out_score=osc,
                                      workspace=ws)
        n_kernels = 2
    elif wl.kind == "prefill":
        ws = torch.empty(dsa.dsa_index_prefill_workspace_bytes(rows, wl.T_k, wl.H, wl.d, wl.topk),
                         dtype=torch.uint8, device=dev)

        def step(qq=q, ww=w, kk=k, oi=out_idx, osc=out_score):
            dsa.dsa_index_prefill(qq, ww, kk, q_off, wl.topk, out_idx=oi, out_score=osc,
                                  workspace=ws)
        n_kernels = 2
    elif args.paged:
        # the same caches scattered over a shuffled pool of pages
        page = args.paged
        B_, t_cap_ = x["k"].shape[0], x["k"].shape[1]
        max_blocks = (t_cap_ + page - 1) // page
        perm = np.random.default_rng(seed + 2).permutation(B_ * max_blocks).astype(np.int32)
        bt = torch.from_numpy(perm.reshape(B_, max_blocks)).to(dev)
        pool = torch.empty((B_ * max_blocks, page, wl.d), dtype=torch.bfloat16, device=dev)
        kpad = torch.nn.functional.pad(k, (0, 0, 0, max_blocks * page - t_cap_))
        pool[bt.reshape(-1).long()] = kpad.reshape(B_ * max_blocks, page, wl.d)
        del kpad, k
        k = pool
        seq_len = torch.from_numpy(x["seq_len"]).to(dev)
        ws = torch.empty(dsa.dsa_index_decode_workspace_bytes(rows, max_blocks * page, wl.H, wl.d, wl.topk),
                         dtype=torch.uint8, device=dev)

        def step(qq=q, ww=w, kk=pool, oi=out_idx, osc=out_score, sl=seq_len):
            dsa.dsa_index_decode_paged(qq, ww, kk, bt, sl, wl.topk, out_idx=oi, out_score=osc, workspace=ws)
        n_kernels = 3
    else:
        seq_len = torch.from_numpy(x["seq_len"]).to(dev)
        ws = torch.empty(dsa.dsa_index_decode_workspace_bytes(rows, wl.t_cap, wl.H, wl.d, wl.topk),
                         dtype=torch.uint8, device=dev)

        def step(qq=q, ww=w, kk=k, oi=out_idx, osc=out_score, sl=seq_len):
            dsa.dsa_index_decode(qq, ww, kk, sl, wl.topk, out_idx=oi, out_score=osc, workspace=ws)
        n_kernels = 3
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    dsa.dsa_profile_enable(True)
    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize(dev)
    if dsa.dsa_index_device_status(ws) != 0:
        raise RuntimeError("device status word set during warm-up")

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id)
    time.sleep(0.3)
    step_ms, kern_ms = [], {}
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    for i in range(args.steps):
        flush.fill_((i + 1) & 0xFF)  # evict the previous step's data from L2 (not timed)
        ev0.record(stream)
        step()
        ev1.record(stream)
        ev1.synchronize()
        step_ms.append(ev0.elapsed_time(ev1))
        per = {}
        for name, ms in dsa.dsa_profile_read():  # a kernel may run more than once per call
            per[name] = per.get(name, 0.0) + ms
        for name, ms in per.items():
            kern_ms.setdefault(name, []).append(ms)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    dsa.dsa_profile_enable(False)
    status = dsa.dsa_index_device_status(ws)

    ms_step = max_over_ranks(float(np.mean(step_ms)), dev)
    value = total_pairs / (ms_step * 1e-3)

    # ---- roofline of the dominant kernel (the fused score + Top-k kernel)
    pk, pk_src = peaks()
    score_ms = float(np.mean(kern_ms.get("score_topk", [float("nan")])))
    if pruned:
        # the dominant kernel is the screen (16 plan rows per query, 2*16*d
        # executed flops per screened pair) or, when the probe sent rows to
        # the dense kernel, the dense pass (2*H*d flops per pair of the query
        # groups it computed)
        screen_ms = float(np.mean(kern_ms.get("screen", [0.0])))
        dense_ms = float(np.mean(kern_ms.get("dense_pass", [0.0])))
        if screen_ms >= dense_ms:
            score_ms = screen_ms
            flops = 2.0 * 16 * wl.d * filter_stats["screened_pairs"]
            kname, tkey = "score_topk_kernel (screen variant)", "screen"
        else:
            score_ms = dense_ms
            flops = 2.0 * wl.H * wl.d * dense_group_pairs
            kname, tkey = "score_topk_kernel (dense pass over flagged rows)", "score_topk_kernel"
        achieved = flops / (score_ms * 1e-3) / 1e12
        peak = float(pk["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": f"bf16_tflops (burst) of {pk_src}",
                "kernel": kname, "kernel_ms": score_ms,
                "traffic": recorded_traffic(wl.name + "_pruned", tkey)}
    elif wl.kind == "prefill":
        flops = 2.0 * wl.H * wl.d * pairs
        achieved = flops / (score_ms * 1e-3) / 1e12
        # FP8 takes its own dtype's peak: the measured bf16 burst figure times
        # the nominal dense FP8 / bf16 ratio (4.5 / 2.25 PFLOP/s)
        peak = float(pk["bf16_tflops"]) * (2.0 if fp8 else 1.0)
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "peak_source": (f"2 x bf16_tflops (burst) of {pk_src} (nominal fp8/bf16 ratio)" if fp8
                                else f"bf16_tflops (burst) of {pk_src}")}
    else:
        nbytes = 2.0 * wl.d * pairs  # every visible key read once
        achieved = nbytes / (score_ms * 1e-3) / 1e9
        peak = float(pk["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": f"hbm_gbs of {pk_src}"}
    if not pruned:
        roof["kernel"] = "score_topk_kernel"
        roof["kernel_ms"] = score_ms
        roof["traffic"] = recorded_traffic(wl.name + ("_fp8" if fp8 else ""), "score_topk_kernel")
    if roof["bound"] == "tensor":
        # the same achieved rate against the other peaks of the dtype: the
        # sustained (power-capped) cuBLAS loop and the datasheet's dense figure
        ratio = 2.0 if fp8 else 1.0
        spec = 2250.0 * ratio
        sus = float(pk["bf16_tflops_sustained"]) * ratio
        roof["frac_vs_sustained"] = roof["achieved"] / sus
        roof["frac_vs_spec"] = roof["achieved"] / spec
        roof["peaks_other"] = {"sustained": sus, ("spec_dense_fp8" if fp8 else "spec_dense_bf16"): spec}

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e and not args.paged:  # (the paged layout has no host-buffer leg)
        hq = torch.from_numpy(np.ascontiguousarray(x["q"]).view(np.int16)).view(torch.bfloat16).pin_memory()
        # (decode keeps its key cache on the device; the other paths take keys from the host)
        hk = (None if wl.kind == "decode" else
              torch.from_numpy(np.ascontiguousarray(x["k"]).view(np.int16)).view(torch.bfloat16).pin_memory())
        hw = torch.from_numpy(x["w"]).pin_memory()
        hoi = torch.empty(out_idx.shape, dtype=torch.int32).pin_memory()
        hos = torch.empty(out_score.shape, dtype=torch.float32).pin_memory()
        extra = {}
        if wl.kind == "decode":
            extra["sl"] = torch.from_numpy(x["seq_len"]).pin_memory()
            dsl = torch.empty_like(seq_len)
        h2d = hq.numel() * 2 + (hk.numel() * 2 if hk is not None else 0) + hw.numel() * 4
        d2h = hoi.numel() * 4 + hos.numel() * 4
        n_e2e = max(3, min(args.steps, 20))
        e_ms = []
        if fp8:
            # FP8 codes and scales in, results out, on one stream
            hq8 = torch.from_numpy(np.ascontiguousarray(x["q8"])).pin_memory()
            hk8 = torch.from_numpy(np.ascontiguousarray(x["k8"])).pin_memory()
            hqs, hks = torch.from_numpy(x["q_scale"]).pin_memory(), torch.from_numpy(x["k_scale"]).pin_memory()
            dq8, dk8, dqs, dks, dw = (torch.empty_like(q8), torch.empty_like(k8), torch.empty_like(qs),
                                      torch.empty_like(ks), torch.empty_like(w))
            h2d = hq8.numel() + hk8.numel() + 4 * (hqs.numel() + hks.numel() + hw.numel())
            e2e_api = "dsa_index_prefill_fp8: codes, scales and weights in, results out (one stream)"

            def e2e_step():
                dq8.copy_(hq8, non_blocking=True)
                dk8.copy_(hk8, non_blocking=True)
                dqs.copy_(hqs, non_blocking=True)
                dks.copy_(hks, non_blocking=True)
                dw.copy_(hw, non_blocking=True)
                step(dq8, dw, dk8, out_idx, out_score, dqs, dks)
                hoi.copy_(out_idx, non_blocking=True)
                hos.copy_(out_score, non_blocking=True)
        elif wl.kind == "prefill" and not pruned:
            # the library's host-buffer entry point: row blocks stream through
            # the device with the copies overlapping the kernels
            hws = torch.empty(dsa.dsa_index_prefill_host_workspace_bytes(rows, wl.T_k, wl.H, wl.d, wl.topk),
                              dtype=torch.uint8, device=dev)
            e2e_api = "dsa_index_prefill_host (pipelined row blocks)"

            def e2e_step():
                dsa.dsa_index_prefill_host(hq, hw, hk, q_off, wl.topk, out_idx=hoi, out_score=hos,
                                           workspace=hws, device=dev)
        elif wl.kind == "decode":
            # a decode step's inputs are the new token's query, head weights and
            # key per sequence (plus the lengths); the key cache of the earlier
            # tokens stays resident in HBM, and the new keys are appended to it
            sl_np = x["seq_len"].astype(np.int64)
            hnew = torch.from_numpy(np.ascontiguousarray(
                x["k"][np.arange(rows), np.maximum(sl_np - 1, 0)]).view(np.int16)).view(torch.bfloat16).pin_memory()
            dq, dw, dnew = torch.empty_like(q), torch.empty_like(w), torch.empty(hnew.shape, dtype=k.dtype, device=dev)
            kc = k.clone()  # the resident cache the new keys are written into
            bidx = torch.arange(rows, device=dev)
            h2d = hq.numel() * 2 + hw.numel() * 4 + rows * 4 + hnew.numel() * 2
            e2e_api = ("dsa_index_decode with a device-resident key cache: query, weights, lengths "
                       "and one new key per sequence in, results out (one stream)")

            def e2e_step():
                dq.copy_(hq, non_blocking=True)
                dw.copy_(hw, non_blocking=True)
                dsl.copy_(extra["sl"], non_blocking=True)
                dnew.copy_(hnew, non_blocking=True)
                kc[bidx, (dsl.long() - 1).clamp_(min=0)] = dnew  # append this step's keys
                step(dq, dw, kc, out_idx, out_score, dsl)
                hoi.copy_(out_idx, non_blocking=True)
                hos.copy_(out_score, non_blocking=True)
        else:
            dq, dk, dw = torch.empty_like(q), torch.empty_like(k), torch.empty_like(w)
            e2e_api = "copies in, device entry point, copies out (one stream)"

            def e2e_step():
                dq.copy_(hq, non_blocking=True)
                dk.copy_(hk, non_blocking=True)
                dw.copy_(hw, non_blocking=True)
                step(dq, dw, dk, out_idx, out_score)
                hoi.copy_(out_idx, non_blocking=True)
                hos.copy_(out_score, non_blocking=True)
        for i in range(n_e2e + 2):
            flush.fill_(i & 0xFF)
            ev0.record(stream)
            e2e_step()
            ev1.record(stream)
            ev1.synchronize()
            if i >= 2:
                e_ms.append(ev0.elapsed_time(ev1))
        em = max_over_ranks(float(np.mean(e_ms)), dev)
        e2e = {"value": total_pairs / (em * 1e-3), "unit": "pairs/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": em, "api": e2e_api}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, nrows, spairs, sdt, cores = oracle_sample_rate(wl, x, target_s=15.0)
        unit = "rows" if wl.kind == "prefill" else "sequences"
        cpu = {"value": rate, "unit": "pairs/s", "cores": cores, "kind": "oracle",
               "sample": f"{nrows} evenly spaced {unit} of {wl.name} ({spairs} pairs, {sdt:.1f} s)"}

    if rank == 0:
        line = {
            "metric": "indexer causal q.k pairs/s" + (" (effective, DoSA)" if pruned else ""),
            "value": value, "unit": "pairs/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
            "dtype": "fp8 (e4m3, fp32 scales)" if fp8 else "bf16", "data": "synthetic",
            "config": dict(workload_config(wl), l2="flushed between steps (256 MiB write)",
                           parallelism=(f"row blocks x{world}" if sharded else f"replicas x{world}"),
                           path=args.path, inputs=args.dtype,
                           **({"page_size": args.paged} if args.paged else {})),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": n_kernels * args.steps, "clocks": clocks, "device_status": status,
            "kernel_ms": {n: float(np.mean(v)) for n, v in kern_ms.items()},
        }
        if filter_stats is not None:
            line["dosa"] = dict(filter_stats, filter_rate=1.0 - filter_stats["survivor_pairs"]
                                / max(filter_stats["screened_pairs"], 1),
                                filter_rate_over="screened rows (all rows, or the probe rows when the "
                                                 "probe sent the chunk to the dense pass)")
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
