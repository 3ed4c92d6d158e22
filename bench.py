#!/usr/bin/env python
"""Benchmark of the batch-1 MXFP4 MoE decode step on B200 (one JSON line on stdout).

Workload (one "step"): the full decode step -- 42 distinct Ling-shaped MoE layers
(hidden 2560, moe_intermediate 768, 512 routed experts top-8 with softmax
renormalisation, one BF16 shared expert of 768, MXFP4 experts: ~67 GB of weights,
so nothing stays in the 126 MB L2 between steps) followed by the 157,184 x 2,560
FP8 LM head with argmax, at M = 1 (decode) and M = 4 (verify window).  Seeded
synthetic weights and tokens; every timed step gets a fresh token row.

value  = algorithmic HBM bytes of the step (weights the method must read + its
         activation I/O, counted from the step's actual routing) / device time,
         summed over ranks (replicas), in GB/s, at M = 1.
e2e    = the same metric through the C-ABI graph launch with the token copied in
         from pinned host memory and logits + argmax copied back, per step.
roofline = the dominant kernel of the step, timed live by CUDA events recorded
         around every launch inside a captured step.
cpu_baseline = the CPU oracle timed on the host on a bounded sample.

--impl reference times the CPU oracle (the reference arm) on the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-step µs and achieved HBM GB/s at M=1/M=4 (fraction of ~8 TB/s)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# DRAM traffic of k_step per layer (read + write): an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum) of the first untraced one-token launch (`--kernel-name-base mangled
# -k regex:k_stepILb1ELb0E -c 1`) in `bench.py --layers 2 --steps 1 --warmup 1
# --no-cpu-baseline --skip-m4 --skip-prefill --skip-head`, valid while the kernel sources
# hash to the value recorded with it (otherwise the roofline's traffic is reported as null).
KSTEP_TRAFFIC = {"bytes_per_layer": (79101696 + 1059072) / 2, "sources_sha256_16": "0fcd417978a35d94",
                 "sources": ("step_kernel.cuh", "decode_kernels.cuh", "common.cuh")}


def kstep_traffic(layers: int):
    import hashlib
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "moe_decode_weight_router_b200", "csrc")
    h = hashlib.sha256()
    for f in KSTEP_TRAFFIC["sources"]:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != KSTEP_TRAFFIC["sources_sha256_16"]:
        return None
    return KSTEP_TRAFFIC["bytes_per_layer"] * layers


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=42)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of CPU-oracle time for cpu_baseline")
    ap.add_argument("--ref-layers", type=int, default=4, help="layers per reference-arm step")
    ap.add_argument("--skip-m4", action="store_true")
    ap.add_argument("--per-layer", action="store_true", help="force the three-kernels-per-layer path")
    ap.add_argument("--skip-prefill", action="store_true", help="skip the prefill-chunk measurement")
    ap.add_argument("--skip-head", action="store_true", help="skip the LM-head comparison and verify window")
    ap.add_argument("--prefill-m", type=int, default=2048, help="tokens of the prefill chunk")
    ap.add_argument("--probe-window", choices=["one", "random", "identical", "disjoint"], default=None,
                    help="byte-accounting probe: one decode step of --layers layers (M=1 for 'one', else an "
                         "M=4 window under the given routing), run twice (the second k_step launch is the "
                         "one to capture); prints its routing and algorithmic bytes")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------
def layer_bytes(S, M, n_unique):
    """Bytes one MoE layer must move: router + shared expert (BF16) + the distinct
    routed experts' MXFP4 codes and scales, plus activation I/O (x in, residual in/out)."""
    router = S.E * S.H * 2
    shared = 3 * S.Is * S.H * 2
    routed = n_unique * S.expert_bytes
    io = M * S.H * (2 + 4 + 4)
    return router + shared + routed + io


def lm_bytes(V, H, M):
    return V * H + V * 4 + M * V * 4 + M * H * 2 + M * 4


def kernel_bytes(S, M, n_unique, V):
    """Per-launch algorithmic bytes of each kernel of a layer (and the LM head)."""
    return {
        "k_dense": S.E * S.H * 2 + 2 * S.Is * S.H * 2 + M * S.H * (2 + 4) + M * (S.E * 4 + S.Is * 4),
        "k_experts13": n_unique * 2 * S.I * (S.H // 2 + S.H // 32) + M * S.H * 2 + n_unique * M * S.I * 4,
        "k_experts2": n_unique * S.H * (S.I // 2 + S.I // 32) + S.Is * S.H * 2 + n_unique * M * S.I * 4
        + M * S.Is * 4 + M * S.H * 8,
        "k_final_norm": M * S.H * (4 + 2),
        "k_lm_gemv": lm_bytes(V, S.H, M),
    }


# ---------------------------------------------------------------------------
# clocks sampler (nvidia-smi during the timed region)
# ---------------------------------------------------------------------------
class Clocks:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuids):
        self.uuids = set(u.lower() for u in uuids if u)
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            if self.uuids and f[1].lower() not in self.uuids:
                continue
            try:
                sm.append(float(f[2]))
                mx.append(float(f[3]))
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for nm, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# replicas: the only cross-rank steps are a barrier and two scalar reductions
# ---------------------------------------------------------------------------
def rank_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_reduce(v, world, device, op):
    """max or sum of a per-rank scalar over the ranks (float64 on `device`)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return t.item()


def replica_gbps(bytes_per_rank, ms_per_rank, world, device):
    """Whole-job rate of N replicas: the bytes all ranks moved over the slowest rank's time."""
    ms = rank_reduce(ms_per_rank, world, device, "max")
    total = rank_reduce(float(bytes_per_rank), world, device, "sum")
    return total / (ms * 1e-3) / 1e9, ms, total


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from moe_decode_weight_router_b200 import (DecodeGraph, DecodeModel, build, decode_step,
                                               decode_step_launch_names, decode_step_workspace_bytes,
                                               lm_head_fp8_quantize, synth)

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    S, V, L = synth.LING, synth.VOCAB, args.layers
    seed = args.seed + 1000 * rank

    # model: L distinct layers + LM head quantised online (once, outside the timed region)
    layers = [synth.layer(S, seed, l, device=dev) for l in range(L)]
    w_lm = synth.lm_head(V, S.H, seed, device=dev)
    lm_q, lm_s = lm_head_fp8_quantize(w_lm)
    torch.cuda.synchronize()
    del w_lm
    torch.cuda.empty_cache()
    model = DecodeModel(layers=layers, lm_q=lm_q, lm_s=lm_s, top_k=S.k, step_path=1 if args.per_layer else 0)

    def barrier():
        rank_barrier(world)

    def max_over_ranks(v):
        return rank_reduce(v, world, dev, "max")

    def sum_over_ranks(v):
        return rank_reduce(v, world, dev, "sum")

    K, W = args.steps, args.warmup
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "")) if hasattr(props, "uuid") else ""
    if uuid and not uuid.startswith("GPU-"):
        uuid = "GPU-" + uuid
    uuids = [None] * world
    if world > 1:
        dist.all_gather_object(uuids, uuid)
    else:
        uuids = [uuid]

    results = {}
    for M in ([1] if args.skip_m4 else [1, 4]):
        xs = [synth.tokens(M, S.H, seed, tid=100 + i, device=dev) for i in range(K + W)]
        ws = torch.empty(decode_step_workspace_bytes(model, M), dtype=torch.uint8, device=dev)
        # routing of every step's token (untimed) -> exact algorithmic bytes per step
        step_bytes, uniq = [], []
        for x in xs:
            r = decode_step(model, x, trace=True, want_logits=False, ws=ws)
            ids = r["ids_trace"].cpu().numpy()
            nu = [len(np.unique(ids[l])) for l in range(L)]
            uniq.append(nu)
            step_bytes.append(sum(layer_bytes(S, M, n) for n in nu) + lm_bytes(V, S.H, M))
        x_buf = xs[0].clone()
        logits = torch.empty((M, V), dtype=torch.float32, device=dev)
        am = torch.empty((M,), dtype=torch.int32, device=dev)
        g = DecodeGraph(model, x_buf, logits, am, ws)
        for i in range(W):
            x_buf.copy_(xs[i])
            g.launch()
        torch.cuda.synchronize()
        clk = Clocks(uuids) if rank == 0 else None
        if clk:
            clk.start()
            time.sleep(0.3)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(K):
            x_buf.copy_(xs[W + i])
            g.launch()
        e1.record()
        torch.cuda.synchronize()
        barrier()
        clocks = clk.stop() if clk else None
        ms_total = max_over_ranks(e0.elapsed_time(e1))
        bytes_rank = float(sum(step_bytes[W:W + K]))
        bytes_all = sum_over_ranks(bytes_rank)
        ms_step = ms_total / K
        # per-step spread (a separate pass: events around each replay, this rank's)
        pe = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(K):
            x_buf.copy_(xs[W + i])
            pe[i][0].record()
            g.launch()
            pe[i][1].record()
        torch.cuda.synchronize()
        per_step = [1000.0 * a.elapsed_time(b) for a, b in pe]
        res = {
            "launches_per_step": len(decode_step_launch_names(model, M)),
            "ms_per_step": ms_step,
            "us_per_step": 1000.0 * ms_step,
            "us_per_step_p10_p50_p90": [float(np.percentile(per_step, q)) for q in (10, 50, 90)],
            "gbps": bytes_all / (ms_total * 1e-3) / 1e9,
            "bytes_per_step": bytes_rank / K,
            "mean_unique_experts": float(np.mean([np.mean(u) for u in uniq[W:W + K]])),
            "clocks": clocks,
        }

        # e2e through the C ABI: pinned host token in, logits + argmax out, per step
        xh = [x.cpu().pin_memory() for x in xs]
        lh = torch.empty((M, V), dtype=torch.float32).pin_memory()
        ah = torch.empty((M,), dtype=torch.int32).pin_memory()
        for i in range(W):
            x_buf.copy_(xh[i], non_blocking=True)
            g.launch()
            lh.copy_(logits, non_blocking=True)
            ah.copy_(am, non_blocking=True)
        torch.cuda.synchronize()
        barrier()
        e0.record()
        for i in range(K):
            x_buf.copy_(xh[W + i], non_blocking=True)
            g.launch()
            lh.copy_(logits, non_blocking=True)
            ah.copy_(am, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        barrier()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1))
        res["e2e"] = {"value": bytes_all / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s", "us_per_step": 1000 * ms_e2e / K,
                      "h2d_bytes_per_step": M * S.H * 2, "d2h_bytes_per_step": M * V * 4 + M * 4}
        g.close()

        # live per-kernel timing: events around every launch inside a captured step
        if M == 1:
            names = decode_step_launch_names(model, M)
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]
            gk = DecodeGraph(model, x_buf, logits, am, ws, events=evs)
            tot = {n: 0.0 for n in set(names)}
            cnt = {n: 0 for n in set(names)}
            kb = {n: 0.0 for n in set(names)}
            reps = max(3, min(K, 10))
            for i in range(reps):
                x_buf.copy_(xs[W + (i % K)])
                gk.launch()
                torch.cuda.synchronize()
                nu = uniq[W + (i % K)]
                for j, n in enumerate(names):
                    tot[n] += evs[2 * j].elapsed_time(evs[2 * j + 1])
                    cnt[n] += 1
                    if n == "k_step":
                        kb[n] += sum(layer_bytes(S, M, u) for u in nu)
                    else:
                        lay = min(j // 3, L - 1)
                        kb[n] += kernel_bytes(S, M, nu[lay], V)[n]
            gk.close()
            ker = {}
            for n in tot:
                avg_ms = tot[n] / cnt[n]
                ker[n] = {"launches_per_step": cnt[n] // reps, "avg_us": 1000 * avg_ms,
                          "share": tot[n] / sum(tot.values()), "gbps": (kb[n] / cnt[n]) / (avg_ms * 1e-3) / 1e9,
                          "bytes_per_launch": kb[n] / cnt[n]}
            res["kernels"] = ker
        results[M] = res

    # LM head: the FP8 head against the BF16 weights it is quantised from (M=1), and the
    # multi-token-prediction verify window (M=4) on synthetic drafts
    if not args.skip_head:
        from moe_decode_weight_router_b200 import lm_head_bf16_gemv, lm_head_fp8_gemv, lm_head_fp8_verify
        w_bf = synth.lm_head(V, S.H, seed, device=dev)
        xh1 = [synth.tokens(1, S.H, seed, tid=300 + i, device=dev) for i in range(K + W)]
        head_us = {}
        for name, fn in (("fp8", lambda x: lm_head_fp8_gemv(x, lm_q, lm_s, want_logits=False)),
                         ("bf16", lambda x: lm_head_bf16_gemv(x, w_bf, want_logits=False))):
            for i in range(W):
                fn(xh1[i])
            torch.cuda.synchronize()
            e0.record()
            for i in range(K):
                fn(xh1[W + i])
            e1.record()
            torch.cuda.synchronize()
            head_us[name] = 1000 * max_over_ranks(e0.elapsed_time(e1)) / K
        del w_bf
        torch.cuda.empty_cache()
        g = torch.Generator(device="cpu")
        g.manual_seed(seed + 11)
        accepted = []
        for i in range(K + W):
            x4 = synth.tokens(4, S.H, seed, tid=500 + i, device=dev)
            _, am4 = lm_head_fp8_gemv(x4, lm_q, lm_s, want_logits=False)
            am4 = am4.cpu()
            drafts = am4[:3].clone()
            keep = torch.rand(3, generator=g) < 0.7
            drafts[~keep] = torch.randint(0, V, (int((~keep).sum()),), generator=g, dtype=torch.int32)
            _, _, acc = lm_head_fp8_verify(x4, lm_q, lm_s, drafts)
            accepted.append(int(acc[0].item()))
        results["head"] = {"fp8_us": head_us["fp8"], "bf16_us": head_us["bf16"],
                           "bf16_over_fp8": head_us["bf16"] / head_us["fp8"],
                           "fp8_gbps": (V * S.H + 4 * V) / (head_us["fp8"] * 1e-6) / 1e9,
                           "bf16_gbps": (2 * V * S.H) / (head_us["bf16"] * 1e-6) / 1e9,
                           "mtp_mean_accept": float(np.mean(accepted)),
                           "mtp_drafts": "each of 3 drafts copies the head's token with probability 0.7, else random"}

    # prefill chunk: one MoE layer for M tokens on the block-scaled tensor cores, each
    # timed call on the next of the L distinct layers (1.6 GB of experts each, > L2)
    if not args.skip_prefill:
        from moe_decode_weight_router_b200 import moe_prefill_layer, moe_prefill_workspace_bytes
        Mp = args.prefill_m
        xp = synth.tokens(Mp, S.H, seed, tid=7, device=dev)
        wsp = torch.empty(moe_prefill_workspace_bytes(Mp, S.H, S.I, S.E, S.k, S.Is), dtype=torch.uint8, device=dev)
        yp = torch.empty((Mp, S.H), dtype=torch.float32, device=dev)
        idp = torch.empty((Mp, S.k), dtype=torch.int32, device=dev)

        def pf(l, ids=False):
            Ly = layers[l % L]
            return moe_prefill_layer(xp, Ly["wr"], Ly["w13c"], Ly["w13s"], Ly["w2c"], Ly["w2s"], Ly["sw13"],
                                     Ly["sw2"], top_k=S.k, ws=wsp, y=yp, want_routing=ids)
        hit = []
        for i in range(min(L, K + W)):
            _, ids, _, _ = pf(i, ids=True)
            hit.append(len(np.unique(ids.cpu().numpy())))
        for i in range(W):
            pf(i)
        torch.cuda.synchronize()
        barrier()
        e0.record()
        for i in range(K):
            pf(W + i)
        e1.record()
        torch.cuda.synchronize()
        barrier()
        ms = max_over_ranks(e0.elapsed_time(e1)) / K
        n_hit = float(np.mean(hit))
        wbytes = S.E * S.H * 2 + n_hit * S.expert_bytes + 3 * S.Is * S.H * 2
        abytes = Mp * S.H * 2 + Mp * S.H * 4
        flops = 2.0 * Mp * S.k * (3 * S.I * S.H) + 2.0 * Mp * (3 * S.Is * S.H) + 2.0 * Mp * S.E * S.H
        results["prefill"] = {"M": Mp, "us_per_chunk": 1000 * ms, "experts_hit": n_hit,
                              "weight_bytes": wbytes, "gbps": world * (wbytes + abytes) / (ms * 1e-3) / 1e9,
                              "tflops": world * flops / (ms * 1e-3) / 1e12, "launches_per_chunk": 10}

    # CPU oracle baseline (rank 0, single GPU only): a bounded sample of the same step
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(model, S, V, args.cpu_budget)
        cpu.update(cpu_baseline_legs(model, S, args.cpu_budget / 4))
    return results, cpu


def _threads():
    n = os.environ.get("OMP_NUM_THREADS")
    if n and n.isdigit():
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(model, S, V, budget_s):
    """Oracle (as it stands) on the host over the same decode step at M = 1: the
    chained layers in order until the time budget is spent (all of them when it
    allows), then the LM head (all rows when the budget allows, else a slice);
    GB/s over the algorithmic bytes actually covered."""
    import numpy as np
    import torch

    import oracle
    from moe_decode_weight_router_b200 import synth

    oracle.lib()

    def fetch_of(Ly):
        def fetch(lst):
            idx = torch.tensor(lst, dtype=torch.long, device=Ly["w13c"].device)
            return {n: synth.bits(Ly[n].index_select(0, idx)) for n in ("w13c", "w13s", "w2c", "w2s")}
        return fetch

    x = synth.bits(synth.tokens(1, S.H, 7, tid=900))
    t_all = 0.0
    nb = 0
    n_done = 0
    for Ly in model.layers:
        spec = [{"wr": synth.bits(Ly["wr"]), "experts": fetch_of(Ly),
                 "shared": {"sw13": synth.bits(Ly["sw13"]), "sw2": synth.bits(Ly["sw2"])}}]
        # host copies of this layer's router/shared weights happen outside the timed calls
        t0 = time.perf_counter()
        ids, w, _, _ = oracle.route(x, spec[0]["wr"], S.k)
        t1 = time.perf_counter()
        ex = spec[0]["experts"](sorted(set(ids.reshape(-1).tolist())))
        t2 = time.perf_counter()
        y = oracle.moe_layer(x, ids, w, _remap(ex, ids), spec[0]["shared"])
        h = (np.vectorize(oracle.bf16_value)(x) if n_done == 0 else h) + y
        x = oracle.rmsnorm_bf16(h)
        t3 = time.perf_counter()
        t_all += (t1 - t0) + (t3 - t2)
        nb += layer_bytes(S, 1, len(np.unique(ids)))
        n_done += 1
        if t_all > budget_s:
            break
    vs = V if t_all < 0.8 * budget_s else 8192
    q = synth.bits(model.lm_q[:vs])
    sc = model.lm_s[:vs].cpu().numpy()
    t0 = time.perf_counter()
    oracle.lmhead_logits(x, q, sc)
    t_all += time.perf_counter() - t0
    nb += lm_bytes(vs, S.H, 1)
    return {"value": nb / t_all / 1e9, "unit": "GB/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{n_done} of {len(model.layers)} chained Ling layers at M=1 + LM head rows [0,{vs}) of {V}; "
                      f"{t_all:.2f} s of oracle time (host copies of the weights excluded)"}


def cpu_baseline_legs(model, S, budget_s):
    """The other oracle legs of the CPU plan, each a bounded sample of its workload:
    one_core  -- the M = 1 step on one host thread (chained layers until budget_s, then
                 8,192 LM-head rows), GB/s over the algorithmic bytes covered;
    m4        -- the M = 4 verify window on all threads (chained layers, routing from
                 the chain), GB/s over the bytes of the distinct experts it touched;
    prefill   -- one M = 2048 prefill chunk of layer 0 (MXFP8 activations): the router
                 over every token, then the layer output of a sample of tokens; the
                 chunk time is the router time plus the per-token time x 2048."""
    import numpy as np
    import torch

    import oracle
    from moe_decode_weight_router_b200 import synth

    def fetch_of(Ly):
        def fetch(lst):
            idx = torch.tensor(lst, dtype=torch.long, device=Ly["w13c"].device)
            return {n: synth.bits(Ly[n].index_select(0, idx)) for n in ("w13c", "w13s", "w2c", "w2s")}
        return fetch

    def chain(M, threads, head_rows):
        oracle.set_threads(threads)
        x = synth.bits(synth.tokens(M, S.H, 8 + M, tid=901))
        h = None
        t_all, nb, n_done = 0.0, 0, 0
        for Ly in model.layers:
            wr = synth.bits(Ly["wr"])
            shared = {"sw13": synth.bits(Ly["sw13"]), "sw2": synth.bits(Ly["sw2"])}
            t0 = time.perf_counter()
            ids, w, _, _ = oracle.route(x, wr, S.k)
            t1 = time.perf_counter()
            ex = fetch_of(Ly)(sorted(set(ids.reshape(-1).tolist())))
            t2 = time.perf_counter()
            y = oracle.moe_layer(x, ids, w, _remap(ex, ids), shared)
            h = (np.vectorize(oracle.bf16_value)(x) if h is None else h) + y
            x = oracle.rmsnorm_bf16(h)
            t3 = time.perf_counter()
            t_all += (t1 - t0) + (t3 - t2)
            nb += layer_bytes(S, M, len(np.unique(ids)))
            n_done += 1
            if t_all > budget_s:
                break
        if head_rows:
            q = synth.bits(model.lm_q[:head_rows])
            sc = model.lm_s[:head_rows].cpu().numpy()
            t0 = time.perf_counter()
            oracle.lmhead_logits(x, q, sc)
            t_all += time.perf_counter() - t0
            nb += lm_bytes(head_rows, S.H, M)
        return nb / t_all / 1e9, n_done, t_all

    legs = {}
    n = _threads()
    v, nl, t = chain(1, 1, 8192)
    legs["one_core"] = {"value": v, "unit": "GB/s", "cores": 1,
                        "sample": f"{nl} chained Ling layers at M=1 + LM-head rows [0,8192); {t:.2f} s"}
    v, nl, t = chain(4, n, 0)
    legs["m4"] = {"value": v, "unit": "GB/s", "cores": n,
                  "sample": f"{nl} chained Ling layers at M=4 (routing from the chain); {t:.2f} s"}
    oracle.set_threads(n)
    # prefill chunk: router over all 2048 tokens, then a sample of tokens' layer outputs
    Mp, ns = 2048, 16
    Ly = model.layers[0]
    x = synth.bits(synth.tokens(Mp, S.H, 11, tid=902))
    t0 = time.perf_counter()
    ids, w, _, _ = oracle.route(x, synth.bits(Ly["wr"]), S.k)
    t_route = time.perf_counter() - t0
    tokens = np.arange(0, Mp, Mp // ns, dtype=np.int32)[:ns]
    ex = fetch_of(Ly)(sorted(set(ids[tokens].reshape(-1).tolist())))
    shared = {"sw13": synth.bits(Ly["sw13"]), "sw2": synth.bits(Ly["sw2"])}
    t0 = time.perf_counter()
    oracle.moe_layer_prefill(x, ids, w, _remap(ex, ids[tokens]), shared, tokens)
    t_tok = (time.perf_counter() - t0) / ns
    legs["prefill"] = {"us_per_chunk": 1e6 * (t_route + t_tok * Mp), "unit": "us", "cores": n,
                       "sample": f"router over {Mp} tokens ({t_route:.2f} s) + layer output of {ns} sampled tokens "
                                 f"({t_tok * 1e3:.1f} ms per token), extrapolated to the {Mp}-token chunk"}
    return legs


def _remap(ex, ids):
    """Expert arrays fetched for sorted(set(ids)) re-indexed by expert id for the oracle."""
    uniq = sorted(set(ids.reshape(-1).tolist()))
    pos = {e: i for i, e in enumerate(uniq)}

    def fetch(lst):
        sel = [pos[e] for e in lst]
        return {n: ex[n][sel] for n in ex}
    return fetch


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle as it stands
# ---------------------------------------------------------------------------
def run_reference(args):
    """The CPU oracle as it stands, on the same metric: each step is a bounded sample
    of the decode step at M = 1 -- ``--ref-layers`` chained Ling layers (two distinct
    layers alternated) and the LM head over 16,384 vocabulary rows."""
    import numpy as np

    import oracle
    from moe_decode_weight_router_b200 import synth

    S, V = synth.LING, synth.VOCAB
    oracle.lib()
    distinct = [{k: synth.bits(v) for k, v in synth.layer(S, args.seed, l, device="cpu").items()} for l in range(2)]
    spec = [{"wr": Ly["wr"], "experts": Ly, "shared": {"sw13": Ly["sw13"], "sw2": Ly["sw2"]}}
            for Ly in (distinct[i % 2] for i in range(args.ref_layers))]
    vs = 16384
    q = synth.bits(synth.e4m3_codes((vs, S.H), args.seed))
    s = synth.row_scales(vs, args.seed).numpy()
    xs = [synth.bits(synth.tokens(1, S.H, args.seed, tid=100 + i)) for i in range(args.steps + args.warmup)]
    for i in range(args.warmup):
        oracle.decode_step(xs[i], spec, q, s, S.k)
    t0 = time.perf_counter()
    nb = 0
    for i in range(args.steps):
        out = oracle.decode_step(xs[args.warmup + i], spec, q, s, S.k)
        nb += sum(layer_bytes(S, 1, len(np.unique(ids))) for ids in out["ids"]) + lm_bytes(vs, S.H, 1)
    dt = time.perf_counter() - t0
    val = nb / dt / 1e9
    sample = f"per step: {args.ref_layers} chained Ling layers at M=1 + LM head rows [0,{vs}) of {V}"
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode step sample (CPU oracle), M=1", "M": 1, "layers": args.ref_layers,
                   "vocab_rows": vs},
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": _threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def probe_window(args):
    """The verify window (M = 4) under a forced routing, for the byte accounting of the
    persistent step: 'identical' repeats one token (every token takes the same 8 experts
    in every layer); 'disjoint' gives token t a large component on hidden dimension t and
    every layer's experts 8t..8t+7 a large router weight on that dimension (each token
    takes its own 8: 32 distinct experts per layer); 'random' is the benchmark's window;
    'one' is the benchmark's one-token step.  Prints the distinct experts of every layer
    and the algorithmic bytes per layer."""
    import numpy as np
    import torch

    from moe_decode_weight_router_b200 import DecodeModel, decode_step, synth
    from moe_decode_weight_router_b200 import build as _b

    _b.build()
    S, dev = synth.LING, "cuda"
    M = 1 if args.probe_window == "one" else 4
    layers = [synth.layer(S, args.seed, l, device=dev) for l in range(args.layers)]
    x = synth.tokens(M, S.H, args.seed, tid=5, device=dev)
    if args.probe_window == "identical":
        x = x[0:1].repeat(M, 1).contiguous()
    elif args.probe_window == "disjoint":
        x[:, :M] = 0
        for t in range(M):
            x[t, t] = 50.0
        for Ly in layers:
            for t in range(M):
                Ly["wr"][8 * t:8 * t + 8, t] = 2.0
    q = synth.e4m3_codes((synth.VOCAB, S.H), args.seed, device=dev)
    s = synth.row_scales(synth.VOCAB, args.seed, device=dev)
    model = DecodeModel(layers=layers, lm_q=q, lm_s=s, top_k=S.k)
    res = None
    for _ in range(2):
        res = decode_step(model, x, trace=True, ws=None if res is None else res["ws"])
    torch.cuda.synchronize()
    ids = res["ids_trace"].cpu().numpy()
    distinct = [int(len(np.unique(ids[l]))) for l in range(args.layers)]
    print(json.dumps({"probe_window": args.probe_window, "M": M, "layers": args.layers,
                      "distinct_experts_per_layer": distinct,
                      "algorithmic_bytes_per_layer": [layer_bytes(S, M, d) for d in distinct]}))
    return 0


def main():
    args = parse_args()
    if args.probe_window:
        return probe_window(args)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return 0
    import datetime

    import torch
    import torch.distributed as dist

    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    results, cpu = run_ours(args, rank, world, local_rank)
    if rank == 0:
        pk, src = peaks()
        hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        r1 = results[1]
        ker = r1.get("kernels", {})
        dom = max(ker, key=lambda n: ker[n]["share"]) if ker else None
        roof = None
        if dom:
            ach = ker[dom]["gbps"]
            traffic = kstep_traffic(args.layers) if dom == "k_step" else None
            roof = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                    "traffic": traffic, "traffic_unit": "bytes per launch (ncu dram read + write)",
                    "peak_source": f"{src} hbm_gbs (copy, burst)"}
        line = {
            "metric": METRIC, "value": r1["gbps"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r1["ms_per_step"], "us_per_step": r1["us_per_step"],
            "us_per_step_p10_p50_p90": r1["us_per_step_p10_p50_p90"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "mxfp4/fp8 weights x bf16 activations, f32 accumulate", "data": "synthetic",
            "frac_of_8tbs": r1["gbps"] / world / NOMINAL_HBM_GBS, "frac_of_measured_hbm": r1["gbps"] / world / hbm,
            "config": {"workload": f"decode step: {args.layers} MoE layers (H2560 I768 E512 top-8 + shared 768, "
                                   "MXFP4) + FP8 LM head 157184x2560, M=1",
                       "M": 1, "layers": args.layers, "hidden": 2560, "experts": 512, "top_k": 8, "vocab": 157184,
                       "l2": "inputs larger than L2: ~67 GB of distinct layer weights streamed per step",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "e2e": {k: v for k, v in r1["e2e"].items()},
            "gpu_launches": r1["launches_per_step"] * args.steps,
            "clocks": r1["clocks"],
            "roofline": roof,
            "kernels": ker,
            "cpu_baseline": cpu,
        }
        if 4 in results:
            r4 = results[4]
            line["m4"] = {"us_per_step": r4["us_per_step"], "us_per_step_p10_p50_p90": r4["us_per_step_p10_p50_p90"],
                          "gbps": r4["gbps"],
                          "frac_of_8tbs": r4["gbps"] / world / NOMINAL_HBM_GBS,
                          "frac_of_measured_hbm": r4["gbps"] / world / hbm,
                          "mean_unique_experts": r4["mean_unique_experts"], "e2e": r4["e2e"], "clocks": r4["clocks"]}
        if "head" in results:
            line["lm_head"] = results["head"]
        if "prefill" in results:
            rp = results["prefill"]
            line["prefill"] = dict(rp, frac_of_measured_hbm=rp["gbps"] / world / hbm,
                                   workload=f"prefill chunk: one MoE layer, M={rp['M']} tokens, MXFP8 activations, "
                                            "tcgen05 block-scaled MMA")
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
