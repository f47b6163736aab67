"""Benchmark of one VeriCache round on B200 (draft attention over the quantised
cache, block verification over the full cache, greedy acceptance).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload (default, one GPU): Llama-3.1-8B attention shapes -- 32 layers,
Hq = 32, Hkv = 8, D = 128, 8 requests at context 32768; KIVI-style 2-bit
cache (group 32, 128-token bf16 residual) in HBM; 30 drafted tokens; the full
bf16 KV (34.4 GB) resident in HBM; vocabulary 128256 with bf16 logits and
geometric accepted-prefix lengths.  One step = one round: 30 draft steps x
32 layers of vc_draft_attn_quant, 32 layers of vc_verify_attn with nq = 31
rows, one vc_accept.  Inputs are synthetic and seeded (no model weights:
query vectors and logits are drawn, not computed).

Reported: ``value`` = draft-attention algorithmic HBM bytes / draft-phase
device time (GB/s); the verify round in microseconds and its HBM fraction;
the roofline of the dominant kernel (the quantised draft attention); an
end-to-end figure with host buffers; the oracle on the host cores.

With ``--gpus N > 1`` (launched by torchrun) every rank runs an independent
replica of the workload (the path has no data exchange); times are the max
over ranks.  ``--impl reference`` times the CPU oracle on a bounded sample of
the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "draft-attn HBM GB/s (% of peak); K=30 verify-round µs vs PCIe/HBM roofline"

WORKLOADS = {
    "llama-3.1-8b-32k-kivi2": dict(NL=32, B=8, Hq=32, Hkv=8, D=128, T=32768, bits=2, G=32, R=128, K=30,
                                   V=128256, logits="bf16", p_mismatch=0.2),
    "llama-3.1-8b-1m-500k-kivi2": dict(NL=32, B=1, Hq=32, Hkv=8, D=128, T=500000, bits=2, G=32, R=128, K=30,
                                       V=128256, logits="bf16", p_mismatch=0.2),
}


def draft_bytes_per_layer(w) -> int:
    """Algorithmic HBM bytes of one quantised draft-attention layer call:
    packed K and V codes, fp16 key scales/zeros per group, fp16 value
    scales/zeros per token, bf16 residual K and V (q and out are negligible)."""
    Lq = w["T"] - w["R"]
    per_head = (2 * Lq * w["D"] * w["bits"] // 8 + (Lq // w["G"]) * w["D"] * 4 + Lq * (w["D"] // w["G"]) * 4
                + w["R"] * w["D"] * 4)
    return per_head * w["Hkv"] * w["B"]


def verify_bytes_per_layer(w) -> int:
    return 4 * w["T"] * w["Hkv"] * w["D"] * w["B"]


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


DRAFT_SOURCES = ["lossless_draft_verify_vc_b200/csrc/vc_draft_quant.cu",
                 "lossless_draft_verify_vc_b200/csrc/vc_splitk.cuh",
                 "lossless_draft_verify_vc_b200/csrc/vc_common.cuh"]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, only while the
    kernel sources still hash to the value recorded with it."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel][workload]
        if e.get("source_hash") == kernel_source_hash(DRAFT_SOURCES):
            return int(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- GPU arm
def build_inputs(w, dev, rank):
    import torch
    from lossless_draft_verify_vc_b200 import synth, vc

    seed0 = 1000 * rank
    NL, B, Hq, Hkv, D, T, K = w["NL"], w["B"], w["Hq"], w["Hkv"], w["D"], w["T"], w["K"]
    nq = K + 1
    caches, kvs = [], []
    for l in range(NL):
        caches.append(synth.random_quant_cache(B, Hkv, T - w["R"], w["R"], D, w["bits"], w["G"],
                                               seed=seed0 + l, device=dev))
        kvs.append(synth.kv_full(B, Hkv, T, D, seed=seed0 + 500 + l, device=dev))
    q_draft = synth.normal((K, NL, B, Hq, D), seed0 + 1, dev)
    q_ver = synth.normal((NL, B, nq, Hq, D), seed0 + 2, dev)
    draft_tok = synth.tokens((B, K), w["V"], seed0 + 3, dev)
    lens = synth.geometric_accept_lengths(B, K, w["p_mismatch"], seed0 + 3)
    ldt = torch.bfloat16 if w["logits"] == "bf16" else torch.float32
    logits = synth.planted_logits(B, K, w["V"], draft_tok.cpu(), lens, seed0 + 4, device="cpu", dtype=ldt).to(dev)
    sh = vc.shape(B, Hq, Hkv, D)
    qcs = [vc.quant_cache(c) for c in caches]
    return dict(caches=caches, kvs=kvs, q_draft=q_draft, q_ver=q_ver, draft_tok=draft_tok, logits=logits,
                lens=lens, sh=sh, qcs=qcs)


def run_gpu(args, w, rank, world):
    import torch
    from lossless_draft_verify_vc_b200 import vc

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    vc.lib()  # fail loudly if the library is missing
    inp = build_inputs(w, dev, rank)
    NL, B, Hq, Hkv, D, T, K, V = w["NL"], w["B"], w["Hq"], w["Hkv"], w["D"], w["T"], w["K"], w["V"]
    nq = K + 1
    sh = inp["sh"]
    ws_d = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, inp["qcs"][0]), dev)
    ws_v = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq), dev)
    ws_a = vc.workspace(vc.vc_accept_workspace_size(B, K, V), dev)
    out_d = torch.empty(B, Hq, D, device=dev)
    out_v = torch.empty(B, nq, Hq, D, device=dev)
    tgt = torch.empty(B, K + 1, dtype=torch.int32, device=dev)
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    cor = torch.empty(B, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        q_draft, q_ver, logits, draft_tok = inp["q_draft"], inp["q_ver"], inp["logits"], inp["draft_tok"]
        if ev: ev[0].record(stream)
        for t in range(K):                      # draft: one token per step, every layer
            for l in range(NL):
                vc.vc_draft_attn_quant(sh, inp["qcs"][l], q_draft[t, l], out_d, ws_d, stream)
        if ev: ev[1].record(stream)
        for l in range(NL):                     # verify: nq rows per request, every layer
            k, v = inp["kvs"][l]
            vc.vc_verify_attn(sh, q_ver[l], k, v, T, nq, out_v, None, ws_v, stream)
        if ev: ev[2].record(stream)
        vc.vc_accept(logits, B, K, V, draft_tok, tgt, acc, cor, ws_a, stream)
        if ev: ev[3].record(stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # warm-up
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert acc.cpu().tolist() == inp["lens"], "acceptance mismatch on the planted logits"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    draft_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    verify_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    accept_ms = sum(e[2].elapsed_time(e[3]) for e in evs)

    # end to end: inputs of every step copied from pinned host memory inside the
    # timed region, results read back to the host
    h_qd = inp["q_draft"].cpu().pin_memory()
    h_qv = inp["q_ver"].cpu().pin_memory()
    h_lg = inp["logits"].cpu().pin_memory()
    h_dt = inp["draft_tok"].cpu().pin_memory()
    d_qd, d_qv = torch.empty_like(inp["q_draft"]), torch.empty_like(inp["q_ver"])
    d_lg, d_dt = torch.empty_like(inp["logits"]), torch.empty_like(inp["draft_tok"])
    h_res = torch.empty(B * (K + 3), dtype=torch.int32).pin_memory()
    e2e_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(args.steps):
        ev = e2e_evs[s]
        ev[0].record(stream)
        d_qd.copy_(h_qd, non_blocking=True)
        for t in range(K):
            for l in range(NL):
                vc.vc_draft_attn_quant(sh, inp["qcs"][l], d_qd[t, l], out_d, ws_d, stream)
        ev[1].record(stream)
        d_qv.copy_(h_qv, non_blocking=True)
        d_lg.copy_(h_lg, non_blocking=True)
        d_dt.copy_(h_dt, non_blocking=True)
        for l in range(NL):
            k, v = inp["kvs"][l]
            vc.vc_verify_attn(sh, d_qv[l], k, v, T, nq, out_v, None, ws_v, stream)
        vc.vc_accept(d_lg, B, K, V, d_dt, tgt, acc, cor, ws_a, stream)
        h_res[:B * (K + 1)].copy_(tgt.view(-1), non_blocking=True)
        h_res[B * (K + 1):B * (K + 2)].copy_(acc, non_blocking=True)
        h_res[B * (K + 2):].copy_(cor, non_blocking=True)
        ev[2].record(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_total_ms = e0.elapsed_time(e1)
    e2e_draft_ms = sum(e[0].elapsed_time(e[1]) for e in e2e_evs)
    h2d = (h_qd.numel() * h_qd.element_size() + h_qv.numel() * h_qv.element_size()
           + h_lg.numel() * h_lg.element_size() + h_dt.numel() * h_dt.element_size())
    d2h = h_res.numel() * h_res.element_size()

    times = torch.tensor([total_ms, draft_ms, verify_ms, accept_ms, e2e_total_ms, e2e_draft_ms], dtype=torch.float64)
    if world > 1:
        tt = times.to(dev)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        times = tt.cpu()
    total_ms, draft_ms, verify_ms, accept_ms, e2e_total_ms, e2e_draft_ms = times.tolist()
    return dict(total_ms=total_ms, draft_ms=draft_ms, verify_ms=verify_ms, accept_ms=accept_ms,
                e2e_total_ms=e2e_total_ms, e2e_draft_ms=e2e_draft_ms, h2d=h2d, d2h=d2h, clocks=clk)


# ----------------------------------------------------------------------------- oracle leg
def oracle_sample(w, budget_s: float):
    """Time the oracle's quantised draft attention on (request 0, KV head 0)
    slices of one layer, repeated until ~budget_s; returns (GB/s, slices,
    seconds, threads)."""
    import numpy as np
    import torch
    from lossless_draft_verify_vc_b200 import synth
    from oracle import attention as A

    try:
        from threadpoolctl import threadpool_info
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count() or 1
    g = w["Hq"] // w["Hkv"]
    c = synth.random_quant_cache(1, 1, w["T"] - w["R"], w["R"], w["D"], w["bits"], w["G"], seed=7, device="cpu")
    cache = dict(bits=c["bits"], group=c["group"], L_q=c["L_q"], R=c["R"], D=c["D"],
                 records=c["records"].numpy(), k_res=c["k_res"].float().numpy(), v_res=c["v_res"].float().numpy())
    q = synth.normal((1, g, w["D"]), 8).float().numpy()
    per_slice = draft_bytes_per_layer(dict(w, B=1, Hkv=1))
    n = 0
    t0 = time.perf_counter()
    while True:
        A.draft_attention_quant(q, cache)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return per_slice * n / el / 1e9, n, el, threads, per_slice


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama-3.1-8b-32k-kivi2", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (small cases for profiler captures; 0 = the workload's)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = dict(WORKLOADS[args.workload])
    if args.layers > 0:
        w["NL"] = args.layers
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    peak, peak_kind = read_peaks()
    nq = w["K"] + 1
    config = {"workload": args.workload, "layers": w["NL"], "requests_per_gpu": w["B"], "context": w["T"],
              "heads": [w["Hq"], w["Hkv"]], "head_dim": w["D"], "bits": w["bits"], "group": w["G"],
              "residual": w["R"], "draft_len": w["K"], "verify_rows": nq, "vocab": w["V"],
              "l2": "inputs larger than L2 (draft cache and full KV are tens of GB; no flush needed)",
              "parallelism": f"replicas x{args.gpus}"}

    if args.impl == "reference":
        if rank != 0:
            return
        budget = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
        vals = []
        for _ in range(args.warmup):
            oracle_sample(w, budget / 4)
        for _ in range(args.steps):
            gbs, n, el, threads, per_slice = oracle_sample(w, budget)
            vals.append(gbs)
        v = statistics.median(vals)
        sample = (f"oracle quantised draft attention on (request 0, KV head 0) of one layer, "
                  f"{per_slice} bytes per slice, ~{budget:.1f} s per step")
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
                "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import torch
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    r = run_gpu(args, w, rank, world)
    K, NL = w["K"], w["NL"]
    db = draft_bytes_per_layer(w)
    vb = verify_bytes_per_layer(w)
    draft_bytes_step = db * K * NL
    value = draft_bytes_step * args.steps * world / (r["draft_ms"] * 1e-3) / 1e9
    launches_draft = K * NL * args.steps
    avg_launch_us = r["draft_ms"] * 1e3 / launches_draft
    achieved = db / (avg_launch_us * 1e-6) / 1e9
    verify_round_us = r["verify_ms"] * 1e3 / args.steps
    verify_gbs = vb * NL / (verify_round_us * 1e-6) / 1e9
    e2e_value = draft_bytes_step * args.steps * world / (r["e2e_draft_ms"] * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["total_ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int2 codes + bf16 -> fp16/bf16 MMA, fp32 accumulate",
        "data": "synthetic (seeded random KV, queries and logits; no model weights)", "config": config,
        "draft_frac_of_hbm_peak": value / world / peak,
        "verify_round_us": verify_round_us,
        "verify_hbm_gbps": verify_gbs, "verify_frac_of_hbm_peak": verify_gbs / peak,
        "accept_us": r["accept_ms"] * 1e3 / args.steps,
        "phases_ms_per_step": {"draft": r["draft_ms"] / args.steps, "verify": r["verify_ms"] / args.steps,
                               "accept": r["accept_ms"] / args.steps},
        "roofline": {"kernel": "vc_draft_attn_quant (draft_quant_kernel)", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs (burst copy)", "unit": "GB/s",
                     "frac": achieved / peak, "traffic": recorded_traffic("draft_quant_kernel", args.workload),
                     "algorithmic_bytes_per_launch": db},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "note": "draft phase timed with its queries copied from pinned host memory; every step also "
                        "copies verify queries, logits and draft tokens in and reads target/accept/correction out"},
        "gpu_launches": (K * NL + NL + 1) * args.steps,
        "clocks": r["clocks"],
    }
    if rank == 0 and world == 1:
        gbs, n, el, threads, per_slice = oracle_sample(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"{n} x (request 0, KV head 0) of one layer ({per_slice} bytes each) "
                                          f"in {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
