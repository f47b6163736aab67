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
import datetime
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
    # quantised draft cache in HBM, full KV resident in HBM
    "llama-3.1-8b-32k-kivi2": dict(kind="resident", streamed_too=True, NL=32, B=8, Hq=32, Hkv=8, D=128, T=32768,
                                   bits=2, G=32, R=128, K=30, V=128256, logits="bf16", p_mismatch=0.2,
                                   host_pool=2),
    # the same shapes at 500K context; verification runs resident and host-streamed
    "llama-3.1-8b-1m-500k-kivi2": dict(kind="resident", streamed_too=True, NL=32, B=1, Hq=32, Hkv=8, D=128,
                                       T=500000, bits=2, G=32, R=128, K=30, V=128256, logits="bf16",
                                       p_mismatch=0.2, host_pool=2),
    # token-dropped draft cache (25% kept per layer-head) in HBM, full KV in pinned host memory
    "qwen-32b-100k-tokdrop4-streamed": dict(kind="streamed", NL=64, B=1, Hq=40, Hkv=8, D=128, T=100000,
                                            n_keep=25000, K=30, V=152064, logits="bf16", p_mismatch=0.2,
                                            host_pool=4),
    # four requests, 4-bit group-64 draft caches, full KV in pinned host memory, staggered by the scheduler
    "llama-70b-4x131k-4bit-stagger": dict(kind="stagger", NL=80, B=1, n_req=4, Hq=64, Hkv=8, D=128, T=131072,
                                          bits=4, G=64, R=128, K=30, V=128256, logits="bf16", p_mismatch=0.2,
                                          host_pool=2),
    # the verification pass through 32 decoder layers with random bf16 weights (Llama-3.1-8B dimensions),
    # full KV resident: tokens verified per second, comparable only in kind (no trained weights)
    "llama-3.1-8b-32k-layers-verify": dict(kind="layers", NL=32, B=8, Hq=32, Hkv=8, D=128, T=32768, K=30,
                                           d_model=4096, d_ff=14336, V=128256),
    # remote prefix caching: each request's compressed prefix cache arrives over an emulated 1.2 GB/s remote
    # link, its full cache is streamed for verification over an emulated 40 GB/s local link
    "llama-3.1-8b-4x32k-kivi2-remote-prefix": dict(kind="remote", NL=32, B=1, n_req=4, Hq=32, Hkv=8, D=128,
                                                   T=32768, bits=2, G=32, R=128, K=30, V=128256, logits="bf16",
                                                   p_mismatch=0.2, host_pool=2, remote_gbps=1.2, local_gbps=40.0,
                                                   rounds=2),
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


def sparse_bytes_per_layer(w) -> int:
    """Algorithmic HBM bytes of one token-dropped draft layer call: the kept
    bf16 K and V rows plus their int32 indices."""
    return w["n_keep"] * w["Hkv"] * (4 * w["D"] + 4) * w["B"]


def measure_pcie_h2d(dev, srcs=(), nbytes: int = 1 << 30, reps: int = 5) -> float:
    """Pinned host -> device copy bandwidth (GB/s, best of reps) of one
    cudaMemcpyAsync: the host-link peak the streamed verification is
    measured against.  Copies a fresh pinned buffer of nbytes and each of
    `srcs` (pinned host tensors: the streamed layers themselves, whose host
    memory may sit elsewhere than a fresh buffer); the best rate counts."""
    import torch
    st = torch.cuda.Stream(dev)
    best = 0.0
    fresh = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    for h in (fresh, *srcs):
        d = torch.empty_like(h, device=dev)
        nb = h.numel() * h.element_size()
        with torch.cuda.stream(st):
            d.copy_(h, non_blocking=True)
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(st)
                d.copy_(h, non_blocking=True)
                e1.record(st)
                e1.synchronize()
                best = max(best, nb / (e0.elapsed_time(e1) * 1e-3) / 1e9)
        del d
    del fresh
    return best


def host_pool(w, dev_dtype, n: int):
    """n distinct pinned host layers of full bf16 K and V [B, Hkv, T, D]; the
    streamed layers cycle through them (the host link moves every layer's
    bytes; only the host RAM they come from is shared)."""
    import torch
    from lossless_draft_verify_vc_b200 import synth
    hk, hv = [], []
    for i in range(n):
        k, v = synth.kv_full(w["B"], w["Hkv"], w["T"], w["D"], seed=900 + i, device="cuda")
        hk.append(k.cpu().pin_memory())
        hv.append(v.cpu().pin_memory())
        del k, v
    return hk, hv


def streamed_verify_pass(vc, ks, sh, q_ver, T, nq, NL, out_v, ws_v, comp):
    """One verification pass over NL layers streamed from host memory: the copy
    of layer l + 2 overlaps the verification of layer l (two staging slots)."""
    ks.prefetch(0)
    if NL > 1:
        ks.prefetch(1)
    for l in range(NL):
        kp, vp = ks.acquire(l, comp)
        vc.vc_verify_attn(sh, q_ver[l], kp, vp, T, nq, out_v, None, ws_v, comp)
        ks.release(l, comp)
        if l + 2 < NL:
            ks.prefetch(l + 2)


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks of the default
    process group (identity without one): multi-GPU times are the slowest
    rank's."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist = torch.distributed
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def whole_job_rate(bytes_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput of independent replicas (GB/s): every rank
    processes the same work per step; the job takes the slowest rank's time."""
    return bytes_per_rank_step * steps * world / (max_ms * 1e-3) / 1e9


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def read_tensor_peak():
    """Dense bf16 tensor-core peak (TFLOP/s): the measured cuBLAS burst figure
    when the box carries one, else the fallback measured earlier on this kind
    of box."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def time_resident_verify_layer(w, dev, reps: int = 20):
    """One layer's block verification with the full K and V resident in HBM
    (the workload's request shape), timed alone with CUDA events over `reps`
    calls alternating two layers (each larger than L2): the HBM and the
    tensor-pipe fractions of the kernel, which the host link hides when the
    cache is streamed."""
    import torch
    from lossless_draft_verify_vc_b200 import synth, vc
    B, Hq, Hkv, D, T, nq = w["B"], w["Hq"], w["Hkv"], w["D"], w["T"], w["K"] + 1
    sh = vc.shape(B, Hq, Hkv, D)
    kv = [synth.kv_full(B, Hkv, T, D, seed=70 + l, device=dev) for l in range(2)]
    q = synth.normal((B, nq, Hq, D), 72, dev)
    out = torch.empty(B, nq, Hq, D, device=dev)
    ws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq), dev)
    comp = torch.cuda.current_stream(dev)
    for l in range(4):
        vc.vc_verify_attn(sh, q, kv[l % 2][0], kv[l % 2][1], T, nq, out, None, ws, comp)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for l in range(reps):
        vc.vc_verify_attn(sh, q, kv[l % 2][0], kv[l % 2][1], T, nq, out, None, ws, comp)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / reps
    byt = 4 * T * Hkv * D * B
    flops = 4 * nq * Hq * T * D * B
    del kv
    torch.cuda.empty_cache()
    return dict(us_per_layer=us, hbm_gbps=byt / (us * 1e-6) / 1e9, tflops=flops / (us * 1e-6) / 1e12,
                bytes_per_layer=byt, flops_per_layer=flops, reps=reps)


def kernel_source_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


DRAFT_SOURCES = ["lossless_draft_verify_vc_b200/csrc/vc_draft_quant.cu",
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
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,timestamp")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        """Starts sampling every 100 ms and returns once the first sample is
        written (at most ~3 s), so that the timed region that follows is
        covered; samples before this point and after stop() are dropped by
        their timestamps."""
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.t0 = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        for _ in range(60):
            if os.path.getsize(self.path) > 0 or self.proc.poll() is not None:
                break
            time.sleep(0.05)
        self.t0 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        t1 = time.time()
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

        def stamp(r):
            try:
                return datetime.datetime.strptime(r[9], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except (ValueError, IndexError):
                return None

        inside = [r for r in rows if self.t0 is not None and stamp(r) is not None and self.t0 - 0.1 <= stamp(r) <= t1]
        rows = inside or rows  # keep every sample when the window holds none (a very short region)
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
    # the draft caches are written once before the loop and never by a kernel
    # of the step: the draft kernel may start copying records early
    for c in caches:
        c["flags"] = vc.VC_CACHE_STATIC
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

    # end to end through the public API: every step copies its inputs from
    # pinned host memory, runs the calls and reads its results back; timed by
    # the host clock (synchronised at the draft phase's end and the step's end)
    h_qd = inp["q_draft"].cpu().pin_memory()
    h_qv = inp["q_ver"].cpu().pin_memory()
    h_lg = inp["logits"].cpu().pin_memory()
    h_dt = inp["draft_tok"].cpu().pin_memory()
    d_qd, d_qv = torch.empty_like(inp["q_draft"]), torch.empty_like(inp["q_ver"])
    d_lg, d_dt = torch.empty_like(inp["logits"]), torch.empty_like(inp["draft_tok"])
    h_out = torch.empty(out_d.shape, dtype=out_d.dtype).pin_memory()
    h_res = torch.empty(B * (K + 3), dtype=torch.int32).pin_memory()
    barrier()
    torch.cuda.synchronize(dev)
    draft_wall, step_wall = [], []
    for s in range(args.steps):
        th0 = time.perf_counter()
        d_qd.copy_(h_qd, non_blocking=True)
        for t in range(K):
            for l in range(NL):
                vc.vc_draft_attn_quant(sh, inp["qcs"][l], d_qd[t, l], out_d, ws_d, stream)
        h_out.copy_(out_d, non_blocking=True)
        stream.synchronize()
        th1 = time.perf_counter()
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
        stream.synchronize()
        th2 = time.perf_counter()
        draft_wall.append((th1 - th0) * 1e3)
        step_wall.append((th2 - th0) * 1e3)
    barrier()
    e2e_draft_ms = sum(draft_wall)
    e2e_total_ms = sum(step_wall)
    h2d = (h_qd.numel() * h_qd.element_size() + h_qv.numel() * h_qv.element_size()
           + h_lg.numel() * h_lg.element_size() + h_dt.numel() * h_dt.element_size())
    d2h = h_out.numel() * h_out.element_size() + h_res.numel() * h_res.element_size()

    compress = time_compress(w, dev, inp) if rank == 0 else None

    streamed = None
    if w.get("streamed_too"):
        streamed = time_streamed_verify(args, w, dev, inp, sh, ws_v, out_v, stream)

    total_ms, draft_ms, verify_ms, accept_ms, e2e_total_ms, e2e_draft_ms = max_over_ranks(
        [total_ms, draft_ms, verify_ms, accept_ms, e2e_total_ms, e2e_draft_ms], dev)
    return dict(total_ms=total_ms, draft_ms=draft_ms, verify_ms=verify_ms, accept_ms=accept_ms,
                e2e_total_ms=e2e_total_ms, e2e_draft_ms=e2e_draft_ms, h2d=h2d, d2h=d2h, clocks=clk, compress=compress,
                streamed=streamed)


def time_compress(w, dev, inp):
    """Building the draft caches on the GPU for one layer of the workload:
    quantising its full K and V into group records + residual, and gathering
    25% kept rows into a kept-row pool.  Device time per call (CUDA events,
    inputs larger than L2) and algorithmic bytes (full rows read, records and
    residual or pool rows written)."""
    import torch
    from lossless_draft_verify_vc_b200 import synth, vc
    B, Hkv, D, T, R, G, bits = w["B"], w["Hkv"], w["D"], w["T"], w["R"], w["G"], w["bits"]
    k, v = inp["kvs"][0]
    k2, v2 = inp["kvs"][1 % len(inp["kvs"])]
    L_q = T - R
    rec_b = 2 * G * D * bits // 8 + 8 * D
    records = torch.empty((B, Hkv, L_q // G, rec_b), dtype=torch.uint8, device=dev)
    kr = torch.empty((B, Hkv, R, D), dtype=torch.bfloat16, device=dev)
    vr = torch.empty_like(kr)
    ws = vc.workspace(vc.vc_compress_workspace_size(), dev)
    sh = inp["sh"]
    n_keep = T // 4
    idx = synth.kept_positions(B, Hkv, T, n_keep, seed=77, device=dev)
    ko = torch.empty((B, Hkv, n_keep, D), dtype=torch.bfloat16, device=dev)
    vo = torch.empty_like(ko)

    def timed(fn, n=10):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(n):
            fn(i)
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) * 1e3 / n

    q_us = timed(lambda i: vc.vc_quantize_cache(sh, k if i % 2 else k2, v if i % 2 else v2, T, bits, G, L_q,
                                                records, kr, vr, R, ws))
    c_us = timed(lambda i: vc.vc_compact_kept(sh, k if i % 2 else k2, v if i % 2 else v2, T, idx, n_keep, ko, vo,
                                              ws))
    flags = vc.vc_workspace_flags(ws)
    q_bytes = 2 * B * Hkv * T * D * 2 + records.numel() + 2 * B * Hkv * R * D * 2
    c_bytes = 2 * 2 * B * Hkv * n_keep * D * 2 + idx.numel() * 4
    del records, kr, vr, ko, vo
    return dict(quantize_us=q_us, quantize_gbps=q_bytes / (q_us * 1e-6) / 1e9, quantize_bytes=q_bytes,
                compact_us=c_us, compact_gbps=c_bytes / (c_us * 1e-6) / 1e9, compact_bytes=c_bytes,
                compact_kept_per_head=n_keep, flags=flags)


def time_streamed_verify(args, w, dev, inp, sh, ws_v, out_v, comp):
    """Verification rounds with every layer's full K and V streamed from
    pinned host memory (double-buffered staging); returns the round time,
    the link bytes per second and the measured link peak."""
    import torch
    from lossless_draft_verify_vc_b200 import vc
    NL, T, nq = w["NL"], w["T"], w["K"] + 1
    hk, hv = host_pool(w, torch.bfloat16, w.get("host_pool", 2))
    pcie = measure_pcie_h2d(dev, (hk[0], hv[0]))
    host_k = [hk[l % len(hk)] for l in range(NL)]
    host_v = [hv[l % len(hv)] for l in range(NL)]
    stage_k = [torch.empty_like(hk[0], device=dev) for _ in range(2)]
    stage_v = [torch.empty_like(hv[0], device=dev) for _ in range(2)]
    copy = torch.cuda.Stream(dev)
    ks = vc.KvStream(host_k, host_v, stage_k, stage_v, copy)
    steps = max(1, min(args.steps, 3))
    for _ in range(1):
        streamed_verify_pass(vc, ks, sh, inp["q_ver"], T, nq, NL, out_v, ws_v, comp)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    copy.wait_event(e0)
    for _ in range(steps):
        streamed_verify_pass(vc, ks, sh, inp["q_ver"], T, nq, NL, out_v, ws_v, comp)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    ks.close()
    ms = e0.elapsed_time(e1) / steps
    link_bytes = 2 * hk[0].numel() * hk[0].element_size() * NL
    return dict(round_us=ms * 1e3, link_gbps=link_bytes / (ms * 1e-3) / 1e9, pcie_peak_gbps=pcie,
                rounds=steps, host_pool_layers=len(hk))


def run_streamed(args, w, rank, world):
    """Token-dropped draft over a kept-row pool in HBM, verification streamed
    per layer from pinned host memory, greedy acceptance."""
    import torch
    from lossless_draft_verify_vc_b200 import synth, vc

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    vc.lib()
    NL, B, Hq, Hkv, D, T, K, V, nk = w["NL"], w["B"], w["Hq"], w["Hkv"], w["D"], w["T"], w["K"], w["V"], w["n_keep"]
    nq = K + 1
    seed0 = 1000 * rank
    sh = vc.shape(B, Hq, Hkv, D)
    # kept-row pools: the n_keep kept K and V rows of every layer-head, addressed
    # through index lists (here the pool slots 0..n_keep-1)
    idx = torch.arange(nk, dtype=torch.int32, device=dev).expand(B, Hkv, nk).contiguous()
    pools = [synth.kv_full(B, Hkv, nk, D, seed=seed0 + l, device=dev) for l in range(NL)]
    scs = [vc.sparse_cache(k, v, idx) for k, v in pools]
    q_draft = synth.normal((K, NL, B, Hq, D), seed0 + 1, dev)
    q_ver = synth.normal((NL, B, nq, Hq, D), seed0 + 2, dev)
    draft_tok = synth.tokens((B, K), V, seed0 + 3, dev)
    lens = synth.geometric_accept_lengths(B, K, w["p_mismatch"], seed0 + 3)
    logits = synth.planted_logits(B, K, V, draft_tok.cpu(), lens, seed0 + 4, device="cpu",
                                  dtype=torch.bfloat16).to(dev)
    ws_d = vc.workspace(vc.vc_draft_attn_sparse_workspace_size(sh, scs[0]), dev)
    ws_v = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq), dev)
    ws_a = vc.workspace(vc.vc_accept_workspace_size(B, K, V), dev)
    out_d = torch.empty(B, Hq, D, device=dev)
    out_v = torch.empty(B, nq, Hq, D, device=dev)
    tgt = torch.empty(B, K + 1, dtype=torch.int32, device=dev)
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    cor = torch.empty(B, dtype=torch.int32, device=dev)
    hk, hv = host_pool(w, torch.bfloat16, w["host_pool"])
    pcie = measure_pcie_h2d(dev, (hk[0], hv[0]))
    host_k = [hk[l % len(hk)] for l in range(NL)]
    host_v = [hv[l % len(hv)] for l in range(NL)]
    stage_k = [torch.empty_like(hk[0], device=dev) for _ in range(2)]
    stage_v = [torch.empty_like(hv[0], device=dev) for _ in range(2)]
    comp = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)
    ks = vc.KvStream(host_k, host_v, stage_k, stage_v, copy)

    def step(ev=None):
        if ev: ev[0].record(comp)
        for t in range(K):
            for l in range(NL):
                vc.vc_draft_attn_sparse(sh, scs[l], q_draft[t, l], out_d, ws_d, comp)
        if ev:
            ev[1].record(comp)
            copy.wait_event(ev[1])  # the timed verification starts its copies here
        streamed_verify_pass(vc, ks, sh, q_ver, T, nq, NL, out_v, ws_v, comp)
        if ev: ev[2].record(comp)
        vc.vc_accept(logits, B, K, V, draft_tok, tgt, acc, cor, ws_a, comp)
        if ev: ev[3].record(comp)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert acc.cpu().tolist() == lens, "acceptance mismatch on the planted logits"
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    for i in range(args.steps):
        step(evs[i])
    t1.record(comp)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ks.close()
    total_ms, draft_ms, verify_ms, accept_ms = max_over_ranks(
        [t0.elapsed_time(t1), sum(e[0].elapsed_time(e[1]) for e in evs), sum(e[1].elapsed_time(e[2]) for e in evs),
         sum(e[2].elapsed_time(e[3]) for e in evs)], dev)
    return dict(total_ms=total_ms, draft_ms=draft_ms, verify_ms=verify_ms, accept_ms=accept_ms,
                clocks=clk, pcie=pcie, link_bytes=2 * hk[0].numel() * hk[0].element_size() * NL,
                host_pool_layers=len(hk))


def run_stagger(args, w, rank, world):
    """Several requests, each a 4-bit draft over its quantised cache and a
    host-streamed verification, run by the scheduler in lock-step and in the
    staggered order; both policies' round times are reported."""
    import torch
    from lossless_draft_verify_vc_b200 import synth, vc

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    vc.lib()
    NL, B, Hq, Hkv, D, T, K, V, n = (w["NL"], w["B"], w["Hq"], w["Hkv"], w["D"], w["T"], w["K"], w["V"],
                                     w["n_req"])
    nq = K + 1
    sh = vc.shape(B, Hq, Hkv, D)
    hk, hv = host_pool(w, torch.bfloat16, w["host_pool"])
    pcie = measure_pcie_h2d(dev, (hk[0], hv[0]))
    copy = torch.cuda.Stream(dev)
    reqs, keep = [], []
    for i in range(n):
        seed0 = 1000 * rank + 100 * i
        caches = [synth.random_quant_cache(B, Hkv, T - w["R"], w["R"], D, w["bits"], w["G"], seed=seed0 + l,
                                           device=dev) for l in range(NL)]
        qcs = [vc.quant_cache(c) for c in caches]
        q_draft = synth.normal((K, NL, B, Hq, D), seed0 + 1, dev)
        q_ver = synth.normal((NL, B, nq, Hq, D), seed0 + 2, dev)
        toks = synth.tokens((B, K), V, seed0 + 3, dev)
        lens = synth.geometric_accept_lengths(B, K, w["p_mismatch"], seed0 + 3)
        logits = synth.planted_logits(B, K, V, toks.cpu(), lens, seed0 + 4, device="cpu",
                                      dtype=torch.bfloat16).to(dev)
        st_k = [torch.empty_like(hk[0], device=dev) for _ in range(2)]
        st_v = [torch.empty_like(hv[0], device=dev) for _ in range(2)]
        out = dict(d=torch.empty(B, Hq, D, device=dev), v=torch.empty(B, nq, Hq, D, device=dev),
                   t=torch.empty(B, K + 1, dtype=torch.int32, device=dev),
                   a=torch.empty(B, dtype=torch.int32, device=dev), c=torch.empty(B, dtype=torch.int32, device=dev))
        dws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qcs[0]), dev)
        vws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq), dev)
        aws = vc.workspace(vc.vc_accept_workspace_size(B, K, V), dev)
        stream = torch.cuda.Stream(dev)
        reqs.append(vc.make_sched_request(sh, vc.VC_DRAFT_QUANT, qcs, q_draft, out["d"], dws,
                                          [hk[l % len(hk)] for l in range(NL)], [hv[l % len(hv)] for l in range(NL)],
                                          st_k, st_v, q_ver, out["v"], vws, T, nq, logits, V, toks, out["t"],
                                          out["a"], out["c"], aws, stream))
        keep.append((caches, qcs, out, lens, q_draft))
    # draft kernel alone (request 0), as in the resident workload
    qcs0, q_draft0, out0 = keep[0][1], keep[0][4], keep[0][2]["d"]
    dws0 = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qcs0[0]), dev)
    comp = torch.cuda.current_stream(dev)
    for l in range(NL):
        vc.vc_draft_attn_quant(sh, qcs0[l], q_draft0[0, l], out0, dws0, comp)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for t in range(K):
        for l in range(NL):
            vc.vc_draft_attn_quant(sh, qcs0[l], q_draft0[t, l], out0, dws0, comp)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    draft_ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    res = {}
    clocks = ClockSampler(dev.index)
    clocks.start()
    for name, pol in (("lockstep", vc.VC_SCHED_LOCKSTEP), ("stagger", vc.VC_SCHED_STAGGER)):
        sch = vc.Sched(reqs, NL, K, pol, copy, timeout_ms=30000)
        sch.run_rounds(1)  # warm-up round
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        st = sch.run_rounds(max(1, min(args.steps, 2)))
        torch.cuda.synchronize(dev)
        sch.close()
        st["elapsed_ms"], st["link_busy_ms"] = max_over_ranks([st["elapsed_ms"], st["link_busy_ms"]], dev)
        for r, (_, _, out, lens, _) in zip(reqs, keep):
            assert out["a"].cpu().tolist() == lens, "acceptance mismatch under the scheduler"
        res[name] = st
    clk = clocks.stop()
    return dict(draft_ms=draft_ms, sched=res, pcie=pcie, clocks=clk,
                link_bytes_per_request=2 * hk[0].numel() * hk[0].element_size() * NL, host_pool_layers=len(hk))


def run_remote(args, w, rank, world):
    """Remote prefix caching: every request's compressed cache (all layers:
    group records and residual) starts in pinned host memory and reaches the
    GPU over the emulated remote link before the request's first draft; each
    round then drafts from it (HBM) and verifies against the full cache
    streamed over the emulated local link.  One run = the fetches plus
    `rounds` rounds of every request, by the scheduler in lock-step and in
    the staggered order."""
    import torch
    from lossless_draft_verify_vc_b200 import synth, vc

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    vc.lib()
    NL, B, Hq, Hkv, D, T, K, V, n = (w["NL"], w["B"], w["Hq"], w["Hkv"], w["D"], w["T"], w["K"], w["V"],
                                     w["n_req"])
    nq = K + 1
    sh = vc.shape(B, Hq, Hkv, D)
    hk, hv = host_pool(w, torch.bfloat16, w["host_pool"])
    copy, remote = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    reqs, keep, fetch = [], [], []
    accepted = 0
    for i in range(n):
        seed0 = 1000 * rank + 100 * i
        caches, src, dst = [], [], []
        for l in range(NL):
            c = synth.random_quant_cache(B, Hkv, T - w["R"], w["R"], D, w["bits"], w["G"], seed=seed0 + l,
                                         device=dev)
            for key in ("records", "k_res", "v_res"):
                src.append(c[key].cpu().pin_memory())
                dst.append(c[key])
                c[key].zero_()  # the device copy is filled by the fetch
            caches.append(c)
        qcs = [vc.quant_cache(c) for c in caches]
        q_draft = synth.normal((K, NL, B, Hq, D), seed0 + 1, dev)
        q_ver = synth.normal((NL, B, nq, Hq, D), seed0 + 2, dev)
        toks = synth.tokens((B, K), V, seed0 + 3, dev)
        lens = synth.geometric_accept_lengths(B, K, w["p_mismatch"], seed0 + 3)
        accepted += sum(a + 1 for a in lens)
        logits = synth.planted_logits(B, K, V, toks.cpu(), lens, seed0 + 4, device="cpu",
                                      dtype=torch.bfloat16).to(dev)
        st_k = [torch.empty_like(hk[0], device=dev) for _ in range(2)]
        st_v = [torch.empty_like(hv[0], device=dev) for _ in range(2)]
        out = dict(d=torch.empty(B, Hq, D, device=dev), v=torch.empty(B, nq, Hq, D, device=dev),
                   t=torch.empty(B, K + 1, dtype=torch.int32, device=dev),
                   a=torch.empty(B, dtype=torch.int32, device=dev), c=torch.empty(B, dtype=torch.int32, device=dev))
        dws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qcs[0]), dev)
        vws = vc.workspace(vc.vc_verify_attn_workspace_size(sh, T, nq), dev)
        aws = vc.workspace(vc.vc_accept_workspace_size(B, K, V), dev)
        stream = torch.cuda.Stream(dev)
        reqs.append(vc.make_sched_request(sh, vc.VC_DRAFT_QUANT, qcs, q_draft, out["d"], dws,
                                          [hk[l % len(hk)] for l in range(NL)], [hv[l % len(hv)] for l in range(NL)],
                                          st_k, st_v, q_ver, out["v"], vws, T, nq, logits, V, toks, out["t"],
                                          out["a"], out["c"], aws, stream))
        keep.append((caches, qcs, out, lens, q_draft))
        fetch.append((src, dst))
    fetch_bytes = sum(t.numel() * t.element_size() for src, _ in fetch for t in src)
    rounds = w.get("rounds", 2)
    # draft kernel alone (request 0, its cache fetched once directly)
    for a_, b_ in zip(*fetch[0]):
        b_.copy_(a_)
    qcs0, q_draft0, out0 = keep[0][1], keep[0][4], keep[0][2]["d"]
    dws0 = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, qcs0[0]), dev)
    comp = torch.cuda.current_stream(dev)
    for l in range(NL):
        vc.vc_draft_attn_quant(sh, qcs0[l], q_draft0[0, l], out0, dws0, comp)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for t in range(K):
        for l in range(NL):
            vc.vc_draft_attn_quant(sh, qcs0[l], q_draft0[t, l], out0, dws0, comp)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    draft_ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    res = {}
    clocks = ClockSampler(dev.index)
    clocks.start()
    for name, pol in (("lockstep", vc.VC_SCHED_LOCKSTEP), ("stagger", vc.VC_SCHED_STAGGER)):
        sch = vc.Sched(reqs, NL, K, pol, copy, timeout_ms=30000)
        sch.set_links(remote, w["remote_gbps"], w["local_gbps"])
        for i, (src, dst) in enumerate(fetch):
            sch.set_fetch(i, src, dst)
        if world > 1:
            torch.distributed.barrier()
        st = sch.run_rounds(rounds)
        torch.cuda.synchronize(dev)
        sch.close()
        for k in ("elapsed_ms", "fetch_ms", "link_busy_ms", "first_draft_ms"):
            st[k] = max_over_ranks([st[k]], dev)[0]
        for (_, _, out, lens, _) in keep:
            assert out["a"].cpu().tolist() == lens, "acceptance mismatch under the scheduler"
        res[name] = st
    clk = clocks.stop()
    return dict(draft_ms=draft_ms, sched=res, clocks=clk, fetch_bytes=fetch_bytes,
                link_bytes_per_request_round=2 * hk[0].numel() * hk[0].element_size() * NL,
                host_pool_layers=len(hk), rounds=rounds, tokens_per_run=accepted * rounds)


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
    ap.add_argument("--kernel", default="", choices=["", "draft", "verify", "accept", "compress"],
                    help="time one kernel of the workload alone (a per-kernel line for profiler captures; "
                         "not the benchmark line)")
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
    config = {"workload": args.workload, "layers": w["NL"], "requests_per_gpu": w["B"] * w.get("n_req", 1),
              "context": w["T"], "heads": [w["Hq"], w["Hkv"]], "head_dim": w["D"], "draft_len": w["K"],
              "verify_rows": nq, "vocab": w["V"],
              "l2": "inputs larger than L2 (draft caches and KV are GBs; no flush needed)",
              "parallelism": f"replicas x{args.gpus}"}
    if "bits" in w:
        config.update(bits=w["bits"], group=w["G"], residual=w["R"])
    if "n_keep" in w:
        config.update(kept_per_head=w["n_keep"], kept_row_pool="idx = pool slots 0..n_keep-1")
    if w["kind"] not in ("resident", "layers") or w.get("streamed_too"):
        config.update(full_kv="pinned host memory, streamed per layer",
                      host_pool_layers=w.get("host_pool", 2))
    if w["kind"] in ("stagger", "remote"):
        config.update(requests=w["n_req"])
    if w["kind"] == "layers":
        config.update(full_kv="resident in HBM", d_model=w["d_model"], d_ff=w["d_ff"],
                      weights="random bf16 (no trained weights)")
    if w["kind"] == "remote":
        config.update(full_kv="pinned host memory, streamed per layer over the emulated local link",
                      draft_cache="pinned host memory, fetched over the emulated remote link",
                      remote_gbps=w["remote_gbps"], local_gbps=w["local_gbps"])

    if args.kernel:
        print(json.dumps(kernel_line(args, w, peak, peak_kind)), flush=True)
        return

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
    if w["kind"] == "streamed":
        line = streamed_line(args, w, rank, world, config, peak, peak_kind)
    elif w["kind"] == "stagger":
        line = stagger_line(args, w, rank, world, config, peak, peak_kind)
    elif w["kind"] == "remote":
        line = remote_line(args, w, rank, world, config, peak, peak_kind)
    elif w["kind"] == "layers":
        line = layers_line(args, w, rank, world, config, peak, peak_kind)
    else:
        line = resident_line(args, w, rank, world, config, peak, peak_kind)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch
        torch.distributed.destroy_process_group()


def _common(args, config, value, peak, peak_kind, r, dtype):
    return {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype, "data": "synthetic (seeded random KV, queries and logits; no model weights)",
            "config": config, "clocks": r["clocks"]}


def kernel_line(args, w, peak, peak_kind):
    """One kernel of the workload timed alone with CUDA events: the quantised
    or token-dropped draft attention of one layer, one resident
    verification layer, one acceptance call over the round's logits, or the
    GPU compression of one layer (quantiser and kept-row compaction)."""
    import torch
    from lossless_draft_verify_vc_b200 import synth, vc
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    vc.lib()
    B = w["B"]
    reps = max(args.steps, 3) * 10
    comp = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if args.kernel == "verify":
        rv = time_resident_verify_layer(w, dev, reps=reps)
        return {"kernel": "vc_verify_attn", "workload": args.workload, "us": rv["us_per_layer"],
                "gbps": rv["hbm_gbps"], "frac_of_hbm_peak": rv["hbm_gbps"] / peak, "tflops": rv["tflops"],
                "peak_kind": peak_kind, "calls": reps}
    if args.kernel == "compress":
        if "bits" not in w:
            return {"kernel": "vc_quantize_cache", "workload": args.workload,
                    "unavailable": "the workload's draft cache is token-dropped, not quantised"}
        kvs = [synth.kv_full(B, w["Hkv"], w["T"], w["D"], seed=s, device=dev) for s in (1, 2)]
        cp = time_compress(w, dev, {"kvs": kvs, "sh": vc.shape(B, w["Hq"], w["Hkv"], w["D"])})
        return {"kernel": "vc_quantize_cache + vc_compact_kept", "workload": args.workload,
                "quantize_us": cp["quantize_us"], "quantize_gbps": cp["quantize_gbps"],
                "quantize_frac_of_hbm_peak": cp["quantize_gbps"] / peak, "compact_us": cp["compact_us"],
                "compact_gbps": cp["compact_gbps"], "compact_frac_of_hbm_peak": cp["compact_gbps"] / peak,
                "flags": cp["flags"], "peak_kind": peak_kind}
    if args.kernel == "accept":
        K, V = w["K"], w["V"]
        dt = torch.bfloat16 if w["logits"] == "bf16" else torch.float32
        toks = synth.tokens((B, K), V, seed=3)
        lens = synth.geometric_accept_lengths(B, K, w["p_mismatch"], seed=3)
        lg = [synth.planted_logits(B, K, V, toks, lens, seed=4 + i, dtype=dt).to(dev) for i in range(4)]
        d = toks.to(dev)
        tgt = torch.empty(B, K + 1, dtype=torch.int32, device=dev)
        acc = torch.empty(B, dtype=torch.int32, device=dev)
        cor = torch.empty_like(acc)
        ws = vc.workspace(vc.vc_accept_workspace_size(B, K, V), dev)
        for i in range(5):
            vc.vc_accept(lg[i % 4], B, K, V, d, tgt, acc, cor, ws, comp)
        torch.cuda.synchronize(dev)
        assert acc.cpu().tolist() == lens
        e0.record(comp)
        for i in range(reps):
            vc.vc_accept(lg[i % 4], B, K, V, d, tgt, acc, cor, ws, comp)
        e1.record(comp)
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) * 1e3 / reps
        nb = B * (K + 1) * V * lg[0].element_size()
        return {"kernel": "vc_accept", "workload": args.workload, "us": us, "gbps": nb / us / 1e3,
                "frac_of_hbm_peak": nb / us / 1e3 / peak, "peak_kind": peak_kind, "calls": reps}
    # draft attention of one layer
    nl = 3
    sh = vc.shape(B, w["Hq"], w["Hkv"], w["D"])
    q = synth.normal((nl, B, w["Hq"], w["D"]), 7, dev)
    out = torch.empty(B, w["Hq"], w["D"], device=dev)
    if "bits" in w:
        caches = [vc.quant_cache(dict(synth.random_quant_cache(B, w["Hkv"], w["T"] - w["R"], w["R"], w["D"],
                                                               w["bits"], w["G"], seed=l, device=dev),
                                      flags=vc.VC_CACHE_STATIC)) for l in range(nl)]
        ws = vc.workspace(vc.vc_draft_attn_quant_workspace_size(sh, caches[0]), dev)
        call = lambda i: vc.vc_draft_attn_quant(sh, caches[i % nl], q[i % nl], out, ws, comp)
        nb, name = draft_bytes_per_layer(w), "vc_draft_attn_quant"
    else:
        keep = []
        caches = []
        for l in range(nl):
            k, v = synth.kv_full(B, w["Hkv"], w["n_keep"], w["D"], seed=40 + l, device=dev)
            idx = torch.arange(w["n_keep"], dtype=torch.int32, device=dev).expand(B, w["Hkv"], -1).contiguous()
            keep.append((k, v, idx))
            caches.append(vc.sparse_cache(k, v, idx))
        ws = vc.workspace(vc.vc_draft_attn_sparse_workspace_size(sh, caches[0]), dev)
        call = lambda i: vc.vc_draft_attn_sparse(sh, caches[i % nl], q[i % nl], out, ws, comp)
        nb, name = sparse_bytes_per_layer(w), "vc_draft_attn_sparse"
    for i in range(6):
        call(i)
    torch.cuda.synchronize(dev)
    e0.record(comp)
    for i in range(reps):
        call(i)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / reps
    return {"kernel": name, "workload": args.workload, "us": us, "gbps": nb / us / 1e3,
            "frac_of_hbm_peak": nb / us / 1e3 / peak, "peak_kind": peak_kind, "calls": reps}


def resident_verify_block(w, peak, peak_kind):
    """JSON block for one resident verification layer of a streamed workload."""
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    rv = time_resident_verify_layer(w, dev)
    tp, tk = read_tensor_peak()
    rv.update({"hbm_frac": rv["hbm_gbps"] / peak, "hbm_peak_kind": f"{peak_kind} hbm_gbs (burst copy)",
               "tensor_frac": rv["tflops"] / tp, "tensor_peak_tflops": tp,
               "tensor_peak_kind": f"{tk} bf16 dense (burst)",
               "note": "one layer of the workload's request with the full K and V in HBM, timed alone; flops = "
                       "4 nq Hq T D (the two products, algorithmic; the kernel runs P.V twice, as bf16 high and "
                       "low parts)"})
    return rv


def streamed_line(args, w, rank, world, config, peak, peak_kind):
    r = run_streamed(args, w, rank, world)
    K, NL = w["K"], w["NL"]
    db = sparse_bytes_per_layer(w)
    value = whole_job_rate(db * K * NL, args.steps, world, r["draft_ms"])
    achieved = db / (r["draft_ms"] * 1e3 / (K * NL * args.steps) * 1e-6) / 1e9
    vr_us = r["verify_ms"] * 1e3 / args.steps
    link = r["link_bytes"] / (vr_us * 1e-6) / 1e9
    line = _common(args, config, value, peak, peak_kind, r, "bf16 rows -> bf16 MMA, fp32 accumulate")
    line.update({
        "ms_per_step": r["total_ms"] / args.steps,
        "draft_frac_of_hbm_peak": value / world / peak,
        "verify_round_us": vr_us, "verify_link_gbps": link, "pcie_peak_gbps": r["pcie"],
        "verify_frac_of_pcie_peak": link / r["pcie"], "accept_us": r["accept_ms"] * 1e3 / args.steps,
        "phases_ms_per_step": {"draft": r["draft_ms"] / args.steps, "verify_streamed": vr_us / 1e3,
                               "accept": r["accept_ms"] / args.steps},
        "roofline": {"kernel": "vc_draft_attn_sparse (draft_sparse_kernel)", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs (burst copy)", "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None, "algorithmic_bytes_per_launch": db},
        "link_roofline": {"phase": "host-streamed verification", "bound": "pcie", "achieved": link,
                          "peak": r["pcie"], "peak_kind": "pinned host->device cudaMemcpyAsync of 1 GiB, measured "
                                                          "in this run", "unit": "GB/s",
                          "frac": link / r["pcie"], "bytes_per_round": r["link_bytes"]},
        # per step: K*NL token-drop draft calls and NL verify calls (each an
        # attention kernel + its chunk-merge kernel), one accept kernel
        "gpu_launches": (2 * K * NL + 2 * NL + 1) * args.steps,
        "verify_resident_layer": resident_verify_block(w, peak, peak_kind),
    })
    return line


def stagger_line(args, w, rank, world, config, peak, peak_kind):
    r = run_stagger(args, w, rank, world)
    K, NL, n = w["K"], w["NL"], w["n_req"]
    db = draft_bytes_per_layer(w)
    value = whole_job_rate(db * K * NL, 1, world, r["draft_ms"])
    lk, sg = r["sched"]["lockstep"], r["sched"]["stagger"]
    per = lambda st: st["elapsed_ms"] / st["rounds"]
    link_bytes_round = r["link_bytes_per_request"] * n
    line = _common(args, config, value, peak, peak_kind, r, "int4 codes + bf16 -> fp16/bf16 MMA, fp32 accumulate")
    line.update({
        "ms_per_step": per(sg),
        "draft_frac_of_hbm_peak": value / world / peak,
        "stagger": {"lockstep_ms_per_round": per(lk), "stagger_ms_per_round": per(sg),
                    "speedup": per(lk) / per(sg),
                    "link_busy_frac_stagger": sg["link_busy_ms"] / sg["elapsed_ms"],
                    "link_busy_frac_lockstep": lk["link_busy_ms"] / lk["elapsed_ms"],
                    "link_gbps_stagger": link_bytes_round / (per(sg) * 1e-3) / 1e9,
                    "pcie_peak_gbps": r["pcie"],
                    "verify_frac_of_pcie_peak_stagger": link_bytes_round / (per(sg) * 1e-3) / 1e9 / r["pcie"],
                    "rounds": sg["rounds"]},
        "roofline": {"kernel": "vc_draft_attn_quant (draft_quant_kernel)", "bound": "hbm",
                     "achieved": db / (r["draft_ms"] * 1e3 / (K * NL) * 1e-6) / 1e9, "peak": peak,
                     "peak_kind": f"{peak_kind} hbm_gbs (burst copy)", "unit": "GB/s",
                     "frac": db / (r["draft_ms"] * 1e3 / (K * NL) * 1e-6) / 1e9 / peak, "traffic": None,
                     "algorithmic_bytes_per_launch": db},
        "gpu_launches": 2 * K * NL,
        "verify_resident_layer": resident_verify_block(w, peak, peak_kind),
    })
    return line


def remote_line(args, w, rank, world, config, peak, peak_kind):
    r = run_remote(args, w, rank, world)
    K, NL, n = w["K"], w["NL"], w["n_req"]
    db = draft_bytes_per_layer(w)
    value = whole_job_rate(db * K * NL, 1, world, r["draft_ms"])
    lk, sg = r["sched"]["lockstep"], r["sched"]["stagger"]
    achieved = db / (r["draft_ms"] * 1e3 / (K * NL) * 1e-6) / 1e9
    local_bytes = r["link_bytes_per_request_round"] * n * r["rounds"]
    line = _common(args, config, value, peak, peak_kind, r, "int2 codes + bf16 -> fp16/bf16 MMA, fp32 accumulate")

    def pol(st):
        return {"ms_per_run": st["elapsed_ms"], "tokens_per_s": r["tokens_per_run"] / (st["elapsed_ms"] * 1e-3),
                "remote_gbps": r["fetch_bytes"] / (st["fetch_ms"] * 1e-3) / 1e9,
                "remote_busy_frac": st["fetch_ms"] / st["elapsed_ms"],
                "local_gbps_while_streaming": local_bytes / (st["link_busy_ms"] * 1e-3) / 1e9,
                "local_busy_frac": st["link_busy_ms"] / st["elapsed_ms"],
                "last_first_draft_ms": st["first_draft_ms"]}

    line.update({
        "ms_per_step": sg["elapsed_ms"],
        "draft_frac_of_hbm_peak": value / world / peak,
        "remote_prefix": {"lockstep": pol(lk), "stagger": pol(sg), "speedup": lk["elapsed_ms"] / sg["elapsed_ms"],
                          "remote_link_gbps_set": w["remote_gbps"], "local_link_gbps_set": w["local_gbps"],
                          "fetch_bytes": r["fetch_bytes"], "rounds_per_run": r["rounds"],
                          "tokens_per_run": r["tokens_per_run"],
                          "note": "one run = every request's compressed cache fetched over the remote link, then "
                                  "`rounds` draft/verify/accept rounds per request; tokens = accepted drafts + the "
                                  "correction per round (planted acceptance)"},
        "roofline": {"kernel": "vc_draft_attn_quant (draft_quant_kernel)", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs (burst copy)", "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None, "algorithmic_bytes_per_launch": db},
        # the timed draft loop: K * NL draft kernels
        "gpu_launches": K * NL,
    })
    return line


def layers_line(args, w, rank, world, config, peak, peak_kind):
    """The verification pass through NL decoder layers (vc_verify_layer) on
    random bf16 weights with the full KV resident: each layer reads its
    weights and its full K and V once."""
    import torch
    from lossless_draft_verify_vc_b200 import synth, vc
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    vc.lib()
    NL, B, Hq, Hkv, D, T, dm, dff = w["NL"], w["B"], w["Hq"], w["Hkv"], w["D"], w["T"], w["d_model"], w["d_ff"]
    nq = w["K"] + 1
    ls = vc.layer_shape(dm, dff, Hq, Hkv, D)
    g = torch.Generator(device=dev).manual_seed(1000 * rank + 5)

    def r(shape, s):
        return (torch.randn(shape, generator=g, device=dev) * s).to(torch.bfloat16)

    layers = []
    for _ in range(NL):
        W = dict(w1=(1 + 0.1 * torch.randn(dm, generator=g, device=dev)).to(torch.bfloat16),
                 w2=(1 + 0.1 * torch.randn(dm, generator=g, device=dev)).to(torch.bfloat16),
                 wqkv=r(((Hq + 2 * Hkv) * D, dm), dm ** -0.5), wo=r((dm, Hq * D), (Hq * D) ** -0.5),
                 wgu=r((2 * dff, dm), dm ** -0.5), wd=r((dm, dff), dff ** -0.5))
        k, v = synth.kv_full(B, Hkv, T, D, seed=len(layers), device=dev)
        layers.append((vc.layer_weights(W), W, k, v))
    x0 = synth.normal((B, nq, dm), 3, dev)
    x = x0.clone()
    ws = vc.workspace(vc.vc_verify_layer_workspace_size(ls, B, nq, T), dev)
    comp = torch.cuda.current_stream(dev)

    def one_pass():
        x.copy_(x0)
        for lw, _, k, v in layers:
            vc.vc_verify_layer(ls, lw, B, nq, T, x, k, v, ws, comp)

    for _ in range(args.warmup):
        one_pass()
    torch.cuda.synchronize(dev)
    assert torch.isfinite(x.float()).all()
    clocks = ClockSampler(dev.index)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for _ in range(args.steps):
        one_pass()
    e1.record(comp)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0] / args.steps
    wbytes = sum(t.numel() * t.element_size() for _, W, _, _ in layers for t in W.values())
    kvbytes = NL * 4 * T * Hkv * D * B
    value = (wbytes + kvbytes) * world / (ms * 1e-3) / 1e9
    line = _common(args, config, value, peak, peak_kind, dict(clocks=clk), "bf16 weights and KV, fp32 accumulate")
    line.update({
        "ms_per_step": ms,
        "note": "value = weight + full-KV bytes read per verification pass / pass time (GB/s); random weights, "
                "so tokens/s are comparable only in kind",
        "verify_pass": {"ms": ms, "tokens_verified_per_s": B * nq * world / (ms * 1e-3),
                        "weight_bytes": wbytes, "kv_bytes": kvbytes, "frac_of_hbm_peak": value / world / peak,
                        "layers": NL, "rows_per_request": nq},
        # per layer: 2 norms, rotary, attention + combine, convert, SwiGLU (+ 4 cuBLAS GEMMs)
        "gpu_launches": NL * 7 * args.steps,
    })
    return line


def resident_line(args, w, rank, world, config, peak, peak_kind):
    r = run_gpu(args, w, rank, world)
    K, NL = w["K"], w["NL"]
    db = draft_bytes_per_layer(w)
    vb = verify_bytes_per_layer(w)
    draft_bytes_step = db * K * NL
    value = whole_job_rate(draft_bytes_step, args.steps, world, r["draft_ms"])
    launches_draft = K * NL * args.steps
    avg_launch_us = r["draft_ms"] * 1e3 / launches_draft
    achieved = db / (avg_launch_us * 1e-6) / 1e9
    verify_round_us = r["verify_ms"] * 1e3 / args.steps
    verify_gbs = vb * NL / (verify_round_us * 1e-6) / 1e9
    e2e_value = whole_job_rate(draft_bytes_step, args.steps, world, r["e2e_draft_ms"])
    e2e_step_value = whole_job_rate(draft_bytes_step, args.steps, world, r["e2e_total_ms"])
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
                "draft_phase_host_ms_per_step": r["e2e_draft_ms"] / args.steps,
                "whole_step_host_ms": r["e2e_total_ms"] / args.steps,
                "whole_step_value": e2e_step_value,
                "note": "host wall clock through the C-ABI calls: value = draft bytes per step / (draft phase: "
                        "queries copied from pinned host memory, K x layers calls, output read back); "
                        "whole_step_* adds the verify-query, logits and draft-token copies, the verification "
                        "and acceptance calls and the read-back of target / accept length / correction"},
        # per step: K*NL quantised draft calls (one kernel each; units are
        # merged in-kernel), NL verify calls (attention kernel + its merge
        # kernel), one accept kernel
        "gpu_launches": (K * NL + 2 * NL + 1) * args.steps,
        "clocks": r["clocks"],
    }
    if r.get("compress"):
        cp = r["compress"]
        line["compress"] = {
            "note": "building one layer's draft caches on the GPU (vc_quantize_cache: full K/V -> group records "
                    "+ residual; vc_compact_kept: 25% kept rows -> pool); device time per call",
            "quantize_us": cp["quantize_us"], "quantize_gbps": cp["quantize_gbps"],
            "quantize_frac_of_hbm_peak": cp["quantize_gbps"] / peak, "quantize_bytes": cp["quantize_bytes"],
            "compact_us": cp["compact_us"], "compact_gbps": cp["compact_gbps"],
            "compact_frac_of_hbm_peak": cp["compact_gbps"] / peak, "compact_bytes": cp["compact_bytes"],
            "flags": cp["flags"]}
    if r.get("streamed"):
        sv = r["streamed"]
        line["verify_streamed"] = {"round_us": sv["round_us"], "link_gbps": sv["link_gbps"],
                                   "pcie_peak_gbps": sv["pcie_peak_gbps"],
                                   "frac_of_pcie_peak": sv["link_gbps"] / sv["pcie_peak_gbps"],
                                   "rounds": sv["rounds"], "host_pool_layers": sv["host_pool_layers"]}
    if rank == 0 and world == 1:
        gbs, n, el, threads, per_slice = oracle_sample(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"{n} x (request 0, KV head 0) of one layer ({per_slice} bytes each) "
                                          f"in {el:.1f} s"}
    return line


if __name__ == "__main__":
    main()
