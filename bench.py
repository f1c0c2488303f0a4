"""Benchmark: 8B-shaped batch-1 decode on the persistent megakernel (one B200 per rank).

Workload (one "step" = one decode step = one launch of the megakernel): Llama-3-8B-shaped
decoder (32 layers, hidden 4096, 32/8 heads x 128, SwiGLU 14336, vocab 128256), seeded
random bf16 weights N(0, 0.02) (16 GB), a 39-token seeded prompt prefilled into the bf16
KV cache, then greedy decode with the next token fed back on the device.  W warm-up steps
and K timed steps follow the prompt, so positions 39 .. 39+W+K-1 are decoded (the default
W=8, K=504 is the 512-step run of that workload).  The weights stream from HBM every step
(15 GB > the 126 MB L2), so no L2 flush is needed between steps.

Other workloads of the same decoder family (`--workload`, each printing its own line; the
default is the one above): `llama8b-ctx4096` (8B shape, batch 1, every step attending over
4096+ cached positions), `chameleon7b-b1` / `-b4` / `-b16` (Chameleon-7B-shaped MHA
decoder, 1, 4 or 16 sequences each at 1024+ cached positions; 16 sequences run the
projections on the tensor cores) and `chameleon7b-qk-b1` / `-b16` (the same with QK-norm).  Their caches are seeded synthetic values standing in for
the prefilled prompts.

Multi-GPU (torchrun, one process per GPU): independent replicas, no collective on the data
path; the timed region is bracketed by a barrier and a device synchronise on every rank and
the slowest rank's time is reported.  `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode ms/token + achieved HBM GB/s (% of peak), 8B-shape bs=1, 1 B200"
PROMPT_LEN = 39
CALIBRATION_STEPS = 6  # untimed decode steps that measure the per-SM schedule (model setup)
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# name: (shape name, sequences, cached positions before decoding (0 = prefill the 39-token prompt))
WORKLOADS = {
    "llama8b": ("LLAMA8B", 1, 0),
    "llama8b-ctx4096": ("LLAMA8B", 1, 4096),
    "chameleon7b-b1": ("CHAMELEON7B", 1, 1024),
    "chameleon7b-b4": ("CHAMELEON7B", 4, 1024),
    "chameleon7b-b4-cuda": ("CHAMELEON7B", 4, 1024),  # the same on the width-4 CUDA-core GEMV
    "chameleon7b-b16": ("CHAMELEON7B", 16, 1024),
    "chameleon7b-qk-b1": ("CHAMELEON7B_QK", 1, 1024),
    "chameleon7b-qk-b16": ("CHAMELEON7B_QK", 16, 1024),
    "attention": (None, 0, 0),  # the standalone decode-attention op, Mirage size
}
WORKLOAD_TEXT = {
    "llama8b": "llama3-8b-shape decode, batch 1, 39-token prompt, greedy",
    "llama8b-ctx4096": "llama3-8b-shape decode, batch 1, 4096 cached positions (synthetic), greedy",
    "chameleon7b-b1": "chameleon-7b-shape MHA decode, batch 1, 1024 cached positions (synthetic), greedy",
    "chameleon7b-b4": "chameleon-7b-shape MHA decode, batch 4 (tensor-core projections), 1024 cached positions "
                      "each (synthetic), greedy",
    "chameleon7b-b4-cuda": "chameleon-7b-shape MHA decode, batch 4 (width-4 CUDA-core GEMV), 1024 cached positions "
                           "each (synthetic), greedy",
    "chameleon7b-b16": "chameleon-7b-shape MHA decode, batch 16 (tensor-core projections), 1024 cached positions "
                       "each (synthetic), greedy",
    "chameleon7b-qk-b1": "chameleon-7b-shape MHA decode with QK-norm (LayerNorm per q/k head before RoPE), "
                         "batch 1, 1024 cached positions (synthetic), greedy",
    "chameleon7b-qk-b16": "chameleon-7b-shape MHA decode with QK-norm, batch 16 (tensor-core projections), "
                          "1024 cached positions each (synthetic), greedy",
    "attention": "standalone decode attention O = softmax(Q.K).V, fp16 Q [64,1,128], K^T [64,128,4096], "
                 "V [64,4096,128], fp32 out, 3 rotating input copies",
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=504)
    p.add_argument("--warmup", type=int, default=8)
    p.add_argument("--impl", default="mk", choices=["mk", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=64)
    p.add_argument("--no-calibrate", action="store_true",
                   help="keep equal rows per SM instead of the schedule calibrated on untimed steps before "
                        "the warm-up")
    p.add_argument("--workload", default="llama8b", choices=sorted(WORKLOADS))
    p.add_argument("--dispatch", default="static", choices=["static", "claim", "claim-paced", "claim-priority"],
                   help="scheduling variant: fixed per-SM queues (default), or projection tasks claimed "
                        "at run time from per-op pools (batch-1 kernel only)")
    p.add_argument("--tasks-per-sm", type=int, default=2, help="pool tasks per SM and projection (--dispatch claim)")
    p.add_argument("--layers", type=int, default=0,
                   help="truncate the decoder to this many layers (profiling captures of a small case); "
                        "0 = the full 32-layer workload")
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, dev, world: int) -> float:
    """The largest of every rank's x (the slowest replica's time); x itself on one rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(shape, positions):
    """Bytes one decode step must read from HBM: every weight once (projections, norms, LM
    head, QK-norm gains and biases), one embedding row, and the K/V actually attended
    (positions 0..p inclusive)."""
    s = shape
    D = s.head_dim
    per_layer = ((s.n_q_heads + 2 * s.n_kv_heads) * D * s.hidden + s.hidden * s.n_q_heads * D
                 + 2 * s.ffn * s.hidden + s.hidden * s.ffn + 2 * s.hidden) * 2
    if getattr(s, "qk_norm", False):
        per_layer += 2 * (s.n_q_heads + s.n_kv_heads) * D * 2
    weights = s.n_layers * per_layer + (s.vocab * s.hidden + s.hidden) * 2 + s.hidden * 2
    kv = [s.n_layers * 2 * s.n_kv_heads * (p + 1) * D * 2 for p in positions]
    return weights, kv


def workload_metric(name):
    if name == "llama8b":
        return METRIC
    return f"decode ms/step + achieved HBM GB/s (% of peak), {name}, 1 B200"


def kernel_source_hash():
    src = os.path.join(ROOT, "persistent_megakernel_decode_04_b200", "csrc", "mk_decode.cu")
    with open(src, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(per_step_alg_bytes):
    """DRAM bytes per launch from the committed ncu summary, scaled to this launch's
    algorithmic bytes; None if the summary is missing or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", "decode_kernel_llama8b_traffic.txt")
    try:
        kv = {}
        for line in open(path):
            if "=" in line and not line.startswith("#"):
                k, v = line.split("=", 1)
                kv[k.strip()] = v.strip()
        if kv.get("kernel_source_sha256_16") != kernel_source_hash():
            return None, "kernel changed since the ncu capture"
        ratio = float(kv["dram_bytes"]) / float(kv["algorithmic_bytes"])
        return ratio * per_step_alg_bytes, kv.get("how", "")
    except Exception:
        return None, "no ncu summary"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu=uuid,{self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        mhz, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            if self.uuid and parts[0] != self.uuid:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------------------------- CPU oracle

def oracle_ms_per_token(weights_full, shape, budget_s=15.0, max_steps=32):
    """Time the CPU oracle on a bounded sample of the same workload: full 32-layer decode
    steps of the 8B shape after a 39-position cache (seeded synthetic values standing in for
    the prefilled prompt), greedy, until `budget_s` of CPU time or `max_steps` steps."""
    import mk_inputs as mi
    import oracle
    d = oracle.Decoder(weights_full, 1, PROMPT_LEN + max_steps + 2)
    d.set_cache(mi.kv_cache_values(0, shape, 1, PROMPT_LEN, sigma=1.0), PROMPT_LEN)
    tok = np.array([1], dtype=np.int32)
    t0 = time.perf_counter()
    n = 0
    while True:
        tok = np.array([oracle.argmax(d.decode(tok)[0])], dtype=np.int32)
        n += 1
        if n >= 3 and (time.perf_counter() - t0 > budget_s or n >= max_steps):
            break
    dt = (time.perf_counter() - t0) / n
    cores = int(os.environ.get("OR_THREADS", os.cpu_count() or 1))
    return dt * 1e3, cores, n


# ------------------------------------------------------------------------------- arms

def run_reference(args, rank, world):
    """The reference arm: the CPU oracle on the same workload (the 8B shape, all 32 layers,
    the 39-token prompt prefilled untimed, then greedy decode), W untimed and K timed steps,
    each step one full oracle decode step.  Rank 0 only."""
    if rank != 0:
        return
    import mk_inputs as mi
    import oracle
    shape = mi.LLAMA8B
    t = time.perf_counter()
    w = mi.make_weights(shape, seed=0)
    d = oracle.Decoder(w, 1, PROMPT_LEN + args.warmup + args.steps + 1)
    rl = d.prefill(mi.prompt(0, 0, PROMPT_LEN, shape.vocab))
    tok = np.array([oracle.argmax(rl[0])], dtype=np.int32)
    for _ in range(args.warmup):
        tok = np.array([oracle.argmax(d.decode(tok)[0])], dtype=np.int32)
    setup_s = time.perf_counter() - t
    t0 = time.perf_counter()
    for _ in range(args.steps):
        tok = np.array([oracle.argmax(d.decode(tok)[0])], dtype=np.int32)
    ms = (time.perf_counter() - t0) / args.steps * 1e3
    cores = int(os.environ.get("OR_THREADS", os.cpu_count() or 1))
    sample = (f"{args.steps} full 32-layer oracle decode steps of the 8B shape after the 39-token prompt "
              f"(prefilled untimed), greedy, measured")
    out = {"impl": "reference", "metric": METRIC, "value": ms, "unit": "ms/token", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded random weights)",
           "config": {"workload": "llama3-8b-shape decode, batch 1, 39-token prompt, greedy",
                      "prompt_len": PROMPT_LEN, "parallelism": "replicas", "weights": "bf16"},
           "cpu_baseline": {"value": ms, "unit": "ms/token", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": ms, "unit": "ms/token", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "setup_s": setup_s}
    print(json.dumps(out), flush=True)


def run_attention(args, rank, world, local):
    """The standalone decode-attention op at the Mirage size: one call per step, inputs rotated
    over three seeded copies (3 x 134 MB > L2) so no call finds its K/V in L2."""
    import torch
    import mk_inputs as mi
    import persistent_megakernel_decode_04_b200 as mk
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    BH, D, L = 64, 128, 4096
    sets = []
    for c in range(3):
        q, kt, v = (torch.from_numpy(mi.normal_f16(c, i + 1, shape).view(np.int16)).to(dev)
                    for i, shape in enumerate(((BH, D), (BH, D, L), (BH, L, D))))
        sets.append((q, kt, v))
    o = torch.empty((BH, D), dtype=torch.float32, device=dev)
    ws = torch.zeros(mk.mk_attention_workspace_bytes(BH, D, L), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for i in range(args.warmup):
        q, kt, v = sets[i % 3]
        mk.mk_attention_decode(q, kt, v, o, BH, D, L, 1.0, ws)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clk:
        start.record(stream)
        for i, (a, b) in enumerate(ev):
            q, kt, v = sets[i % 3]
            a.record(stream)
            mk.mk_attention_decode(q, kt, v, o, BH, D, L, 1.0, ws)
            b.record(stream)
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if mk.mk_attention_status(ws, BH, D, L) != mk.MK_OK:
        raise SystemExit("attention reported an error status")
    us = np.array([a.elapsed_time(b) for a, b in ev]) * 1e3
    total_us = start.elapsed_time(stop) * 1e3 / args.steps
    alg = BH * L * D * 2 * 2 + BH * D * 2 + BH * D * 4  # K and V once, q, o
    peak, peak_kind = measured_peaks()
    achieved = alg / (us.mean() * 1e-6) / 1e9
    # end to end: host inputs (pinned) copied in and o copied out every call
    hq, hk, hv = (t.cpu().pin_memory() for t in sets[0])
    ho = torch.empty_like(o, device="cpu").pin_memory()
    q, kt, v = sets[0]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, min(args.e2e_steps, 16))
    e0.record(stream)
    for _ in range(n_e2e):
        q.copy_(hq, non_blocking=True)
        kt.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        mk.mk_attention_decode(q, kt, v, o, BH, D, L, 1.0, ws)
        ho.copy_(o, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if rank == 0:
        out = {"metric": "standalone decode attention us/call + achieved HBM GB/s, Mirage size, 1 B200",
               "value": float(us.mean()), "unit": "us/call", "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": float(us.mean()) / 1e3, "higher_is_better": False,
               "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic (seeded N(0,1))",
               "config": {"workload": WORKLOAD_TEXT["attention"], "BH": BH, "head_dim": D, "keys": L,
                          "l2": "3 rotating input copies (402 MB > L2)"},
               "us_p50": float(np.median(us)), "us_per_call_back_to_back": total_us,
               "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                            "frac": achieved / peak, "traffic": None, "peak_kind": peak_kind,
                            "algorithmic_bytes_per_launch": alg},
               "e2e": {"value": e0.elapsed_time(e1) * 1e3 / n_e2e, "unit": "us/call",
                       "h2d_bytes_per_step": (BH * D + 2 * BH * L * D) * 2, "d2h_bytes_per_step": BH * D * 4,
                       "steps": n_e2e},
               "gpu_launches": args.steps, "clocks": clk.summary()}
        print(json.dumps(out), flush=True)


def run_mk(args, rank, world, local):
    import torch
    import torch.distributed as dist
    import mk_inputs as mi
    import persistent_megakernel_decode_04_b200 as mk

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600),
                                device_id=dev)
    shape_name, B, ctx0 = WORKLOADS[args.workload]
    base = getattr(mi, shape_name)
    shape = base if args.layers <= 0 else base.with_layers(args.layers)
    calib_steps = 0 if (args.no_calibrate or args.dispatch != "static") else CALIBRATION_STEPS
    total_steps = calib_steps + args.warmup + args.steps
    max_seq = (ctx0 or PROMPT_LEN) + total_steps + args.e2e_steps + 8
    os.environ.setdefault("MK_INPUT_THREADS", str(max(1, (os.cpu_count() or 1) // max(1, world))))
    weights = mi.make_weights(shape, seed=0)
    stream = torch.cuda.current_stream(dev)
    cfg = mk.Config.from_shape(shape, B, max_seq)
    if args.workload.endswith("-cuda"):
        cfg.tc_min_batch = 5  # batches up to 4 on the CUDA-core GEMV
    m = mk.Megakernel(cfg, weights, local, stream=stream)
    info = m.info()
    cpu_baseline = rank == 0 and not args.no_cpu_baseline and args.workload == "llama8b"
    if not cpu_baseline:
        del weights
    if ctx0 == 0:
        prompt = torch.from_numpy(mi.prompt(0, 0, PROMPT_LEN, shape.vocab)[None].astype(np.int32)).to(dev)
        logits = m.prefill(prompt)
        tok = torch.argmax(logits[0]).to(torch.int32).reshape(1)
    else:
        # seeded synthetic cache standing in for the prefilled prompts, filled layer by layer
        gen = torch.Generator(device=dev)
        gen.manual_seed(1234)
        kvv = m.kv_view()
        for l in range(shape.n_layers):
            vals = torch.randn((2, B, shape.n_kv_heads, ctx0, shape.head_dim), generator=gen, device=dev)
            kvv[l, :, :B, :, :ctx0, :] = vals.to(torch.bfloat16).view(torch.int16)
            del vals
        m.set_positions([ctx0] * B)
        tok = torch.from_numpy(mi.prompt(0, 0, B, shape.vocab).astype(np.int32)).to(dev)
    calibrated = False
    if args.dispatch != "static":  # pools are cut in equal shares: no per-SM calibration
        m.set_dispatch({"claim": mk.MK_DISPATCH_CLAIM, "claim-paced": mk.MK_DISPATCH_CLAIM_PACED,
                        "claim-priority": mk.MK_DISPATCH_CLAIM_PRIORITY}[args.dispatch], args.tasks_per_sm)
    elif calib_steps:
        # the schedule: per-SM streaming speed measured on untimed traced decode steps
        # (3 rounds x 2 steps) and every projection's rows re-partitioned, before the warm-up
        m.calibrate(tok, steps=2, rounds=3)
        calibrated = True
    for _ in range(args.warmup):
        _, nt = m.decode(tok)
        tok = nt.clone()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    pos0 = m.positions()[0]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(uuid) as clk:
        start.record(stream)
        for a, b in ev:
            a.record(stream)
            _, nt = m.decode(tok)
            b.record(stream)
            tok = nt  # next step reads this step's greedy token on the device
        stop.record(stream)
        torch.cuda.synchronize(dev)
    status = m.sync_status()
    if status != mk.MK_OK:
        raise SystemExit(f"decode reported status {status}: {mk.mk_last_error(m.ctx)}")
    elapsed_ms = start.elapsed_time(stop)
    step_ms = np.array([a.elapsed_time(b) for a, b in ev])
    max_ms = max_over_ranks(elapsed_ms, dev, world)
    if world > 1:
        dist.barrier()

    # end to end through the C ABI with host buffers: token in from pinned host memory,
    # logits and next token back to pinned host memory, every step
    host_tok = torch.zeros(B, dtype=torch.int32, pin_memory=True)
    host_logits = torch.empty((B, shape.vocab), dtype=torch.float32, pin_memory=True)
    host_next = torch.zeros(B, dtype=torch.int32, pin_memory=True)
    dev_tok = torch.zeros(B, dtype=torch.int32, device=dev)
    host_tok.copy_(tok.cpu())
    m.set_positions([pos0 + args.steps] * B)
    n_e2e = min(args.e2e_steps, max_seq - (pos0 + args.steps) - 1)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        dev_tok.copy_(host_tok, non_blocking=True)
        lg, nt = m.decode(dev_tok)
        host_logits.copy_(lg, non_blocking=True)
        host_next.copy_(nt, non_blocking=True)
        stream.synchronize()
        host_tok.copy_(host_next)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_max = max_over_ranks(e0.elapsed_time(e1), dev, world)
    if m.sync_status() != mk.MK_OK:
        raise SystemExit("decode reported an error in the end-to-end loop")

    if rank == 0:
        positions = list(range(pos0, pos0 + args.steps))
        wbytes, kvbytes = algorithmic_bytes(shape, positions)
        alg = wbytes + B * float(np.mean(kvbytes))  # every sequence attends over its own cache
        mean_ms = float(step_ms.mean())
        peak, peak_kind = measured_peaks()
        achieved = alg / (mean_ms * 1e-3) / 1e9
        traffic, traffic_note = (profiled_traffic(alg) if args.workload == "llama8b" and args.dispatch == "static"
                                 else (None, "no ncu summary"))
        # whole job: slowest rank's time over all ranks' steps (replicas decode concurrently)
        value = max_ms / (args.steps * world)
        out = {
            "metric": workload_metric(args.workload), "value": value,
            "unit": "ms/token" if B == 1 else "ms/step", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded random weights)",
            "config": {"workload": WORKLOAD_TEXT[args.workload]
                                   + ("" if args.layers <= 0 else f" (truncated to {args.layers} layers)"),
                       "prompt_len": PROMPT_LEN if ctx0 == 0 else None, "cached_positions": ctx0 or None,
                       "decode_positions": [pos0, pos0 + args.steps - 1], "batch_per_gpu": B,
                       "global_batch": world * B, "parallelism": "replicas", "weights": "bf16",
                       "schedule": (f"run-time claims from per-op pools, {args.tasks_per_sm} tasks per SM"
                                    + (", paced by the workers" if args.dispatch == "claim-paced" else "")
                                    + (", attention chunks claimed first (priority)"
                                       if args.dispatch == "claim-priority" else "")
                                    if args.dispatch != "static" else
                                    f"calibrated per-SM rows ({calib_steps} untimed calibration steps "
                                    f"before the warm-up)" if calibrated else "equal rows per SM"),
                       "l2": "inputs larger than L2 (15 GB of weights streamed per step)"},
            "ms_per_step_p50": float(np.median(step_ms)), "tokens_per_s": 1e3 / (max_ms / args.steps) * world * B,
            "hbm_gbs": achieved, "hbm_frac_of_measured": achieved / peak, "hbm_frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
            "bound_ms_at_8tbs": alg / NOMINAL_HBM_GBS / 1e6,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": alg, "traffic_note": traffic_note},
            "e2e": {"value": (e2e_max / n_e2e) if n_e2e > 0 else None, "unit": "ms/token" if B == 1 else "ms/step",
                    "h2d_bytes_per_step": 4 * B, "d2h_bytes_per_step": B * (shape.vocab * 4 + 4), "steps": n_e2e},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
            "kernel": {"n_sms": info["n_sms"], "n_tasks": info["n_tasks"], "smem_bytes": info["smem_bytes"]},
        }
        if cpu_baseline:
            ms, cores, n = oracle_ms_per_token(weights, shape)
            out["cpu_baseline"] = {
                "value": ms, "unit": "ms/token", "cores": cores, "kind": "oracle",
                "sample": f"{n} full 32-layer oracle decode steps of the 8B shape after a 39-position "
                          f"synthetic cache, greedy, measured (about 15 s of CPU time)"}
        print(json.dumps(out), flush=True)
    m.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.gpus != world and world == 1 and args.gpus > 1:
        print(json.dumps({"error": f"--gpus {args.gpus} needs torchrun with {args.gpus} processes"}))
        sys.exit(2)
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.workload == "attention":
        run_attention(args, rank, world, local)
    else:
        run_mk(args, rank, world, local)


if __name__ == "__main__":
    main()
