#!/usr/bin/env python
"""Benchmark of the gated delta rule token mixer on B200.

Headline: gdr_fwd on the layer-shaped workload (B=4, T=4096, H=16,
dk=dv=128, bf16 q/k/v/o, fp32 gates and state, random S0), throughput in
Mtok/s (tokens = B*T, all heads).  One step = one gdr_fwd call, i.e. one pass
of the whole chunkwise forward (staging, cumulative decay, decay-masked
beta K K^T, triangular solve, W/U products, sequential state pass, outputs,
final state) over one batch.  Inputs are synthetic (seeded), resident in HBM
before the timed region, and larger than the 126 MB L2 (q, k, v alone are
201 MB), so no L2 flush is needed between steps.

Also reported on the same JSON line: the roofline of the forward kernel, the
end-to-end number through the public API with host buffers, the oracle's CPU
throughput, clocks sampled during the timed region, the number of kernels
launched, and secondary measurements of the decode step (HBM roofline),
the backward and the Gated DeltaNet-2 forward.

Multi-GPU (torchrun): the (batch, head) units are independent, so every
rank runs its own batch with no collective on the data path (weak scaling);
time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference there is for
this method) on the host cores, on rank 0.
"""
import argparse
import json
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "gated-delta-rule fwd Mtok/s (H16,128×128,T4K,bf16); % TC peak; decode % HBM BW"
WORKLOAD = "layer_fwd"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-secondary", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--profile-bwd", metavar="B,T,H", default=None,
                   help="only run gdr_bwd twice on seeded bf16 d=128 inputs of this shape "
                        "(a short command for profilers) and exit")
    p.add_argument("--profile-gdn2", metavar="B,T,H", default=None,
                   help="only run gdr2_fwd twice on seeded bf16 d=128 inputs of this shape and exit")
    p.add_argument("--profile-fwd", metavar="B,T,H", default=None,
                   help="only run gdr_fwd twice on seeded bf16 d=128 inputs of this shape and exit "
                        "(long sequences over few heads take the parallel-segment path)")
    p.add_argument("--profile-gdn2-bwd", metavar="B,T,H", default=None,
                   help="only run gdr2_bwd twice on seeded bf16 d=128 inputs of this shape and exit")
    p.add_argument("--profile-step", action="store_true",
                   help="only run gdr_step three times on the decode workload (B256 H16 d128 bf16, "
                        "268 MB fp32 state) and exit")
    p.add_argument("--profile-block-bwd", metavar="B,T,H", default=None,
                   help="only run the block prologue backward (K=4) three times on seeded bf16 d=128 "
                        "inputs of this shape and exit")
    p.add_argument("--profile-block", metavar="B,T,H", default=None,
                   help="only run the block prologue (K=4) and epilogue twice each on seeded bf16 "
                        "d=128 inputs of this shape and exit")
    return p.parse_args()


def profile_fwd(shape):
    """Two gdr_fwd calls on the seeded layer recipe (bf16, d = 128, S0 = 0),
    then a status check."""
    import gated_delta_rule_91_b200 as gdr
    B, T, H = (int(x) for x in shape.split(","))
    x = synth.gdr_inputs(B, T, H, 128, 128, "bf16", seed=1)
    d = {n: x[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")}
    for _ in range(2):
        gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None)
    torch.cuda.synchronize()
    gdr.check_status()
    print(json.dumps({"profile_fwd": shape, "status": "ok"}))


def profile_step():
    """Three decode steps on the decode workload's state and first inputs,
    then a status check."""
    import gated_delta_rule_91_b200 as gdr
    w = synth.WORKLOADS["decode"]
    S = synth.decode_state(w.B, w.H, w.dk, w.dv, w.seed).cuda()
    x = {n: t.cuda() for n, t in synth.decode_step_inputs(w.B, w.H, w.dk, w.dv, w.dtype, w.seed, 0).items()}
    for _ in range(3):
        gdr.gdr_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
    torch.cuda.synchronize()
    gdr.check_status()
    print(json.dumps({"profile_step": "decode", "status": "ok"}))


def profile_gdn2_bwd(shape):
    """Two Gated DeltaNet-2 backward calls on the seeded GDN-2 recipe (bf16,
    d = 128, S0 ~ N(0, 0.02), dO ~ N(0, 1) seeded 7), then a status check."""
    import gated_delta_rule_91_b200 as gdr
    B, T, H = (int(x) for x in shape.split(","))
    x = synth.gdr2_inputs(B, T, H, 128, 128, "bf16", seed=4, s0_std=0.02)
    d = {n: (x[n].cuda() if x[n] is not None else None) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}
    dO = torch.randn(d["q"].shape, generator=torch.Generator().manual_seed(7)).to(d["q"].dtype).cuda()
    for _ in range(2):
        gdr.gdr2_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], dO)
    torch.cuda.synchronize()
    gdr.check_status()
    print(json.dumps({"profile_gdn2_bwd": shape, "status": "ok"}))


def profile_block(shape):
    """Two block prologue calls (ShortConv K=4, SiLU, q/k L2) and two block
    epilogue calls (RMSNorm, SiLU gate) on the seeded block recipe, bf16,
    d = 128, then a status check."""
    import gated_delta_rule_91_b200 as gdr
    B, T, H = (int(x) for x in shape.split(","))
    px = {n: (t.cuda() if t is not None else None)
          for n, t in synth.block_prologue_inputs(B, T, H, 128, 128, 4, "bf16", seed=21, state=False).items()}
    ex = {n: (t.cuda() if t is not None else None)
          for n, t in synth.block_epilogue_inputs(B, T, H, 128, "bf16", seed=22).items()}
    for _ in range(2):
        gdr.gdr_block_prologue(px["xq"], px["xk"], px["xv"], px["wq"], px["wk"], px["wv"], px["bq"],
                               px["bk"], px["bv"], eps=1e-6)
    for _ in range(2):
        gdr.gdr_block_epilogue(ex["o"], ex["g"], ex["weight"], 1e-6)
    torch.cuda.synchronize()
    gdr.check_status()
    print(json.dumps({"profile_block": shape, "status": "ok"}))


def profile_block_bwd(shape):
    """Three block prologue backward calls (ShortConv K=4, SiLU, q/k L2) on
    the bench's seeded inputs (bf16, d = 128, dy ~ N(0, 1) seeded 25), then a
    status check."""
    import gated_delta_rule_91_b200 as gdr
    B, T, H = (int(x) for x in shape.split(","))
    d, K = 128, 4
    px = {n: (t.cuda() if t is not None else None)
          for n, t in synth.block_prologue_inputs(B, T, H, d, d, K, "bf16", seed=21, state=False).items()}
    pg = torch.Generator().manual_seed(25)
    dys = [torch.randn(B, T, H, d, generator=pg).to(torch.bfloat16).cuda() for _ in range(3)]
    ws = torch.empty(gdr.lib().gdr_block_prologue_bwd_workspace_bytes(H, d, d, K), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        gdr.gdr_block_prologue_bwd(px["xq"], px["xk"], px["xv"], px["wq"], px["wk"], px["wv"], *dys,
                                   px["bq"], px["bk"], px["bv"], eps=1e-6, workspace=ws)
    torch.cuda.synchronize()
    gdr.check_status()
    print(json.dumps({"profile_block_bwd": shape, "status": "ok"}))


def profile_gdn2(shape):
    """Two Gated DeltaNet-2 forward calls on the seeded GDN-2 recipe
    (bf16, d = 128, S0 ~ N(0, 0.02)), then a status check."""
    import gated_delta_rule_91_b200 as gdr
    B, T, H = (int(x) for x in shape.split(","))
    x = synth.gdr2_inputs(B, T, H, 128, 128, "bf16", seed=4, s0_std=0.02)
    d = {n: (x[n].cuda() if x[n] is not None else None) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}
    for _ in range(2):
        gdr.gdr2_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    torch.cuda.synchronize()
    gdr.check_status()
    print(json.dumps({"profile_gdn2": shape, "status": "ok"}))


def profile_bwd(shape):
    """Two backward calls on seeded layer-recipe inputs (bf16, d = 128,
    S0 ~ N(0, 0.02), dO drawn with the inputs), then a status check."""
    import gated_delta_rule_91_b200 as gdr
    B, T, H = (int(x) for x in shape.split(","))
    x = synth.gdr_inputs(B, T, H, 128, 128, "bf16", seed=1, s0_std=0.02, with_dO=True)
    d = {n: (x[n].cuda() if x[n] is not None else None)
         for n in ("q", "k", "v", "log_alpha", "beta", "S0", "dO")}
    for _ in range(2):
        gdr.gdr_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"])
    torch.cuda.synchronize()
    gdr.check_status()
    print(json.dumps({"profile_bwd": shape, "status": "ok"}))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# ---------------------------------------------------------------------------
# workload arithmetic: algorithmic bytes and FLOPs per launch -- what the
# algorithm must read, write and compute, the units the roofline divides by
# ---------------------------------------------------------------------------
def fwd_bytes(B, T, H, dk, dv, esize=2, with_s0=True, with_st=True):
    per_tok_head = 2 * dk * esize + dv * esize + 8 + dv * esize   # q,k,v in; gates; o out
    state = B * H * dv * dk * 4 * (int(with_s0) + int(with_st))
    return B * T * H * per_tok_head + state


def fwd_flops(B, T, H, dk, dv, C=64):
    # 2*dk*dv per token for each of W S^T, Q S^T and the state update (=6 dk dv)
    # plus 2*C per token for each of K K^T, Q K^T (dk), U^g, P U (dv) and W (dk)
    return B * T * H * (6 * dk * dv + 2 * C * (3 * dk + 2 * dv))


def bwd_flops(B, T, H, d, C=64):
    return B * T * H * (12 * d * d + 20 * C * d + 4 * C * C)


def step_bytes(B, H, dk, dv, esize=2):
    return 2 * B * H * dv * dk * 4 + B * H * (2 * dk + dv) * esize + 2 * B * H * 4 + B * H * dv * esize


def gdr2_bytes(B, T, H, dk, dv, esize=2):
    per = 2 * dk * esize + dv * esize + 4 * dk + 4 * dk + 4 * dv + dv * esize
    return B * T * H * per + 2 * B * H * dv * dk * 4


def step2_bytes(B, H, dk, dv, esize=2):
    """Gated DeltaNet-2 decode step: the fp32 state read and written, q, k,
    v and o, and the per-channel gates log alpha, b (dk) and w (dv) in fp32."""
    return (2 * B * H * dv * dk * 4 + (2 * dk + 2 * dv) * B * H * esize
            + (2 * dk + dv) * B * H * 4)


def prologue_bytes(B, T, H, dk, dv, K, esize=2):
    """Block prologue: read xq, xk, xv and write q, k, v once, plus the fp32
    conv taps and biases (the conv state is not used on this workload)."""
    elems = B * T * H * (2 * dk + dv)
    return 2 * elems * esize + H * (2 * dk + dv) * (K + 1) * 4


def epilogue_bytes(B, T, H, dv, esize=2):
    """Block epilogue: read o and g, write y; the fp32 norm weight."""
    return 3 * B * T * H * dv * esize + dv * 4


def prologue_bwd_bytes(B, T, H, dk, dv, K, esize=2):
    """Block prologue backward: read x and dy of the three streams, write dx;
    the fp32 taps and biases in, their gradients out."""
    C = H * (2 * dk + dv)
    return 3 * B * T * C * esize + 2 * C * (K + 1) * 4


def epilogue_bwd_bytes(B, T, H, dv, esize=2):
    """Block epilogue backward: read o, g and dy, write do and dg; the fp32
    weight in and dweight out."""
    return 5 * B * T * H * dv * esize + 2 * dv * 4


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.5)  # let the sampler come up before the timed region

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, begin):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        inside = [s for t, s in self.samples if self.t0 - 0.05 <= t <= self.t1 + 0.15]
        used = inside if inside else [s for _, s in self.samples][-3:]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for s in used:
            parts = [p.strip() for p in s.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(used),
                "samples_in_timed_region": len(inside)}


# ---------------------------------------------------------------------------
def shard_seed(base_seed, rank):
    """Each rank draws its own batch (independent (b, h) units, weak scaling)."""
    return base_seed + 7919 * rank


def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device="cuda"):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def traffic_from_profile(kernel_tag):
    """DRAM bytes per launch recorded in profiles/<kernel_tag>.md, if the
    recorded kernel source hash matches the current source; else None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", kernel_tag + ".md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    src = fields.get("kernel_source")
    sha = fields.get("kernel_source_sha256")
    tb = fields.get("traffic_bytes_per_launch")
    if not (src and sha and tb):
        return None
    h = hashlib.sha256()
    for rel in src.split(","):
        p = os.path.join(ROOT, rel.strip())
        if not os.path.exists(p):
            return None
        with open(p, "rb") as f:
            h.update(f.read())
    if h.hexdigest() != sha:
        return None
    return float(tb)


def workload_config(world):
    """The `config` object of both arms' JSON lines (identical by construction)."""
    w = synth.WORKLOADS[WORKLOAD]
    return {"workload": WORKLOAD, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
            "io_dtype": "bf16", "gates_state_dtype": "f32", "S0": "N(0,0.02)",
            "l2": "inputs_exceed_l2 (q,k,v 201 MB > 126 MB L2); no flush",
            "parallelism": "dp%d (independent (b,h) shards, no collective)" % world}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _np(x):
    return {n: (t.double().numpy() if t is not None else None) for n, t in x.items()}


def _time_oracle(fn, min_s=0.0):
    """Run fn once (at least once, repeated until min_s seconds); seconds per run."""
    reps, t0 = 0, time.time()
    while True:
        fn()
        reps += 1
        if time.time() - t0 >= min_s:
            break
    return (time.time() - t0) / reps, reps


def cpu_baseline(w):
    """The fp64 oracle on the host cores: the headline workload (repeated for
    10 s), and once each the other workloads' oracle work -- the tiny fp32
    workload and the Gated DeltaNet-2 workload in full, all 1024 decode steps,
    the long workload's forward at full length and its backward on the first
    2048 tokens (tokens/s of that slice)."""
    import oracle
    a = _np(synth.workload_inputs(WORKLOAD))
    dt, reps = _time_oracle(lambda: oracle.gdr_fwd(a["q"], a["k"], a["v"], a["log_alpha"], a["beta"], a["S0"]),
                            10.0)
    per = {}
    wt = synth.WORKLOADS["tiny_f32"]
    t = _np(synth.workload_inputs("tiny_f32"))
    s, r = _time_oracle(lambda: oracle.gdr_fwd(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], t["S0"]), 1.0)
    per["tiny_f32"] = {"tok_per_s": wt.B * wt.T / s, "s_per_run": s, "runs": r}
    w4 = synth.WORKLOADS["gdn2_fwd"]
    g = _np(synth.workload_inputs("gdn2_fwd"))
    s, r = _time_oracle(lambda: oracle.gdr2_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["S0"]))
    per["gdn2_fwd"] = {"tok_per_s": w4.B * w4.T / s, "s_per_run": s, "runs": r}
    del g
    # decode: the 1024 steps' inputs are drawn outside the timed loop, 64 at a time
    wd = synth.WORKLOADS["decode"]
    S = synth.decode_state(wd.B, wd.H, wd.dk, wd.dv, wd.seed).double().numpy()
    spent = 0.0
    for c0 in range(0, wd.steps, 64):
        xs = [_np(synth.decode_step_inputs(wd.B, wd.H, wd.dk, wd.dv, wd.dtype, wd.seed, st))
              for st in range(c0, min(c0 + 64, wd.steps))]
        t0 = time.time()
        for xx in xs:
            oracle.gdr_step_inplace(xx["q"], xx["k"], xx["v"], xx["log_alpha"], xx["beta"], S)
        spent += time.time() - t0
    per["decode"] = {"tok_per_s": wd.B * wd.steps / spent, "s_total": spent, "steps": wd.steps}
    del S
    wl = synth.WORKLOADS["long_fwd_bwd"]
    l = _np(synth.workload_inputs("long_fwd_bwd"))
    s, r = _time_oracle(lambda: oracle.gdr_fwd(l["q"], l["k"], l["v"], l["log_alpha"], l["beta"], l["S0"]))
    per["long_fwd"] = {"tok_per_s": wl.B * wl.T / s, "s_per_run": s, "runs": r}
    Ts = 2048
    sl = {n: (v[:, :Ts].copy() if v is not None and v.ndim >= 3 else v) for n, v in l.items()}
    s, r = _time_oracle(lambda: oracle.gdr_bwd(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], None,
                                               sl["dO"], None))
    per["long_bwd_T2048_slice"] = {"tok_per_s": wl.B * Ts / s, "s_per_run": s, "runs": r,
                                   "note": "backward on the first 2048 tokens (all 16 heads); the full "
                                           "65,536 tokens would take about 32x as long"}
    return {"value": w.B * w.T / dt / 1e6, "unit": "Mtok/s", "cores": oracle.num_threads(),
            "cpu_model": cpu_model(), "kind": "oracle",
            "sample": "the full workload B=%d T=%d H=%d d=%d, run %d time(s) back to back, "
                      "fp64 sequential recurrence, OpenMP over (b,h)" % (w.B, w.T, w.H, w.dk, reps),
            "per_workload": per}


def run_reference(args, rank, world):
    """fp64 CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    w = synth.WORKLOADS[WORKLOAD]
    x = synth.workload_inputs(WORKLOAD)
    a = {n: (x[n].double().numpy() if x[n] is not None else None) for n in x}

    def step(i):
        b = i % w.B
        S0 = a["S0"][b:b + 1] if a["S0"] is not None else None
        oracle.gdr_fwd(a["q"][b:b + 1], a["k"][b:b + 1], a["v"][b:b + 1],
                       a["log_alpha"][b:b + 1], a["beta"][b:b + 1], S0)

    for i in range(args.warmup):
        step(i)
    t0 = time.time()
    for i in range(args.steps):
        step(i)
    dt = (time.time() - t0) / args.steps
    value = w.T / dt / 1e6
    sample = "one batch element (b = step mod %d) of the workload per step: T=%d, all %d heads" % (
        w.B, w.T, w.H)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Mtok/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(world),
            "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": oracle.num_threads(),
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def secondary(pk):
    """Decode step, backward and Gated DeltaNet-2 forward (one GPU, rank 0)."""
    import gated_delta_rule_91_b200 as gdr
    out = {}
    ev = lambda: torch.cuda.Event(enable_timing=True)

    # decode: B256 H16 d128, state 268 MB read + written per step
    w = synth.WORKLOADS["decode"]
    S = synth.decode_state(w.B, w.H, w.dk, w.dv, w.seed).cuda()
    xs = [synth.decode_step_inputs(w.B, w.H, w.dk, w.dv, w.dtype, w.seed, t) for t in range(8)]
    xs = [{n: t.cuda() for n, t in x.items()} for x in xs]
    o = torch.empty(w.B, w.H, w.dv, dtype=torch.bfloat16, device="cuda")
    for i in range(5):
        x = xs[i % 8]
        gdr.gdr_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, o=o)
    n = 100
    e0, e1 = ev(), ev()
    torch.cuda.synchronize()
    e0.record()
    for i in range(n):
        x = xs[i % 8]
        gdr.gdr_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, o=o)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / n
    gbs = step_bytes(w.B, w.H, w.dk, w.dv) / (us * 1e-6) / 1e9
    out["decode"] = {"workload": "decode B=256 H=16 d=128 bf16", "us_per_step": us,
                     "tok_per_s": w.B / (us * 1e-6), "achieved_gbs": gbs,
                     "hbm_frac": gbs / pk["hbm_gbs"]}
    del S, xs

    # Gated DeltaNet-2 decode on the same shape (per-channel gates, b in (0, 1))
    S = synth.decode_state(w.B, w.H, w.dk, w.dv, w.seed).cuda()
    x2 = synth.gdr2_inputs(w.B, 8, w.H, w.dk, w.dv, "bf16", seed=w.seed)
    xs2 = [{n: x2[n][:, t].contiguous().cuda() for n in ("q", "k", "v", "log_alpha", "b", "w")} for t in range(8)]
    call2 = lambda x: gdr.gdr2_step(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], S, o=o)
    for i in range(5):
        call2(xs2[i % 8])
    e0, e1 = ev(), ev()
    torch.cuda.synchronize()
    e0.record()
    for i in range(n):
        call2(xs2[i % 8])
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / n
    gbs = step2_bytes(w.B, w.H, w.dk, w.dv) / (us * 1e-6) / 1e9
    out["gdn2_decode"] = {"workload": "GDN-2 decode B=256 H=16 d=128 bf16", "us_per_step": us,
                          "tok_per_s": w.B / (us * 1e-6), "achieved_gbs": gbs, "hbm_frac": gbs / pk["hbm_gbs"]}
    del S, xs2

    # backward at full length T=65536 (timed only when the backward is built)
    w = synth.WORKLOADS["long_fwd_bwd"]
    x = synth.workload_inputs("long_fwd_bwd")
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    try:
        reps = 3
        t0 = ev(); t1 = ev(); t2 = ev()
        gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])  # warm-up
        gdr.gdr_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"])
        torch.cuda.synchronize()
        t0.record()
        for _ in range(reps):
            gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
        t1.record()
        for _ in range(reps):
            gdr.gdr_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["dO"])
        t2.record()
        torch.cuda.synchronize()
        fms, bms = t0.elapsed_time(t1) / reps, t1.elapsed_time(t2) / reps
        out["long_fwd_bwd"] = {
            "workload": "B=1 T=65536 H=16 d=128 bf16",
            "fwd_ms": fms, "bwd_ms": bms,
            "fwd_tc_frac": fwd_flops(w.B, w.T, w.H, w.dk, w.dv) / (fms * 1e-3) / (pk["bf16_tflops"] * 1e12),
            "bwd_tc_frac": bwd_flops(w.B, w.T, w.H, w.dk) / (bms * 1e-3) / (pk["bf16_tflops"] * 1e12)}
    except Exception as e:  # backward not built yet
        out["long_fwd_bwd"] = {"unavailable": str(e).splitlines()[0][:200]}
    del d, x

    # Gated DeltaNet-2 forward
    w = synth.WORKLOADS["gdn2_fwd"]
    x = synth.workload_inputs("gdn2_fwd")
    d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    try:
        call = lambda: gdr.gdr2_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
        call()
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        e0.record()
        for _ in range(5):
            call()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 5
        out["gdn2_fwd"] = {"workload": "B=4 T=4096 H=16 d=128 bf16", "ms": ms,
                           "mtok_per_s": w.B * w.T / (ms * 1e-3) / 1e6,
                           "tc_frac": fwd_flops(w.B, w.T, w.H, w.dk, w.dv) / (ms * 1e-3) / (pk["bf16_tflops"] * 1e12),
                           "hbm_frac": gdr2_bytes(w.B, w.T, w.H, w.dk, w.dv) / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
        # the same workload with the erase gate in (0, 2) (negative-eigenvalue range)
        d["b"].mul_(2.0)
        call()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(5):
            call()
        e1.record()
        torch.cuda.synchronize()
        ms2 = e0.elapsed_time(e1) / 5
        out["gdn2_fwd_b_0_2"] = {"workload": "B=4 T=4096 H=16 d=128 bf16, b in (0, 2)", "ms": ms2,
                                 "mtok_per_s": w.B * w.T / (ms2 * 1e-3) / 1e6}
        # Gated DeltaNet-2 backward on the same workload (dO ~ N(0, 1), dS_T = 0)
        d["b"].mul_(0.5)
        dO = torch.randn(d["q"].shape, generator=torch.Generator().manual_seed(7)).to(d["q"].dtype).cuda()
        bcall = lambda: gdr.gdr2_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], dO)
        bcall()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(3):
            bcall()
        e1.record()
        torch.cuda.synchronize()
        bms = e0.elapsed_time(e1) / 3
        out["gdn2_bwd"] = {"workload": "B=4 T=4096 H=16 d=128 bf16", "ms": bms,
                           "mtok_per_s": w.B * w.T / (bms * 1e-3) / 1e6,
                           "tc_frac": bwd_flops(w.B, w.T, w.H, w.dk) / (bms * 1e-3) / (pk["bf16_tflops"] * 1e12),
                           "kernels": "cluster recompute; tensor-core dS pass (dL/dS in TMEM); tensor-core per-chunk products, chain rule and dlog alpha suffix sums; CUDA-core paths only for chunks decaying past e^20"}
    except Exception as e:
        out["gdn2_fwd"] = {"unavailable": str(e).splitlines()[0][:200]}
    del d, x
    out.update(block_lines(pk))
    out.update(seq_split_line())
    return out


def seq_split_line(R=8):
    """One rank's share of the long sequence (B1 T65536 H16 d128 bf16) split
    into R segments: both forward passes of its 8192-token segment, the
    combine as the last rank (R - 1 segment maps) and the output correction.
    The all-gather of (M, N) is not timed on one GPU; its size is reported."""
    import gated_delta_rule_91_b200 as gdr
    x = synth.workload_inputs("long_fwd_bwd")
    T = x["q"].shape[1]
    Ts = T // R
    d = {n: x[n][:, :Ts].contiguous().cuda() for n in ("q", "k", "v", "log_alpha", "beta")}
    B, _, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    M_all = torch.zeros(R, B, H, dk, dk, device="cuda")
    N_all = torch.zeros(R, B, H, dv, dk, device="cuda")

    def rank_work():
        o0, qt, N, M = gdr.gdr_seg_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"])
        S_in, _ = gdr.gdr_seg_combine(M_all, N_all, R - 1, None, want_final=True)
        gdr.gdr_seg_fixup(qt, S_in, o0)

    for _ in range(2):
        rank_work()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        rank_work()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 3
    return {"seq_split_8": {"workload": "B=1 T=65536 H=16 d=128 bf16 split into %d segments of %d tokens" % (R, Ts),
                            "rank_ms": ms, "exchange_bytes_per_rank": (dk * dk + dv * dk) * 4 * B * H,
                            "note": "per-rank device time without the all-gather; the unsplit forward is long_fwd_bwd.fwd_ms"}}


def block_lines(pk):
    """The block's prologue (ShortConv, SiLU, q/k L2) and epilogue (RMSNorm,
    SiLU gate) on the layer workload, alone and around the forward."""
    import gated_delta_rule_91_b200 as gdr
    out = {}
    B, T, H, d, K = 4, 4096, 16, 128, 4
    px = {n: (t.cuda() if t is not None else None)
          for n, t in synth.block_prologue_inputs(B, T, H, d, d, K, "bf16", seed=21, state=False).items()}
    ex = {n: (t.cuda() if t is not None else None)
          for n, t in synth.block_epilogue_inputs(B, T, H, d, "bf16", seed=22).items()}
    gx = {n: (t.cuda() if t is not None else None)
          for n, t in synth.gdr_inputs(B, T, H, d, d, "bf16", seed=23).items()}
    q, k, v = (torch.empty(B, T, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    o = torch.empty_like(q)
    y = torch.empty_like(q)
    pro = lambda: gdr.gdr_block_prologue(px["xq"], px["xk"], px["xv"], px["wq"], px["wk"], px["wv"],
                                         px["bq"], px["bk"], px["bv"], eps=1e-6, q=q, k=k, v=v)
    epi = lambda oo: gdr.gdr_block_epilogue(oo, ex["g"], ex["weight"], 1e-6, y=y)
    mix = lambda: gdr.gdr_fwd(q, k, v, gx["log_alpha"], gx["beta"], gx["S0"], o=o)

    def timed(fn, reps=20):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    us_p = timed(pro) * 1e3
    gbs_p = prologue_bytes(B, T, H, d, d, K) / (us_p * 1e-6) / 1e9
    out["block_prologue"] = {"workload": "B=4 T=4096 H=16 dk=dv=128 bf16, ShortConv K=4 + SiLU + q/k L2",
                             "us": us_p, "achieved_gbs": gbs_p, "hbm_frac": gbs_p / pk["hbm_gbs"]}
    pg = torch.Generator().manual_seed(25)
    dys = [torch.randn(B, T, H, d, generator=pg).to(torch.bfloat16).cuda() for _ in range(3)]
    pws = torch.empty(gdr.lib().gdr_block_prologue_bwd_workspace_bytes(H, d, d, K), dtype=torch.uint8,
                      device="cuda")
    pro_bwd = lambda: gdr.gdr_block_prologue_bwd(px["xq"], px["xk"], px["xv"], px["wq"], px["wk"], px["wv"],
                                                 *dys, px["bq"], px["bk"], px["bv"], eps=1e-6, workspace=pws)
    us_pb = timed(pro_bwd) * 1e3
    gbs_pb = prologue_bwd_bytes(B, T, H, d, d, K) / (us_pb * 1e-6) / 1e9
    out["block_prologue_bwd"] = {"workload": "B=4 T=4096 H=16 dk=dv=128 bf16, backward of ShortConv K=4 + SiLU "
                                             "+ q/k L2 (dx, dw, dbias; 2 launches)",
                                 "us": us_pb, "achieved_gbs": gbs_pb, "hbm_frac": gbs_pb / pk["hbm_gbs"]}
    us_e = timed(lambda: epi(ex["o"])) * 1e3
    gbs_e = epilogue_bytes(B, T, H, d) / (us_e * 1e-6) / 1e9
    out["block_epilogue"] = {"workload": "B=4 T=4096 H=16 dv=128 bf16, RMSNorm + SiLU gate",
                             "us": us_e, "achieved_gbs": gbs_e, "hbm_frac": gbs_e / pk["hbm_gbs"]}
    dy = torch.randn(B, T, H, d, generator=torch.Generator().manual_seed(24)).to(torch.bfloat16).cuda()
    ws = torch.empty(gdr.lib().gdr_block_epilogue_bwd_workspace_bytes(d), dtype=torch.uint8, device="cuda")
    us_b = timed(lambda: gdr.gdr_block_epilogue_bwd(ex["o"], ex["g"], ex["weight"], dy, 1e-6, workspace=ws)) * 1e3
    gbs_b = epilogue_bwd_bytes(B, T, H, d) / (us_b * 1e-6) / 1e9
    out["block_epilogue_bwd"] = {"workload": "B=4 T=4096 H=16 dv=128 bf16, backward of RMSNorm + SiLU gate "
                                             "(do, dg, dweight; 2 launches)",
                                 "us": us_b, "achieved_gbs": gbs_b, "hbm_frac": gbs_b / pk["hbm_gbs"]}

    def chain():
        pro()
        mix()
        epi(o)

    ms = timed(chain, reps=10)
    out["block_mixer_fwd"] = {"workload": "B=4 T=4096 H=16 d=128 bf16: prologue -> gdr_fwd -> epilogue",
                              "ms": ms, "mtok_per_s": B * T / (ms * 1e-3) / 1e6}
    return out


def main():
    args = parse_args()
    if args.profile_bwd:
        profile_bwd(args.profile_bwd)
        return
    if args.profile_gdn2:
        profile_gdn2(args.profile_gdn2)
        return
    if args.profile_block:
        profile_block(args.profile_block)
        return
    if args.profile_block_bwd:
        profile_block_bwd(args.profile_block_bwd)
        return
    if args.profile_gdn2_bwd:
        profile_gdn2_bwd(args.profile_gdn2_bwd)
        return
    if args.profile_fwd:
        profile_fwd(args.profile_fwd)
        return
    if args.profile_step:
        profile_step()
        return
    rank, world, local = dist_init(args)
    if args.impl == "reference":
        run_reference(args, rank, world)  # no process group: rank 0 alone works
        return

    import gated_delta_rule_91_b200 as gdr

    torch.cuda.set_device(local)
    pk = peaks()
    w = synth.WORKLOADS[WORKLOAD]
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    x = synth.gdr_inputs(B, T, H, dk, dv, w.dtype, seed=shard_seed(w.seed, rank), s0_std=w.s0_std)
    d = {n: x[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    o = torch.empty(B, T, H, dv, dtype=torch.bfloat16, device="cuda")
    ST = torch.empty(B, H, dv, dk, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        gdr.gdr_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], o=o, S_T=ST)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier(world)
    torch.cuda.synchronize()
    n0 = gdr.launch_count()
    clocks.mark(True)
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    barrier(world)
    launches = gdr.launch_count() - n0
    clk = clocks.stop()
    total_ms = evs[0].elapsed_time(evs[-1])
    per_launch = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(total_ms, world)
    ms_step = total_ms / args.steps
    value = world * B * T / (ms_step * 1e-3) / 1e6

    # roofline of the forward kernel (one launch per step)
    avg_launch_s = sum(per_launch) / len(per_launch) * 1e-3
    nbytes = fwd_bytes(B, T, H, dk, dv)
    nflops = fwd_flops(B, T, H, dk, dv)
    achieved = nbytes / avg_launch_s / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / pk["hbm_gbs"], "traffic": traffic_from_profile("gdr_fwd_layer_fwd"),
            "algorithmic_bytes_per_launch": nbytes, "peak_source": pk["source"],
            "tensor": {"achieved_tflops": nflops / avg_launch_s / 1e12,
                       "peak_tflops": pk["bf16_tflops"],
                       "frac": nflops / avg_launch_s / 1e12 / pk["bf16_tflops"],
                       "algorithmic_flops_per_launch": nflops}}

    # end to end through the public API with host buffers
    h = {n: x[n].pin_memory() for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    sh = torch.empty(ST.shape, dtype=ST.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h.values())
    d2h = oh.numel() * oh.element_size() + sh.numel() * sh.element_size()

    # one batch element at a time on two streams, so element b+1's upload
    # overlaps element b's forward and download (the copy engines run both
    # directions at once); every call is the public gdr_fwd on a batch slice
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]

    def e2e_step():
        start = torch.cuda.Event()
        start.record(stream)
        done = []
        for bi in range(B):
            sb = streams[bi % 2]
            sb.wait_event(start)
            with torch.cuda.stream(sb):
                for n in h:
                    if h[n] is not None:
                        d[n][bi].copy_(h[n][bi], non_blocking=True)
                gdr.gdr_fwd(d["q"][bi:bi + 1], d["k"][bi:bi + 1], d["v"][bi:bi + 1],
                            d["log_alpha"][bi:bi + 1], d["beta"][bi:bi + 1],
                            d["S0"][bi:bi + 1] if d["S0"] is not None else None,
                            o=o[bi:bi + 1], S_T=ST[bi:bi + 1])
                oh[bi].copy_(o[bi], non_blocking=True)
                sh[bi].copy_(ST[bi], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(sb)
                done.append(ev)
        for ev in done:
            stream.wait_event(ev)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ea.elapsed_time(eb) / args.e2e_steps, world)
    e2e = {"value": world * B * T / (e2e_ms * 1e-3) / 1e6, "unit": "Mtok/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    extra = None
    if rank == 0 and world == 1 and not args.no_secondary:
        del h, oh, sh
        extra = secondary(pk)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "Mtok/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": workload_config(world),
                "roofline": roof, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
                "cpu_baseline": cpu, "secondary": extra}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
