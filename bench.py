#!/usr/bin/env python
"""Benchmark of the VQ3R hot path on B200.

One step = one pass of the whole path over a 64-expert MoE layer
(w1, w3: 2048 x 7168; w2: 7168 x 2048 per expert, bf16, Student-t(4) rows
with log-normal row factors; 2.82 G weights):
  encode (row scale + greedy 3-stage assignment), repack of the indices into
  the tiled GEMV layout, decode to fp32, relative Frobenius error of each
  matrix, and the MoE decode step (8 active experts: gate/up and down GEMV
  of all 8 experts in one grouped call, B = 1).
Each matrix kind of the layer is stacked into one call.  The decode step
rotates over the 8 disjoint 8-expert groups of the layer so that its 132 MB
of indices per step come from HBM, not L2 (the layer's 5.6 GB of weights
exceed L2 as well).

Prints one JSON line (rank 0).  --impl reference times the CPU oracle on a
bounded sample of the same workload instead.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth import workloads as wl  # noqa: E402

METRIC = "VQ3R encode Gweights/s (vs fp32 peak); decode-GEMV GB/s vs HBM roofline, 1 B200"
# The definition's work: 3 stages x 256 codewords x 8 dims x (sub, mul, add) / 8 weights.
FLOPS_PER_WEIGHT = 2304
VQ4P_FLOPS_PER_WEIGHT = 768  # 4 stages x 64 codewords x 8 dims x (sub, mul, add) / 8 weights
# What the encoder executes: a screening pass per (vector, codeword) of 8 fused multiply-adds on the FP32 pipe
# and 5 ALU-pipe operations of bookkeeping (max and min for the second smallest, a compare, two selects), plus
# the definition's scan for the rare vectors whose margin test fails.  The ALU pipe (64 lanes per SM) bounds it.
ALU_OPS_PER_VEC_CODEWORD = 5
ENC_ALU_OPS_PER_WEIGHT = 3 * 256 * ALU_OPS_PER_VEC_CODEWORD / 8  # 480
ALU_LANES_PER_SM = 64
# DRAM bytes (read + write) per weight of the encode kernel: dram__bytes_read.sum + dram__bytes_write.sum of the
# ncu capture in profiles/encode_kernel_moe-layer-8-experts.md (117.4 M weights).  Set to None when the encode
# kernel changes, until it is captured again.
ENCODE_DRAM_BYTES_PER_WEIGHT = (235115264 + 8597760) / 117440512
SM_COUNT_NOMINAL = 148
FP32_LANES_PER_SM = 128


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="vq3r", choices=["vq3r", "reference"])
    ap.add_argument("--experts", type=int, default=64)
    ap.add_argument("--gemv-iters", type=int, default=200)
    ap.add_argument("--gemm-iters", type=int, default=10,
                    help="timed calls of the prefill product (8 experts' w1, 512 tokens each); 0 skips it")
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep-experts", type=int, default=256,
                    help="experts of the scale-sweep workload (Student-t(3) with 0.1%% outliers at 20 sigma) whose "
                         "encode and decode-GEMV are measured after the timed step; 0 skips it")
    ap.add_argument("--no-expert-quality", action="store_true",
                    help="skip the single-expert quality table (VQ3R beside the oracle's rtn4-row)")
    return ap.parse_args()


def load_codebooks(name):
    """Codebooks written by tests/golden/make_codebooks.py (hex float32 text)."""
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", "codebooks_%s.txt" % name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            rows.append([int(t, 16) for t in line.split()])
    return np.array(rows, dtype=np.uint32).view(np.float32).reshape((4, 64, 8) if name.startswith("vq4p_") else (3, 256, 8))


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("sm_max_mhz", 1965.0)), "measured"
    except Exception:
        return 6650.0, 1965.0, "fallback"


def bf16_peak():
    """Measured dense bf16 tensor throughput (burst), else the fallback figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
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
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- workload

def layer_gemv_bytes(B, experts):
    """Algorithmic bytes of one GEMV call over the stacked matrices of every expert of the layer."""
    total = 0
    for k in (wl.W1, wl.W3, wl.W2):
        rows, cols = wl.mat_shape(k)
        total += experts * (3 * rows * cols // 8 + 2 * rows + 4 * B * rows) + 2 * B * cols
    return total


def moe_step_bytes(B, n_exp=8):
    """Algorithmic bytes of one MoE decode step: index planes, scales, x, y."""
    gu_rows, gu_cols = wl.mat_shape(wl.W1)
    dn_rows, dn_cols = wl.mat_shape(wl.W2)
    idx = n_exp * (2 * 3 * gu_rows * gu_cols // 8 + 3 * dn_rows * dn_cols // 8)
    scales = n_exp * 2 * (2 * gu_rows + dn_rows)
    x = 2 * B * gu_cols + 2 * n_exp * B * dn_cols
    y = 4 * B * n_exp * (2 * gu_rows + dn_rows)
    return idx + scales + x + y


class Layer:
    """The layer on one GPU: inputs, outputs, workspaces and the step."""

    def __init__(self, torch, vq, dev, experts, expert0, B_list):
        self.torch, self.vq, self.dev = torch, vq, dev
        self.E = experts
        seed, dist = wl.LAYER["seed"], wl.expert_dist()
        stream = torch.cuda.current_stream().cuda_stream
        self.cb = torch.from_numpy(load_codebooks("layer")).to(dev)
        self.kinds = (wl.W1, wl.W3, wl.W2)
        self.W, self.idx, self.sc, self.dec, self.err, self.err_ws, self.tiles = {}, {}, {}, {}, {}, {}, {}
        for k in self.kinds:
            rows, cols = wl.mat_shape(k)
            W = torch.empty((experts * rows, cols), dtype=torch.bfloat16, device=dev)
            for e in range(experts):
                synth.fill_rows_device(W[e * rows:(e + 1) * rows].data_ptr(), cols, 0, rows, seed,
                                       wl.tag(expert0 + e, k), dist, stream=stream)
            self.W[k] = W
            self.idx[k] = torch.empty((3, experts * rows, cols // 8), dtype=torch.uint8, device=dev)
            self.tiles[k] = torch.empty(vq.vq3r_tiles_size(experts * rows, cols), dtype=torch.uint8, device=dev)
            self.sc[k] = torch.empty(experts * rows, dtype=torch.int16, device=dev)
            self.dec[k] = torch.empty((experts * rows, cols), dtype=torch.float32, device=dev)
            self.err[k] = torch.empty(1, dtype=torch.float64, device=dev)
            self.err_ws[k] = torch.empty(vq.vq3r_rel_frobenius_workspace_size(experts * rows, cols),
                                         dtype=torch.uint8, device=dev)
        self.weights = sum(self.W[k].numel() for k in self.kinds)
        # decode-step inputs and outputs per batch size
        self.groups = max(1, experts // 8)
        self.moe = {}
        for B in B_list:
            xu = torch.empty((B, wl.HIDDEN), dtype=torch.bfloat16, device=dev)
            synth.fill_rows_device(xu.data_ptr(), wl.HIDDEN, 0, B, wl.ACT_SEED, wl.tag(0, wl.X_GATEUP),
                                   synth.normal(), stream=stream)
            xd = torch.empty((8, B, wl.INTER), dtype=torch.bfloat16, device=dev)
            for j in range(8):
                synth.fill_rows_device(xd[j].data_ptr(), wl.INTER, 0, B, wl.ACT_SEED, wl.tag(j, wl.X_DOWN),
                                       synth.normal(), stream=stream)
            plans = []
            for g in range(self.groups):
                ex = [g * 8 + j for j in range(min(8, experts))]
                p1, p2 = [], []
                for j, e in enumerate(ex):
                    for k in (wl.W1, wl.W3):
                        rows, cols = wl.mat_shape(k)
                        p1.append(dict(idx=self.tiles[k], scales=self.sc[k], codebooks=self.cb, x=xu, row0=e * rows,
                                       rows=rows, layout="tiles", cols=cols,
                                       y=torch.empty((B, rows), dtype=torch.float32, device=dev)))
                    rows, cols = wl.mat_shape(wl.W2)
                    p2.append(dict(idx=self.tiles[wl.W2], scales=self.sc[wl.W2], codebooks=self.cb, x=xd[j],
                                   row0=e * rows, rows=rows, layout="tiles", cols=cols,
                                   y=torch.empty((B, rows), dtype=torch.float32, device=dev)))
                # the whole step (gate/up and down of the 8 experts) is one grouped call
                d = vq._descs(p1 + p2)
                plans.append((d, len(p1) + len(p2), p1 + p2, vq.lib().vq3r_gemv_workspace_size(d, len(p1) + len(p2), B)))
            wsz = max(p[3] for p in plans)
            ws = torch.zeros(wsz, dtype=torch.uint8, device=dev)
            self.moe[B] = (plans, ws, xu, xd)
        self._gemv_calls = {}

    # --- the parts of a step (each enqueues on the current stream) ---

    def encode(self):
        for k in self.kinds:
            self.encode_kind(k)

    def encode_kind(self, k):
        self.vq.vq3r_encode(self.W[k], self.cb, self.idx[k], self.sc[k])

    def pack(self):
        for k in self.kinds:
            self.vq.vq3r_pack_tiles(self.idx[k], out=self.tiles[k])

    def decode(self):
        for k in self.kinds:
            self.vq.vq3r_decode(self.idx[k], self.sc[k], self.cb, out=self.dec[k])

    def errors(self):
        for k in self.kinds:
            self.vq.vq3r_rel_frobenius_error(self.W[k], self.idx[k], self.sc[k], self.cb, out=self.err[k],
                                             workspace=self.err_ws[k])

    def gemv(self, B, group):
        # the C call with its arguments bound once per batch size (on the stream current at that time, the
        # default stream everywhere in this script): the decode step takes about 30 us, so per-call Python work
        # (a stream object, tensor attributes) would otherwise starve the GPU
        call = self._gemv_calls.get(B)
        if call is None:
            plans, ws, _, _ = self.moe[B]
            fn, s = self.vq.lib().vq3r_gemv, self.torch.cuda.current_stream().cuda_stream
            wp, wn = ws.data_ptr(), ws.numel()
            args = [p[:2] for p in plans]
            err = self.vq.VQ3RError

            def call(g):
                d, n = args[g % len(args)]
                st = fn(d, n, B, 1, wp, wn, s)
                if st:
                    raise err(st, "vq3r_gemv")
            self._gemv_calls[B] = call
        call(group)

    def layer_gemv_plan(self, B):
        """One grouped call over the stacked w1, w3, w2 of every expert of the layer (shared x per kind):
        the steady-state rate of the GEMV kernel, with the per-call start and reduction amortised."""
        _, _, xu, xd = self.moe[B]
        mats = []
        for k in self.kinds:
            rows, cols = wl.mat_shape(k)
            mats.append(dict(idx=self.tiles[k], scales=self.sc[k], codebooks=self.cb, x=xu if cols == wl.HIDDEN else xd[0],
                             rows=self.E * rows, layout="tiles", cols=cols,
                             y=self.torch.empty((B, self.E * rows), dtype=self.torch.float32, device=self.dev)))
        d = self.vq._descs(mats)
        ws = self.torch.zeros(self.vq.lib().vq3r_gemv_workspace_size(d, len(mats), B), dtype=self.torch.uint8,
                              device=self.dev)
        return d, len(mats), ws, mats

    def layer_gemv(self, plan, B):
        d, n, ws, _ = plan
        st = self.vq.lib().vq3r_gemv(d, n, B, 1, ws.data_ptr(), ws.numel(), self.torch.cuda.current_stream().cuda_stream)
        if st:
            raise self.vq.VQ3RError(st, "vq3r_gemv")

    LAUNCHES_PER_STEP = 3 * 2 + 3 + 3 * 1 + 3 * 2 + 1  # encode, pack, decode, error, gemv (kernels)


def bench_config(experts):
    """The workload both arms report (the reference arm times bounded row samples of it)."""
    rows_w13, cols_w13 = wl.mat_shape(wl.W1)
    rows_w2, cols_w2 = wl.mat_shape(wl.W2)
    return {"workload": "moe-layer-64x3-bf16: encode + tile repack + decode(fp32) + rel-Frobenius of the layer, "
                        "then moe-decode-step-8-experts GEMV (B=1)",
            "experts_per_gpu": experts, "weights_per_gpu": experts * (2 * rows_w13 * cols_w13 + rows_w2 * cols_w2),
            "matrices": "w1,w3 2048x7168; w2 7168x2048 per expert, stacked per kind",
            "l2": "inputs larger than L2 (5.6 GB layer); GEMV rotates 8 disjoint 8-expert groups (1.06 GB of indices)"}


def errs_plain_w1(layer):
    return float(layer.err[wl.W1].item())


# ----------------------------------------------------------------------------- CPU oracle sample

def cpu_oracle_sample(seconds, experts=64):
    """Time the oracle (as it stands) on a bounded row sample of the same layer:
    encode + decode + error + GEMV of sampled rows of each matrix kind."""
    import oracle
    seed, dist = wl.LAYER["seed"], wl.expert_dist()
    cb = load_codebooks("layer")
    rng = np.random.default_rng(0)

    def run(nrows):
        t_work, n_w = 0.0, 0
        for k in (wl.W1, wl.W3, wl.W2):
            rows, cols = wl.mat_shape(k)
            picks = rng.integers(0, experts * rows, size=nrows)
            W = np.stack([synth.fill_row_list(cols, [r % rows], seed, wl.tag(int(r // rows), k), dist)[0]
                          for r in picks])
            x = synth.fill_rows(cols, 0, 1, wl.ACT_SEED, wl.tag(0, wl.X_GATEUP), synth.normal())
            t0 = time.perf_counter()
            idx, sc = oracle.encode(W, "bf16", cb)
            Wd = oracle.decode(idx, sc, cb)
            oracle.rel_frobenius(W, "bf16", Wd)
            oracle.gemv(Wd, x, "bf16")
            t_work += time.perf_counter() - t0
            n_w += W.size
        return t_work, n_w

    t, n = run(16)
    per_w = t / n
    nrows = max(16, int(seconds / (per_w * (2 * 7168 + 2048))))
    t, n = run(nrows)
    cores = oracle.max_threads()
    # the same work on one core, on a tenth of the rows (reported beside the all-core figure)
    oracle.set_threads(1)
    try:
        t1, n1 = run(max(4, nrows // 10))
    finally:
        oracle.set_threads(cores)
    return {"value": n / t / 1e9, "unit": "Gweights/s", "cores": cores, "kind": "oracle",
            "sample": "%d sampled rows of each of w1, w3, w2 of the 64-expert layer (%d weights): encode + decode + "
                      "rel-Frobenius + binary64 GEMV, %.1f s" % (nrows, n, t),
            "one_core": {"value": n1 / t1 / 1e9, "unit": "Gweights/s", "weights": n1, "seconds": t1}}


def expert_rtn4_quality():
    """The single-expert workload (w1, w3: 2048 x 7168, w2: 7168 x 2048, Student-t(4) x log-normal rows, seed 1):
    the oracle's rtn4-row baseline error of each matrix (symmetric per-row int4, fp16 scale, 4.01 bits/weight).
    Part of the CPU leg: the oracle on host cores, before CUDA starts."""
    import oracle
    cfg, dist = wl.EXPERT, wl.expert_dist()
    out = {}
    t0 = time.perf_counter()
    for k, name in ((wl.W1, "w1"), (wl.W3, "w3"), (wl.W2, "w2")):
        rows, cols = wl.mat_shape(k)
        W = synth.fill_rows(cols, 0, rows, cfg["seed"], wl.tag(0, k), dist)
        Wq, _ = oracle.rtn4_row(W, "bf16")
        out[name] = oracle.rel_frobenius(W, "bf16", Wq)
    out["seconds"] = time.perf_counter() - t0
    return out


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on a bounded sample, same metric and config."""
    if rank != 0:
        return
    import oracle
    cb = load_codebooks("layer")
    seed, dist = wl.LAYER["seed"], wl.expert_dist()
    rng = np.random.default_rng(1)
    rows_per_step = 128
    samples = []
    for it in range(args.warmup + args.steps):
        mats = []
        for k in (wl.W1, wl.W3, wl.W2):
            rows, cols = wl.mat_shape(k)
            picks = rng.integers(0, args.experts * rows, size=rows_per_step)
            W = np.stack([synth.fill_row_list(cols, [r % rows], seed, wl.tag(int(r // rows), k), dist)[0]
                          for r in picks])
            mats.append((W, synth.fill_rows(cols, 0, 1, wl.ACT_SEED, wl.tag(0, wl.X_GATEUP), synth.normal())))
        t0 = time.perf_counter()
        n = 0
        for W, x in mats:
            idx, sc = oracle.encode(W, "bf16", cb)
            Wd = oracle.decode(idx, sc, cb)
            oracle.rel_frobenius(W, "bf16", Wd)
            oracle.gemv(Wd, x, "bf16")
            n += W.size
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            samples.append((dt, n))
    t = sum(s[0] for s in samples)
    n = sum(s[1] for s in samples)
    v = n / t / 1e9
    desc = ("each step: %d sampled rows of each of w1, w3, w2 of the 64-expert layer (%d weights): encode + decode + "
            "rel-Frobenius + binary64 GEMV" % (rows_per_step, samples[0][1]))
    out = {"metric": METRIC, "value": v, "unit": "Gweights/s", "impl": "reference", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / len(samples),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
           "config": bench_config(args.experts),
           "cpu_baseline": {"value": v, "unit": "Gweights/s", "cores": oracle.max_threads(), "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": v, "unit": "Gweights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------- ranks

def rank_expert0(rank, experts):
    """First expert of a rank's layer: rank r encodes experts experts*r .. experts*r + experts - 1 (weak scaling;
    the shards are disjoint, and each is the same data a single process would generate for those experts)."""
    return rank * experts


def max_over_ranks(torch, value, world, device):
    """The slowest rank's time (every rank takes the same collective step)."""
    if world == 1:
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def timed_region(torch, fn, reps):
    """Mean ms of reps calls of fn (after one untimed call), CUDA events on the current stream."""
    fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def whole_job_rate(world, weights_per_rank, ms):
    """Gweights/s of the whole job: every rank's weights over the slowest rank's time."""
    return world * weights_per_rank / ms / 1e6


# ----------------------------------------------------------------------------- main

def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE %d: launch N>1 with torchrun" % (args.gpus, world))

    # CPU baseline first (the oracle on host cores, before CUDA starts)
    cpu = None
    rtn4 = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(args.cpu_seconds, args.experts)
        if not args.no_expert_quality:
            rtn4 = expert_rtn4_quality()

    import torch
    import residual_vector_quantization_b200 as vq
    from datetime import timedelta
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    B_list = (1, 4, 8, 32)
    layer = Layer(torch, vq, dev, args.experts, rank_expert0(rank, args.experts), B_list)
    torch.cuda.synchronize()
    hbm_gbs, sm_max_mhz, peak_src = peaks()
    props = torch.cuda.get_device_properties(dev)
    sms = props.multi_processor_count
    # The definition's distance has every operation rounded (no fused multiply-add): one operation per FP32
    # lane and clock.  The screened encoder is bound by the ALU pipe instead.
    fp32_peak_tflops = sms * FP32_LANES_PER_SM * 1 * sm_max_mhz * 1e6 / 1e12
    alu_peak_tops = sms * ALU_LANES_PER_SM * sm_max_mhz * 1e6 / 1e12

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(i, marks=None):
        if marks: marks[0].record()
        layer.encode()
        if marks: marks[1].record()
        layer.pack()
        if marks: marks[2].record()
        layer.decode()
        if marks: marks[3].record()
        layer.errors()
        if marks: marks[4].record()
        layer.gemv(1, i)
        if marks: marks[5].record()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()

    clocks = ClockSampler(local)
    clocks.start()
    marks = [[ev() for _ in range(6)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t0, t1 = ev(), ev()
    t0.record()
    for i in range(args.steps):
        step(args.warmup + i, marks[i])
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(torch, t0.elapsed_time(t1), world, dev)
    part = lambda a, b: [marks[i][a].elapsed_time(marks[i][b]) for i in range(args.steps)]  # noqa: E731
    enc_ms = statistics.mean(part(0, 1))
    pack_ms = statistics.mean(part(1, 2))
    dec_ms = statistics.mean(part(2, 3))
    err_ms = statistics.mean(part(3, 4))
    gv1_ms = statistics.mean(part(4, 5))

    # decode-step GEMV sweep over batch sizes (not part of the step), rotating expert groups
    gemv = {}
    for B in B_list:
        for i in range(3):
            layer.gemv(B, i)
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record()
        for i in range(args.gemv_iters):
            layer.gemv(B, i)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / args.gemv_iters
        gbs = moe_step_bytes(B) / ms / 1e6
        gemv[str(B)] = {"us_per_step": 1e3 * ms, "GB/s": gbs, "frac_hbm": gbs / hbm_gbs,
                        "tokens_per_s": B / ms * 1e3}

    # the same kernel over the whole layer in one call (all experts' indices, 3 stacked matrices)
    layer_sweep = {}
    for B in B_list:
        plan = layer.layer_gemv_plan(B)
        for i in range(2):
            layer.layer_gemv(plan, B)
        torch.cuda.synchronize()
        a, b = ev(), ev()
        iters = 10 if B <= 8 else 3
        a.record()
        for i in range(iters):
            layer.layer_gemv(plan, B)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / iters
        nbytes = layer_gemv_bytes(B, layer.E)
        layer_sweep[str(B)] = {"us_per_call": 1e3 * ms, "GB/s": nbytes / ms / 1e6, "frac_hbm": nbytes / ms / 1e6 / hbm_gbs}
        del plan

    # achievable streaming bandwidth of this GPU, for context beside the copy-bandwidth fractions: a read-only
    # reduction and a write-only fill of 4 GiB (torch's kernels; not part of the path)
    stream_bw = None
    if args.gemm_iters > 0:
        buf = torch.empty(1 << 30, dtype=torch.float32, device=dev)
        buf.fill_(1.0)
        acc = torch.empty((), dtype=torch.float32, device=dev)
        rd, wr = [], []
        for _ in range(4):
            a, b, c = ev(), ev(), ev()
            a.record()
            torch.sum(buf, dim=0, out=acc)
            b.record()
            buf.fill_(2.0)
            c.record()
            torch.cuda.synchronize()
            rd.append(a.elapsed_time(b))
            wr.append(b.elapsed_time(c))
        nbytes = buf.numel() * 4
        stream_bw = {"read_GB/s": nbytes / min(rd[1:]) / 1e6, "write_GB/s": nbytes / min(wr[1:]) / 1e6,
                     "bytes": nbytes, "how": "torch.sum and Tensor.fill_ over a 4 GiB float32 buffer, best of 3"}
        del buf, acc

    # the prefill product on the tensor cores: the gate projections of 8 experts, 512 seeded random tokens each,
    # in one vq3r_gemm call (weights rebuilt from the tiled indices, bf16, fp32 accumulation)
    prefill = None
    if args.gemm_iters > 0:
        T, E8 = 512, min(8, layer.E)
        rows, cols = wl.mat_shape(wl.W1)
        gen = torch.Generator(device=dev)
        gen.manual_seed(wl.ACT_SEED)
        xs = torch.randn((E8, T, cols), generator=gen, device=dev).to(torch.bfloat16)
        ys = torch.empty((E8, T, rows), dtype=torch.float32, device=dev)
        mats = [dict(idx=layer.tiles[wl.W1], scales=layer.sc[wl.W1], codebooks=layer.cb, cols=cols, row0=e * rows,
                     rows=rows, x=xs[e], y=ys[e]) for e in range(E8)]
        for i in range(3):
            vq.vq3r_gemm(mats)
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record()
        for i in range(args.gemm_iters):
            vq.vq3r_gemm(mats)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / args.gemm_iters
        tflops = 2.0 * E8 * T * rows * cols / ms / 1e9
        peak_tc, peak_tc_src = bf16_peak()
        prefill = {"config": "%d experts x w1 %dx%d, %d tokens each, one call" % (E8, rows, cols, T), "ms": ms,
                   "TFLOP/s": tflops, "frac_bf16_peak": tflops / peak_tc, "bf16_peak_tflops": peak_tc,
                   "peak_source": peak_tc_src}
        del xs, ys, mats

    # codebook training on the GPU: Lloyd, 3 stages x 20 iterations on 65536 seeded random 8-vectors (the size of
    # the layer's training sample)
    train = None
    if args.gemm_iters > 0:
        gen = torch.Generator(device=dev)
        gen.manual_seed(wl.LAYER_SEED)
        vecs = torch.randn((65536, 8), generator=gen, device=dev)
        cbk = torch.empty((3, 256, 8), dtype=torch.float32, device=dev)
        trc = torch.empty((3, 21), dtype=torch.float64, device=dev)
        wst = torch.empty(vq.vq3r_train_workspace_size(65536), dtype=torch.uint8, device=dev)
        vq.vq3r_train(vecs, 20, codebooks=cbk, trace=trc, workspace=wst)
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record()
        vq.vq3r_train(vecs, 20, codebooks=cbk, trace=trc, workspace=wst)
        b.record()
        torch.cuda.synchronize()
        train = {"vectors": 65536, "stages": 3, "iters": 20, "ms": a.elapsed_time(b)}
        del vecs, wst

    # VQ4P (page §5: 4 stages x 64 codewords, packed 6-bit indices, the same 3.00 bits/weight) on the layer's
    # stacked gate matrix, beside VQ3R's decode of the same matrix: encode, decode to fp32, error
    vq4p = None
    if args.gemm_iters > 0:
        k = wl.W1
        cb4 = torch.from_numpy(load_codebooks("vq4p_layer")).to(dev)
        pl = torch.empty_like(layer.idx[k])
        sc4 = torch.empty_like(layer.sc[k])
        e4 = torch.empty(1, dtype=torch.float64, device=dev)
        n_w = layer.W[k].numel()

        def timed(fn, reps):
            fn()
            torch.cuda.synchronize()
            a, b = ev(), ev()
            a.record()
            for _ in range(reps):
                fn()
            b.record()
            torch.cuda.synchronize()
            return a.elapsed_time(b) / reps

        enc4_ms = timed(lambda: vq.vq4p_encode(layer.W[k], cb4, pl, sc4), 2)
        dec4_ms = timed(lambda: vq.vq4p_decode(pl, sc4, cb4, out=layer.dec[k]), 3)
        dec3_ms = timed(lambda: vq.vq3r_decode(layer.idx[k], layer.sc[k], layer.cb, out=layer.dec[k]), 3)
        err4_ms = timed(lambda: vq.vq4p_rel_frobenius_error(layer.W[k], pl, sc4, cb4, out=e4,
                                                            workspace=layer.err_ws[k]), 3)
        vq4p = {"matrix": "w1 of the layer, %d x %d stacked" % tuple(layer.W[k].shape),
                "encode_ms": enc4_ms, "encode_Gweights/s": n_w / enc4_ms / 1e6,
                "encode_definition_equivalent_tflops": VQ4P_FLOPS_PER_WEIGHT * n_w / enc4_ms / 1e9,
                "encode_frac_alu": 4 * 64 * ALU_OPS_PER_VEC_CODEWORD / 8 * n_w / enc4_ms / 1e9 / alu_peak_tops,
                "decode_f32_ms": dec4_ms, "decode_f32_frac_hbm": n_w * 4.375 / dec4_ms / 1e6 / hbm_gbs,
                "vq3r_decode_f32_ms": dec3_ms, "decode_speedup_vs_vq3r": dec3_ms / dec4_ms,
                "rel_frobenius_ms": err4_ms, "rel_frobenius_frac_hbm": n_w * 2.375 / err4_ms / 1e6 / hbm_gbs,
                "error": float(e4.item()), "vq3r_error": float(layer.err[k].item())}
        del pl, sc4

        # the 8-expert decode step with VQ4P weights beside VQ3R's over the same experts and x: experts 0-15 of
        # every kind, the two 8-expert groups alternating (264 MB of indices, more than L2)
        t4 = {}
        for kk in layer.kinds:
            rows, cols = wl.mat_shape(kk)
            p4, s4 = vq.vq4p_encode(layer.W[kk][:16 * rows], cb4)
            t4[kk] = (vq.vq3r_pack_tiles(p4), s4)
            del p4
        ws4 = torch.zeros(256, dtype=torch.uint8, device=dev)
        L4, stream4 = vq.lib(), torch.cuda.current_stream().cuda_stream
        step4 = {}
        for B in (1, 4):
            _, _, xu, xd = layer.moe[B]
            res = {}
            for fmt, fn in (("vq3r", L4.vq3r_gemv), ("vq4p", L4.vq4p_gemv)):
                calls = []
                for g in range(2):
                    mats = []
                    for j in range(8):
                        for kk in layer.kinds:
                            rows, cols = wl.mat_shape(kk)
                            idx_k, sc_k, cb_k = (t4[kk][0], t4[kk][1], cb4) if fmt == "vq4p" else \
                                (layer.tiles[kk], layer.sc[kk], layer.cb)
                            mats.append(dict(idx=idx_k, scales=sc_k, codebooks=cb_k, x=xd[j] if kk == wl.W2 else xu,
                                             row0=(8 * g + j) * rows, rows=rows, layout="tiles", cols=cols,
                                             y=torch.empty((B, rows), dtype=torch.float32, device=dev)))
                    calls.append((vq._descs(mats), len(mats), mats))

                def call(i, fn=fn, calls=calls, fmt=fmt):
                    d, n, _ = calls[i % 2]
                    st = fn(d, n, B, 1, ws4.data_ptr(), ws4.numel(), stream4)
                    if st:
                        raise vq.VQ3RError(st, fmt + "_gemv")

                for i in range(4):
                    call(i)
                torch.cuda.synchronize()
                a, b = ev(), ev()
                a.record()
                for i in range(args.gemv_iters):
                    call(i)
                b.record()
                torch.cuda.synchronize()
                ms = a.elapsed_time(b) / args.gemv_iters
                res[fmt] = {"us_per_step": 1e3 * ms, "frac_hbm": moe_step_bytes(B) / ms / 1e6 / hbm_gbs}
            step4[str(B)] = res
        vq4p["decode_step_8_experts"] = step4
        del t4, cb4

    # outlier-aware variant (page "XFP", 权重分解): a sparse FP16 residual of cols/512 entries per row on top of
    # the layer's VQ3R encoding: selection, decode and error with outliers, the MoE decode step with the sparse add,
    # and the error gain on the sweep distribution (Student-t(3) with 0.1% of weights at 20 sigma)
    outl = None
    if args.gemm_iters > 0:
        def timed_ms(fn, reps):
            fn()
            torch.cuda.synchronize()
            a, b = ev(), ev()
            a.record()
            for _ in range(reps):
                fn()
            b.record()
            torch.cuda.synchronize()
            return a.elapsed_time(b) / reps

        oc, ov, sel = {}, {}, {}
        for k in layer.kinds:
            rows_t, cols = layer.W[k].shape
            kk = cols // 512
            oc[k] = torch.empty((rows_t, kk), dtype=torch.int16, device=dev)
            ov[k] = torch.empty((rows_t, kk), dtype=torch.int16, device=dev)
            sel[k] = timed_ms(lambda: vq.vq3r_outliers(layer.W[k], layer.idx[k], layer.sc[k], layer.cb, kk, oc[k],
                                                        ov[k]), 2)
        k1 = wl.W1
        n1 = layer.W[k1].numel()
        e1 = torch.empty(1, dtype=torch.float64, device=dev)
        dec_o = timed_ms(lambda: vq.vq3r_decode_outliers(layer.idx[k1], layer.sc[k1], layer.cb, oc[k1], ov[k1],
                                                         out=layer.dec[k1]), 3)
        dec_p = timed_ms(lambda: vq.vq3r_decode(layer.idx[k1], layer.sc[k1], layer.cb, out=layer.dec[k1]), 3)
        err_o = timed_ms(lambda: vq.vq3r_rel_frobenius_error_outliers(layer.W[k1], layer.idx[k1], layer.sc[k1],
                                                                      layer.cb, oc[k1], ov[k1], out=e1,
                                                                      workspace=layer.err_ws[k1]), 3)
        err_with = float(e1.item())
        # the MoE decode step (B = 1) with the outliers: one call whose lookup kernel adds them
        # (vq3r_gemv_with_outliers), and for comparison the two-launch form (vq3r_gemv, then vq3r_gemv_outliers)
        plans, ws1, xu, xd = layer.moe[1]
        otl = {k: vq.vq3r_pack_outliers(oc[k], ov[k]) for k in layer.kinds}  # one-time layout for the fused call
        fdescs = []
        for g in range(layer.groups):
            d, n, mats = plans[g][:3]
            mo = []
            for i, m in enumerate(mats):
                kind = (wl.W1, wl.W3)[i % 2] if i < 16 else wl.W2
                mo.append(dict(m, otiles=otl[kind]))
            fdescs.append((d, vq._outlier_tiles(mo), n))
        odescs = []
        for g in range(layer.groups):
            mats = plans[g][2]
            om = []
            for j in range(min(8, layer.E)):
                e = g * 8 + j
                for slot, kind in ((2 * j, wl.W1), (2 * j + 1, wl.W3), (16 + j, wl.W2)):
                    rows, cols = wl.mat_shape(kind)
                    om.append(dict(ocols=oc[kind], ovals=ov[kind], cols=cols, row0=e * rows, rows=rows,
                                   x=xu if kind != wl.W2 else xd[j], y=mats[slot]["y"]))
            odescs.append(vq._outlier_descs(om))
        L = vq.lib()

        def step_plain(i):
            layer.gemv(1, i)

        def step_two_launch(i):
            layer.gemv(1, i)
            d = odescs[i % layer.groups]
            st = L.vq3r_gemv_outliers(d, len(d), 1, 1, torch.cuda.current_stream().cuda_stream)
            if st:
                raise vq.VQ3RError(st, "vq3r_gemv_outliers")

        def step_out(i):
            d, od, n = fdescs[i % layer.groups]
            st = L.vq3r_gemv_with_outliers(d, od, n, 1, 1, ws1.data_ptr(), ws1.numel(),
                                           torch.cuda.current_stream().cuda_stream)
            if st:
                raise vq.VQ3RError(st, "vq3r_gemv_with_outliers")

        reps = max(8, args.gemv_iters)
        t_plain = timed_ms(lambda: [step_plain(i) for i in range(reps)], 1) / reps
        t_out = timed_ms(lambda: [step_out(i) for i in range(reps)], 1) / reps
        t_two = timed_ms(lambda: [step_two_launch(i) for i in range(reps)], 1) / reps
        # error gain on 8 experts' w1 of the sweep distribution
        rows, cols = wl.mat_shape(wl.W1)
        Ws = torch.empty((8 * rows, cols), dtype=torch.bfloat16, device=dev)
        for e in range(8):
            synth.fill_rows_device(Ws[e * rows:(e + 1) * rows].data_ptr(), cols, 0, rows, wl.SWEEP["seed"],
                                   wl.tag(e, wl.W1), wl.sweep_dist(), stream=torch.cuda.current_stream().cuda_stream)
        cbs = torch.from_numpy(load_codebooks("sweep")).to(dev)
        idx_s, sc_s = vq.vq3r_encode(Ws, cbs)
        es0 = float(vq.vq3r_rel_frobenius_error(Ws, idx_s, sc_s, cbs).item())
        sweep_gain = {}
        for kk in (cols // 512, cols // 128):
            ocs, ovs = vq.vq3r_outliers(Ws, idx_s, sc_s, cbs, kk)
            sweep_gain[str(kk)] = float(vq.vq3r_rel_frobenius_error_outliers(Ws, idx_s, sc_s, cbs, ocs, ovs).item())
        del Ws, idx_s, sc_s, ocs, ovs
        outl = {"budget": "cols/512 per row (14 for 7168 columns, 4 for 2048): %.4f extra bits/weight"
                          % (32.0 / 512),
                "select_ms": {str(k): sel[k] for k in layer.kinds},
                "select_Gweights/s": sum(layer.W[k].numel() for k in layer.kinds) / sum(sel.values()) / 1e6,
                "decode_f32_w1_ms": dec_o, "decode_f32_w1_plain_ms": dec_p,
                "rel_frobenius_w1_ms": err_o, "rel_frobenius_w1_frac_hbm": n1 * 2.375 / err_o / 1e6 / hbm_gbs,
                "error_w1": err_with, "error_w1_plain": errs_plain_w1(layer),
                "moe_step_B1_us": 1e3 * t_out, "moe_step_B1_plain_us": 1e3 * t_plain,
                "moe_step_B1_two_launch_us": 1e3 * t_two, "moe_step_B1_ratio_to_plain": t_out / t_plain,
                "sweep_8x_w1_error_plain": es0, "sweep_8x_w1_error_with_outliers": sweep_gain}
        del oc, ov, odescs, fdescs, otl

    # the single-expert workload's quality table: VQ3R error of w1, w3, w2 (this library, expert codebooks) beside
    # the oracle's rtn4-row error of the same matrices (computed in the CPU leg), outside the timed region
    quality = None
    if rtn4 is not None:
        cbe = torch.from_numpy(load_codebooks("expert")).to(dev)
        vq3 = {}
        for k, name in ((wl.W1, "w1"), (wl.W3, "w3"), (wl.W2, "w2")):
            rows, cols = wl.mat_shape(k)
            We = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
            synth.fill_rows_device(We.data_ptr(), cols, 0, rows, wl.EXPERT["seed"], wl.tag(0, k), wl.expert_dist(),
                                   stream=torch.cuda.current_stream().cuda_stream)
            ie, se = vq.vq3r_encode(We, cbe)
            vq3[name] = float(vq.vq3r_rel_frobenius_error(We, ie, se, cbe).item())
            del We, ie, se
        quality = {"workload": wl.EXPERT["name"] + ", seed %d" % wl.EXPERT["seed"],
                   "vq3r_3.00bpw": vq3, "rtn4_row_4.01bpw_oracle": {n: rtn4[n] for n in ("w1", "w3", "w2")},
                   "bits_per_weight": {"vq3r": {"w1": 3 + 16 / 7168, "w3": 3 + 16 / 7168, "w2": 3 + 16 / 2048},
                                       "rtn4_row": {"w1": 4 + 16 / 7168, "w3": 4 + 16 / 7168, "w2": 4 + 16 / 2048}}}

    # the scale-sweep workload: 256 experts x {w1, w3: 2048 x 7168; w2: 7168 x 2048}, Student-t(3) rows with 0.1%
    # of the weights at +-20 sigma, seed 4 (11.27 G weights, 22.5 GB of bf16): encode of each stacked matrix kind,
    # then the decode-GEMV at B = 1, 4, 8, 32 over all experts, as one call over the three stacked matrices and as
    # 8-expert decode steps rotating over all 32 disjoint groups
    sweep = None
    if args.sweep_experts > 0:
        E5 = args.sweep_experts
        st5 = torch.cuda.current_stream().cuda_stream
        cb5 = torch.from_numpy(load_codebooks("sweep")).to(dev)
        W5, I5, S5 = {}, {}, {}
        for k in layer.kinds:
            rows, cols = wl.mat_shape(k)
            W5[k] = torch.empty((E5 * rows, cols), dtype=torch.bfloat16, device=dev)
            for e in range(E5):
                synth.fill_rows_device(W5[k][e * rows:(e + 1) * rows].data_ptr(), cols, 0, rows, wl.SWEEP["seed"],
                                       wl.tag(e, k), wl.sweep_dist(), stream=st5)
            I5[k] = torch.empty((3, E5 * rows, cols // 8), dtype=torch.uint8, device=dev)
            S5[k] = torch.empty(E5 * rows, dtype=torch.int16, device=dev)
        n5 = sum(W5[k].numel() for k in layer.kinds)

        def enc5():
            for k in layer.kinds:
                vq.vq3r_encode(W5[k], cb5, I5[k], S5[k])

        enc5_ms = timed_region(torch, enc5, 2)
        del W5
        torch.cuda.empty_cache()
        T5 = {k: vq.vq3r_pack_tiles(I5[k]) for k in layer.kinds}
        del I5
        enc5_tflops = FLOPS_PER_WEIGHT * n5 / enc5_ms / 1e9
        gv_all, gv_steps = {}, {}
        for B in B_list:
            _, _, xu, xd = layer.moe[B]
            mats = []
            for k in layer.kinds:
                rows, cols = wl.mat_shape(k)
                mats.append(dict(idx=T5[k], scales=S5[k], codebooks=cb5, x=xu if cols == wl.HIDDEN else xd[0],
                                 rows=E5 * rows, layout="tiles", cols=cols,
                                 y=torch.empty((B, E5 * rows), dtype=torch.float32, device=dev)))
            d = vq._descs(mats)
            ws5 = torch.zeros(max(256, vq.lib().vq3r_gemv_workspace_size(d, 3, B)), dtype=torch.uint8, device=dev)
            def call():
                st = vq.lib().vq3r_gemv(d, 3, B, 1, ws5.data_ptr(), ws5.numel(), st5)
                if st:
                    raise vq.VQ3RError(st, "vq3r_gemv")

            ms = timed_region(torch, call, 3 if B <= 8 else 2)
            nbytes = layer_gemv_bytes(B, E5)
            gv_all[str(B)] = {"us_per_call": 1e3 * ms, "GB/s": nbytes / ms / 1e6,
                              "frac_hbm": nbytes / ms / 1e6 / hbm_gbs}
            del mats, d
            groups = []
            for g in range(E5 // 8):
                ms_ = []
                for j in range(8):
                    e = g * 8 + j
                    for k in (wl.W1, wl.W3):
                        rows, cols = wl.mat_shape(k)
                        ms_.append(dict(idx=T5[k], scales=S5[k], codebooks=cb5, x=xu, row0=e * rows, rows=rows,
                                        layout="tiles", cols=cols,
                                        y=torch.empty((B, rows), dtype=torch.float32, device=dev)))
                for j in range(8):
                    e = g * 8 + j
                    rows, cols = wl.mat_shape(wl.W2)
                    ms_.append(dict(idx=T5[wl.W2], scales=S5[wl.W2], codebooks=cb5, x=xd[j], row0=e * rows,
                                    rows=rows, layout="tiles", cols=cols,
                                    y=torch.empty((B, rows), dtype=torch.float32, device=dev)))
                groups.append((vq._descs(ms_), ms_))

            def steps():
                for dg, _ in groups:
                    st = vq.lib().vq3r_gemv(dg, 24, B, 1, ws5.data_ptr(), ws5.numel(), st5)
                    if st:
                        raise vq.VQ3RError(st, "vq3r_gemv")

            ms = timed_region(torch, steps, 2) / len(groups)
            gv_steps[str(B)] = {"us_per_step": 1e3 * ms, "GB/s": moe_step_bytes(B) / ms / 1e6,
                                "frac_hbm": moe_step_bytes(B) / ms / 1e6 / hbm_gbs, "tokens_per_s": B / ms * 1e3}
            del groups, ws5
        sweep = {"workload": wl.SWEEP["name"] + ", seed %d, %d experts" % (wl.SWEEP["seed"], E5), "weights": n5,
                 "index_bytes": 3 * n5 // 8,
                 "encode": {"ms": enc5_ms, "Gweights/s": n5 / enc5_ms / 1e6,
                            "definition_equivalent_tflops": enc5_tflops,
                            "definition_equivalent_frac_fma_counted_fp32_peak": enc5_tflops / (2 * fp32_peak_tflops),
                            "executed_alu_frac": ENC_ALU_OPS_PER_WEIGHT * n5 / enc5_ms / 1e9 / alu_peak_tops},
                 "gemv_all_experts_one_call": gv_all,
                 "gemv_decode_steps_8_experts_rotating_32_groups": gv_steps}
        del T5, S5
        torch.cuda.empty_cache()

    # end to end through the public API with host buffers: every step uploads the layer from pinned host memory
    # and reads its results back (indices, scales, errors, y).  The device inputs and index outputs are double
    # buffered and the copies are pipelined per matrix kind: a kind's encode starts once its weights have arrived
    # (upload on its own stream) and its indices are read back as soon as it is encoded (a third stream), so the
    # copies overlap the compute of the same and the neighbouring steps; every copy lies between the start and
    # end events.
    e2e = None
    if args.e2e_steps > 0:
        hostW = {k: torch.empty(layer.W[k].shape, dtype=layer.W[k].dtype, pin_memory=True) for k in layer.kinds}
        hostI = {k: torch.empty(layer.idx[k].shape, dtype=torch.uint8, pin_memory=True) for k in layer.kinds}
        hostS = {k: torch.empty(layer.sc[k].shape, dtype=torch.int16, pin_memory=True) for k in layer.kinds}
        hostE = torch.empty(3, dtype=torch.float64, pin_memory=True)
        hostY = torch.empty((8 * 7168 + 16 * 2048,), dtype=torch.float32, pin_memory=True)
        for k in layer.kinds:
            hostW[k].copy_(layer.W[k])
        W0, I0 = dict(layer.W), dict(layer.idx)
        Wbuf = [W0, {k: torch.empty_like(W0[k]) for k in layer.kinds}]
        Ibuf = [I0, {k: torch.empty_like(I0[k]) for k in layer.kinds}]
        torch.cuda.synchronize()
        h2d = sum(hostW[k].numel() * hostW[k].element_size() for k in layer.kinds)
        d2h = sum(hostI[k].numel() + 2 * hostS[k].numel() for k in layer.kinds) + 24 + 4 * hostY.numel()
        s_comp = torch.cuda.current_stream()
        s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
        K = args.e2e_steps
        nk = len(layer.kinds)
        ev_up = [[ev() for _ in range(nk)] for _ in range(K)]
        ev_enc = [[ev() for _ in range(nk)] for _ in range(K)]
        ev_comp = [ev() for _ in range(K)]
        ev_down = [ev() for _ in range(K)]
        barrier()
        a, b = ev(), ev()
        a.record(s_comp)
        for i in range(K):
            bi = i % 2
            with torch.cuda.stream(s_up):
                s_up.wait_event(a)
                if i >= 2:
                    s_up.wait_event(ev_comp[i - 2])  # step i - 2 has finished with this input buffer
                for j, k in enumerate(layer.kinds):
                    Wbuf[bi][k].copy_(hostW[k], non_blocking=True)
                    ev_up[i][j].record(s_up)
            if i >= 2:
                s_comp.wait_event(ev_down[i - 2])  # step i - 2's indices have been read back
            layer.W, layer.idx = Wbuf[bi], Ibuf[bi]
            # the step (as in the timed loop), each kind's encode once its weights are on the device and its
            # index read-back once it is encoded
            for j, k in enumerate(layer.kinds):
                s_comp.wait_event(ev_up[i][j])
                layer.encode_kind(k)
                ev_enc[i][j].record(s_comp)
                with torch.cuda.stream(s_down):
                    s_down.wait_event(ev_enc[i][j])
                    hostI[k].copy_(Ibuf[bi][k], non_blocking=True)
            with torch.cuda.stream(s_down):
                ev_down[i].record(s_down)
            layer.pack()
            layer.decode()
            layer.errors()
            layer.gemv(1, i)
            for k in layer.kinds:
                hostS[k].copy_(layer.sc[k], non_blocking=True)
            for j, k in enumerate(layer.kinds):
                hostE[j:j + 1].copy_(layer.err[k], non_blocking=True)
            plans = layer.moe[1][0][i % layer.groups]
            off = 0
            for m in plans[2]:
                n = m["y"].numel()
                hostY[off:off + n].copy_(m["y"].view(-1), non_blocking=True)
                off += n
            ev_comp[i].record(s_comp)
        s_comp.wait_event(ev_down[K - 1])
        s_comp.wait_event(ev_up[K - 1][nk - 1])
        b.record(s_comp)
        torch.cuda.synchronize()
        layer.W, layer.idx = W0, I0
        e2e_ms = max_over_ranks(torch, a.elapsed_time(b) / K, world, dev)
        e2e = {"value": whole_job_rate(world, layer.weights, e2e_ms), "unit": "Gweights/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": K,
               "overlap": "uploads and index read-backs on their own streams, pipelined per matrix kind, "
                          "double-buffered device buffers"}
        del Wbuf, Ibuf

    errs = {str(k): float(layer.err[k].item()) for k in layer.kinds}
    ms_step = total_ms / args.steps
    value = whole_job_rate(world, layer.weights, ms_step)  # Gweights/s over the whole path
    enc_tflops = FLOPS_PER_WEIGHT * layer.weights / enc_ms / 1e9
    enc_tops = ENC_ALU_OPS_PER_WEIGHT * layer.weights / enc_ms / 1e9
    dev_err = vq.vq3r_device_error()
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "Gweights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": bench_config(args.experts),
            "roofline": {"bound": "alu", "achieved": enc_tops, "peak": alu_peak_tops, "unit": "Top/s",
                         "frac": enc_tops / alu_peak_tops,
                         "traffic": (None if ENCODE_DRAM_BYTES_PER_WEIGHT is None
                                     else ENCODE_DRAM_BYTES_PER_WEIGHT * layer.weights / 3),
                         "kernel": "vq3r_encode (row scale + screened greedy assignment; per launch = one stacked "
                                   "matrix kind, 3 per step).  achieved = the ALU-pipe operations the screened "
                                   "encoder executes, %d per weight (3 stages x 256 codewords x %d bookkeeping "
                                   "operations / 8), per second; peak = %d SMs x %d ALU lanes x %.0f MHz; traffic = "
                                   "DRAM bytes per launch from the committed ncu capture"
                                   % (ENC_ALU_OPS_PER_WEIGHT, ALU_OPS_PER_VEC_CODEWORD, sms, ALU_LANES_PER_SM,
                                      sm_max_mhz),
                         "definition_equivalent": {
                             "flops_per_weight": FLOPS_PER_WEIGHT, "achieved_tflops": enc_tflops,
                             "frac_of_fma_counted_fp32_peak": enc_tflops / (2 * fp32_peak_tflops),
                             "fma_counted_fp32_peak_tflops": 2 * fp32_peak_tflops,
                             "frac_of_non_fma_fp32_ceiling": enc_tflops / fp32_peak_tflops,
                             "non_fma_fp32_ceiling_tflops": fp32_peak_tflops,
                             "note": "the definition's arithmetic (3 x 256 x 8 x (sub, mul, add) per 8 weights) "
                                     "credited at the kernel's rate; the kernel reaches the same indices with a "
                                     "screen and runs the definition's scan only where the screen's margin fails, "
                                     "so the rate can exceed the non-FMA ceiling of the operations it credits"}},
            "kernels": {
                "encode": {"ms": enc_ms, "Gweights/s": layer.weights / enc_ms / 1e6, "TFLOP/s": enc_tflops},
                "pack_tiles": {"ms": pack_ms, "GB/s": 2 * 0.375 * layer.weights / pack_ms / 1e6},
                "decode_f32": {"ms": dec_ms, "GB/s": layer.weights * (4 + 0.375) / dec_ms / 1e6,
                               "frac_hbm": layer.weights * 4.375 / dec_ms / 1e6 / hbm_gbs},
                "rel_frobenius": {"ms": err_ms, "GB/s": layer.weights * (2 + 0.375) / err_ms / 1e6,
                                  "frac_hbm": layer.weights * 2.375 / err_ms / 1e6 / hbm_gbs, "errors": errs},
                "gemv_in_step_B1": {"us": 1e3 * gv1_ms, "GB/s": moe_step_bytes(1) / gv1_ms / 1e6,
                                    "frac_hbm": moe_step_bytes(1) / gv1_ms / 1e6 / hbm_gbs},
                "gemv_sweep": gemv,
                "gemv_layer_sweep": layer_sweep,
                "gemm_prefill": prefill,
                "train_lloyd": train,
                "vq4p": vq4p,
                "outliers": outl,
                "expert_quality": quality,
                "sweep_256_experts": sweep,
                "stream_bandwidth": stream_bw,
                "hbm_peak_gbs": hbm_gbs, "peak_source": peak_src},
            "e2e": e2e,
            "gpu_launches": Layer.LAUNCHES_PER_STEP * args.steps,
            "clocks": clk,
            "device_error": dev_err,
        }
        if cpu is not None:
            out["cpu_baseline"] = cpu
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
