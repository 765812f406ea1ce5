"""Benchmark of the packed-ternary decode path on B200.

One step = one decode token at M = 1 through the synthetic 8B-geometry linear stack (36 layers,
each as four fused launches: q|k|v 6144x4096, o 4096x4096, gate|up 24576x4096, down 4096x12288,
i.e. all 252 ternary linears) plus the int8 output head 151936x4096 with fused argmax, bf16
activations. Weights are packed on the device from the seeded generator (synth), activations
are N(0,1) bf16; every input of a step (2.37 GB) is far larger than the 126 MB L2, so each step
streams its weights from HBM.

Prints one JSON line (rank 0). --impl reference times the CPU oracle instead (the same workload,
a bounded sample per step, extrapolated to a token).

The timed region replays CUDA graphs of captured steps (kernels launched with programmatic
dependent launch); each kernel reads its activations only after the previous kernel finished,
as in a real decode chain. Extra rows measure the other scope rows (single GEMV, int8 mode,
0.6B stack, small-M sweep, base-3 unpack).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ternary GEMV HBM GB/s & 8B linear-stack tok/s at M=1 (fraction of HBM peak)"
# DRAM bytes (read + write) of the stream kernel per full 8B step, from an ncu capture of the
# 4-layer profile case (batch-8b-4layers-bf16: 195.43 MB read + 5.26 MB written) scaled by the
# units processed (36 / 4 layers). None whenever that kernel has changed since the counters were
# taken.
STREAM_TRAFFIC_PER_STEP = 9 * (195.43e6 + 5.26e6)
SEED = 0x7E2A2026
L2_BYTES = 126 * 1024 * 1024


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------------------------
# synthetic model on the device
class Linear:
    """A fused packed-ternary launch: rows of several projections stacked (same input)."""

    def __init__(self, W, N, K, parts):
        self.W, self.N, self.K, self.parts = W, N, K, parts

    @property
    def bytes(self):
        # algorithmic bytes of one M=1 launch: planes + scales + activation in + output out
        return self.N * self.K // 4 + 2 * self.N + 2 * self.K + 4 * self.N


def build_linear(model, layer, projs, seed=SEED, interleave=False):
    """interleave (two projections of equal shape, e.g. gate and up): rows in groups of eight,
    16j .. 16j + 7 from the first projection's rows 8j .. 8j + 7, then the second's (the layout of
    the dependent chain's SwiGLU epilogue)."""
    import torch
    import bit_gemv_tern_b200 as tg
    import synth
    import synth.cuda as sc
    shapes = {p: (N, K) for p, N, K in synth.linear_shapes(model)}
    K = shapes[projs[0]][1]
    N = sum(shapes[p][0] for p in projs)
    tr = torch.empty(N * K, dtype=torch.int8, device="cuda")
    scales, r = [], 0
    for p in projs:
        n = shapes[p][0]
        tid = synth.tensor_id(layer, p)
        sc.trits_into(tr[r * K:(r + n) * K], seed, tid, K, synth.trit_probs(model, layer, p))
        scales.append(synth.row_scales(seed, tid, n))
        r += n
    scale = np.concatenate(scales)
    if interleave:
        n = N // 2
        tr = tr.view(2, n // 8, 8, K).transpose(0, 1).contiguous().view(-1)
        scale = scale.reshape(2, n // 8, 8).transpose(1, 0, 2).reshape(-1).copy()
    W = tg.TernMatrix.empty(N, K)
    W.scale.copy_(torch.from_numpy(scale.view(np.float16)))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    tg.tern_pack(tg.TERN_SRC_INT8_TRITS, tr, N, K, W.planes, flag)
    assert tg.tern_read_flag(flag) == 0
    del tr
    return Linear(W, N, K, projs)


class Stack:
    """A model's fused linears + int8 head with activations for M rows, on the device."""

    def __init__(self, model, M=1, seed=SEED, layers=None):
        import torch
        import synth
        import synth.cuda as sc
        g = synth.GEOMETRY[model]
        self.model, self.M = model, M
        self.L = g["layers"] if layers is None else layers
        self.V, self.d = g["vocab"], g["d"]
        self.linears, self.x_tid = [], []
        for layer in range(self.L):
            for grp, projs in synth.FUSED_GROUPS:
                # gate|up rows interleaved by eight (the dependent chain fuses SwiGLU into its epilogue;
                # the independent batches only see the outputs in another order)
                self.linears.append(build_linear(model, layer, projs, seed, interleave=grp == "gate_up"))
                self.x_tid.append(synth.act_tensor_id(model, layer, grp))
        htid = synth.head_tensor_id(model)
        self.head_W = torch.empty(self.V * self.d, dtype=torch.int8, device="cuda")
        sc.head_into(self.head_W, seed, htid, self.d)
        self.head_s = torch.from_numpy(synth.head_scales(seed, htid, self.V).view(np.float16)).cuda()
        # activations: one bf16 [M, K] per fused launch + the head input, in one contiguous buffer
        xs = [synth.activations(seed, tid, M, lin.K) for tid, lin in zip(self.x_tid, self.linears)]
        xs.append(synth.activations(seed, synth.head_act_tensor_id(model), M, self.d))
        self.x_offsets, off = [], 0
        for a in xs:
            self.x_offsets.append(off)
            off += a.size
        self.x_host = torch.empty(off, dtype=torch.int16, pin_memory=True)
        flat = np.concatenate([a.reshape(-1) for a in xs]).view(np.int16)
        self.x_host.numpy()[:] = flat
        self.x = self.x_host.cuda()
        self.y = [torch.empty(M * lin.N, dtype=torch.float32, device="cuda") for lin in self.linears]
        # int8 mode inputs (quantised once; a full model fuses this into the producing kernel)
        self.q = torch.empty(off, dtype=torch.int8, device="cuda")
        self.sx = torch.empty(len(xs) * M, dtype=torch.float32, device="cuda")
        self.argmax = torch.empty(M, dtype=torch.int32, device="cuda")
        self.maxval = torch.empty(M, dtype=torch.float32, device="cuda")
        import bit_gemv_tern_b200 as tg
        self.ws = torch.zeros(tg.i8_head_workspace_bytes(self.V, M), dtype=torch.uint8, device="cuda")
        self.result_host = torch.empty(2 * M, dtype=torch.int32, pin_memory=True)
        self._batches = {}
        for i, (o, a) in enumerate(zip(self.x_offsets, xs)):
            K = a.shape[1]
            tg.tern_quantize_act(self.x[o:o + M * K], M, K, self.q[o:o + M * K], self.sx[i * M:(i + 1) * M])
        torch.cuda.synchronize()

    def xs(self, i):
        K = self.linears[i].K if i < len(self.linears) else self.d
        o = self.x_offsets[i]
        return self.x[o:o + self.M * K], self.q[o:o + self.M * K], self.sx[i * self.M:(i + 1) * self.M]

    @property
    def stack_bytes(self):
        return sum(l.bytes + (self.M - 1) * (2 * l.K + 4 * l.N) for l in self.linears)

    @property
    def head_bytes(self):
        return self.V * self.d + 2 * self.V + 2 * self.M * self.d + 8 * self.M

    def batch(self, mode):
        """The stack's M = 1 GEMVs as one tern_gemv_batch (independent activations)."""
        import bit_gemv_tern_b200 as tg
        if mode not in self._batches:
            act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
            entries = []
            for i, lin in enumerate(self.linears):
                xb, q, sx = self.xs(i)
                entries.append((lin.W, xb if mode == "bf16" else q, None if mode == "bf16" else sx, self.y[i]))
            self._batches[mode] = tg.GemvBatch(entries, act)
        return self._batches[mode]

    def int8_fused_batch(self):
        """The stack's GEMVs in int8 mode with the per-token quantiser fused into the batch's operand
        preparation (bf16 activations in, s_x written by the prep): no separate quantiser launch."""
        import torch
        import bit_gemv_tern_b200 as tg
        if "int8_fused" not in self._batches:
            self.sx_fused = torch.empty(len(self.linears) * self.M, dtype=torch.float32, device="cuda")
            entries, pros = [], []
            for i, lin in enumerate(self.linears):
                xb, _, _ = self.xs(i)
                entries.append((lin.W, None, self.sx_fused[i * self.M:(i + 1) * self.M], self.y[i]))
                pros.append((tg.TERN_PRO_BF16, xb, None, 0.0))
            self._batches["int8_fused"] = tg.GemvBatch(entries, tg.TERN_ACT_INT8, M=self.M, prologues=pros)
        return self._batches["int8_fused"]

    def launch_step_int8_fused(self):
        """int8-mode decode step with every quantisation inside it: the stack's batch (quantiser fused
        into its prep launch), then the head input's quantiser and the int8 head."""
        import bit_gemv_tern_b200 as tg
        self.int8_fused_batch()()
        xb, q, sx = self.xs(len(self.linears))
        tg.tern_quantize_act(xb, self.M, self.d, q, sx)
        tg.i8_head_gemv_argmax(self.head_W, self.head_s, self.V, self.d, self.M, tg.TERN_ACT_INT8, q, sx,
                               self.argmax, self.maxval, None, self.ws)

    def launch_stack(self, mode="bf16", pdl=False, chained=False):
        """M = 1: one batched launch pair for all linears (their activations are independent
        inputs); chained=True launches one GEMV per linear instead, each waiting for the previous
        kernel before reading its activation (a decode chain)."""
        import bit_gemv_tern_b200 as tg
        act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
        fl = tg.TERN_FLAG_PDL if pdl else 0
        if self.M == 1 and not chained:
            self.batch(mode)(flags=fl)
            return
        for i, lin in enumerate(self.linears):
            xb, q, sx = self.xs(i)
            if self.M == 1:
                tg.tern_gemv(lin.W, act, xb if act == tg.TERN_ACT_BF16 else q, None if act == tg.TERN_ACT_BF16 else sx,
                             self.y[i], flags=fl)
            else:
                tg.tern_gemm_small_m(lin.W, self.M, act, xb if act == tg.TERN_ACT_BF16 else q,
                                     None if act == tg.TERN_ACT_BF16 else sx, self.y[i], flags=fl)

    def launch_head(self, mode="bf16", pdl=False):
        import bit_gemv_tern_b200 as tg
        act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
        xb, q, sx = self.xs(len(self.linears))
        tg.i8_head_gemv_argmax(self.head_W, self.head_s, self.V, self.d, self.M, act,
                               xb if act == tg.TERN_ACT_BF16 else q, None if act == tg.TERN_ACT_BF16 else sx,
                               self.argmax, self.maxval, None, self.ws, flags=tg.TERN_FLAG_PDL if pdl else 0)

    @property
    def launches_per_step(self):
        return 3 if self.M == 1 else len(self.linears) + 1


def capture(fn, steps, events=None):
    """CUDA graph of `steps` repetitions of fn(step_index, events)."""
    import torch
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=s):
        for i in range(steps):
            fn(i)
    torch.cuda.current_stream().wait_stream(s)
    return g


def timed_replays(graphs_and_counts):
    """Replay graphs back to back between two events; returns elapsed ms."""
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for g, n in graphs_and_counts:
        for _ in range(n):
            g.replay()
    b.record()
    b.synchronize()
    return a.elapsed_time(b)


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu, self.proc, self.path = gpu_index, None, None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        try:
            rows = [l.split(",") for l in open(self.path).read().strip().splitlines() if l.strip()]
            os.unlink(self.path)
        except Exception:
            return out
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1])); mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if sm:
            out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                   "samples": len(sm)}
        return out


# ---------------------------------------------------------------------------------------------
def _oracle_sample(rows=256, model="8b"):
    """Inputs for the CPU oracle: `rows` rows of each fused launch of `model` and 4x as many head
    rows."""
    import oracle
    import synth
    shapes = {p: (N, K) for p, N, K in synth.linear_shapes(model)}
    fused = [(grp, sum(shapes[p][0] for p in projs), shapes[projs[0]][1]) for grp, projs in synth.FUSED_GROUPS]
    mats = []
    for grp, N, K in fused:
        t = synth.trits(SEED, 9000 + K, rows, K)
        mats.append((grp, N, K, oracle.pack(t), synth.row_scales(SEED, 9000 + K, rows),
                     synth.activations(SEED, 9000 + K, 1, K)))
    d = synth.GEOMETRY[model]["d"]
    head = (synth.head_weights(SEED, 9999, 4 * rows, d), synth.head_scales(SEED, 9999, 4 * rows),
            synth.activations(SEED, 9999, 1, d))
    return mats, head, rows, model


def _oracle_token_seconds(sample, threads, budget_s):
    """Time the oracle on the sample (repeating calls until budget_s is spent) and scale by rows to
    one token of the sample's model: layers x 4 fused launches + the vocabulary-row head.
    Returns (s/token, s measured)."""
    import oracle
    import synth
    mats, head, rows, model = sample
    L, V = synth.GEOMETRY[model]["layers"], synth.GEOMETRY[model]["vocab"]
    spent, reps = 0.0, 0
    tot = {}
    while True:
        for grp, N, K, pl, s, x in mats:
            t0 = time.perf_counter()
            oracle.gemm_bf16(pl, s, K, x, nthreads=threads)
            dt = time.perf_counter() - t0
            tot[grp] = tot.get(grp, 0.0) + dt
            spent += dt
        t0 = time.perf_counter()
        oracle.head_bf16(head[0], head[1], head[2], nthreads=threads)
        dt = time.perf_counter() - t0
        tot["head"] = tot.get("head", 0.0) + dt
        spent += dt
        reps += 1
        if spent >= budget_s:
            break
    t_token = sum(tot[grp] / (reps * rows) * N * L for grp, N, K, _, _, _ in mats)
    t_token += tot["head"] / (reps * 4 * rows) * V
    return t_token, spent


def token_bytes(model):
    """Algorithmic bytes of one M = 1 token of `model`: per fused linear the packed planes N*K/4,
    the fp16 scales 2N, the bf16 activation 2K and the fp32 outputs 4N; the int8 head V*d + 2V
    (+ its activation and result)."""
    import synth
    g = synth.GEOMETRY[model]
    shapes = {p: (N, K) for p, N, K in synth.linear_shapes(model)}
    b = 0
    for _, projs in synth.FUSED_GROUPS:
        N, K = sum(shapes[p][0] for p in projs), shapes[projs[0]][1]
        b += N * K // 4 + 2 * N + 2 * K + 4 * N
    return g["layers"] * b + g["vocab"] * g["d"] + 2 * g["vocab"] + 2 * g["d"] + 8


def _oracle_gemv_seconds(threads, budget_s):
    """The oracle on the whole single-GEMV workload (N = 3072, K = 1024, M = 1), repeated until
    budget_s is spent; returns s per GEMV."""
    import oracle
    import synth
    N, K = 3072, 1024
    pl = oracle.pack(synth.trits(SEED, 1, N, K))
    s, x = synth.row_scales(SEED, 1, N), synth.activations(SEED, 1, 1, K)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.gemm_bf16(pl, s, K, x, nthreads=threads)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return (time.perf_counter() - t0) / reps


def cpu_baseline(budget_s=12.0):
    """The oracle on this host's cores on a bounded sample of the 8B token, scaled to tok/s; with
    the same on one thread and the oracle's GB/s (the workload's algorithmic bytes over its time)
    for the single GEMV, the 0.6B token and the 8B token."""
    threads = os.cpu_count() or 1
    sample = _oracle_sample()
    t_token, spent = _oracle_token_seconds(sample, threads, budget_s)
    t_token_1, spent_1 = _oracle_token_seconds(sample, 1, budget_s / 3)
    t_06, spent_06 = _oracle_token_seconds(_oracle_sample(model="0.6b"), threads, budget_s / 4)
    t_gemv = _oracle_gemv_seconds(threads, 1.0)
    gemv_bytes = 3072 * 1024 // 4 + 2 * 3072 + 2 * 1024 + 4 * 3072
    per_config = {
        "gemv_3072x1024_m1": {"gbs": gemv_bytes / t_gemv / 1e9, "us_per_call": t_gemv * 1e6},
        "0.6b_token_m1": {"gbs": token_bytes("0.6b") / t_06 / 1e9, "tok_s": 1.0 / t_06},
        "8b_token_m1": {"gbs": token_bytes("8b") / t_token / 1e9, "tok_s": 1.0 / t_token,
                        "gbs_1thread": token_bytes("8b") / t_token_1 / 1e9, "tok_s_1thread": 1.0 / t_token_1},
    }
    return {"value": 1.0 / t_token, "unit": "tok/s", "cores": threads, "kind": "oracle",
            "value_1thread": 1.0 / t_token_1, "per_config": per_config,
            "sample": f"{sample[2]} rows of each fused 8B launch (q|k|v, o, gate|up, down; full K) and "
                      f"{4 * sample[2]} head rows (K=4096), fp64 oracle, calls repeated for {spent:.1f} s "
                      f"({spent_1:.1f} s on 1 thread), per-row time scaled to 36 layers + the 151936-row head; "
                      f"0.6B the same at its widths ({spent_06:.1f} s); the single GEMV whole"}


# ---------------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step times the oracle on a bounded sample of the
    token (sized so that warm-up + steps take about a minute), extrapolated to tok/s."""
    if rank != 0:
        return 0
    threads = os.cpu_count() or 1
    sample = _oracle_sample()
    per_step = max(0.002, 60.0 / (args.steps + args.warmup))
    for _ in range(args.warmup):
        _oracle_token_seconds(sample, threads, per_step)
    toks, spent = [], 0.0
    for _ in range(args.steps):
        t, sp = _oracle_token_seconds(sample, threads, per_step)
        toks.append(t)
        spent += sp
    t_token = statistics.median(toks)
    cb = {"value": 1.0 / t_token, "unit": "tok/s", "cores": threads, "kind": "oracle",
          "sample": f"per step: {sample[2]} rows of each fused 8B launch and {4 * sample[2]} head rows, "
                    f"oracle calls repeated for >= {per_step * 1000:.0f} ms, per-row time scaled to a token; "
                    f"median over {args.steps} steps ({spent:.1f} s measured)"}
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * t_token,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "8b_linear_stack_m1_bf16_plus_int8_head", "model": "neutrino-1-8b-geometry",
                       "global_batch": 1, "seq_len": 1, "parallelism": "none (host cores)"},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def rank_barrier(dist):
    """Barrier over the replica ranks (no-op on one GPU)."""
    if dist is not None:
        dist.barrier()


def max_over(dist, v, device):
    """The maximum of a per-rank time over all replica ranks (the slowest rank sets the clock)."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world, steps, ms):
    """Whole-job units per second: every rank processed `steps` units in `ms` (the max over ranks)."""
    return world * steps / (ms / 1000.0)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-rows", action="store_true", help="skip the extra scope rows")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--profile", default=None, choices=sorted(PROFILE_CASES),
                    help="run one small case 4 times (3 warm-up launches + 1) for an ncu capture, then exit")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        rank_barrier(dist)

    def max_over_ranks(v):
        return max_over(dist, v, "cuda")

    import bit_gemv_tern_b200 as tg
    from bit_gemv_tern_b200 import build as _b
    _b.build()
    hbm_peak, bf16_peak, bf16_sust, peak_kind = peaks()
    if args.profile:
        return run_profile_case(args.profile)

    stack = Stack("8b", M=1)
    n_linear = len(stack.linears)
    S = min(args.steps, 100)
    R, rem = divmod(args.steps, S)
    ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(S)]

    # One step = the stack's two launches (operand prep, persistent stream) then the head. The
    # kernels of a step are launched without programmatic dependent launch: a head launched early
    # only waits resident next to the stream's tail, and measured slower (the stream kernel itself
    # always overlaps its own prep).
    def step_plain(i):
        stack.launch_stack("bf16", pdl=False)
        stack.launch_head("bf16", pdl=False)

    def step_events(i):
        ev[i][0].record()
        stack.launch_stack("bf16", pdl=False)
        ev[i][1].record()
        stack.launch_head("bf16", pdl=False)
        ev[i][2].record()

    g_main = capture(step_plain, S)
    g_rem = capture(step_plain, rem) if rem else None
    g_warm = capture(step_plain, args.warmup)
    g_warm.replay()
    torch.cuda.synchronize()

    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = timed_replays([(g_main, R)] + ([(g_rem, 1)] if g_rem else []))
    barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(ms)
    clocks = clk.summary()
    ms_step = ms / args.steps
    value = replica_throughput(world, args.steps, ms)

    # dominant kernel: the batched stream of the stack, timed per step with CUDA events recorded on
    # the launching stream between the step's launches (a second timed pass over S steps, so that
    # the events do not sit inside the throughput's timed region)
    g_ev = capture(step_events, S)
    g_ev.replay()
    torch.cuda.synchronize()
    timed_replays([(g_ev, 1)])
    stack_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(S)]
    head_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(S)]
    gemv_s = statistics.median(stack_ms) / 1000.0
    gemv_gbs = stack.stack_bytes / gemv_s / 1e9
    head_gbs = stack.head_bytes / (statistics.median(head_ms) / 1000.0) / 1e9
    step_bytes = stack.stack_bytes + stack.head_bytes
    del g_ev

    # end to end through the C ABI: H2D of the step's activations, the step, D2H of the argmax
    g_one = capture(step_plain, 1)
    n_e2e = min(args.steps, 300)
    res = torch.empty(2, dtype=torch.int32, device="cuda")
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(n_e2e):
        stack.x.copy_(stack.x_host, non_blocking=True)
        g_one.replay()
        res[0:1].copy_(stack.argmax)
        res[1:2].copy_(stack.maxval.view(torch.int32))
        stack.result_host.copy_(res, non_blocking=True)
        torch.cuda.current_stream().synchronize()
    e2e_s = max_over_ranks(time.perf_counter() - t0)
    e2e = {"value": world * n_e2e / e2e_s, "unit": "tok/s",
           "h2d_bytes_per_step": int(stack.x_host.numel() * 2), "d2h_bytes_per_step": 8, "steps": n_e2e,
           "note": "per step: pinned-host activations -> device, graph of the step's launches, argmax + max logit -> host, stream sync"}

    rows = {}
    if not args.no_rows:
        rows = extra_rows(stack, torch, tg, hbm_peak, bf16_peak)
    cb = None
    if rank == 0 and not args.no_cpu:
        cb = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "8b_linear_stack_m1_bf16_plus_int8_head",
                       "model": "neutrino-1-8b-geometry (36 x 7 ternary linears as 144 fused launches + int8 head 151936x4096)",
                       "global_batch": world, "seq_len": 1, "parallelism": f"replicas x{world}" if world > 1 else "none",
                       "step_bytes": step_bytes, "l2": "inputs larger than L2: every step streams 2.37 GB of weights from HBM",
                       "graph": f"{S}-step CUDA graph x {R}" + (f" + {rem}-step graph" if rem else "") + ", no events inside; per-kernel times from a second pass with events"},
            "gbs": step_bytes / (ms_step / 1000.0) / 1e9,
            "hbm_frac_step": step_bytes / (ms_step / 1000.0) / 1e9 / hbm_peak,
            "roofline": {"bound": "hbm", "kernel": "k_batch_prep + k_batch_stream<bf16> (all 144 fused GEMVs of the step in one persistent launch)",
                         "achieved": gemv_gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gemv_gbs / hbm_peak,
                         "peak_kind": f"{peak_kind} hbm_gbs (copy)", "traffic": STREAM_TRAFFIC_PER_STEP,
                         "traffic_note": "dram read+write bytes per step, ncu capture of 4 layers x 9",
                         "algorithmic_bytes_per_step": stack.stack_bytes, "launches": n_linear,
                         "head": {"kernel": "k_head<bf16,1>", "achieved": head_gbs, "frac": head_gbs / hbm_peak}},
            "cpu_baseline": cb,
            "e2e": e2e,
            "clocks": clocks,
            "gpu_launches": stack.launches_per_step * args.steps,
            "rows": rows,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _profile_batch(mode):
    def run():
        st = Stack("8b", M=1, layers=4)
        return lambda: st.launch_stack(mode)
    return run


def _profile_smallm(M, tc=False):
    def run():
        st = Stack("8b", M=1, layers=4)
        sv = StackView(st, M)
        return lambda: sv.launch_stack("bf16", tc=tc)
    return run


def _profile_chain(mode):
    def run():
        st = Stack("8b", M=1, layers=4)
        ch = Chain(st, mode)
        return ch.chain
    return run


def _profile_head(mode):
    def run():
        st = Stack("8b", M=1, layers=0)
        return lambda: st.launch_head(mode)
    return run


def _profile_prefill(proj):
    def run():
        ps = PrefillSet(M=4096, projs=(proj,))
        return ps.launch
    return run


def _profile_base3():
    def run():
        import torch
        import synth
        import synth.cuda as sc
        import bit_gemv_tern_b200 as tg
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        items = []
        for p, N, K in synth.linear_shapes("8b"):
            t = torch.empty(N * K, dtype=torch.int8, device="cuda")
            sc.trits_into(t, SEED, synth.tensor_id(0, p), K)
            e = torch.empty(tg.tern_base3_bytes(N, K), dtype=torch.uint8, device="cuda")
            tg.tern_base3_encode(t, N, K, e, flag)
            del t
            items.append((e, N, K, torch.empty(N * K // 16, dtype=torch.int32, device="cuda")))
        return lambda: tg.tern_pack_batch(tg.TERN_SRC_BASE3, items, flag)
    return run


def _profile_fv5():
    def run():
        import torch
        import synth
        import synth.cuda as sc
        import bit_gemv_tern_b200 as tg
        gen = torch.Generator(device="cuda").manual_seed(SEED)
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        entries = []
        for p, N, K in synth.linear_shapes("8b"):
            t = torch.empty(N * K, dtype=torch.int8, device="cuda")
            h = torch.empty(N * K, dtype=torch.int8, device="cuda")
            sc.trits_into(t, SEED, synth.tensor_id(1, p), K)
            sc.trits_into(h, SEED + 1, synth.tensor_id(1, p), K)
            codes = t * (1 + (h == 1).to(torch.int8))
            del t, h
            planes = torch.empty(N * 3 * K // 32, dtype=torch.int32, device="cuda")
            tg.tern_fv5_pack(codes, N, K, planes, flag)
            del codes
            lo = 0.01 + 0.04 * torch.rand(N * (K // 256), device="cuda", generator=gen)
            scales = torch.stack([lo, lo * (2 + torch.rand(N * (K // 256), device="cuda", generator=gen))], 1).contiguous()
            x = torch.from_numpy(synth.activations(SEED, 8000 + K, 1, K).view(np.int16)).cuda()
            entries.append((tg.Fv5Matrix(planes, scales, N, K), x, None, torch.empty(N, dtype=torch.float32, device="cuda")))
        return lambda: tg.tern_fv5_gemv_batch(entries, tg.TERN_ACT_BF16)
    return run


def _profile_pack():
    def run():
        import torch
        import synth
        import synth.cuda as sc
        import bit_gemv_tern_b200 as tg
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        items = []
        for p, N, K in synth.linear_shapes("8b"):
            t = torch.empty(N * K, dtype=torch.int8, device="cuda")
            sc.trits_into(t, SEED, synth.tensor_id(0, p), K)
            items.append((t, N, K, torch.empty(N * K // 16, dtype=torch.int32, device="cuda")))
        return lambda: tg.tern_pack_batch(tg.TERN_SRC_INT8_TRITS, items, flag)
    return run


# Small cases for ncu captures (inputs > L2, a few hundred MB on the device):
#   batch-8b-4layers-*: 4 layers of the 8B stack (16 fused GEMVs, 193 MB of planes) as one batch
#   head-8b-*:          the int8 head 151936 x 4096 (622 MB)
#   prefill-8b-gate-*:  one 12288 x 4096 linear at M = 4096 tokens (tcgen05 prefill)
#   base3-8b-1layer:    the transport of one 8B layer's seven tensors (86.9 MB) in one batched call
#   fv5-8b-1layer-batched: one 8B layer's seven linears as five-valued weights (78.6 MB), M = 1, bf16,
#                       in one tern_fv5_gemv_batch call
#   pack-8b-1layer:     the int8 trits of one 8B layer's seven tensors (193 MB) in one batched call
#   smallm-8b-4layers-m8-bf16(-tc): the 16 fused GEMVs of 4 layers at M = 8 in bf16 mode, on the
#                       default (mma.sync) kernels or, with -tc, on the tcgen05 ones
PROFILE_CASES = {
    "batch-8b-4layers-bf16": _profile_batch("bf16"),
    "batch-8b-4layers-int8": _profile_batch("int8"),
    "head-8b-bf16": _profile_head("bf16"),
    "smallm-8b-4layers-m8-bf16": _profile_smallm(8),
    "smallm-8b-4layers-m8-bf16-tc": _profile_smallm(8, tc=True),
    "chain-8b-4layers-bf16": _profile_chain("bf16"),
    "prefill-8b-gate-m4096": _profile_prefill("gate"),
    "base3-8b-1layer": _profile_base3(),
    "fv5-8b-1layer-batched": _profile_fv5(),
    "pack-8b-1layer": _profile_pack(),
}


def run_profile_case(name):
    import torch
    import bit_gemv_tern_b200 as tg
    fn = PROFILE_CASES[name]()
    for _ in range(4):
        fn()
    torch.cuda.synchronize()
    st = tg.tern_device_status()
    print(f"profile case {name}: status {st}", flush=True)
    return 0 if st == tg.TERN_OK else 1


def gbs_of(nbytes, ms):
    return nbytes / (ms / 1000.0) / 1e9


def extra_rows(stack, torch, tg, hbm_peak, bf16_peak):
    """The other scope rows, each timed with CUDA events over graph replays."""
    out = {}

    # int8-activation mode on the same 8B stack, every quantisation inside the step (the stack's
    # quantiser fused into its prep launch, one quantiser launch for the head input)
    reps = 50
    g = capture(lambda i: stack.launch_step_int8_fused(), 10)
    g.replay()
    ms = timed_replays([(g, reps // 10)]) / reps
    nb = stack.stack_bytes + stack.head_bytes
    out["8b_stack_m1_int8"] = {"tok_s": 1000.0 / ms, "ms": ms, "gbs": gbs_of(nb, ms), "frac": gbs_of(nb, ms) / hbm_peak,
                               "launches_per_step": 4,
                               "note": "bf16 activations in; quantiser fused into the batch prep; head input quantised in the step"}
    # the same with activations quantised once before the timed region (kernel-only comparison)
    g = capture(lambda i: (stack.launch_stack("int8"), stack.launch_head("int8")), 10)
    g.replay()
    ms = timed_replays([(g, reps // 10)]) / reps
    nb = stack.stack_bytes - sum(l.K for l in stack.linears) + stack.head_bytes - stack.d
    out["8b_stack_m1_int8_prequantised"] = {"tok_s": 1000.0 / ms, "ms": ms, "gbs": gbs_of(nb, ms),
                                            "frac": gbs_of(nb, ms) / hbm_peak}
    # a decode chain whose linears depend on one another through their prologues
    out["8b_decode_chain_m1"] = chain_row(stack, torch, hbm_peak)
    # speculative-verify rounds: k drafts + 1 through the stack and the head with on-device acceptance
    out["verify_round_8b_bf16"] = verify_rows(stack, torch, tg, hbm_peak)
    # decode-chain variant: one launch per fused linear, each waiting for its predecessor (PDL)
    g = capture(lambda i: (stack.launch_stack("bf16", pdl=True, chained=True), stack.launch_head("bf16")), 10)
    g.replay()
    ms = timed_replays([(g, 5)]) / 50
    nb = stack.stack_bytes + stack.head_bytes
    out["8b_stack_m1_bf16_chained"] = {"tok_s": 1000.0 / ms, "ms": ms, "gbs": gbs_of(nb, ms), "frac": gbs_of(nb, ms) / hbm_peak,
                                      "launches_per_step": len(stack.linears) + 1}
    # stack only (no head), bf16
    g = capture(lambda i: stack.launch_stack("bf16"), 10)
    g.replay()
    ms = timed_replays([(g, 5)]) / 50
    out["8b_stack_only_m1_bf16"] = {"tok_s": 1000.0 / ms, "ms": ms, "gbs": gbs_of(stack.stack_bytes, ms),
                                    "frac": gbs_of(stack.stack_bytes, ms) / hbm_peak}

    # single GEMV 3072 x 1024 (the small configuration), L2 defeated by rotating replicas
    import synth
    reps_w = int(math.ceil(3 * L2_BYTES / (3072 * 1024 // 4)))
    lin = build_linear("0.6b", 0, ("gate",))
    planes = torch.empty(reps_w * lin.W.planes.numel(), dtype=torch.int32, device="cuda")
    for r in range(reps_w):
        planes[r * lin.W.planes.numel():(r + 1) * lin.W.planes.numel()].copy_(lin.W.planes)
    mats = [tg.TernMatrix(planes[r * lin.W.planes.numel():(r + 1) * lin.W.planes.numel()], lin.W.scale, 3072, 1024)
            for r in range(reps_w)]
    x = torch.from_numpy(synth.activations(SEED, 7, 1, 1024).view(np.int16)).cuda()
    y = torch.empty(3072, dtype=torch.float32, device="cuda")
    g = capture(lambda i: tg.tern_gemv(mats[i], tg.TERN_ACT_BF16, x, None, y, flags=tg.TERN_FLAG_PDL), reps_w)
    g.replay()
    ms = timed_replays([(g, 4)]) / (4 * reps_w)
    out["gemv_3072x1024_bf16"] = {"us": ms * 1000.0, "gbs": gbs_of(lin.bytes, ms), "frac": gbs_of(lin.bytes, ms) / hbm_peak,
                                  "replicas": reps_w}
    del planes, mats

    # 0.6B stack + tied head (the second configuration)
    s06 = Stack("0.6b", M=1)
    g = capture(lambda i: (s06.launch_stack("bf16"), s06.launch_head("bf16")), 20)
    g.replay()
    ms = timed_replays([(g, 10)]) / 200
    nb = s06.stack_bytes + s06.head_bytes
    out["0.6b_stack_m1_bf16"] = {"tok_s": 1000.0 / ms, "ms": ms, "gbs": gbs_of(nb, ms), "frac": gbs_of(nb, ms) / hbm_peak,
                                 "launches_per_step": s06.launches_per_step}
    del s06

    # small-M sweep on the 8B stack + head (speculative verify)
    out["small_m_8b_bf16"] = small_m_sweep(stack, hbm_peak)

    # prefill: M = 4096 tokens through each of the 7 distinct 8B linear shapes (tcgen05)
    out["prefill_8b_m4096"] = prefill_row(torch, tg, bf16_peak)

    # pack of int8 trits into the planes: the seven tensors of one 8B layer per call
    out["pack_8b_layer"] = pack_row(torch, tg, hbm_peak)

    # base-3 transport unpack of all 8B trits (bit-exact expansion into the planes)
    out["base3_unpack_8b"] = base3_row(stack, torch, tg, hbm_peak)
    # order-0 rANS transport of all 8B trits: decode into the planes in one launch
    out["rans_decode_8b"] = rans_row(torch, tg, hbm_peak)
    # five-valued (FV5-style) weights and the block-scaled (FV5B-style) head
    out["fv5_8b"] = fv5_rows(stack, torch, tg, hbm_peak)
    return out


class Chain:
    """One decode token through the 8B stack as a dependent chain in one cooperative launch
    (tern_chain_run): each fused linear's activation is computed from an earlier linear's output.
    Per layer: q|k|v <- RMSNorm(h); o <- cast of the q part of the q|k|v output (standing in for
    attention, which is not a linear); gate|up <- RMSNorm(o output), its SwiGLU fused into its
    epilogue (gate and up rows interleaved); down <- that SwiGLU; the next layer's h = the down
    output. No residual adds (not part of the path). Then the head on the RMSNorm of the last h (a
    prologue launch and the head launch). Weights are the stack's; gains and the entry h are seeded
    synthetic inputs."""

    def __init__(self, stack, mode="bf16"):
        import torch
        import synth
        import bit_gemv_tern_b200 as tg
        self.stack, self.mode = stack, mode
        act = tg.TERN_ACT_BF16 if mode == "bf16" else tg.TERN_ACT_INT8
        d = stack.d
        self.h0 = torch.from_numpy(synth.residual(SEED, 0, 1, d).reshape(-1)).cuda()
        self.gains = [torch.from_numpy(synth.norm_gains(SEED, i, d).view(np.int16)).cuda() for i in range(2 * stack.L + 1)]
        self.h = {}
        self.sx = torch.empty(len(stack.linears), dtype=torch.float32, device="cuda")
        items = []
        for i, lin in enumerate(stack.linears):
            layer, grp = divmod(i, 4)
            sx = self.sx[i:i + 1] if act == tg.TERN_ACT_INT8 else None
            if grp == 0:
                it = tg.ChainItem(lin.W, tg.TERN_PRO_RMSNORM, stack.y[i], src_item=i - 1 if i else -1,
                                  src=None if i else self.h0, gain=self.gains[2 * layer], eps=1e-6, x_scale=sx)
            elif grp == 1:
                it = tg.ChainItem(lin.W, tg.TERN_PRO_CAST, stack.y[i], src_item=i - 1, x_scale=sx)
            elif grp == 2:
                self.h[i] = torch.empty(lin.N // 2, dtype=torch.int16, device="cuda")
                it = tg.ChainItem(lin.W, tg.TERN_PRO_RMSNORM, stack.y[i], src_item=i - 1, gain=self.gains[2 * layer + 1],
                                  eps=1e-6, swiglu_out=True, h=self.h[i], x_scale=sx)
            else:
                it = tg.ChainItem(lin.W, tg.TERN_PRO_BF16, stack.y[i], src_item=i - 1, src_h=True, x_scale=sx)
            items.append(it)
        self.chain = tg.Chain(items, act)
        self.last = stack.y[len(stack.linears) - 1]
        self.x_head = torch.empty(d, dtype=torch.int16, device="cuda")
        self.q_head = torch.empty(d, dtype=torch.int8, device="cuda")
        self.sx_head = torch.empty(1, dtype=torch.float32, device="cuda")

    def launch(self):
        import bit_gemv_tern_b200 as tg
        st = self.stack
        self.chain()
        tg.tern_act_prologue(tg.TERN_PRO_RMSNORM, self.last, self.gains[-1], 1e-6, 1, st.d, self.x_head)
        if self.mode == "bf16":
            tg.i8_head_gemv_argmax(st.head_W, st.head_s, st.V, st.d, 1, tg.TERN_ACT_BF16, self.x_head, None,
                                   st.argmax, st.maxval, None, st.ws)
        else:
            tg.tern_quantize_act(self.x_head, 1, st.d, self.q_head, self.sx_head)
            tg.i8_head_gemv_argmax(st.head_W, st.head_s, st.V, st.d, 1, tg.TERN_ACT_INT8, self.q_head, self.sx_head,
                                   st.argmax, st.maxval, None, st.ws)

    @property
    def launches(self):
        return 3 + (1 if self.mode == "int8" else 0)


def _timed_direct(fn, n):
    """fn() launched n times between two events on the current stream; returns elapsed ms."""
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(n):
        fn()
    b.record()
    b.synchronize()
    return a.elapsed_time(b)


def chain_row(stack, torch, hbm_peak):
    """The dependent decode chain, timed as direct launches (the chain kernel is a cooperative launch;
    a CUDA graph of it is tried too and reported when capture succeeds)."""
    import bit_gemv_tern_b200 as tg
    out = {}
    for mode in ("bf16", "int8"):
        ch = Chain(stack, mode)
        for _ in range(3):
            ch.launch()
        torch.cuda.synchronize()
        assert tg.tern_device_status() == tg.TERN_OK
        ms = _timed_direct(ch.launch, 50) / 50
        mc = _timed_direct(ch.chain, 50) / 50
        assert tg.tern_device_status() == tg.TERN_OK
        nb = stack.stack_bytes + stack.head_bytes
        row = {"tok_s": 1000.0 / ms, "ms": ms, "gbs": nb / (ms / 1000.0) / 1e9,
               "frac": nb / (ms / 1000.0) / 1e9 / hbm_peak, "launches_per_token": ch.launches,
               "chain_kernel_ms": mc, "chain_kernel_frac": stack.stack_bytes / (mc / 1000.0) / 1e9 / hbm_peak,
               "timing": "direct launches"}
        try:
            g = capture(lambda i: ch.launch(), 10)
            g.replay()
            torch.cuda.synchronize()
            mg = timed_replays([(g, 5)]) / 50
            row["graph_ms"], row["graph_tok_s"] = mg, 1000.0 / mg
            del g
        except Exception as e:                    # capture of a cooperative launch refused
            row["graph"] = "capture failed: %s" % str(e).splitlines()[0][:120]
            torch.cuda.synchronize()
        out[mode] = row
        del ch
    return out


def small_m_sweep(stack, hbm_peak, Ms=(1, 2, 3, 4, 5, 6, 7, 8, 12, 16)):
    """One pass of M rows through the 8B stack + head per M (bf16): mma.sync kernels up to M = 8,
    tcgen05 from M = 9. Then the stack alone in int8 mode at M = 5, 8, 16 on both kernel families
    (activations quantised once)."""
    out = {}
    for M in Ms:
        sm = stack if M == 1 else StackView(stack, M)
        g = capture(lambda i: (sm.launch_stack("bf16"), sm.launch_head("bf16")), 5)
        g.replay()
        ms = timed_replays([(g, 4)]) / 20
        nb = sm.stack_bytes + sm.head_bytes
        out[str(M)] = {"pass_us": ms * 1000.0, "frac": gbs_of(nb, ms) / hbm_peak, "tokens_per_s": M * 1000.0 / ms,
                       "gbs": gbs_of(nb, ms), "launches_per_pass": 3, "kernel": "tcgen05" if M >= 9 else "mma.sync"}
        del g
    int8 = {}
    for M in (5, 8, 16):
        sm = StackView(stack, M)
        row = {}
        for name, tc in (("tcgen05", True), ("mma_sync", False)):
            g = capture(lambda i: sm.launch_stack("int8", tc=tc), 5)
            g.replay()
            ms = timed_replays([(g, 4)]) / 20
            nb = sm.stack_bytes - sum(l.K for l in sm.linears) * M
            row[name + "_pass_us"] = ms * 1000.0
            row[name + "_frac"] = gbs_of(nb, ms) / hbm_peak
            del g
        int8[str(M)] = row
    out["int8_stack_only"] = int8
    return out


def verify_rows(stack, torch, tg, hbm_peak):
    """k drafted tokens + 1 through the 8B stack (one small-M batch) and the head with the acceptance
    count on the device. Drafts equal to the target's own greedy tokens (from a previous pass) give
    the all-accepted round (k + 1 tokens); drafts that all miss give 1 token."""
    out = {}
    for k in (1, 3, 6):
        M = k + 1
        sv = StackView(stack, M)
        accept = torch.empty(2, dtype=torch.int32, device="cuda")
        draft = torch.empty(k, dtype=torch.int32, device="cuda")
        sv.launch_stack("bf16")
        sv.launch_head("bf16")
        torch.cuda.synchronize()
        hits = sv.argmax[:k].clone()

        def round_(i):
            sv.launch_stack("bf16")
            tg.i8_head_verify(stack.head_W, stack.head_s, sv.V, sv.d, M, tg.TERN_ACT_BF16, sv.x[:M * sv.d], None,
                              draft, sv.argmax, sv.maxval, accept, sv.ws)
        row = {}
        for case, d in (("all_accepted", hits), ("none_accepted", hits + 1)):
            draft.copy_(d)
            g = capture(round_, 5)
            g.replay()
            torch.cuda.synchronize()
            n = int(accept[0].item())
            ms = timed_replays([(g, 4)]) / 20
            row[case] = {"pass_us": ms * 1000.0, "accepted": n, "tokens_per_round": n + 1,
                         "tokens_per_s": (n + 1) * 1000.0 / ms}
            del g
        nb = sv.stack_bytes + sv.head_bytes
        row["frac_hbm"] = nb / (row["all_accepted"]["pass_us"] / 1e6) / 1e9 / hbm_peak
        out[f"k{k}"] = row
        del sv
    return out


class PrefillSet:
    """The seven distinct 8B linear shapes (layer 0 weights) with M bf16 activation rows each."""

    def __init__(self, M=4096, projs=("q", "k", "v", "o", "gate", "up", "down")):
        import torch
        import synth
        self.M = M
        self.lins = [build_linear("8b", 0, (p,)) for p in projs]
        self.X = {}
        for lin in self.lins:
            if lin.K not in self.X:
                self.X[lin.K] = torch.from_numpy(synth.activations(SEED, 6000 + lin.K, M, lin.K).view(np.int16)).cuda()
        self.Y = [torch.empty(M * lin.N, dtype=torch.float32, device="cuda") for lin in self.lins]

    @property
    def flops(self):
        return sum(2.0 * self.M * lin.N * lin.K for lin in self.lins)

    def launch(self):
        import bit_gemv_tern_b200 as tg
        for lin, y in zip(self.lins, self.Y):
            tg.tern_gemm_prefill(lin.W, self.M, self.X[lin.K], y)


def prefill_row(torch, tg, bf16_peak):
    ps = PrefillSet()
    g = capture(lambda i: ps.launch(), 1)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    reps = 10
    ms = timed_replays([(g, reps)]) / reps
    tf = ps.flops / (ms / 1000.0) / 1e12
    st = tg.tern_device_status()
    per = {}
    for lin, y in zip(ps.lins, ps.Y):
        g1 = capture(lambda i, lin=lin, y=y: tg.tern_gemm_prefill(lin.W, ps.M, ps.X[lin.K], y), 1)
        g1.replay()
        m1 = timed_replays([(g1, reps)]) / reps
        per["x".join(map(str, (lin.N, lin.K)))] = {"ms": m1, "tflops": 2.0 * ps.M * lin.N * lin.K / (m1 / 1000.0) / 1e12}
    del ps
    return {"ms_per_set": ms, "tflops": tf, "frac": tf / bf16_peak, "peak": f"{peaks()[3]} bf16 dense (burst)",
            "flops_per_set": 1.5805e12, "status": st, "shapes": per}


class StackView:
    """The 8B stack's weights with M activation rows (for the small-M sweep)."""

    def __init__(self, base, M):
        import torch
        import synth
        self.base, self.M, self.linears, self.V, self.d = base, M, base.linears, base.V, base.d
        self.x = torch.from_numpy(synth.activations(SEED, 5000 + M, M, 12288).view(np.int16)).cuda()
        self.y = [torch.empty(M * l.N, dtype=torch.float32, device="cuda") for l in base.linears]
        self.argmax = torch.empty(M, dtype=torch.int32, device="cuda")
        self.maxval = torch.empty(M, dtype=torch.float32, device="cuda")
        import bit_gemv_tern_b200 as tg
        self.ws = torch.zeros(tg.i8_head_workspace_bytes(self.V, M), dtype=torch.uint8, device="cuda")

    stack_bytes = Stack.stack_bytes
    head_bytes = Stack.head_bytes

    def launch_stack(self, mode="bf16", pdl=False, tc=False):
        """All 144 fused linears as one batched small-M launch pair (each reads its X [M][K]; int8
        mode: q [M][K] and s_x [M], quantised once); tc: the tcgen05 kernels where the mma.sync
        ones are the default (every list but bf16 of 9..16 rows)."""
        import torch
        import bit_gemv_tern_b200 as tg
        key = "_batch_" + mode
        if not hasattr(self, key):
            if mode == "bf16":
                entries = [(lin.W, self.x[:self.M * lin.K], None, self.y[i]) for i, lin in enumerate(self.linears)]
                setattr(self, key, tg.GemvBatch(entries, tg.TERN_ACT_BF16, M=self.M))
            else:
                self.q = torch.empty(self.M * 12288, dtype=torch.int8, device="cuda")
                self.sxq = torch.empty(self.M, dtype=torch.float32, device="cuda")
                self.qk = {}
                entries = []
                for i, lin in enumerate(self.linears):
                    if lin.K not in self.qk:
                        q = torch.empty(self.M * lin.K, dtype=torch.int8, device="cuda")
                        sx = torch.empty(self.M, dtype=torch.float32, device="cuda")
                        tg.tern_quantize_act(self.x[:self.M * lin.K], self.M, lin.K, q, sx)
                        self.qk[lin.K] = (q, sx)
                    q, sx = self.qk[lin.K]
                    entries.append((lin.W, q, sx, self.y[i]))
                setattr(self, key, tg.GemvBatch(entries, tg.TERN_ACT_INT8, M=self.M))
        getattr(self, key)(flags=(tg.TERN_FLAG_PDL if pdl else 0) | (tg.TERN_FLAG_TCGEN05 if tc else 0))

    def launch_head(self, mode="bf16", pdl=False):
        import bit_gemv_tern_b200 as tg
        tg.i8_head_gemv_argmax(self.base.head_W, self.base.head_s, self.V, self.d, self.M, tg.TERN_ACT_BF16,
                               self.x[:self.M * self.d], None, self.argmax, self.maxval, None, self.ws,
                               flags=tg.TERN_FLAG_PDL if pdl else 0)


def pack_row(torch, tg, hbm_peak):
    """int8 trits of the seven tensors of one 8B layer (193 MB, > L2) packed into their planes by
    one tern_pack_batch call (one launch); bytes = N*K in + N*K/4 out per tensor."""
    import synth
    import synth.cuda as sc
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    items, nb, trits = [], 0, 0
    for p, N, K in synth.linear_shapes("8b"):
        t = torch.empty(N * K, dtype=torch.int8, device="cuda")
        sc.trits_into(t, SEED, synth.tensor_id(1, p), K, synth.trit_probs("8b", 1, p))
        items.append((t, N, K, torch.empty(N * K // 16, dtype=torch.int32, device="cuda")))
        nb += N * K + N * K // 4
        trits += N * K
    g = capture(lambda i: tg.tern_pack_batch(tg.TERN_SRC_INT8_TRITS, items, flag), 1)
    g.replay()
    reps = 10
    ms = timed_replays([(g, reps)]) / reps
    assert tg.tern_read_flag(flag) == 0
    gbs = nb / (ms / 1000.0) / 1e9
    layers = synth.GEOMETRY["8b"]["layers"]
    return {"ms": ms, "gbs": gbs, "frac": gbs / hbm_peak, "trits": trits, "bytes": nb, "tensors": len(items),
            "launches": 1, "ms_8b_equivalent": ms * layers}


def base3_row(stack, torch, tg, hbm_peak):
    """All 252 ternary tensors of the 8B (6.95e9 trits) expanded from the base-3 transport into
    the planes by one tern_pack_batch call (one launch)."""
    import synth
    import synth.cuda as sc
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    items, nb, trits = [], 0, 0
    L = synth.GEOMETRY["8b"]["layers"]
    for layer in range(L):
        for p, N, K in synth.linear_shapes("8b"):
            t = torch.empty(N * K, dtype=torch.int8, device="cuda")
            sc.trits_into(t, SEED, synth.tensor_id(layer, p), K, synth.trit_probs("8b", layer, p))
            e = torch.empty(tg.tern_base3_bytes(N, K), dtype=torch.uint8, device="cuda")
            tg.tern_base3_encode(t, N, K, e, flag)
            del t
            items.append((e, N, K, torch.empty(N * K // 16, dtype=torch.int32, device="cuda")))
            nb += e.numel() + N * K // 4
            trits += N * K
    assert tg.tern_read_flag(flag) == 0
    g = capture(lambda i: tg.tern_pack_batch(tg.TERN_SRC_BASE3, items, flag), 1)
    g.replay()
    reps = 5
    ms = timed_replays([(g, reps)]) / reps
    assert tg.tern_read_flag(flag) == 0
    out = {"ms": ms, "gbs": nb / (ms / 1000.0) / 1e9, "frac": nb / (ms / 1000.0) / 1e9 / hbm_peak,
           "trits": trits, "bytes": nb, "tensors": len(items), "launches": 1}
    del items
    return out


def rans_row(torch, tg, hbm_peak):
    """All 252 ternary tensors of the 8B coded by the device encoder (order-0 rANS, one stream per
    row), then decoded into their planes by one tern_rans_decode call (one launch). Bytes = payload
    + row ends read, planes written."""
    import synth
    import synth.cuda as sc
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    L = synth.GEOMETRY["8b"]["layers"]
    shapes = synth.linear_shapes("8b")
    Nmax = max(N for _, N, _ in shapes)
    Kmax = max(K for _, _, K in shapes)
    bound = max(tg.tern_rans_payload_bound(N, K) for _, N, K in shapes)
    ws = torch.empty(max(tg.tern_rans_workspace_bytes(N, K) for _, N, K in shapes), dtype=torch.uint8, device="cuda")
    buf = torch.empty(bound, dtype=torch.uint8, device="cuda")
    t = torch.empty(Nmax * Kmax, dtype=torch.int8, device="cuda")
    entries, payload_bytes, trits = [], 0, 0
    for layer in range(L):
        for p, N, K in shapes:
            sc.trits_into(t[:N * K], SEED, synth.tensor_id(layer, p), K, synth.trit_probs("8b", layer, p))
            freq = torch.empty(3, dtype=torch.int16, device="cuda")
            row_end = torch.empty(N, dtype=torch.int32, device="cuda")
            tg.tern_rans_encode(t[:N * K], N, K, freq, row_end, buf, ws, flag)
            assert tg.tern_read_flag(flag) == 0
            n = int(row_end[-1].item()) & 0xFFFFFFFF
            payload = buf[:n].clone()
            entries.append((freq, row_end, payload, N, K, torch.empty(N * K // 16, dtype=torch.int32, device="cuda")))
            payload_bytes += n + 4 * N
            trits += N * K
    del t, ws, buf
    g = capture(lambda i: tg.tern_rans_decode(entries, flag), 1)
    g.replay()
    reps = 3
    ms = timed_replays([(g, reps)]) / reps
    assert tg.tern_read_flag(flag) == 0
    nb = payload_bytes + trits // 4
    out = {"ms": ms, "gbs": nb / (ms / 1000.0) / 1e9, "frac": nb / (ms / 1000.0) / 1e9 / hbm_peak,
           "trits": trits, "transport_bytes": payload_bytes, "bits_per_trit": 8.0 * payload_bytes / trits,
           "tensors": len(entries), "launches": 1}
    del entries
    return out


def fv5_rows(stack, torch, tg, hbm_peak):
    """Three 8B layers' seven linears (21 launches, 235 MB > L2) as five-valued weights at M = 1
    (codes: the 8B trits, magnitude 2 where a second trit stream draws +1; fp32 s_lo in
    [0.01, 0.05), s_hi = 2..3 x s_lo, seeded), then the FV5B-style head 151936 x 4096 (the stack's
    int8 head weights with one fp32 scale per 256-weight block). bf16 activations."""
    import synth
    import synth.cuda as sc
    gen = torch.Generator(device="cuda").manual_seed(SEED)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    mats, xs, ys, nbytes = [], {}, [], 0
    for layer in range(1, 4):
        for p, N, K in synth.linear_shapes("8b"):
            t = torch.empty(N * K, dtype=torch.int8, device="cuda")
            h = torch.empty(N * K, dtype=torch.int8, device="cuda")
            sc.trits_into(t, SEED, synth.tensor_id(layer, p), K, synth.trit_probs("8b", layer, p))
            sc.trits_into(h, SEED + 1, synth.tensor_id(layer, p), K)
            codes = t * (1 + (h == 1).to(torch.int8))
            del t, h
            planes = torch.empty(N * 3 * K // 32, dtype=torch.int32, device="cuda")
            tg.tern_fv5_pack(codes, N, K, planes, flag)
            del codes
            lo = 0.01 + 0.04 * torch.rand(N * (K // 256), device="cuda", generator=gen)
            hi = lo * (2 + torch.rand(N * (K // 256), device="cuda", generator=gen))
            scales = torch.stack([lo, hi], 1).contiguous()
            mats.append(tg.Fv5Matrix(planes, scales, N, K))
            if K not in xs:
                xs[K] = torch.from_numpy(synth.activations(SEED, 8000 + K, 1, K).view(np.int16)).cuda()
            ys.append(torch.empty(N, dtype=torch.float32, device="cuda"))
            nbytes += N * K * 3 // 8 + N * (K // 256) * 8 + 2 * K + 4 * N
    assert tg.tern_read_flag(flag) == 0

    def pass_(i):
        for W, y in zip(mats, ys):
            tg.tern_fv5_gemm(W, 1, tg.TERN_ACT_BF16, xs[W.K], None, y)
    g = capture(pass_, 2)
    g.replay()
    torch.cuda.synchronize()
    ms = timed_replays([(g, 5)]) / 10
    out = {"linears_3_layers_m1_bf16": {"ms": ms, "gbs": nbytes / (ms / 1000.0) / 1e9,
                                        "frac": nbytes / (ms / 1000.0) / 1e9 / hbm_peak, "bytes": nbytes,
                                        "launches": len(mats), "bits_per_weight": 3.25}}
    del g
    # the same 21 linears as one tern_fv5_gemv_batch call (one persistent launch)
    entries = [(W, xs[W.K], None, y) for W, y in zip(mats, ys)]
    g = capture(lambda i: tg.tern_fv5_gemv_batch(entries, tg.TERN_ACT_BF16), 2)
    g.replay()
    torch.cuda.synchronize()
    ms = timed_replays([(g, 5)]) / 10
    out["linears_3_layers_m1_bf16_batched"] = {"ms": ms, "gbs": nbytes / (ms / 1000.0) / 1e9,
                                               "frac": nbytes / (ms / 1000.0) / 1e9 / hbm_peak, "launches": 1}
    del mats, g, entries
    V, d = stack.V, stack.d
    S = (0.001 + 0.02 * torch.rand(V * (d // 256), device="cuda", generator=gen)).contiguous()
    xb = torch.from_numpy(synth.activations(SEED, 8100, 1, d).view(np.int16)).cuda()
    am = torch.empty(1, dtype=torch.int32, device="cuda")
    mv = torch.empty(1, dtype=torch.float32, device="cuda")
    g = capture(lambda i: tg.fv5b_head_gemv_argmax(stack.head_W, S, V, d, 1, tg.TERN_ACT_BF16, xb, None, am, mv,
                                                    None, stack.ws), 5)
    g.replay()
    torch.cuda.synchronize()
    ms = timed_replays([(g, 4)]) / 20
    hb = V * d + V * (d // 256) * 4 + 2 * d + 8
    out["fv5b_head_151936x4096_m1_bf16"] = {"us": ms * 1000.0, "gbs": hb / (ms / 1000.0) / 1e9,
                                            "frac": hb / (ms / 1000.0) / 1e9 / hbm_peak}
    return out


if __name__ == "__main__":
    sys.exit(main())
