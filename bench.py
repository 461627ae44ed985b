#!/usr/bin/env python
"""Benchmark of the sketched linear layer on B200.

Default workload: LLaMA-2-7B-shaped decode (the seven layer shapes q/k/v/o
4096x4096, gate/up 11008x4096, down 4096x11008; 4-bit indices, 8 groups per
row, fp16 LUTs; X bf16 N(0,1) at 1 and at 16 tokens).  One step = the seven
layers at T=1 followed by the seven layers at T=16.  Their inputs are
independent activations, so by default each token count's seven layers are
one grouped call (sk_linear_fwd_group, one launch); --decode-groups block
groups only the layers that share an input in a decoder block, layer makes
one call per layer.
The metric is algorithmic bytes per second (packed indices + LUTs +
activations in + outputs out), the LUT-GEMV's HBM roofline quantity.

Other workloads (--workload) time the training products (forward, input
gradient and LUT gradient per layer) in TFLOP/s and the 70B multi-task
serving shapes; they print the same JSON contract.

Multi-GPU (torchrun, one process per GPU): decode and serving run as
independent replicas; the training workloads run data-parallel, each rank on
its own token batch, with one NCCL all-reduce of the fp32 LUT gradient per
layer on a side stream.  Both scale weakly.

Timing: W warm-up steps, then K steps captured as CUDA graphs and replayed back
to back, bracketed by a barrier and a device synchronisation on each side,
timed with CUDA events on the launching stream; multi-GPU runs take the max
over ranks.  Inputs exceed L2: the weights rotate over several copies whose
total is well above the 126 MB L2, so every layer reads its indices from HBM.
Per-kernel durations come from external CUDA events captured between the
launches inside the same graphs.

`--impl reference` times the CPU oracle (plain NumPy float64) on a bounded
sample of the same workload on the host cores: the reported baseline, not a
target.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LUT-GEMV GB/s (% HBM peak) & fwd+bwd TFLOP/s (% bf16 peak), sketched linear"

WORKLOADS = {
    # name: (layer shapes, bits, gpr, token batches, ntask, products, unit)
    "decode7b": dict(shapes="LLAMA2_7B", bits=4, gpr=8, batches=(1, 16), ntask=1, ops=("fwd",),
                     desc="LLaMA-2-7B-shaped decode, 7 layers, 4-bit, GPR=8, T=1 and T=16"),
    "finetune7b": dict(shapes="LLAMA2_7B", bits=2, gpr=8, batches=(8192,), ntask=1, ops=("fwd", "dx", "dlut"),
                       desc="7B-shaped fine-tune step, 7 layers, 2-bit, GPR=8, T=8192: Y, dX, dLUT"),
    "finetune7b_mt": dict(shapes="LLAMA2_7B", bits=2, gpr=8, batches=(8192,), ntask=8, ops=("fwd", "dx", "dlut"),
                          desc="7B-shaped multi-task fine-tune step, 7 layers, 2-bit, GPR=8, 8 LUT sets, T=8192: Y, dX, dLUT"),
    "train13b": dict(shapes="LLAMA2_13B", bits=3, gpr=1, batches=(4096,), ntask=1, ops=("fwd", "dx", "dlut"),
                     desc="LLaMA-2-13B-shaped fwd+bwd, 7 layers, 3-bit, GPR=1, T=4096"),
    "serve70b_decode": dict(shapes="LLAMA3_70B", bits=4, gpr=4, batches=(1, 64), ntask=8, ops=("fwd",),
                            desc="LLaMA-3-70B-shaped multi-task decode, 7 layers, 4-bit, GPR=4, 8 LUT sets, B=1 and 64"),
    "serve70b_prefill": dict(shapes="LLAMA3_70B", bits=4, gpr=4, batches=(4096,), ntask=8, ops=("fwd",),
                             desc="LLaMA-3-70B-shaped multi-task prefill, 7 layers, 4-bit, GPR=4, 8 LUT sets, T=4096"),
}

# The sketching stage (SpaLLM section 2.2) of one LLaMA-2-7B block: four
# distinct layer inputs (q/k/v share one, gate/up share one), seven weights,
# the pages' calibration set of 128 sequences of 2048 tokens.
SKETCH_METRIC = "sketching stage: weights sketched per second (Gram, inverse factor, weighted Lloyd, mapping)"
SKETCH_INPUTS = (("qkv", (0, 1, 2)), ("o", (3,)), ("gate_up", (4, 5)), ("down", (6,)))
WORKLOADS["sketch7b"] = dict(shapes="LLAMA2_7B", bits=4, gpr=8, batches=(128 * 2048,), ntask=1, ops=("sketch",),
                             desc="sketching stage of one LLaMA-2-7B block: 128x2048 calibration tokens, "
                                  "4-bit, GPR=8, damp 0.01, at most 100 Lloyd updates")
# float64 FMA lanes per SM per cycle on B200 (NVIDIA's 37 TFLOP/s FP64 at the
# 1965 MHz boost clock over 148 SMs); the fp64 stages report against this
FP64_LANES_PER_SM = 64

# the fine-tune workload measured beside the default decode workload: the
# metric names both the LUT-GEMV bandwidth and the fwd+bwd throughput
TRAIN_WORKLOAD = "finetune7b"

L2_BYTES = 126 * 1024 * 1024
# Integer-ALU cost of one 4-bit lookup (byte-permute network) and the integer
# pipe's issue rate per SM on B200, measured with a throughput probe.
ALU_OPS_PER_4BIT_WEIGHT = 2.25
INT_LANES_PER_SM = 64


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode7b")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layers", default=None,
                    help="comma-separated layer indices to run (a subset for profiling); default all")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-groups", choices=("block", "all", "layer"), default="all",
                    help="decode forward calls: 'all' one grouped call for the seven projections of a "
                         "token count (their inputs are independent here), 'block' groups only the "
                         "projections that share an input in a decoder block (q/k/v, gate/up), 'layer' "
                         "one call per layer")
    ap.add_argument("--no-train", action="store_true",
                    help="with the default decode workload, skip the fine-tune block (the metric's fwd+bwd half)")
    ap.add_argument("--launch-events", choices=("groups", "on", "off"), default="groups",
                    help="timing events captured between launches: 'groups' only where the kernel "
                         "changes (each event costs a few microseconds), 'on' between every launch")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


_LAYER_SUBSET = None


def layer_shapes(w):
    from compressive_fine_tuning_b200 import synth
    shapes = getattr(synth, w["shapes"])
    if _LAYER_SUBSET is not None:
        shapes = [shapes[i] for i in _LAYER_SUBSET]
    return shapes


def is_hbm_bound(w):
    return w["ops"] == ("fwd",) and max(w["batches"]) <= 64


def launch_bytes(n, d, bits, gpr, T, ntask_present=1):
    """Algorithmic bytes of one forward launch: packed indices, the LUT sets
    the batch uses, X in, Y out."""
    k = 1 << bits
    return n * d * bits // 8 + ntask_present * n * gpr * k * 2 + T * d * 2 + T * n * 2


def launch_flops(n, d, T, op):
    return 2 * T * n * d  # each of Y, dX and the dense part of dLUT is one T x n x d contraction


def fwd_tc_kernel_name(T, ntask):
    """The tensor-core forward kernel for a batch: 256-token tiles (more than
    128 tokens per LUT set on average) run on a CTA pair unless SK_TC_PAIR=0."""
    per = -(-T // ntask)
    pair = per > 128 and os.environ.get("SK_TC_PAIR", "1") != "0"
    return "fwd_tc_pair_kernel" if pair else "fwd_tc_kernel"


def kernel_name(op, T, w):
    """The library kernel a launch of this kind runs (the dispatch rules of sk_api.cu)."""
    if op == "fwd":
        if w["ntask"] > 1:
            if w["bits"] == 4 and T == 1:
                return "decode_group_kernel"
            return fwd_tc_kernel_name(T, w["ntask"]) + " (routed)"
        path = os.environ.get("SK_FWD_PATH", "")
        if w["bits"] == 4 and T <= 16 and path not in ("gemv", "tc"):
            return "decode_group_kernel"
        if path == "gemv" or (T == 1 and path != "tc"):
            return "gemv_fwd_single_kernel"
        return fwd_tc_kernel_name(T, 1)
    routed = " (routed)" if w["ntask"] > 1 else ""
    if op == "dx":
        if T < 64:
            return "simt_bwd_input_kernel"
        # 256-column blocks on CTA pairs unless SK_DX_PAIR=0
        return ("dx_tc_pair_kernel" if os.environ.get("SK_DX_PAIR", "1") != "0" else "dx_tc_kernel") + routed
    if T < 64:
        return "simt_bwd_lut_kernel"
    # 256-row blocks on CTA pairs unless SK_DLUT_PAIR=0
    return ("dlut_tc_pair_kernel" if os.environ.get("SK_DLUT_PAIR", "1") != "0" else "dlut_tc_kernel") + routed


def kernels_per_launch(op, T, w):
    """Library kernels one API call of this kind launches: the routed forward
    adds the routing and gather kernels, the tensor-core LUT gradient adds its
    reduction of partial bins."""
    if op == "fwd" and w["ntask"] > 1 and not (T == 1 and w["bits"] == 4):
        return 3                    # route, gather, forward
    if op == "dx" and w["ntask"] > 1 and T >= 64:
        return 3                    # route, gather, input gradient
    if op == "dlut" and T >= 64:
        return 5 if w["ntask"] > 1 else 2   # (route, two gathers,) bins, reduction
    return 1


def traffic_per_launch(kname, workload, units_per_launch):
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload (profiles/traffic.json), scaled from the captured launch to
    the average launch by algorithmic units; None when there is no capture or
    any of the kernel's sources changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[f"{kname.split(' ')[0]}@{workload}"]
        h = hashlib.sha256()
        for name in rec["source"]:
            with open(os.path.join(ROOT, "compressive_fine_tuning_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return rec["dram_bytes"] * units_per_launch / rec["algorithmic_units"]
    except Exception:
        return None


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # the samples go to a scratch file next to the run (SK_CLOCKS_DIR, else
        # the system temporary directory)
        base = os.environ.get("SK_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(base, f"clocks_gpu{gpu_index}_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sms.append(float(p[1])); maxs.append(float(p[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, p[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs), "reasons": sorted(reasons),
                "samples": len(sms)}


# ---------------------------------------------------------------------------
# the CPU oracle baseline
# ---------------------------------------------------------------------------

def cpu_baseline(w, budget_s=15.0, seed=0):
    """Time the oracle on a bounded sample of the workload: whole layers, but
    only as many tokens / layers as fit in about `budget_s` of CPU time."""
    import oracle
    from compressive_fine_tuning_b200 import synth
    shapes = layer_shapes(w)
    bits, gpr = w["bits"], w["gpr"]
    units, done, t0 = 0.0, [], time.perf_counter()
    for li, (n, d) in enumerate(shapes):
        for T in w["batches"]:
            Ts = min(T, 64)  # token sample for large batches
            c = synth.layer_case(seed + li, n=n, d=d, bits=bits, gpr=gpr, T=Ts, ntask=w["ntask"],
                                 with_task=w["ntask"] > 1)
            s0 = time.perf_counter()
            if "fwd" in w["ops"]:
                oracle.forward(c.x, c.idx, c.lut, c.task)
            if "dx" in w["ops"]:
                oracle.backward_input(c.dy, c.idx, c.lut, c.task)
            if "dlut" in w["ops"]:
                oracle.backward_lut(c.x, c.dy, c.idx, gpr, 1 << bits, task=c.task, ntask=w["ntask"])
            dt = time.perf_counter() - s0
            if is_hbm_bound(w):
                present = min(w["ntask"], Ts)
                units += launch_bytes(n, d, bits, gpr, Ts, present)
            else:
                units += sum(launch_flops(n, d, Ts, op) for op in w["ops"])
            done.append((li, Ts, dt))
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    el = sum(x[2] for x in done)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    return units, el, cores, done


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

# A decoder block's projections in the order a block runs them; the members
# of a group read the same input (q/k/v; gate/up), so a real block can issue
# each group as one call.
BLOCK_GROUPS = ((0, 1, 2), (3,), (4, 5), (6,))


def decode_groups(w, how, nlayers):
    """The forward groups of a decode workload (one library call each), or
    None for per-layer calls: 'block' groups the layers that share an input in
    a decoder block, 'all' issues the seven projections (independent inputs
    here) as one call, 'layer' one call per layer."""
    if not (is_hbm_bound(w) and w["ops"] == ("fwd",) and w["bits"] == 4 and w["ntask"] == 1) or how == "layer":
        return None
    if _LAYER_SUBSET is not None or nlayers != 7:
        return [tuple(range(nlayers))] if how == "all" else None
    if how == "all":
        return [tuple(range(7))]
    return [g for g in BLOCK_GROUPS]


def weight_copy(step, batch_index, n_batches, copies):
    """The weight copy that token batch `batch_index` of step `step` reads:
    the batches of all steps walk the copies in order, so a copy is read again
    only after every other copy has been."""
    return (step * n_batches + batch_index) % copies


def make_layers(w, seed, device, copies):
    """Build the layer set once on the host, then `copies` device copies of
    the packed weights and LUTs (distinct buffers, so rotation defeats L2)."""
    import torch
    from compressive_fine_tuning_b200 import sk, synth
    shapes = layer_shapes(w)
    bits, gpr, ntask = w["bits"], w["gpr"], w["ntask"]
    layers = []
    for li, (n, d) in enumerate(shapes):
        rng = synth.rng_for(seed * 100 + li)
        idx = torch.from_numpy(synth.make_idx(rng, n, d, bits)).to(device)
        packed = sk.pack(idx, bits)
        del idx
        lut = torch.from_numpy(synth.make_lut(rng, ntask, n, gpr, bits)).to(device)
        sets = [(packed, lut)] + [(packed.clone(), lut.clone()) for _ in range(copies - 1)]
        layers.append(dict(n=n, d=d, sets=sets))
    return layers


def run_ours(args, w, rank, world, device):
    import torch
    import torch.distributed as dist
    from compressive_fine_tuning_b200 import sk, synth

    bits, gpr, ntask = w["bits"], w["gpr"], w["ntask"]
    shapes = layer_shapes(w)
    weight_bytes = sum(n * d * bits // 8 for n, d in shapes)
    copies = max(2, int(np.ceil(3 * L2_BYTES / weight_bytes)) + 1)
    layers = make_layers(w, args.seed, device, copies)
    rng = synth.rng_for(10_000 + rank)

    # how the forward launches are grouped (decode workloads): each group is
    # one library call; layers of a group that read the same input in a
    # decoder block (q/k/v, gate/up) share one X
    fwd_groups = decode_groups(w, args.decode_groups, len(layers))
    share_x = {}
    for grp in fwd_groups or ():
        for li in grp:
            if args.decode_groups == "block":
                share_x[li] = grp[0]

    # activations / gradients per (layer, batch)
    acts = {}
    for li, L in enumerate(layers):
        for T in w["batches"]:
            X = torch.from_numpy(synth.make_bf16(rng, (T, L["d"]), synth.X_STD).view(np.int16)).to(device).view(torch.bfloat16)
            dY = torch.from_numpy(synth.make_bf16(rng, (T, L["n"]), synth.DY_STD).view(np.int16)).to(device).view(torch.bfloat16)
            task = torch.from_numpy(synth.make_task(rng, T, ntask)).to(device) if ntask > 1 else None
            if share_x.get(li, li) != li:
                X = acts[(share_x[li], T)]["X"]
                task = acts[(share_x[li], T)]["task"]
            outs = dict(Y=torch.empty((T, L["n"]), dtype=torch.bfloat16, device=device))
            if "dx" in w["ops"]:
                outs["dX"] = torch.empty((T, L["d"]), dtype=torch.bfloat16, device=device)
            if "dlut" in w["ops"]:
                outs["dl"] = torch.empty((ntask, L["n"], gpr, 1 << bits), dtype=torch.float32, device=device)
            acts[(li, T)] = dict(X=X, dY=dY, task=task, **outs)

    # launch list of one step: (layers, T, op, units); `layers` is a tuple of
    # layer indices, several for a grouped forward
    hbm_bound = is_hbm_bound(w)
    plan = []
    for T in w["batches"]:
        if fwd_groups is not None:
            for grp in fwd_groups:
                u = 0
                for li in grp:
                    a, L = acts[(li, T)], layers[li]
                    present = ntask if a["task"] is None else int(torch.unique(a["task"]).numel())
                    u += launch_bytes(L["n"], L["d"], bits, gpr, T, present)
                plan.append((tuple(grp), T, "fwd", u))
            continue
        for li, L in enumerate(layers):
            for op in w["ops"]:
                if hbm_bound:
                    a = acts[(li, T)]
                    present = ntask if a["task"] is None else int(torch.unique(a["task"]).numel())
                    u = launch_bytes(L["n"], L["d"], bits, gpr, T, present)
                else:
                    u = launch_flops(L["n"], L["d"], T, op)
                plan.append(((li,), T, op, u))
    step_units = sum(p[3] for p in plan)
    # LUT lookups of each forward launch: every weight once per LUT set present
    plan_lookups = []
    for (members, T, op, u) in plan:
        lk = 0
        for li in members:
            a, L = acts[(li, T)], layers[li]
            present = 1 if a["task"] is None else int(torch.unique(a["task"]).numel())
            lk += L["n"] * L["d"] * present
        plan_lookups.append(lk if op == "fwd" else 0)

    # every (step, token batch) reads its own copy of the weights: consecutive
    # batches of a step do not share a copy, and a copy comes back only after
    # all the others (more than 3x L2 of index bytes) have been streamed
    batch_pos = {T: bi for bi, T in enumerate(w["batches"])}

    def copy_of(s, T):
        return weight_copy(s, batch_pos[T], len(w["batches"]), copies)

    def call(members, T, op, s, X_of, task, out_of, dy_of=None):
        """One library call of the plan: X_of(li), dy_of(li) and out_of(li)
        give the tensors (device-resident or staged views)."""
        dy_of = dy_of or (lambda li: acts[(li, T)]["dY"])
        if len(members) > 1 or fwd_groups is not None:
            ls = [(layers[li]["sets"][copy_of(s, T)][0], layers[li]["sets"][copy_of(s, T)][1], X_of(li))
                  for li in members]
            sk.linear_fwd_group(ls, bits, task, outs=[out_of(li) for li in members])
            return
        li = members[0]
        L = layers[li]
        packed, lut = L["sets"][copy_of(s, T)]
        if op == "fwd":
            sk.linear_fwd(packed, lut, bits, X_of(li), task, out=out_of(li))
        elif op == "dx":
            sk.linear_bwd_input(packed, lut, bits, L["d"], dy_of(li), task, out=out_of(li))
        else:
            sk.linear_bwd_lut(packed, bits, gpr, X_of(li), dy_of(li), task, ntask, out=out_of(li))

    out_key = {"fwd": "Y", "dx": "dX", "dlut": "dl"}

    def launch(members, T, op, s):
        call(members, T, op, s, lambda li: acts[(li, T)]["X"], acts[(members[0], T)]["task"],
             lambda li: acts[(li, T)][out_key[op]])

    # data-parallel fine-tuning: every rank runs its own T tokens (weak
    # scaling) and the LUT gradients are summed over ranks, one all-reduce per
    # layer on a side stream, joined at the end of the step
    reducer = None
    if world > 1 and "dlut" in w["ops"]:
        from compressive_fine_tuning_b200 import dp
        reducer = dp.LutGradReducer()

    def after(op, members, T):
        if reducer is not None and op == "dlut":
            for li in members:
                reducer.submit(acts[(li, T)]["dl"])

    def end_step():
        if reducer is not None:
            reducer.wait()

    stream = torch.cuda.Stream(device)
    K, W = args.steps, args.warmup
    # NCCL calls are issued eagerly (no graph capture) so that every rank's
    # collectives stay in plain stream order
    use_graphs = reducer is None

    # warm-up (eager), also the first-call setup of every kernel
    with torch.cuda.stream(stream):
        for s in range(W):
            for (li, T, op, u) in plan:
                launch(li, T, op, s)
                after(op, li, T)
            end_step()
    torch.cuda.synchronize(device)

    # event boundaries: before the first launch, then wherever the kernel type
    # (op, token count) changes, and after the last launch
    kinds = [(op, T) for (li, T, op, u) in plan]
    if args.launch_events == "on":
        bounds = list(range(len(plan) + 1))
    elif args.launch_events == "groups":
        bounds = [0] + [j for j in range(1, len(plan)) if kinds[j] != kinds[j - 1]] + [len(plan)]
    else:
        bounds = []

    def record_step(s, evs):
        if 0 in evs:
            evs[0].record()
        for j, (li, T, op, u) in enumerate(plan):
            launch(li, T, op, W + s)
            after(op, li, T)
            if j + 1 in evs:
                evs[j + 1].record()
        end_step()

    # capture one graph per timed step, with external timing events at the boundaries
    graphs, ev = [], []
    for s in range(K):
        evs = {b: torch.cuda.Event(enable_timing=True, external=use_graphs) for b in bounds}
        if use_graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                record_step(s, evs)
            graphs.append(g)
        ev.append(evs)
    torch.cuda.synchronize(device)
    for g in graphs[:2]:  # replay warm-up
        g.replay()
    torch.cuda.synchronize(device)

    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        start.record(stream)
        if use_graphs:
            for g in graphs:
                g.replay()
        else:
            for s in range(K):
                record_step(s, ev[s])
        stop.record(stream)
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    ms = start.elapsed_time(stop)
    if world > 1:
        t = torch.tensor([ms], device=device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())

    # time per kernel type: groups of launches between boundary events; without
    # events the step time is spread over the launches in proportion to units
    groups = []   # (kind, units, ms per step)
    if bounds:
        for a0, a1 in zip(bounds[:-1], bounds[1:]):
            t = sum(ev[s][a0].elapsed_time(ev[s][a1]) for s in range(K)) / K
            groups.append((kinds[a0], sum(p[3] for p in plan[a0:a1]), t, a1 - a0))
    else:
        groups.append((kinds[0], step_units, ms / K, len(plan)))
    total_units = step_units * K * world
    value = total_units / (ms / 1e3)
    res = dict(ms=ms, value=value, plan=plan, lookups=plan_lookups, groups=groups, step_units=step_units,
               hbm_bound=hbm_bound, clocks=clocks, copies=copies, weight_bytes=weight_bytes)

    # end-to-end through the public API with host buffers (one rank's view)
    if not args.no_e2e:
        # every step copies its inputs (X, dY, task ids of every launch) from
        # pinned host memory in one transfer and reads all its results back in
        # one transfer; the launches read and write views of the staging buffers
        def slab(nbytes):
            return (nbytes + 255) // 256 * 256

        needs = {"fwd": ("X", "task"), "dx": ("dY", "task"), "dlut": ("X", "dY", "task")}
        # staging offsets per distinct input tensor (layers of a group may share
        # one X) and per output
        in_views, out_views, in_off, out_off = {}, {}, 0, 0
        for (members, T, op, u) in plan:
            for li in members:
                a = acts[(li, T)]
                for name in needs[op]:
                    t = a[name]
                    if t is None or id(t) in in_views:
                        continue
                    in_views[id(t)] = (in_off, t)
                    in_off += slab(t.numel() * t.element_size())
                out = a[out_key[op]]
                out_views[(li, T, op)] = (out_off, out)
                out_off += slab(out.numel() * out.element_size())
        # one pinned host copy of the inputs and one of the results; two device
        # staging sets, so that the copies of one step overlap the launches of
        # the next (the inputs of step s + 1 go in and the results of step s
        # come out while step s + 1 computes), as a serving or training loop
        # would run; every step still copies all its inputs in and all its
        # results out inside the timed region
        hin = torch.empty(in_off, dtype=torch.uint8, pin_memory=True)
        hout = torch.empty(out_off, dtype=torch.uint8, pin_memory=True)
        din = [torch.empty(in_off, dtype=torch.uint8, device=device) for _ in range(2)]
        dout = [torch.empty(out_off, dtype=torch.uint8, device=device) for _ in range(2)]

        def view(buf, off, like):
            nb = like.numel() * like.element_size()
            return buf[off:off + nb].view(like.dtype).view(like.shape)

        for key, (off, t) in in_views.items():
            view(hin, off, t).copy_(t.cpu())
        dev_in = [{key: view(din[b], off, t) for key, (off, t) in in_views.items()} for b in range(2)]
        dev_out = [{key: view(dout[b], off, t) for key, (off, t) in out_views.items()} for b in range(2)]

        def staged(b, li, T, name):
            t = acts[(li, T)][name]
            return None if t is None else dev_in[b][id(t)]

        # bytes that cross the bus per step: each input once, each result once
        h2d = sum(t.numel() * t.element_size() for (_, t) in in_views.values())
        d2h = sum(t.numel() * t.element_size() for (_, t) in out_views.values())
        # transfers are issued in pieces of at most 64 MiB (one piece for a
        # decode step)
        piece = 64 << 20

        def copy_in_pieces(dst, src):
            for o in range(0, src.numel(), piece):
                dst[o:o + piece].copy_(src[o:o + piece], non_blocking=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        h2d_stream, d2h_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, in_free = [ev(), ev()], [ev(), ev()]
        out_ready, out_free = [ev(), ev()], [ev(), ev()]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        staged_dy = {}
        e0.record(stream)
        h2d_stream.wait_event(e0)
        d2h_stream.wait_event(e0)
        for s in range(K):
            b = s % 2
            with torch.cuda.stream(h2d_stream):
                if s >= 2:
                    h2d_stream.wait_event(in_free[b])
                copy_in_pieces(din[b], hin)
                in_ready[b].record(h2d_stream)
            with torch.cuda.stream(stream):
                stream.wait_event(in_ready[b])
                if s >= 2:
                    stream.wait_event(out_free[b])
                for (members, T, op, u) in plan:
                    if "dY" in needs[op]:
                        for li in members:
                            staged_dy[li] = staged(b, li, T, "dY")
                    call(members, T, op, W + s, lambda li: staged(b, li, T, "X"), staged(b, members[0], T, "task"),
                         lambda li: dev_out[b][(li, T, op)], dy_of=lambda li: staged_dy[li])
                    if reducer is not None and op == "dlut":
                        for li in members:
                            reducer.submit(dev_out[b][(li, T, op)])
                        reducer.wait()
                out_ready[b].record(stream)
                in_free[b].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(out_ready[b])
                copy_in_pieces(hout, dout[b])
                out_free[b].record(d2h_stream)
        stream.wait_stream(d2h_stream)
        stream.wait_stream(h2d_stream)
        e1.record(stream)
        torch.cuda.synchronize(device)
        ems = e0.elapsed_time(e1)
        if world > 1:
            t = torch.tensor([ems], device=device, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        res["e2e"] = dict(value=total_units / (ems / 1e3), h2d=h2d, d2h=d2h, ms=ems)
    return res


# ---------------------------------------------------------------------------
# the sketching stage (dense weights + calibration activations -> sketch)
# ---------------------------------------------------------------------------

def sketch_factor_launches(d, nb=64):
    """Kernel launches of one inverse factor of a d x d Gram matrix (the
    launch loops of the library, counted)."""
    n = 2                                              # damping, reversal
    for k0 in range(0, d, 2 * nb):                     # Cholesky super-blocks
        for h in range(2):
            kk = k0 + h * nb
            if kk >= d:
                break
            rest = d - kk - min(nb, d - kk)
            n += 1 + (1 if rest > 0 else 0) + (1 if h == 0 and rest > 0 else 0)
        n += 1 if d - k0 - min(d - k0, 2 * nb) > 0 else 0
    n += 1                                             # identity
    for r0 in range(0, d, 2 * nb):                     # inverse super-blocks
        for h in range(2):
            rr = r0 + h * nb
            if rr >= d:
                break
            n += 1 + (1 if h == 0 and d - rr - min(nb, d - rr) > 0 else 0)
        n += 1 if d - r0 - min(d - r0, 2 * nb) > 0 else 0
    return n + 2                                       # reversal, column norms


def sketch_cpu_baseline(budget_rows=32, tokens=4096, seed=0):
    """The oracle's sketching stage on a bounded sample: the q_proj input with
    `tokens` calibration tokens (Gram matrix and inverse factor of the full
    4096-wide input), then Lloyd and the mapping for `budget_rows` rows."""
    import oracle
    from compressive_fine_tuning_b200 import synth
    n, d = synth.LLAMA2_7B[0]
    c = synth.sketch_case(seed + 777, budget_rows, d, tokens)
    t0 = time.perf_counter()
    h = oracle.damped(oracle.gram(c.x), 0.01)
    u, hd = oracle.inverse_factor(h)
    lut = oracle.lloyd_luts(c.theta, hd, 4, 8, 100)
    oracle.sketch_round(c.theta, u, lut)
    el = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    sample = (f"q_proj input (d={d}): Gram of {tokens} tokens, inverse factor, then Lloyd and mapping "
              f"of {budget_rows} of the {n} rows")
    return budget_rows * d, el, cores, sample


def sketch_inputs():
    """The distinct layer inputs and the weights that read them (restricted to
    --layers when given)."""
    out = []
    for name, members in SKETCH_INPUTS:
        m = tuple(li for li in members if _LAYER_SUBSET is None or li in _LAYER_SUBSET)
        if m:
            out.append((name, m))
    return out


def run_sketch(args, w, rank, device):
    """Time the sketching stage of one 7B block per step; stage boundaries
    carry CUDA events on the launching stream."""
    import torch
    from compressive_fine_tuning_b200 import sk, synth
    shapes = synth.LLAMA2_7B
    bits, gpr, s_tok = w["bits"], w["gpr"], w["batches"][0]
    g = torch.Generator(device=device).manual_seed(args.seed * 1000 + rank)
    # calibration activations: N(0, 1) times a per-column scale exp(N(0, 0.5)), bf16
    X = {}
    for name, members in sketch_inputs():
        d = shapes[members[0]][1]
        scale = torch.exp(torch.randn(d, generator=g, device=device) * synth.CALIB_COL_SIGMA)
        X[name] = (torch.randn((s_tok, d), generator=g, device=device) * scale).to(torch.bfloat16)
    theta = {li: torch.randn((shapes[li][0], shapes[li][1]), generator=g, device=device) * synth.LUT_STD
             for _, members in sketch_inputs() for li in members}
    stage_names = ("gram", "factor", "lloyd", "round")

    def step(evs=None, host=None):
        out = []
        mark = (lambda nm: evs.append((nm, torch.cuda.Event(enable_timing=True)))) if evs is not None else None
        for name, members in sketch_inputs():
            if mark: mark("gram"); evs[-1][1].record()
            xin = X[name] if host is None else host["X"][name].to(device, non_blocking=True)
            H = sk.gram(xin)
            if mark: mark("factor"); evs[-1][1].record()
            U, hd = sk.inverse_factor(H, 0.01)
            for li in members:
                th = theta[li] if host is None else host["theta"][li].to(device, non_blocking=True)
                if mark: mark("lloyd"); evs[-1][1].record()
                lut, _ = sk.lloyd(th, hd, bits, gpr, 100)
                if mark: mark("round"); evs[-1][1].record()
                idx = sk.sketch_round(th, U, lut, bits)
                out.append((sk.pack(idx, bits), lut))
        if mark: mark("end"); evs[-1][1].record()
        return out

    K, W = args.steps, args.warmup
    for _ in range(W):
        step()
    torch.cuda.synchronize(device)
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    all_evs = []
    t0 = torch.cuda.Event(enable_timing=True); t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    t0.record()
    for _ in range(K):
        evs = []
        step(evs)
        all_evs.append(evs)
    t1.record()
    torch.cuda.synchronize(device)
    clocks = sampler.stop() if sampler else None
    ms = t0.elapsed_time(t1)
    per_stage = {nm: 0.0 for nm in stage_names}
    for evs in all_evs:
        for (nm, e), (_, e2) in zip(evs[:-1], evs[1:]):
            per_stage[nm] += e.elapsed_time(e2)
    used = [li for _, m in sketch_inputs() for li in m]
    weights = sum(shapes[li][0] * shapes[li][1] for li in used)
    # algorithmic work per stage and step
    # (the Gram matrix is symmetric: its upper triangle, s * d * (d + 1) flops)
    work = {"gram": sum(float(s_tok) * shapes[m[0]][1] * (shapes[m[0]][1] + 1) for _, m in sketch_inputs()),
            "factor": sum(2.0 / 3.0 * shapes[m[0]][1] ** 3 for _, m in sketch_inputs()),
            "round": sum(float(shapes[li][0]) * shapes[li][1] ** 2 for li in used)}
    res = dict(ms=ms, per_stage=per_stage, work=work, weights=weights, clocks=clocks)
    if not args.no_e2e:
        host = {"X": {k: v.cpu().pin_memory() for k, v in X.items()},
                "theta": {li: t.cpu().pin_memory() for li, t in theta.items()}}
        step(host=host)
        torch.cuda.synchronize(device)
        h2d = sum(v.numel() * v.element_size() for v in host["X"].values()) + \
            sum(t.numel() * t.element_size() for t in host["theta"].values())
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        out = step(host=host)
        back = [(p.cpu(), l.cpu()) for p, l in out]
        e1.record()
        torch.cuda.synchronize(device)
        d2h = sum(p.numel() * p.element_size() + l.numel() * l.element_size() for p, l in back)
        res["e2e"] = dict(ms=e0.elapsed_time(e1), h2d=h2d, d2h=d2h)
    return res


def main_sketch(args, w, world, rank, local):
    pk = peaks()
    config = {"workload": args.workload, "desc": w["desc"], "bits": w["bits"], "gpr": w["gpr"],
              "calibration_tokens": w["batches"][0], "layers": [list(x) for x in layer_shapes(w)],
              "inputs": {nm: list(m) for nm, m in sketch_inputs()},
              "parallelism": "single" if world == 1 else f"replicas{world} (one block per rank)",
              "l2": "calibration activations (2-6 GB per input) and weights exceed L2"}
    unit = "weights/s"
    if args.impl == "reference":
        if rank != 0:
            return 0
        best = None
        for _ in range(max(1, min(args.steps, 2))):
            wts, el, cores, sample = sketch_cpu_baseline(seed=args.seed)
            best = el if best is None else min(best, el)
        v = wts / best
        print(json.dumps({"impl": "reference", "metric": SKETCH_METRIC, "value": v, "unit": unit, "n_gpus": 1,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": best * 1e3,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "config": config,
                          "cpu_baseline": {"value": v, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
                          "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return 0
    import torch
    import torch.distributed as dist
    import datetime
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    device = torch.device("cuda", torch.cuda.current_device())
    if world > 1:
        dist.barrier()
    res = run_sketch(args, w, rank, device)
    ms = res["ms"]
    if world > 1:
        t = torch.tensor([ms], device=device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    K = args.steps
    step_ms = ms / K
    st = {k: v / K for k, v in res["per_stage"].items()}
    dom = max(st, key=st.get)
    mhz = (res["clocks"] or {}).get("sm_mhz") or 1965.0
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    fp64_peak = sms * FP64_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
    rates = {}
    for k, v in st.items():
        if k in res["work"]:
            rates[k] = res["work"][k] / (v / 1e3) / 1e12
    if dom == "gram":
        roof = {"bound": "tensor", "achieved": rates["gram"], "peak": pk["bf16_sus"], "unit": "TFLOP/s",
                "frac": rates["gram"] / pk["bf16_sus"], "kernel": "gram_tc_kernel",
                "peak_source": pk["source"] + " bf16_tflops_sustained"}
    elif dom in ("factor", "round"):
        roof = {"bound": "alu", "achieved": rates[dom], "peak": fp64_peak, "unit": "TFLOP/s (fp64)",
                "frac": rates[dom] / fp64_peak,
                "kernel": "gemm_sub_f64_kernel (" + ("Cholesky and triangular inverse" if dom == "factor"
                                                     else "mapping: later-column compensation") + ")",
                "peak_source": f"{FP64_LANES_PER_SM} fp64 FMA lanes/cycle/SM (nominal) x SMs x median SM clock"}
    else:
        roof = {"bound": "alu", "achieved": None, "peak": None, "unit": None, "frac": None, "kernel": "lloyd_kernel"}
    roof["traffic"] = None
    roof["share"] = st[dom] / step_ms
    roof["stages_ms"] = st
    roof["stage_rates_tflops"] = rates
    roof["fp64_peak_tflops"] = fp64_peak
    from compressive_fine_tuning_b200 import synth
    shapes = synth.LLAMA2_7B
    n_launch = 0
    for _, members in sketch_inputs():
        n_launch += 1 + sketch_factor_launches(shapes[members[0]][1])          # Gram, inverse factor
        for li in members:
            nr = (shapes[li][1] + 127) // 128
            n_launch += 1 + 1 + nr + (nr - 1) + 1                              # Lloyd; copy; blocks, GEMMs; pack
    line = {"metric": SKETCH_METRIC, "value": res["weights"] * world / (step_ms / 1e3), "unit": unit,
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "roofline": roof, "gpu_launches": n_launch * K, "clocks": res["clocks"]}
    if "e2e" in res:
        e = res["e2e"]
        line["e2e"] = {"value": res["weights"] / (e["ms"] / 1e3), "unit": unit, "h2d_bytes_per_step": e["h2d"],
                       "d2h_bytes_per_step": e["d2h"]}
    if not args.no_cpu_baseline:
        wts, el, cores, sample = sketch_cpu_baseline(seed=args.seed)
        line["cpu_baseline"] = {"value": wts / el, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample}
    print(json.dumps(line))
    return 0


def fmt_units(w):
    hbm = is_hbm_bound(w)
    return ("GB/s", 1e9) if hbm else ("TFLOP/s", 1e12)


def main():
    global _LAYER_SUBSET
    args = parse()
    w = WORKLOADS[args.workload]
    if args.layers:
        _LAYER_SUBSET = [int(x) for x in args.layers.split(",")]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if w["ops"] == ("sketch",):
        return main_sketch(args, w, world, rank, local)
    unit, scale = fmt_units(w)
    pk = peaks()
    config = workload_config(args.workload, w, world)

    if args.impl == "reference":
        if rank != 0:
            return 0
        units, el, cores, done = cpu_baseline(w, budget_s=12.0, seed=args.seed)
        per_step = el
        K = args.steps
        # each reference step is one bounded sample (the same sample every step)
        for _ in range(max(0, min(K, 3) - 1)):
            u2, e2, _, _ = cpu_baseline(w, budget_s=12.0, seed=args.seed)
            per_step = min(per_step, e2)
        v = units / per_step / scale
        sample = "; ".join(f"layer {li} T={T}" for li, T, _ in done)
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": 1, "steps": K,
                "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": v, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
                "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist
    import datetime
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", torch.cuda.current_device())
    line = measure(args, args.workload, w, config, world, rank, device, pk)
    if args.workload == "decode7b" and not args.no_train and _LAYER_SUBSET is None:
        # the metric's second half: the fwd+bwd TFLOP/s of the 7B-shaped
        # fine-tune step, measured in the same run on the same GPU(s)
        torch.cuda.empty_cache()
        tw = WORKLOADS[TRAIN_WORKLOAD]
        tconfig = workload_config(TRAIN_WORKLOAD, tw, world)
        train = measure(args, TRAIN_WORKLOAD, tw, tconfig, world, rank, device, pk)
        if line is not None:
            line["train"] = {k: train[k] for k in ("value", "unit", "ms_per_step", "steps", "warmup", "dtype",
                                                   "config", "roofline", "gpu_launches", "clocks", "e2e",
                                                   "cpu_baseline") if k in train}
            line["train"]["metric"] = "fwd+bwd TFLOP/s (% bf16 peak), sketched linear: Y, dX and dLUT per layer"
            line["train"]["higher_is_better"] = True
            line["gpu_launches"] += train["gpu_launches"]
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    print(json.dumps(line))
    return 0


def workload_config(name, w, world):
    return {"workload": name, "desc": w["desc"], "bits": w["bits"], "gpr": w["gpr"],
            "tokens": list(w["batches"]), "ntask": w["ntask"], "layers": [list(s) for s in layer_shapes(w)],
            "parallelism": ("single" if world == 1 else
                            f"dp{world} (tokens per rank; LUT-gradient all-reduce)" if "dlut" in w["ops"]
                            else f"replicas{world}"),
            "l2": "weights rotate over copies totalling > 3x L2; every (step, token batch) reads its own copy",
            "layer_subset": _LAYER_SUBSET}


def measure(args, name, w, config, world, rank, device, pk):
    """Time one workload on the GPU arm; rank 0 gets the JSON line (others None)."""
    import torch
    unit, scale = fmt_units(w)
    res = run_ours(args, w, rank, world, device)
    if rank != 0:
        return None

    # the dominant kernel: the kernel type (op, tokens) with the largest share of
    # the step; its achieved rate = its algorithmic units / its measured time
    by_kind = {}
    for kind, units, t, nl in res["groups"]:
        a = by_kind.setdefault(kind, [0.0, 0.0, 0])
        a[0] += units; a[1] += t; a[2] += nl
    dom = max(by_kind, key=lambda k: by_kind[k][1])
    units, t_ms, nl = by_kind[dom]
    step_ms = res["ms"] / args.steps
    op, T = dom
    kname = kernel_name(op, T, w)
    if res["hbm_bound"]:
        achieved = units / (t_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "traffic": traffic_per_launch(kname, name, units / max(nl, 1)),
                "kernel": kname, "launches_per_step": nl, "share": t_ms / step_ms,
                "peak_source": pk["source"] + " hbm_gbs (copy)"}
    else:
        achieved = units / (t_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_sus"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_sus"], "traffic": traffic_per_launch(kname, name, units / max(nl, 1)),
                "kernel": kname, "launches_per_step": nl, "share": t_ms / step_ms,
                "peak_source": pk["source"] + " bf16_tflops_sustained (a kernel timed inside a long step)"}
    if res["hbm_bound"] and kname.startswith("decode_group_kernel") and w["bits"] == 4:
        # The decode kernel is bound by the integer pipe, not by HBM: every 4-bit
        # lookup costs 2.25 integer-ALU lane operations at least (16 byte permutes
        # and 2 masks per eight weights), and the integer pipe issues 64 lanes per
        # cycle per SM on this GPU (measured).  A weight is looked up once per
        # LUT set present in the batch.  Reported beside the HBM roofline.
        lookups = sum(lk for (members, T_, op_, u_), lk in zip(res["plan"], res["lookups"]) if (op_, T_) == dom)
        mhz = (res["clocks"] or {}).get("sm_mhz") or 1965.0
        ops = lookups * ALU_OPS_PER_4BIT_WEIGHT / (t_ms / 1e3)
        alu_peak = torch.cuda.get_device_properties(device).multi_processor_count * INT_LANES_PER_SM * mhz * 1e6
        roof["alu"] = {"achieved": ops / 1e12, "peak": alu_peak / 1e12, "unit": "T int-lane-ops/s",
                       "frac": ops / alu_peak, "ops_per_weight": ALU_OPS_PER_4BIT_WEIGHT,
                       "peak_source": f"{INT_LANES_PER_SM} integer lanes/cycle/SM (measured) x SMs x median SM clock"}
    roof["by_kernel"] = {f"{kernel_name(k[0], k[1], w)} T={k[1]}": {
        "rate": v[0] / (v[1] / 1e3) / scale, "unit": unit, "share": v[1] / step_ms} for k, v in by_kind.items()}

    line = {"metric": METRIC, "value": res["value"] / scale, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
            "roofline": roof, "gpu_launches": sum(kernels_per_launch(op, T, w) for (_, T, op, _) in res["plan"]) * args.steps,
            "clocks": res["clocks"]}
    if "e2e" in res:
        e = res["e2e"]
        line["e2e"] = {"value": e["value"] / scale, "unit": unit, "h2d_bytes_per_step": e["h2d"],
                       "d2h_bytes_per_step": e["d2h"],
                       "copies": "every step's inputs in and results out, overlapped with the neighbouring "
                                 "steps' launches (two device staging sets, one copy stream per direction)"}
    if not args.no_cpu_baseline and world == 1:
        units, el, cores, done = cpu_baseline(w, budget_s=12.0 if res["hbm_bound"] else 8.0, seed=args.seed)
        line["cpu_baseline"] = {"value": units / el / scale, "unit": unit, "cores": cores, "kind": "oracle",
                                "sample": "; ".join(f"layer {li} T={T}" for li, T, _ in done)}
    return line


if __name__ == "__main__":
    sys.exit(main())
