#!/usr/bin/env python
"""Benchmark of the B200 selective scan (S6) and decode step.

One JSON line on rank 0.  A step is one pass of the whole hot path over one batch:
for the scan workloads one ``ssm_selective_scan_fwd`` call (discretise, recurrence,
readout, skip, gate, final state), for the decode workload one ``ssm_state_step`` call,
for bwd130m one ``ssm_selective_scan_bwd`` call (all gradients of the scan);
the conv workloads time the causal convolution in front of the scan
(``ssm_causal_conv1d_fwd`` with its final window, or one ``ssm_causal_conv1d_step``).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mamba2p8b]
  python bench.py --impl reference ...        # the fp64 CPU oracle, timed on host cores

Workloads (selective_state_space_45_b200.inputs.CONFIGS): mamba2p8b (default: batch 4,
L 4096, d_inner 5120, N 16, bf16 in/out, fp32 state), mamba130m, long1m, decode, the
backward's bwd130m, and the convolution's conv130m, conv2p8b, convstep.
Multi-GPU: every rank runs its own replica (channels are independent; the path has no
exchange step), timing is the max over ranks, value counts all ranks' work.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "selective-scan GB/s & tokens·channels/s (1 B200), % of HBM/MUFU roofline"
UNIT = "tokens*channels/s"
N_SM = 148
MUFU_EX2_PER_CLK_PER_SM = 16        # SFU ex2 throughput per SM per clock
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_SM_MHZ = 1965.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba2p8b",
                    choices=["mamba130m", "mamba2p8b", "mamba2p8b_d4736", "mamba2p8b_d5920",
                             "long1m", "long1m_slow", "decode", "tiny",
                             "conv130m", "conv2p8b", "convstep", "bwd130m", "decode4", "ssd130m"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0,
                    help="CPU seconds the oracle baseline may spend")
    ap.add_argument("--segments", type=int, default=0,
                    help="scan workloads: force this many time segments per sequence "
                         "(ssm_scan_force_segments; 0 = the library's own choice)")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_dist(world, backend, timeout_s=120):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist if world > 1 else None


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(dist, value, device="cpu"):
    """Max of a float over all ranks (identity on one rank)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(dist, value, device="cpu"):
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ peaks, clocks, traffic

def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        bf16 = p.get("bf16_tflops")
        return dict(hbm_gbs=float(p["hbm_gbs"]), sm_max_mhz=float(p.get("sm_max_mhz", FALLBACK_SM_MHZ)),
                    bf16_tflops=float(bf16) if bf16 is not None else FALLBACK_BF16_TFLOPS,
                    source="measured (MEASURED_PEAKS.json)")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=FALLBACK_HBM_GBS, sm_max_mhz=FALLBACK_SM_MHZ,
                    bf16_tflops=FALLBACK_BF16_TFLOPS, source="fallback")


# translation unit of libssm.so that holds each kernel and its launch logic
KERNEL_UNIT = {"scan_fwd_kernel": "scan_api.cu", "state_step_kernel": "step_api.cu",
               "state_steps_kernel": "step_api.cu", "ssd_tc_kernel": "ssd_api.cu",
               "scan_bwd_kernel": "bwd_api.cu",
               "causal_conv1d_vec_kernel": "conv_api.cu", "conv1d_step_kernel": "conv_api.cu"}


def kernel_source_hash(kernel):
    """Hash of the sources (kernel, headers, launch code) a kernel is built from."""
    from selective_state_space_45_b200.build import source_hash
    return source_hash(KERNEL_UNIT[kernel])


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if taken on these sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f).get("%s %s" % (kernel, workload))
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return float(rec["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock / throttle sampling every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return dict(sm_mhz=statistics.median(sm) if sm else None,
                    sm_max_mhz=float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                    reasons=reasons, samples=len(rows))


# ------------------------------------------------------------------ workloads

def scan_counts(batch, dim, L, N, in_size, out_size):
    """Algorithmic bytes (each input read once, each output written once) and work."""
    streams = batch * dim * L * (3 * in_size + out_size)          # x, delta, z in; y out
    bc = 2 * batch * L * N * in_size                               # B, C in
    params = dim * N * 4 + 2 * dim * 4                             # A; D and delta_bias
    state = batch * dim * N * 4                                    # final state out
    return dict(bytes=streams + bc + params + state, exps=batch * L * dim * N,
                tokch=batch * L * dim)


def conv_counts(batch, dim, L, K, in_size, out_size):
    streams = batch * dim * L * (in_size + out_size)              # x in; u out
    params = dim * (K + 1) * 4                                     # taps and bias
    window = batch * dim * (K - 1) * 4                             # final window out
    return dict(bytes=streams + params + window, exps=batch * dim * L, tokch=batch * dim * L)


def conv_step_counts(batch, dim, K, in_size, out_size):
    window = 2 * batch * dim * (K - 1) * 4                         # read + write in place
    streams = batch * dim * (in_size + out_size)                   # x in; u out
    params = dim * (K + 1) * 4
    return dict(bytes=window + streams + params, exps=batch * dim, tokch=batch * dim)


def bwd_counts(batch, dim, L, N, in_size, g_size):
    """Backward: inputs read once (x, delta, z, B, C, dy, parameters), gradients written
    once.  Work: 2 ex2 per (t, d, n) -- the states recomputed forward and the decay again
    in the reverse walk, the least a backward that keeps no N-expanded tensor in HBM
    needs."""
    streams = batch * dim * L * (3 * in_size + g_size + 3 * g_size)   # x, delta, z, dy in; dx, ddelta, dz out
    bc = 2 * batch * L * N * (in_size + g_size)                       # B, C in; dB, dC out
    params = 2 * (dim * N * 4 + 2 * dim * 4)                          # A, D, bias in; dA, dD, dbias out
    return dict(bytes=streams + bc + params, exps=2 * batch * L * dim * N, tokch=batch * L * dim)


def ssd_counts(batch, L, heads, P, N, in_size, out_size, Q=128):
    """SSD by chunks: x, B, C, a read once and y written once; work = the four chunk products
    (scores C B^T, masked scores times x, C times the entering state, B^T times the weighted
    inputs), 2 flops per multiply-add, over whole chunks."""
    toks = batch * L * heads
    byts = toks * (P * in_size + 2 * N * in_size + 4 + P * out_size)
    nchunk = batch * heads * (-(-L // Q))
    flops = nchunk * 2 * (Q * Q * N + Q * Q * P + 2 * Q * N * P)
    return dict(bytes=byts, flops=flops, exps=0, tokch=toks * P)


def workload_kind(name):
    if name.startswith("ssd"):
        return "ssd"
    if name.startswith("bwd"):
        return "bwd"
    if name == "decode4":
        return "decodemulti"
    if name == "decode":
        return "decode"
    if name == "convstep":
        return "convstep"
    if name.startswith("conv"):
        return "conv"
    return "scan"


def steps_counts(ntok, batch, dim, N, in_size, out_size):
    """ntok decode tokens in one call: the state read and written once."""
    c = step_counts(batch, dim, N, in_size, out_size)
    state = 2 * batch * dim * N * 4
    per_tok = c["bytes"] - state - (dim * N * 4 + dim * 4)
    return dict(bytes=state + ntok * per_tok + dim * N * 4 + dim * 4, exps=ntok * c["exps"],
                tokch=ntok * c["tokch"])


def step_counts(batch, dim, N, in_size, out_size):
    state = 2 * batch * dim * N * 4                                # read + write in place
    streams = batch * dim * (3 * in_size + out_size)               # x, delta, z in; y out
    bc = 2 * batch * N * in_size
    params = dim * N * 4 + dim * 4
    return dict(bytes=state + streams + bc + params, exps=batch * dim * N, tokch=batch * dim)


class Workload:
    """Device-resident inputs of one workload, rotated over enough copies that the
    bytes touched between two uses of the same copy exceed the L2 cache."""

    def __init__(self, name, device, seed=0):
        import torch
        from selective_state_space_45_b200 import inputs
        self.name, self.device = name, device
        self.cfg = dict(inputs.CONFIGS[name])
        self.kind = workload_kind(name)
        c = self.cfg
        dt = c["dtype"]
        esz = torch.tensor([], dtype=dt).element_size()
        if self.kind == "scan":
            self.counts = scan_counts(c["batch"], c["dim"], c["seqlen"], c["dstate"], esz, esz)
        elif self.kind == "ssd":
            self.counts = ssd_counts(c["batch"], c["seqlen"], c["heads"], c["headdim"], c["dstate"],
                                     esz, esz)
        elif self.kind == "bwd":
            self.counts = bwd_counts(c["batch"], c["dim"], c["seqlen"], c["dstate"], esz, esz)
        elif self.kind == "decode":
            self.counts = step_counts(c["batch"], c["dim"], c["dstate"], esz, esz)
        elif self.kind == "decodemulti":
            self.counts = steps_counts(c["ntok"], c["batch"], c["dim"], c["dstate"], esz, esz)
        elif self.kind == "conv":
            self.counts = conv_counts(c["batch"], c["dim"], c["seqlen"], c["width"], esz, esz)
        else:
            self.counts = conv_step_counts(c["batch"], c["dim"], c["width"], esz, esz)
        per_set = self.counts["bytes"]
        self.nsets = max(1, min(4, -(-int(2.5 * L2_BYTES) // per_set)))
        self.sets = []
        for s in range(self.nsets):
            inp = inputs.make_config_inputs(name, device=device, seed=seed + s)
            if self.kind == "scan":
                inp["y"] = torch.empty(inp["x"].shape, device=device, dtype=dt)
                inp["fs"] = torch.empty(c["batch"], c["dim"], c["dstate"], device=device)
            elif self.kind == "ssd":
                inp["y"] = torch.empty(inp["x"].shape, device=device, dtype=dt)
            elif self.kind == "bwd":
                for k in ("dx", "ddelta", "dz"):
                    inp[k] = torch.empty(inp["x"].shape, device=device, dtype=dt)
                for k in ("dB", "dC"):
                    inp[k] = torch.empty(inp["B"].shape, device=device, dtype=dt)
                inp["dA"] = torch.empty(inp["A"].shape, device=device)
                inp["dD"] = torch.empty(c["dim"], device=device)
                inp["dbias"] = torch.empty(c["dim"], device=device)
            elif self.kind == "conv":
                inp["u"] = torch.empty(inp["x"].shape, device=device, dtype=dt)
                inp["fw"] = torch.empty(c["batch"], c["dim"], c["width"] - 1, device=device)
            elif self.kind == "decodemulti":
                inp["y"] = torch.empty(c["ntok"], c["batch"], c["dim"], device=device, dtype=dt)
            else:
                inp["y" if self.kind == "decode" else "u"] = torch.empty(
                    c["batch"], c["dim"], device=device, dtype=dt)
            self.sets.append(inp)

    def launch(self, i, stream=None):
        import selective_state_space_45_b200 as ssm
        s = self.sets[i % self.nsets]
        if self.kind == "scan":
            ssm.ssm_selective_scan_fwd(s["x"], s["delta"], s["delta_bias"], True, s["A"], s["B"],
                                       s["C"], s["D"], s["z"], s["y"], s["fs"], stream)
        elif self.kind == "ssd":
            ssm.ssm_ssd_fwd(s["x"], s["a"], s["B"], s["C"], s["y"], None, None, stream)
        elif self.kind == "decodemulti":
            k = self.cfg["ntok"]
            t = ((i // self.nsets) % (s["x"].shape[0] // k)) * k
            ssm.ssm_state_step_multi(s["state"], s["x"][t:t + k], s["delta"][t:t + k], s["A"],
                                     s["B"][t:t + k], s["C"][t:t + k], s["D"], s["z"][t:t + k],
                                     s["y"], stream)
        elif self.kind == "bwd":
            ssm.ssm_selective_scan_bwd(s["x"], s["delta"], s["delta_bias"], True, s["A"], s["B"], s["C"],
                                       s["D"], s["z"], None, s["dy"], None, s["dx"], s["ddelta"], s["dA"],
                                       s["dB"], s["dC"], s["dD"], s["dz"], s["dbias"], None, stream)
        elif self.kind == "decode":
            t = (i // self.nsets) % s["x"].shape[0]
            ssm.ssm_state_step(s["state"], s["x"][t], s["delta"][t], s["A"], s["B"][t], s["C"][t],
                               s["D"], s["z"][t], s["y"], stream)
        elif self.kind == "conv":
            ssm.ssm_causal_conv1d_fwd(s["x"], s["weight"], s["bias"], None, s["u"], s["fw"], True,
                                      stream)
        else:
            t = (i // self.nsets) % s["x"].shape[0]
            ssm.ssm_causal_conv1d_step(s["window"], s["x"][t], s["weight"], s["bias"], s["u"], True,
                                       stream)

    def description(self):
        return describe_workload(self.name)


def describe_workload(name):
    """The workload's name and shape, as both arms print it in ``config.workload``."""
    from selective_state_space_45_b200 import inputs
    c = inputs.CONFIGS[name]
    kind = workload_kind(name)
    io = str(c["dtype"]).split(".")[-1]
    if kind == "conv":
        return ("%s-shaped causal depthwise conv1d + SiLU: batch %d, L %d, d_inner %d, width %d, "
                "%s x and u, fp32 taps/bias/final window" % (name[4:], c["batch"], c["seqlen"],
                                                             c["dim"], c["width"], io))
    if kind == "convstep":
        return ("decode conv1d step: batch %d, d_inner %d, width %d, fp32 window in place, one %s "
                "token per sequence" % (c["batch"], c["dim"], c["width"], io))
    if kind == "ssd":
        return ("%s-shaped Mamba-2 SSD by 128-token chunks: batch %d, L %d, %d heads x %d, state %d, "
                "%s x/B/C and y, fp32 a" % (name[3:], c["batch"], c["seqlen"], c["heads"],
                                           c["headdim"], c["dstate"], io))
    if kind == "decodemulti":
        return ("decode, %d tokens per call on the carried state: batch %d, d_inner %d, N %d, "
                "fp32 state in place, %s tokens" % (c["ntok"], c["batch"], c["dim"], c["dstate"], io))
    if kind == "bwd":
        return ("%s-shaped selective scan backward (states recomputed): batch %d, L %d, d_inner %d, "
                "N %d, %s inputs, dy and gradients, fp32 A/D/bias gradients"
                % (name[3:], c["batch"], c["seqlen"], c["dim"], c["dstate"], io))
    if kind == "scan":
        return ("%s-shaped selective scan: batch %d, L %d, d_inner %d, N %d, %s x/delta/z/B/C "
                "and y, fp32 A/D/bias/state" % (name, c["batch"], c["seqlen"], c["dim"],
                                                 c["dstate"], str(c["dtype"]).split(".")[-1]))
    return ("decode state step: batch %d, d_inner %d, N %d, fp32 state in place, one %s token "
            "per sequence" % (c["batch"], c["dim"], c["dstate"], str(c["dtype"]).split(".")[-1]))


def kernel_name(kind):
    return dict(scan="scan_fwd_kernel", decode="state_step_kernel", conv="causal_conv1d_vec_kernel",
                convstep="conv1d_step_kernel", bwd="scan_bwd_kernel",
                decodemulti="state_steps_kernel", ssd="ssd_tc_kernel")[kind]


# ------------------------------------------------------------------ CPU oracle timing

def host_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_sample(name, n_target_tokch, seed=0):
    """Inputs of a channel sample of workload ``name`` (CPU tensors widened to fp64 by the
    oracle): all sequences, the first k channels, k chosen for ~n_target_tokch units."""
    import torch
    from selective_state_space_45_b200 import inputs
    c = inputs.CONFIGS[name]
    kind = workload_kind(name)
    if kind == "convstep":
        k = int(max(1, min(c["dim"], n_target_tokch // c["batch"])))
        inp = inputs.make_conv_step_inputs(c["batch"], k, 1, c["width"], c["dtype"], device="cpu",
                                           seed=seed)
        sample = dict(window=inp["window"], x=inp["x"][0], weight=inp["weight"], bias=inp["bias"])
        return kind, sample, c["batch"] * k, "%d sequences x %d of %d channels, one token" % (
            c["batch"], k, c["dim"])
    if kind == "conv":
        per_channel = c["batch"] * c["seqlen"]
        k = int(max(1, min(c["dim"], n_target_tokch // per_channel)))
        inp = inputs.make_conv_inputs(c["batch"], k, c["seqlen"], c["width"], c["dtype"], device="cpu",
                                      seed=seed)
        return kind, inp, per_channel * k, "%d sequences x %d of %d channels, all %d tokens" % (
            c["batch"], k, c["dim"], c["seqlen"])
    if kind == "bwd":
        per_channel = c["batch"] * c["seqlen"]
        k = int(max(1, min(c["dim"], n_target_tokch // per_channel)))
        L = c["seqlen"]
        if k == 1 and n_target_tokch < per_channel:  # one channel of one sequence, shortened
            L = int(max(64, min(L, n_target_tokch)))
            inp = inputs.make_scan_bwd_inputs(1, 1, L, c["dstate"], c["dtype"], device="cpu", seed=seed)
            return kind, inp, L, "1 channel of 1 sequence, first %d of %d tokens" % (L, c["seqlen"])
        inp = inputs.make_scan_bwd_inputs(c["batch"], k, L, c["dstate"], c["dtype"], device="cpu",
                                          seed=seed)
        return kind, inp, per_channel * k, "%d sequences x %d of %d channels, all %d tokens" % (
            c["batch"], k, c["dim"], L)
    if kind == "ssd":
        per_head = c["batch"] * c["seqlen"] * c["headdim"]
        k = int(max(1, min(c["heads"], n_target_tokch // per_head)))
        inp = inputs.make_ssd_inputs(c["batch"], c["seqlen"], k, c["headdim"], c["dstate"], c["dtype"],
                                     device="cpu", seed=seed)
        return kind, inp, per_head * k, "%d sequences x %d of %d heads, all %d tokens" % (
            c["batch"], k, c["heads"], c["seqlen"])
    if kind == "decodemulti":
        k = int(max(1, min(c["dim"], n_target_tokch // (c["batch"] * c["ntok"]))))
        inp = inputs.make_decode_inputs(c["batch"], k, c["dstate"], c["ntok"], c["dtype"], device="cpu",
                                        seed=seed)
        return kind, inp, c["ntok"] * c["batch"] * k, "%d sequences x %d of %d channels, %d tokens" % (
            c["batch"], k, c["dim"], c["ntok"])
    if name == "decode":
        k = int(max(1, min(c["dim"], n_target_tokch // c["batch"])))
        inp = inputs.make_decode_inputs(c["batch"], k, c["dstate"], 1, c["dtype"], device="cpu",
                                        seed=seed)
        sample = dict(state=inp["state"], x=inp["x"][0], delta=inp["delta"][0], A=inp["A"],
                      B=inp["B"][0], C=inp["C"][0], D=inp["D"], z=inp["z"][0])
        return "decode", sample, c["batch"] * k, "%d sequences x %d of %d channels, one token" % (
            c["batch"], k, c["dim"])
    per_channel = c["batch"] * c["seqlen"]
    k = int(max(1, min(c["dim"], n_target_tokch // per_channel)))
    L = c["seqlen"]
    if k == 1 and n_target_tokch < per_channel:  # one channel of one sequence, shortened
        L = int(max(64, min(L, n_target_tokch)))
        inp = inputs.make_scan_inputs(1, 1, L, c["dstate"], c["dtype"], device="cpu", seed=seed,
                                      dt_dist=c["dt_dist"], a_dist=c.get("a_dist", "index"))
        return "scan", inp, L, "1 channel of 1 sequence, first %d of %d tokens" % (L, c["seqlen"])
    inp = inputs.make_scan_inputs(c["batch"], k, L, c["dstate"], c["dtype"], device="cpu", seed=seed,
                                  dt_dist=c["dt_dist"], a_dist=c.get("a_dist", "index"))
    return "scan", inp, per_channel * k, "%d sequences x %d of %d channels, all %d tokens" % (
        c["batch"], k, c["dim"], L)


def _oracle_call(kind, inp, threads):
    import oracle
    if kind == "scan":
        oracle.scan(x=inp["x"], delta=inp["delta"], A=inp["A"], B=inp["B"], C=inp["C"], D=inp["D"],
                    z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True, nthreads=threads)
    elif kind == "ssd":
        oracle.ssd_loop(inp["x"], inp["a"], inp["B"], inp["C"])
    elif kind == "decodemulti":
        h = inp["state"]
        for t in range(inp["x"].shape[0]):
            _, h = oracle.step(h, inp["x"][t], inp["delta"][t], inp["A"], inp["B"][t], inp["C"][t],
                               D=inp["D"], z=inp["z"][t])
    elif kind == "bwd":
        oracle.scan_bwd(inp["dy"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                        z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=True)
    elif kind == "conv":
        oracle.causal_conv1d(inp["x"], inp["weight"], bias=inp["bias"])
    elif kind == "convstep":
        oracle.conv1d_step(inp["window"], inp["x"], inp["weight"], bias=inp["bias"])
    else:
        oracle.step(inp["state"], inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                    z=inp["z"])


def oracle_rate(name, threads, budget_s):
    """Time the oracle as it stands on a bounded sample sized to about ``budget_s`` seconds."""
    kind, inp, units, what = _oracle_sample(name, 2048 * 16)
    t0 = time.perf_counter()
    _oracle_call(kind, inp, threads)
    probe = max(time.perf_counter() - t0, 1e-4)
    rate = units / probe
    kind, inp, units, what = _oracle_sample(name, int(rate * budget_s))
    t0 = time.perf_counter()
    _oracle_call(kind, inp, threads)
    wall = time.perf_counter() - t0
    return dict(value=units / wall, unit=UNIT, cores=threads if kind == "scan" else 1, kind="oracle",
                sample=what, seconds=round(wall, 3))


def run_reference(args):
    """The fp64 oracle timed on the host cores, step by step, on bounded samples."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    threads = host_threads()
    # size each step so that warm-up + timed steps take about two minutes in total
    per_step_s = max(0.02, min(30.0, 120.0 / max(1, args.steps + args.warmup)))
    kind, inp, units, what = _oracle_sample(args.workload, 2048 * 16)
    t0 = time.perf_counter()
    _oracle_call(kind, inp, threads)
    rate = units / max(time.perf_counter() - t0, 1e-4)
    kind, inp, units, what = _oracle_sample(args.workload, int(rate * per_step_s))
    for _ in range(args.warmup):
        _oracle_call(kind, inp, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_call(kind, inp, threads)
    wall = time.perf_counter() - t0
    value = units * args.steps / wall
    cores = threads if kind == "scan" else 1
    line = dict(metric=METRIC, value=value, unit=UNIT, impl="reference", n_gpus=args.gpus,
                steps=args.steps, warmup=args.warmup, ms_per_step=1e3 * wall / args.steps,
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                data="synthetic", config=dict(workload=describe_workload(args.workload), sample=what),
                cpu_baseline=dict(value=value, unit=UNIT, cores=cores, kind="oracle", sample=what),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def count_kernel_nodes(graph):
    """Kernel launches inside a captured CUDA graph (our kernels: the library is the only
    thing launched in the capture), or None if the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        h = rt.cudaGraph_t(init_value=int(graph.raw_cuda_graph()))
        err, _, n = rt.cudaGraphGetNodes(h, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(h, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        count = 0
        for node in nodes[:n]:
            err, kind = rt.cudaGraphNodeGetType(node)
            if err == rt.cudaError_t.cudaSuccess and kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                count += 1
        return count
    except Exception:  # noqa: BLE001 -- an inspection aid only
        return None


def time_e2e_scan(wl, steps):
    """time_e2e for the whole-sequence scan, pipelined over slices of the batch (or, for
    one sequence, of the channels): per slice, its inputs go up on one stream, its scan
    runs on a second and its outputs come back on a third, so that the two copy
    directions overlap each other and the scans.  Every step still copies all of its
    inputs from pinned host memory and reads all of its outputs back."""
    import torch
    import selective_state_space_45_b200 as ssm
    dev = wl.sets[0]
    batch, dim, L = dev["x"].shape
    names_in = ["x", "delta", "z", "B", "C", "A", "D", "delta_bias"]
    host = {}
    for n in names_in:
        host[n] = torch.empty(dev[n].shape, dtype=dev[n].dtype, pin_memory=True)
        host[n].copy_(dev[n])
    outs = {n: torch.empty(dev[n].shape, dtype=dev[n].dtype, pin_memory=True) for n in ("y", "fs")}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs.values())
    if batch >= 2:                      # one slice per sequence; shared parameters with the first
        slices = [(b, b + 1, 0, dim) for b in range(batch)]
        shared = ["A", "D", "delta_bias"]
    else:                               # one sequence: four channel ranges; B, C with the first
        k = 4
        cuts = [dim * i // k for i in range(k + 1)]
        slices = [(0, 1, cuts[i], cuts[i + 1]) for i in range(k)]
        shared = ["B", "C"]

    def view(t, n, sl):
        b0, b1, d0, d1 = sl
        if n in ("A",):
            return t[d0:d1]
        if n in ("D", "delta_bias"):
            return t[d0:d1]
        if n in ("B", "C"):
            return t[b0:b1]
        return t[b0:b1, d0:d1]

    s_up, s_run, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ns = len(slices)
    ev_up = [torch.cuda.Event() for _ in range(ns)]
    ev_run = [torch.cuda.Event() for _ in range(ns)]
    ev_down = [torch.cuda.Event() for _ in range(ns)]
    main = torch.cuda.current_stream()
    for e in ev_up + ev_run + ev_down:
        e.record(main)

    def one():
        for i, sl in enumerate(slices):
            s_up.wait_event(ev_run[i])          # this slice's inputs are free again
            with torch.cuda.stream(s_up):
                for n in names_in:
                    if n in shared and i > 0:
                        continue
                    if n in shared:             # every slice's scan reads these: wait for them
                        s_up.wait_event(ev_run[ns - 1])
                    view(dev[n], n, sl if n not in shared else (0, batch, 0, dim)).copy_(
                        view(host[n], n, sl if n not in shared else (0, batch, 0, dim)), non_blocking=True)
                ev_up[i].record(s_up)
            s_run.wait_event(ev_up[i])
            s_run.wait_event(ev_up[0])
            s_run.wait_event(ev_down[i])        # this slice's outputs have been read back
            b0, b1, d0, d1 = sl
            ssm.ssm_selective_scan_fwd(view(dev["x"], "x", sl), view(dev["delta"], "delta", sl),
                                       view(dev["delta_bias"], "delta_bias", sl), True,
                                       view(dev["A"], "A", sl), view(dev["B"], "B", sl),
                                       view(dev["C"], "C", sl), view(dev["D"], "D", sl),
                                       view(dev["z"], "z", sl), view(dev["y"], "y", sl),
                                       view(dev["fs"], "fs", sl), stream=s_run)
            ev_run[i].record(s_run)
            s_down.wait_event(ev_run[i])
            with torch.cuda.stream(s_down):
                for n in ("y", "fs"):
                    view(outs[n], n, sl).copy_(view(dev[n], n, sl), non_blocking=True)
                ev_down[i].record(s_down)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for st in (s_up, s_run, s_down):
        st.wait_event(e0)
    for _ in range(steps):
        one()
    for st in (s_up, s_run, s_down):
        main.wait_stream(st)
    e1.record(main)
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1e3
    return dict(value=wl.counts["tokch"] * steps / sec, unit=UNIT, h2d_bytes_per_step=h2d,
                d2h_bytes_per_step=d2h, ms_per_step=1e3 * sec / steps,
                pipeline="%d slices: uploads, scans and read-backs on three streams" % ns)


def time_e2e(wl, steps, stream):
    """The same metric through the public API with HOST buffers: every step copies its
    inputs from pinned host memory, runs the call and reads the outputs back."""
    import torch
    import selective_state_space_45_b200 as ssm
    if wl.kind == "scan":
        return time_e2e_scan(wl, steps)
    dev = wl.sets[0]
    # per-token inputs of the decode kinds are [steps, ...]: one token's slice travels
    per_token = {"decode": ("x", "delta", "z", "B", "C"), "convstep": ("x",),
                 "decodemulti": ("x", "delta", "z", "B", "C")}.get(wl.kind, ())
    ntok = wl.cfg.get("ntok", 1)
    names_in, names_out = dict(
        scan=(["x", "delta", "z", "B", "C", "A", "D", "delta_bias"], ["y", "fs"]),
        bwd=(["x", "delta", "z", "B", "C", "A", "D", "delta_bias", "dy"],
             ["dx", "ddelta", "dz", "dB", "dC", "dA", "dD", "dbias"]),
        decode=(["state", "x", "delta", "z", "B", "C", "A", "D"], ["y", "state"]),
        decodemulti=(["state", "x", "delta", "z", "B", "C", "A", "D"], ["y", "state"]),
        ssd=(["x", "a", "B", "C"], ["y"]),
        conv=(["x", "weight", "bias"], ["u", "fw"]),
        convstep=(["window", "x", "weight", "bias"], ["u", "window"]))[wl.kind]

    def dev_view(n):
        if n not in per_token:
            return dev[n]
        return dev[n][0:ntok] if wl.kind == "decodemulti" else dev[n][0]

    host = {}
    for n in names_in:
        src = dev_view(n)
        host[n] = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
        host[n].copy_(src)
    outs = {n: torch.empty(dev[n].shape, dtype=dev[n].dtype, pin_memory=True) for n in names_out}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs.values())

    def one():
        for n in names_in:
            dev_view(n).copy_(host[n], non_blocking=True)
        if wl.kind == "scan":
            ssm.ssm_selective_scan_fwd(dev["x"], dev["delta"], dev["delta_bias"], True, dev["A"],
                                       dev["B"], dev["C"], dev["D"], dev["z"], dev["y"], dev["fs"])
        elif wl.kind == "ssd":
            ssm.ssm_ssd_fwd(dev["x"], dev["a"], dev["B"], dev["C"], dev["y"])
        elif wl.kind == "decodemulti":
            ssm.ssm_state_step_multi(dev["state"], dev_view("x"), dev_view("delta"), dev["A"],
                                     dev_view("B"), dev_view("C"), dev["D"], dev_view("z"), dev["y"])
        elif wl.kind == "bwd":
            ssm.ssm_selective_scan_bwd(dev["x"], dev["delta"], dev["delta_bias"], True, dev["A"], dev["B"],
                                       dev["C"], dev["D"], dev["z"], None, dev["dy"], None, dev["dx"],
                                       dev["ddelta"], dev["dA"], dev["dB"], dev["dC"], dev["dD"], dev["dz"],
                                       dev["dbias"], None)
        elif wl.kind == "decode":
            ssm.ssm_state_step(dev["state"], dev["x"][0], dev["delta"][0], dev["A"], dev["B"][0],
                               dev["C"][0], dev["D"], dev["z"][0], dev["y"])
        elif wl.kind == "conv":
            ssm.ssm_causal_conv1d_fwd(dev["x"], dev["weight"], dev["bias"], None, dev["u"], dev["fw"])
        else:
            ssm.ssm_causal_conv1d_step(dev["window"], dev["x"][0], dev["weight"], dev["bias"], dev["u"])
        for n in names_out:
            outs[n].copy_(dev[n], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            one()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            one()
        e1.record(stream)
        torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1e3
    return dict(value=wl.counts["tokch"] * steps / sec, unit=UNIT, h2d_bytes_per_step=h2d,
                d2h_bytes_per_step=d2h, ms_per_step=1e3 * sec / steps)


def sfu_probe_rate(ssm, device, stream, sm_mhz):
    """The SFU ex2 rate measured on this GPU by the library's probe (ssm_sfu_probe: 8
    independent ex2 chains per thread, 2048 threads per SM), timed with CUDA events on the
    launching stream.  Reported beside the derived peak, not used as the denominator."""
    import torch
    blocks, iters = N_SM * 8, 4096
    out = torch.empty(blocks * 256, device=device, dtype=torch.float32)
    ssm.ssm_sfu_probe(out, blocks, 64, stream)             # load and warm up
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        ssm.ssm_sfu_probe(out, blocks, iters, stream)
        e1.record(stream)
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1e3
    n = blocks * 256 * 8 * iters
    return dict(gexp_s=n / sec / 1e9, ex2_per_clk_per_sm=n / sec / (N_SM * sm_mhz * 1e6),
                at_sm_mhz=sm_mhz, ex2=n, ms=1e3 * sec)


def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    import selective_state_space_45_b200 as ssm
    ssm.load_library()
    if args.segments:
        if workload_kind(args.workload) != "scan":
            raise SystemExit("bench.py: --segments applies to the scan workloads only")
        ssm.ssm_scan_force_segments(args.segments)

    wl = Workload(args.workload, device, seed=rank)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            wl.launch(i, stream)
    torch.cuda.synchronize()
    barrier(dist, device)

    # The K timed steps are captured once into a CUDA graph and replayed: host launch
    # overhead (ctypes marshalling, tens of microseconds) would otherwise sit between
    # short kernels and count as device time.
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
        for i in range(args.steps):
            wl.launch(args.warmup + i, stream)
    graph.instantiate()
    launches = count_kernel_nodes(graph)
    with torch.cuda.stream(stream):
        graph.replay()                    # first replay uploads the graph; untimed
    torch.cuda.synchronize()
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local).start()
    time.sleep(0.3)                       # let the sampler take its first reading
    torch.cuda.synchronize()
    barrier(dist, device)
    with torch.cuda.stream(stream):
        t_begin.record(stream)
        graph.replay()
        t_end.record(stream)
    torch.cuda.synchronize()
    barrier(dist, device)
    clocks = sampler.stop()
    del graph

    local_sec = t_begin.elapsed_time(t_end) / 1e3
    sec = max_over_ranks(dist, local_sec, device)
    kern_ms = 1e3 * sec / args.steps      # average step (kernel) duration over the timed region
    total_units = sum_over_ranks(dist, wl.counts["tokch"] * args.steps, device)

    e2e = time_e2e(wl, args.e2e_steps, stream)
    e2e_val = sum_over_ranks(dist, e2e["value"], device)

    peaks = load_peaks()
    kern_s = kern_ms / 1e3
    gbs = wl.counts["bytes"] / kern_s / 1e9
    if wl.kind in ("scan", "bwd"):
        peak_gexp = N_SM * MUFU_EX2_PER_CLK_PER_SM * peaks["sm_max_mhz"] * 1e6 / 1e9
        achieved = wl.counts["exps"] / kern_s / 1e9
        roof = dict(bound="alu", achieved=achieved, peak=peak_gexp, unit="Gexp/s",
                    frac=achieved / peak_gexp,
                    traffic=None if args.segments else recorded_traffic(kernel_name(wl.kind), wl.name),
                    kernel=kernel_name(wl.kind), kernel_ms=kern_ms,
                    peak_basis=("148 SMs x 16 ex2/clk/SM x %.0f MHz max SM clock; the 16 ex2/clk/SM "
                                "is the SFU rate of the CUDA programming guide's throughput table "
                                "for compute capability 10.x; sfu_probe measures it on this GPU"
                                % peaks["sm_max_mhz"]),
                    hbm=dict(achieved_gbs=gbs, peak_gbs=peaks["hbm_gbs"], frac=gbs / peaks["hbm_gbs"],
                             peak_source=peaks["source"]),
                    sfu_probe=sfu_probe_rate(ssm, device, stream,
                                             clocks.get("sm_mhz") or peaks["sm_max_mhz"]))
    elif wl.kind == "ssd":
        tfl = wl.counts["flops"] / kern_s / 1e12
        roof = dict(bound="hbm", achieved=gbs, peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=gbs / peaks["hbm_gbs"],
                    traffic=recorded_traffic(kernel_name(wl.kind), wl.name),
                    kernel=kernel_name(wl.kind), kernel_ms=kern_ms,
                    peak_basis="measured copy bandwidth, burst (%s)" % peaks["source"],
                    tensor=dict(achieved_tflops=tfl, peak_tflops=peaks.get("bf16_tflops"),
                                frac=(tfl / peaks["bf16_tflops"]) if peaks.get("bf16_tflops") else None,
                                note="bf16 tensor-core work of the chunk products"))
    else:
        roof = dict(bound="hbm", achieved=gbs, peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=gbs / peaks["hbm_gbs"],
                    traffic=recorded_traffic(kernel_name(wl.kind), wl.name),
                    kernel=kernel_name(wl.kind), kernel_ms=kern_ms,
                    peak_basis="measured copy bandwidth, burst (%s)" % peaks["source"])

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_rate(args.workload, host_threads(), args.cpu_budget_s)

    if rank == 0:
        c = wl.cfg
        config = dict(workload=wl.description(), batch=c["batch"],
                      d_inner=c.get("dim", c.get("heads", 0) * c.get("headdim", 0)),
                      parallelism="replicas x%d" % world,
                      l2=("%d rotating input sets of %.0f MB (%.0f MB touched per cycle) > 126 MB L2"
                          % (wl.nsets, wl.counts["bytes"] / 1e6, wl.nsets * wl.counts["bytes"] / 1e6)))
        if "dstate" in c:
            config.update(dstate=c["dstate"])
        if "width" in c:
            config.update(width=c["width"])
        if "heads" in c:
            config.update(heads=c["heads"], headdim=c["headdim"], chunk=128)
        if "seqlen" in c:
            config.update(seqlen=c["seqlen"], global_batch=c["batch"] * world)
        if wl.kind == "scan":
            config.update(segments=args.segments if args.segments else "auto")
        line = dict(metric=METRIC, value=total_units / sec, unit=UNIT, n_gpus=world, steps=args.steps,
                    warmup=args.warmup, ms_per_step=1e3 * sec / args.steps, higher_is_better=True,
                    scaling="weak", vs_baseline=None, dtype="f32",
                    io_dtype=str(c["dtype"]).split(".")[-1], data="synthetic", config=config,
                    gb_per_s=gbs * world, roofline=roof, cpu_baseline=cpu,
                    e2e=dict(value=e2e_val, unit=UNIT, h2d_bytes_per_step=e2e["h2d_bytes_per_step"],
                             d2h_bytes_per_step=e2e["d2h_bytes_per_step"]),
                    gpu_launches=launches if launches is not None else args.steps,
                    timing="one CUDA graph of the %d timed steps, replayed once between CUDA events"
                           % args.steps,
                    clocks=clocks, impl="ours")
        print(json.dumps(line), flush=True)
    barrier(dist, device)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
