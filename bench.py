#!/usr/bin/env python
"""Benchmark of the gated delta-rule hot path on B200: one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl {native,reference}] [--no-also] [--no-e2e]

A step is one pass of the layer over one batch of synthetic input (seeded,
recipe in gated_delta_rule_forward_b200/inputs.py).  The headline workload is
the largest single-GPU one, the long-context forward: Gated DeltaNet, bf16
q/k/v/o, fp32 state, B=1 T=65536 H=16 dk=dv=128.  The line also carries the
other workloads ("also": KLA on the same shape, the 350M-model layer (GDN and
DeltaNet, B=8 T=2048 H=8), KDA / KLA / GDN-2 at the 1.3B-model shape, and
the decode of 256 sequences x 16 heads: 1024 seeded steps from the
long-context forward's final state, broadcast, the 350M layer fed raw
projections and logits, the kernels applying the input transforms, and the
350M layer's chunked backward), each with its own roofline:
achieved HBM bandwidth of the algorithmic bytes, and for the forwards also
the tensor-core rate of the chunked algorithm's flops.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a
device synchronisation on each side, CUDA events on the launching stream, max
over ranks.  Two input sets are rotated so that a step never finds its inputs
in L2 (each set is larger than the 126 MB L2).  Multi-GPU (torchrun) is weak
scaling: every rank runs its own batch, with no data-path collective.

--impl reference times the fp64 CPU oracle (the only reference that exists)
on the machine's host cores, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (variant, B, T, H, dk, dv); decode workloads use N = B and no T
    "gdn_fwd_350m": ("gdn", 8, 2048, 8, 128, 128),
    "deltanet_fwd_350m": ("deltanet", 8, 2048, 8, 128, 128),
    "kda_fwd_1p3b": ("kda", 4, 4096, 16, 128, 128),
    "kla_fwd_1p3b": ("kla", 4, 4096, 16, 128, 128),
    "gdn2_fwd_1p3b": ("gdn2", 4, 4096, 16, 128, 128),
    "gdn_fwd_64k": ("gdn", 1, 65536, 16, 128, 128),
    "kla_fwd_64k": ("kla", 1, 65536, 16, 128, 128),
    "gdn_decode_256x16": ("gdn", 256, None, 16, 128, 128),
    "gdn_fwd_350m_raw": ("gdn", 8, 2048, 8, 128, 128),
    "gdn_bwd_350m": ("gdn", 8, 2048, 8, 128, 128),
    "kda_bwd_1p3b": ("kda", 4, 4096, 16, 128, 128),
    "gdn2_bwd_1p3b": ("gdn2", 4, 4096, 16, 128, 128),
}
BWD_WORKLOADS = {"gdn_bwd_350m", "kda_bwd_1p3b", "gdn2_bwd_1p3b"}   # the chunked backward (gradients of o and the final state)
RAW_WORKLOADS = {"gdn_fwd_350m_raw"}   # raw projections and logits in; the kernels apply the transforms
DEFAULT = "gdn_fwd_64k"
DECODE_STEPS = 1024         # the decode chain after the long-context prefill
DECODE_PREFILL = "gdn_fwd_64k"
ORACLE_SAMPLE_TOKENS = 4096  # the oracle's timed sample of a long forward: its first tokens, every head
METRIC = "gated-delta-rule layer tokens/s (fwd, decode) at 1 B200; % of bf16 TC / HBM roofline"
_CSRC = "gated_delta_rule_forward_b200/csrc/"
_TC = [_CSRC + f for f in ("chunk_common.cuh", "tc_util.cuh", "tma_host.cuh")]
KERNEL_SOURCES = {   # sources whose text keys a recorded ncu traffic figure
    "chunk64_split": [_CSRC + "chunk_split.cu", _CSRC + "chunk_split.cuh", _CSRC + "chunk_record.cuh"] + _TC,
    "token_bf16io": [_CSRC + "token_fwd.cu"],
    "token_f32io": [_CSRC + "token_fwd.cu"],
    "decode": [_CSRC + "decode.cu"],
    "chunk64_backward": [_CSRC + "chunk_bwd.cu", _CSRC + "chunk_bwd.cuh", _CSRC + "chunk_split.cu"] + _TC,
}


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def _code_only(text):
    """Source text without // and /* */ comments or blank lines: what a
    comment-only edit leaves unchanged (string literals hold no comment
    markers in these sources)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_hash(kernel):
    """Hash of the code (comments stripped) of a kernel's sources: keys the
    recorded ncu traffic, so that a figure taken on other code is not used."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES.get(kernel, []) + ["gated_delta_rule_forward_b200/csrc/common.cuh"]:
        p = os.path.join(ROOT, rel)
        if os.path.exists(p):
            h.update(_code_only(open(p, encoding="utf-8").read()).encode())
    return h.hexdigest()[:12]


def recorded_traffic(kernel, workload):
    """DRAM bytes per step (all launches of one forward / decode call) from a
    committed ncu summary, if it was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == kernel and f[1] == workload:
            if f[2] == source_hash(kernel):
                return float(f[3])
    return None


def fwd_bytes(variant, B, T, H, dk, dv, io_bytes=2):
    """Algorithmic HBM bytes of one forward launch: every input read once, o and
    the final state written once, no initial state (zeros)."""
    th = B * T * H
    b = th * (2 * dk + 2 * dv) * io_bytes
    if variant != "gdn2":
        b += th * 4                                    # beta / eta
    if variant in ("gdn", "kla"):
        b += th * 4                                    # scalar log decay
    elif variant in ("kda", "gdn2"):
        b += th * dk * 4                               # channel-wise log decay
    if variant == "gdn2":
        b += 2 * th * dk * 4                           # erase and write gates
    b += B * H * dk * dv * 4                           # final state
    return b


def fwd_flops(variant, B, T, H, dk, dv, C=64):
    """Flops of the chunked algorithm per forward call (the tensor-core rate's
    numerator): per token-head 2 C dk (K K^T) + 2 C dk (Q K^T) + 2 C dk (W) +
    2 C dv (U') + 2 dk dv (W S) + 2 dk dv (Q S) + 2 C dv (P E) + 2 dk dv (K~^T E)
    = 10 C d + 6 d^2 at dk = dv = d; GDN-2 adds the second Gram pair, R, and the
    two state-free terms: 18 C d + 8 d^2."""
    d = dk
    per = (18 * C * d + 8 * d * d) if variant == "gdn2" else (10 * C * d + 6 * d * d)
    return B * T * H * per


def bwd_bytes(variant, B, T, H, dk, dv, io_bytes=2):
    """Algorithmic HBM bytes of one backward call: q, k, v, d_o and the gates
    read once; dq, dk, dv, the gate gradients and the initial state's gradient
    written once (no initial state, no final-state gradient)."""
    th = B * T * H
    b = th * (2 * dk + 2 * dv) * io_bytes + th * (2 * dk + dv) * io_bytes
    if variant != "gdn2":
        b += th * 4 * 2                                # beta in, d beta out
    if variant in ("gdn", "kla"):
        b += th * 4 * 2                                # log decay in, its gradient out
    elif variant in ("kda", "gdn2"):
        b += th * dk * 4 * 2                           # per-channel log decay in, its gradient out
    if variant == "gdn2":
        b += 2 * th * dk * 4 * 2                       # erase and write gates in, their gradients out
    b += B * H * dk * dv * 4                           # initial state's gradient
    return b


def decode_bytes(variant, N, H, dk, dv, io_bytes=2):
    nh = N * H
    b = nh * dk * dv * 4 * 2 + nh * (2 * dk + 2 * dv) * io_bytes
    if variant != "gdn2":
        b += nh * 4
    if variant in ("gdn", "kla"):
        b += nh * 4
    elif variant in ("kda", "gdn2"):
        b += nh * dk * 4
    if variant == "gdn2":
        b += 2 * nh * dk * 4
    return b


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.samples, self.proc, self.gpu = [], None, gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [s for t, s in self.samples if t0 - 0.15 <= t <= t1 + 0.15] or [s for _, s in self.samples]
        if not rows:
            return None
        sm = sorted(float(r[0]) for r in rows if r[0].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v.strip() == "Active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """Maximum of a per-rank scalar (a device time) over all ranks."""
    if world == 1:
        return x
    dev = "cpu" if torch.distributed.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, steps, ms_max, world):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


# ----------------------------------------------------------------------------- native arm
def make_device_sets(name, seed):
    """Two device-resident input sets of a forward workload (and the host copy)."""
    from gated_delta_rule_forward_b200.inputs import make_inputs, make_raw_inputs
    variant, B, T, H, dk, dv = WORKLOADS[name]
    make = make_raw_inputs if name in RAW_WORKLOADS else make_inputs
    d = make(variant, B, T, H, dk, dv, dtype=torch.bfloat16, seed=seed)
    dev = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    # second set: the same tensors rolled along the head axis (distinct values and addresses)
    dev2 = {k: (None if v is None else torch.roll(v, 1, dims=-2 if v.dim() == 4 else -1).contiguous())
            for k, v in dev.items()}
    return [dev, dev2], d


def gates(d):
    return {k: d[k] for k in ("beta", "log_g", "erase_b", "write_w")}


def run_forward_workload(name, K, W, world, e2e=False, seed=0):
    import gated_delta_rule_forward_b200 as gdr
    variant, B, T, H, dk, dv = WORKLOADS[name]
    sets, host = make_device_sets(name, seed)
    outs = [torch.empty(B, T, H, dv, device="cuda", dtype=torch.bfloat16) for _ in sets]
    finals = [torch.empty(B, H, dk, dv, device="cuda", dtype=torch.float32) for _ in sets]
    kernel = gdr.forward_kernel_name(variant, torch.bfloat16, B, T, H, dk, dv, 0)
    launches = gdr.forward_launches(variant, torch.bfloat16, B, T, H, dk, dv, 0)

    raw = name in RAW_WORKLOADS

    def step(i):
        d = sets[i % 2]
        gdr.forward(d["q"], d["k"], d["v"], variant=variant, **gates(d), out=outs[i % 2],
                    final_state=finals[i % 2], chunk=0, raw_inputs=raw)

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t_wall0 = time.time()
    for i in range(K):
        starts[i].record()
        step(i)
        ends[i].record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = starts[0].elapsed_time(ends[-1])
    total_ms = max_over_ranks(total_ms, world)
    launch_ms = sum(per) / K                  # one kernel per step: its average duration
    res = {
        "workload": name, "variant": variant, "B": B, "T": T, "H": H, "dk": dk, "dv": dv, "raw_inputs": raw,
        "kernel": kernel, "launches_per_step": launches, "ms_per_step": total_ms / K,
        "launch_ms": launch_ms, "tokens_per_step": B * T, "wall": (t_wall0, t_wall1),
        "alg_bytes": fwd_bytes(variant, B, T, H, dk, dv), "alg_flops": fwd_flops(variant, B, T, H, dk, dv),
    }
    res["value"] = job_throughput(B * T, K, total_ms, world)
    if e2e:
        res["e2e"] = forward_e2e(name, host, K, W, world)
    return res


def run_backward_workload(name, K, W, world, seed=0):
    """The chunked backward of a forward workload: the gradients of <d_o, o> with
    respect to every input (the forward's products and carry re-run inside)."""
    import gated_delta_rule_forward_b200 as gdr
    from gated_delta_rule_forward_b200.inputs import random_output_grad
    variant, B, T, H, dk, dv = WORKLOADS[name]
    sets, _ = make_device_sets(name, seed)
    grads = [random_output_grad(B, T, H, dv, seed + 11 + j).cuda() for j in range(2)]

    def step(i):
        d = sets[i % 2]
        gdr.backward(d["q"], d["k"], d["v"], grads[i % 2], variant=variant, **gates(d), scale=dk ** -0.5)

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t_wall0 = time.time()
    for i in range(K):
        starts[i].record()
        step(i)
        ends[i].record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(starts[0].elapsed_time(ends[-1]), world)
    res = {"workload": name, "variant": variant, "B": B, "T": T, "H": H, "dk": dk, "dv": dv,
           "kernel": "chunk64_backward", "launches_per_step": 9, "ms_per_step": total_ms / K,
           "launch_ms": sum(per) / K, "tokens_per_step": B * T, "wall": (t_wall0, t_wall1),
           "alg_bytes": bwd_bytes(variant, B, T, H, dk, dv)}
    res["value"] = job_throughput(B * T, K, total_ms, world)
    return res


def streamed_e2e(pinned_sets, out_specs, call, K, W, world):
    """K steps of (H2D of the step's inputs from pinned host memory, `call`, D2H
    of its outputs into pinned host memory), double-buffered over three streams:
    step i+1's copy-in and step i-1's copy-out run while step i computes, as a
    stream of batches is served.  Every step's own copies are inside the timed
    region.  Returns the milliseconds of the K steps (max over ranks)."""
    # each step's inputs packed into one pinned buffer: one H2D copy per step
    keys = [k for k, v in pinned_sets[0].items() if v is not None]
    layout, off = {}, 0
    for k in keys:
        t = pinned_sets[0][k]
        layout[k] = (off, t.dtype, t.shape)
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    packed = []
    for src in pinned_sets:
        buf = torch.empty(off, dtype=torch.uint8).pin_memory()
        for k, (o, _, _) in layout.items():
            flat = src[k].reshape(-1).view(torch.uint8)
            buf[o:o + flat.numel()].copy_(flat)
        packed.append(buf)
    bufs = [torch.empty(off, dtype=torch.uint8, device="cuda") for _ in range(2)]
    dev = [{k: bufs[j][o:o + torch.Size(sh).numel() * torch.empty(0, dtype=dt).element_size()].view(dt).view(sh)
            for k, (o, dt, sh) in layout.items()} for j in range(2)]
    outs = [[torch.empty(sh, device="cuda", dtype=dt) for sh, dt in out_specs] for _ in range(2)]
    hosts = [[torch.empty(sh, dtype=dt).pin_memory() for sh, dt in out_specs] for _ in range(2)]
    comp = torch.cuda.current_stream()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]       # the call of the buffer pair finished
    out_free = [torch.cuda.Event() for _ in range(2)]   # its output read back

    def step(i):
        j = i % 2
        src = pinned_sets[i % len(pinned_sets)]
        cin.wait_event(done[j])            # inputs of step i-2 consumed
        with torch.cuda.stream(cin):
            bufs[j].copy_(packed[i % len(packed)], non_blocking=True)
        in_ready[j].record(cin)
        comp.wait_event(in_ready[j])
        comp.wait_event(out_free[j])       # output of step i-2 read back
        call({k: dev[j].get(k) for k in src}, outs[j])
        done[j].record(comp)
        cout.wait_event(done[j])
        with torch.cuda.stream(cout):
            for h, o in zip(hosts[j], outs[j]):
                h.copy_(o, non_blocking=True)
        out_free[j].record(cout)

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    cin.wait_event(s)
    cout.wait_event(s)
    for i in range(K):
        step(i)
    for j in range(2):
        comp.wait_event(out_free[j])
    e.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(s.elapsed_time(e), world), off


E2E_NOTE = ("one packed H2D of the step's inputs, the call, D2H of its outputs; double-buffered on three "
            "streams (copies of neighbouring steps overlap)")


def forward_e2e(name, host, K, W, world):
    """Public-API forward throughput with host buffers: every step copies its
    inputs in from pinned host memory and its output back, inside the timed region."""
    import gated_delta_rule_forward_b200 as gdr
    variant, B, T, H, dk, dv = WORKLOADS[name]
    pinned = {k: (None if v is None else v.pin_memory()) for k, v in host.items()}
    shapes = [((B, T, H, dv), torch.bfloat16), ((B, H, dk, dv), torch.float32)]
    d2h = B * T * H * dv * 2 + B * H * dk * dv * 4

    def call(d, outs):
        gdr.forward(d["q"], d["k"], d["v"], variant=variant, **gates(d), out=outs[0], final_state=outs[1])

    ms, h2d = streamed_e2e([pinned], shapes, call, K, W, world)
    return {"value": job_throughput(B * T, K, ms, world), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / K, "schedule": E2E_NOTE}


def prefill_state(world_seed):
    """Final state [1, H, dk, dv] of the long-context forward (the decode's prefill)."""
    import gated_delta_rule_forward_b200 as gdr
    from gated_delta_rule_forward_b200.inputs import make_inputs
    variant, B, T, H, dk, dv = WORKLOADS[DECODE_PREFILL]
    d = {k: (None if v is None else v.cuda())
         for k, v in make_inputs(variant, B, T, H, dk, dv, dtype=torch.bfloat16, seed=world_seed).items()}
    _, S = gdr.forward(d["q"], d["k"], d["v"], variant=variant, **gates(d), chunk=0)
    torch.cuda.synchronize()
    return S


def run_decode_workload(name, K, W, world, e2e=False, chain=True, seed=0):
    """Decode of N sequences x H heads.  With `chain` (the long-context protocol):
    the state starts as the long-context forward's final state broadcast to the N
    sequences, and DECODE_STEPS steps with inputs seeded 1000 + s are timed as one
    chain; otherwise K steps of that chain are timed."""
    import gated_delta_rule_forward_b200 as gdr
    from gated_delta_rule_forward_b200.inputs import make_decode_inputs
    variant, N, _, H, dk, dv = WORKLOADS[name]
    n_steps = DECODE_STEPS if chain else K
    n_inputs = min(n_steps, DECODE_STEPS)
    steps = [{k: (None if v is None else v.cuda()) for k, v in
              make_decode_inputs(variant, N, H, s, dk, dv).items()} for s in range(n_inputs)]
    start = prefill_state(seed).expand(N, H, dk, dv).contiguous()
    state = start.clone()
    out = torch.empty(N, H, dv, device="cuda", dtype=torch.bfloat16)

    def step(i):
        d = steps[i % n_inputs]
        gdr.decode_step(d["q"], d["k"], d["v"], state, variant=variant, **gates(d), out=out)

    for i in range(W):
        step(i)
    state.copy_(start)                  # the timed chain starts from the prefill state
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    s.record()
    for i in range(n_steps):
        step(i)
    e.record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e), world)
    res = {"workload": name, "variant": variant, "N": N, "H": H, "dk": dk, "dv": dv, "kernel": "decode",
           "launches_per_step": 1, "steps_timed": n_steps, "ms_per_step": ms / n_steps,
           "launch_ms": ms / n_steps, "tokens_per_step": N,
           "value": job_throughput(N, n_steps, ms, world), "alg_bytes": decode_bytes(variant, N, H, dk, dv),
           "wall": (t_wall0, t_wall1),
           "protocol": (f"{n_steps} steps from the {DECODE_PREFILL} final state broadcast to {N} sequences, "
                        "inputs seeded 1000 + step")}
    if e2e:
        res["e2e"] = decode_e2e(name, steps[:16], state, K, W, world)
    return res


def decode_e2e(name, dev_steps, state, K, W, world):
    """Public-API decode throughput with host buffers: every step copies its
    token inputs in from pinned host memory (the state stays on the device) and
    its output back, inside the timed region."""
    import gated_delta_rule_forward_b200 as gdr
    variant, N, _, H, dk, dv = WORKLOADS[name]
    pinned = [{k: (None if v is None else v.cpu().pin_memory()) for k, v in d.items()} for d in dev_steps]
    d2h = N * H * dv * 2

    def call(d, outs):
        gdr.decode_step(d["q"], d["k"], d["v"], state, variant=variant, **gates(d), out=outs[0])

    ms, h2d = streamed_e2e(pinned, [((N, H, dv), torch.bfloat16)], call, K, W, world)
    return {"value": job_throughput(N, K, ms, world), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / K, "schedule": E2E_NOTE}


def roofline(res, peaks):
    """Algorithmic bytes of one call over its event-timed duration.  A call of the
    two-kernel path is one preparation and one carry launch; the pair is timed
    together (the workspace between them is not algorithmic traffic)."""
    achieved = res["alg_bytes"] / (res["launch_ms"] / 1e3) / 1e9
    traffic = recorded_traffic(res["kernel"], res["workload"])
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
            "peak_source": peaks["source"], "alg_bytes_per_launch": res["alg_bytes"],
            "launches_timed": res["launches_per_step"]}


def roofline_tensor(res, peaks):
    """The chunked algorithm's flops (fwd_flops) over the call's event-timed
    duration, against the measured dense bf16 tensor peak (the carry's fp16 and
    the channel-decay Gram product's tf32 operands run on the same units; tf32
    at half the bf16 rate, which this figure does not discount)."""
    achieved = res["alg_flops"] / (res["launch_ms"] / 1e3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(achieved / peaks["bf16_tflops"], 4), "peak_source": peaks["source"],
            "alg_flops_per_launch": res["alg_flops"]}


def cpu_baseline(name):
    """The oracle as it stands, on the host cores, on a bounded sample of the workload."""
    import oracle
    from gated_delta_rule_forward_b200.inputs import make_decode_inputs, make_inputs, random_state
    variant, B, T, H, dk, dv = WORKLOADS[name]
    if T is None:   # decode: whole steps of all N sequences
        d = make_decode_inputs(variant, B, H, 0, dk, dv)
        S = random_state(B, H, dk, dv, 7)
        passes, t0 = 0, time.perf_counter()
        while passes == 0 or time.perf_counter() - t0 < 2.0:
            _, S = oracle.decode_step(variant, d["q"], d["k"], d["v"], S, **gates(d))
            passes += 1
        dt = time.perf_counter() - t0
        return {"value": passes * B / dt, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
                "sample": f"{passes} decode step(s) of all {B} sequences x {H} heads, fp64, {dt:.2f} s wall"}
    if name in BWD_WORKLOADS:   # backward: one sequence's gradients per pass
        from gated_delta_rule_forward_b200.inputs import random_output_grad
        d = make_inputs(variant, 1, T, H, dk, dv, dtype=torch.bfloat16, seed=0)
        dO = random_output_grad(1, T, H, dv, 1)
        passes, t0 = 0, time.perf_counter()
        while passes == 0 or time.perf_counter() - t0 < 2.0:
            oracle.backward(variant, d["q"], d["k"], d["v"], dO, **gates(d), scale=dk ** -0.5)
            passes += 1
        dt = time.perf_counter() - t0
        return {"value": passes * T / dt, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
                "sample": f"{passes} backward pass(es) of 1 of {B} sequences x {T} tokens x {H} heads, fp64, "
                          f"{dt:.2f} s wall"}
    Ts = min(T, ORACLE_SAMPLE_TOKENS)
    d = make_inputs(variant, B, Ts, H, dk, dv, dtype=torch.bfloat16, seed=0)
    oracle.forward(variant, **{k: (None if v is None else v[:, :64]) for k, v in d.items()})  # build/load
    passes, t0 = 0, time.perf_counter()
    while passes == 0 or time.perf_counter() - t0 < 2.0:     # >= 2 s wall on all host cores
        oracle.forward(variant, **d)
        passes += 1
    dt = time.perf_counter() - t0
    what = "the whole workload" if Ts == T else f"the first {Ts} of its {T} tokens"
    return {"value": passes * B * Ts / dt, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{passes} pass(es) of {what} ({B} sequence(s) x {Ts} tokens x {H} heads), fp64, "
                      f"{dt:.2f} s wall"}


def native(args):
    world, rank, local = dist_setup()
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    peaks = load_peaks()
    sampler = ClockSampler(local)
    sampler.start()
    t0 = time.time()
    if args.workload in BWD_WORKLOADS:
        main = run_backward_workload(args.workload, args.steps, args.warmup, world, seed=rank)
    elif WORKLOADS[args.workload][2] is None:
        main = run_decode_workload(args.workload, args.steps, args.warmup, world, e2e=not args.no_e2e,
                                   chain=False, seed=rank)
    else:
        main = run_forward_workload(args.workload, args.steps, args.warmup, world, e2e=not args.no_e2e,
                                    seed=rank)   # each rank its own sequences
    t1 = time.time()
    also = []
    if not args.no_also:
        for name in WORKLOADS:
            if name == args.workload:
                continue
            k = max(3, args.steps // 4) if "64k" in name else args.steps
            if name in BWD_WORKLOADS:
                r = run_backward_workload(name, max(3, args.steps // 4), args.warmup, world, seed=rank)
            elif WORKLOADS[name][2] is None:
                r = run_decode_workload(name, k, args.warmup, world, chain=True, seed=rank)
            else:
                r = run_forward_workload(name, k, args.warmup, world, seed=rank)
            r["roofline"] = roofline(r, peaks)
            if "alg_flops" in r:
                r["roofline_tensor"] = roofline_tensor(r, peaks)
            r["unit"] = "tokens/s"
            r.pop("wall", None)
            also.append(r)
    sampler.stop()
    clocks = sampler.summary(*main["wall"])
    cpu = cpu_baseline(args.workload) if rank == 0 and world == 1 else None
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    variant, B, T, H, dk, dv = WORKLOADS[args.workload]
    shape = ({"sequences_per_gpu": B, "heads": H, "dk": dk, "dv": dv, "tokens_per_step": B} if T is None else
             {"batch_per_gpu": B, "seq_len": T, "heads": H, "dk": dk, "dv": dv})
    line = {
        "metric": METRIC, "value": round(main["value"], 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(main["ms_per_step"], 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; q,k L2-normalised, v ~ N(0,1), sigmoid / -softplus gates)",
        "config": {"workload": args.workload, "variant": variant, **shape, "global_batch": B * world,
                   "kernel": main["kernel"],
                   "state": "fp32", "parallelism": f"dp{world}",
                   "l2": "inputs > L2; two input sets rotated between steps"},
        "roofline": roofline(main, peaks),
        "roofline_tensor": roofline_tensor(main, peaks) if "alg_flops" in main else None,
        "cpu_baseline": cpu,
        "e2e": main.get("e2e"),
        "gpu_launches": main["launches_per_step"] * args.steps,
        "clocks": clocks,
        "also": also,
        "wall_s": round(t1 - t0, 2),
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- reference arm
def reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    import oracle
    from gated_delta_rule_forward_b200.inputs import make_decode_inputs, make_inputs, random_state
    variant, B, T, H, dk, dv = WORKLOADS[args.workload]
    if T is None:   # decode: one step of all N sequences per step
        d = make_decode_inputs(variant, B, H, 0, dk, dv)
        S = random_state(B, H, dk, dv, 7)
        run = lambda: oracle.decode_step(variant, d["q"], d["k"], d["v"], S, **gates(d))
        tokens = B
        sample = f"one decode step of all {B} sequences x {H} heads per step, fp64"
    elif args.workload in BWD_WORKLOADS:   # backward: one of the B sequences' gradients per step
        from gated_delta_rule_forward_b200.inputs import random_output_grad
        d = make_inputs(variant, 1, T, H, dk, dv, dtype=torch.bfloat16, seed=0)
        dO = random_output_grad(1, T, H, dv, 1)
        run = lambda: oracle.backward(variant, d["q"], d["k"], d["v"], dO, **gates(d), scale=dk ** -0.5)
        tokens = T
        sample = f"the backward of 1 of {B} sequences x {T} tokens x {H} heads per step, fp64"
    else:           # forward: one of the B sequences per step (its first tokens if it is long)
        Ts = min(T, ORACLE_SAMPLE_TOKENS)
        d = make_inputs(variant, 1, Ts, H, dk, dv, dtype=torch.bfloat16, seed=0)
        run = lambda: oracle.forward(variant, **d)
        tokens = Ts
        sample = (f"1 of {B} sequences x {T} tokens x {H} heads per step, fp64" if Ts == T else
                  f"the first {Ts} of the {T} tokens of 1 of {B} sequence(s) x {H} heads per step, fp64")
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = tokens * args.steps / dt
    cores = oracle.max_threads()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": args.workload, "variant": variant, "batch_per_gpu": B, "seq_len": T,
                   "heads": H, "dk": dk, "dv": dv, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT, choices=list(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-also", action="store_true", help="only the headline workload")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        reference(args)
    else:
        native(args)


if __name__ == "__main__":
    main()
