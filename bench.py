#!/usr/bin/env python
"""Benchmark: MFA decode attention on B200 (KV-tokens/s and HBM roofline).

One step = one MFA decode-attention call (all 64 heads of every sequence over its
whole cached context, split over the SMs and merged) on the headline workload:
batch 64, context 4096, contiguous bf16 KV cache, q/K/V ~ N(0, 1), scale 1/16.
Inputs are synthetic (seeded), resident in HBM before the timed region; three
copies of the 256 MiB cache rotate so that no step reads a cache that is still
L2-resident (each copy is larger than the 126 MB L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch of 64
sequences (weak scaling; the sequences are independent, so there is no
data-path collective); time is the max over ranks.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_attention_08_b200 import inputs as gen  # noqa: E402

HEADLINE = 2
METRIC = "MFA decode KV-tokens/s and HBM GB/s (% of B200 peak) at 4K ctx, 1 GPU"
UNIT = "KV-tokens/s"
L2_BYTES = 126 * 1024 * 1024


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the oracle's CPU-baseline sample")
    ap.add_argument("--profile", choices=["decode", "paged", "fp8", "qproj", "lse_merge", "gqa",
                                          "out_proj", "kv_append", "fused"],
                    default=None,
                    help="profiling case for ncu: plain launches of one kernel family on a "
                         "reduced workload that still exceeds L2")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(gpus: int):
    """Join the job's process group (one rank per GPU; NCCL, or gloo without
    CUDA) from the rendezvous environment torchrun or spawn_ranks sets."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(
            "nccl" if torch.cuda.is_available() else "gloo",
            timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def _free_port() -> int:
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _spawned_rank(local, world, port, target, target_args):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(local),
                      LOCAL_RANK=str(local), WORLD_SIZE=str(world), LOCAL_WORLD_SIZE=str(world))
    os.environ.setdefault("NCCL_DEBUG", "INFO")        # NCCL's init lines show the rank count
    os.environ.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
    target(*target_args)


def spawn_ranks(n: int, target, *target_args):
    """Run target(*target_args) in n fresh processes, rank r on GPU r, with the
    rendezvous environment torchrun would set (127.0.0.1, a free port): what
    `bench.py --gpus N` does when it is not already running under torchrun."""
    import torch.multiprocessing as mp
    mp.spawn(_spawned_rank, args=(n, _free_port(), target, target_args), nprocs=n, join=True)


def _dist_device() -> str:
    return "cpu" if torch.distributed.get_backend() == "gloo" else "cuda"


def dist_max(x: float, world: int) -> float:
    """Max over ranks of a per-rank elapsed time (the only cross-rank reduction)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_dist_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank_step: int, steps: int, world: int, t_max: float) -> float:
    """Whole-job throughput: units every rank processed over the slowest rank's time."""
    return units_per_rank_step * steps * world / t_max


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


# ---------------------------------------------------------------------------
# clocks (nvidia-smi sampled in the background around the timed region)
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], swp=f[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        pmax = max(r["power"] for r in rows)
        loaded = [r for r in rows if r["power"] >= 0.5 * pmax] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples_under_load": len(loaded),
                "power_w_max": pmax}


# ---------------------------------------------------------------------------
# algorithmic bytes (what the operation must move at minimum)
# ---------------------------------------------------------------------------
def decode_alg_bytes(dec: gen.DecodeInputs, out_bytes: int = 2) -> int:
    """K and V rows of every valid token once, q and out once, lengths, page table."""
    T = dec.total_tokens
    kv_elem = 1 if dec.kv_dtype == "e4m3" else 2
    B = dec.batch
    b = T * 2 * 256 * kv_elem + B * 64 * 256 * (2 + out_bytes) + B * 4
    if dec.page_table is not None:
        b += sum((int(L) + dec.page_size - 1) // dec.page_size for L in dec.seq_lens.tolist()) * 4
    return b


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def recorded_traffic(kernel_tag: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.txt")
    if not os.path.exists(path):
        return None, None
    fields = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    src = hashlib.sha256()
    for f in ("decode_kernel.cu", "sm100.cuh", "mfa_internal.h"):
        src.update(open(os.path.join(ROOT, "decode_attention_08_b200", "csrc", f), "rb").read())
    if fields.get("kernel_source_sha256") != src.hexdigest():
        return None, path
    try:
        return float(fields["dram_bytes_per_launch"]), path
    except (KeyError, ValueError):
        return None, path


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
class DecodeStep:
    """One decode-attention call per replay, captured in CUDA graphs (one graph
    per rotating cache copy)."""

    def __init__(self, dec: gen.DecodeInputs, copies: int, out_dtype=torch.bfloat16,
                 num_splits: int = 0):
        from decode_attention_08_b200 import mfa
        self.mfa = mfa
        self.dec = dec
        self.q = dec.q.cuda()
        self.lens = dec.seq_lens.cuda()
        self.pt = None if dec.page_table is None else dec.page_table.cuda()
        self.kv = []
        for i in range(copies):
            self.kv.append((dec.k.cuda(), dec.v.cuda()))
        self.out = torch.empty(dec.batch, 64, 256, dtype=out_dtype, device="cuda")
        self.num_splits = num_splits
        self.ws = torch.zeros(mfa.decode_workspace_size(dec.batch, num_splits), dtype=torch.uint8,
                              device="cuda")
        self.graphs = []
        self.stream = torch.cuda.Stream()

    def call(self, i: int):
        k, v = self.kv[i % len(self.kv)]
        self.mfa.decode_attention_ex(self.q, k, v, self.pt, self.lens, self.out,
                                     self.dec.softmax_scale, self.dec.kv_dtype,
                                     k_scale=self.dec.k_scale, v_scale=self.dec.v_scale,
                                     num_splits=self.num_splits, workspace=self.ws)

    def capture(self, steps_per_graph: int = 10):
        """One graph per rotating cache copy holding a single step, plus graphs
        of `steps_per_graph` consecutive steps (copies rotating inside) so that
        consecutive steps overlap through programmatic dependent launch."""
        with torch.cuda.stream(self.stream):
            for i in range(len(self.kv)):
                self.call(i)  # first launch outside capture (sets kernel attributes)
        torch.cuda.synchronize()
        for i in range(len(self.kv)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self.call(i)
            self.graphs.append(g)
        self.multi = []
        self.per_multi = steps_per_graph
        for start in range(len(self.kv)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                for j in range(steps_per_graph):
                    self.call(start + j)
            self.multi.append(g)
        torch.cuda.synchronize()

    def replay(self, i: int):
        self.graphs[i % len(self.graphs)].replay()

    def run(self, k: int, first: int = 0):
        """Exactly k steps (steps first .. first + k - 1)."""
        i = first
        while k - (i - first) >= self.per_multi:
            self.multi[i % len(self.multi)].replay()
            i += self.per_multi
        while i - first < k:
            self.replay(i)
            i += 1
        return i


def time_steps(step: DecodeStep, k: int, world: int):
    """K replays bracketed by barrier + synchronize; CUDA events on the replay stream."""
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(step.stream):
        s.record(step.stream)
        step.run(k)
        e.record(step.stream)
    torch.cuda.synchronize()
    barrier(world)
    return s.elapsed_time(e) / 1e3


def single_call_us(step: DecodeStep, n: int = 30) -> float:
    """Latency of one call with nothing overlapping it: each replay of a
    one-call graph (cache copies rotating) sits between two synchronisations;
    the median device time between CUDA events on its stream, in us."""
    times = []
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    for i in range(n):
        torch.cuda.synchronize()
        with torch.cuda.stream(step.stream):
            s.record(step.stream)
            step.replay(i)
            e.record(step.stream)
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) * 1e3)
    return statistics.median(times)


# untimed load before each attention workload's timed region, so every one is
# timed in the same sustained state as the headline (the GPU at its power cap)
SUSTAIN_S = 1.0


def sustain(step: DecodeStep, seconds: float):
    """Untimed load so the clock samples reflect the steady state."""
    t0 = time.time()
    i = 0
    with torch.cuda.stream(step.stream):
        while time.time() - t0 < seconds:
            i = step.run(60, i)
            step.stream.synchronize()


def spot_parity(dec: gen.DecodeInputs, out: torch.Tensor, n: int = 8):
    """Sampled outputs against the float64 oracle (test infrastructure)."""
    from oracle import oracle as orc
    rng = np.random.default_rng(4242)
    pairs = sorted(set(zip(rng.integers(0, dec.batch, n).tolist(), rng.integers(0, 64, n).tolist())))
    kvd = orc.E4M3 if dec.kv_dtype == "e4m3" else orc.BF16
    pt = None if dec.page_table is None else dec.page_table.numpy()
    ref, _ = orc.decode(gen.bits(dec.q), gen.bits(dec.k), gen.bits(dec.v), dec.seq_lens.numpy(),
                        dec.softmax_scale, kv_dtype=kvd, page_table=pt,
                        page_size=dec.page_size or 64, k_scale=dec.k_scale, v_scale=dec.v_scale,
                        select=pairs)
    o = out.float().cpu().numpy()
    got = np.stack([o[b, h] for b, h in pairs])
    return float(np.max(np.abs(got - ref))), len(pairs)


def e2e_decode(dec: gen.DecodeInputs, step: DecodeStep, k: int, world: int):
    """Same metric through the public API (plain entry point) with host buffers:
    every step copies q and seq_lens from pinned host memory, runs the call, and
    reads the output back. The KV cache is device-resident state. As a serving
    loop would, the copies run on their own streams, double-buffered, so step
    i + 1's inputs go up and step i - 1's output comes back while step i's call
    runs; the timed region spans the first upload to the last read-back."""
    from decode_attention_08_b200 import mfa
    nb = 2
    q_h = [dec.q.pin_memory() for _ in range(nb)]
    lens_h = [dec.seq_lens.pin_memory() for _ in range(nb)]
    out_h = [torch.empty(dec.batch, 64, 256, dtype=torch.bfloat16).pin_memory()
             for _ in range(nb)]
    q_d = [torch.empty_like(q_h[0], device="cuda") for _ in range(nb)]
    lens_d = [torch.empty_like(lens_h[0], device="cuda") for _ in range(nb)]
    out_d = [torch.empty(dec.batch, 64, 256, dtype=torch.bfloat16, device="cuda")
             for _ in range(nb)]
    st = step.stream
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nb)]    # inputs of buffer j uploaded
    ev_c = [torch.cuda.Event() for _ in range(nb)]     # call on buffer j done
    ev_out = [torch.cuda.Event() for _ in range(nb)]   # output of buffer j read back

    def one(i, first):
        j = i % nb
        kk, vv = step.kv[i % len(step.kv)]
        with torch.cuda.stream(s_in):
            if not first:
                s_in.wait_event(ev_c[j])          # the call two steps back has read q_d[j]
            q_d[j].copy_(q_h[j], non_blocking=True)
            lens_d[j].copy_(lens_h[j], non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(st):
            st.wait_event(ev_in[j])
            if not first:
                st.wait_event(ev_out[j])          # out_d[j] of two steps back is read back
            mfa.decode_attention(q_d[j], kk, vv, step.pt, lens_d[j], out_d[j],
                                 dec.softmax_scale, dec.kv_dtype)
            ev_c[j].record(st)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[j])
            out_h[j].copy_(out_d[j], non_blocking=True)
            ev_out[j].record(s_out)

    for i in range(3):
        one(i, i < nb)
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(s_in)
    for i in range(k):
        one(i, False)
    e.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    t = dist_max(s.elapsed_time(e) / 1e3, world)
    h2d = q_h[0].numel() * q_h[0].element_size() + lens_h[0].numel() * 4
    d2h = out_h[0].numel() * out_h[0].element_size()
    return t, h2d, d2h


def cpu_model() -> str:
    """The host CPU's model name (/proc/cpuinfo), for the CPU-baseline record."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(dec: gen.DecodeInputs, seconds: float):
    """The float64 oracle on whole sequences of the same workload, until about
    `seconds` of CPU work; KV-tokens/s over the sample."""
    from oracle import oracle as orc
    orc.build()
    q = gen.bits(dec.q)
    k = gen.bits(dec.k)
    v = gen.bits(dec.v)
    lens = dec.seq_lens.numpy()
    done_tokens = 0
    nseq = 0
    t0 = time.time()
    b = 0
    while time.time() - t0 < seconds and nseq < dec.batch:
        sel = [(b, h) for h in range(64)]
        orc.decode(q, k, v, lens, dec.softmax_scale, select=sel)
        done_tokens += int(lens[b])
        nseq += 1
        b += 1
    t = time.time() - t0
    return {"value": done_tokens / t, "unit": UNIT, "cores": orc.num_threads(), "cpu": cpu_model(),
            "kind": "oracle",
            "sample": f"{nseq} of {dec.batch} sequences (all 64 heads, L=4096 each) of the "
                      f"headline workload, float64 C oracle, {t:.1f} s"}


def other_workloads(hbm_peak: float, mfa_us: float):
    """Kernel-level numbers of the other workloads (one call per replay)."""
    res = {}
    res[gen.GQA_WORKLOAD["name"]] = time_gqa(hbm_peak, mfa_us)
    torch.cuda.empty_cache()
    for idx in (1, 3, 4, 5):
        dec, proj = gen.make_workload(idx)
        big = decode_alg_bytes(dec) > L2_BYTES
        copies = 2 if big else 1
        num_splits = dec.meta.get("num_splits", 0)
        step = DecodeStep(dec, copies, num_splits=num_splits)
        step.capture()
        for i in range(5):
            step.replay(i)
        sustain(step, SUSTAIN_S)
        n = 50 if big else 500
        t = time_steps(step, n, 1) / n
        alg = decode_alg_bytes(dec)
        err, ns = spot_parity(dec, step.out)
        entry = {"us_per_call": t * 1e6, "single_call_us": single_call_us(step),
                 "kv_tokens_per_s": dec.total_tokens / t,
                 "seq_per_s": dec.batch / t, "alg_bytes": alg, "gbs": alg / t / 1e9,
                 "frac_of_measured_hbm": alg / t / 1e9 / hbm_peak,
                 "spot_max_abs_err": err, "spot_samples": ns,
                 "l2": "2 rotating copies" if big else "L2-resident (latency)"}
        if num_splits:
            entry["num_splits"] = num_splits
            step0 = DecodeStep(dec, copies, num_splits=0)
            step0.capture()
            for i in range(5):
                step0.replay(i)
            sustain(step0, SUSTAIN_S)
            t0 = time_steps(step0, n, 1) / n
            entry["auto_split_us_per_call"] = t0 * 1e6
            entry["auto_split_gbs"] = alg / t0 / 1e9
            del step0
        if proj is not None:
            entry["qproj"] = time_qproj(proj, hbm_peak)
            torch.cuda.empty_cache()
            entry["fused_qproj_attention"] = time_fused(dec, proj, hbm_peak, t * 1e6,
                                                        entry["qproj"]["us_per_call"])
        res[gen.WORKLOADS[idx]["name"]] = entry
        del step
        torch.cuda.empty_cache()
    for batch, kv in ((64, "bf16"), (128, "e4m3")):
        res[f"mfa_kv_append_b{batch}_h7168_{kv}"] = time_kv_append(batch, kv, hbm_peak)
        torch.cuda.empty_cache()
    for batch in (8, 64):
        res[f"mfa_output_proj_b{batch}_16384x7168"] = time_out_proj(batch, hbm_peak)
        torch.cuda.empty_cache()
    for batch in (8, 64):
        res[f"mfa_lse_merge_b{batch}_s8"] = time_lse_merge(8, batch, hbm_peak)
        torch.cuda.empty_cache()
    return res


class GqaStep(DecodeStep):
    """DecodeStep over the grouped-query comparison kernel (same rotation and graphs)."""

    def __init__(self, inp: gen.GqaInputs, copies: int):
        from decode_attention_08_b200 import mfa
        self.mfa = mfa
        self.dec = inp
        self.q = inp.q.cuda()
        self.lens = inp.seq_lens.cuda()
        self.pt = None
        self.kv = [(inp.k.cuda(), inp.v.cuda()) for _ in range(copies)]
        self.out = torch.empty(inp.batch, 64, 128, dtype=torch.bfloat16, device="cuda")
        self.num_splits = 0
        self.ws = torch.empty(mfa.decode_workspace_size(inp.batch, 0), dtype=torch.uint8,
                              device="cuda")
        self.graphs = []
        self.stream = torch.cuda.Stream()

    def call(self, i: int):
        k, v = self.kv[i % len(self.kv)]
        self.mfa.gqa_decode_attention(self.q, k, v, None, self.lens, self.out,
                                      self.dec.softmax_scale, workspace=self.ws)


def time_gqa(hbm_peak: float, mfa_us: float):
    """The grouped-query comparison workload (same batch, context and cache bytes
    per token as the headline), timed like the headline."""
    inp = gen.make_gqa_workload()
    step = GqaStep(inp, copies=3)
    step.capture()
    for i in range(5):
        step.replay(i)
    sustain(step, SUSTAIN_S)  # the headline's conditions (power-capped clock)
    n = 200
    t = time_steps(step, n, 1) / n
    T = inp.total_tokens
    alg = T * 1024 + inp.batch * 64 * 128 * 4 + inp.batch * 4
    return {"us_per_call": t * 1e6, "single_call_us": single_call_us(step),
            "kv_tokens_per_s": T / t, "alg_bytes": alg, "gbs": alg / t / 1e9,
            "frac_of_measured_hbm": alg / t / 1e9 / hbm_peak,
            "mfa_headline_us_per_call": mfa_us, "gqa_over_mfa_time": t * 1e6 / mfa_us,
            "shape": "64 q heads x 128 in 2 groups, 2 key + 2 value heads x 128 (1024 B/token, "
                     "as MFA's 1 + 1 heads x 256), bf16 cache and output",
            "l2": "3 rotating device copies of the cache"}


class FusedStep(DecodeStep):
    """The query projection then the attention in one call (mfa_qproj_decode_attention)."""

    def __init__(self, dec: gen.DecodeInputs, proj: gen.ProjInputs, copies: int, num_splits: int):
        super().__init__(dec, copies, num_splits=num_splits)
        mfa = self.mfa
        self.x, self.wa, self.wb = proj.x.cuda(), proj.w_qa.cuda(), proj.w_qb.cuda()
        self.qf = torch.empty(dec.batch, 64 * 256, dtype=torch.bfloat16, device="cuda")
        self.wsf = torch.zeros(mfa.qproj_decode_workspace_size(dec.batch, self.x.shape[1],
                                                               self.wa.shape[1], num_splits),
                               dtype=torch.uint8, device="cuda")

    def call(self, i: int):
        k, v = self.kv[i % len(self.kv)]
        self.mfa.qproj_decode_attention(self.x, self.wa, self.wb, self.qf, k, v, self.pt,
                                        self.lens, self.out, self.dec.softmax_scale,
                                        num_splits=self.num_splits, workspace=self.wsf)


def time_fused(dec: gen.DecodeInputs, proj: gen.ProjInputs, hbm_peak: float, attn_us: float,
               proj_us: float):
    """Projection + attention as one call, against the two timed separately."""
    step = FusedStep(dec, proj, 2, dec.meta.get("num_splits", 0))
    step.capture()
    for i in range(5):
        step.replay(i)
    sustain(step, SUSTAIN_S)
    n = 50
    t = time_steps(step, n, 1) / n
    alg = decode_alg_bytes(dec) + sum(x.numel() * 2 for x in (proj.x, proj.w_qa, proj.w_qb))
    res = {"us_per_call": t * 1e6, "single_call_us": single_call_us(step),
           "sum_of_separate_us": attn_us + proj_us, "alg_bytes": alg, "gbs": alg / t / 1e9,
           "frac_of_measured_hbm": alg / t / 1e9 / hbm_peak,
           "note": "mfa_qproj_decode_attention: x[8,7168] -> W_qa -> W_qb -> q, then the 16-way "
                   "split attention; algorithmic bytes = weights + x + the attention's"}
    del step
    return res


def time_qproj(proj: gen.ProjInputs, hbm_peak: float):
    from decode_attention_08_b200 import mfa
    x, wa, wb = proj.x.cuda(), proj.w_qa.cuda(), proj.w_qb.cuda()
    q = torch.empty(x.shape[0], wb.shape[1], dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(mfa.query_proj_workspace_size(x.shape[0], x.shape[1], wa.shape[1]),
                     dtype=torch.uint8, device="cuda")
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for _ in range(3):
            mfa.query_proj_ex(x, wa, wb, q, ws)
    torch.cuda.synchronize()
    # rotate through enough weight copies to exceed L2
    copies = [(wa, wb)] + [(wa.clone(), wb.clone()) for _ in range(2)]
    graphs = []
    for a, b in copies:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            mfa.query_proj_ex(x, a, b, q, ws)
        graphs.append(g)
    for i in range(6):
        graphs[i % 3].replay()
    torch.cuda.synchronize()
    n = 200
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(st):
        s.record(st)
        for i in range(n):
            graphs[i % 3].replay()
        e.record(st)
    torch.cuda.synchronize()
    t = s.elapsed_time(e) / 1e3 / n
    alg = (wa.numel() + wb.numel() + x.numel() + q.numel()) * 2
    flops = 2 * x.shape[0] * (wa.numel() + wb.numel())
    return {"us_per_call": t * 1e6, "alg_bytes": alg, "gbs": alg / t / 1e9,
            "frac_of_measured_hbm": alg / t / 1e9 / hbm_peak, "tflops": flops / t / 1e12,
            "note": "batch <= 8: one persistent kernel (split-K latent GEMM, deterministic merge, up-projection whose weights fill the ring while the latent forms); larger batches: two launches"}


def time_kv_append(batch: int, kv_dtype: str, hbm_peak: float):
    """The new token's key/value projection and cache append of a decode batch
    (contiguous cache of 4097 rows per sequence, row 4096 written). The weights
    rotate through 20 device copies (147 MB > L2): in a decode step the other
    layers' weights pass through L2 between two appends of one layer."""
    from decode_attention_08_b200 import mfa
    inp = gen.make_kv_append_inputs(3000 + batch, batch)
    x = inp.x.cuda()
    copies = [(inp.w_k.cuda(), inp.w_v.cuda()) for _ in range(20)]
    fp8 = kv_dtype == "e4m3"
    shape = (batch, 4097, 256)
    kc = torch.zeros(shape, dtype=torch.uint8 if fp8 else torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    pos = torch.full((batch,), 4096, dtype=torch.int32, device="cuda")
    ws = torch.empty(mfa.kv_append_workspace_size(batch, x.shape[1]), dtype=torch.uint8,
                     device="cuda")
    sc = (0.02, 0.02) if fp8 else (1.0, 1.0)
    st = torch.cuda.Stream()

    def call(i):
        wk, wv = copies[i % len(copies)]
        mfa.kv_append(x, wk, wv, kc, vc, pos, kv_dtype=kv_dtype, k_scale=sc[0], v_scale=sc[1],
                      workspace=ws, stream=st)

    with torch.cuda.stream(st):
        for i in range(3):
            call(i)
    torch.cuda.synchronize()
    graphs = []
    for i in range(len(copies)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            call(i)
        graphs.append(g)
    for i in range(len(copies)):
        graphs[i].replay()
    torch.cuda.synchronize()
    n = 200
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(st):
        s.record(st)
        for i in range(n):
            graphs[i % len(graphs)].replay()
        e.record(st)
    torch.cuda.synchronize()
    status = mfa.read_status()
    t = s.elapsed_time(e) / 1e3 / n
    esz = 1 if fp8 else 2
    alg = (2 * x.shape[1] * 256 * 2 + x.numel() * 2 + batch * 2 * 256 * esz + batch * 4)
    return {"us_per_call": t * 1e6, "alg_bytes": alg, "gbs": alg / t / 1e9,
            "frac_of_measured_hbm": alg / t / 1e9 / hbm_peak, "status": status,
            "note": "split-K projection x [W_k | W_v] (one launch) + merge-and-store kernel; "
                    "weights rotate through 20 copies (> L2)"}


def time_out_proj(batch: int, hbm_peak: float):
    """The attention layer's output projection [B, 16384] x [16384, 7168]; two
    weight copies (235 MB each, > L2) alternate."""
    from decode_attention_08_b200 import mfa
    inp = gen.make_out_proj_inputs(4000 + batch, batch)
    o = inp.o.cuda()
    copies = [inp.w_o.cuda(), inp.w_o.cuda()]
    y = torch.empty(batch, copies[0].shape[1], dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(mfa.output_proj_workspace_size(batch, o.shape[1], y.shape[1]),
                     dtype=torch.uint8, device="cuda")
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for i in range(3):
            mfa.output_proj(o, copies[i % 2], y, workspace=ws, stream=st)
    torch.cuda.synchronize()
    graphs = []
    for w in copies:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            mfa.output_proj(o, w, y, workspace=ws, stream=st)
        graphs.append(g)
    for i in range(4):
        graphs[i % 2].replay()
    torch.cuda.synchronize()
    n = 50
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(st):
        s.record(st)
        for i in range(n):
            graphs[i % 2].replay()
        e.record(st)
    torch.cuda.synchronize()
    status = mfa.read_status()
    t = s.elapsed_time(e) / 1e3 / n
    alg = (copies[0].numel() + o.numel() + y.numel()) * 2
    return {"us_per_call": t * 1e6, "alg_bytes": alg, "gbs": alg / t / 1e9,
            "frac_of_measured_hbm": alg / t / 1e9 / hbm_peak, "status": status,
            "tflops": 2 * batch * copies[0].numel() / t / 1e12,
            "note": "split-K GEMM (weights as the MMA's A operand) + in-order merge kernel"}


def time_lse_merge(parts: int, batch: int, hbm_peak: float):
    """The merge of a sequence split over `parts` GPUs (the exchange step's
    compute): `parts` (O, lse) parts per sequence; enough input copies rotate
    that the inputs exceed L2, one graph replays a call on each copy."""
    from decode_attention_08_b200 import mfa
    inp = gen.make_lse_merge_inputs(4100 + batch, parts, batch)
    per_copy = (inp.o_parts.numel() + inp.lse_parts.numel()) * 4
    n_copies = max(2, -(-2 * L2_BYTES // per_copy))
    o_parts = [inp.o_parts.cuda() for _ in range(n_copies)]
    lse_parts = [inp.lse_parts.cuda() for _ in range(n_copies)]
    out = torch.empty(batch, 64, 256, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for i in range(3):
            mfa.lse_merge(o_parts[i % n_copies], lse_parts[i % n_copies], out, stream=st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for i in range(n_copies):
            mfa.lse_merge(o_parts[i], lse_parts[i], out, stream=st)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    reps = 5
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(st):
        s.record(st)
        for _ in range(reps):
            g.replay()
        e.record(st)
    torch.cuda.synchronize()
    status = mfa.read_status()
    t = s.elapsed_time(e) / 1e3 / (reps * n_copies)
    alg = per_copy + out.numel() * 2
    return {"us_per_call": t * 1e6, "alg_bytes": alg, "gbs": alg / t / 1e9,
            "frac_of_measured_hbm": alg / t / 1e9 / hbm_peak, "status": status,
            "copies": n_copies,
            "note": "log-sum-exp merge of a sequence split over GPUs, bf16 output"}


def run_ours(args, world, rank, local):
    from decode_attention_08_b200 import build, mfa
    build.build()
    mfa.lib()
    hbm_peak, bf16_peak, peak_kind = peaks()

    dec, _ = gen.make_workload(HEADLINE)
    step = DecodeStep(dec, copies=3)
    step.capture()
    for i in range(max(3, args.warmup)):
        step.replay(i)
    torch.cuda.synchronize()
    # the same K steps right after warm-up, before sustained load brings the
    # GPU to its power cap (reported beside the sustained value)
    burst = dist_max(time_steps(step, args.steps, world), world)
    sampler = ClockSampler(local)
    sampler.start()
    sustain(step, 1.0)
    secs = time_steps(step, args.steps, world)
    sustain(step, 0.3)
    clocks = sampler.stop()
    t_max = dist_max(secs, world)

    T = dec.total_tokens
    value = weak_scaling_value(T, args.steps, world, t_max)
    per_launch = secs / args.steps
    alg = decode_alg_bytes(dec)
    achieved = alg / per_launch / 1e9
    traffic, _ = recorded_traffic("mfa_decode_kernel_b64_l4096_bf16")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": t_max / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/K/V, bf16)",
        "config": {"workload": gen.WORKLOADS[HEADLINE]["name"], "batch_per_gpu": dec.batch,
                   "seq_len": 4096, "q_heads": 64, "head_dim": 256, "kv_heads": 1,
                   "kv_cache": "contiguous bf16", "out": "bf16", "softmax_scale": 1 / 16,
                   "split": "balanced over SMs + LSE combine",
                   "l2": "3 rotating device copies of the 256 MiB cache (each > L2)",
                   "launch": "CUDA graphs of consecutive C-ABI calls (programmatic dependent launch between steps)",
                   "parallelism": f"dp{world} (independent sequences per GPU)"},
        "hbm_gbs": achieved,
        "seq_per_s": dec.batch * args.steps * world / t_max,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_kind": peak_kind,
                     "kernel": "one decode-attention call: mfa_decode_kernel + mfa_combine_kernel (programmatic dependent launch)",
                     "alg_bytes_per_launch": alg},
        "clocks": clocks,
        "gpu_launches": 2 * args.steps,
        "burst": {"value": weak_scaling_value(T, args.steps, world, burst),
                  "ms_per_step": burst / args.steps * 1e3,
                  "frac_of_measured_hbm": alg / (burst / args.steps) / 1e9 / hbm_peak,
                  "note": "the same steps timed right after warm-up, before a second of "
                          "sustained load brings the GPU to its 1000 W power cap; value, "
                          "roofline and clocks above are the sustained measurement"},
    }
    # one isolated call (nothing before or after it on the GPU) next to the
    # pipelined per-step time above
    line["single_call_us"] = single_call_us(step)
    if rank == 0:
        err, ns = spot_parity(dec, step.out)
        line["parity"] = {"spot_max_abs_err": err, "samples": ns, "tol": 2e-3}
    t_e2e, h2d, d2h = e2e_decode(dec, step, min(args.steps, 200), world)
    n_e2e = min(args.steps, 200)
    line["e2e"] = {"value": T * n_e2e * world / t_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h,
                   "note": "public API (mfa_decode_attention) per step: q + seq_lens H2D from "
                           "pinned memory, the call, output D2H; KV cache device-resident; "
                           "copies on their own streams, double-buffered, overlapping the "
                           "neighbouring steps' calls"}
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(dec, args.cpu_seconds)
    if rank == 0 and world == 1 and not args.no_extra:
        del step
        torch.cuda.empty_cache()
        line["other_workloads"] = other_workloads(hbm_peak, per_launch * 1e6)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, world, rank):
    """The oracle (float64 C, host cores) as the reference arm; each step is a
    bounded sample (one sequence, all 64 heads) of the headline workload."""
    if rank != 0:
        return
    from oracle import oracle as orc
    orc.build()
    dec, _ = gen.make_workload(HEADLINE)
    q, k, v = gen.bits(dec.q), gen.bits(dec.k), gen.bits(dec.v)
    lens = dec.seq_lens.numpy()

    def one(i):
        b = i % dec.batch
        orc.decode(q, k, v, lens, dec.softmax_scale, select=[(b, h) for h in range(64)])
        return int(lens[b])

    for i in range(max(3, args.warmup)):
        one(i)
    t0 = time.time()
    toks = sum(one(i) for i in range(args.steps))
    t = time.time() - t0
    value = toks / t
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) q/K/V, bf16)", "impl": "reference",
        "config": {"workload": gen.WORKLOADS[HEADLINE]["name"], "batch_per_gpu": dec.batch,
                   "seq_len": 4096, "q_heads": 64, "head_dim": 256, "kv_heads": 1},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.num_threads(), "cpu": cpu_model(),
                         "kind": "oracle",
                         "sample": "per step one sequence (all 64 heads, L=4096) of the "
                                   "headline workload, float64 C oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """Small case for Nsight Compute: plain (non-graph) launches, inputs > L2,
    a few hundred MB on the device."""
    from decode_attention_08_b200 import build, mfa
    build.build()
    torch.cuda.set_device(0)
    if args.profile == "lse_merge":
        # a sequence batch split over 8 GPUs: 8 parts x 256 sequences (134 MB > L2)
        inp = gen.make_lse_merge_inputs(4200, 8, 256)
        o, l = inp.o_parts.cuda(), inp.lse_parts.cuda()
        out = torch.empty(256, 64, 256, dtype=torch.bfloat16, device="cuda")
        for _ in range(args.warmup + args.steps):
            mfa.lse_merge(o, l, out)
    elif args.profile == "qproj":
        proj = gen.make_proj_inputs(2005, 8)
        x, wa, wb = proj.x.cuda(), proj.w_qa.cuda(), proj.w_qb.cuda()
        q = torch.empty(8, wb.shape[1], dtype=torch.bfloat16, device="cuda")
        for _ in range(args.warmup + args.steps):
            mfa.query_proj(x, wa, wb, q)
    elif args.profile == "out_proj":
        inp = gen.make_out_proj_inputs(4008, 8)
        o, wo = inp.o.cuda(), inp.w_o.cuda()
        y = torch.empty(8, wo.shape[1], dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(mfa.output_proj_workspace_size(8, o.shape[1], wo.shape[1]),
                         dtype=torch.uint8, device="cuda")
        for _ in range(args.warmup + args.steps):
            mfa.output_proj(o, wo, y, ws)
    elif args.profile == "kv_append":
        inp = gen.make_kv_append_inputs(3064, 64)
        x, wk, wv = inp.x.cuda(), inp.w_k.cuda(), inp.w_v.cuda()
        kc = torch.zeros(64, 4096, 256, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        pos = torch.full((64,), 4000, dtype=torch.int32, device="cuda")
        for _ in range(args.warmup + args.steps):
            mfa.kv_append(x, wk, wv, kc, vc, pos)
    elif args.profile == "gqa":
        inp = gen.make_gqa_inputs(1100, 48, 4096)
        step = GqaStep(inp, copies=1)
        for i in range(args.warmup + args.steps):
            step.call(i)
    elif args.profile == "fused":
        dec, proj = gen.make_workload(5)
        step = FusedStep(dec, proj, 1, dec.meta.get("num_splits", 0))
        for i in range(args.warmup + args.steps):
            step.call(i)
    else:
        if args.profile == "decode":
            dec = gen.make_decode_inputs(1002, 48, 4096)
        elif args.profile == "fp8":
            dec = gen.make_decode_inputs(1004, 96, 4096, kv_dtype="e4m3")
        else:
            lens = gen.workload_lengths(3)[:40].tolist()
            dec = gen.make_decode_inputs(1003, 40, lens, page_size=64)
        step = DecodeStep(dec, copies=1)
        for i in range(args.warmup + args.steps):
            step.call(i)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": args.profile, "launch_groups": args.warmup + args.steps,
                      "status": mfa.read_status()}))


def main(argv=None, runner=None):
    """Entry point. `runner(args, world, rank, local)` runs one rank's work
    (default: the benchmark itself)."""
    args = parse_args(argv)
    if args.profile:
        run_profile_case(args)
        return
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # launch one rank per GPU ourselves (under torchrun they already exist)
        spawn_ranks(args.gpus, main, sys.argv[1:] if argv is None else list(argv), runner)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        (runner or run_ours)(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
