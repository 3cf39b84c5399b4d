"""Benchmark of the contextually sparse LoRA hot path on one Llama-2-7B-shaped
SwiGLU FFN layer (d=4096, d_ff=11008, batch 8 x seq 512, last 25% of each
sequence dense output tokens, SVD rank 8, LoRA rank 16 on gate/up/down,
sparsity 50%, bf16, forward + backward).

One step = slora_ffn_fwd_bwd: estimate + select + sliced forward + sliced
backward for one batch.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): data parallel, every rank runs its
own batch (weak scaling); the six LoRA gradients, packed in one flat buffer,
are summed across ranks with one NCCL all-reduce per step.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from contextual_sparsity_lora_svd_b200 import synth  # noqa: E402

WORKLOAD = synth.WORKLOADS[1]
METRIC = "sparse LoRA fwd+bwd tokens/s; sliced-GEMM % bf16 peak; estimator HBM GB/s"
UNIT = "tokens/s"


def measured_traffic(kernel_file, summary):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when the kernel source changed since the capture."""
    import hashlib
    try:
        src = os.path.join(ROOT, "contextual_sparsity_lora_svd_b200", "csrc", kernel_file)
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
        vals = {}
        for line in open(os.path.join(ROOT, "profiles", summary)):
            if ":" in line and line.split(":")[0] in ("traffic_bytes_per_launch",
                                                      "kernel_source_sha256"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
        if vals.get("kernel_source_sha256") != sha:
            return None
        return float(vals["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return dict(hbm=m["hbm_gbs"], bf16=m["bf16_tflops"], bf16_sus=m["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every `period` s."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period: float = 0.002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period, self.stop_ev = period, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_ev.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": [],
                    "samples": 0}
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ inputs
_CASE = {}


def make_case(batch=None, seq=None):
    """The full workload (default) or its first `batch` sequences of length
    `seq`: the same weights and the same leading rows of X and dOut."""
    import dataclasses
    w = WORKLOAD
    if "full" not in _CASE:
        tok = synth.Tokens.uniform(w["batch"], w["seq"], w["out_frac"])
        _CASE["full"] = synth.ffn_case(tok, w["d"], w["d_ff"], w["r_svd"], w["r_lora"],
                                       w["sparsity"], bf16=True, workload=1, fast=True)
    full = _CASE["full"]
    if batch is None and seq is None:
        return full
    assert seq == w["seq"]
    tok = synth.Tokens.uniform(batch, seq, w["out_frac"])
    return dataclasses.replace(full, tokens=tok, X=full.X[:tok.T], dOut=full.dOut[:tok.T])


class GpuLayer:
    """Device copies of one layer plus outputs/grads/workspace for bench steps."""

    def __init__(self, case, L):
        self.L, self.case = L, case
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(
            torch.bfloat16).cuda()
        w = WORKLOAD
        d, F, r, rs = w["d"], w["d_ff"], w["r_lora"], w["r_svd"]
        self.d, self.F, self.r = d, F, r
        self.t = {k: bf(getattr(case, k)) for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
        for k in ("Wg", "Wu", "Wd"):
            self.t[k] = bf(getattr(case, k).W)
        # offline prepare (not timed): estimator factors of gate/up, Wd^T for the down proj
        self.t["Wd_t"] = torch.empty(F, d, dtype=torch.bfloat16, device="cuda")
        for nm, n, k in (("g", F, d), ("u", F, d)):
            self.t["L" + nm] = torch.empty(k, rs, device="cuda")
            self.t["U" + nm] = torch.empty(n, rs, device="cuda")
            L.slora_svd_prepare(self.t["W" + nm], rs, self.t["L" + nm], self.t["U" + nm], seed=7)
        Ld = torch.empty(F, rs, device="cuda")
        Ud = torch.empty(d, rs, device="cuda")
        L.slora_svd_prepare(self.t["Wd"], rs, Ld, Ud, W_t=self.t["Wd_t"], seed=7)
        del self.t["Wd"]
        t = self.t
        self.layer = L.ffn_layer_struct(d, F, rs, r, case.lora_scale, t["Wg"], t["Wu"], t["Wd_t"],
                                        t["Ag"], t["Bg"], t["Au"], t["Bu"], t["Ad"], t["Bd"],
                                        t["Lg"], t["Ug"], t["Lu"], t["Uu"])
        self.io = [self.make_io(bf(case.X), bf(case.dOut))]
        self.X, self.dOut, self.out, self.dX, self.gflat = (self.io[0][k] for k in
                                                            ("X", "dOut", "out", "dX", "gflat"))
        need = L.workspace_size("slora_ffn_fwd_bwd", self.io[0]["args"])
        self.ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        self.ws_bytes = L.c_sz(need)

    def make_io(self, X, dOut):
        """Per-step inputs, outputs and LoRA gradients (one flat fp32 buffer)."""
        L, d, F, r = self.L, self.d, self.F, self.r
        T = self.case.tokens.T
        io = {"X": X, "dOut": dOut,
              "out": torch.empty(T, d, dtype=torch.bfloat16, device="cuda"),
              "dX": torch.empty(T, d, dtype=torch.bfloat16, device="cuda"),
              "idx": torch.empty(F, dtype=torch.int32, device="cuda")}
        shapes = [(r, d), (F, r), (r, d), (F, r), (r, F), (d, r)]
        io["gflat"] = torch.zeros(sum(a * b for a, b in shapes), device="cuda")
        grads, o = [], 0
        for a, b in shapes:
            grads.append(io["gflat"][o:o + a * b].view(a, b))
            o += a * b
        io["gstruct"] = L.ffn_grads_struct(*grads)
        tok = self.case.tokens
        io["args"], io["keep"] = L.ffn_args(L.BF16, self.layer, tok.batch, tok.seq, tok.ctx_len,
                                            self.case.sparsity, io["X"], io["dOut"], io["out"],
                                            io["dX"], io["gstruct"], io["idx"])
        return io

    def step(self, stream, io=None):
        import ctypes
        L = self.L
        io = io or self.io[0]
        st = L.lib().slora_ffn_fwd_bwd(*io["args"], L.ptr(self.ws), ctypes.byref(self.ws_bytes),
                                       stream.cuda_stream)
        if st != 0:
            raise L.SloraError("slora_ffn_fwd_bwd", st, L.lib().slora_last_error_string().decode())


# ------------------------------------------------------------ CPU oracle
def oracle_step_time(case, reps=1):
    """Seconds for the oracle's fwd+bwd of `case` (estimate, select, sliced
    fwd/bwd), on this host's cores.  Estimator factors: the closed-form top-r
    singular triplets of the construction."""
    from oracle import slora_oracle as O
    r = WORKLOAD["r_svd"]
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=case.lora_scale)
    for nm, sw in (("g", case.Wg), ("u", case.Wu)):
        lay["L" + nm] = sw.V[:, :r] * sw.s[None, :r]
        lay["U" + nm] = sw.U[:, :r].copy()
    tok = case.tokens
    t0 = time.perf_counter()
    for _ in range(reps):
        O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay, case.sparsity)
    return (time.perf_counter() - t0) / reps


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def set_threads():
    n = str(host_cores())
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ.setdefault(v, n)
    torch.set_num_threads(int(n))


CPU_SAMPLE = dict(batch=1, seq=512)  # one sequence: 384 context + 128 output tokens


def cpu_baseline():
    case = make_case(**CPU_SAMPLE)
    oracle_step_time(case)  # warm the BLAS pools
    t = oracle_step_time(case, reps=3)
    T = case.tokens.T
    return {"value": T / t, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
            "sample": f"{CPU_SAMPLE['batch']} x {CPU_SAMPLE['seq']} tokens of the same layer "
                      f"(ctx 384 + out 128), fp64 NumPy oracle, 3 reps after 1 warm-up"}


# ------------------------------------------------------------------- arms
def config_dict(world):
    w = WORKLOAD
    return {"workload": w["name"], "model": "Llama-2-7B FFN layer (random init, decaying spectrum)",
            "global_batch": w["batch"] * world, "seq_len": w["seq"], "d": w["d"],
            "d_ff": w["d_ff"], "ctx_frac": 1 - w["out_frac"], "sparsity": w["sparsity"],
            "r_svd": w["r_svd"], "r_lora": w["r_lora"],
            "parallelism": f"dp{world}" if world > 1 else "single",
            "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
            "launch": "one slora_ffn_fwd_bwd call captured as a CUDA graph, replayed per step "
                      "(per-kernel times from a separate eager pass)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    set_threads()
    case = make_case(**CPU_SAMPLE)
    for _ in range(args.warmup):
        oracle_step_time(case)
    ts = [oracle_step_time(case) for _ in range(args.steps)]
    T = case.tokens.T
    v = T / float(np.mean(ts))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(ts)),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(world),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                             "sample": f"each step: {T} tokens ({CPU_SAMPLE['batch']} x "
                                       f"{CPU_SAMPLE['seq']}) of the workload, fp64 NumPy oracle"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world):
    from contextual_sparsity_lora_svd_b200 import _lib as L
    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    pk = peaks()
    case = make_case()
    if world > 1:
        # weak scaling: every rank runs its own 8 x 512-token batch, drawn from
        # its own seeds (same layer weights on every rank)
        import dataclasses
        T, d = case.X.shape
        seed = 1000 * 1 + 1_000_003 * (rank + 1)
        case = dataclasses.replace(
            case, X=synth.round_bf16(synth.gaussian((T, d), 1.0, seed)),
            dOut=synth.round_bf16(synth.gaussian((T, d), 1.0, seed + 1)))
    G = GpuLayer(case, L)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    T = case.tokens.T

    from contextual_sparsity_lora_svd_b200 import dp

    def one_step():
        # each rank runs its own block of sequences (weak scaling: 8 x 512 tokens
        # per GPU), selecting from its own context tokens; the LoRA gradients are
        # then summed over ranks (one NCCL all-reduce of the flat fp32 buffer)
        G.step(stream)
        dp.allreduce_grads(G.gflat)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    # one step captured as a CUDA graph per buffer set (the library call is
    # capture-safe: fixed buffers and tensor maps per workspace); the headline
    # and end-to-end passes replay it, the per-kernel profiled pass runs eagerly
    if len(G.io) < 2:
        G.io.append(G.make_io(torch.empty_like(G.X), torch.empty_like(G.dOut)))

    def capture(io):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            G.step(torch.cuda.current_stream(), io)
        return g

    graphs = [capture(io) for io in G.io]
    torch.cuda.synchronize()

    def graph_step():
        graphs[0].replay()
        dp.allreduce_grads(G.gflat)

    for _ in range(args.warmup):
        graph_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()

    def timed(profile, step_fn):
        """K steps bracketed by CUDA events on the launching stream, L2 flushed
        (outside the events) before each; with `profile` every launch of the
        library is also bracketed by events, per kernel class."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        if profile:
            L.profile_enable(True)
        n0 = L.launch_count()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            step_fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        launches = L.launch_count() - n0
        prof = None
        if profile:
            prof = {c: L.profile_read(c) for c in L.KERNEL_CLASSES}
            L.profile_enable(False)
        return float(sum(a.elapsed_time(b) for a, b in ev)), launches, prof

    if args.profile_region:
        torch.cuda.profiler.start()
    with ClockSampler(dev) as clk:
        ms, _, _ = timed(False, graph_step)
    if args.profile_region:
        torch.cuda.profiler.stop()
    # per-kernel durations: a second timed pass with events around every launch
    ms_prof, launches_prof, prof = timed(True, one_step)
    launches = launches_prof  # the graph replays the same launches as the eager step
    ms = dp.max_over_ranks(ms, device="cuda")
    ms_step = ms / args.steps
    value = world * T / (ms_step / 1e3)

    # ---- end to end through the public API with host buffers: every step's
    # inputs go host->device and its outputs device->host inside the timed
    # region; copies run on their own streams, double-buffered, so step i+1's
    # upload and step i-1's download overlap step i's compute.
    Xh = G.X.cpu().pin_memory()
    dOh = G.dOut.cpu().pin_memory()
    outs = [{k: torch.empty_like(io[k], device="cpu").pin_memory() for k in ("out", "dX", "gflat")}
            for io in G.io]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    e2e_steps = max(2, min(args.steps, 10))
    up = [torch.cuda.Event() for _ in range(2)]      # inputs of set i landed
    done = [torch.cuda.Event() for _ in range(2)]    # compute on set i finished
    down = [torch.cuda.Event() for _ in range(2)]    # outputs of set i read back
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d_s)
    stream.wait_event(e0)
    d2h_s.wait_event(e0)

    def upload(i):
        io = G.io[i % 2]
        with torch.cuda.stream(h2d_s):
            if i >= 2:
                h2d_s.wait_event(done[i % 2])  # step i-2 has finished reading this set
            io["X"].copy_(Xh, non_blocking=True)
            io["dOut"].copy_(dOh, non_blocking=True)
            up[i % 2].record(h2d_s)

    upload(0)
    for i in range(e2e_steps):
        if i + 1 < e2e_steps:
            upload(i + 1)
        io = G.io[i % 2]
        stream.wait_event(up[i % 2])
        if i >= 2:
            stream.wait_event(down[i % 2])  # step i-2's outputs are read back
        graphs[i % 2].replay()
        dp.allreduce_grads(io["gflat"])
        done[i % 2].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(done[i % 2])
            for k in ("out", "dX", "gflat"):
                outs[i % 2][k].copy_(io[k], non_blocking=True)
            down[i % 2].record(d2h_s)
    e1.record(d2h_s)
    torch.cuda.synchronize()
    e2e_ms = dp.max_over_ranks(e0.elapsed_time(e1) / e2e_steps, device="cuda")
    h2d = Xh.numel() * 2 + dOh.numel() * 2
    d2h = sum(outs[0][k].numel() * outs[0][k].element_size() for k in ("out", "dX", "gflat"))

    # ---- roofline of the dominant kernel class (by device time)
    kernels = {}
    ktot = sum(v[1] for v in prof.values())
    for c, (n, kms, work) in prof.items():
        if n:
            kernels[c] = {"launches_per_step": n / args.steps, "ms_per_step": kms / args.steps,
                          "share": kms / ktot if ktot > 0 else None,
                          "share_of_step": kms / ms_prof if ms_prof > 0 else None}
    gemm_cls = max(("gemm_tc", "gemm_simt"), key=lambda c: prof[c][1])
    n_g, ms_g, fl_g = prof[gemm_cls]
    achieved = fl_g / (ms_g / 1e3) / 1e12 if ms_g > 0 else 0.0
    traffic = (measured_traffic("gemm_tc.cu", "tc_gemm_llama2_7b_ffn_bf16.md")
               if gemm_cls == "gemm_tc" else None)
    roof = {"kernel": gemm_cls, "bound": "tensor", "achieved": achieved, "peak": pk["bf16"],
            "unit": "TFLOP/s", "frac": achieved / pk["bf16"], "traffic": traffic,
            "peak_kind": f"bf16 burst, {pk['src']}",
            "frac_of_sustained": achieved / pk["bf16_sus"],
            "flops_per_launch": fl_g / max(n_g, 1), "ms_per_launch": ms_g / max(n_g, 1)}
    n_e, ms_e, by_e = prof["estimate"]
    n_s, ms_s, by_s = prof["select"]
    est = {"ms_per_step": (ms_e + ms_s) / args.steps,
           "GB/s": (by_e + by_s) / ((ms_e + ms_s) / 1e3) / 1e9 if ms_e + ms_s > 0 else None}
    if est["GB/s"]:
        est["frac_hbm"] = est["GB/s"] / pk["hbm"]
    # The FFN score is bound by arithmetic, not HBM: per (context token, channel)
    # pair it needs 2 r_svd FMAs and two MUFU ops (exp, reciprocal) for the silu.
    # Per SM and clock: 128 fp32 FMA lanes, 16 MUFU lanes; 148 SMs at the sampled
    # SM clock (the maximum when NVML gave none).
    w = WORKLOAD
    pairs = w["batch"] * (w["seq"] - int(round(w["out_frac"] * w["seq"]))) * w["d_ff"]
    mhz = clk.summary().get("sm_mhz") or clk.summary().get("sm_max_mhz") or 1965.0
    hz = float(mhz) * 1e6
    t_fma = pairs * 2 * w["r_svd"] / (128 * 148 * hz)
    t_mufu = pairs * 2 / (16 * 148 * hz)
    if ms_e > 0:
        est["score_alu"] = {"bound": "alu", "pairs": pairs, "bound_us": 1e6 * max(t_fma, t_mufu),
                            "achieved_us": 1e3 * ms_e / args.steps,
                            "frac": 1e6 * max(t_fma, t_mufu) / (1e3 * ms_e / args.steps)}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Llama-2-7B-shaped inputs, random-init decaying-spectrum "
                    "weights)",
            "config": config_dict(world), "roofline": roof, "estimator": est,
            "kernels": kernels, "gpu_launches": int(launches),
            "clocks": clk.summary(),
            "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "overlap": "double-buffered: H2D, compute and D2H on separate streams"},
            "profiled_ms_per_step": ms_prof / args.steps,
            "impl": "ours"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        set_threads()
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def torchrun_argv(argv, n, script=None, port=None):
    """Command that runs `script` (this file by default) with `argv` as N
    ranks on this node, one process per GPU, rendezvous on 127.0.0.1."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
            "--master-port", str(port or free_port()),
            os.path.abspath(script or __file__), *argv]


def launch(argv, n, script=None, timeout_s=None) -> int:
    """Starts N ranks of `script` under torch.distributed.run and returns the
    launcher's exit status."""
    import subprocess
    return subprocess.run(torchrun_argv(argv, n, script), timeout=timeout_s).returncode


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-region", action="store_true",
                    help="bracket the timed steps with cudaProfilerStart/Stop (for ncu "
                         "--profile-from-start off)")
    args = ap.parse_args()
    if args.gpus < 1:
        raise SystemExit("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: start the N ranks ourselves
        raise SystemExit(launch(sys.argv[1:], args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        from contextual_sparsity_lora_svd_b200 import dp
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dp.init_from_env("nccl", timeout_s=120)
    try:
        run_ours(args, rank, world)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
