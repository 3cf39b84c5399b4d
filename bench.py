"""Benchmark of the contextually sparse LoRA hot path on B200.

Workloads (synthetic Llama-shaped inputs, random-init decaying-spectrum
weights; `--workload`, default the first):

  llama2-7b-ffn-bf16      one SwiGLU FFN layer, d=4096, d_ff=11008, batch 8 x
                          seq 512 (last 25% of each sequence dense output
                          tokens), SVD rank 8, LoRA rank 16 on gate/up/down,
                          sparsity 50%: one step = slora_ffn_fwd_bwd (estimate
                          + select + sliced forward + sliced backward).
  llama2-7b-attn-qk-bf16  the q/k/v/o LoRA linears of one attention layer,
                          32 heads x 128, batch 4 x seq 1024: q/k sliced per
                          head at 50% by the QK-norm estimate, v/o dense;
                          variants: rotate-half pair selection, v/o sliced.
  llama2-7b-stack32-bf16  32 layers of the two above with the per-layer ratio
                          table (layers 0-3 dense, FFN 0.5 -> 0.9, q/k 0.3 ->
                          0.6) and the progressive schedule (dense for the
                          first 10% of a run).
  llama3-8b-layer-bf16    one Llama-3-8B-shaped layer (d_ff=14336, GQA 32 q /
                          8 kv heads), 8192 tokens: sparsity x SVD-rank sweep
                          at seq 1024 and a sequence sweep at 50% / rank 8.
  llama2-7b-decoder32-bf16  the 32-layer stack's whole training step with the
                          attention core, RMS norms and residuals (forward of
                          every layer, then backward), beside the same stack
                          run dense.

Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME]

Timing: the step's library calls are captured once as a CUDA graph and
replayed; CUDA events on the launching stream bracket each step; a 256 MiB
write flushes L2 between steps, outside the events.  A second, eager pass
brackets every library launch with events for the per-kernel-class times.
Multi-GPU (one process per GPU, started by `--gpus N` itself): data parallel,
every rank runs its own batch (weak scaling); the LoRA gradients, packed in
one flat fp32 buffer per layer, are summed over ranks with one NCCL
all-reduce per step.
"""
from __future__ import annotations

import argparse
import hashlib
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

METRIC = "sparse LoRA fwd+bwd tokens/s; sliced-GEMM % bf16 peak; estimator HBM GB/s"
UNIT = "tokens/s"
WORKLOAD_NAMES = ["llama2-7b-ffn-bf16", "llama2-7b-attn-qk-bf16", "llama2-7b-stack32-bf16",
                  "llama3-8b-layer-bf16", "llama2-7b-decoder32-bf16"]


# ------------------------------------------------------------------ peaks
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return dict(hbm=m["hbm_gbs"], bf16=m["bf16_tflops"], bf16_sus=m["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def measured_traffic(kernel_file, workload):
    """DRAM bytes per launch of the dominant kernel from one ncu capture
    (profiles/ncu_traffic.json), or None when the kernel source changed since."""
    try:
        src = os.path.join(ROOT, "contextual_sparsity_lora_svd_b200", "csrc", kernel_file)
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            rec = json.load(f).get(kernel_file, {}).get(workload)
        if not rec or rec.get("source_sha256") != sha:
            return None
        return float(rec["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


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


# ------------------------------------------------------------------ host
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


def to_host(t):
    return t.detach().double().cpu().numpy()


# ------------------------------------------------------------- configs
L2_NOTE = "flushed between timed steps (256 MiB write, outside the events)"


def workload_config(name, world):
    """The `config` object of a workload's JSON line (both arms)."""
    par = f"dp{world}" if world > 1 else "single"
    if name == "llama2-7b-ffn-bf16":
        w = synth.WORKLOADS[1]
        return {"workload": name, "model": "Llama-2-7B FFN layer (random init, decaying spectrum)",
                "global_batch": w["batch"] * world, "seq_len": w["seq"], "d": w["d"],
                "d_ff": w["d_ff"], "ctx_frac": 1 - w["out_frac"], "sparsity": w["sparsity"],
                "r_svd": w["r_svd"], "r_lora": w["r_lora"], "parallelism": par, "l2": L2_NOTE,
                "launch": "one slora_ffn_fwd_bwd call captured as a CUDA graph, replayed per "
                          "step (per-kernel times from an eager pass)"}
    if name == "llama2-7b-attn-qk-bf16":
        w = synth.WORKLOADS[2]
        return {"workload": name, "model": "Llama-2-7B attention q/k/v/o LoRA linears "
                                           "(random init)",
                "global_batch": w["batch"] * world, "seq_len": w["seq"], "d": w["d"],
                "heads": w["heads"], "kv_heads": w["kv_heads"], "head_dim": w["head_dim"],
                "ctx_frac": 0.75, "qk_sparsity": w["sparsity"], "v_o": "dense LoRA",
                "r_svd": w["r_svd"], "r_lora": w["r_lora"], "parallelism": par,
                "attention_core": "excluded (its output and input gradients are synthetic "
                                  "tensors)", "l2": L2_NOTE}
    if name == "llama2-7b-stack32-bf16":
        from contextual_sparsity_lora_svd_b200.schedule import llama2_7b_stack
        w = synth.WORKLOADS[3]
        t = llama2_7b_stack()
        return {"workload": name, "model": "32 Llama-2-7B layers: q/k/v/o LoRA linears + SwiGLU "
                                           "FFN",
                "global_batch": w["batch"] * world, "seq_len": w["seq"], "layers": w["layers"],
                "d": w["d"], "d_ff": w["d_ff"], "heads": w["heads"], "r_svd": w["r_svd"],
                "r_lora": w["r_lora"], "ffn_sparsity": list(t.ffn), "qk_sparsity": list(t.qk),
                "v_o": "dense LoRA",
                "excluded": "attention core, norms, embeddings (their tensors are synthetic; "
                            "every layer reads the same X)", "parallelism": par, "l2": L2_NOTE}
    if name == "llama2-7b-decoder32-bf16":
        from contextual_sparsity_lora_svd_b200.schedule import llama2_7b_stack
        w = synth.WORKLOADS[3]
        t = llama2_7b_stack()
        return {"workload": name, "model": "32 Llama-2-7B decoder layers: RMS norms, q/k/v/o "
                                           "LoRA linears, rotary embedding, causal attention, "
                                           "residuals, SwiGLU FFN",
                "global_batch": w["batch"] * world, "seq_len": w["seq"], "layers": w["layers"],
                "d": w["d"], "d_ff": w["d_ff"], "heads": w["heads"], "r_svd": w["r_svd"],
                "r_lora": w["r_lora"], "ffn_sparsity": list(t.ffn), "qk_sparsity": list(t.qk),
                "v_o": "dense LoRA", "ffn_backward": "from the forward state kept in each "
                                                     "layer's FFN workspace (slora_ffn_bwd)",
                "excluded": "embeddings, final norm and loss (a synthetic output gradient)",
                "parallelism": par, "l2": L2_NOTE,
                "launch": "the whole step (forward of 32 layers, then backward) captured as one "
                          "CUDA graph"}
    w = synth.WORKLOADS[4]
    return {"workload": name, "model": "Llama-3-8B layer: q/k/v/o LoRA linears (GQA 32/8) + "
                                       "SwiGLU FFN",
            "tokens": w["tokens"], "headline_point": {"sparsity": 0.5, "r_svd": 8, "seq": 1024},
            "d": w["d"], "d_ff": w["d_ff"], "heads": w["heads"], "kv_heads": w["kv_heads"],
            "r_lora": w["r_lora"], "parallelism": par, "l2": L2_NOTE}


# ------------------------------------------------------------- GPU inputs
class WeightFactory:
    """Decaying-spectrum weights W = c Q1 diag(i^-0.7) Q2^T (RMS 0.02) built on
    the GPU with torch (benchmark inputs only).  Q1, Q2 come from the QR of a
    seeded Gaussian per shape; further weights of the same shape reuse them
    under a seeded row permutation and column sign flip (still orthonormal),
    so a 32-layer stack gets distinct weights without 200 QRs."""

    def __init__(self):
        self.base = {}

    def _q(self, n, m, tag):
        key = (n, m, tag)
        if key not in self.base:
            g = torch.Generator(device="cuda").manual_seed(n * 1_000_003 + m * 31 + tag)
            a = torch.randn(n, m, device="cuda", generator=g)
            q, r = torch.linalg.qr(a)
            self.base[key] = q * torch.sign(torch.diagonal(r))[None, :]
        return self.base[key]

    def weight(self, n, k, seed):
        m = min(n, k)
        g = torch.Generator(device="cuda").manual_seed(int(seed))
        q1 = self._q(n, m, 1)[torch.randperm(n, device="cuda", generator=g)]
        q2 = self._q(k, m, 2)[torch.randperm(k, device="cuda", generator=g)]
        sg = torch.randint(0, 2, (m,), device="cuda", generator=g).float() * 2 - 1
        s = torch.arange(1, m + 1, device="cuda", dtype=torch.float64) ** (-0.7)
        c = 0.02 * np.sqrt(n * k / float(torch.sum(s * s)))
        w = (q1 * (sg * (c * s).float())[None, :]) @ q2.T
        return w.to(torch.bfloat16)


def lora_pair(n, k, r, seed):
    g = torch.Generator(device="cuda").manual_seed(int(seed))
    A = (torch.randn(r, k, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    B = (torch.randn(n, r, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    return A, B


def randn_bf16(shape, seed):
    g = torch.Generator(device="cuda").manual_seed(int(seed))
    return torch.randn(*shape, device="cuda", generator=g).to(torch.bfloat16)


def prepare_factors(L, W, r):
    n, k = W.shape
    Lf = torch.empty(k, r, device="cuda")
    Uf = torch.empty(n, r, device="cuda")
    L.slora_svd_prepare(W, r, Lf, Uf, seed=7)
    return Lf, Uf


def ffn_weights_gpu(L, wf, d, d_ff, r_svds, r_lora, seed):
    """Device weights of one FFN layer and its estimator factors per rank."""
    w = {"Wg": wf.weight(d_ff, d, seed + 2), "Wu": wf.weight(d_ff, d, seed + 3)}
    w["Wd_t"] = wf.weight(d, d_ff, seed + 4).t().contiguous()
    w["Ag"], w["Bg"] = lora_pair(d_ff, d, r_lora, seed + 5)
    w["Au"], w["Bu"] = lora_pair(d_ff, d, r_lora, seed + 7)
    w["Ad"], w["Bd"] = lora_pair(d, d_ff, r_lora, seed + 9)
    fac = {}
    for r in r_svds:
        fac[r] = prepare_factors(L, w["Wg"], r) + prepare_factors(L, w["Wu"], r)
    return w, fac


def attn_weights_gpu(L, wf, d, H, KV, hd, r_svds, r_lora, seed, vo=False):
    nq, nkv = H * hd, KV * hd
    w = {"Wq": wf.weight(nq, d, seed + 12), "Wk": wf.weight(nkv, d, seed + 13),
         "Wv": wf.weight(nkv, d, seed + 14), "Wo": wf.weight(d, nq, seed + 15)}
    if vo:
        w["Wo_t"] = w["Wo"].t().contiguous()
    for nm, n, k, sd in (("q", nq, d, 16), ("k", nkv, d, 18), ("v", nkv, d, 20),
                         ("o", d, nq, 22)):
        w["A" + nm], w["B" + nm] = lora_pair(n, k, r_lora, seed + sd)
    fac = {}
    for r in r_svds:
        f = {}
        f["Lq"], f["Uq"] = prepare_factors(L, w["Wq"], r)
        f["Lk"], f["Uk"] = prepare_factors(L, w["Wk"], r)
        if vo:
            f["Lv"], f["Uv"] = prepare_factors(L, w["Wv"], r)
        fac[r] = f
    return w, fac


# ------------------------------------------------------------------ timing
class Harness:
    def __init__(self, L, dev, world, profile_region=False):
        self.L, self.dev, self.world = L, dev, world
        self.stream = torch.cuda.current_stream()
        self.flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        # bracket the first timed region with cudaProfilerStart/Stop (for ncu
        # --profile-from-start off)
        self.profile_region = profile_region

    def capture(self, fn):
        """CUDA graph of fn() on a side capture stream (one library step)."""
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        return g

    def barrier(self):
        torch.cuda.synchronize()
        if self.world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    def time_steps(self, step, steps, after=None):
        """Total ms of `steps` calls of step(), each bracketed by events on the
        launching stream with an L2 flush before it (outside the events)."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        self.barrier()
        region, self.profile_region = self.profile_region, False
        if region:
            torch.cuda.profiler.start()
        for i in range(steps):
            self.flush_buf.zero_()
            ev[i][0].record(self.stream)
            step()
            if after:
                after()
            ev[i][1].record(self.stream)
        torch.cuda.synchronize()
        if region:
            torch.cuda.profiler.stop()
        return float(sum(a.elapsed_time(b) for a, b in ev))

    def profile(self, step, steps, after=None):
        """Eager pass with events around every library launch: (total ms,
        launches, {class: (launches, ms, work)})."""
        L = self.L
        L.profile_enable(True)
        n0 = L.launch_count()
        ms = self.time_steps(step, steps, after)
        launches = L.launch_count() - n0
        prof = {c: L.profile_read(c) for c in L.KERNEL_CLASSES}
        L.profile_enable(False)
        return ms, launches, prof


def kernel_table(prof, steps, ms_prof):
    out = {}
    ktot = sum(v[1] for v in prof.values())
    for c, (n, kms, work) in prof.items():
        if n:
            out[c] = {"launches_per_step": n / steps, "ms_per_step": kms / steps,
                      "share": kms / ktot if ktot > 0 else None,
                      "share_of_step": kms / ms_prof if ms_prof > 0 else None}
    return out


def gemm_roofline(prof, pk, kernel_file="gemm_tc.cu", workload=None):
    n_g, ms_g, fl_g = prof["gemm_tc"]
    achieved = fl_g / (ms_g / 1e3) / 1e12 if ms_g > 0 else 0.0
    return {"kernel": "tc_gemm2_kernel (tcgen05 sliced GEMMs)", "bound": "tensor",
            "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
            "frac": achieved / pk["bf16"],
            "traffic": measured_traffic(kernel_file, workload) if workload else None,
            "peak_kind": f"bf16 burst, {pk['src']}",
            "frac_of_sustained": achieved / pk["bf16_sus"],
            "flops_per_launch": fl_g / max(n_g, 1), "ms_per_launch": ms_g / max(n_g, 1)}


def sm_count():
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


# --------------------------------------------------- standalone estimator
class Estimator:
    """One standalone slora_estimate_select call (its own workspace), for the
    estimate+select measurement by algorithmic bytes: X_C read once, both
    factor pairs, the scores written and the indices written."""

    def __init__(self, L, crit, X, batch, seq, ctx_len, L0, U0, L1, U1, r, s, heads=0, kv=0,
                 hd=0):
        import ctypes
        from contextual_sparsity_lora_svd_b200.layers import _Call
        self.L = L
        n0, n1 = U0.shape[0], U1.shape[0]
        self.tok, self.keep = L.make_tokens(batch, seq, ctx_len)
        self.k_out = L.c_i32(0)
        nidx = max(n0 + n1, (heads + kv) * hd)
        self.idx = torch.empty(nidx, dtype=torch.int32, device="cuda")
        self.scores = torch.empty(max(n0, n1), device="cuda")
        d = X.shape[1]
        args = [crit, L.ptr(X), L.BF16, ctypes.byref(self.tok), d, L.ptr(L0), L.ptr(U0), n0,
                L.ptr(L1), L.ptr(U1), n1, r, heads, kv, hd, float(s), L.ptr(self.idx),
                ctypes.byref(self.k_out), L.ptr(self.scores)]
        self.call = _Call("slora_estimate_select", args)
        need = self.call.need()
        self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
        T_C = int(sum(int(c) for c in ctx_len))
        crit_ffn = crit in (L.CRIT_FFN, L.CRIT_FFN_GRAM)
        n_scores = n0 if crit_ffn else (kv * hd // (2 if crit == L.CRIT_QK_ROPE_PAIR else 1))
        n_out = int(self.k_out.value) * (1 if crit_ffn else heads + kv)
        nfac = 2 if crit != L.CRIT_L2 else 1
        self.bytes = (T_C * d * 2 + (nfac * d + n0 + (n1 if nfac == 2 else 0)) * r * 4 +
                      n_scores * 4 + n_out * 4)
        self.pairs = T_C * n0 if crit == L.CRIT_FFN else 0
        self.r = r

    def __call__(self):
        self.call(self.ws.data_ptr(), self.L.c_sz(self.ws.numel()),
                  torch.cuda.current_stream().cuda_stream)


def measure_estimator(H, est, steps, pk, clk_mhz):
    """Standalone estimate+select: graph replay time with L2 flushed, the
    launch breakdown from an eager pass, and the HBM / ALU fractions."""
    g = H.capture(est)
    for _ in range(3):
        g.replay()
    ms = H.time_steps(g.replay, steps) / steps
    ms_p, launches, prof = H.profile(est, steps)
    out = {"us_per_call": ms * 1e3, "bytes": est.bytes, "GB/s": est.bytes / (ms / 1e3) / 1e9,
           "launches_per_call": launches / steps,
           "kernels_us": {c: v[1] * 1e3 / steps for c, v in prof.items() if v[0]}}
    out["frac_hbm"] = out["GB/s"] / pk["hbm"]
    if est.pairs:
        # activation-norm score: per (context token, channel) pair two MUFU
        # ops (exp and reciprocal of the silu) on 16 MUFU lanes per SM and
        # clock, 2 r FMAs on 128 FMA lanes (the MUFU term binds)
        hz = float(clk_mhz) * 1e6
        nsm = sm_count()
        t_mufu = est.pairs * 2 / (16 * nsm * hz)
        t_fma = est.pairs * 2 * est.r / (128 * nsm * hz)
        bound = max(t_mufu, t_fma)
        score_us = out["kernels_us"].get("estimate", 0.0)
        out["score_alu"] = {"bound": "alu", "pairs": est.pairs, "bound_us": bound * 1e6,
                            "score_kernel_us": score_us,
                            "frac": bound * 1e6 / score_us if score_us > 0 else None,
                            "sm_mhz": clk_mhz}
    del g
    return out


# -------------------------------------------------------------- e2e helper
def e2e_measure(H, graphs, sets, in_keys, out_keys, steps, after=None):
    """End to end through the public API with host buffers: each step uploads
    its inputs from pinned host memory and reads back its outputs.  With two
    distinct buffer sets the copies run on their own streams, double-buffered
    (step i+1's upload and step i-1's read-back overlap step i); with one set
    every step runs upload, compute and read-back in order."""
    hin = {k: sets[0][k].cpu().pin_memory() for k in in_keys}
    hout = [{k: torch.empty_like(s[k], device="cpu").pin_memory() for k in out_keys}
            for s in sets]
    stream = H.stream
    H.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sets[0] is sets[1]:
        e0.record(stream)
        for i in range(steps):
            for k in in_keys:
                sets[0][k].copy_(hin[k], non_blocking=True)
            graphs[0].replay()
            if after:
                after(0)
            for k in out_keys:
                hout[0][k].copy_(sets[0][k], non_blocking=True)
        e1.record(stream)
    else:
        h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
        up = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        down = [torch.cuda.Event() for _ in range(2)]
        e0.record(h2d_s)
        stream.wait_event(e0)
        d2h_s.wait_event(e0)

        def upload(i):
            s_ = sets[i % 2]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(done[i % 2])  # step i-2 has finished reading this set
                for k in in_keys:
                    s_[k].copy_(hin[k], non_blocking=True)
                up[i % 2].record(h2d_s)

        upload(0)
        for i in range(steps):
            if i + 1 < steps:
                upload(i + 1)
            stream.wait_event(up[i % 2])
            if i >= 2:
                stream.wait_event(down[i % 2])  # step i-2's outputs are read back
            graphs[i % 2].replay()
            if after:
                after(i % 2)
            done[i % 2].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(done[i % 2])
                for k in out_keys:
                    hout[i % 2][k].copy_(sets[i % 2][k], non_blocking=True)
                down[i % 2].record(d2h_s)
        e1.record(d2h_s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = sum(v.numel() * v.element_size() for v in hin.values())
    d2h = sum(v.numel() * v.element_size() for v in hout[0].values())
    return ms, h2d, d2h


# =================================================================== FFN
def ffn_case_numpy(batch=None, seq=None, _cache={}):
    """The FFN workload's inputs (numpy, shared with the CPU oracle): the full
    8 x 512 batch, or its first `batch` sequences."""
    import dataclasses
    w = synth.WORKLOADS[1]
    if "full" not in _cache:
        tok = synth.Tokens.uniform(w["batch"], w["seq"], w["out_frac"])
        _cache["full"] = synth.ffn_case(tok, w["d"], w["d_ff"], w["r_svd"], w["r_lora"],
                                        w["sparsity"], bf16=True, workload=1, fast=True)
    full = _cache["full"]
    if batch is None:
        return full
    tok = synth.Tokens.uniform(batch, seq, w["out_frac"])
    return dataclasses.replace(full, tokens=tok, X=full.X[:tok.T], dOut=full.dOut[:tok.T])


def oracle_ffn_time(case, r, s=None, reps=1):
    from oracle import slora_oracle as O
    lay = dict(Wg=case.Wg.W, Wu=case.Wu.W, Wd=case.Wd.W, Ag=case.Ag, Bg=case.Bg, Au=case.Au,
               Bu=case.Bu, Ad=case.Ad, Bd=case.Bd, scale=case.lora_scale)
    for nm, sw in (("g", case.Wg), ("u", case.Wu)):
        lay["L" + nm] = sw.V[:, :r] * sw.s[None, :r]
        lay["U" + nm] = sw.U[:, :r].copy()
    tok = case.tokens
    t0 = time.perf_counter()
    for _ in range(reps):
        O.ffn_fwd_bwd(case.X, case.dOut, tok.batch, tok.seq, tok.ctx_len, lay,
                      case.sparsity if s is None else s)
    return (time.perf_counter() - t0) / reps


def cpu_baseline_ffn(reps=3):
    case = ffn_case_numpy(1, 512)
    oracle_ffn_time(case, 8)
    t = oracle_ffn_time(case, 8, reps=reps)
    return {"value": case.tokens.T / t, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
            "sample": "1 x 512 tokens of the same layer (ctx 384 + out 128), fp64 NumPy oracle, "
                      f"{reps} reps after 1 warm-up"}


def run_ffn(args, H, pk, rank, world):
    from contextual_sparsity_lora_svd_b200 import dp
    from contextual_sparsity_lora_svd_b200.layers import FfnLayer
    L = H.L
    wl = synth.WORKLOADS[1]
    d, F, r, rs = wl["d"], wl["d_ff"], wl["r_lora"], wl["r_svd"]
    case = ffn_case_numpy()
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(
        torch.bfloat16).cuda()
    Xn, dOn = case.X, case.dOut
    if world > 1:  # weak scaling: each rank its own batch, same weights
        T = Xn.shape[0]
        seed = 1000 + 1_000_003 * (rank + 1)
        Xn = synth.round_bf16(synth.gaussian((T, d), 1.0, seed))
        dOn = synth.round_bf16(synth.gaussian((T, d), 1.0, seed + 1))
    w = {k: bf(getattr(case, k)) for k in ("Ag", "Bg", "Au", "Bu", "Ad", "Bd")}
    w["Wg"], w["Wu"] = bf(case.Wg.W), bf(case.Wu.W)
    w["Wd_t"] = bf(case.Wd.W.T)
    w["Lg"], w["Ug"] = prepare_factors(L, w["Wg"], rs)
    w["Lu"], w["Uu"] = prepare_factors(L, w["Wu"], rs)
    tok = case.tokens
    sets = []
    layers = []
    for i in range(2):  # two buffer sets (the end-to-end pass double-buffers)
        X, dO = bf(Xn), bf(dOn)
        lay = FfnLayer(w, d, F, rs, r, case.lora_scale, tok.batch, tok.seq, tok.ctx_len,
                       wl["sparsity"], X, dO)
        layers.append(lay)
        sets.append({"X": X, "dOut": dO, "out": lay.out, "dX": lay.dX, "gflat": lay.gflat})
    ws = torch.empty(max(l.workspace_bytes() for l in layers), dtype=torch.uint8, device="cuda")
    graphs = [H.capture(lambda l=l: l.step(ws)) for l in layers]
    allreduce = (lambda i=0: dp.allreduce_grads(layers[i].gflat)) if world > 1 else None
    for _ in range(args.warmup):
        graphs[0].replay()
        if allreduce:
            allreduce()
    T = tok.T
    with ClockSampler(H.dev) as clk:
        ms = H.time_steps(graphs[0].replay, args.steps, allreduce)
    ms_prof, launches, prof = H.profile(lambda: layers[0].step(ws), args.steps, allreduce)
    ms = dp.max_over_ranks(ms, device="cuda")
    ms_step = ms / args.steps
    e2e_steps = max(2, min(args.steps, 10))
    e2e_ms, h2d, d2h = e2e_measure(H, graphs, sets, ("X", "dOut"), ("out", "dX", "gflat"),
                                   e2e_steps,
                                   (lambda i: dp.allreduce_grads(layers[i].gflat))
                                   if world > 1 else None)
    e2e_ms = dp.max_over_ranks(e2e_ms, device="cuda")
    mhz = clk.summary().get("sm_mhz") or clk.summary().get("sm_max_mhz") or 1965.0
    est = Estimator(L, L.CRIT_FFN, layers[0].X, tok.batch, tok.seq, tok.ctx_len, w["Lg"],
                    w["Ug"], w["Lu"], w["Uu"], rs, wl["sparsity"])
    est_m = measure_estimator(H, est, args.steps, pk, mhz)
    n_e, ms_e, _ = prof["estimate"]
    n_s, ms_s, _ = prof["select"]
    # the per-sequence variant: one channel set per sequence (same inputs)
    ps = FfnLayer(w, d, F, rs, r, case.lora_scale, tok.batch, tok.seq, tok.ctx_len,
                  wl["sparsity"], layers[0].X, layers[0].dOut, per_sequence=True)
    ws_ps = torch.empty(ps.workspace_bytes(), dtype=torch.uint8, device="cuda")
    ps.step(ws_ps)  # eager first: the library creates its lane streams outside the capture
    g_ps = H.capture(lambda: ps.step(ws_ps))
    g_ps.replay()
    n_ps = max(3, args.steps // 2)
    ms_ps = dp.max_over_ranks(H.time_steps(g_ps.replay, n_ps), device="cuda") / n_ps
    del g_ps, ps, ws_ps
    est_m["in_step_us"] = {"score_and_select": (ms_e + ms_s) * 1e3 / args.steps,
                           "note": "inside slora_ffn_fwd_bwd the projection X_C [Lg|Lu] rides "
                                   "the LoRA X A^T stream over X (class 'skinny')"}
    line = {"metric": METRIC, "value": world * T / (ms_step / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Llama-2-7B-shaped inputs, random-init decaying-spectrum "
                    "weights)",
            "config": workload_config(wl["name"], world),
            "roofline": gemm_roofline(prof, pk, workload=wl["name"]),
            "estimator": est_m,
            "per_sequence_sets": {"ms_per_step": ms_ps, "tokens_per_s": world * T / (ms_ps / 1e3),
                                  "vs_per_batch_set": ms_step / ms_ps,
                                  "call": "slora_ffn_fwd_bwd_per_seq (one channel set per "
                                          "sequence; same inputs)"},
            "kernels": kernel_table(prof, args.steps, ms_prof), "gpu_launches": int(launches),
            "clocks": clk.summary(),
            "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "overlap": "double-buffered: H2D, compute and D2H on separate streams"},
            "profiled_ms_per_step": ms_prof / args.steps, "impl": "ours"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        set_threads()
        line["cpu_baseline"] = cpu_baseline_ffn()
    return line


# ============================================================= attention
_ATTN_INPUTS = {}


def oracle_attn_inputs(batch, seq, d, H, KV, hd, r_svd, r_lora):
    """Random inputs of the attention linears' oracle timing (weights of the
    workload's shapes; their values do not change the oracle's cost)."""
    key = (batch, seq, d, H, KV, hd, r_svd, r_lora)
    if key not in _ATTN_INPUTS:
        tok = synth.Tokens.uniform(batch, seq, 0.25)
        rg = synth.rng(4242)
        nq, nkv = H * hd, KV * hd
        W = {"q": rg.standard_normal((nq, d)) * 0.02, "k": rg.standard_normal((nkv, d)) * 0.02,
             "v": rg.standard_normal((nkv, d)) * 0.02, "o": rg.standard_normal((d, nq)) * 0.02}
        _ATTN_INPUTS[key] = dict(
            tok=tok, X=rg.standard_normal((tok.T, d)), Xo=rg.standard_normal((tok.T, nq)), W=W,
            A={m: rg.standard_normal((r_lora, W[m].shape[1])) * 0.02 for m in W},
            B={m: rg.standard_normal((W[m].shape[0], r_lora)) * 0.02 for m in W},
            fac={m: (rg.standard_normal((d, r_svd)), rg.standard_normal((W[m].shape[0], r_svd)))
                 for m in ("q", "k", "v")})
    return _ATTN_INPUTS[key]


def oracle_attn_time(batch, seq, d, H, KV, hd, r_svd, r_lora, s_qk, reps=1, vo=0.0, pairs=False):
    """Seconds for the oracle's q/k estimate + select and the four linears'
    forward and backward on `batch` x `seq` tokens."""
    from oracle import slora_oracle as O
    I = oracle_attn_inputs(batch, seq, d, H, KV, hd, r_svd, r_lora)
    tok, X, W, A, B, fac = I["tok"], I["X"], I["W"], I["A"], I["B"], I["fac"]
    C, Orow = O.context_rows(tok.batch, tok.seq, tok.ctx_len)
    t0 = time.perf_counter()
    for _ in range(reps):
        if s_qk > 0:
            est = O.estimate_select_qk_pairs if pairs else O.estimate_select_qk
            iq, ik, _, _ = est(X, tok.batch, tok.seq, tok.ctx_len, *fac["q"], *fac["k"], H, KV,
                               hd, s_qk)
            sides = {"q": ("out_rows", iq), "k": ("out_rows", ik)}
        else:
            sides = {"q": ("none", None), "k": ("none", None)}
        if vo > 0:
            io, iv, _, _ = O.estimate_select_l2(X, tok.batch, tok.seq, tok.ctx_len, *fac["v"], H,
                                                KV, hd, vo)
            sides["v"] = ("out_rows", iv)
            sides["o"] = ("in_cols", io)
        else:
            sides["v"] = ("none", None)
            sides["o"] = ("none", None)
        for m in ("q", "k", "v", "o"):
            side, idx = sides[m]
            Xin = X if m != "o" else I["Xo"]
            Xout = None
            if side == "in_cols":
                Xin, Xout = Xin[C][:, idx], Xin[Orow]
            Yc, Yo, XA = O.linear_fwd(side, Xin, Xout, tok.batch, tok.seq, tok.ctx_len, W[m], A[m],
                                      B[m], 1.0, idx)
            O.linear_bwd(side, Xin, Xout, XA, np.ones_like(Yc),
                         np.ones_like(Yo) if Yo is not None else None, tok.batch, tok.seq,
                         tok.ctx_len, W[m], A[m], B[m], 1.0, idx)
    return (time.perf_counter() - t0) / reps


def cpu_baseline_attn(d=4096, H=32, KV=32, hd=128, s=0.5, reps=2):
    oracle_attn_time(1, 1024, d, H, KV, hd, 8, 16, s)
    t = oracle_attn_time(1, 1024, d, H, KV, hd, 8, 16, s, reps=reps)
    return {"value": 1024 / t, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
            "sample": f"1 x 1024 tokens (ctx 768 + out 256) of the same layer shapes, q/k "
                      f"estimate+select and q/k/v/o fwd+bwd, fp64 NumPy oracle, {reps} reps "
                      "after 1 warm-up"}


def build_attn(L, w, fac, d, H, KV, hd, r_svd, r_lora, batch, seq, s_qk, seed, pairs=False,
               vo=0.0):
    from contextual_sparsity_lora_svd_b200.layers import AttnLinears
    T = batch * seq
    ctx = [seq - int(round(0.25 * seq))] * batch
    X = randn_bf16((T, d), seed)
    attn_out = randn_bf16((T, H * hd), seed + 1)
    dY_o = randn_bf16((T, d), seed + 2)
    dq = randn_bf16((T, H * hd), seed + 3)
    dk = randn_bf16((T, KV * hd), seed + 4)
    dv = randn_bf16((T, KV * hd), seed + 5)
    ww = dict(w)
    ww.update(fac[r_svd])
    return AttnLinears(ww, d, H, KV, hd, r_svd, r_lora, 1.0, batch, seq, ctx, s_qk, X, attn_out,
                       dY_o, dq, dk, dv, pairs=pairs, vo_sparsity=vo)


def time_runner(H, runners, steps, warmup, ws=None):
    """Graph-replay ms per step of running `runners` in order."""
    if ws is None:
        ws = torch.empty(max(r.workspace_bytes() for r in runners), dtype=torch.uint8,
                         device="cuda")

    def step():
        for r in runners:
            r.step(ws)
    g = H.capture(step)
    for _ in range(warmup):
        g.replay()
    ms = H.time_steps(g.replay, steps) / steps
    return ms, g, step, ws


def run_attn(args, H, pk, rank, world):
    from contextual_sparsity_lora_svd_b200 import dp
    L = H.L
    wl = synth.WORKLOADS[2]
    d, Hh, KV, hd, rs, r = wl["d"], wl["heads"], wl["kv_heads"], wl["head_dim"], wl["r_svd"], \
        wl["r_lora"]
    batch, seq, s = wl["batch"], wl["seq"], wl["sparsity"]
    wf = WeightFactory()
    w, fac = attn_weights_gpu(L, wf, d, Hh, KV, hd, (rs,), r, 2000, vo=True)
    base = build_attn(L, w, fac, d, Hh, KV, hd, rs, r, batch, seq, s, 2100 + 97 * rank)
    T = batch * seq
    grads_flat = base.gflat
    allreduce = (lambda: dp.allreduce_grads(grads_flat)) if world > 1 else None
    ws = torch.empty(base.workspace_bytes(), dtype=torch.uint8, device="cuda")
    g = H.capture(lambda: base.step(ws))
    for _ in range(args.warmup):
        g.replay()
        if allreduce:
            allreduce()
    with ClockSampler(H.dev) as clk:
        ms = H.time_steps(g.replay, args.steps, allreduce)
    # per-launch event timings with the parallel branches issued one after
    # another, so that no launch's time includes another branch's work
    base.serial = True
    ms_prof, launches, prof = H.profile(lambda: base.step(ws), args.steps, allreduce)
    base.serial = False
    ms = dp.max_over_ranks(ms, device="cuda")
    ms_step = ms / args.steps
    mhz = clk.summary().get("sm_mhz") or 1965.0
    # end to end: X, the attention-output stand-in and the upstream gradients
    # go up, the four linears' outputs and the LoRA gradients come back; a
    # second runner (same weights, its own buffers and inputs) double-buffers
    base2 = build_attn(L, w, fac, d, Hh, KV, hd, rs, r, batch, seq, s, 2150 + 97 * rank)
    g2 = H.capture(lambda: base2.step(ws))
    sets = [{"X": b.X, "attn_out": b.attn_out, "dY_o": b.dY_o, "Yq": b.bufs["q"][0],
             "Yk": b.bufs["k"][0], "Yo": b.bufs["o"][0], "dXq": b.dX["q"], "grads": b.gflat}
            for b in (base, base2)]
    e2e_ms, h2d, d2h = e2e_measure(H, [g, g2], sets, ("X", "attn_out", "dY_o"),
                                   ("Yq", "Yk", "Yo", "dXq", "grads"), max(2, min(args.steps, 10)),
                                   (lambda i: dp.allreduce_grads(sets[i]["grads"]))
                                   if world > 1 else None)
    # the q/k estimator alone, by algorithmic bytes
    est = Estimator(L, L.CRIT_QK, base.X, batch, seq, [768] * batch, fac[rs]["Lq"],
                    fac[rs]["Uq"], fac[rs]["Lk"], fac[rs]["Uk"], rs, s, heads=Hh, kv=KV, hd=hd)
    est_m = measure_estimator(H, est, args.steps, pk, mhz)
    variants = {}
    for name, kw, crit in (("qk_rope_pairs", dict(pairs=True), L.CRIT_QK_ROPE_PAIR),
                           ("vo_sliced_l2", dict(vo=s), L.CRIT_L2)):
        v = build_attn(L, w, fac, d, Hh, KV, hd, rs, r, batch, seq, s, 2100, **kw)
        vms, vg, _, _ = time_runner(H, [v], args.steps, args.warmup)
        del vg
        if crit == L.CRIT_L2:
            e = Estimator(L, crit, base.X, batch, seq, [768] * batch, fac[rs]["Lv"],
                          fac[rs]["Uv"], fac[rs]["Lv"], fac[rs]["Uv"], rs, s, heads=Hh, kv=KV,
                          hd=hd)
        else:
            e = Estimator(L, crit, base.X, batch, seq, [768] * batch, fac[rs]["Lq"],
                          fac[rs]["Uq"], fac[rs]["Lk"], fac[rs]["Uk"], rs, s, heads=Hh, kv=KV,
                          hd=hd)
        em = measure_estimator(H, e, args.steps, pk, mhz)
        variants[name] = {"ms_per_step": vms, "tokens_per_s": world * T / (vms / 1e3),
                          "estimator_us": em["us_per_call"], "estimator_frac_hbm": em["frac_hbm"]}
        del v, e
    dense = build_attn(L, w, fac, d, Hh, KV, hd, rs, r, batch, seq, 0.0, 2100)
    dms, dg, _, _ = time_runner(H, [dense], args.steps, args.warmup)
    del dg, dense
    variants["dense_lora"] = {"ms_per_step": dms, "tokens_per_s": world * T / (dms / 1e3)}
    line = {"metric": METRIC, "value": world * T / (ms_step / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded inputs, random-init decaying-spectrum weights built on "
                    "the GPU)",
            "config": workload_config(wl["name"], world),
            "roofline": gemm_roofline(prof, pk),
            "estimator": est_m, "variants": variants,
            "kernels": kernel_table(prof, args.steps, ms_prof), "gpu_launches": int(launches),
            "clocks": clk.summary(),
            "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "profiled_ms_per_step": ms_prof / args.steps, "impl": "ours"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        set_threads()
        line["cpu_baseline"] = cpu_baseline_attn()
    return line


# ================================================================= stack
def run_stack(args, H, pk, rank, world):
    from contextual_sparsity_lora_svd_b200 import dp
    from contextual_sparsity_lora_svd_b200.layers import FfnLayer
    from contextual_sparsity_lora_svd_b200.schedule import ProgressiveSchedule, llama2_7b_stack
    L = H.L
    wl = synth.WORKLOADS[3]
    d, F, Hh, KV, hd = wl["d"], wl["d_ff"], wl["heads"], wl["kv_heads"], wl["head_dim"]
    rs, r, batch, seq, nl = wl["r_svd"], wl["r_lora"], wl["batch"], wl["seq"], wl["layers"]
    T = batch * seq
    ctx = [seq - int(round(0.25 * seq))] * batch
    table = llama2_7b_stack()
    wf = WeightFactory()
    X = randn_bf16((T, d), 3000 + 97 * rank)
    dOut = randn_bf16((T, d), 3001 + 97 * rank)
    t_setup = time.perf_counter()
    layer_w = []
    for l in range(nl):
        fw, ffac = ffn_weights_gpu(L, wf, d, F, (rs,), r, 3100 + 10 * l)
        fw["Lg"], fw["Ug"], fw["Lu"], fw["Uu"] = ffac[rs]
        aw, afac = attn_weights_gpu(L, wf, d, Hh, KV, hd, (rs,), r, 3100 + 10 * l)
        layer_w.append((fw, aw, afac))
    torch.cuda.synchronize()
    t_setup = time.perf_counter() - t_setup

    def runners(sparse):
        out = []
        for l, (fw, aw, afac) in enumerate(layer_w):
            sf, sq = (table.ffn[l], table.qk[l]) if sparse else (0.0, 0.0)
            out.append(build_attn(L, aw, afac, d, Hh, KV, hd, rs, r, batch, seq, sq, 3500 + l))
            out.append(FfnLayer(fw, d, F, rs, r, 1.0, batch, seq, ctx, sf, X, dOut))
        return out

    sparse_r = runners(True)
    ws = torch.empty(max(x.workspace_bytes() for x in sparse_r), dtype=torch.uint8,
                     device="cuda")
    flats = [x.gflat for x in sparse_r if hasattr(x, "gflat")]
    allreduce = (lambda: [dp.allreduce_grads(f) for f in flats]) if world > 1 else None

    def sparse_step():
        for x in sparse_r:
            x.step(ws)
    g = H.capture(sparse_step)
    for _ in range(args.warmup):
        g.replay()
        if allreduce:
            allreduce()
    with ClockSampler(H.dev) as clk:
        ms = H.time_steps(g.replay, args.steps, allreduce)
    for x in sparse_r:  # per-launch timings with the parallel branches one after another
        x.serial = True
    ms_prof, launches, prof = H.profile(sparse_step, args.steps, allreduce)
    for x in sparse_r:
        x.serial = False
    ms = dp.max_over_ranks(ms, device="cuda")
    ms_sparse = ms / args.steps
    e2e_steps = max(2, min(args.steps, 5))
    # end to end: the batch's input and output gradient go up, every layer's
    # LoRA gradients come back
    sets = [{"X": X, "dOut": dOut, "grads": torch.cat(
        [f for f in flats] + [torch.cat([gg.view(-1) for gg in x.grads.values()])
                              for x in sparse_r if not hasattr(x, "gflat")])}] * 2
    grads_cat = sets[0]["grads"]

    def gather_grads(_i):
        torch.cat([f for f in flats] + [torch.cat([gg.view(-1) for gg in x.grads.values()])
                                        for x in sparse_r if not hasattr(x, "gflat")],
                  out=grads_cat)
    e2e_ms, h2d, d2h = e2e_measure(H, [g, g], sets, ("X", "dOut"), ("grads",), e2e_steps,
                                   gather_grads)
    del g
    # the dense phase of the progressive schedule: every layer dense
    dense_r = runners(False)
    ms_dense, gd, _, _ = time_runner(H, dense_r, max(2, args.steps // 2), 1, ws)
    del gd, dense_r
    sch = ProgressiveSchedule(table, total_steps=1000)
    run_ms = sum(n * (ms_dense if f == 0.0 else ms_sparse) for _, n, f in sch.phases())
    line = {"metric": METRIC, "value": world * T / (ms_sparse / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_sparse, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded inputs, random-init decaying-spectrum weights built on "
                    "the GPU, distinct per layer)",
            "config": workload_config(wl["name"], world),
            "roofline": gemm_roofline(prof, pk),
            "progressive": {"dense_phase_ms_per_step": ms_dense,
                            "sparse_phase_ms_per_step": ms_sparse,
                            "run_steps": 1000, "dense_steps": sch.dense_steps,
                            "run_tokens_per_s": world * T * 1000 / (run_ms / 1e3),
                            "speedup_sparse_vs_dense": ms_dense / ms_sparse},
            "kernels": kernel_table(prof, args.steps, ms_prof), "gpu_launches": int(launches),
            "clocks": clk.summary(), "setup_s": t_setup,
            "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "profiled_ms_per_step": ms_prof / args.steps, "impl": "ours"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        set_threads()
        # one sparse layer (layer 17: FFN 0.7, q/k 0.45) of attention linears +
        # FFN on 1 x 1024 tokens, scaled by 32 layers
        fcase = synth.ffn_case(synth.Tokens.uniform(1, 1024, 0.25), d, F, rs, r, table.ffn[17],
                               bf16=True, workload=3, layer=17, fast=True)
        t_f = oracle_ffn_time(fcase, rs)
        t_a = oracle_attn_time(1, 1024, d, Hh, KV, hd, rs, r, table.qk[17])
        line["cpu_baseline"] = {"value": 1024 / (nl * (t_f + t_a)), "unit": UNIT,
                                "cores": host_cores(), "kind": "oracle",
                                "sample": "one layer (layer 17 ratios) of attention linears + FFN "
                                          "on 1 x 1024 tokens, fp64 NumPy oracle, time x 32 "
                                          "layers"}
    return line


# ============================================================ decoder stack
def decoder_weights(L, wf, d, F, Hh, KV, hd, rs, r, seed):
    """One decoder layer's device tensors: attention and FFN weights with their
    LoRA pairs and estimator factors, and the two RMS gains."""
    fw, ffac = ffn_weights_gpu(L, wf, d, F, (rs,), r, seed)
    fw["Lg"], fw["Ug"], fw["Lu"], fw["Uu"] = ffac[rs]
    aw, afac = attn_weights_gpu(L, wf, d, Hh, KV, hd, (rs,), r, seed)
    w = dict(fw)
    w.update(aw)
    w.update(afac[rs])
    g = torch.Generator(device="cuda").manual_seed(int(seed) + 40)
    for k in ("g1", "g2"):
        w[k] = (1.0 + 0.1 * torch.randn(d, device="cuda", generator=g)).to(torch.bfloat16)
    return w


def oracle_decoder_layer(d, F, Hh, KV, hd, rs, r, _cache={}):
    """Random-weight float64 layer of the given shapes for the oracle timing
    (the timing does not depend on the spectrum)."""
    key = (d, F, Hh, KV, hd, rs, r)
    if key not in _cache:
        rng = np.random.default_rng(11)
        lay = {"scale": 1.0}
        for nm, n, k in (("q", Hh * hd, d), ("k", KV * hd, d), ("v", KV * hd, d),
                         ("o", d, Hh * hd), ("g", F, d), ("u", F, d), ("d", d, F)):
            lay["W" + nm] = rng.standard_normal((n, k)) / np.sqrt(k)
            lay["A" + nm] = rng.standard_normal((r, k)) * 0.02
            lay["B" + nm] = rng.standard_normal((n, r)) * 0.02
            if nm in ("q", "k", "g", "u"):
                lay["L" + nm] = rng.standard_normal((k, rs)) / np.sqrt(k)
                lay["U" + nm] = rng.standard_normal((n, rs)) / np.sqrt(rs)
        lay["g1"] = 1.0 + 0.1 * rng.standard_normal(d)
        lay["g2"] = 1.0 + 0.1 * rng.standard_normal(d)
        _cache.clear()
        _cache[key] = lay
    return _cache[key]


def oracle_decoder_time(seq, d, F, Hh, KV, hd, rs, r, s_qk, s_ffn):
    """Seconds of the oracle's step (forward with its own selections, then
    backward) for one decoder layer on 1 x seq tokens."""
    from oracle import stack_oracle as S
    lay = oracle_decoder_layer(d, F, Hh, KV, hd, rs, r)
    rng = np.random.default_rng(12)
    x, dy = rng.standard_normal((seq, d)), rng.standard_normal((seq, d))
    ctx = [seq - int(round(0.25 * seq))]
    t0 = time.perf_counter()
    S.stack_fwd_bwd(x, dy, [lay], 1, seq, ctx, Hh, KV, hd, qk_sparsity=[s_qk],
                    ffn_sparsity=[s_ffn])
    return time.perf_counter() - t0


def run_decoder(args, H, pk, rank, world):
    """The 32-layer decoder stack's whole training step (layers.DecoderStack):
    sparse q/k feeding the attention core, v/o, residuals, RMS norms and the
    sparse FFN, forward through all layers then backward, with the per-layer
    ratio table; and the same stack dense (every layer at ratio 0)."""
    from contextual_sparsity_lora_svd_b200 import dp
    from contextual_sparsity_lora_svd_b200.layers import DecoderStack
    from contextual_sparsity_lora_svd_b200.schedule import ProgressiveSchedule, llama2_7b_stack
    L = H.L
    wl = synth.WORKLOADS[3]
    d, F, Hh, KV, hd = wl["d"], wl["d_ff"], wl["heads"], wl["kv_heads"], wl["head_dim"]
    rs, r, batch, seq, nl = wl["r_svd"], wl["r_lora"], wl["batch"], wl["seq"], wl["layers"]
    T = batch * seq
    ctx = [seq - int(round(0.25 * seq))] * batch
    table = llama2_7b_stack()
    wf = WeightFactory()
    X = randn_bf16((T, d), 3000 + 97 * rank)
    dY = randn_bf16((T, d), 3001 + 97 * rank)
    t_setup = time.perf_counter()
    layers = [decoder_weights(L, wf, d, F, Hh, KV, hd, rs, r, 3100 + 10 * l) for l in range(nl)]
    torch.cuda.synchronize()
    t_setup = time.perf_counter() - t_setup
    sparse = DecoderStack(layers, d, Hh, KV, hd, F, rs, r, 1.0, batch, seq, ctx, list(table.qk),
                          list(table.ffn), X, dY)
    ws = torch.empty(sparse.workspace_bytes(), dtype=torch.uint8, device="cuda")
    allreduce = (lambda: dp.allreduce_grads(sparse.gflat)) if world > 1 else None
    g = H.capture(lambda: sparse.step(ws))
    for _ in range(args.warmup):
        g.replay()
        if allreduce:
            allreduce()
    with ClockSampler(H.dev) as clk:
        ms = H.time_steps(g.replay, args.steps, allreduce)
    # per-launch event timings with the parallel branches issued one after
    # another, so that no launch's time includes another branch's work
    sparse.serial = True
    ms_prof, launches, prof = H.profile(lambda: sparse.step(ws), args.steps, allreduce)
    sparse.serial = False
    ms = dp.max_over_ranks(ms, device="cuda")
    ms_sparse = ms / args.steps
    e2e_steps = max(2, min(args.steps, 5))
    sets = [{"X": X, "dY": dY, "grads": sparse.gflat}] * 2
    e2e_ms, h2d, d2h = e2e_measure(H, [g, g], sets, ("X", "dY"), ("grads",), e2e_steps)
    del g
    del sparse
    torch.cuda.empty_cache()
    # the same stack with every layer dense (the first phase of the schedule)
    dense = DecoderStack(layers, d, Hh, KV, hd, F, rs, r, 1.0, batch, seq, ctx, [0.0] * nl,
                         [0.0] * nl, X, dY)
    wsd = torch.empty(dense.workspace_bytes(), dtype=torch.uint8, device="cuda")
    gd = H.capture(lambda: dense.step(wsd))
    gd.replay()
    nd = max(2, args.steps // 2)
    ms_dense = dp.max_over_ranks(H.time_steps(gd.replay, nd), device="cuda") / nd
    del gd, dense, wsd
    sch = ProgressiveSchedule(table, total_steps=1000)
    run_ms = sum(n * (ms_dense if f == 0.0 else ms_sparse) for _, n, f in sch.phases())
    n_a, ms_a, fl_a = prof["attention"]
    att = fl_a / (ms_a / 1e3) / 1e12 if ms_a > 0 else 0.0
    line = {"metric": METRIC, "value": world * T / (ms_sparse / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_sparse, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded inputs, random-init decaying-spectrum weights built on "
                    "the GPU, distinct per layer)",
            "config": workload_config("llama2-7b-decoder32-bf16", world),
            "roofline": gemm_roofline(prof, pk),
            "attention_core": {"kernels": "attn_fwd_tc_kernel / attn_bwd_dkv_tc_kernel + "
                                          "attn_bwd_dq_tc_kernel (tcgen05, tensor-memory "
                                          "accumulators)",
                               "work": "algorithmic: 2 causal products forward, 5 backward "
                                       "(the dQ kernel's recomputed S and dP not counted)",
                               "achieved": att, "unit": "TFLOP/s",
                               "peak": pk["bf16"], "frac": att / pk["bf16"],
                               "ms_per_step": ms_a / args.steps,
                               "flops_per_step": fl_a / args.steps},
            "dense_vs_sparse": {"dense_ms_per_step": ms_dense, "sparse_ms_per_step": ms_sparse,
                                "speedup": ms_dense / ms_sparse,
                                "run_steps": 1000, "dense_steps": sch.dense_steps,
                                "run_tokens_per_s": world * T * 1000 / (run_ms / 1e3)},
            "kernels": kernel_table(prof, args.steps, ms_prof), "gpu_launches": int(launches),
            "clocks": clk.summary(), "setup_s": t_setup,
            "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "profiled_ms_per_step": ms_prof / args.steps, "impl": "ours"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        set_threads()
        t = oracle_decoder_time(1024, d, F, Hh, KV, hd, rs, r, table.qk[17], table.ffn[17])
        line["cpu_baseline"] = {"value": 1024 / (nl * t), "unit": UNIT, "cores": host_cores(),
                                "kind": "oracle",
                                "sample": "one decoder layer (layer 17 ratios) on 1 x 1024 "
                                          "tokens, random weights of its shapes, fp64 NumPy "
                                          "oracle, time x 32 layers"}
    return line


# ========================================================== llama3 sweep
def run_llama3(args, H, pk, rank, world):
    from contextual_sparsity_lora_svd_b200.layers import FfnLayer
    L = H.L
    wl = synth.WORKLOADS[4]
    d, F, Hh, KV, hd, r = wl["d"], wl["d_ff"], wl["heads"], wl["kv_heads"], wl["head_dim"], \
        wl["r_lora"]
    Ttot = wl["tokens"]
    wf = WeightFactory()
    fw, ffac = ffn_weights_gpu(L, wf, d, F, wl["r_svds"], r, 4000)
    aw, afac = attn_weights_gpu(L, wf, d, Hh, KV, hd, wl["r_svds"], r, 4000)
    X = randn_bf16((Ttot, d), 4100 + 97 * rank)
    dOut = randn_bf16((Ttot, d), 4101 + 97 * rank)
    points = [(s, rs, 1024) for s in wl["sparsities"] for rs in wl["r_svds"]]
    points += [(0.5, 8, q) for q in wl["seqs"] if q != 1024]
    steps = max(3, min(args.steps, 8))
    table = []
    center = None
    ws = None
    for s, rs, seq in points:
        batch = Ttot // seq
        ctx = [seq - int(round(0.25 * seq))] * batch
        w = dict(fw)
        w["Lg"], w["Ug"], w["Lu"], w["Uu"] = ffac[rs]
        attn = build_attn(L, aw, afac, d, Hh, KV, hd, rs, r, batch, seq, s, 4200)
        ffn = FfnLayer(w, d, F, rs, r, 1.0, batch, seq, ctx, s, X, dOut)
        need = max(attn.workspace_bytes(), ffn.workspace_bytes())
        if ws is None or ws.numel() < need:
            ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        ms, g, step, _ = time_runner(H, [attn, ffn], steps, 2, ws)
        row = {"sparsity": s, "r_svd": rs, "seq": seq, "batch": batch, "ms_per_step": ms,
               "tokens_per_s": world * Ttot / (ms / 1e3)}
        if (s, rs, seq) == (0.5, 8, 1024):
            with ClockSampler(H.dev) as clk:
                ms_c = H.time_steps(g.replay, args.steps) / args.steps
            attn.serial = True  # per-launch timings with the parallel branches one after another
            ms_prof, launches, prof = H.profile(step, args.steps)
            attn.serial = False
            est = Estimator(L, L.CRIT_QK, X, batch, seq, ctx, afac[rs]["Lq"], afac[rs]["Uq"],
                            afac[rs]["Lk"], afac[rs]["Uk"], rs, s, heads=Hh, kv=KV, hd=hd)
            center = dict(ms=ms_c, prof=prof, launches=launches, ms_prof=ms_prof,
                          clk=clk.summary(),
                          est=measure_estimator(H, est, args.steps, pk,
                                                clk.summary().get("sm_mhz") or 1965.0))
            sets = [{"X": X, "dOut": dOut, "out": ffn.out, "dX": ffn.dX, "g": ffn.gflat}] * 2
            center["e2e"] = e2e_measure(H, [g, g], sets, ("X", "dOut"), ("out", "dX", "g"), 4)
        else:
            attn.serial = True
            _, _, prof_pt = H.profile(step, 2)
            attn.serial = False
            n_g, ms_g, fl_g = prof_pt["gemm_tc"]
            row["gemm_tflops"] = fl_g / (ms_g / 1e3) / 1e12 if ms_g > 0 else None
        table.append(row)
        del g, attn, ffn
        torch.cuda.empty_cache()
    c = center
    e2e_ms, h2d, d2h = c["e2e"]
    line = {"metric": METRIC, "value": world * Ttot / (c["ms"] / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": c["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded inputs, random-init decaying-spectrum weights built on "
                    "the GPU)",
            "config": workload_config(wl["name"], world),
            "roofline": gemm_roofline(c["prof"], pk), "estimator_qk": c["est"],
            "sweep": table, "kernels": kernel_table(c["prof"], args.steps, c["ms_prof"]),
            "gpu_launches": int(c["launches"]), "clocks": c["clk"],
            "e2e": {"value": world * Ttot / (e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "impl": "ours"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        set_threads()
        fcase = synth.ffn_case(synth.Tokens.uniform(1, 1024, 0.25), d, F, 8, r, 0.5, bf16=True,
                               workload=4, fast=True)
        t_f = oracle_ffn_time(fcase, 8)
        t_a = oracle_attn_time(1, 1024, d, Hh, KV, hd, 8, r, 0.5)
        line["cpu_baseline"] = {"value": 1024 / (t_f + t_a), "unit": UNIT, "cores": host_cores(),
                                "kind": "oracle",
                                "sample": "1 x 1024 tokens of the headline point (s 0.5, rank 8) "
                                          "attention linears + FFN, fp64 NumPy oracle"}
    return line


RUNNERS = {"llama2-7b-ffn-bf16": run_ffn, "llama2-7b-attn-qk-bf16": run_attn,
           "llama2-7b-stack32-bf16": run_stack, "llama3-8b-layer-bf16": run_llama3,
           "llama2-7b-decoder32-bf16": run_decoder}


# ------------------------------------------------------------- reference
def run_reference(args, rank, world):
    """The oracle (the plain CPU implementation) on a bounded sample of the
    workload, per step, on this host's cores; rank 0 only."""
    if rank != 0:
        return
    set_threads()
    name = args.workload
    if name == "llama2-7b-ffn-bf16":
        case = ffn_case_numpy(1, 512)
        fn, T = (lambda: oracle_ffn_time(case, 8)), case.tokens.T
        sample = "1 x 512 tokens (ctx 384 + out 128) of the layer"
    elif name == "llama2-7b-attn-qk-bf16":
        fn, T = (lambda: oracle_attn_time(1, 1024, 4096, 32, 32, 128, 8, 16, 0.5)), 1024
        sample = "1 x 1024 tokens (ctx 768 + out 256) of the layer's q/k/v/o linears"
    elif name == "llama2-7b-decoder32-bf16":
        from contextual_sparsity_lora_svd_b200.schedule import llama2_7b_stack
        t = llama2_7b_stack()

        def fn():
            return 32 * oracle_decoder_time(1024, 4096, 11008, 32, 32, 128, 8, 16, t.qk[17],
                                            t.ffn[17])
        T = 1024
        sample = "1 x 1024 tokens of one decoder layer (layer 17 ratios), x 32 layers"
    else:
        wl = synth.WORKLOADS[3 if name == "llama2-7b-stack32-bf16" else 4]
        F, KV = wl["d_ff"], wl["kv_heads"]
        layers = 32 if name == "llama2-7b-stack32-bf16" else 1
        fcase = synth.ffn_case(synth.Tokens.uniform(1, 1024, 0.25), 4096, F, 8, 16, 0.5,
                               bf16=True, workload=4, fast=True)

        def fn():
            return layers * (oracle_ffn_time(fcase, 8) +
                             oracle_attn_time(1, 1024, 4096, 32, KV, 128, 8, 16, 0.5))
        T = 1024
        sample = f"1 x 1024 tokens of one layer (attention linears + FFN), x {layers} layers"
    for _ in range(args.warmup):
        fn()
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        r = fn()
        ts.append(r if name in ("llama2-7b-stack32-bf16", "llama3-8b-layer-bf16",
                                "llama2-7b-decoder32-bf16")
                  else time.perf_counter() - t0)
    v = T / float(np.mean(ts))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(ts)),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(name, world),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                             "sample": f"each step: {sample}, fp64 NumPy oracle"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world):
    from contextual_sparsity_lora_svd_b200 import _lib as L
    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    H = Harness(L, dev, world, args.profile_region)
    line = RUNNERS[args.workload](args, H, peaks(), rank, world)
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
    ap.add_argument("--workload", choices=WORKLOAD_NAMES, default=WORKLOAD_NAMES[0])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-region", action="store_true",
                    help="bracket the first timed steps with cudaProfilerStart/Stop (for ncu "
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
