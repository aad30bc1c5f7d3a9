#!/usr/bin/env python
"""Benchmark of the WSVD low-rank decode step on B200.

A step is one pass of the hot path over one batch: the latent append of the
new token (block-Hadamard rotation, projection through A_Kh / A_Vh, int8/int4
quantisation into the cache) followed by the decode-step attention over the
per-head low-rank cache (split-L kernel + combine).  Workloads without an
append (ragged int4, comparison shapes) time the decode alone.

Prints ONE JSON line (rank 0).  `value` is tokens*heads/s over the whole job
(sum over sequences of the attended length times heads, divided by the device
time of the timed steps, max over ranks).  Inputs are resident in HBM before
the timed region; L2 is flushed (a 256 MiB write) between timed steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl wsvd|reference]

Under torchrun (N > 1) every rank runs an independent replica of the workload
(the decode has no exchange step); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as WL  # noqa: E402

METRIC = "low-rank decode-attention step µs, tokens·heads/s, HBM GB/s vs ~8 TB/s peak"
UNIT = "tokens*heads/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
HOST_LEAD_CYCLES = 100_000  # device sleep (~50-75 us) before each timed step


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def source_digest(files):
    """Digest of the kernel sources with comments and blank space removed, so
    that an edit of comments alone does not retire a capture (the sources
    hold no string literal with a comment marker)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "rank_kv_cache_wsvd_b200", "csrc", f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {"append": ["append.cu", "append_core.cuh", "common.cuh", "wsvd_internal.h", "api.cu"],
                  "step": ["decode.cu", "append_core.cuh", "common.cuh", "wsvd_internal.h", "api.cu"],
                  "decode": ["decode.cu", "shared.cu", "common.cuh", "wsvd_internal.h", "api.cu"],
                  "prefill_gemm": ["prefill.cu", "common.cuh", "wsvd_internal.h", "tc05.cuh"],
                  "grouped": ["grouped.cu", "common.cuh", "wsvd_internal.h", "tc05.cuh"]}


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_digest") != source_digest(KERNEL_SOURCES[kernel]):
        return None
    return float(e["dram_bytes_per_launch"])


class ClockSampler:
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [ln.split(", ") for ln in out.strip().splitlines() if ln.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def replica_throughput(units_local: float, seconds_local: float, world: int, device="cuda"):
    """Whole-job throughput of N independent replicas: every rank processed
    `units_local` units; the job's duration is the slowest rank's (max over
    ranks).  Returns (units per second over all ranks, max seconds)."""
    if world == 1:
        return units_local / seconds_local, seconds_local
    import torch
    import torch.distributed as dist
    t = torch.tensor([seconds_local], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    t_max = float(t.item())
    return units_local * world / t_max, t_max


# ----------------------------------------------------------------------------- workloads
def attended_tokens(w: WL.Workload, lens_after: np.ndarray) -> int:
    return int(lens_after.sum()) * w.H


def alg_bytes_decode(w: WL.Workload, lens: np.ndarray, w8: bool = False) -> int:
    rb = w.r * w.bits // 8
    codes = int(lens.sum()) * w.H * 2 * (rb + 2)
    weights = 2 * w.H * (w.r * w.Hd + w.Hd * 4) if w8 else 2 * w.H * w.r * w.Hd * 2  # B_K, B_V (+ column scales)
    io = w.B * w.H * w.Hd * (2 + 4)
    return codes + weights + io


def alg_bytes_append(w: WL.Workload, w8: bool = False) -> int:
    rb = w.r * w.bits // 8
    weights = 2 * w.H * (w.E * w.r + w.r * 4) if w8 else 2 * w.H * w.E * w.r * 2  # A_K, A_V (+ column scales)
    return weights + w.B * w.E * 2 + w.B * w.H * 2 * (rb + 2) + w.B * 4 * 2


class WsvdStep:
    """Device-resident inputs of one workload and the launches of one step."""

    def __init__(self, w: WL.Workload, seed: int = 0, w8: bool = False):
        import torch

        import rank_kv_cache_wsvd_b200 as W
        self.W, self.torch, self.w, self.w8 = W, torch, w, w8
        self.has_append = w.append_steps > 0
        lens_full = WL.seq_lens(w, seed)
        lens0 = lens_full - 1 if self.has_append else lens_full
        d = WL.decode_inputs(w, seed=seed, lens=lens_full)
        if self.has_append:  # the new token's row is produced by the append inside each step
            for b in range(w.B):
                n = int(lens0[b])
                d.lat_k[b, :, n:] = 0
                d.lat_v[b, :, n:] = 0
                d.scale_k[b, :, n:] = 0
                d.scale_v[b, :, n:] = 0
        cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        qdt = torch.float16 if w.q_dtype == "fp16" else torch.bfloat16
        self.q = cu(d.q_bits.view(np.int16)).view(qdt)
        self.lat_k, self.lat_v = cu(d.lat_k), cu(d.lat_v)
        self.scale_k, self.scale_v = cu(d.scale_k), cu(d.scale_v)
        self.B_k, self.B_v = cu(d.Bk), cu(d.Bv)
        if w8:  # int8 weights, one fp32 scale per output column
            bkq, sbk = WL.quantize_weights_w8(d.Bk)
            bvq, sbv = WL.quantize_weights_w8(d.Bv)
            self.B_k, self.B_v, self.sB_k, self.sB_v = cu(bkq), cu(bvq), cu(sbk), cu(sbv)
        self.lens0 = cu(lens0.astype(np.int32))
        self.lens = self.lens0.clone()
        self.lens_after = lens_full.astype(np.int64)
        self.out = torch.empty((w.B, w.H, w.Hd), dtype=torch.float32, device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.ws = W.workspace(W.wsvd_decode_workspace_size(w.B, w.H, w.r))
        if self.has_append:
            ai = WL.append_inputs(w, seed=seed, steps=1)
            self.x = cu(ai.x_bits[0].view(np.int16)).view(torch.bfloat16)
            self.A_k, self.A_v = cu(ai.A_k), cu(ai.A_v)
            if w8:
                akq, sak = WL.quantize_weights_w8(ai.A_k)
                avq, sav = WL.quantize_weights_w8(ai.A_v)
                self.A_k, self.A_v, self.sA_k, self.sA_v = cu(akq), cu(avq), cu(sak), cu(sav)
            self.ws_app = W.workspace(W.wsvd_append_workspace_size())
            # the step's host inputs in one pinned buffer, q right after x (one copy per step)
            nx, nq = w.B * w.E, w.B * w.H * w.Hd
            io = torch.empty(nx + nq, dtype=torch.int16).pin_memory()
            io[:nx] = torch.from_numpy(ai.x_bits[0].view(np.int16).reshape(-1).copy())
            io[nx:] = torch.from_numpy(d.q_bits.view(np.int16).reshape(-1).copy())
            self.x_host = io[:nx].view(torch.bfloat16).view(w.B, w.E)
            self.q_host = io[nx:].view(qdt).view(w.B, w.H, w.Hd)
        else:
            self.q_host = torch.from_numpy(d.q_bits.view(np.int16).copy()).view(qdt).pin_memory()
        self.out_host = torch.empty((w.B, w.H, w.Hd), dtype=torch.float32).pin_memory()
        # kernels per step: one when the append and the decode run as one kernel, else the append and
        # the decode's one or two (cluster kernel, or q' + split-L grid)
        if self.has_append:
            self.launches_per_step = W.wsvd_step_launch_count(w.B, w.H, w.Hd, w.E, w.r, w.bits, w.L_cap,
                                                              w.hadamard_block, w8)
        else:
            self.launches_per_step = W.wsvd_decode_launch_count(w.B, w.H, w.Hd, w.r, w.bits, w.L_cap)
        self.one_kernel = self.has_append and self.launches_per_step == 1

    def reset(self):
        self.lens.copy_(self.lens0)

    def append(self):
        if not self.has_append:
            return
        if self.w8:
            self.W.wsvd_latent_append_w8(self.x, self.A_k, self.A_v, self.sA_k, self.sA_v, self.lens, self.lat_k,
                                         self.lat_v, self.scale_k, self.scale_v, bits=self.w.bits,
                                         hadamard_block=self.w.hadamard_block, workspace_buf=self.ws_app,
                                         err=self.err)
        else:
            self.W.wsvd_latent_append(self.x, self.A_k, self.A_v, self.lens, self.lat_k, self.lat_v, self.scale_k,
                                      self.scale_v, bits=self.w.bits, hadamard_block=self.w.hadamard_block,
                                      workspace_buf=self.ws_app, err=self.err)

    def decode(self):
        if self.w8:
            self.W.wsvd_decode_attention_w8(self.q, self.lat_k, self.lat_v, self.scale_k, self.scale_v, self.B_k,
                                            self.B_v, self.sB_k, self.sB_v, self.lens, bits=self.w.bits,
                                            out=self.out, workspace_buf=self.ws, err=self.err)
        else:
            self.W.wsvd_decode_attention(self.q, self.lat_k, self.lat_v, self.scale_k, self.scale_v, self.B_k,
                                         self.B_v, self.lens, bits=self.w.bits, out=self.out, workspace_buf=self.ws,
                                         err=self.err)

    def step(self):
        """One step through the public API: the one-call append + decode when
        the workload appends, else the decode."""
        if not self.has_append:
            self.decode()
            return
        if self.w8:
            self.W.wsvd_append_and_decode_w8(self.x, self.A_k, self.A_v, self.sA_k, self.sA_v, self.lens, self.lat_k,
                                             self.lat_v, self.scale_k, self.scale_v, self.q, self.B_k, self.B_v,
                                             self.sB_k, self.sB_v, bits=self.w.bits,
                                             hadamard_block=self.w.hadamard_block, out=self.out,
                                             append_ws=self.ws_app, decode_ws=self.ws, err=self.err)
            return
        self.W.wsvd_append_and_decode(self.x, self.A_k, self.A_v, self.lens, self.lat_k, self.lat_v, self.scale_k,
                                      self.scale_v, self.q, self.B_k, self.B_v, bits=self.w.bits,
                                      hadamard_block=self.w.hadamard_block, out=self.out, append_ws=self.ws_app,
                                      decode_ws=self.ws, err=self.err)

    def e2e_step(self):
        """Public-API step with host buffers: H2D of the step inputs, append,
        decode, D2H of the result."""
        if self.has_append:
            self.x.copy_(self.x_host, non_blocking=True)
        self.q.copy_(self.q_host, non_blocking=True)
        self.step()
        self.out_host.copy_(self.out, non_blocking=True)

    def e2e_callable(self, graph=True):
        """The public call of one step from host buffers: StepFromHost (fp16
        weights, appending workloads) -- one launch of the captured step graph,
        or with graph=False one wsvd_append_and_decode_host call -- else the
        Python-level copies around the device call."""
        if self.has_append and not self.w8:
            self.e2e_call_name = ("wsvd_step_host_graph_launch (wsvd_append_and_decode_host captured once)" if graph
                                  else "wsvd_append_and_decode_host")
            return self.W.StepFromHost(self.x_host, self.A_k, self.A_v, self.lens, self.lat_k, self.lat_v,
                                       self.scale_k, self.scale_v, self.q_host, self.B_k, self.B_v, self.out_host,
                                       bits=self.w.bits, hadamard_block=self.w.hadamard_block, err=self.err,
                                       graph=graph)
        self.e2e_call_name = "copies + " + ("wsvd_append_and_decode_w8" if self.has_append else "wsvd_decode_attention")
        return self.e2e_step

    def e2e_bytes(self):
        h2d = self.q_host.numel() * 2 + (self.x_host.numel() * 2 if self.has_append else 0)
        return h2d, self.out_host.numel() * 4


def time_comparisons(w: WL.Workload, steps: int, warmup: int, flush):
    """Dense fp16 flash-decode and shared-latent SVD decode on the same shapes."""
    import torch

    import rank_kv_cache_wsvd_b200 as W
    res = {}
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ww = w.with_(R=w.R or 512)
    dd = WL.dense_inputs(ww, seed=0)
    q = cu(dd["q_bits"].view(np.int16)).view(torch.float16 if w.q_dtype == "fp16" else torch.bfloat16)
    K, V, lens = cu(dd["K"]), cu(dd["V"]), cu(dd["seq_lens"])
    del dd
    wsd = W.workspace(W.dense_decode_workspace_size(w.B, w.H, w.Hd))
    out = torch.empty((w.B, w.H, w.Hd), dtype=torch.float32, device="cuda")
    t = _time_loop(lambda: W.dense_decode_attention(q, K, V, lens, out=out, workspace_buf=wsd), steps, warmup, flush)
    nb = int(WL.seq_lens(w).sum()) * w.H * 2 * w.Hd * 2
    res["dense_fp16"] = {"us": t * 1e6, "alg_bytes": nb, "gbs": nb / t / 1e9}
    del K, V
    sd = WL.shared_inputs(ww, seed=0)
    lk, lv, bk, bv = cu(sd["lat_k"]), cu(sd["lat_v"]), cu(sd["Bk"]), cu(sd["Bv"])
    del sd
    wss = W.workspace(W.shared_decode_workspace_size(w.B, w.H, ww.R))
    t = _time_loop(lambda: W.shared_latent_svd_decode(q, lk, lv, bk, bv, lens, out=out, workspace_buf=wss), steps,
                   warmup, flush)
    ntok = int(WL.seq_lens(w).sum())
    per_head = ntok * w.H * 2 * ww.R * 2
    unique = ntok * 2 * ww.R * 2 + 2 * w.H * ww.R * w.Hd * 2
    res["shared_latent_R%d" % ww.R] = {"us": t * 1e6, "per_head_reconstruction_bytes": per_head,
                                       "unique_bytes": unique, "unique_gbs": unique / t / 1e9}
    return res


def time_prefill(w: WL.Workload, T: int, steps: int, warmup: int, flush):
    """The prefill latent write of a T-token block per sequence (the image
    tokens of the prompt) into an empty cache: device time per call, events
    around it, L2 flushed and the lengths reset before each call.  The work is
    a GEMM [B*T x E] . [E x 2*H*r]; the kernels multiply it twice (the hi and
    lo fp16 halves of the rotated activations), so the tensor-core FLOPs are
    twice the useful ones."""
    import torch

    import rank_kv_cache_wsvd_b200 as W
    pi = WL.prefill_inputs(w, seed=0, T=T)
    x = torch.from_numpy(pi.x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    A_k, A_v = torch.from_numpy(pi.A_k).cuda(), torch.from_numpy(pi.A_v).cuda()
    L_cap = max(w.L_cap, T)
    rb = w.r * w.bits // 8
    lk = torch.zeros((w.B, w.H, L_cap, rb), dtype=torch.uint8, device="cuda")
    lv = torch.zeros_like(lk)
    sk = torch.zeros((w.B, w.H, L_cap), dtype=torch.float16, device="cuda")
    sv = torch.zeros_like(sk)
    lens = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = W.workspace(W.wsvd_prefill_workspace_size(w.B, T, w.E))
    call = lambda: W.wsvd_latent_prefill(x, A_k, A_v, lens, lk, lv, sk, sv, bits=w.bits,
                                         hadamard_block=w.hadamard_block, workspace_buf=ws, err=err)
    for _ in range(max(3, warmup)):
        lens.zero_()
        call()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush.zero_()
        lens.zero_()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"prefill device error word {int(err.item())}")
    t = sum(a.elapsed_time(b) for a, b in evs) / 1e3 / steps
    M, N = w.B * T, 2 * w.H * w.r
    flops = 2.0 * M * w.E * N
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peak = json.load(open(pk))["bf16_tflops"] if os.path.exists(pk) else 1590.0
    return {"T": T, "us": t * 1e6, "launches": 3, "useful_tflops": flops / t / 1e12,
            "tensor_tflops": 2 * flops / t / 1e12, "peak_tflops": peak,
            "peak_kind": "measured bf16 burst (fp16 has the same nominal rate)" if os.path.exists(pk) else "fallback",
            "frac_useful": flops / t / 1e12 / peak, "frac_tensor": 2 * flops / t / 1e12 / peak,
            "weights_bytes": 2 * w.H * w.E * w.r * 2, "activation_bytes": M * w.E * 2,
            "note": "tcgen05 kind::f16 128x64 tiles, TMA-fed, accumulators in tensor memory (hi + lo split of the "
                    "rotated activations); rotation + split and the length advance are separate launches"}


def _time_loop(fn, steps, warmup, flush):
    """Device time per call of `fn`: events on the launching stream around the
    call; before each call the L2 is flushed and a device sleep keeps the host
    ahead, as in the timed steps."""
    import torch
    for _ in range(max(3, warmup)):
        fn()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush.zero_()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / 1e3 / steps


# ----------------------------------------------------------------------------- sweep
SWEEP = ["long_r16", "long_r32", "long_r64", "cmp_l2048", "cmp_l8192", "ragged"]


def device_decode_inputs(w: WL.Workload, seed: int):
    """Decode inputs of a full-size workload built on the device (seconds, not
    the minutes the host generator needs at these sizes) with the workload's
    recipe: latents N(0,1) (or Student-t nu = 3 with the workload's x20
    outlier channels) per (b, h, token, channel), per-token scale
    fp16(max|x| / Q), codes round-half-even(x / scale) clamped to +-Q, int4
    packed two per byte (element 2j low nibble); q and B_K, B_V drawn by the
    host generator.  Measurement inputs only: parity tests use workloads.py."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 + seed)
    lens = WL.seq_lens(w, seed)
    Q = 127 if w.bits == 8 else 7
    rb = w.r * w.bits // 8
    gains = torch.from_numpy(WL._outlier_channels(w, seed)).float().cuda() if w.latent != "normal" else None

    def lat():
        out = torch.empty((w.B, w.H, w.L_cap, rb), dtype=torch.uint8, device="cuda")
        sc = torch.empty((w.B, w.H, w.L_cap), dtype=torch.float16, device="cuda")
        for b in range(w.B):
            x = torch.randn((w.H, w.L_cap, w.r), generator=g, device="cuda")
            if gains is not None:  # Student-t with 3 degrees of freedom: z / sqrt(chi2_3 / 3)
                c = torch.randn((3, w.H, w.L_cap, w.r), generator=g, device="cuda").square().sum(0)
                x = x / torch.sqrt(c / 3.0) * gains[:, None, :]
            s16 = (x.abs().amax(-1) / Q).half()
            s = s16.float()[..., None]
            codes = torch.where(s > 0, torch.round(x / torch.where(s > 0, s, torch.ones_like(s))),
                                torch.zeros_like(x)).clamp_(-Q, Q).to(torch.int16)
            if w.bits == 8:
                out[b] = codes.to(torch.int8).view(torch.uint8)
            else:
                nib = (codes & 0xF).to(torch.uint8)
                out[b] = nib[..., 0::2] | (nib[..., 1::2] << 4)
            sc[b] = s16
        return out, sc

    lk, sk = lat()
    lv, sv = lat()
    q, qb = WL.query(w, seed)
    bk, bv = WL.up_proj(w, seed)
    qdt = torch.float16 if w.q_dtype == "fp16" else torch.bfloat16
    qt = torch.from_numpy(qb.view(np.int16).copy()).cuda().view(qdt)
    return dict(q=qt, lat_k=lk, lat_v=lv, scale_k=sk, scale_v=sv, B_k=torch.from_numpy(bk).cuda(),
                B_v=torch.from_numpy(bv).cuda(), seq_lens=torch.from_numpy(lens.astype(np.int32)).cuda(),
                lens=lens)


def run_sweep(names, steps: int, flush, peak: float):
    """Decode-only timing of the 4K-32K workloads: the WSVD decode and the
    in-library dense fp16 decode on the same shape (events around each call,
    L2 flushed before it, host kept ahead), with the HBM fraction of the WSVD
    decode and its speedup against 0.85 x the KV-byte ratio."""
    import torch

    import rank_kv_cache_wsvd_b200 as W
    rows = {}
    for name in names:
        w = WL.PRESETS[name]
        t = device_decode_inputs(w, 0)
        lens = t.pop("lens")
        ws = W.workspace(W.wsvd_decode_workspace_size(w.B, w.H, w.r))
        out = torch.empty((w.B, w.H, w.Hd), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        call = lambda: W.wsvd_decode_attention(t["q"], t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], t["B_k"],
                                               t["B_v"], t["seq_lens"], bits=w.bits, out=out, workspace_buf=ws,
                                               err=err)
        t_w = _time_loop(call, steps, 5, flush)
        if int(err.item()) != 0:
            raise RuntimeError(f"sweep {name}: device error word {int(err.item())}")
        del t
        K = torch.randn((w.B, w.H, w.L_cap, w.Hd), device="cuda").half()
        V = torch.randn_like(K)
        qd = torch.randn((w.B, w.H, w.Hd), device="cuda").half()
        lens_t = torch.from_numpy(lens.astype(np.int32)).cuda()
        wsd = W.workspace(W.dense_decode_workspace_size(w.B, w.H, w.Hd))
        t_d = _time_loop(lambda: W.dense_decode_attention(qd, K, V, lens_t, out=out, workspace_buf=wsd), steps, 5,
                         flush)
        del K, V
        nb = alg_bytes_decode(w, lens)
        dense_bytes = int(lens.sum()) * w.H * 2 * w.Hd * 2
        ratio = dense_bytes / (int(lens.sum()) * w.H * 2 * (w.r * w.bits // 8 + 2))
        gbs = nb / t_w / 1e9
        rows[name] = {"decode_us": t_w * 1e6, "alg_bytes": nb, "gbs": gbs, "frac": gbs / peak,
                      "dense_fp16_us": t_d * 1e6, "dense_gbs": dense_bytes / t_d / 1e9,
                      "speedup_vs_dense": t_d / t_w, "kv_byte_ratio": ratio, "speedup_target": 0.85 * ratio,
                      "launches": W.wsvd_decode_launch_count(w.B, w.H, w.Hd, w.r, w.bits, w.L_cap),
                      "tokens_heads_per_s": int(lens.sum()) * w.H / t_w}
        torch.cuda.empty_cache()
    return rows


# ----------------------------------------------------------------------------- grouped / multi-token decode
# (workload, Hq query heads, Tq tokens per step): G = Hq / w.H query heads per latent head.
GROUPED = {
    "gqa_llava": (WL.LLAVA7B.with_(H=8), 32, 1),      # LLaVA layer, 4 query heads per latent head
    "multi_long": (WL.LONG[32].with_(H=8), 32, 4),    # 32K context, G 4, 4 tokens per step: 16 queries per head
}


def alg_bytes_grouped(w: WL.Workload, lens, Hq: int, Tq: int) -> int:
    rb = w.r * w.bits // 8
    return int(np.sum(lens)) * w.H * 2 * (rb + 2) + 2 * w.H * w.r * w.Hd * 2 + w.B * Tq * Hq * w.Hd * (2 + 4)


def run_grouped(name: str, steps: int, flush, peak: float):
    """Device time of one wsvd_decode_multi call on a grouped workload (events
    around the call, L2 flushed before it), its HBM fraction, the tensor-core
    work it executes, and for comparison the one-query kernel run once per
    query of a head (what serving these queries without the grouped kernel
    reads: the cache once per query)."""
    import torch

    import rank_kv_cache_wsvd_b200 as W
    w, Hq, Tq = GROUPED[name]
    G = Hq // w.H
    t = device_decode_inputs(w, 0)
    lens = t.pop("lens")
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    qdt = torch.float16 if w.q_dtype == "fp16" else torch.bfloat16
    q = torch.randn((w.B, Tq, Hq, w.Hd), generator=g, device="cuda").to(qdt)
    ws = W.workspace(W.wsvd_decode_multi_workspace_size(w.B, Tq, Hq, w.H, w.r, w.L_cap))
    out = torch.empty((w.B, Tq, Hq, w.Hd), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    call = lambda: W.wsvd_decode_multi(q, t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], t["B_k"], t["B_v"],
                                       t["seq_lens"], bits=w.bits, out=out, workspace_buf=ws, err=err)
    t_g = _time_loop(call, steps, 5, flush)
    if int(err.item()) != 0:
        raise RuntimeError(f"grouped {name}: device error word {int(err.item())}")
    q1 = q[:, 0, ::G].contiguous()  # one query per latent head
    ws1 = W.workspace(W.wsvd_decode_workspace_size(w.B, w.H, w.r))
    out1 = torch.empty((w.B, w.H, w.Hd), dtype=torch.float32, device="cuda")
    t_1 = _time_loop(lambda: W.wsvd_decode_attention(q1, t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"],
                                                     t["B_k"], t["B_v"], t["seq_lens"], bits=w.bits, out=out1,
                                                     workspace_buf=ws1), steps, 5, flush)
    nq = G * Tq
    nb = alg_bytes_grouped(w, lens, Hq, Tq)
    units = sum(max(0, int(n) - Tq + 1 + tq) for n in lens for tq in range(Tq)) * Hq  # attended (token, query head)
    tiles = int(np.sum((lens + 127) // 128)) * w.H * ((nq + 15) // 16)
    nq_cta = 4 if nq <= 4 else (8 if nq <= 8 else 16)
    ns, no = (3 * nq_cta + 15) // 16 * 16, 2 * nq_cta
    mo = 64 if w.r <= 64 else 128
    mma_ops = tiles * (2 * 128 * ns * max(32, w.r) + 2 * mo * no * 128)  # executed (padded) MMA operations
    del t
    torch.cuda.empty_cache()
    return {"workload": w.name, "Hq": Hq, "Hkv": w.H, "G": G, "Tq": Tq, "us": t_g * 1e6, "alg_bytes": nb,
            "gbs": nb / t_g / 1e9, "frac": nb / t_g / 1e9 / peak, "units_per_s": units / t_g,
            "tensor_tops_executed": mma_ops / t_g / 1e12,
            "one_query_kernel_us": t_1 * 1e6, "one_query_kernel_x_queries_us": t_1 * 1e6 * nq,
            "speedup_vs_one_query_per_call": t_1 * nq / t_g}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample_step(w: WL.Workload, seed: int, heads: int, cache={}):
    """One step of the float64 oracle on `heads` heads of every sequence (the
    bounded CPU sample): the full latent append of the new token (rotation,
    projection, quantiser, row write, length advance) when the workload
    appends, then the decode of every sampled (b, h).  Returns the
    tokens*heads it attended."""
    import oracle as O
    key = (w.name, seed, heads)
    if key not in cache:
        lens = WL.seq_lens(w, seed)
        q, _ = WL.query(w, seed)
        bk, bv = WL.up_proj(w, seed)
        blocks = {(b, h): WL.latent_cache_block(w, seed, b, h) for b in range(w.B) for h in range(heads)}
        app = None
        if w.append_steps:
            ai = WL.append_inputs(w, seed=seed, steps=1)
            rb = w.r * w.bits // 8
            lat = np.zeros((w.B, heads, w.L_cap, rb), np.uint8)
            sc = np.zeros((w.B, heads, w.L_cap), np.float16)
            app = (ai.x[0], ai.A_k[:heads], ai.A_v[:heads], (lens - 1).astype(np.int32), lat, sc)
        cache[key] = (lens, q, bk, bv, blocks, app)
    lens, q, bk, bv, blocks, app = cache[key]
    if app is not None:
        x, ak, av, lens0, lat, sc = app
        O.latent_append(x, ak, av, lens0, lat, sc, lat, sc, w.r, w.bits, w.hadamard_block)
    n = 0
    for (b, h), (lk, sk, lv, sv) in blocks.items():
        O.wsvd_decode_head(q[b, h], lk, sk, lv, sv, bk[h], bv[h], int(lens[b]), w.r, w.bits)
        n += int(lens[b])
    return n


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def _cpu_leg(w: WL.Workload, budget_s: float, heads: int, threads):
    """Oracle steps for about budget_s seconds; threads=None leaves the BLAS
    pools as they are (all cores), else limits them to that many threads."""
    from contextlib import nullcontext
    try:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(limits=threads) if threads else nullcontext()
    except Exception:
        ctx = nullcontext()
    with ctx:
        cores = cpu_threads()
        oracle_sample_step(w, 0, heads)  # inputs built outside the timing
        t0 = time.perf_counter()
        n_tok, n_steps = 0, 0
        while True:
            n_tok += oracle_sample_step(w, 0, heads)
            n_steps += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = time.perf_counter() - t0
    return {"value": n_tok / dt, "unit": UNIT, "cores": cores, "steps": n_steps, "seconds": dt}


def run_cpu_sample(w: WL.Workload, budget_s: float, heads: int):
    """The float64 oracle as it stands on a bounded sample, timed twice: with
    its BLAS pools limited to one thread and with all of the host's cores.
    The line's value is the all-cores leg."""
    one = _cpu_leg(w, budget_s / 2, heads, 1)
    allc = _cpu_leg(w, budget_s / 2, heads, None)
    work = ("latent append (rotate, project, quantise, write) + " if w.append_steps else "") + "decode"
    return {"value": allc["value"], "unit": UNIT, "cores": allc["cores"], "kind": "oracle",
            "sample": f"float64 oracle steps over {heads} of {w.H} heads of every sequence ({work}); "
                      f"{len(os.sched_getaffinity(0))} host cores available",
            "single_thread": one, "all_cores": allc}


def sample_heads(w: WL.Workload) -> int:
    """Heads per oracle step: about 12800 attended token-heads (tens of ms of float64 work)."""
    per_head_tokens = w.B * (w.L_cap if not isinstance(w.lens, tuple) else sum(w.lens) // 2)
    return max(1, min(w.H, 12800 // max(1, per_head_tokens)))


def run_prefill_line(w: WL.Workload, args, world: int, rank: int, barrier):
    """`--op prefill`: one JSON line for the prompt-block latent write (tokens
    written per second), each rank an independent replica."""
    import torch
    if not w.prefill_tokens:
        raise SystemExit(f"workload {w.name} has no prefill block")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    barrier()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.25)
    pf = time_prefill(w, w.prefill_tokens, args.steps, args.warmup, flush)
    clk = clocks.stop()
    barrier()
    t = pf["us"] * 1e-6
    value, t_total = replica_throughput(w.B * w.prefill_tokens * args.steps, t * args.steps, world)
    if rank == 0:
        line = {
            "metric": "prefill latent write: prompt tokens written into the low-rank cache per second",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_total / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16 (hi + lo split), f32 accumulate", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.prefill_tokens, "E": w.E, "H": w.H, "r": w.r,
                       "latent_bits": w.bits, "l2": "flushed between timed calls (256 MiB write)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "tensor", "kernel": "prefill (rotate + GEMM/quantise + advance, 3 launches)",
                         "achieved": pf["tensor_tflops"], "peak": pf["peak_tflops"], "unit": "TFLOP/s",
                         "frac": pf["frac_tensor"], "peak_kind": pf["peak_kind"],
                         "traffic": ncu_traffic("prefill_gemm", "llava7b" if w is WL.LLAVA7B else w.name),
                         "traffic_kernel": "prefill_gemm_kernel (DRAM bytes per launch, ncu)",
                         "useful_tflops": pf["useful_tflops"]},
            "prefill": pf, "gpu_launches": 3 * args.steps, "clocks": clk,
        }
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="wsvd", choices=["wsvd", "reference"])
    ap.add_argument("--workload", default="llava7b", choices=sorted(WL.PRESETS))
    ap.add_argument("--cpu-seconds", type=float, default=16.0,
                    help="CPU baseline budget, split between the one-thread and all-cores legs")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the decode-only sweep over the 4K-32K workloads (default line only)")
    ap.add_argument("--no-extras", action="store_true", help="skip the CPU baseline, e2e and comparison timings")
    ap.add_argument("--weights", default="fp16", choices=["fp16", "int8"],
                    help="low-rank factors A, B as fp16, or int8 with per-column scales (W8)")
    ap.add_argument("--op", default="step", choices=["step", "prefill", "grouped"],
                    help="step: the decode step (append + decode); prefill: the prompt-block latent write alone; "
                         "grouped: the grouped-query / multi-token decode (--grouped-workload)")
    ap.add_argument("--grouped-workload", default="multi_long", choices=sorted(GROUPED))
    args = ap.parse_args()
    w = WL.PRESETS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        heads = sample_heads(w)
        for _ in range(max(0, args.warmup)):
            oracle_sample_step(w, 0, heads)
        t0 = time.perf_counter()
        n = sum(oracle_sample_step(w, 0, heads) for _ in range(args.steps))
        dt = time.perf_counter() - t0
        v = n / dt
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": w.name, "sample_heads": heads},
                "cpu_baseline": {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                                 "sample": f"{heads} of {w.H} heads of every sequence per step"},
                "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist

    import rank_kv_cache_wsvd_b200 as W
    W.load()  # fails loudly if the library is missing
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    if args.op == "grouped":
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        barrier()
        clocks = ClockSampler(torch.cuda.current_device())
        clocks.start()
        time.sleep(0.25)
        gr = run_grouped(args.grouped_workload, args.steps, flush, peaks()[0])
        clk = clocks.stop()
        barrier()
        t = gr["us"] * 1e-6
        value, t_total = replica_throughput(gr["units_per_s"] * t * args.steps, t * args.steps, world)
        if rank == 0:
            peak, kind = peaks()
            print(json.dumps({
                "metric": "grouped / multi-token low-rank decode: attended (token, query head) pairs per second",
                "value": value, "unit": "token*query_heads/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": t_total / args.steps * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "s8 x s8 -> s32 scores, f16 x f16 -> f32 values",
                "data": "synthetic",
                "config": {"workload": args.grouped_workload, "shape": gr["workload"], "Hq": gr["Hq"],
                           "Hkv": gr["Hkv"], "Tq": gr["Tq"], "l2": "flushed between timed calls (256 MiB write)",
                           "parallelism": f"replicas x{world}"},
                "roofline": {"bound": "hbm", "kernel": "grouped_decode_kernel (1 launch)", "achieved": gr["gbs"],
                             "peak": peak, "unit": "GB/s", "frac": gr["gbs"] / peak, "peak_kind": kind,
                             "traffic": ncu_traffic("grouped", args.grouped_workload),
                             "traffic_kernel": "grouped_decode_kernel (DRAM bytes per launch, ncu)",
                             "alg_bytes_per_launch": gr["alg_bytes"],
                             "tensor_tops_executed": gr["tensor_tops_executed"]},
                "grouped": gr, "gpu_launches": args.steps, "clocks": clk}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    if args.op == "prefill":
        run_prefill_line(w, args, world, rank, barrier)
        if world > 1:
            dist.destroy_process_group()
        return

    w8 = args.weights == "int8"
    st = WsvdStep(w, seed=rank, w8=w8)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    for _ in range(3):  # first calls (library load, per-device setup) outside everything timed
        st.reset()
        st.append()
        st.decode()
        st.reset()
        st.step()
    torch.cuda.synchronize()
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        st.reset()
        st.step()
    torch.cuda.synchronize()
    barrier()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.25)
    # Timed region: per step one call of the public step (append, then the
    # decode launched behind it), bracketed by events on its stream.  Before
    # the first event (outside the timed interval) the L2 is flushed, the
    # lengths are reset and a device sleep keeps the host ahead of the device.
    evs = []
    for _ in range(args.steps):
        flush.zero_()
        st.reset()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record()
        st.step()
        e[1].record()
        evs.append(e)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    t_step = sum(e[0].elapsed_time(e[1]) for e in evs) / 1e3
    # Per-kernel durations (the roofline's denominators): inside the step the
    # decode overlaps the append, so each kernel is timed here as its own
    # launch, events around it, under the same flush and host lead.
    # At least 100 samples: the two kernels are close at small shapes and the
    # event clock ticks in about a microsecond.
    n_b = min(max(args.steps, 100), 300)
    evs = []
    for _ in range(n_b):
        flush.zero_()
        st.reset()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        st.append()
        e[1].record()
        st.decode()
        e[2].record()
        evs.append(e)
    torch.cuda.synchronize()
    t_app = sum(e[0].elapsed_time(e[1]) for e in evs) / 1e3 / n_b * args.steps if st.has_append else 0.0
    t_dec = sum(e[1].elapsed_time(e[2]) for e in evs) / 1e3 / n_b * args.steps
    t_sep = sum(e[0].elapsed_time(e[2]) for e in evs) / 1e3 / n_b
    # Context (not part of `value`): the step replayed from one CUDA graph.
    g_step = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        st.reset()
        st.step()
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(g_step):
        st.step()
    n_g = min(args.steps, 300)
    evs = []
    for _ in range(n_g):
        flush.zero_()
        st.reset()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record()
        g_step.replay()
        e[1].record()
        evs.append(e)
    torch.cuda.synchronize()
    t_graph = sum(e[0].elapsed_time(e[1]) for e in evs) / 1e3 / n_g
    del g_step
    units_local = attended_tokens(w, st.lens_after) * args.steps
    value, t_total = replica_throughput(units_local, t_step, world)
    if int(st.err.item()) != 0:
        raise RuntimeError(f"device error word {int(st.err.item())}")

    ms_per_step = t_total / args.steps * 1e3
    peak, peak_kind = peaks()
    dec_bytes = alg_bytes_decode(w, st.lens_after, w8)
    app_bytes = alg_bytes_append(w, w8) if st.has_append else 0
    per_app = t_app / args.steps
    per_dec = t_dec / args.steps
    if st.one_kernel:
        dom, nbytes, dur, launches = "step", app_bytes + dec_bytes, t_step / args.steps, \
            "wsvd one-kernel step (append + decode, 1 launch)"
    elif st.has_append and per_app >= per_dec:
        dom, nbytes, dur, launches = "append", app_bytes, per_app, "wsvd latent append (1 launch)"
    else:
        dom, nbytes, dur, launches = "decode", dec_bytes, per_dec, \
            "wsvd decode (1 launch: split-L + last-arriver combine)"
    achieved = nbytes / dur / 1e9
    traffic = ncu_traffic(dom, args.workload + ("_w8" if w8 else ""))

    extras = {}
    if not args.no_extras and rank == 0:
        # End to end through the public API with host buffers: one library call
        # per step (x and q brought in from pinned host memory, append, decode,
        # out delivered to pinned host memory) and a stream synchronisation;
        # host wall clock around the two.
        # The length reset that lets every step append the same row is done
        # before the clock starts.
        n_e2e = max(50, min(args.steps, 500))
        stream = torch.cuda.current_stream()

        def wall_per_step(fn):
            for _ in range(10):
                st.reset()
                fn()
            torch.cuda.synchronize()
            total = 0.0
            for _ in range(n_e2e):
                st.reset()
                stream.synchronize()
                t0 = time.perf_counter()
                fn()
                stream.synchronize()
                total += time.perf_counter() - t0
            return total

        fn = st.e2e_callable(graph=True)
        t_e2e = wall_per_step(fn)
        call_name = st.e2e_call_name
        direct = None
        if st.has_append and not w8:
            fd = st.e2e_callable(graph=False)
            direct = {"us_per_step": wall_per_step(fd) / n_e2e * 1e6, "call": st.e2e_call_name}
        if hasattr(fn, "close"):
            fn.close()
        h2d, d2h = st.e2e_bytes()
        extras["e2e"] = {"value": attended_tokens(w, st.lens_after) * n_e2e / t_e2e, "unit": UNIT,
                         "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                         "us_per_step": t_e2e / n_e2e * 1e6,
                         "timing": "host wall clock around one library call + stream sync per step",
                         "call": call_name}
        if direct is not None:
            extras["e2e"]["direct_call"] = direct
        extras["comparisons_same_shape"] = time_comparisons(w, min(args.steps, 200), 5, flush)
        extras["comparisons_same_shape"]["wsvd_decode"] = {"us": per_dec * 1e6, "alg_bytes": dec_bytes,
                                                           "gbs": dec_bytes / per_dec / 1e9}
        if st.has_append and w.prefill_tokens:
            extras["prefill"] = time_prefill(w, w.prefill_tokens, min(args.steps, 200), 5, flush)
        extras["cpu_baseline"] = run_cpu_sample(w, args.cpu_seconds, sample_heads(w))
        if not args.no_sweep and args.workload == "llava7b":
            extras["grouped"] = {k: run_grouped(k, 300, flush, peaks()[0]) for k in GROUPED}
            extras["sweep"] = run_sweep(SWEEP, 300, flush, peaks()[0])
            extras["sweep"]["note"] = ("decode-only, events around each call, L2 flushed before it; frac = "
                                       "algorithmic GB/s / peak (%s); target frac >= 0.70 and speedup_vs_dense "
                                       ">= speedup_target = 0.85 x kv_byte_ratio" % peaks()[1])

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "Hd": w.Hd, "r": w.r,
                       "latent_bits": w.bits, "weights": args.weights,
                       "attended_tokens_per_seq": [int(x) for x in st.lens_after],
                       "step": ("append + decode" if st.has_append else "decode"),
                       "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"replicas x{world}",
                       "launch": ("one wsvd_append_and_decode call per step (one kernel: append and decode); "
                                  "events around the call" if st.one_kernel else
                                  "one wsvd_append_and_decode call per step (decode launched behind the "
                                  "append as a programmatic dependent); events around the call"
                                  if st.has_append else "one wsvd_decode_attention call per step; events around it")},
            "step_us": ms_per_step * 1e3,
            "breakdown_us": {"append": per_app * 1e6, "decode": per_dec * 1e6,
                             "two_calls": t_sep * 1e6,
                             "note": "each kernel as its own launch, events around it (same flush and host lead)"},
            "graph_step_us": t_graph * 1e6,
            "hbm_gbs": (dec_bytes + app_bytes) / (t_total / args.steps) / 1e9,
            "roofline": {"bound": "hbm", "kernel": launches, "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind, "traffic": traffic,
                         "alg_bytes_per_launch": nbytes, "frac_of_nominal_8TBs": achieved / NOMINAL_HBM_GBS},
            "gpu_launches": st.launches_per_step * args.steps,
            "clocks": clk,
        }
        for k in ("cpu_baseline", "e2e", "comparisons_same_shape", "prefill", "sweep", "grouped"):
            if k in extras:
                line[k] = extras[k]
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
