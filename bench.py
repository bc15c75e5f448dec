"""Benchmark of the Mamba-2 layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one prefill layer call over one batch of the Nemotron-3-Nano-shaped
long-context workload (1 sequence x 262144 tokens, 64 heads x 64, d_state 128,
8 groups, chunk 128, conv 4, bf16 I/O, fp32 state): causal conv1d+SiLU, then
the chunked SSD scan (dt softplus, chunk cumsum, C.B^T o L times X, chunk
states, state passing, C.h + D.x), with inputs resident in HBM.  Rank 0
prints one JSON line.  Next to the headline prefill number the line carries:
  roofline      the scan kernel's achieved HBM GB/s on the headline workload
                (algorithmic bytes per launch / its CUDA-event duration)
                against the measured peak;
  prefill       the same measurement (layer tokens/s, scan and conv rooflines)
                for each prefill workload: the FRANKENSTALLM-H 3B layer (8 x
                2048 tokens, 40 heads), the Nemotron-H 8B layer (4 x 4096
                tokens, 128 heads) and the headline one;
  decode        one decode step of the 256-sequence, 128-head workload
                (conv-cache roll, conv + SiLU and state update in one
                kernel), its GB/s; the two-kernel form beside it;
  backward      the scan's backward pass on the 3B layer;
  mixer         the whole Mamba-2 mixer of the 3B layer (in_proj, the path,
                gated RMSNorm, out_proj; d_model 2560) and its in_proj linear
                layer alone, against the bf16 tensor peak;
  e2e           the headline prefill step through the public one-call entry
                point (ssd_conv_scan_fwd) with the step's inputs copied from
                pinned host memory and y + final state copied back, inside the
                timed region; the sequence goes through in pieces (conv cache
                and state carried over) so that copies and compute overlap;
  cpu_baseline  the fp64 oracle timed on this host's cores on a bounded sample
                (a 4096-token prefix of the headline workload).
Multi-GPU: one process per GPU (torchrun); each rank runs its own batch
(independent sequences, no data-path collective): weak scaling.
``--impl reference`` times the fp64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from ssd_selective_scan_b200 import shard, synth  # noqa: E402

METRIC = "SSD prefill scan tokens/s/layer & % roofline; decode state-update HBM GB/s"
HEADLINE = 3                      # the largest single-GPU prefill workload
PREFILL_CONFIGS = (1, 2, 3)
PREFILL = synth.CONFIGS[HEADLINE]
BWD = synth.CONFIGS[1]            # the backward pass is timed on the 3B layer
MIXER = synth.CONFIGS[1]          # the whole mixer is timed on the 3B layer ...
MIXER_D_MODEL = 2560              # ... with its d_model
DECODE = synth.CONFIGS[4]
RAGGED = synth.CONFIGS[1]         # ragged prefill: the 3B layer's tokens packed as prompts of mixed lengths
ORACLE_PREFIX = 4096              # tokens of the headline workload the oracle times
E2E_PIECES = 8                    # the end-to-end leg streams the sequence in this many pieces
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# ----------------------------------------------------------------------------
# algorithmic work (bytes the method must move; FLOPs of the causal tiles)
# ----------------------------------------------------------------------------

def scan_bytes_per_token(s) -> int:
    """x, B, C, dt read and y written once: e * (2*H*P + 2*G*N + H)."""
    return s.elem_bytes * (2 * s.H * s.P + 2 * s.G * s.N + s.H)


def scan_flops_per_token(s) -> int:
    """causal C.B^T (G*Q*N) + causal (..)X (H*Q*P) + chunk state and C.h (4*H*P*N)."""
    return s.G * s.Q * s.N + s.H * s.Q * s.P + 4 * s.H * s.P * s.N


def conv_bytes_per_token(s) -> int:
    return 2 * s.elem_bytes * s.conv_dim


def decode_state_update_bytes(s) -> int:
    """fp32 state read + written, x/B/C/dt read, y written."""
    return 8 * s.b * s.H * s.P * s.N + s.elem_bytes * s.b * (s.H * s.P + 2 * s.G * s.N + s.H + s.H * s.P)


def scan_bwd_bytes_per_token(s) -> int:
    """Backward pass: x, B, C, dt, dy read; dx, dB, dC, ddt written."""
    return s.elem_bytes * (3 * s.H * s.P + 4 * s.G * s.N + 2 * s.H)


def scan_bwd_flops_per_token(s) -> int:
    """Backward pass, the chunked matrix form: causal C.B^T (G*Q*N), causal
    dY.X^T and M3^T.dY (2*H*Q*P), causal M1.B and M1^T.C (2*H*Q*N), and the
    five state products S, dS, (Ec o dY).h0, (El o X).g, B.g^T (10*H*P*N)."""
    return s.G * s.Q * s.N + 2 * s.H * s.Q * s.P + 2 * s.H * s.Q * s.N + 10 * s.H * s.P * s.N


def linear_flops(M, N, K) -> int:
    return 2 * M * N * K


def mixer_flops(s, d_model) -> int:
    """in_proj + out_proj products, plus the scan's causal-tile FLOPs."""
    M = s.b * s.L
    nproj = 2 * s.H * s.P + 2 * s.G * s.N + s.H
    return linear_flops(M, nproj, d_model) + linear_flops(M, d_model, s.H * s.P) + scan_flops_per_token(s) * M


def decode_step_bytes(s) -> int:
    """The one-kernel decode step: fp32 state read + written, conv cache read +
    written (k columns), the token's xBC and dt read, y written."""
    return 8 * s.b * s.H * s.P * s.N + s.elem_bytes * s.b * (2 * s.k * s.conv_dim + s.conv_dim + s.H + s.H * s.P)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0, source="fallback")


def scan_kernel_traffic(kernel_tag: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(kernel_tag)
        if e and e.get("source_sha") == source_digest():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# The sources the tensor-core scan kernel is compiled from.
SCAN_SOURCES = ("chunk_scan_tc.cu", "sm100.cuh", "common.cuh", "kernels.h")


def source_digest() -> str:
    """Digest of the scan kernel's code with comments and whitespace removed,
    so that an edit to the documentation alone keeps the counters valid."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ssd_selective_scan_b200", "csrc")
    for name in SCAN_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update((name + " " + " ".join(text.split())).encode())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        # nvidia-smi ignores CUDA_VISIBLE_DEVICES: address the GPU by UUID
        try:
            self.gpu = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.gpu = str(device.index or 0)
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for r in csv.reader(f):
                    if len(r) >= 9:
                        rows.append([c.strip() for c in r])
            os.unlink(self.path)
        except Exception:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# the prefill step, the decode step, and their timing
# ----------------------------------------------------------------------------

class PrefillStep:
    def __init__(self, s, seed, dev, layer_call: bool = False):
        from ssd_selective_scan_b200 import layer
        self.layer = layer
        self.s = s
        inp = synth.layer_inputs(s, seed)
        self.host = inp
        self.d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
        self.conv_state = torch.zeros(s.b, s.conv_dim, s.k, dtype=s.torch_dtype, device=dev)
        self.u = torch.empty(s.b, s.L, s.conv_dim, dtype=s.torch_dtype, device=dev)
        self.y = torch.empty(s.b, s.L, s.H, s.P, dtype=s.torch_dtype, device=dev)
        self.fs = torch.empty(s.b, s.H, s.P, s.N, dtype=torch.float32, device=dev)
        self.views = layer.split_channels(self.u, s.H, s.P, s.G, s.N)
        need = layer.chunk_scan_workspace_bytes(s.b, s.L, s.H, s.P, s.N, s.G, s.Q, s.torch_dtype)
        self.ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev) if need else None
        self.ws_layer = None
        if layer_call:
            need = layer.conv_scan_workspace_bytes(s.b, s.L, s.H, s.P, s.N, s.G, s.Q, s.k, s.torch_dtype)
            self.ws_layer = torch.empty(need, dtype=torch.uint8, device=dev)

    def conv(self):
        d = self.d
        self.layer.conv1d_silu(d["xBC"], d["w"], d["bias"], self.conv_state, out=self.u)

    def scan(self):
        d, s = self.d, self.s
        x, B, C = self.views
        self.layer.chunk_scan_fwd(x, B, C, d["dt_raw"], d["A"], d["dt_bias"], d["D"], None,
                                  Q=s.Q, y=self.y, final_state=self.fs, workspace=self.ws)

    def __call__(self):
        self.conv()
        self.scan()

    def layer_call(self):
        """The same two kernels through the one-call prefill entry point."""
        d, s = self.d, self.s
        self.layer.conv_scan_fwd(d["xBC"], d["w"], d["dt_raw"], d["A"], s.H, s.P, s.G, s.N,
                                 bias=d["bias"], conv_state=self.conv_state, dt_bias=d["dt_bias"],
                                 D=d["D"], Q=s.Q, y=self.y, final_state=self.fs,
                                 workspace=self.ws_layer)


class BackwardStep:
    """The scan's backward pass on the scan inputs of a prefill workload."""

    def __init__(self, s, seed, dev):
        from ssd_selective_scan_b200 import layer
        self.layer = layer
        self.s = s
        inp = synth.scan_inputs(s, seed)
        self.d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
        g = torch.Generator().manual_seed(seed + 1)
        self.dy = torch.randn(s.b, s.L, s.H, s.P, generator=g).to(s.torch_dtype).to(dev)
        self.views = layer.split_channels(self.d["u"], s.H, s.P, s.G, s.N)
        need = layer.chunk_scan_bwd_workspace_bytes(s.b, s.L, s.H, s.P, s.N, s.G, s.torch_dtype)
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)

    def __call__(self):
        d, s = self.d, self.s
        x, B, C = self.views
        self.layer.chunk_scan_bwd(x, B, C, d["dt_raw"], d["A"], self.dy, d["dt_bias"], d["D"], None,
                                  None, want_dinit=False, workspace=self.ws)


class MixerStep:
    """The whole mixer (and its in_proj alone) on a prefill workload."""

    def __init__(self, s, d_model, seed, dev):
        from ssd_selective_scan_b200 import layer
        self.layer = layer
        self.s, self.d_model = s, d_model
        inp = synth.mixer_inputs(s, d_model, seed)
        self.d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
        self.out = torch.empty(s.b, s.L, d_model, dtype=torch.bfloat16, device=dev)
        self.fs = torch.empty(s.b, s.H, s.P, s.N, dtype=torch.float32, device=dev)
        need = layer.mixer_workspace_bytes(s.b, s.L, d_model, s.H, s.P, s.N, s.G, s.Q, s.k)
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        self.zx = torch.empty(s.b * s.L, self.d["W_in"].shape[0], dtype=torch.bfloat16, device=dev)

    def __call__(self):
        d, s = self.d, self.s
        self.layer.mixer_forward(d["hidden"], d["W_in"], d["conv_w"], d["dt_bias"], d["A"], d["D"], d["norm_w"],
                                 d["W_out"], s.H, s.P, s.G, s.N, Q=s.Q, out=self.out, final_state=self.fs,
                                 workspace=self.ws)

    def in_proj(self):
        self.layer.linear(self.d["hidden"].view(-1, self.d_model), self.d["W_in"], y=self.zx)


class RaggedStep:
    """The ragged scan (ssd_chunk_scan_fwd_varlen) on a prefill workload's
    tokens packed as a batch of prompts: a seeded length mix, or the
    workload's own equal lengths."""

    def __init__(self, s, seed, dev, lens=None):
        from ssd_selective_scan_b200 import layer
        self.layer = layer
        T = s.b * s.L
        self.lens = synth.ragged_lengths(T, seed) if lens is None else list(lens)
        self.s = s.with_(b=1, L=T)
        inp = synth.scan_inputs(self.s, seed)
        u = inp["u"][0].to(dev)
        x, B, C = layer.split_channels(u, s.H, s.P, s.G, s.N)
        self.x, self.B, self.C = x.view(T, s.H, s.P), B.view(T, s.G, s.N), C.view(T, s.G, s.N)
        self.dt = inp["dt_raw"][0].contiguous().to(dev)
        self.A, self.dtb, self.D = inp["A"].to(dev), inp["dt_bias"].to(dev), inp["D"].to(dev)
        offs = [0]
        for n in self.lens:
            offs.append(offs[-1] + n)
        self.cu = torch.tensor(offs, dtype=torch.int32, device=dev)
        self.y = torch.empty(T, s.H, s.P, dtype=s.torch_dtype, device=dev)
        self.fs = torch.empty(len(self.lens), s.H, s.P, s.N, dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        need = layer.chunk_scan_varlen_workspace_bytes(len(self.lens), T, s.H, s.P, s.N, s.G, s.Q, s.torch_dtype)
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.layer.chunk_scan_fwd_varlen(self.x, self.B, self.C, self.dt, self.A, self.cu, self.dtb, self.D, None,
                                         Q=self.s.Q, y=self.y, final_state=self.fs, workspace=self.ws,
                                         status=self.status)


class DecodeStep:
    def __init__(self, s, seed, dev):
        from ssd_selective_scan_b200 import layer
        self.layer = layer
        self.s = s
        inp = synth.decode_inputs(s, seed)
        self.d = {k: v.to(dev) for k, v in inp.items()}
        self.u = torch.empty(s.b, s.conv_dim, dtype=s.torch_dtype, device=dev)
        self.y = torch.empty(s.b, s.H, s.P, dtype=s.torch_dtype, device=dev)
        self.views = layer.split_channels(self.u, s.H, s.P, s.G, s.N)
        self.ws = layer.decode_step_workspace(s.b, s.G, dev)

    def conv(self):
        d, s = self.d, self.s
        self.layer.conv1d_silu(d["xBC"].view(s.b, 1, s.conv_dim), d["w"], None, d["conv_state"],
                               out=self.u.view(s.b, 1, s.conv_dim))

    def update(self):
        d = self.d
        x, B, C = self.views
        self.layer.state_update(d["state"], x, B, C, d["dt_raw"], d["A"], d["dt_bias"], d["D"],
                                y=self.y)

    def __call__(self):
        """One decode token per sequence through the one-kernel decode step,
        one CTA per (sequence, head) with its workspace of arrival counters."""
        d, s = self.d, self.s
        self.layer.decode_step(d["xBC"], d["w"], d["conv_state"], d["state"], d["dt_raw"], d["A"],
                               s.H, s.P, s.G, s.N, dt_bias=d["dt_bias"], D=d["D"], y=self.y, workspace=self.ws)

    def per_group(self):
        """The same step, one CTA per (sequence, group), no workspace."""
        d, s = self.d, self.s
        self.layer.decode_step(d["xBC"], d["w"], d["conv_state"], d["state"], d["dt_raw"], d["A"],
                               s.H, s.P, s.G, s.N, dt_bias=d["dt_bias"], D=d["D"], y=self.y)


def _events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def workload_config(s) -> dict:
    """The `config` block of a prefill workload (the same in both arms)."""
    return {"workload": s.name, "batch": s.b, "seq_len": s.L, "heads": s.H, "head_dim": s.P,
            "d_state": s.N, "groups": s.G, "chunk": s.Q, "conv": s.k, "state_dtype": "f32",
            "per_rank_batch": s.b,
            "l2": f"inputs larger than L2 (xBC {s.b * s.L * s.conv_dim * s.elem_bytes / 1e6:.0f} MB, "
                  f"conv output the same, per step)",
            "step": "conv1d+SiLU then chunked SSD scan (one prefill layer)"}


def scan_roofline(s, scan_ms: float, peaks: dict, traffic) -> dict:
    tokens = s.b * s.L
    scan_bytes = scan_bytes_per_token(s) * tokens
    flops = scan_flops_per_token(s) * tokens
    achieved = scan_bytes / (scan_ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "chunk_scan", "achieved": achieved,
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
            "traffic": traffic, "algorithmic_bytes_per_launch": scan_bytes,
            "algorithmic_flops_per_launch": flops,
            "tensor_frac": flops / (scan_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "peak_source": peaks["source"], "launch_ms": scan_ms}


def time_prefill(step, K, W, barrier, max_over_ranks):
    """W untimed steps, then K timed steps with per-kernel CUDA events on the
    launching stream.  Returns (ms per step, mean conv ms, mean scan ms), each
    the max over ranks."""
    for _ in range(W):
        step()
    ev_scan = _events(2 * K)
    ev_conv = _events(2 * K)
    t0, t1 = _events(2)
    barrier()
    t0.record()
    for i in range(K):
        ev_conv[2 * i].record()
        step.conv()
        ev_conv[2 * i + 1].record()
        ev_scan[2 * i].record()
        step.scan()
        ev_scan[2 * i + 1].record()
    t1.record()
    barrier()
    ms_step = max_over_ranks(t0.elapsed_time(t1) / K)
    scan_ms = max_over_ranks(statistics.mean(ev_scan[2 * i].elapsed_time(ev_scan[2 * i + 1]) for i in range(K)))
    conv_ms = max_over_ranks(statistics.mean(ev_conv[2 * i].elapsed_time(ev_conv[2 * i + 1]) for i in range(K)))
    return ms_step, conv_ms, scan_ms


def run_ours(args, rank, world, dev):
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(v: float) -> float:
        return shard.max_over_ranks(v, dev)

    K = args.steps
    peaks = load_peaks()

    # the other prefill workloads, each measured the same way
    blocks = {}
    for cfg in PREFILL_CONFIGS:
        if cfg == HEADLINE:
            continue
        s = synth.CONFIGS[cfg]
        st = PrefillStep(s, shard.rank_seed(synth.config_seed(cfg), rank), dev)
        ms_step, conv_ms, scan_ms = time_prefill(st, K, args.warmup, barrier, max_over_ranks)
        tokens = s.b * s.L
        blocks[s.name] = {
            "tokens_per_s": shard.aggregate_tokens_per_s(tokens, world, ms_step), "ms_per_step": ms_step,
            "scan": scan_roofline(s, scan_ms, peaks, scan_kernel_traffic(f"chunk_scan@{s.name}")),
            "conv": {"ms": conv_ms, "GB/s": conv_bytes_per_token(s) * tokens / (conv_ms * 1e-3) / 1e9,
                     "frac_hbm": conv_bytes_per_token(s) * tokens / (conv_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}}
        del st
        torch.cuda.empty_cache()

    # the headline workload, with the clocks sampled over its timed region
    s = PREFILL
    step = PrefillStep(s, shard.rank_seed(synth.config_seed(HEADLINE), rank), dev, layer_call=True)
    barrier()
    with ClockSampler(dev) as clk:
        ms_step, conv_ms, scan_ms = time_prefill(step, K, args.warmup, barrier, max_over_ranks)
        # keep the sampler alive over a longer stretch of identical work so the
        # clock record has enough samples (not part of the timed number)
        t_end = time.time() + max(0.0, 1.5 - ms_step * K / 1e3)
        while time.time() < t_end:
            for _ in range(5):
                step()
            torch.cuda.synchronize()
    clocks = clk.summary()
    tokens = s.b * s.L
    head_roof = scan_roofline(s, scan_ms, peaks, scan_kernel_traffic(f"chunk_scan@{s.name}"))
    blocks[s.name] = {
        "tokens_per_s": shard.aggregate_tokens_per_s(tokens, world, ms_step), "ms_per_step": ms_step,
        "scan": head_roof,
        "conv": {"ms": conv_ms, "GB/s": conv_bytes_per_token(s) * tokens / (conv_ms * 1e-3) / 1e9,
                 "frac_hbm": conv_bytes_per_token(s) * tokens / (conv_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}}

    # end to end through the public API: every step copies its inputs from
    # pinned host memory and its results back.  The sequence goes through in
    # E2E_PIECES pieces (chunked prefill: the conv cache and the state carry
    # from piece to piece, bit-identical to one call), so the copies in, the
    # layer and the copies out of different pieces overlap on three streams.
    pin_x = step.host["xBC"].pin_memory()
    pin_dt = step.host["dt_raw"].pin_memory()
    out_y = torch.empty(step.y.shape, dtype=step.y.dtype, pin_memory=True)
    out_fs = torch.empty(step.fs.shape, dtype=torch.float32, pin_memory=True)
    KE = max(3, min(10, K // 4))
    npiece = E2E_PIECES if (s.b == 1 and s.L % (E2E_PIECES * s.Q) == 0) else 1
    plen = s.L // npiece
    st_in, st_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    comp = torch.cuda.current_stream(dev)
    prev_comp = [None] * npiece   # the previous step's events, per piece
    prev_out = [None] * npiece
    d = step.d

    def e2e_step():
        ev_start = torch.cuda.Event()   # the step's copies start inside the timed region
        ev_start.record(comp)
        st_in.wait_event(ev_start)
        for i in range(npiece):
            a, b = i * plen, (i + 1) * plen
            ev_in = torch.cuda.Event()
            with torch.cuda.stream(st_in):
                if prev_comp[i] is not None:
                    st_in.wait_event(prev_comp[i])   # the previous step's layer has read this piece
                d["xBC"][:, a:b].copy_(pin_x[:, a:b], non_blocking=True)
                d["dt_raw"][:, a:b].copy_(pin_dt[:, a:b], non_blocking=True)
                ev_in.record(st_in)
            comp.wait_event(ev_in)
            if prev_out[i] is not None:
                comp.wait_event(prev_out[i])         # the previous step's y of this piece is out
            step.layer.conv_scan_fwd(d["xBC"][:, a:b], d["w"], d["dt_raw"][:, a:b], d["A"], s.H, s.P, s.G, s.N,
                                     bias=d["bias"], conv_state=step.conv_state, dt_bias=d["dt_bias"], D=d["D"],
                                     init_state=step.fs if i > 0 else None, Q=s.Q, y=step.y[:, a:b],
                                     final_state=step.fs, workspace=step.ws_layer)
            ev_c = torch.cuda.Event()
            ev_c.record(comp)
            prev_comp[i] = ev_c
            ev_out = torch.cuda.Event()
            with torch.cuda.stream(st_out):
                st_out.wait_event(ev_c)
                out_y[:, a:b].copy_(step.y[:, a:b], non_blocking=True)
                if i == npiece - 1:
                    out_fs.copy_(step.fs, non_blocking=True)
                ev_out.record(st_out)
            prev_out[i] = ev_out
        comp.wait_event(prev_out[npiece - 1])        # the step ends when its results are on the host

    for _ in range(2):
        e2e_step()
    e0, e1 = _events(2)
    barrier()
    e0.record()
    for _ in range(KE):
        e2e_step()
    e1.record()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / KE)
    h2d = pin_x.numel() * pin_x.element_size() + pin_dt.numel() * pin_dt.element_size()
    d2h = out_y.numel() * out_y.element_size() + out_fs.numel() * 4
    del step, pin_x, pin_dt, out_y, out_fs
    torch.cuda.empty_cache()

    # decode: one token per sequence through the one-kernel decode step (the
    # state is rewritten in place, so consecutive steps are valid work)
    dec = DecodeStep(DECODE, shard.rank_seed(synth.config_seed(4), rank), dev)
    for _ in range(max(3, args.warmup)):
        dec()
    KD = max(10, K)
    d0, d1 = _events(2)
    barrier()
    d0.record()
    for _ in range(KD):
        dec()
    d1.record()
    barrier()
    dec_ms = max_over_ranks(d0.elapsed_time(d1) / KD)
    # the one-kernel step without the workspace (one CTA per sequence and group)
    for _ in range(3):
        dec.per_group()
    d4, d5 = _events(2)
    barrier()
    d4.record()
    for _ in range(KD):
        dec.per_group()
    d5.record()
    barrier()
    grp_ms = max_over_ranks(d4.elapsed_time(d5) / KD)
    # the same step as two kernels (conv roll, then the state update alone), for comparison
    for _ in range(3):
        dec.conv(); dec.update()
    ev_u = _events(2 * KD)
    d2, d3 = _events(2)
    barrier()
    d2.record()
    for i in range(KD):
        dec.conv()
        ev_u[2 * i].record()
        dec.update()
        ev_u[2 * i + 1].record()
    d3.record()
    barrier()
    two_ms = max_over_ranks(d2.elapsed_time(d3) / KD)
    upd_ms = max_over_ranks(statistics.mean(ev_u[2 * i].elapsed_time(ev_u[2 * i + 1]) for i in range(KD)))
    del dec
    torch.cuda.empty_cache()

    # the backward pass of the scan on the 3B layer
    bwd = BackwardStep(BWD, shard.rank_seed(synth.config_seed(1), rank), dev)
    for _ in range(3):
        bwd()
    KB = max(3, min(20, K))
    b0, b1 = _events(2)
    barrier()
    b0.record()
    for _ in range(KB):
        bwd()
    b1.record()
    barrier()
    bwd_ms = max_over_ranks(b0.elapsed_time(b1) / KB)
    del bwd
    torch.cuda.empty_cache()

    # the whole mixer of the 3B layer, and its in_proj alone
    mx = MixerStep(MIXER, MIXER_D_MODEL, shard.rank_seed(synth.config_seed(1), rank), dev)
    KM = max(3, min(20, K))

    def time_fn(fn, n):
        for _ in range(3):
            fn()
        a0, a1 = _events(2)
        barrier()
        a0.record()
        for _ in range(n):
            fn()
        a1.record()
        barrier()
        return max_over_ranks(a0.elapsed_time(a1) / n)
    mix_ms = time_fn(mx, KM)
    lin_ms = time_fn(mx.in_proj, KM)
    del mx
    torch.cuda.empty_cache()

    # the ragged scan: the 3B layer's 16384 tokens as a mix of prompt
    # lengths, and as its own 8 equal sequences (against the dense call)
    rag = RaggedStep(RAGGED, shard.rank_seed(synth.config_seed(1), rank), dev)
    rag_ms = time_fn(rag, KM)
    rag_lens = rag.lens
    rag_status = int(rag.status.item())
    del rag
    req = RaggedStep(RAGGED, shard.rank_seed(synth.config_seed(1), rank), dev, lens=[RAGGED.L] * RAGGED.b)
    req_ms = time_fn(req, KM)
    del req
    torch.cuda.empty_cache()
    if rag_status != 0:
        raise RuntimeError(f"ragged scan reported status {rag_status}")

    if rank != 0:
        return None
    btok = BWD.b * BWD.L
    mtok = MIXER.b * MIXER.L
    rtok = RAGGED.b * RAGGED.L
    rbytes = scan_bytes_per_token(RAGGED) * rtok
    nproj = 2 * MIXER.H * MIXER.P + 2 * MIXER.G * MIXER.N + MIXER.H
    line = {
        "metric": METRIC,
        "value": shard.aggregate_tokens_per_s(tokens, world, ms_step),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(s),
        "roofline": head_roof,
        "scan_only": {"tokens_per_s": tokens / (scan_ms * 1e-3), "ms": scan_ms},
        "conv": blocks[s.name]["conv"],
        "prefill": blocks,
        "decode": {"workload": DECODE.name,
                   "kernel": "decode_step_head (conv-cache roll, conv + SiLU, state update: one launch, "
                             "one CTA per sequence and head, ssd_decode_step_ws)",
                   "ms_per_step": dec_ms,
                   "GB/s": decode_step_bytes(DECODE) / (dec_ms * 1e-3) / 1e9,
                   "frac_hbm": decode_step_bytes(DECODE) / (dec_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                   "tokens_per_s": world * DECODE.b / (dec_ms * 1e-3),
                   "per_group_kernel_ms_per_step": grp_ms,
                   "two_kernel_ms_per_step": two_ms, "state_update_ms": upd_ms,
                   "state_update_GB/s": decode_state_update_bytes(DECODE) / (upd_ms * 1e-3) / 1e9,
                   "state_update_frac_hbm": decode_state_update_bytes(DECODE) / (upd_ms * 1e-3) / 1e9 /
                                            peaks["hbm_gbs"]},
        "backward": {"workload": BWD.name,
                     "kernels": "chunk states (tcgen05), state passing, chunk gradients (tcgen05), head sums",
                     "ms": bwd_ms, "tokens_per_s": world * btok / (bwd_ms * 1e-3),
                     "GB/s": scan_bwd_bytes_per_token(BWD) * btok / (bwd_ms * 1e-3) / 1e9,
                     "frac_hbm": scan_bwd_bytes_per_token(BWD) * btok / (bwd_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "TFLOP/s": scan_bwd_flops_per_token(BWD) * btok / (bwd_ms * 1e-3) / 1e12,
                     "frac_bf16_peak": scan_bwd_flops_per_token(BWD) * btok / (bwd_ms * 1e-3) / 1e12 /
                                       peaks["bf16_tflops"]},
        "ragged": {"workload": f"{RAGGED.name} tokens as {len(rag_lens)} prompts of 64-4096 tokens "
                               "(seeded log-uniform mix)",
                   "kernel": "ssd_chunk_scan_fwd_varlen (preparation kernel + tensor-core scan, one head per item)",
                   "tokens": rtok, "nseq": len(rag_lens), "ms": rag_ms,
                   "tokens_per_s": world * rtok / (rag_ms * 1e-3),
                   "GB/s": rbytes / (rag_ms * 1e-3) / 1e9,
                   "frac_hbm": rbytes / (rag_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                   "equal_lengths_ms": req_ms,
                   "dense_scan_ms": blocks[RAGGED.name]["scan"]["launch_ms"]},
        "mixer": {"workload": MIXER.name, "d_model": MIXER_D_MODEL,
                  "kernels": "in_proj (tcgen05 linear), conv1d+SiLU, chunk scan, gated RMSNorm, out_proj",
                  "ms": mix_ms, "tokens_per_s": world * mtok / (mix_ms * 1e-3),
                  "TFLOP/s": mixer_flops(MIXER, MIXER_D_MODEL) / (mix_ms * 1e-3) / 1e12,
                  "frac_bf16_peak": mixer_flops(MIXER, MIXER_D_MODEL) / (mix_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                  "in_proj": {"M": mtok, "N": nproj, "K": MIXER_D_MODEL, "ms": lin_ms,
                              "TFLOP/s": linear_flops(mtok, nproj, MIXER_D_MODEL) / (lin_ms * 1e-3) / 1e12,
                              "frac_bf16_peak": linear_flops(mtok, nproj, MIXER_D_MODEL) / (lin_ms * 1e-3) / 1e12 /
                                                peaks["bf16_tflops"]}},
        "e2e": {"value": shard.aggregate_tokens_per_s(tokens, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pieces": npiece},
        "gpu_launches": 2 * K,   # conv + scan per timed prefill step
        "clocks": clocks,
    }
    return line


# ----------------------------------------------------------------------------
# the fp64 oracle on the host (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------

def oracle_sample(tokens: int = ORACLE_PREFIX):
    """One oracle prefill-layer call on the first `tokens` tokens of the
    headline workload (the same seeded inputs, cut to a prefix)."""
    import oracle
    s = PREFILL
    inp = synth.layer_inputs(s, synth.config_seed(HEADLINE))
    f = lambda t: None if t is None else t[:, :tokens].to(torch.float64).numpy()
    g = lambda t: None if t is None else t.to(torch.float64).numpy()
    args = (f(inp["xBC"]), g(inp["w"]), g(inp["bias"]), None, f(inp["dt_raw"]), g(inp["A"]),
            g(inp["dt_bias"]), g(inp["D"]), None, s.H, s.P, s.G, s.N)
    del inp
    threads = min(oracle.default_threads(), s.b * s.H)

    def run():
        t = time.perf_counter()
        oracle.layer_prefill(*args, nthreads=threads)
        return time.perf_counter() - t
    return s.b * tokens, run, threads


def cpu_baseline(min_seconds: float = 10.0, max_runs: int = 50):
    """The oracle on a 4096-token prefix of the headline workload, repeated
    until about `min_seconds` of CPU time have passed (a bounded sample: at
    most `max_runs` runs)."""
    ntok, run, threads = oracle_sample()
    run()  # warm (compile, page in)
    secs, runs = 0.0, 0
    while secs < min_seconds and runs < max_runs:
        secs += run()
        runs += 1
    return {"value": runs * ntok / secs, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{runs} runs of the first {ORACLE_PREFIX} of {PREFILL.L} tokens of the headline "
                      f"workload ({PREFILL.H} heads), conv1d+SiLU and token-by-token scan in fp64, "
                      f"{threads} threads",
            "seconds": secs}


def run_reference(args):
    ntok, run, threads = oracle_sample()
    for _ in range(args.warmup):
        run()
    secs = [run() for _ in range(args.steps)]
    total = sum(secs)
    v = args.steps * ntok / total
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(PREFILL),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: the fp64 oracle (conv1d+SiLU, token-by-token "
                                   f"recurrence) on the first {ORACLE_PREFIX} of the workload's "
                                   f"{PREFILL.L} tokens, {threads} threads"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_one_kernel(args, dev):
    """Launch one kernel of the bench workloads alone (for ncu captures)."""
    if args.kernel == "decode":
        fn = DecodeStep(DECODE, synth.config_seed(4), dev)
    elif args.kernel in ("mixer", "linear"):
        s = MIXER if args.seq_len is None else MIXER.with_(L=args.seq_len)
        mx = MixerStep(s, MIXER_D_MODEL, synth.config_seed(1), dev)
        fn = mx if args.kernel == "mixer" else mx.in_proj
    elif args.kernel == "bwd":
        s = BWD if args.seq_len is None else BWD.with_(L=args.seq_len)
        fn = BackwardStep(s, synth.config_seed(1), dev)
    elif args.kernel == "ragged":
        fn = RaggedStep(RAGGED, synth.config_seed(1), dev)
    else:
        s = synth.CONFIGS[args.workload]
        if args.seq_len is not None:
            s = s.with_(L=args.seq_len)
        st = PrefillStep(s, synth.config_seed(args.workload), dev)
        st.conv()
        fn = st.scan if args.kernel == "scan" else st.conv
    for _ in range(args.warmup):
        fn()
    e0, e1 = _events(2)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    workload = {"decode": DECODE.name, "mixer": MIXER.name, "linear": MIXER.name, "bwd": BWD.name,
                "ragged": RAGGED.name + " as a prompt-length mix"}.get(args.kernel, args.workload)
    print(json.dumps({"kernel": args.kernel, "workload": workload, "seq_len": args.seq_len,
                      "launches": args.steps, "ms_per_launch": e0.elapsed_time(e1) / args.steps}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=["scan", "conv", "decode", "bwd", "mixer", "linear", "ragged"],
                    help="launch only this kernel (warmup + steps launches) and print its mean "
                         "CUDA-event time; for profiler captures")
    ap.add_argument("--workload", type=int, choices=PREFILL_CONFIGS, default=HEADLINE,
                    help="prefill workload of --kernel scan|conv")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="--kernel only: a shorter sequence of the same workload (small captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    import datetime
    import torch.distributed as dist
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    from ssd_selective_scan_b200 import binding
    binding.load()
    if args.kernel:
        run_one_kernel(args, dev)
        return 0
    line = run_ours(args, rank, world, dev)
    if rank == 0:
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
