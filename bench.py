#!/usr/bin/env python3
"""Benchmark of the selective-scan forward on B200 (one JSON line on rank 0).

Default workload: the largest single-GPU configuration, the Mamba-2.8B-shaped long
sequence (batch 1, d_inner 5120, seqlen 65536, d_state 16, bf16 activations, fp32
state, softplus delta, D skip, z gate, final state). One pass = one
ssm_selective_scan_fwd call over one batch: softplus, discretisation, recurrence,
readout, gate (and, for workloads with a conv, the fused conv + SiLU).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long|m130|bidir|...]
                  [--passes-per-step P] [--impl ours|reference]

A bench step is P passes over P batches (P >= 1 chosen so that a step takes at least
25 ms, unless given), the inputs of successive passes alternating between two
input sets. Timing: W untimed steps, then K steps bracketed by a barrier and a
device synchronisation, timed with CUDA events on the launching stream; the max over
ranks is reported. Every scan pass streams more than the 126 MB L2 and no input set
is touched again before another set's bytes have gone through L2, so no flush is
inserted. Under torchrun every rank runs its own replica of the workload (the path
needs no exchange between GPUs): weak scaling.

`--impl reference` times the CPU oracle (double precision, single thread per
process) on a bounded sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mamba_selective_scan_sm_b200 import synth  # noqa: E402

METRIC = "selective-scan fwd B*D*L elems/s and achieved HBM GB/s vs B200 peak (1 GPU)"
L2_BYTES = 126 * 1024 * 1024
SFU_EX2_PER_CLK_PER_SM = 16      # MUFU.EX2 results per clock per SM (a standalone ex2 loop on B200)
FP32_LANES_PER_SM = 128          # FP32 FMA lanes per SM per clock (4 SMSPs x 32)
N_SM = 148


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="long", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--chunks", type=int, default=0, help="num_chunks passed to the scan (0 = auto)")
    ap.add_argument("--passes-per-step", type=int, default=0,
                    help="passes (one batch each) per bench step; 0 = enough for 25 ms")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's sequence length (a smaller case of the same "
                         "shape for profiler captures; the bench line names it)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ bytes --

def algorithmic_bytes(w) -> int:
    """Compulsory HBM bytes of one step: every input read once, every output written once."""
    es = 2 if w.dtype == "bf16" else 4
    if w.name.startswith("decode"):
        rows = w.batch * w.dim
        return (rows * w.dstate * 4 * 2          # state read + write
                + rows * 4 * es * 2              # conv state read + write
                + rows * es * 3                  # x, dt, z
                + rows * es                      # y
                + w.batch * w.dstate * es * 2    # B_t, C_t
                + w.dim * (w.dstate + 4 + 4) * 4)  # A, D, dt_bias, conv w/b
    rows = w.batch * w.dim
    L = w.seqlen
    if w.extra.get("conv_only"):                  # x read, y write, taps and bias
        return rows * L * es * 2 + w.dim * (w.conv_width + 1) * 4
    act = rows * L * es * 4                       # u (or x), delta, z read; y write
    bc = (w.dim * w.dstate * 4 * 2 if w.extra.get("bc_shared")       # B, C fixed per channel
          else w.batch * w.dstate * L * es * 2)   # B, C
    dirs = 2 if w.bidirectional else 1
    a_par = w.extra["a_heads"] if w.extra.get("a_heads") else w.dim * w.dstate
    params = (a_par + w.dim * 2) * 4 * dirs + (w.dim * (w.conv_width + 1) * 4 if w.conv_width else 0)
    fstate = rows * w.dstate * 4 * dirs if (w.final_state or w.bidirectional) else 0
    if "packed" in w.extra:                       # per sequence: final state, offsets
        nseq = len(synth.packed_lengths(L, *w.extra["packed"]))
        fstate = nseq * w.dim * w.dstate * 4 + (nseq + 1) * 4
    return act + bc + params + fstate


def exp_count(w) -> int:
    if w.extra.get("conv_only"):
        return w.batch * w.dim * w.seqlen         # one SiLU per output
    dirs = 2 if w.bidirectional else 1
    steps = max(w.seqlen, 1) * (w.steps if w.steps else 1)
    per_state = 1 if w.extra.get("a_heads") else w.dstate   # A per head: one exp per step
    return w.batch * w.dim * steps * per_state * dirs


def fp32_ops(w) -> int:
    """FP32 operations the recurrence cannot avoid: per state and step dBu = du * B,
    h = dA * h + dBu (one FMA) and the readout C * h (one FMA)."""
    dirs = 2 if w.bidirectional else 1
    return 3 * w.batch * w.dim * max(w.seqlen, 1) * w.dstate * dirs


# ---------------------------------------------------------------- traffic --

# each family: its kernel, the shared device headers, its launcher and the host code
# that picks its variant (all of which decide what the captured launch did)
KERNEL_SOURCES = {
    "scan": ("scan_kernel.cuh", "device_common.cuh", "scan_params.h", "scan_launch.cuh",
             "scan_variants.h", "scan_bf16.cu", "scan_f32.cu", "scan_bf16_ext.cu",
             "scan_f32_ext.cu", "scan_bf16_m2.cu", "scan_f32_m2.cu", "kernels.cu", "ssm_api.cu"),
    "decode": ("decode_kernel.cuh", "device_common.cuh", "scan_params.h", "kernels.cu",
               "ssm_api.cu"),
    "conv": ("conv_kernel.cuh", "device_common.cuh", "scan_params.h", "kernels.cu",
             "ssm_api.cu"),
}


def kernel_source_digest(kind: str) -> str:
    """sha256 over the CUDA sources of one kernel family (what an ncu capture describes)."""
    import hashlib
    d = os.path.join(ROOT, "mamba_selective_scan_sm_b200", "csrc")
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")


def recorded_traffic(key, path=TRAFFIC_JSON):
    """DRAM bytes (read + write) per pass of workload `key`'s dominant kernel, from the
    committed ncu capture record, if that capture was taken of the current sources;
    else None."""
    try:
        with open(path) as f:
            rows = json.load(f)["rows"]
    except (OSError, ValueError, KeyError):
        return None
    kind = "decode" if key.startswith("decode") else ("conv" if key == "conv" else "scan")
    digest = kernel_source_digest(kind)
    for r in rows:
        if r.get("workload") == key and r.get("sources_sha256") == digest:
            try:
                return float(r["bytes"])
            except (KeyError, TypeError, ValueError):
                return None
    return None


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs. start() returns
    once the first sample has arrived (or after a few seconds), so that the sampler is
    running when the timed region begins."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.reader = None

    def start(self, wait_s: float = 3.0):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        first = threading.Event()

        def read():
            for line in self.proc.stdout:
                self.lines.append((time.perf_counter(), line))
                first.set()
        self.reader = threading.Thread(target=read, daemon=True)
        self.reader.start()
        first.wait(wait_s)

    def stop(self, window=None):
        """Median SM clock and throttle reasons over the samples that arrived inside
        `window` (perf_counter seconds; all samples if none did), with their count."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.reader is not None:
            self.reader.join(timeout=5)
        rows = []
        inside = [ln for t, ln in self.lines if window and window[0] <= t <= window[1]]
        for line in inside or [ln for _, ln in self.lines]:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), max=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                            ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": rows[0]["max"],
                "reasons": sorted(reasons), "samples": len(self.lines),
                "samples_under_load": len(inside),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------- workload --

class ScanWorkload:
    """A scan workload: one pass is one ssm_selective_scan_fwd call over one batch.

    Device inputs come in SETS independent copies and successive passes alternate
    between them (each set is its own batch of the same shape), so a pass never finds
    the previous pass's inputs in L2."""

    SETS = 2

    def __init__(self, w, device, chunks):
        import torch
        self.w = w
        self.torch = torch
        self.device = device
        self.chunks = chunks
        inp = synth.scan_inputs(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, w.conv_width,
                                w.bidirectional, seed=0, a_heads=w.extra.get("a_heads", 0),
                                bc_shared=bool(w.extra.get("bc_shared")))
        self.host_inp = inp
        self.tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        par = lambda k: torch.from_numpy(inp[k]).to(device) if inp.get(k) is not None else None
        self.p = {k: par(k) for k in ("A", "D", "delta_bias", "conv_w", "conv_b", "A_rev", "D_rev",
                                      "delta_bias_rev")}
        self.cl = bool(w.extra.get("channel_last"))
        first = self._make_set(inp)
        self.sets = [first] + [self._clone_set(first) for _ in range(self.SETS - 1)]
        self.base, self.t, self.out = self.sets[0]
        self.k = 0
        self.starts = None
        rows = w.batch
        if "packed" in w.extra:
            lens = synth.packed_lengths(w.seqlen, *w.extra["packed"])
            st = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
            self.starts = torch.from_numpy(st).to(device)
            rows = len(lens)
        shp = (rows, w.dim, w.dstate)
        self.fs = torch.empty(shp, device=device) if (w.final_state or w.bidirectional) else None
        self.fsr = torch.empty(shp, device=device) if w.bidirectional else None
        import mamba_selective_scan_sm_b200 as ssm
        self.ssm = ssm
        n = ssm.ssm_selective_scan_workspace_size(self.t["u"], self.p["A"],
                                                  conv_weight=self.p["conv_w"] if w.conv_width else None,
                                                  A_rev=self.p["A_rev"], num_chunks=chunks,
                                                  seq_starts=self.starts, channel_last=self.cl,
                                                  dstate=w.dstate,
                                                  bc_shared=bool(w.extra.get("bc_shared")))
        self.ws = torch.empty(max(n, 1), dtype=torch.uint8, device=device)
        # a two-pass carry (asked for, or chosen for a small grid) adds the summary launch
        self.launches_per_pass = 2 if (n > 0 and not w.bidirectional) else 1
        self.h = None          # pinned host buffers of the end-to-end measurement

    def _views(self, base):
        """The scan's tensors (views) of one set's base tensors."""
        if not self.cl:
            return dict(base)
        D, N, R = self.w.dim, self.w.dstate, self.w.extra["dt_rank"]
        xz, xdbl = base["xz"], base["xdbl"]
        return {"u": xz[..., :D], "z": xz[..., D:], "delta": base["dt"],
                "B": xdbl[..., R:R + N], "C": xdbl[..., R + N:]}

    def _make_set(self, inp):
        torch, w = self.torch, self.w
        act = lambda k: torch.from_numpy(inp[k]).to(self.device).to(self.tdt)
        if self.cl:
            # the Mamba block's own tensors: x and z are the two halves of the in_proj
            # output, B and C columns of the x_proj output (after its dt_rank columns)
            B, D, L, N, R = w.batch, w.dim, w.seqlen, w.dstate, w.extra["dt_rank"]
            cl = lambda k: act(k).transpose(1, 2)
            xz = torch.cat([cl("u"), cl("z")], dim=2).contiguous()
            xdbl = torch.zeros(B, L, R + 2 * N, dtype=self.tdt, device=self.device)
            xdbl[..., R:R + N] = cl("B")
            xdbl[..., R + N:] = cl("C")
            base = {"xz": xz, "xdbl": xdbl, "dt": cl("delta").contiguous()}
            out = torch.empty(B, L, D, dtype=self.tdt, device=self.device)
        else:
            base = {k: act(k) for k in ("u", "delta", "z", "B", "C")}
            out = torch.empty_like(base["u"])
        return base, self._views(base), out

    def _clone_set(self, s):
        base = {k: v.clone() for k, v in s[0].items()}
        return base, self._views(base), self.torch.empty_like(s[2])

    def launch(self, t, out):
        w, p = self.w, self.p
        conv = w.conv_width > 0
        self.ssm.ssm_selective_scan_fwd(
            t["u"], t["delta"], p["A"], t["B"], t["C"], p["D"], t["z"], p["delta_bias"], True,
            False, p["conv_w"] if conv else None, p["conv_b"] if conv else None, p["A_rev"],
            p["D_rev"], p["delta_bias_rev"], out=out, num_chunks=self.chunks,
            workspace=self.ws, final_state=self.fs, final_state_rev=self.fsr,
            seq_starts=self.starts, channel_last=self.cl)

    def unit(self):
        """One pass over the next input set."""
        _, t, out = self.sets[self.k % self.SETS]
        self.k += 1
        self.launch(t, out)

    def e2e_setup(self):
        torch = self.torch
        # the tensors a caller hands over (channel-last: the projection outputs whole)
        self.h = {k: v.cpu().pin_memory() for k, v in self.base.items()}
        self.hout = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
                     for _ in range(self.SETS)]
        self.h2d = sum(v.numel() * v.element_size() for v in self.h.values())
        self.d2h = self.hout[0].numel() * self.hout[0].element_size()
        self.s_h2d, self.s_d2h = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_serial(self):
        """Upload one batch, scan it, read the result back, all on the current stream."""
        base, t, out = self.sets[0]
        for k, v in self.h.items():
            base[k].copy_(v, non_blocking=True)
        self.launch(t, out)
        self.hout[0].copy_(out, non_blocking=True)

    def e2e_pipelined(self, n):
        """n batches: batch i's upload (copy stream), scan (current stream) and read-back
        (second copy stream) overlap the neighbouring batches' through the two sets."""
        torch = self.torch
        cur = torch.cuda.current_stream()
        Event = lambda: torch.cuda.Event()
        up = [Event() for _ in range(n)]
        done = [Event() for _ in range(n)]
        back = [Event() for _ in range(n)]
        for i in range(n):
            base, t, out = self.sets[i % self.SETS]
            with torch.cuda.stream(self.s_h2d):
                if i >= self.SETS:                  # the set's previous scan has read it
                    self.s_h2d.wait_event(done[i - self.SETS])
                for k, v in self.h.items():
                    base[k].copy_(v, non_blocking=True)
                up[i].record(self.s_h2d)
            cur.wait_event(up[i])
            if i >= self.SETS:                      # the set's previous result is back
                cur.wait_event(back[i - self.SETS])
            self.launch(t, out)
            done[i].record(cur)
            with torch.cuda.stream(self.s_d2h):
                self.s_d2h.wait_event(done[i])
                self.hout[i % self.SETS].copy_(out, non_blocking=True)
                back[i].record(self.s_d2h)
        cur.wait_event(back[n - 1])
        cur.wait_stream(self.s_h2d)

    def elems(self):
        return self.w.batch * self.w.dim * self.w.seqlen


class ConvWorkload:
    """The standalone causal conv1d + SiLU (ssm_causal_conv1d_fwd) on the m130 shape.

    One launch's 100 MB (x read, y written) would fit the 126 MB L2, so launches rotate
    over SETS independent input/output pairs: a launch's tensors were last touched SETS - 1
    launches earlier, with ~200 MB of other traffic in between. A launch (~21 us) is
    shorter than the binding's host-side call and than the gap between two graph
    replays, so one CUDA graph holds REP launches cycling over the sets and a pass replays
    it: REP batches per pass (the end-to-end leg calls the binding itself)."""

    SETS = 3
    REP = 30

    def __init__(self, w, device):
        import torch
        import mamba_selective_scan_sm_b200 as ssm
        self.w, self.torch, self.ssm = w, torch, ssm
        inp = synth.scan_inputs(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, w.conv_width, seed=0)
        self.host_inp = inp
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        x = torch.from_numpy(inp["u"]).to(device).to(tdt)
        self.xs = [x.clone() for _ in range(self.SETS)]
        self.outs = [torch.empty_like(x) for _ in range(self.SETS)]
        self.x, self.out = self.xs[0], self.outs[0]
        self.cw = torch.from_numpy(inp["conv_w"]).to(device)
        self.cb = torch.from_numpy(inp["conv_b"]).to(device)
        self.k = 0
        self.launches_per_pass = self.REP
        self.h = None
        self.launch(0)                                  # load the kernel outside the capture
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side), torch.cuda.graph(self.graph, stream=side):
            for i in range(self.REP):
                self.launch(i % self.SETS)
        torch.cuda.current_stream().wait_stream(side)

    def launch(self, i):
        self.ssm.ssm_causal_conv1d_fwd(self.xs[i], self.cw, self.cb, True, out=self.outs[i])

    def unit(self):
        self.graph.replay()

    def e2e_setup(self):
        self.h = self.x.cpu().pin_memory()
        self.hout = self.torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d = self.h.numel() * self.h.element_size()
        self.d2h = self.hout.numel() * self.hout.element_size()

    def e2e_serial(self):
        i = self.k % self.SETS
        self.k += 1
        self.xs[i].copy_(self.h, non_blocking=True)
        self.launch(i)
        self.hout.copy_(self.outs[i], non_blocking=True)

    e2e_pipelined = None
    batches_per_unit = REP                            # e2e_serial moves one batch

    def elems(self):
        return self.REP * self.w.batch * self.w.dim * self.w.seqlen


class DecodeWorkload:
    """The decode configuration: 64 successive single-token updates of every (b, d) row.

    One bench step replays a CUDA graph of the 64 token launches (no host launch
    overhead between tokens). The state of one layer (at B256 D5120 N16: 84 MB fp32 + 10.5
    MB conv state) would fit the 126 MB L2, so the tokens rotate over LAYERS independent state
    buffers (one per layer of a model): a token's state was last touched LAYERS - 1
    launches earlier, and ~190 MB of other traffic has gone through L2 since."""

    LAYERS = 3

    def __init__(self, w, device):
        import torch
        import mamba_selective_scan_sm_b200 as ssm
        self.w, self.torch, self.ssm = w, torch, ssm
        inp = synth.decode_inputs(w.batch, w.dim, w.dstate, w.steps, 4, w.dtype, seed=0,
                                  a_heads=w.extra.get("a_heads", 0))
        self.host_inp = inp
        bf = torch.bfloat16
        st = torch.from_numpy(inp["state"]).to(device)
        cs = torch.from_numpy(inp["conv_state"]).to(device).to(bf)
        self.states = [st.clone() for _ in range(self.LAYERS)]
        self.css = [cs.clone() for _ in range(self.LAYERS)]
        self.seq = {k: torch.from_numpy(inp[k]).to(device).to(bf) for k in ("x", "dt", "z", "B", "C")}
        self.p = {k: torch.from_numpy(inp[k]).to(device) for k in ("A", "D", "dt_bias", "conv_w", "conv_b")}
        self.outs = torch.empty(w.steps, w.batch, w.dim, dtype=bf, device=device)
        self.launches_per_pass = w.steps
        self.h = None
        self.tokens()                                   # load the kernels outside the capture
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side), torch.cuda.graph(self.graph, stream=side):
            self.tokens()
        torch.cuda.current_stream().wait_stream(side)

    def tokens(self):
        q, p = self.seq, self.p
        for s in range(self.w.steps):
            layer = s % self.LAYERS
            self.ssm.ssm_selective_state_update(self.states[layer], self.css[layer], q["x"][s],
                                                q["dt"][s], p["A"], q["B"][s], q["C"][s], p["D"],
                                                q["z"][s], p["dt_bias"], True, p["conv_w"],
                                                p["conv_b"], out=self.outs[s])

    def unit(self):
        self.graph.replay()

    def e2e_setup(self):
        torch = self.torch
        self.h = {k: v.cpu().pin_memory() for k, v in self.seq.items()}
        self.hout = torch.empty(self.outs.shape, dtype=self.outs.dtype).pin_memory()
        self.h2d = sum(v.numel() * v.element_size() for v in self.h.values())
        self.d2h = self.hout.numel() * self.hout.element_size()

    def e2e_serial(self):
        for k, v in self.h.items():
            self.seq[k].copy_(v, non_blocking=True)
        self.unit()
        self.hout.copy_(self.outs, non_blocking=True)

    e2e_pipelined = None

    def elems(self):
        return self.w.batch * self.w.dim * self.w.steps


# ------------------------------------------------------------ cpu oracle --

def oracle_sample(w, seconds=10.0):
    """Time the CPU oracle on a bounded sample of the workload; returns (elems/s, desc, cores)."""
    import oracle
    if w.name.startswith("decode"):
        inp = synth.decode_inputs(1, 256, w.dstate, 4, 4, w.dtype, seed=0,
                                  a_heads=4 if w.extra.get("a_heads") else 0)
        t0 = time.perf_counter()
        n = 0
        st, cs = inp["state"], inp["conv_state"]
        while time.perf_counter() - t0 < seconds:
            for s in range(4):
                _, st, cs = oracle.state_update(st, cs, inp["x"][s], inp["dt"][s], inp["A"],
                                                inp["B"][s], inp["C"][s], inp["D"], inp["z"][s],
                                                inp["dt_bias"], True, inp["conv_w"], inp["conv_b"])
                n += 256
        dt = time.perf_counter() - t0
        return n / dt, f"{n} single-token channel updates (batch 1, d_inner 256) of the decode workload", 1
    if w.extra.get("conv_only"):
        inp = synth.scan_inputs(1, 64, w.seqlen, w.dstate, w.dtype, w.conv_width, seed=0)
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < seconds:
            oracle.causal_conv1d(inp["u"], inp["conv_w"], inp["conv_b"], True)
            n += 64 * w.seqlen
        dt = time.perf_counter() - t0
        return n / dt, f"{n // w.seqlen} channels x seqlen {w.seqlen} of the {w.name} workload", 1
    chans_per_call = 16
    # A per head: the sample's 16 channels form one head
    inp = synth.scan_inputs(1, chans_per_call, w.seqlen, w.dstate, w.dtype, w.conv_width,
                            w.bidirectional, seed=0, a_heads=1 if w.extra.get("a_heads") else 0,
                            bc_shared=bool(w.extra.get("bc_shared")))
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.scan_channels(inp, [(0, d) for d in range(chans_per_call)], conv=w.conv_width > 0,
                             bidirectional=w.bidirectional)
        n += chans_per_call * w.seqlen
        if time.perf_counter() - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    return n / dt, (f"{n // w.seqlen} channels x seqlen {w.seqlen} of the {w.name} workload "
                    f"({n} elements, {dt:.1f} s)"), 1


# -------------------------------------------------------------------- main --

def _oracle_worker(job):
    """One process of the all-core oracle timing: the single-threaded sample."""
    key, seconds = job
    return oracle_sample(synth.WORKLOADS[key], seconds)


class OraclePool:
    """The oracle on every host core: one spawned process per core, each timing the
    single-threaded oracle on its own channels for the same window; the throughputs
    add up. (Spawned, not forked: the parent may already hold a CUDA context.)"""

    def __init__(self):
        import multiprocessing
        self.cores = len(os.sched_getaffinity(0))
        self.pool = multiprocessing.get_context("spawn").Pool(self.cores)

    def sample(self, key, seconds):
        res = self.pool.map(_oracle_worker, [(key, seconds)] * self.cores)
        value = sum(r[0] for r in res)
        return value, f"{res[0][1]}, on each of {self.cores} processes", self.cores

    def close(self):
        self.pool.close()
        self.pool.join()


def run_reference(args, w, rank):
    if rank != 0:
        return
    # each step a bounded sample: the whole run stays near a minute of host time
    per_step = min(2.0, max(0.2, 60.0 / max(args.steps + args.warmup, 1)))
    pool = OraclePool()
    steps_v = []
    for _ in range(args.warmup):
        pool.sample(args.workload, per_step)
    t_all = time.perf_counter()
    for _ in range(args.steps):
        v, desc, cores = pool.sample(args.workload, per_step)
        steps_v.append(v)
    wall = time.perf_counter() - t_all
    pool.close()
    value = statistics.median(steps_v)
    line = {
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": "elems/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": wall / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args),
        "cpu_baseline": {"value": value, "unit": "elems/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "elems/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


STEP_MIN_MS = 25.0


def passes_for(pass_ms, min_ms=STEP_MIN_MS):
    """Passes per bench step so that a step lasts at least min_ms (at least one)."""
    if pass_ms <= 0:
        return 1
    return max(1, int(-(-min_ms // pass_ms)))


def config_of(w, args, passes=1):
    c = {"workload": w.name, "batch": w.batch, "d_inner": w.dim, "seqlen": w.seqlen,
         "d_state": w.dstate, "conv_width": w.conv_width, "bidirectional": w.bidirectional,
         "final_state": w.final_state, "parallelism": f"replicas x{args.gpus}",
         "passes_per_step": passes,
         "step": (f"{passes} pass(es), each one call over one batch of the shape above; "
                  "successive passes alternate between two input sets")}
    if w.steps:
        c["tokens_per_step"] = w.steps
        c["launch"] = f"one CUDA graph of {w.steps} token launches per step"
    ab = algorithmic_bytes(w)
    if w.extra.get("conv_only"):
        c["l2"] = (f"launches rotate over {ConvWorkload.SETS} input/output pairs "
                   f"({ConvWorkload.SETS * ab / 1e6:.0f} MB > 126 MB L2)")
        c["launch"] = (f"one CUDA graph of {ConvWorkload.REP} launches per pass, "
                       f"each one batch of the shape above")
    elif w.name.startswith("decode"):
        es = 2 if w.dtype == "bf16" else 4
        layer_mb = w.batch * w.dim * (w.dstate * 4 + w.conv_width * es) / 1e6   # SSM + conv state
        c["l2"] = (f"state rotated over {DecodeWorkload.LAYERS} layers "
                   f"({DecodeWorkload.LAYERS * layer_mb:.0f} MB of state > 126 MB L2): no step "
                   "finds its state in L2")
    else:
        c["l2"] = ("inputs larger than L2 ({:.0f} MB/step > 126 MB)".format(ab / 1e6)
                   if ab > L2_BYTES else "working set {:.0f} MB/step fits L2: L2-warm".format(ab / 1e6))
    if args.chunks:
        c["num_chunks"] = args.chunks
    if "packed" in w.extra:
        c["sequences"] = len(synth.packed_lengths(w.seqlen, *w.extra["packed"]))
    if w.extra.get("channel_last"):
        c["layout"] = (f"channel-last views: u, z of one (B, L, {2 * w.dim}) tensor, B, C of one "
                       f"(B, L, {w.extra['dt_rank'] + 2 * w.dstate}) tensor")
    return c


# ------------------------------------------------------------- replicas --
# Every rank runs its own replica of the workload (the path needs no exchange between
# GPUs); the host logic below is what ties the ranks together, and the CPU tests run it
# under gloo.

def init_ranks(backend, device=None, timeout_s=120):
    """Join the process group (RANK / WORLD_SIZE / MASTER_* from the environment) when
    more than one rank runs; returns the world size."""
    import datetime
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 and not dist.is_initialized():
        kw = {"device_id": device} if device is not None and backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world


def max_over_ranks(value, device):
    """The largest of every rank's value (each rank's timed region ends when its last
    step does: the job's time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms):
    """Whole-job throughput: the units all ranks processed over the job's time."""
    return units_per_rank * world / (ms * 1e-3)


def leave_ranks():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


def workload_of(args):
    """The named workload, with the sequence length overridden if asked."""
    import dataclasses
    w = synth.WORKLOADS[args.workload]
    if args.seqlen and not w.name.startswith("decode"):
        w = dataclasses.replace(w, seqlen=args.seqlen,
                                name=f"{w.name} (seqlen overridden: {args.seqlen})")
    return w


def main():
    args = parse()
    w = workload_of(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    world = init_ranks("nccl", device)

    if w.name.startswith("decode"):
        wl = DecodeWorkload(w, device)
    elif w.extra.get("conv_only"):
        wl = ConvWorkload(w, device)
    else:
        wl = ScanWorkload(w, device, args.chunks)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # passes per bench step: enough for 25 ms (the same number on every rank)
    for _ in range(2):
        wl.unit()
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(3):
        wl.unit()
    c1.record(stream)
    torch.cuda.synchronize()
    passes = args.passes_per_step or passes_for(c0.elapsed_time(c1) / 3, STEP_MIN_MS)
    passes = int(max_over_ranks(passes, device))

    def step():
        for _ in range(passes):
            wl.unit()

    for _ in range(max(args.warmup, 3)):
        step()
    barrier()

    # per-step timing of the step's launches, for the roofline
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    w0 = time.perf_counter()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        ev[2 * i].record(stream)
        step()
        ev[2 * i + 1].record(stream)
    t1.record(stream)
    barrier()
    clocks = sampler.stop((w0, time.perf_counter()))
    ms_total = t0.elapsed_time(t1)
    per_pass = [ev[2 * i].elapsed_time(ev[2 * i + 1]) / passes for i in range(args.steps)]
    ms_total = max_over_ranks(ms_total, device)
    ms_step = ms_total / args.steps
    elems = wl.elems() * passes
    value = job_throughput(elems, world, ms_step)

    # end to end through the public binding: every batch's inputs uploaded from pinned
    # host memory, scanned, its result read back; a step is the same `passes` batches
    e2e = None
    if not args.no_e2e:
        wl.e2e_setup()

        def timed(fn, reps):
            fn()
            barrier()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            barrier()
            return max_over_ranks(a.elapsed_time(b) / reps, device)

        k = max(3, min(args.steps, 10))
        ms_serial = timed(wl.e2e_serial, k)        # per batch
        bpu = getattr(wl, "batches_per_unit", 1)   # batches one pass of the device leg holds
        batch_elems = wl.elems() // bpu
        e2e = {"unit": "elems/s", "h2d_bytes_per_step": wl.h2d * passes * bpu,
               "d2h_bytes_per_step": wl.d2h * passes * bpu}
        serial = {"value": job_throughput(batch_elems, world, ms_serial), "ms_per_batch": ms_serial,
                  "how": "upload, scan and read-back of one batch back to back on one stream"}
        if wl.e2e_pipelined is not None:
            nb = max(4, k)
            ms_pipe = timed(lambda: wl.e2e_pipelined(nb), 1) / nb
            e2e.update(value=job_throughput(batch_elems, world, ms_pipe), ms_per_step=ms_pipe * passes * bpu,
                       ms_per_batch=ms_pipe,
                       how=(f"{nb} batches: uploads on one copy stream, scans on the compute "
                            "stream, read-backs on a second copy stream, two device input sets"),
                       serial=serial)
        else:
            e2e.update(value=serial["value"], ms_per_step=ms_serial * passes * bpu,
                       ms_per_batch=ms_serial, how=serial["how"])

    if rank == 0:
        hbm_peak, peak_kind = measured_peaks()
        ab = algorithmic_bytes(w)
        # a decode or conv pass is a graph of back-to-back launches of one kernel
        mean_launch_ms = statistics.mean(per_pass) / (
            wl.launches_per_pass if (w.name.startswith("decode") or w.extra.get("conv_only")) else 1)
        achieved = ab / (mean_launch_ms * 1e-3) / 1e9
        sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
        exps = exp_count(w) / (w.steps if w.steps else 1) if w.name.startswith("decode") else exp_count(w)
        sfu_peak = N_SM * SFU_EX2_PER_CLK_PER_SM * sm_mhz * 1e6
        sfu_ach = exps / (mean_launch_ms * 1e-3)
        hbm = {"achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
               "peak_kind": f"{peak_kind} HBM copy bandwidth",
               "algorithmic_bytes_per_launch": ab}
        sfu = {"achieved": sfu_ach / 1e9, "peak": sfu_peak / 1e9, "unit": "Gex2/s",
               "frac": sfu_ach / sfu_peak, "exp2_per_launch": exps,
               "peak_kind": (f"{N_SM} SMs x {SFU_EX2_PER_CLK_PER_SM} ex2/clk/SM (measured) x "
                             f"{sm_mhz:.0f} MHz (sampled SM clock)")}
        traffic = None if args.seqlen else recorded_traffic(args.workload)
        if w.name.startswith("decode") or w.extra.get("conv_only"):
            roof = dict(bound="hbm", **{k: hbm[k] for k in ("achieved", "peak", "unit", "frac")},
                        traffic=traffic, peak_kind=hbm["peak_kind"],
                        algorithmic_bytes_per_launch=ab, mean_launch_ms=mean_launch_ms, sfu=sfu)
        elif w.extra.get("a_heads"):
            # A per head: one exp per (b, d, l); the floor is the FP32 pipe, three
            # operations per (b, d, l, n), 128 lanes per SM per clock
            ops = fp32_ops(w)
            fp_peak = N_SM * FP32_LANES_PER_SM * sm_mhz * 1e6
            fp_ach = ops / (mean_launch_ms * 1e-3)
            roof = dict(bound="alu", achieved=fp_ach / 1e12, peak=fp_peak / 1e12, unit="Tops/s",
                        frac=fp_ach / fp_peak, traffic=traffic,
                        peak_kind=(f"{N_SM} SMs x {FP32_LANES_PER_SM} FP32 lanes x {sm_mhz:.0f} MHz "
                                   "(sampled SM clock)"),
                        fp32_ops_per_launch=ops, mean_launch_ms=mean_launch_ms, hbm=hbm, sfu=sfu)
        else:
            # one exp per (b, d, l, n) is the binding roof at d_state 16; HBM alongside
            roof = dict(bound="alu", **{k: sfu[k] for k in ("achieved", "peak", "unit", "frac")},
                        traffic=traffic, peak_kind=sfu["peak_kind"],
                        exp2_per_launch=exps, mean_launch_ms=mean_launch_ms, hbm=hbm)
        line = {
            "metric": METRIC,
            "value": value, "unit": "elems/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded; value distributions of the Mamba init)",
            "config": config_of(w, args, passes),
            "roofline": roof,
            "hbm_gbs": achieved,
            "e2e": e2e,
            "gpu_launches": args.steps * passes * wl.launches_per_pass,
            "clocks": clocks,
        }
        if not args.no_cpu_baseline and world == 1:
            v1, desc1, _ = oracle_sample(w, seconds=10.0)
            pool = OraclePool()
            pool.sample(args.workload, 1.0)                 # workers warm
            v, desc, cores = pool.sample(args.workload, 10.0)
            pool.close()
            line["cpu_baseline"] = {"value": v, "unit": "elems/s", "cores": cores,
                                    "kind": "oracle", "sample": desc,
                                    "single_core": {"value": v1, "cores": 1, "sample": desc1}}
        print(json.dumps(line), flush=True)
    leave_ranks()


if __name__ == "__main__":
    main()
