#!/usr/bin/env python
"""Benchmark of the R-SWA / SR-SWA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl ours|reference]

A step is one decode step of the whole batch through the C ABI:
  configs 1, 2 (R-SWA):   rswa_decode_append (ring append fused into the decode)
  configs 4, 5 (SR-SWA):  srswa_step (ring append, router and gathered attention in
                          one launch; --unfused: rswa_append + srswa_route + srswa_decode)
  configs 6, 7:           configs 2 and 4 over an FP8 (E4M3) prefix, quantised
                          once before timing: rswa_append + rswa_decode_fp8
                          (+ srswa_route + srswa_decode_fp8)
  config 8 (SR-SWA chunked prefill): srswa_route_tokens + srswa_prefill (grouping by
                          routed block set, band part and routed part on tcgen05)
  config 9 (page2d rotary encoding of a prefill chunk's q and k): rswa_rope_page2d
  config 10:              config 4 with the page2d encoding of q and k_new inside the
                          same launch: srswa_step_rope (--unfused: rswa_append_rope +
                          srswa_route + srswa_decode)
  config 13:              config 2 with the page2d encoding inside the fused step:
                          rswa_decode_append_rope
  configs 11, 12:         configs 6 and 7 with an FP8 ring as well: rswa_append_fp8 +
                          rswa_decode_fp8kv (+ srswa_route + srswa_decode_fp8kv)
(the router's block index keys are pooled once per prefix, before timing).
The default workload is the batched R-SWA decode: 512 sequences, 16 heads,
head_dim 128, a 10-page prefix (2560 visual + 32 prompt tokens) and a full
128-slot ring with write pointers uniform in [0, 128).

The K timed steps are captured in one CUDA graph and replayed once (after W
eager warm-up steps and one untimed replay); CUDA events with external
record nodes bracket the attention (and route) kernel launches of every 8th
step inside the graph, so the kernels' average durations are measured on
their own stream inside the timed region (an event node adds several
microseconds to the step it sits in, so bracketing every step would slow the
step being timed; the sampled steps' extra time stays in the step time).
Inputs (the prefix K/V) are larger than L2, so no flush is needed between
steps. Under torchrun every rank runs its own batch (weak scaling,
no data-path collective); the timing is the max over ranks.

--impl reference runs the CPU oracle (test infrastructure, fp64) on a bounded
sample of each step's sequences on the host cores and reports the same
metric, extrapolated from the sample.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode attn steps/s & achieved HBM GB/s (fraction of peak) on 1 B200"
FALLBACK_HBM_GBS = 6650.0
EVENT_EVERY = 8  # kernel durations are bracketed with CUDA events in every 8th timed step
TIMING_NOTE = (f"K steps in one CUDA graph replay timed by CUDA events (ms_per_step); kernel durations from event "
               f"brackets around the kernels of every {EVENT_EVERY}th step (avg_launch_us): an event node between "
               "two kernels also ends programmatic dependent launch there, so a bracket includes the launch gap "
               "that the un-bracketed steps hide, and a one-kernel step's bracket can exceed ms_per_step")


# ----------------------------------------------------------------------------- workloads

def workload(cfg: int) -> dict:
    from long_context_decode_swa_b200 import synth
    if cfg == 1:
        m = synth.ocr_prefix_len(1)
        return dict(kind="rswa", B=1, H=16, D=128, n=128, plen=[m], cap=m, wp0=37,
                    name="R-SWA decode, 1 sequence, 16 heads, head_dim 128, prefix 288 (256 visual + 32 prompt), "
                         "full 128-slot ring from slot 37")
    if cfg == 2:
        m = synth.ocr_prefix_len(10)
        return dict(kind="rswa", B=512, H=16, D=128, n=128, plen=[m] * 512, cap=m, wp0=None,
                    name="R-SWA batched decode, 512 sequences, 16 heads, head_dim 128, prefix 2592 "
                         "(10 pages x 256 visual + 32 prompt), full 128-slot ring, wp ~ U[0,128)")
    if cfg == 3:
        m = synth.ocr_prefix_len(40)
        return dict(kind="prefill", B=4, H=16, D=128, n=128, plen=[m] * 4, cap=m, T=4096, wp0=None,
                    name="R-SWA chunked prefill, 4 sequences, 16 heads, head_dim 128, prefix 10272 (40 pages x 256 "
                         "visual + 32 prompt), 4096 output-side queries, causal band 128")
    if cfg == 4:
        return dict(kind="srswa", B=64, H=16, D=128, n=128, plen=[32768] * 64, cap=32768, wp0=None,
                    name="SR-SWA decode, 64 sequences, 16 heads, head_dim 128, 32768-token history (1024 blocks "
                         "of 32), index dim 32, 1.5-entmax top-16 + log-prob bias, full 128-slot ring")
    if cfg == 5:
        pages = synth.log_uniform_pages(16, 32, 400, seed=5005)
        plen = [256 * p for p in pages]
        return dict(kind="srswa", B=16, H=16, D=128, n=128, plen=plen, cap=102400, wp0=None,
                    name="SR-SWA long-horizon decode, 16 sequences, 16 heads, head_dim 128, ragged histories "
                         "8192-102400 tokens (log-uniform pages x 256), top-16 blocks + 128-slot ring")
    if cfg == 8:
        return dict(kind="srswa_prefill", B=4, H=16, D=128, n=128, plen=[32768] * 4, cap=32768, T=4096, wp0=None,
                    name="SR-SWA chunked prefill, 4 sequences, 16 heads, head_dim 128, 32768-token history (1024 "
                         "blocks), 4096 output-side queries each routed to its own top-16 blocks (planted, 32 "
                         "directions cycled over the tokens) + causal band 128")
    if cfg == 9:
        return dict(kind="rope", B=4, H=16, D=128, n=128, plen=[0] * 4, cap=0, T=4096, wp0=None,
                    name="page2d rotary encoding of a prefill chunk, 4 sequences x 4096 tokens, 16 heads, head_dim "
                         "128, q and k (bf16 in, bf16 out), tokens on pages of 200-2000 tokens, base 10000, page_mod 2")
    if cfg == 10:
        w = workload(4)
        w["rope"] = True
        w["name"] += "; page2d rotary encoding of q and the new key inside the same launch (srswa_step_rope)"
        return w
    if cfg == 13:
        w = workload(2)
        w["rope"] = True
        w["name"] += "; page2d rotary encoding of q and the new key inside the fused step (rswa_decode_append_rope)"
        return w
    if cfg in (11, 12):  # configs 6 and 7 with the ring in FP8 too (row scales)
        w = workload(6 if cfg == 11 else 7)
        w["fp8_ring"] = True
        w["name"] += "; ring K/V stored as E4M3 codes with one f32 scale per row"
        return w
    if cfg in (6, 7):  # the batched R-SWA and the 32K-history SR-SWA workloads over an FP8 (E4M3) prefix
        w = workload(2 if cfg == 6 else 4)
        w["fp8"] = True
        w["name"] += "; prefix K/V stored as E4M3 codes with per-(sequence, head, 32-token block) f32 scales"
        return w
    raise SystemExit(f"config {cfg} is not a decode benchmark here")


def prefill_flops(w: dict) -> float:
    """FLOPs the method must do per prefill launch: per (b, h) and query i, q.k and p.v over its
    visible keys (prefix_len + min(n, i + 1)), 2 x 2 x D FLOPs per key."""
    T, n, D, H = w["T"], w["n"], w["D"], w["H"]
    band = sum(min(n, i + 1) for i in range(T))
    return float(sum(4 * D * (m * T + band) for m in w["plen"]) * H)


def srswa_prefill_flops(w: dict, blk, logp) -> float:
    """FLOPs of the SR-SWA prefill attention: per (b, h) and query t, 4 x 128 x (the valid rows of
    its routed blocks with finite bias + its band min(n, t + 1))."""
    import numpy as np
    T, n, D, H = w["T"], w["n"], w["D"], w["H"]
    total = 0
    for b, m in enumerate(w["plen"]):
        c = blk[b].astype(np.int64)
        ok = (c >= 0) & np.isfinite(logp[b])
        rows = np.where(ok, np.minimum(32, m - 32 * c), 0).sum()
        band = sum(min(n, t + 1) for t in range(T))
        total += 4 * D * (int(rows) + band)
    return float(total * H)


def algorithmic_bytes(w: dict, blk_rows=None) -> dict:
    """Bytes the method must move per attention launch (and per route launch).

    R-SWA: per (b, h): (prefix_len + ring fill) K and V rows of 256 B each, the
    query (256 B), the f32 output (512 B) and lse (4 B). With an FP8 prefix a
    prefix row is 128 B of codes each for K and V, plus two f32 scales per block.
    SR-SWA: the same with the routed blocks' valid rows in place of the prefix.
    Router: per sequence the block keys (128 B per block), q_idx (128 B) and the
    top-k outputs (8 B each).
    """
    H, n = w["H"], w["n"]
    per_q = 256 + 512 + 4
    ring_row = 264 if w.get("fp8_ring") else 512  # FP8 ring: 128 + 128 B of codes + two 4-byte row scales
    # an FP8 prefix row is 128 + 128 B of codes, plus 8 B of scales per 32-row block
    row = 256 if w.get("fp8") else 512
    if w["kind"] == "rswa":
        attn = sum(m * row + (8 * ((m + 31) // 32) if w.get("fp8") else 0) + n * ring_row + per_q
                   for m in w["plen"]) * H
        return dict(attn=attn, route=0)
    rows = blk_rows if blk_rows is not None else [16 * 32] * w["B"]
    attn = sum(r * row + (8 * ((r + 31) // 32) if w.get("fp8") else 0) + n * ring_row + per_q for r in rows) * H
    route = sum(((m + 31) // 32) * 128 + 128 + 16 * 8 for m in w["plen"])
    return dict(attn=attn, route=route)


def l2_note(w: dict, nbytes: dict) -> str:
    """How the timed steps relate to the 126 MB L2 (no flush is issued between steps)."""
    B, H, n = w["B"], w["H"], w["n"]
    kv_store = sum(w["plen"]) * H * 512
    ring = B * H * n * 512
    if w["kind"] == "rswa":
        if nbytes["attn"] > 4e8:
            return f"inputs larger than L2 (each step reads {nbytes['attn'] / 1e9:.2f} GB of K/V); no flush"
        return "working set fits in L2; numbers are L2-resident"
    gathered = nbytes["attn"] - ring
    return (f"no flush: routed prefix blocks change every step (32 planted query directions, cycled; "
            f"{gathered / 1e6:.0f} MB gathered per step out of a {kv_store / 1e9:.1f} GB K/V store, a direction "
            f"recurs after 32 steps); the {ring / 1e6:.0f} MB ring is re-read every step, as in decode, and may "
            f"hit L2")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (200 ms) during the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="rswa_clocks_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        self.t0 = time.time()

    def stop(self, t_begin: float, t_end: float) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            rows.append((ts, parts))
        try:
            os.remove(self.path)
        except OSError:
            pass
        inside = [p for ts, p in rows if t_begin - 0.15 <= ts <= t_end + 0.15] or [p for _, p in rows[-3:]]
        sm = [float(p[2]) for p in inside if p[2].replace(".", "").isdigit()]
        smax = [float(p[3]) for p in inside if p[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in inside for i in range(4) if p[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(inside),
                "power_w_max": max((float(p[4]) for p in inside if p[4].replace(".", "").isdigit()), default=None)}


# ----------------------------------------------------------------------------- helpers

def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(kind: str) -> str:
    """Hash of the code the measured kernel is built from (kind: dense, sparse, prefill, srswa_prefill or rope), with
    comments and blank lines removed: a traffic record stays valid across comment edits only."""
    import re
    files = {"prefill": ["prefill.cu", "tcgen05.cuh", "common.cuh"], "rope": ["rope.cu", "common.cuh"],
             "srswa_prefill": ["srswa_prefill.cu", "prefill.cu", "tcgen05.cuh", "common.cuh"]}.get(
        kind, ["decode.cu", "common.cuh", "internal.h"])
    h = hashlib.sha256()
    for f in files:
        src = open(os.path.join(ROOT, "long_context_decode_swa_b200", "csrc", f), encoding="utf-8").read()
        if f == "internal.h":  # only the argument and workspace structs the decode kernel is built from
            a = src.index("struct DecodeArgs")
            b = src.index("};", src.index("struct WorkspacePlan")) + 2
            src = src[a:b]
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("\n".join(line.rstrip() for line in src.splitlines() if line.strip()).encode())
    h.update(kind.encode())
    return h.hexdigest()[:16]


def committed_traffic(key: str, src_hash: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on this kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    try:
        for line in open(p):
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            if len(parts) >= 3 and parts[0] == key and parts[1] == src_hash:
                return float(parts[2])
    except OSError:
        pass
    return None


def dist_setup(args):
    import torch

    from long_context_decode_swa_b200 import replicas
    world, rank, local = replicas.env_rank()
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit("--gpus N > 1 must be launched with torchrun (one process per GPU)")
    torch.cuda.set_device(local)
    if world > 1:
        replicas.init("nccl", timeout_s=120.0, device=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    from long_context_decode_swa_b200 import replicas
    replicas.barrier()


def max_over_ranks(world, x: float) -> float:
    from long_context_decode_swa_b200 import replicas
    return replicas.max_over_ranks(x, device="cuda")


# ----------------------------------------------------------------------------- our arm

class Problem:
    """Device-resident inputs and state of one rank's batch, plus the step function."""

    def __init__(self, w: dict, steps_total: int, seed: int):
        import torch

        import long_context_decode_swa_b200 as rswa
        from long_context_decode_swa_b200 import synth
        self.rswa = rswa
        self.w = w
        B, H, D, n = w["B"], w["H"], w["D"], w["n"]
        self.c = synth.decode_case(B, H, D, w["plen"], w["cap"], n, steps_total, seed=seed, device="cuda",
                                   wp0=w["wp0"], fill0=n, poison=False)
        self.dims = rswa.dims_of(self.c.pk, self.c.ring_k)
        self.ws = rswa.new_workspace(self.dims, rswa.OP_DECODE)
        self.out = torch.empty((B, H, D), dtype=torch.float32, device="cuda")
        self.lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
        self.sparse = w["kind"] == "srswa"
        self.fp8 = bool(w.get("fp8"))
        # SR-SWA over a bf16 prefix and ring: the whole step (append + router + attention) in one
        # launch (srswa_step), unless unfused is asked for
        self.fused_route = self.sparse and not self.fp8 and not w.get("fp8_ring") and not w.get("unfused")
        if self.fp8:  # the stored cache: the bf16 prefix quantised once, by the library
            self.k8, self.v8, self.ks, self.vs = rswa.fp8_prefix_buffers(self.c.pk)
            rswa.rswa_quantize_prefix(self.c.pk, self.c.pv, self.c.prefix_len, self.k8, self.v8, self.ks, self.vs,
                                      status=self.ws)
        self.fp8_ring = bool(w.get("fp8_ring"))
        if self.fp8_ring:  # a full FP8 ring: n appends of random rows before timing
            self.ring8 = rswa.fp8_ring_buffers(self.c.ring_k.shape)
            g = synth._gen(seed + 3, "cuda")
            for _ in range(n):
                kk = synth.randn_bf16((B, H, D), g, "cuda")
                vv = synth.randn_bf16((B, H, D), g, "cuda")
                rswa.rswa_append_fp8(*self.ring8, kk, vv, self.c.wp, self.c.fill, status=self.ws)
        self.rope = bool(w.get("rope"))
        if self.rope:  # this step's token positions ([steps][B]) and the encoded query
            tok, page = synth.page_positions(B, steps_total, seed=seed + 2)
            self.tok = tok.t().contiguous().to("cuda")
            self.page = page.t().contiguous().to("cuda")
            self.q_rot = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
        if self.sparse:
            n_dirs = 32
            pl = synth.plant_router_keys(w["plen"], w["cap"], n_dirs=n_dirs, seed=seed + 1, device="cuda")
            nb_cap = (w["cap"] + 31) // 32
            self.kbar = torch.empty((B, nb_cap, 32), dtype=torch.float32, device="cuda")
            rswa.srswa_index_pool(pl.k_idx, self.c.prefix_len, self.kbar)
            self.q_idx = pl.q_idx                           # [n_dirs][B][32]
            self.n_dirs = n_dirs
            self.blk = torch.empty((B, 16), dtype=torch.int32, device="cuda")
            self.logp = torch.empty((B, 16), dtype=torch.float32, device="cuda")
            self.ws_route = rswa.new_workspace(self.dims, rswa.OP_ROUTE)
            self.ws = rswa.new_workspace(self.dims, rswa.OP_SRSWA_ROUTED if self.fused_route else
                                         rswa.OP_SRSWA_DECODE)
            del pl
        torch.cuda.synchronize()

    def step(self, i: int, q=None, k_new=None, v_new=None, ev=None, pos=None):
        """Launches one decode step (1 to 3 kernels) on the current stream; returns the launch count.
        pos: this step's (tok_pos, page) for the encoding configs (default: the device-resident ones)."""
        c, r = self.c, self.rswa
        q = c.q[i] if q is None else q
        k_new = c.k_new[i] if k_new is None else k_new
        v_new = c.v_new[i] if v_new is None else v_new
        if self.rope:
            tok, page = pos if pos is not None else (self.tok[i % self.tok.shape[0]], self.page[i % self.page.shape[0]])
        if self.fused_route:
            if ev is not None:
                ev[0].record()
            if self.rope:
                r.srswa_step_rope(q, k_new, v_new, self.q_idx[i % self.n_dirs], self.kbar, c.pk, c.pv, c.prefix_len,
                                  c.ring_k, c.ring_v, c.wp, c.fill, tok, page, self.blk, self.logp, self.out, self.ws,
                                  lse=self.lse, scale=c.scale)
            else:
                r.srswa_step(q, k_new, v_new, self.q_idx[i % self.n_dirs], self.kbar, c.pk, c.pv, c.prefix_len,
                             c.ring_k, c.ring_v, c.wp, c.fill, self.blk, self.logp, self.out, self.ws, lse=self.lse,
                             scale=c.scale)
            if ev is not None:
                ev[1].record()
            return 1
        if not self.fp8 and not self.sparse and not (self.rope and self.w.get("unfused")):
            # R-SWA over a bf16 prefix: the fused step (ring append, and the encoding when asked
            # for, inside the decode launch), measured faster there
            if ev is not None:
                ev[0].record()
            if self.rope:
                r.rswa_decode_append_rope(q, k_new, v_new, c.pk, c.pv, c.prefix_len, c.ring_k, c.ring_v, c.wp,
                                          c.fill, tok, page, self.out, self.ws, lse=self.lse, scale=c.scale)
            else:
                r.rswa_decode_append(q, k_new, v_new, c.pk, c.pv, c.prefix_len, c.ring_k, c.ring_v, c.wp, c.fill,
                                     self.out, self.ws, lse=self.lse, scale=c.scale)
            if ev is not None:
                ev[1].record()
            return 1
        if self.fp8_ring:
            r.rswa_append_fp8(*self.ring8, k_new, v_new, c.wp, c.fill, status=self.ws)
            if self.sparse:
                if ev is not None:
                    ev[2].record()
                r.srswa_route(self.q_idx[i % self.n_dirs], self.kbar, c.prefix_len, self.blk, self.logp,
                              self.ws_route, prefix_cap=self.w["cap"])
                if ev is not None:
                    ev[3].record()
            if ev is not None:
                ev[0].record()
            if self.sparse:
                r.srswa_decode_fp8kv(q, self.k8, self.v8, self.ks, self.vs, c.prefix_len, self.blk, self.logp,
                                     *self.ring8, c.wp, c.fill, self.out, self.ws, lse=self.lse, scale=c.scale)
            else:
                r.rswa_decode_fp8kv(q, self.k8, self.v8, self.ks, self.vs, c.prefix_len, *self.ring8, c.wp, c.fill,
                                    self.out, self.ws, lse=self.lse, scale=c.scale)
            if ev is not None:
                ev[1].record()
            return 3 if self.sparse else 2
        if self.rope:
            if ev is not None:
                ev[4].record()
            q = r.rswa_append_rope(c.ring_k, c.ring_v, k_new, v_new, c.wp, c.fill, q, tok, page, q_out=self.q_rot,
                                   status=self.ws)
            if ev is not None:
                ev[5].record()
        else:
            r.rswa_append(c.ring_k, c.ring_v, k_new, v_new, c.wp, c.fill, status=self.ws)
        if not self.sparse:
            if ev is not None:
                ev[0].record()
            if self.fp8:
                r.rswa_decode_fp8(q, self.k8, self.v8, self.ks, self.vs, c.prefix_len, c.ring_k, c.ring_v, c.wp,
                                  c.fill, self.out, self.ws, lse=self.lse, scale=c.scale)
            else:
                r.rswa_decode(q, c.pk, c.pv, c.prefix_len, c.ring_k, c.ring_v, c.wp, c.fill, self.out, self.ws,
                              lse=self.lse, scale=c.scale)
            if ev is not None:
                ev[1].record()
            return 2
        if ev is not None:
            ev[2].record()
        r.srswa_route(self.q_idx[i % self.n_dirs], self.kbar, c.prefix_len, self.blk, self.logp, self.ws_route,
                      prefix_cap=self.w["cap"])
        if ev is not None:
            ev[3].record()
            ev[0].record()
        if self.fp8:
            r.srswa_decode_fp8(q, self.k8, self.v8, self.ks, self.vs, c.prefix_len, self.blk, self.logp, c.ring_k,
                               c.ring_v, c.wp, c.fill, self.out, self.ws, lse=self.lse, scale=c.scale)
        else:
            r.srswa_decode(q, c.pk, c.pv, c.prefix_len, self.blk, self.logp, c.ring_k, c.ring_v, c.wp, c.fill,
                           self.out, self.ws, lse=self.lse, scale=c.scale)
        if ev is not None:
            ev[1].record()
        return 3


class PrefillProblem:
    """Device-resident inputs of one rank's prefill chunk; a step is one rswa_prefill launch."""

    def __init__(self, w: dict, seed: int):
        import torch

        import long_context_decode_swa_b200 as rswa
        from long_context_decode_swa_b200 import synth
        self.rswa = rswa
        self.w = w
        self.d = synth.prefill_case(w["B"], w["H"], w["D"], w["plen"], w["cap"], w["T"], seed=seed, device="cuda",
                                    poison=False)
        B, H, T, D = self.d["q"].shape
        self.out = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
        self.lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
        self.ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        self.sparse = False
        torch.cuda.synchronize()

    def step(self, i: int, q=None, k_new=None, v_new=None, ev=None):
        d = self.d
        if ev is not None:
            ev[0].record()
        self.rswa.rswa_prefill(d["q"] if q is None else q, d["k_out"] if k_new is None else k_new,
                               d["v_out"] if v_new is None else v_new, d["pk"], d["pv"], d["prefix_len"], self.out,
                               self.ws, lse=self.lse, scale=d["scale"], ring=self.w["n"])
        if ev is not None:
            ev[1].record()
        return 1


class SrswaPrefillProblem:
    """SR-SWA chunked prefill: a step is srswa_route_tokens (every query routed) + srswa_prefill."""

    def __init__(self, w: dict, seed: int):
        import torch

        import long_context_decode_swa_b200 as rswa
        from long_context_decode_swa_b200 import synth
        self.rswa = rswa
        self.w = w
        B, H, T = w["B"], w["H"], w["T"]
        self.d = synth.prefill_case(B, H, w["D"], w["plen"], w["cap"], T, seed=seed, device="cuda", poison=False)
        pl = synth.plant_router_keys(w["plen"], w["cap"], n_dirs=32, seed=seed + 1, device="cuda")
        nb_cap = (w["cap"] + 31) // 32
        self.kbar = torch.empty((B, nb_cap, 32), dtype=torch.float32, device="cuda")
        rswa.srswa_index_pool(pl.k_idx, self.d["prefix_len"], self.kbar)
        self.q_tok = pl.q_idx[torch.arange(T, device="cuda") % 32].permute(1, 0, 2).contiguous()   # [B][T][32]
        del pl
        self.blk = torch.empty((B, T, 16), dtype=torch.int32, device="cuda")
        self.logp = torch.empty((B, T, 16), dtype=torch.float32, device="cuda")
        self.out = torch.empty((B, H, T, w["D"]), dtype=torch.float32, device="cuda")
        self.lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
        self.ws = rswa.srswa_prefill_workspace(B, H, T, w["cap"], ring=w["n"])
        self.ws_route = torch.zeros(256, dtype=torch.uint8, device="cuda")
        self.sparse = True
        torch.cuda.synchronize()

    def step(self, i: int, q=None, k_new=None, v_new=None, ev=None):
        d, r = self.d, self.rswa
        if ev is not None:
            ev[2].record()
        r.srswa_route_tokens(self.q_tok, self.kbar, d["prefix_len"], self.blk, self.logp, self.ws_route,
                             prefix_cap=self.w["cap"])
        if ev is not None:
            ev[3].record()
            ev[0].record()
        r.srswa_prefill(d["q"] if q is None else q, d["k_out"] if k_new is None else k_new,
                        d["v_out"] if v_new is None else v_new, d["pk"], d["pv"], d["prefix_len"], self.blk,
                        self.logp, self.out, self.ws, lse=self.lse, scale=d["scale"], ring=self.w["n"])
        if ev is not None:
            ev[1].record()
        return 2


def measured_tensor_peak(sustained: bool):
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["bf16_tflops_sustained" if sustained else "bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return (1400.0 if sustained else 1590.0), "fallback"


def run_ours(args, w: dict, world: int, rank: int, local: int) -> dict:
    import torch
    K, W = args.steps, args.warmup
    if w["kind"] in ("prefill", "srswa_prefill"):
        return run_prefill(args, w, world, rank, local)
    if w["kind"] == "rope":
        return run_rope(args, w, world, rank, local)
    prob = Problem(w, K + W, seed=1000 * args.config + rank)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(W):
            prob.step(K + i)
    stream.synchronize()
    # capture the K timed steps; external event records bracket the attention (and route) kernels of
    # every EVENT_EVERY-th step (an event node costs several microseconds of step time, so bracketing
    # every step would slow the step it measures)
    sampled = list(range(0, K, EVENT_EVERY))
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)] for _ in sampled]
    graph = torch.cuda.CUDAGraph()
    launches = 0
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            launches += prob.step(i, ev=evs[i // EVENT_EVERY] if i % EVENT_EVERY == 0 else None)
    graph.replay()                      # untimed replay
    torch.cuda.synchronize()
    status = prob.rswa.check_status(prob.ws)
    if status:
        raise RuntimeError(f"device status 0x{status:x} during warm-up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        start.record()
        graph.replay()
        end.record()
    end.synchronize()
    t_wall1 = time.time()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop(t_wall0, t_wall1)
    ms_total = start.elapsed_time(end)
    attn_ms = [e[0].elapsed_time(e[1]) for e in evs]
    route_ms = [e[2].elapsed_time(e[3]) for e in evs] if prob.sparse and not prob.fused_route else []
    rope_ms = [e[4].elapsed_time(e[5]) for e in evs] if prob.rope and w.get("unfused") else []
    ms_max = max_over_ranks(world, ms_total)
    del graph

    # routed rows of the last step (for the SR-SWA byte count)
    blk_rows = None
    if prob.sparse:
        blk = prob.blk.cpu().tolist()
        lp = prob.logp.cpu().tolist()
        blk_rows = []
        for b in range(w["B"]):
            m = w["plen"][b]
            blk_rows.append(sum(min(32, m - 32 * c) for c, l in zip(blk[b], lp[b]) if c >= 0 and l > -math.inf))
    nbytes = algorithmic_bytes(w, blk_rows)
    if not prob.fp8 and (not prob.sparse or prob.fused_route):
        # the fused step also writes this step's K and V row into the ring
        nbytes["attn"] += w["B"] * w["H"] * 512
        if prob.rope:  # and reads the step's two int32 positions per sequence
            nbytes["attn"] += w["B"] * 8
    if prob.fused_route:  # one kernel moves the router's bytes too
        nbytes = dict(attn=nbytes["attn"] + nbytes["route"], route=0)
    attn_avg_s = statistics.mean(attn_ms) / 1e3
    achieved = nbytes["attn"] / attn_avg_s / 1e9
    peak, peak_src = measured_peak()
    key = f"{'srswa_step' if prob.fused_route else ('srswa' if prob.sparse else 'rswa')}_decode_config{args.config}"
    traffic = committed_traffic(key, kernel_source_hash("sparse" if prob.sparse else "dense"))

    # ---- e2e through the public API: pinned host inputs -> device -> append/decode -> host result ----
    e2e = run_e2e(prob, K, W) if not args.no_e2e else {"ms": float("nan"), "h2d": 0, "d2h": 0}
    e2e_ms = max_over_ranks(world, e2e["ms"])
    B, H, D = w["B"], w["H"], w["D"]
    steps_per_s = world * K / (ms_max / 1e3)
    res = {
        "metric": METRIC,
        "value": steps_per_s,
        "unit": "steps/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_max / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "storage_dtype": ("e4m3 prefix (f32 block scales) + " + ("e4m3 ring (f32 row scales)" if prob.fp8_ring
                                                                  else "bf16 ring")) if prob.fp8 else "bf16",
        "data": "synthetic",
        "impl": "ours",
        "config": config_of(w, args, world),
        "timing": TIMING_NOTE,
        "qtok_per_s": steps_per_s * B * H,
        "seq_tok_per_s": steps_per_s * B,
        "hbm_gbs_step": world * K * (nbytes["attn"] + nbytes["route"]) / (ms_max / 1e3) / 1e9,
        "bytes_per_step": {"attn": nbytes["attn"], "route": nbytes["route"]},
        "roofline": {"bound": "hbm", "kernel": ("srswa step kernel: decode_kernel<true, bf16> with the ring append and "
                                                "the router fused" if prob.fused_route else
                                                ("srswa decode_kernel<true" if prob.sparse else "rswa decode_kernel<false")
                                                + (", fp8>" if prob.fp8 else (", bf16>" if prob.sparse else
                                                                              ", bf16> with the fused ring append")))
                                               + (", the page2d encoding inside" if prob.rope and not w.get("unfused")
                                                  else ""),
                     "achieved": achieved,
                     "peak": peak,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else
                     "fallback 6650 GB/s", "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes_per_launch": nbytes["attn"], "avg_launch_us": attn_avg_s * 1e6},
        "kernels_us": {"attention": attn_avg_s * 1e6,
                       **({"route": statistics.mean(route_ms) * 1e3} if route_ms else {}),
                       **({"append_rope": statistics.mean(rope_ms) * 1e3} if rope_ms else {})},
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": {"value": world * K / (e2e_ms / 1e3), "unit": "steps/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e_ms / K},
    }
    return res


def run_prefill(args, w: dict, world: int, rank: int, local: int) -> dict:
    import torch
    K, W = args.steps, args.warmup
    sparse = w["kind"] == "srswa_prefill"
    prob = (SrswaPrefillProblem if sparse else PrefillProblem)(w, seed=1000 * args.config + rank)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(W):
            prob.step(i)
    stream.synchronize()
    sampled = list(range(0, K, EVENT_EVERY))
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4 if sparse else 2)] for _ in sampled]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            prob.step(i, ev=evs[i // EVENT_EVERY] if i % EVENT_EVERY == 0 else None)
    graph.replay()
    torch.cuda.synchronize()
    if prob.rswa.check_status(prob.ws):
        raise RuntimeError("device status set during warm-up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        start.record()
        graph.replay()
        end.record()
    end.synchronize()
    t1 = time.time()
    barrier(world)
    clk = clocks.stop(t0, t1)
    ms_total = start.elapsed_time(end)
    ms_max = max_over_ranks(world, ms_total)
    kern_s = statistics.mean(e[0].elapsed_time(e[1]) for e in evs) / 1e3
    route_s = statistics.mean(e[2].elapsed_time(e[3]) for e in evs) / 1e3 if sparse else 0.0
    del graph
    sustained = ms_total > 1000.0
    peak, src = measured_tensor_peak(sustained)
    if sparse:
        flops = srswa_prefill_flops(w, prob.blk.cpu().numpy(), prob.logp.cpu().numpy())
    else:
        flops = prefill_flops(w)
    achieved = flops / kern_s / 1e12
    e2e = run_prefill_e2e(prob, K, W) if not args.no_e2e else {"ms": float("nan"), "h2d": 0, "d2h": 0}
    e2e_ms = max_over_ranks(world, e2e["ms"])
    B, H, T = w["B"], w["H"], w["T"]
    value = world * K / (ms_max / 1e3)
    return {
        "metric": METRIC, "value": value, "unit": "prefill chunks/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16-mma/f32-acc", "storage_dtype": "bf16", "data": "synthetic", "impl": "ours",
        "config": config_of(w, args, world),
        "timing": TIMING_NOTE,
        "qtok_per_s": value * B * H * T,
        "roofline": ({"bound": "tensor", "kernel": "SR-SWA prefill attention: group_prep_kernel + group_kernel + "
                                                 "prefill_kernel (band and ring, tcgen05) + routed_kernel (routed "
                                                 "blocks, tcgen05)",
                      "achieved": achieved, "peak": peak,
                      "peak_source": f"{src} bf16 {'sustained' if sustained else 'burst'} (MEASURED_PEAKS.json); "
                                     "FLOPs counted per query over its own routed rows and band",
                      "unit": "TFLOP/s", "frac": achieved / peak,
                      "traffic": committed_traffic(f"srswa_prefill_config{args.config}",
                                                 kernel_source_hash("srswa_prefill")),
                      "algorithmic_flops_per_launch": flops, "avg_launch_us": kern_s * 1e6} if sparse else
                     {"bound": "tensor", "kernel": "prefill_kernel (tcgen05)", "achieved": achieved, "peak": peak,
                      "peak_source": f"{src} bf16 {'sustained' if sustained else 'burst'} (MEASURED_PEAKS.json)",
                      "unit": "TFLOP/s", "frac": achieved / peak,
                      "traffic": committed_traffic(f"rswa_prefill_config{args.config}", kernel_source_hash("prefill")),
                      "algorithmic_flops_per_launch": flops, "avg_launch_us": kern_s * 1e6}),
        "kernels_us": {"prefill": kern_s * 1e6, **({"route": route_s * 1e6} if sparse else {})},
        # SR-SWA: route_tokens, group_prep, group, band prefill, routed; dense: the prefill kernel
        "gpu_launches": K * (5 if sparse else 1),
        "clocks": clk,
        "e2e": {"value": world * K / (e2e_ms / 1e3), "unit": "prefill chunks/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e_ms / K},
    }


class RopeProblem:
    """A prefill chunk's q and k (bf16 [B][T][H][D]) with their page positions; a step is one
    rswa_rope_page2d launch encoding both into separate outputs."""

    def __init__(self, w: dict, seed: int):
        import torch

        import long_context_decode_swa_b200 as rswa
        from long_context_decode_swa_b200 import synth
        self.rswa = rswa
        self.w = w
        B, T, H, D = w["B"], w["T"], w["H"], w["D"]
        g = synth._gen(seed, "cuda")
        self.q = synth.randn_bf16((B, T, H, D), g, "cuda")
        self.k = synth.randn_bf16((B, T, H, D), g, "cuda")
        tok, page = synth.page_positions(B, T, seed=seed + 1)
        self.tok, self.page = tok.to("cuda"), page.to("cuda")
        self.q_out, self.k_out = torch.empty_like(self.q), torch.empty_like(self.k)
        torch.cuda.synchronize()

    def step(self, i: int, q=None, k=None, ev=None):
        if ev is not None:
            ev[0].record()
        self.rswa.rswa_rope_page2d(self.q if q is None else q, self.tok, self.page, q_out=self.q_out,
                                   k=self.k if k is None else k, k_out=self.k_out, base=10000.0, page_mod=2)
        if ev is not None:
            ev[1].record()
        return 1


def rope_bytes(w: dict) -> float:
    """Bytes the encoding must move per launch: q and k read and written once (2 B per element)
    and the two int32 positions of every token."""
    elems = w["B"] * w["T"] * w["H"] * w["D"]
    return float(2 * 2 * 2 * elems + 2 * 4 * w["B"] * w["T"])


def run_rope(args, w: dict, world: int, rank: int, local: int) -> dict:
    import torch
    K, W = args.steps, args.warmup
    prob = RopeProblem(w, seed=1000 * args.config + rank)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(W):
            prob.step(i)
    stream.synchronize()
    sampled = list(range(0, K, EVENT_EVERY))
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in sampled]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            prob.step(i, ev=evs[i // EVENT_EVERY] if i % EVENT_EVERY == 0 else None)
    graph.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        start.record()
        graph.replay()
        end.record()
    end.synchronize()
    t1 = time.time()
    barrier(world)
    clk = clocks.stop(t0, t1)
    ms_max = max_over_ranks(world, start.elapsed_time(end))
    kern_s = statistics.mean(e[0].elapsed_time(e[1]) for e in evs) / 1e3
    del graph
    nbytes = rope_bytes(w)
    achieved = nbytes / kern_s / 1e9
    peak, peak_src = measured_peak()
    e2e = run_rope_e2e(prob, K, W) if not args.no_e2e else {"ms": float("nan"), "h2d": 0, "d2h": 0}
    e2e_ms = max_over_ranks(world, e2e["ms"])
    B, H, T = w["B"], w["H"], w["T"]
    value = world * K / (ms_max / 1e3)
    return {
        "metric": METRIC, "value": value, "unit": "encoded chunks/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "storage_dtype": "bf16", "data": "synthetic", "impl": "ours",
        "config": config_of(w, args, world),
        "timing": TIMING_NOTE,
        "tok_per_s": value * B * T,
        "roofline": {"bound": "hbm", "kernel": "rope_kernel (page2d, q and k)", "achieved": achieved, "peak": peak,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else
                     "fallback 6650 GB/s", "unit": "GB/s", "frac": achieved / peak,
                     "traffic": committed_traffic(f"rope_config{args.config}", kernel_source_hash("rope")),
                     "algorithmic_bytes_per_launch": nbytes, "avg_launch_us": kern_s * 1e6},
        "kernels_us": {"rope": kern_s * 1e6},
        "gpu_launches": K,
        "clocks": clk,
        "e2e": {"value": world * K / (e2e_ms / 1e3), "unit": "encoded chunks/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e_ms / K},
    }


def run_rope_e2e(prob: RopeProblem, K: int, W: int) -> dict:
    """Pinned host q and k -> device -> rswa_rope_page2d -> encoded q and k back to the host."""
    import torch
    hq, hk = prob.q.cpu().pin_memory(), prob.k.cpu().pin_memory()
    dq, dk = torch.empty_like(prob.q), torch.empty_like(prob.k)
    oq = torch.empty(prob.q.shape, dtype=torch.bfloat16, pin_memory=True)
    ok = torch.empty(prob.k.shape, dtype=torch.bfloat16, pin_memory=True)
    stream = torch.cuda.Stream()

    def one(i):
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        prob.step(i, q=dq, k=dk)
        oq.copy_(prob.q_out, non_blocking=True)
        ok.copy_(prob.k_out, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(W):
            one(i)
    stream.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s.record()
        for i in range(K):
            one(i)
        e.record()
    e.synchronize()
    return {"ms": s.elapsed_time(e), "h2d": 2 * hq.numel() * 2, "d2h": 2 * oq.numel() * 2}


def run_prefill_e2e(prob: PrefillProblem, K: int, W: int) -> dict:
    import torch
    d = prob.d
    hq = d["q"].cpu().pin_memory()
    hk = d["k_out"].cpu().pin_memory()
    hv = d["v_out"].cpu().pin_memory()
    dq, dk, dv = torch.empty_like(d["q"]), torch.empty_like(d["k_out"]), torch.empty_like(d["v_out"])
    hout = torch.empty(prob.out.shape, dtype=torch.float32, pin_memory=True)
    hlse = torch.empty(prob.lse.shape, dtype=torch.float32, pin_memory=True)
    stream = torch.cuda.Stream()

    def one(i):
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        prob.step(i, q=dq, k_new=dk, v_new=dv)
        hout.copy_(prob.out, non_blocking=True)
        hlse.copy_(prob.lse, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(W):
            one(i)
    stream.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s.record()
        for i in range(K):
            one(i)
        e.record()
    e.synchronize()
    return {"ms": s.elapsed_time(e), "h2d": 3 * hq.numel() * 2, "d2h": hout.numel() * 4 + hlse.numel() * 4}


def run_e2e(prob: Problem, K: int, W: int) -> dict:
    import torch
    c = prob.c
    B, H, D = c.q.shape[1:]
    pool = min(K, 16)
    hq = [torch.empty((B, H, D), dtype=torch.bfloat16, pin_memory=True) for _ in range(pool)]
    hk = [torch.empty((B, H, D), dtype=torch.bfloat16, pin_memory=True) for _ in range(pool)]
    hv = [torch.empty((B, H, D), dtype=torch.bfloat16, pin_memory=True) for _ in range(pool)]
    for j in range(pool):
        hq[j].copy_(c.q[j])
        hk[j].copy_(c.k_new[j])
        hv[j].copy_(c.v_new[j])
    dq = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
    dk, dv = torch.empty_like(dq), torch.empty_like(dq)
    hout = torch.empty((B, H, D), dtype=torch.float32, pin_memory=True)
    hlse = torch.empty((B, H), dtype=torch.float32, pin_memory=True)
    stream = torch.cuda.Stream()

    if prob.rope:  # the step's token positions come from the host too
        hpos = [torch.empty((2, B), dtype=torch.int32, pin_memory=True) for _ in range(pool)]
        for j in range(pool):
            hpos[j][0].copy_(prob.tok[j % prob.tok.shape[0]])
            hpos[j][1].copy_(prob.page[j % prob.page.shape[0]])
        dpos = torch.empty((2, B), dtype=torch.int32, device="cuda")

    def one(j):
        dq.copy_(hq[j % pool], non_blocking=True)
        dk.copy_(hk[j % pool], non_blocking=True)
        dv.copy_(hv[j % pool], non_blocking=True)
        if prob.rope:
            dpos.copy_(hpos[j % pool], non_blocking=True)
        prob.step(0, q=dq, k_new=dk, v_new=dv, pos=(dpos[0], dpos[1]) if prob.rope else None)
        hout.copy_(prob.out, non_blocking=True)
        hlse.copy_(prob.lse, non_blocking=True)

    with torch.cuda.stream(stream):
        for j in range(W):
            one(j)
    stream.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s.record()
        for j in range(K):
            one(j)
        e.record()
    e.synchronize()
    h2d = 3 * B * H * D * 2 + (2 * B * 4 if prob.rope else 0)
    d2h = B * H * D * 4 + B * H * 4
    return {"ms": s.elapsed_time(e), "h2d": h2d, "d2h": d2h}


# ----------------------------------------------------------------------------- oracle (CPU) arms

def oracle_sample_step(w: dict, sample: int, seed: int):
    """Inputs for `sample` sequences of the workload, on the host, for the oracle."""
    from long_context_decode_swa_b200 import synth
    plen = w["plen"][:sample]
    cap = max(plen)
    c = synth.decode_case(sample, w["H"], w["D"], plen, cap, w["n"], 1, seed=seed, wp0=w["wp0"], fill0=w["n"],
                          poison=False)
    u = synth.to_u16
    st = dict(q=u(c.q[0]), k=u(c.k_new[0]), v=u(c.v_new[0]), pk=u(c.pk), pv=u(c.pv), plen=c.prefix_len.numpy(),
              rk=u(c.ring_k).copy(), rv=u(c.ring_v).copy(), wp=c.wp.numpy().copy(), fill=c.fill.numpy().copy(),
              scale=c.scale)
    import oracle
    if w.get("fp8"):
        st["k8"], st["ks"] = oracle.quantize_prefix(st["pk"], st["plen"])
        st["v8"], st["vs"] = oracle.quantize_prefix(st["pv"], st["plen"])
    if w.get("fp8_ring"):  # a full FP8 ring: n appends of random rows
        import numpy as np
        st["ring8"] = list(oracle.fp8_ring(sample, w["H"], w["n"], w["D"]))
        rng = np.random.default_rng(seed + 3)
        for _ in range(w["n"]):
            kk = oracle.bf16_round(rng.standard_normal((sample, w["H"], w["D"])))
            vv = oracle.bf16_round(rng.standard_normal((sample, w["H"], w["D"])))
            oracle.append_fp8(*st["ring8"], kk, vv, st["wp"], st["fill"])
    if w.get("rope"):
        tok, page = synth.page_positions(sample, 1, seed=seed + 2)
        st["tok"], st["page"] = tok[:, 0].numpy().copy(), page[:, 0].numpy().copy()
    if w["kind"] == "srswa":
        pl = synth.plant_router_keys(plen, cap, n_dirs=1, seed=seed + 1)
        st["k_idx"] = u(pl.k_idx)
        st["q_idx"] = pl.q_idx[0].numpy()
    return st


def oracle_step(st: dict, w: dict):
    import oracle
    if w.get("rope"):  # the page2d encoding of this step's query and key, rounded to bf16
        st = dict(st, q=oracle.bf16_round(oracle.rope_page2d(st["q"], st["tok"], st["page"])))
        k = oracle.bf16_round(oracle.rope_page2d(st["k"], st["tok"], st["page"]))
    else:
        k = st["k"]
    if w.get("fp8_ring"):
        oracle.append_fp8(*st["ring8"], k, st["v"], st["wp"], st["fill"])
        if w["kind"] == "rswa":
            return oracle.rswa_decode_fp8kv(st["q"], st["k8"], st["v8"], st["ks"], st["vs"], st["plen"], *st["ring8"],
                                            st["wp"], st["fill"], st["scale"])
        kbar = st.get("kbar")
        if kbar is None:
            kbar = st["kbar"] = oracle.index_pool(st["k_idx"], st["plen"])
        r = oracle.route(st["q_idx"], kbar, st["plen"])
        return oracle.srswa_decode_fp8kv(st["q"], st["k8"], st["v8"], st["ks"], st["vs"], st["plen"], r["blk_idx"],
                                         r["blk_logp"], *st["ring8"], st["wp"], st["fill"], st["scale"])
    oracle.append(st["rk"], st["rv"], k, st["v"], st["wp"], st["fill"])
    if w["kind"] == "rswa":
        if w.get("fp8"):
            return oracle.rswa_decode_fp8(st["q"], st["k8"], st["v8"], st["ks"], st["vs"], st["plen"], st["rk"],
                                          st["rv"], st["wp"], st["fill"], st["scale"])
        return oracle.rswa_decode(st["q"], st["pk"], st["pv"], st["plen"], st["rk"], st["rv"], st["wp"], st["fill"],
                                  st["scale"])
    kbar = st.get("kbar")
    if kbar is None:
        kbar = st["kbar"] = oracle.index_pool(st["k_idx"], st["plen"])   # once per prefix, as on the GPU
    r = oracle.route(st["q_idx"], kbar, st["plen"])
    if w.get("fp8"):
        return oracle.srswa_decode_fp8(st["q"], st["k8"], st["v8"], st["ks"], st["vs"], st["plen"], r["blk_idx"],
                                       r["blk_logp"], st["rk"], st["rv"], st["wp"], st["fill"], st["scale"])
    return oracle.srswa_decode(st["q"], st["pk"], st["pv"], st["plen"], r["blk_idx"], r["blk_logp"], st["rk"],
                               st["rv"], st["wp"], st["fill"], st["scale"])


PREFILL_ORACLE_ROWS = 64  # query rows per sampled sequence in the prefill oracle arms


def oracle_prefill_case(w: dict, sample: int, seed: int):
    """Host inputs of `sample` sequences of a prefill workload, PREFILL_ORACLE_ROWS rows each
    (evenly spaced over the chunk), and the work fraction they stand for."""
    import numpy as np

    import oracle
    from long_context_decode_swa_b200 import synth
    plen = w["plen"][:sample]
    d = synth.prefill_case(sample, w["H"], w["D"], plen, w["cap"], w["T"], seed=seed, poison=False)
    u = synth.to_u16
    st = dict(q=u(d["q"]), k=u(d["k_out"]), v=u(d["v_out"]), pk=u(d["pk"]), pv=u(d["pv"]),
              plen=d["prefix_len"].numpy(), scale=d["scale"])
    rows = np.unique(np.linspace(0, w["T"] - 1, PREFILL_ORACLE_ROWS).astype(np.int32))
    st["rows"] = rows
    if w["kind"] == "srswa_prefill":
        pl = synth.plant_router_keys(plen, w["cap"], n_dirs=32, seed=seed + 1)
        kbar = oracle.index_pool(u(pl.k_idx), st["plen"])
        q_tok = pl.q_idx.numpy()[rows % 32].transpose(1, 0, 2).copy()          # routes of the sampled rows
        b_rows, l_rows = oracle.route_tokens(q_tok, kbar, st["plen"])
        st["blk"] = np.full((sample, w["T"], 16), -1, np.int32)
        st["logp"] = np.full((sample, w["T"], 16), -np.inf)
        st["blk"][:, rows], st["logp"][:, rows] = b_rows, l_rows
        st["q_tok"], st["kbar"] = q_tok, kbar
    return st, (sample / w["B"]) * (len(rows) / w["T"])


def oracle_prefill_step(st: dict, w: dict):
    import oracle
    if w["kind"] == "srswa_prefill":
        st["blk_rows"] = oracle.route_tokens(st["q_tok"], st["kbar"], st["plen"])      # the step's routing
        return oracle.srswa_prefill(st["q"], st["k"], st["v"], st["pk"], st["pv"], st["plen"], st["blk"],
                                    st["logp"], st["scale"], st["rows"], w["n"])
    return oracle.rswa_prefill(st["q"], st["k"], st["v"], st["pk"], st["pv"], st["plen"], st["scale"], st["rows"],
                               w["n"])


ROPE_ORACLE_TOKENS = 512  # tokens of one sequence per oracle step of the encoding config


def oracle_rope_case(w: dict, seed: int):
    """Host q, k and positions of ROPE_ORACLE_TOKENS tokens of one sequence, and the work
    fraction of a chunk they stand for."""
    from long_context_decode_swa_b200 import synth
    g = synth._gen(seed, "cpu")
    shape = (ROPE_ORACLE_TOKENS, w["H"], w["D"])
    q, k = synth.randn_bf16(shape, g, "cpu"), synth.randn_bf16(shape, g, "cpu")
    tok, page = synth.page_positions(1, ROPE_ORACLE_TOKENS, seed=seed + 1)
    st = dict(q=synth.to_u16(q), k=synth.to_u16(k), tok=tok[0].numpy().copy(), page=page[0].numpy().copy())
    return st, ROPE_ORACLE_TOKENS / (w["B"] * w["T"])


def oracle_rope_step(st: dict):
    import oracle
    return (oracle.bf16_round(oracle.rope_page2d(st["q"], st["tok"], st["page"])),
            oracle.bf16_round(oracle.rope_page2d(st["k"], st["tok"], st["page"])))


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo", encoding="utf-8"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w: dict, budget_s: float = 12.0, budget_1thread_s: float = 3.0) -> dict:
    """The oracle as it stands, on all host threads (the reported value) and, over the same
    sample for a shorter time, on one thread."""
    import oracle
    step, frac, unit, what, lo, hi = _cpu_baseline_case(w, budget_s)
    threads = oracle.get_threads()
    dt, reps = _time_steps(step, budget_s, lo, hi)
    try:
        oracle.set_threads(1)
        dt1, reps1 = _time_steps(step, budget_1thread_s, 1, hi)
    finally:
        oracle.set_threads(threads)
    return {"value": frac / dt, "unit": unit, "cores": threads, "kind": "oracle",
            "sample": f"{what}, {reps} steps timed; {unit} extrapolated by the sample fraction; fp64 C oracle "
                      f"(OpenMP over independent problems)",
            "value_1thread": frac / dt1, "steps_1thread": reps1, "host_cpus": os.cpu_count(),
            "cpu_model": cpu_model()}


def _time_steps(step, budget_s: float, min_reps: int, max_reps: int):
    reps, t0 = 0, time.perf_counter()
    while reps < min_reps or (time.perf_counter() - t0 < budget_s and reps < max_reps):
        step()
        reps += 1
    return (time.perf_counter() - t0) / reps, reps


def _cpu_baseline_case(w: dict, budget_s: float):
    """(step function, work fraction of one full step, unit, sample description, min / max
    timed steps) of a bounded oracle sample of the workload, warmed up once."""
    if w["kind"] == "rope":
        st, frac = oracle_rope_case(w, seed=77)
        oracle_rope_step(st)
        return (lambda: oracle_rope_step(st)), frac, "encoded chunks/s", \
            f"{ROPE_ORACLE_TOKENS} of {w['B'] * w['T']} tokens (all heads, q and k)", 2, 200
    if w["kind"] in ("prefill", "srswa_prefill"):
        st, frac = oracle_prefill_case(w, 1, seed=77)
        oracle_prefill_step(st, w)
        return (lambda: oracle_prefill_step(st, w)), frac, "prefill chunks/s", \
            f"1 of {w['B']} sequences, {len(st['rows'])} of {w['T']} query rows (all heads)", 1, 20
    sample = min(w["B"], 2)
    st = oracle_sample_step(w, sample, seed=77)
    oracle_step(st, w)                               # warm (and pool the router keys)
    t0 = time.perf_counter()
    oracle_step(st, w)
    one = time.perf_counter() - t0
    # grow the sample to fill about budget_s of CPU work
    sample = int(max(1, min(w["B"], sample * budget_s / max(one, 1e-3) / 3)))
    st = oracle_sample_step(w, sample, seed=78)
    oracle_step(st, w)
    return (lambda: oracle_step(st, w)), sample / w["B"], "steps/s", \
        f"{sample} of {w['B']} sequences per step (all heads)", 2, 50


def config_of(w: dict, args, world: int) -> dict:
    """The `config` object of a workload, the same for both arms."""
    B = w["B"]
    c = {"workload": w["name"], "config_index": args.config, "batch_per_gpu": B, "global_batch": B * world,
         "heads": w["H"], "head_dim": w["D"], "ring": w["n"], "parallelism": f"replicas x{world}"}
    if w["kind"] == "rope":
        nbytes = rope_bytes(w)
        c.pop("ring")
        c["chunk"] = w["T"]
        c["l2"] = (f"no flush: each step streams {nbytes / 1e9:.2f} GB through L2 ({nbytes / 2e9:.2f} GB read, "
                   "as much written), twice its 126 MB, in the same order every step")
    elif w["kind"] in ("prefill", "srswa_prefill"):
        c["chunk"] = w["T"]
        c["prefix_tokens_mean"] = statistics.mean(w["plen"])
        c["l2"] = "no flush: the prefix K/V of the chunk exceed L2; each step recomputes the same chunk"
    else:
        c["prefix_tokens_mean"] = statistics.mean(w["plen"])
        c["l2"] = l2_note(w, algorithmic_bytes(w))
    return c


def run_reference(args, w: dict) -> dict:
    """The oracle as the reference arm, on the host cores, K timed steps of a bounded sample.

    Each step runs the oracle on a sample of the workload; `value` is extrapolated to the
    whole workload by the sample fraction, while `ms_per_step` is the measured time of one
    sampled step (so steps x ms_per_step is the timed region's real length)."""
    import oracle
    if w["kind"] == "rope":
        st, frac = oracle_rope_case(w, seed=99)
        step = lambda: oracle_rope_step(st)  # noqa: E731
        unit = "encoded chunks/s"
        what = f"{ROPE_ORACLE_TOKENS} of {w['B'] * w['T']} tokens per step (all heads, q and k)"
    elif w["kind"] in ("prefill", "srswa_prefill"):
        st, frac = oracle_prefill_case(w, 1, seed=99)
        step = lambda: oracle_prefill_step(st, w)  # noqa: E731
        unit = "prefill chunks/s"
        what = f"1 of {w['B']} sequences, {len(st['rows'])} of {w['T']} query rows per step (all heads)"
    else:
        sample = min(w["B"], {1: 1, 2: 8, 4: 2, 5: 1, 6: 8, 7: 2, 10: 2, 11: 8, 12: 2, 13: 8}.get(args.config, 1))
        st = oracle_sample_step(w, sample, seed=99)
        step = lambda: oracle_step(st, w)  # noqa: E731
        frac = sample / w["B"]
        unit = "steps/s"
        what = f"{sample} of {w['B']} sequences per step (all heads)"
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = frac / dt
    cb = {"value": value, "unit": unit, "cores": oracle.get_threads(), "kind": "oracle",
          "sample": f"{what}; {unit} extrapolated by the sample fraction ({frac:.4g}); fp64 C oracle on the host "
                    f"cores"}
    return {"metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "ms_per_full_step_extrapolated": 1e3 / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": config_of(w, args, 1), "cpu_baseline": cb,
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


SWEEP_LENGTHS = (8192, 16384, 32768, 65536, 102400)


def run_length_sweep(args, world: int, rank: int, local: int, lengths=SWEEP_LENGTHS) -> dict:
    """The SR-SWA step at uniform history lengths (16 sequences, top-16 + 128-slot ring).

    The attention reads the same 640 rows per (sequence, head) at every length; only the
    router's block-key scan (128 B per 32-token block) grows with the history."""
    import torch
    rows = []
    for m in lengths:
        w = workload(5)
        w["plen"] = [m] * w["B"]
        w["cap"] = m
        w["name"] = f"SR-SWA decode, 16 sequences, 16 heads, head_dim 128, uniform history {m} tokens"
        if getattr(args, "unfused", False):
            w["unfused"] = True
        r = run_ours(args, w, world, rank, local)
        rows.append({"history": m, "ms_per_step": r["ms_per_step"], "steps_per_s": r["value"],
                     "kernels_us": r["kernels_us"], "attn_hbm_frac": r["roofline"]["frac"],
                     "route_bytes_share": r["bytes_per_step"]["route"] / (r["bytes_per_step"]["attn"] +
                                                                          r["bytes_per_step"]["route"]),
                     "clocks": r["clocks"]})
        torch.cuda.empty_cache()
    steps = [x["ms_per_step"] for x in rows]
    return {"metric": "SR-SWA decode step latency vs history length", "unit": "ms/step", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": False, "data": "synthetic",
            "impl": "ours", "sweep": rows, "max_over_min": max(steps) / min(steps)}


EXTRA_CONFIGS = (1, 3, 4, 5)
EXTRA_SWEEP = (8192, 102400)


def summary(r: dict) -> dict:
    """The figures of one workload's run kept in the default line's `configs` object."""
    rf = r["roofline"]
    keep = ("bound", "kernel", "achieved", "peak", "peak_source", "unit", "frac", "traffic",
            "algorithmic_bytes_per_launch", "algorithmic_flops_per_launch", "avg_launch_us")
    return {"workload": r["config"]["workload"], "value": r["value"], "unit": r["unit"],
            "ms_per_step": r["ms_per_step"], "steps": r["steps"], "warmup": r["warmup"],
            **({"qtok_per_s": r["qtok_per_s"]} if "qtok_per_s" in r else {}),
            **({"hbm_gbs_step": r["hbm_gbs_step"]} if "hbm_gbs_step" in r else {}),
            "kernels_us": r["kernels_us"], "gpu_launches": r["gpu_launches"],
            "roofline": {k: rf[k] for k in keep if k in rf}, "clocks": r["clocks"], "l2": r["config"].get("l2")}


def run_extra_configs(args, world: int, rank: int, local: int) -> dict:
    """Configs 1, 3, 4 and 5 and the two ends of the SR-SWA length sweep, each with its own
    K timed steps, kernel brackets, roofline and clocks (no e2e or CPU legs)."""
    import copy

    import torch
    out = {}
    for cfg in EXTRA_CONFIGS:
        a = copy.copy(args)
        a.config = cfg
        a.no_e2e = True
        out[str(cfg)] = summary(run_ours(a, workload(cfg), world, rank, local))
        torch.cuda.empty_cache()
    a = copy.copy(args)
    a.config = 5
    a.no_e2e = True
    sw = run_length_sweep(a, world, rank, local, EXTRA_SWEEP)
    out["length_sweep"] = {"what": sw["metric"] + " (16 sequences, uniform histories)", "unit": sw["unit"],
                           "points": [{"history": x["history"], "ms_per_step": x["ms_per_step"],
                                       "kernels_us": x["kernels_us"], "clocks": x["clocks"]} for x in sw["sweep"]],
                           "max_over_min": sw["max_over_min"]}
    return out


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=None, choices=list(range(1, 14)),
                    help="the workload (default 2, which also runs configs 1, 3, 4, 5 into `configs`)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (a smaller case, e.g. for an ncu capture)")
    ap.add_argument("--prefix", type=int, default=None,
                    help="override every sequence's prefix length (and the capacity) of the workload")
    ap.add_argument("--unfused", action="store_true",
                    help="SR-SWA workloads: append + srswa_route + srswa_decode (three launches) instead of srswa_step")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="with the default workload, skip the other configs' lines in `configs`")
    ap.add_argument("--length-sweep", action="store_true",
                    help="SR-SWA latency against history length: 16 sequences at uniform lengths "
                         f"{SWEEP_LENGTHS}, one JSON line with every length's step and kernel times")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    extras = args.config is None and not args.no_extra_configs and args.batch is None and args.prefix is None
    if args.config is None:
        args.config = 2
    w = workload(args.config)
    if args.batch is not None:
        reps = (args.batch + len(w["plen"]) - 1) // len(w["plen"])
        w["plen"] = (w["plen"] * reps)[:args.batch]
        w["name"] = w["name"].replace(f"{w['B']} sequences", f"{args.batch} sequences")
        w["B"] = args.batch
    if args.unfused:
        w["unfused"] = True
        w["name"] += " [append, router and attention as three launches]"
    if args.prefix is not None:
        w["plen"] = [args.prefix] * w["B"]
        w["cap"] = args.prefix
        w["name"] += f" [prefix overridden: {args.prefix}]"

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, w)), flush=True)
        return

    world, rank, local = dist_setup(args)
    try:
        if args.length_sweep:
            res = run_length_sweep(args, world, rank, local)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        res = run_ours(args, w, world, rank, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(w)
        if extras and world == 1:
            import torch
            torch.cuda.empty_cache()
            res["configs"] = run_extra_configs(args, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        from long_context_decode_swa_b200 import replicas
        replicas.shutdown()


if __name__ == "__main__":
    main()
