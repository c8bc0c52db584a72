#!/usr/bin/env python
"""Decode-step benchmark of the variable-precision weight read path on B200.

Default workload (one GPU): every linear layer of one Qwen3-0.6B-shaped decode
step (28 layers x {q 1024->2048, k/v 1024->1024, o 2048->1024, gate/up
1024->3072, down 3072->1024} + tied lm_head 1024->151936, 197 GEMVs), random
N(0, 0.02) weights quantized to int8 (absmax per row per 128 columns) and held
in the plane store, every block read at D4, an independent bf16 N(0, 1) input
per layer, batch 1; the logit gate (entropy and top-2 margin over the 151936
logits) runs on the head output, and a seeded 16% of steps escalate to D8 by
adding the residual planes to every GEMV and re-running the gate.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fl|reference]

Prints one JSON line. `value` is weight bytes read per second (GB/s) over the
whole job; `tokens_per_s` the decode steps per second. With N > 1 (torchrun)
each rank runs its own replica of the step (independent decode streams), so
scaling is weak and `value` sums the ranks; time is the max over ranks.
--impl reference times the CPU oracle on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "weight-bytes GB/s and fraction of HBM peak at batch 1; decode-step tokens/s"
WORKLOAD = ("qwen3-0.6b-shaped decode step: 197 GEMVs (28 layers x q,k,v,o,gate,up,down + tied head "
            "1024x151936) read at D4 from the plane store, logit gate over 151936 logits fused into the same launch; "
            "a step escalates D4->D8 (residual planes + gate) when the gate says so, decided on the device; 25 "
            "rotating input sets, entropy threshold set so 4 of them (16%) escalate; batch 1")


SPEC_HBM_GBS = 8000.0   # B200 HBM3e, the vendor's figure (context beside the measured copy peak)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=["fl", "reference"], default="fl")
    ap.add_argument("--no-extra", action="store_true", help="skip the per-config kernel measurements")
    ap.add_argument("--shard", action="store_true",
                    help="split every layer's blocks over the ranks (strong scaling) instead of one replica per GPU")
    ap.add_argument("--profile", choices=["none", "step", "residual", "kquant", "kernels", "layer"], default="none",
                    help="short run for an ncu capture: 'step' = the decode step only, 'residual' = the decode "
                         "step's D4 -> D8 residual pass (gate fused) three times, 'kquant' = the K-quant "
                         "step only, 'kernels' = one pass of every per-config kernel measurement, 'layer' = "
                         "three fl_gemv_depth calls on one layer (--shape, --batch, --level); no JSON "
                         "timing claims")
    ap.add_argument("--shape", default="4096,4096", help="--profile layer: out,in")
    ap.add_argument("--batch", type=int, default=1, help="--profile layer: tokens per call")
    ap.add_argument("--level", type=int, default=3, help="--profile layer: depth level of every block (3 = D6)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples, every 10 ms, from before the warm-up to the
    end of the timing (a device-timed region of a few ms would otherwise fall between samples),
    plus NVML readings taken right before and right after the timed region itself."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = {}

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "10"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def mark(self, key):
        """NVML reading of the SM clock and the active throttle reasons, stored under key."""
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            names = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
                     0x4: "sw_power_cap"}
            self.marks[key] = {"sm_mhz": mhz, "reasons": sorted(n for b, n in names.items() if bits & b)}
        except Exception as e:
            self.marks[key] = {"error": str(e)[:120]}

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        window = "10 ms nvidia-smi samples from before the warm-up to the end of the kernel timing"
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": window,
                    **self.marks}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "window": window, **self.marks}


def src_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "variable_precision_weight_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel_key):
    """Per-launch DRAM bytes from the committed ncu summary, if taken on the current source."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel_key]
        if rec.get("source_sha") != src_sha(*rec["sources"]):
            return None
        return rec
    except Exception:
        return None


def device_ok(fl, what):
    """The kernels' error words after a timed region: a bounded wait that ran out (or a bad list
    entry) makes that region's outputs invalid, so its number is not printed."""
    try:
        fl.fl_device_status()
    except fl.FlError as e:
        raise SystemExit(json.dumps({"error": f"device status after {what}: {e}", "value": None}))
    return "ok"


def max_over_ranks(t, world, device="cuda"):
    """The job's time: the slowest rank's (every rank calls this; one all-reduce)."""
    if world <= 1:
        return t
    import torch
    import torch.distributed as dist
    tt = torch.tensor([t], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_rate(units_per_rank, world, t):
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / t


# ----------------------------------------------------------------------------- GPU workload

def gpu_int8_layer(torch, out, inn, gen):
    """N(0, 0.02) weights -> int8 codes (absmax / 127 per row per 128 columns, round half to even)."""
    w = torch.randn((out, inn), generator=gen, device="cuda", dtype=torch.float32).mul_(0.02)
    wg = w.view(out, inn // 128, 128)
    s = wg.abs().amax(dim=2).div_(127.0)
    safe = torch.where(s > 0, s, torch.ones_like(s))
    q = torch.round(wg / safe[..., None]).clamp_(-127, 127)
    q = torch.where((s > 0)[..., None], q, torch.zeros_like(q)).to(torch.int8).view(out, inn)
    return q, s.contiguous()


def plane_layer(torch, fl, out, inn, gen, keep_block0=False):
    q, s = gpu_int8_layer(torch, out, inn, gen)
    store = torch.empty(fl.fl_plane_store_bytes(out, inn), dtype=torch.uint8, device="cuda")
    fl.fl_pack_planes(q, s, out, inn, store)
    if keep_block0:  # the first 64-row block's codes and scales, for the in-run output check
        return store, (q[:64].cpu().numpy(), s[:64].cpu().numpy())
    return store


def block_reference(q, s, level, x_bits):
    """Plain float64 outputs of one 64-row block read at `level` (the depth rule written out:
    w_d = s (u_d - 128 + c_d), u = q + 128 with its low 8 - d bits cleared, c_d = (2^(8-d) - 1) / 2)
    and the bar's mass sum_c |w_d| |x_c|."""
    import numpy as np
    d = 2 * level
    u = q.astype(np.int64) + 128
    ud = u & ~((1 << (8 - d)) - 1)
    cd = ((1 << (8 - d)) - 1) / 2.0
    w = np.repeat(s.astype(np.float64), 128, axis=1) * (ud - 128 + cd)
    x = (x_bits.astype(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return w @ x, np.abs(w) @ np.abs(x)


def plane_bytes(inn, level):
    """Algorithmic bytes of one 64-row block read at `level`: scales + level planes."""
    G = inn // 128
    return 256 * G + 2048 * G * level if level > 0 else 0


class DecodeStep:
    """The Qwen3-0.6B-shaped step on one GPU. NSETS independent input sets rotate over the
    steps; each set's step is one CUDA graph: the D4 pass with the logit gate fused, then the
    D4->D8 residual pass (gate fused) conditioned on the device on the first pass's escalate
    flag. The entropy threshold is calibrated once so that 4 of the 25 sets escalate."""

    NSETS = 25
    NESC = 4

    def __init__(self, torch, fl, seed):
        from variable_precision_weight_b200 import synth
        self.torch, self.fl = torch, fl
        gen = torch.Generator(device="cuda")
        gen.manual_seed(seed)
        self.shapes = synth.qwen3_step_shapes()
        self.stores = []
        tot_in = sum(i for _, _, i in self.shapes)
        tot_out = sum(o for _, o, _ in self.shapes)
        self.xs = torch.empty((self.NSETS, tot_in), dtype=torch.int16, device="cuda")
        self.xs_b = torch.empty_like(self.xs)   # second input buffer (the end-to-end run double-buffers)
        self.y = torch.empty(tot_out, dtype=torch.float32, device="cuda")
        self.h2d_bytes = tot_in * 2
        items = [[] for _ in range(self.NSETS)]
        items_r = [[] for _ in range(self.NSETS)]
        items_b = [[] for _ in range(self.NSETS)]
        items_rb = [[] for _ in range(self.NSETS)]
        oi = oo = 0
        self.bytes_d4 = self.bytes_res = 0
        self.levels = []
        # problems whose first 64-row block the run checks: the first layer, the first down
        # projection (in 3072) and the head
        self.sample_idx = (0, 6, len(self.shapes) - 1)
        self.samples = {}
        for pi, (name, o, i) in enumerate(self.shapes):
            st = plane_layer(torch, fl, o, i, gen, keep_block0=pi in self.sample_idx)
            if pi in self.sample_idx:
                st, qs = st
                self.samples[pi] = (qs, oi, oo, i)
            self.stores.append(st)
            d4 = torch.full((o // 64,), 2, dtype=torch.uint8, device="cuda")
            d8 = torch.full((o // 64,), 4, dtype=torch.uint8, device="cuda")
            self.levels += [d4, d8]
            ys = self.y[oo:oo + o]
            for j in range(self.NSETS):
                xs, xb = self.xs[j, oi:oi + i], self.xs_b[j, oi:oi + i]
                items[j].append((st, o, i, d4, None, xs, ys))
                items_r[j].append((st, o, i, d4, d8, xs, ys))
                items_b[j].append((st, o, i, d4, None, xb, ys))
                items_rb[j].append((st, o, i, d4, d8, xb, ys))
            self.bytes_d4 += (o // 64) * plane_bytes(i, 2)
            self.bytes_res += (o // 64) * (256 * (i // 128) + 2048 * (i // 128) * 2)
            oi += i
            oo += o
        self.vocab = self.shapes[-1][1]
        self.prob_d4 = [fl.gemv_problems(it) for it in items]
        self.prob_res = [fl.gemv_problems(it) for it in items_r]
        self.prob_d4_b = [fl.gemv_problems(it) for it in items_b]
        self.prob_res_b = [fl.gemv_problems(it) for it in items_rb]
        self.n = len(items[0])
        # gate outputs per set (one 32-byte row, so one device->host copy reads a step's result)
        self.gates = torch.zeros((self.NSETS, 8), dtype=torch.int32, device="cuda")
        wsb = fl.fl_gemv_gate_workspace_bytes(1)
        self.gate_ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        self.runs = torch.zeros(1, dtype=torch.int32, device="cuda")  # residual passes that ran
        self.hx = [synth.bf16_normal((tot_in,), seed, 99, j).view("int16") for j in range(self.NSETS)]
        for j in range(self.NSETS):
            self.xs[j].copy_(torch.from_numpy(self.hx[j]))
        self.tau_h, self.tau_m = self._calibrate(wsb)
        self.specs = [self._spec(j, wsb) for j in range(self.NSETS)]

    def _spec(self, j, wsb, tau_h=None, tau_m=None):
        torch, g = self.torch, self.gates[j]
        return self.fl.gate_spec(self.n - 1, self.tau_h if tau_h is None else tau_h,
                                 self.tau_m if tau_m is None else tau_m, g[0:1].view(torch.float32),
                                 g[1:2].view(torch.float32), g[2:4], g[4:5].view(torch.uint8)[0:1], self.gate_ws, wsb)

    def _calibrate(self, wsb):
        """Entropy threshold between the NESC-th and next largest entropies of the sets' D4
        logits; the margin threshold below every set's margin (it never decides)."""
        import numpy as np
        torch = self.torch
        for j in range(self.NSETS):
            self.fl.fl_gemv_batched_gate(self.prob_d4[j], self.n, 1, 0, self._spec(j, wsb, 1e30, -1.0))
        torch.cuda.synchronize()
        H = self.gates[:, 0].view(torch.float32).cpu().numpy().astype(np.float64)
        M = self.gates[:, 1].view(torch.float32).cpu().numpy().astype(np.float64)
        h = np.sort(H)[::-1]
        self.calib = {"entropy_sorted": h.tolist(), "margin_min": float(M.min())}
        tau_h, tau_m = float(0.5 * (h[self.NESC - 1] + h[self.NESC])), float(0.5 * M.min())
        self.esc_sets = [bool(H[j] > tau_h or M[j] < tau_m) for j in range(self.NSETS)]
        return tau_h, tau_m

    def check_outputs(self, j):
        """The sampled blocks of the step last run (input set j) against block_reference at the
        level the device ran (D8 for an escalating set, else D4): the largest error as a fraction
        of the path's bar 2e-3 sum |w||x| + 1e-5."""
        import numpy as np
        lv = 4 if self.esc_sets[j] else 2
        y = self.y.cpu().numpy()
        worst = 0.0
        for pi, ((q, s), oi, oo, i) in self.samples.items():
            yref, mass = block_reference(q, s, lv, self.hx[j][oi:oi + i])
            err = np.abs(y[oo:oo + 64].astype(np.float64) - yref)
            worst = max(worst, float((err / (2e-3 * mass + 1e-5)).max()))
        return {"input_set": j, "level": f"D{2 * lv}", "blocks": len(self.samples), "max_err_ratio": worst,
                "ok": worst <= 1.0}

    def step_graph_body(self, j, buf=0):
        fl = self.fl
        d4, res = (self.prob_d4, self.prob_res) if buf == 0 else (self.prob_d4_b, self.prob_res_b)
        fl.fl_gemv_batched_gate(d4[j], self.n, 1, 0, self.specs[j])
        esc = self.gates[j, 4:5].view(self.torch.uint8)[0:1]
        fl.fl_gemv_batched_gate_if(res[j], self.n, 1, 1, self.specs[j], esc, self.runs)

    def gemv_only(self):
        # the step's dominant kernel as the step runs it (D4 pass, gate fused)
        self.fl.fl_gemv_batched_gate(self.prob_d4[0], self.n, 1, 0, self.specs[0])

    def capture(self):
        torch = self.torch
        for j in range(self.NSETS):
            self.step_graph_body(j)
        torch.cuda.synchronize()
        self.g = []
        for j in range(self.NSETS):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                self.step_graph_body(j)
            self.g.append(gr)
        # all NSETS steps in order in one graph, so each launch's set-up overlaps the previous
        # kernel's tail (programmatic launches) across step boundaries too
        self.gAll = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.gAll):
            for j in range(self.NSETS):
                self.step_graph_body(j)
        self.gK = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.gK):
            self.gemv_only()
        torch.cuda.synchronize()

    def capture_first(self, k):
        """One graph of the first k sets' steps in order (a run whose step count is not a whole
        number of rounds replays it once, so every timed step overlaps its neighbours)."""
        self.gFirst = None
        if k > 0:
            self.gFirst = self.torch.cuda.CUDAGraph()
            with self.torch.cuda.graph(self.gFirst):
                for j in range(k):
                    self.step_graph_body(j)
            self.torch.cuda.synchronize()


def time_loop(torch, body, steps):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for k in range(steps):
        body(k)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e-3


# ----------------------------------------------------------------------------- per-config kernel lines

def kquant_step(torch, fl):
    """The Llama-3.2-1B-shaped K-quant step (96 Q4_K + 17 Q6_K tensors, seeded Gaussian weights
    encoded on the host), resident on the device: (problems, tensors to keep alive, record bytes)."""
    import concurrent.futures as cf
    from variable_precision_weight_b200 import synth
    mix = synth.llama32_kquant_mix()

    def make(k):
        name, o, i, tp = mix[k]
        return synth.encode_kquant(synth.gaussian_weights(o, i, 4, k), tp)

    with cf.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 4)) as ex:
        blobs = list(ex.map(make, range(len(mix))))
    items, keep, nbytes = [], [], 0
    for k, ((name, o, i, tp), blob) in enumerate(zip(mix, blobs)):
        blk = torch.from_numpy(blob).cuda()
        x = torch.from_numpy(synth.bf16_normal((1, i), 4, 1000 + k).view("int16")).cuda()
        y = torch.empty((1, o), device="cuda")
        keep += [blk, x, y]
        items.append((blk, tp, o, i, x, y))
        nbytes += blk.numel()
    return items, keep, nbytes


def in_pass_measurement(torch, fl, step, peak, f=0.16, rounds=40):
    """The decode step with the in-pass level decision instead of the gate: the D4 pass, the
    share rule (the draft score's top f of every layer's blocks rise to D8), then the residual
    pass from D4 to the decided levels. One graph holds the 25 input sets' steps in order."""
    import numpy as np
    n, NS = step.n, step.NSETS
    tot_out = step.y.numel()
    lv_to, score, lifted, counts, dec_items, res_items = [], [], [], [], [], [[] for _ in range(NS)]
    oo = oi = 0
    bytes_res = bytes_scales = 0
    for k, (name, o, i) in enumerate(step.shapes):
        t = torch.empty(o // 64, dtype=torch.uint8, device="cuda")
        c = torch.empty(o // 64, dtype=torch.float32, device="cuda")
        u = torch.empty(o // 64, dtype=torch.int32, device="cuda")
        lv_to.append(t)
        score.append(c)
        lifted.append(u)
        ys = step.y[oo:oo + o]
        dec_items.append((step.stores[k], o, i, ys, t, c, u))
        for j in range(NS):
            res_items[j].append((step.stores[k], o, i, step.levels[2 * k], t, step.xs[j, oi:oi + i], ys))
        up = int(np.floor(np.float64(np.float32(f)) * (o // 64)))    # the kernel's count of rising blocks
        counts.append(up)
        bytes_res += up * (256 * (i // 128) + 2048 * (i // 128) * 2)
        bytes_scales += (o // 64) * 256 * (i // 128)
        oo += o
        oi += i
    assert oo == tot_out
    dec = fl.decide_problems(dec_items)
    # the two-launch form (score, then one CTA per layer selects): on this step the one-launch
    # form (counters; the last CTA to score a layer selects it) measured slower, 16.4 us
    params = fl.decide_params(fl.FL_DECIDE_SHARE, 2, 4, 0.0, f)
    res = [fl.gemv_problems(it) for it in res_items]
    lists = fl.block_lists(lifted, counts)          # the residual reads the lifted blocks only

    def one(j):
        fl.fl_gemv_batched(step.prob_d4[j], n, 1, 0)
        fl.fl_level_decide(dec, n, 1, params)
        fl.fl_gemv_batched_listed(res[j], *lists, n, 1, 1)

    for j in range(NS):
        one(j)
    torch.cuda.synchronize()
    got = sum(int((t > 2).sum().item()) for t in lv_to)
    g_all, g_dec, g_res = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_all):
        for j in range(NS):
            one(j)
    with torch.cuda.graph(g_dec):
        for j in range(NS):
            fl.fl_level_decide(dec, n, 1, params)
    with torch.cuda.graph(g_res):                  # the residual passes alone, last decided levels
        for j in range(NS):
            fl.fl_gemv_batched_listed(res[j], *lists, n, 1, 1)
    for _ in range(3):
        g_all.replay()
        g_dec.replay()
        g_res.replay()
    t = time_loop(torch, lambda k: g_all.replay(), rounds) / (rounds * NS)
    td = time_loop(torch, lambda k: g_dec.replay(), rounds) / (rounds * NS)
    tr = time_loop(torch, lambda k: g_res.replay(), rounds) / (rounds * NS)
    g_lad = torch.cuda.CUDAGraph()                 # the score launch alone (ladder rule)
    ladder = fl.decide_params(fl.FL_DECIDE_LADDER, 2, 4, 1.0, 0.0)
    with torch.cuda.graph(g_lad):
        for j in range(NS):
            fl.fl_level_decide(dec, n, 1, ladder)
    g_lad.replay()
    tl = time_loop(torch, lambda k: g_lad.replay(), rounds) / (rounds * NS)
    nbytes = step.bytes_d4 + bytes_res
    return {"f": f, "lifted_blocks": got, "lifted_expected": sum(counts), "us_per_step": t * 1e6,
            "bytes_per_step": nbytes, "GBps": nbytes / t / 1e9, "frac": nbytes / t / 1e9 / peak,
            "tokens_per_s": 1.0 / t, "decide_us": td * 1e6, "decide_ladder_us": tl * 1e6, "residual_us": tr * 1e6,
            "residual_GBps": bytes_res / tr / 1e9,
            "decide_bytes": bytes_scales + 4 * tot_out, "decide_GBps": (bytes_scales + 4 * tot_out) / td / 1e9,
            "launches_per_step": 4}


def spec_measurement(torch, fl, step, peak, K=4, rounds=20):
    """Verified speculation on the decode step: windows of K steps, each K gated D4 draft passes
    (batch 1), one gated residual pass at batch K over the window (the D8 logits of all K steps
    from one read of the low planes) and the acceptance, on the device. The 25 input sets give
    25 // K windows, one graph."""
    n, W = step.n, step.NSETS // K
    wins = []
    for w in range(W):
        items_d, items_v, keep = [[] for _ in range(K)], [], []
        oi = 0
        for k, (name, o, i) in enumerate(step.shapes):
            x = torch.empty((K, i), dtype=torch.int16, device="cuda")
            for t in range(K):
                x[t].copy_(step.xs[w * K + t, oi:oi + i])
            y = torch.empty((K, o), dtype=torch.float32, device="cuda")
            keep += [x, y]
            d4, d8 = step.levels[2 * k], step.levels[2 * k + 1]
            for t in range(K):
                items_d[t].append((step.stores[k], o, i, d4, None, x[t], y[t]))
            items_v.append((step.stores[k], o, i, d4, d8, x, y))
            oi += i
        wsb = fl.fl_gemv_gate_workspace_bytes(K)
        g = {"ws": torch.zeros(wsb, dtype=torch.uint8, device="cuda"),
             "ent": torch.empty(K, dtype=torch.float32, device="cuda"),
             "mar": torch.empty(K, dtype=torch.float32, device="cuda"),
             "esc": torch.empty(K, dtype=torch.uint8, device="cuda"),
             "dtop": torch.empty((K, 2), dtype=torch.int32, device="cuda"),
             "vtop": torch.empty((K, 2), dtype=torch.int32, device="cuda"),
             "res": torch.empty(2, dtype=torch.int32, device="cuda")}
        specs = [fl.gate_spec(n - 1, step.tau_h, step.tau_m, g["ent"][t:t + 1], g["mar"][t:t + 1], g["dtop"][t],
                              g["esc"][t:t + 1], g["ws"], wsb) for t in range(K)]
        spec_v = fl.gate_spec(n - 1, step.tau_h, step.tau_m, g["ent"], g["mar"], g["vtop"], g["esc"], g["ws"], wsb)
        wins.append((g, keep, [fl.gemv_problems(it) for it in items_d], fl.gemv_problems(items_v), specs, spec_v))
    totals = torch.zeros(2, dtype=torch.int32, device="cuda")

    def all_windows():
        for g, keep, pd, pv, specs, spec_v in wins:
            for t in range(K):
                fl.fl_gemv_batched_gate(pd[t], n, 1, 0, specs[t])
            fl.fl_gemv_batched_gate(pv, n, K, 1, spec_v)
            fl.fl_spec_accept(g["dtop"], g["vtop"], K, g["res"], totals)

    all_windows()
    torch.cuda.synchronize()
    acc, emi = (int(v) for v in totals.cpu().tolist())
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        all_windows()
    for _ in range(3):
        gr.replay()
    t = time_loop(torch, lambda k: gr.replay(), rounds) / rounds
    bytes_round = W * (K * step.bytes_d4 + step.bytes_res)
    d8_per_token = sum((o // 64) * plane_bytes(i, 4) for _, o, i in step.shapes)
    return {"k": K, "windows": W, "accepted": acc, "emitted": emi, "us_per_window": t / W * 1e6,
            "tokens_per_s": emi / t, "bytes_per_emitted_token": bytes_round / emi,
            "vs_all_d8_bytes_per_token": bytes_round / emi / d8_per_token,
            "GBps": bytes_round / t / 1e9, "frac": bytes_round / t / 1e9 / peak,
            "launches_per_window": K + 2}


def extra_measurements(torch, fl, peak):
    """One line per other configuration: its kernel's weight-byte rate, timed over CUDA-graph replays
    with enough rotating copies of the weights that every replay reads past the 126 MB L2."""
    import numpy as np
    from variable_precision_weight_b200 import synth
    out = {}
    gen = torch.Generator(device="cuda")

    def graph_time(fn, reps):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize()
        t = time_loop(torch, lambda k: g.replay(), reps)
        return t / reps

    # config 0: 1024 x 1024, 16 blocks at seeded depths; D4 pass + residual to D8
    gen.manual_seed(100)
    ncp = 320
    stores = [plane_layer(torch, fl, 1024, 1024, gen) for _ in range(ncp)]
    lv = torch.from_numpy(synth.seeded_levels(16, 0, 2)).cuda()
    x = torch.from_numpy(synth.bf16_normal((1, 1024), 0, 3).view("int16")).cuda()
    y = torch.empty((1, 1024), device="cuda")
    nbytes = sum(plane_bytes(1024, int(l)) for l in lv.cpu().numpy())
    items = [(s, 1024, 1024, lv, None, x, y) for s in stores]
    arr = fl.gemv_problems(items[:256])
    t = graph_time(lambda: fl.fl_gemv_batched(arr, 256, 1, 0), 50)
    out["cfg0_1024x1024_mixed_depth"] = {"layers_per_launch": 256, "us_per_layer": t / 256 * 1e6,
                                         "GBps": 256 * nbytes / t / 1e9, "frac": 256 * nbytes / t / 1e9 / peak}
    w0 = fl.plane_weight(stores[0], 1024, 1024)
    wsb = fl.fl_gemv_workspace_bytes(1024, 1024, 1)
    ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
    t1 = graph_time(lambda: fl.fl_gemv_depth(w0, lv, x, 1, y, ws, wsb), 200)
    out["cfg0_single_call_latency_us"] = t1 * 1e6
    try:
        # D4 everywhere, then the residual to D8 (256 layers per launch each)
        d4 = torch.full((16,), 2, dtype=torch.uint8, device="cuda")
        d8 = torch.full((16,), 4, dtype=torch.uint8, device="cuda")
        a4 = fl.gemv_problems([(s_, 1024, 1024, d4, None, x, y) for s_ in stores[:256]])
        ar = fl.gemv_problems([(s_, 1024, 1024, d4, d8, x, y) for s_ in stores[:256]])
        tp = graph_time(lambda: (fl.fl_gemv_batched(a4, 256, 1, 0), fl.fl_gemv_batched(ar, 256, 1, 1)), 50)
        pb = 16 * (plane_bytes(1024, 2) + 256 * 8 + 2048 * 8 * 2)   # D4 read, then scales + planes 2, 3
        out["cfg0_d4_then_residual_to_d8"] = {"layers_per_launch": 256, "us_per_layer": tp / 256 * 1e6,
                                              "GBps": 256 * pb / tp / 1e9, "frac": 256 * pb / tp / 1e9 / peak}
        # hot: one layer's weights 256 times per launch, so they stay in L2
        ah = fl.gemv_problems([(stores[0], 1024, 1024, lv, None, x, y)] * 256)
        th = graph_time(lambda: fl.fl_gemv_batched(ah, 256, 1, 0), 50)
        out["cfg0_mixed_depth_l2_resident"] = {"us_per_layer": th / 256 * 1e6, "GBps": 256 * nbytes / th / 1e9}
    except Exception as e:  # a measurement that fails is reported, not fatal to the line
        out["cfg0_d4_then_residual_to_d8"] = {"error": str(e)[:200]}
    del stores, items, arr
    torch.cuda.empty_cache()

    try:
        # the standalone logit gate over the Qwen3-0.6B vocab (151,936 fp32 logits, batch 1), and
        # the packer (int8 codes + scales -> plane store) on the head's 1024 -> 151936 shape
        V = 151936
        z = torch.randn((1, V), device="cuda", generator=gen)
        ge, gm = torch.empty(1, device="cuda"), torch.empty(1, device="cuda")
        gt, gs = torch.empty((1, 2), dtype=torch.int32, device="cuda"), torch.empty(1, dtype=torch.uint8, device="cuda")
        tgt = graph_time(lambda: fl.fl_logit_gate(z, V, 1, 10.0, 1e-3, ge, gm, gt, gs), 200)
        out["gate_151936_logits"] = {"us": tgt * 1e6, "GBps": 4 * V / tgt / 1e9}
        qh = torch.randint(-127, 128, (V, 1024), dtype=torch.int8, device="cuda", generator=gen)
        sh = torch.rand((V, 8), device="cuda", generator=gen)
        sth = torch.empty(fl.fl_plane_store_bytes(V, 1024), dtype=torch.uint8, device="cuda")
        tpk = graph_time(lambda: fl.fl_pack_planes(qh, sh, V, 1024, sth), 20)
        pk_bytes = qh.numel() + sh.numel() * 4 + sth.numel()
        out["pack_1024x151936"] = {"us": tpk * 1e6, "GBps": pk_bytes / tpk / 1e9, "frac": pk_bytes / tpk / 1e9 / peak,
                                   "bytes": pk_bytes}
        del qh, sh, sth
    except Exception as e:
        out["gate_151936_logits"] = {"error": str(e)[:200]}

    # config 2: lens map over 14708 blocks (8 lenses) -> per-layer levels -> 35 layers x [64 n_b, 2048]
    nb = 14708
    xy, cxy, r = synth.lens_inputs(nb, 8, 2, 1)
    stops = synth.even_stops(3, 1)
    p = fl.lens_params(0.3, 0.75, 1, 4, stops, 0)
    xy_d, c_d, r_d = (torch.from_numpy(a).cuda() for a in (xy, cxy, r))
    lev = torch.empty(nb, dtype=torch.uint8, device="cuda")
    cnt = torch.zeros(5, dtype=torch.int32, device="cuda")
    tl = graph_time(lambda: fl.fl_level_map(xy_d, nb, c_d, r_d, 8, p, lev, None), 500)
    fl.fl_level_map(xy_d, nb, c_d, r_d, 8, p, lev, cnt)
    torch.cuda.synchronize()
    counts = cnt.cpu().numpy().astype(np.int64)
    mem_bits = float((counts * np.array([0, 2, 4, 6, 8])).sum() / counts.sum())
    gen.manual_seed(200)
    per = synth.lens_stack_layers(nb, 35)
    items, b0, nbytes, keep = [], 0, 0, []
    lv_host = lev.cpu().numpy()
    xs = torch.from_numpy(synth.bf16_normal((35, 2048), 2, 2).view("int16")).cuda()
    ys = torch.empty((35, 64 * max(per)), device="cuda")
    for l, n in enumerate(per):
        st = plane_layer(torch, fl, 64 * n, 2048, gen)
        keep.append(st)
        items.append((st, 64 * n, 2048, lev[b0:b0 + n], None, xs[l], ys[l]))
        nbytes += sum(plane_bytes(2048, int(v)) for v in lv_host[b0:b0 + n])
        b0 += n
    arr = fl.gemv_problems(items)
    t = graph_time(lambda: fl.fl_gemv_batched(arr, 35, 1, 0), 100)
    out["cfg2_lens_stack_14708_blocks"] = {"level_map_us": tl * 1e6, "memory_bits": mem_bits,
                                           "level_counts": counts.tolist(), "gemv_us": t * 1e6,
                                           "GBps": nbytes / t / 1e9, "frac": nbytes / t / 1e9 / peak,
                                           "bytes": nbytes}
    del keep, items, arr
    torch.cuda.empty_cache()

    # config 3: large shapes at D6 (literal lens reading: glass D6, kappa = D6), batch 1/4/8/16
    for (o, i) in ((14336, 4096), (4096, 14336), (4096, 4096)):
        per_copy = (o // 64) * plane_bytes(i, 3)
        ncp = max(2, int(np.ceil(300e6 / per_copy)))
        gen.manual_seed(300 + o)
        stores = [plane_layer(torch, fl, o, i, gen) for _ in range(ncp)]
        lv6 = torch.full((o // 64,), 3, dtype=torch.uint8, device="cuda")
        for batch in (1, 4, 8, 16, 32):
            x = torch.from_numpy(synth.bf16_normal((batch, i), 3, batch).view("int16")).cuda()
            y = torch.empty((batch, o), device="cuda")
            wsb = fl.fl_gemv_workspace_bytes(o, i, batch)
            ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
            wts = [fl.plane_weight(s, o, i) for s in stores]

            def run():
                for w in wts:
                    fl.fl_gemv_depth(w, lv6, x, batch, y, ws, wsb)
            t = graph_time(run, 20) / ncp
            out[f"cfg3_{i}to{o}_b{batch}_D6"] = {"us": t * 1e6, "GBps": per_copy / t / 1e9,
                                                 "frac": per_copy / t / 1e9 / peak,
                                                 "tflops": 2 * batch * o * i / t / 1e12}
        try:
            # the g = 1 variant at batch 1: kappa = D8 inside 4 lenses drawn by the config-2 rule
            nbk = o // 64
            bxy, bc, br = synth.lens_inputs(nbk, 4, 3, o)
            pg = fl.lens_params(0.3, 1.0, 3, 4, synth.even_stops(4, 3), 0)
            lvg = torch.empty(nbk, dtype=torch.uint8, device="cuda")
            fl.fl_level_map(torch.from_numpy(bxy).cuda(), nbk, torch.from_numpy(bc).cuda(), torch.from_numpy(br).cuda(),
                            4, pg, lvg, None)
            torch.cuda.synchronize()
            lvh = lvg.cpu().numpy()
            bg = sum(plane_bytes(i, int(v)) for v in lvh)
            x1 = torch.from_numpy(synth.bf16_normal((1, i), 3, 1).view("int16")).cuda()
            y1 = torch.empty((1, o), device="cuda")
            wsb1 = fl.fl_gemv_workspace_bytes(o, i, 1)
            ws1 = torch.zeros(max(wsb1, 16), dtype=torch.uint8, device="cuda")

            def run_g():
                for w in wts:
                    fl.fl_gemv_depth(w, lvg, x1, 1, y1, ws1, wsb1)
            tg = graph_time(run_g, 20) / ncp
            out[f"cfg3_{i}to{o}_b1_g1"] = {"us": tg * 1e6, "GBps": bg / tg / 1e9, "frac": bg / tg / 1e9 / peak,
                                           "d8_blocks": int((lvh == 4).sum()), "blocks": nbk}
        except Exception as e:
            out[f"cfg3_{i}to{o}_b1_g1"] = {"error": str(e)[:200]}
        del stores
        torch.cuda.empty_cache()

    # config 4: Llama-3.2-1B-shaped K-quant step (96 Q4_K + 17 Q6_K tensors), batch 1
    items, keep, nbytes = kquant_step(torch, fl)
    arr = fl.kquant_problems(items)
    t = graph_time(lambda: fl.fl_gemv_kquant_batched(arr, len(items), 1), 100)
    tr = traffic_record("kquant_gemv_llama32_1b_step")
    out["cfg4_llama32_1b_kquant_step"] = {"us": t * 1e6, "GBps": nbytes / t / 1e9, "frac": nbytes / t / 1e9 / peak,
                                          "tokens_per_s": 1.0 / t, "bytes": nbytes,
                                          "traffic": tr["bytes_per_launch"] if tr else None}
    del keep, items, arr
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- CPU oracle timing

def cpu_baseline(budget_s=12.0):
    """The oracle as it stands (OpenMP over output rows, all host cores) on a bounded sample of the step:
    the 28 GEMVs of layers 0-3 of the Qwen3-0.6B shapes at D4, passed over repeatedly for ~budget_s."""
    import numpy as np
    import oracle
    from variable_precision_weight_b200 import synth
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    shapes = synth.qwen3_step_shapes()[:28]
    layers = []
    for k, (name, o, i) in enumerate(shapes):
        q, s = synth.int8_layer(o, i, 9, k)
        layers.append((q, s, synth.bf16_normal((1, i), 9, 1000 + k), np.full(o // 64, 2, np.uint8),
                       (o // 64) * plane_bytes(i, 2)))
    t_total, nbytes, passes = 0.0, 0, 0
    while t_total < budget_s:
        for q, s, x, lv, nb in layers:
            t0 = time.perf_counter()
            oracle.gemv_depth(q, s, lv, x, nthreads=cores)
            t_total += time.perf_counter() - t0
            nbytes += nb
        passes += 1
    # the same sample on one thread, for about a tenth of the time
    t1, b1 = 0.0, 0
    while t1 < budget_s / 10:
        for q, s, x, lv, nb in layers:
            t0 = time.perf_counter()
            oracle.gemv_depth(q, s, lv, x, nthreads=1)
            t1 += time.perf_counter() - t0
            b1 += nb
    return {"value": nbytes / t_total / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} passes over the 28 GEMVs of layers 0-3 at D4 "
                      f"({nbytes / passes / 1e6:.1f} MB of weight bytes per pass), {t_total:.1f} s",
            "tokens_per_s_equiv": nbytes / t_total / (316616704),
            "single_thread_value": b1 / t1 / 1e9, "cpu_model": cpu_model()}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ----------------------------------------------------------------------------- arms

def run_reference(args, rank):
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    from variable_precision_weight_b200 import synth
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    # one step = the oracle's D4 read of one 1024 x 1024 layer of the step (a bounded sample)
    q, s = synth.int8_layer(1024, 1024, 9, 0)
    x = synth.bf16_normal((1, 1024), 9, 1)
    lv = np.full(16, 2, np.uint8)
    for _ in range(args.warmup):
        oracle.gemv_depth(q, s, lv, x, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gemv_depth(q, s, lv, x, nthreads=cores)
    t = time.perf_counter() - t0
    nbytes = 16 * plane_bytes(1024, 2)
    v = nbytes * args.steps / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample_per_step": "one 1024x1024 GEMV of the step at D4"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": "one 1024x1024 layer at D4 per step"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_fl(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    from variable_precision_weight_b200 import fl

    torch.cuda.set_device(local_rank)
    peak, peak_kind = load_peaks()
    if args.profile == "layer":
        from variable_precision_weight_b200 import synth
        o, i = (int(v) for v in args.shape.split(","))
        gen = torch.Generator(device="cuda")
        gen.manual_seed(300 + o)
        w = fl.plane_weight(plane_layer(torch, fl, o, i, gen), o, i)
        lv = torch.full((o // 64,), args.level, dtype=torch.uint8, device="cuda")
        x = torch.from_numpy(synth.bf16_normal((args.batch, i), 3, args.batch).view("int16")).cuda()
        y = torch.empty((args.batch, o), device="cuda")
        wsb = fl.fl_gemv_workspace_bytes(o, i, args.batch)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        for k in range(3):
            fl.fl_gemv_depth(w, lv, x, args.batch, y, ws, wsb)
        torch.cuda.synchronize()
        fl.fl_device_status()
        return 0
    if args.profile == "kquant":
        items, keep, _ = kquant_step(torch, fl)
        arr = fl.kquant_problems(items)
        for k in range(3):
            fl.fl_gemv_kquant_batched(arr, len(items), 1)
        torch.cuda.synchronize()
        return 0
    step = DecodeStep(torch, fl, seed=1000 + rank)
    if args.profile == "residual":
        # after the 25 calibration launches: the D4 -> D8 residual pass (gate fused) of input
        # set 0, three times, as the step runs it when the gate escalates
        for k in range(3):
            fl.fl_gemv_batched_gate(step.prob_res[0], step.n, 1, 1, step.specs[0])
        torch.cuda.synchronize()
        fl.fl_device_status()
        return 0
    step.capture()
    NS = step.NSETS

    if args.profile != "none":
        for k in range(3):
            step.g[k].replay()
        torch.cuda.synchronize()
        if args.profile == "kernels":
            extra_measurements(torch, fl, peak)
        return 0

    # the timed steps: whole rounds of the NS sets as one graph each, then one graph holding the
    # remaining sets' steps in order: every launch overlaps its neighbours for any step count
    rem = args.steps % NS
    step.capture_first(rem)

    def body(r):
        if r < args.steps // NS:
            step.gAll.replay()
        else:
            step.gFirst.replay()

    clk = ClockSampler(local_rank)
    clk.__enter__()
    for k in range(args.warmup):
        step.g[k % NS].replay()
    step.gAll.replay()
    if step.gFirst is not None:
        step.gFirst.replay()
    step.runs.zero_()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n_calls = args.steps // NS + (1 if rem else 0)
    clk.mark("nvml_before_timed_region")
    t = time_loop(torch, body, n_calls)
    clk.mark("nvml_after_timed_region")
    t = max_over_ranks(t, world)
    status = device_ok(fl, "the timed steps")
    parity = step.check_outputs((args.steps - 1) % NS)
    n_esc = int(step.runs.item())                 # residual passes the device decided to run
    value = job_rate(args.steps * step.bytes_d4 + n_esc * step.bytes_res, world, t) / 1e9
    tok_s = job_rate(args.steps, world, t)

    # dominant kernel alone: the step's D4 pass (gate fused), graph-replayed back to back
    reps = max(200, args.steps // 10)
    tk = time_loop(torch, lambda k: step.gK.replay(), reps) / reps
    clk.__exit__(None, None, None)
    device_ok(fl, "the roofline launch timing")
    achieved = step.bytes_d4 / tk / 1e9
    spread = {}
    try:  # the launch's own spread: 100 replays, each bracketed by events
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(100)]
        for e0, e1 in evs:
            e0.record()
            step.gK.replay()
            e1.record()
        torch.cuda.synchronize()
        us = np.array([e0.elapsed_time(e1) * 1e3 for e0, e1 in evs])
        spread = {"us_p10": float(np.percentile(us, 10)), "us_p50": float(np.percentile(us, 50)),
                  "us_p90": float(np.percentile(us, 90)),
                  "frac_p50": step.bytes_d4 / (float(np.percentile(us, 50)) * 1e-6) / 1e9 / peak}
    except Exception as e:
        spread = {"spread_error": str(e)[:200]}

    # end to end: each step copies its inputs host->device (pinned) and reads the gate result back.
    # Rounds of the NS input sets alternate between two device input buffers: while a round
    # computes from one, its copy stream fills the other with the next round's inputs (the input
    # sets are independent), and each step's result is read back on a third stream as soon as the
    # step is done. One CUDA graph per buffer holds a round with its copies as graph nodes; the
    # round's last copy and read-back complete before its graph does. The first round's inputs
    # are copied before timing, so the timed region holds one input copy per step it runs (for
    # the following round) and every step's read-back.
    hx = [torch.from_numpy(step.hx[j]).pin_memory() for j in range(NS)]
    hres = torch.empty((NS, 8), dtype=torch.int32).pin_memory()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = (step.xs, step.xs_b)

    def round_with_copies(buf):
        cap = torch.cuda.current_stream()
        ev_done = [torch.cuda.Event() for _ in range(NS)]
        ev_fork, ev_in, ev_out = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
        ev_fork.record(cap)
        s_in.wait_event(ev_fork)
        s_out.wait_event(ev_fork)
        with torch.cuda.stream(s_in):                 # the next round's inputs, into the other buffer
            for j in range(NS):
                bufs[1 - buf][j].copy_(hx[j], non_blocking=True)
        for j in range(NS):
            step.step_graph_body(j, buf)
            ev_done[j].record(cap)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[j])
                hres[j].copy_(step.gates[j], non_blocking=True)      # step j's result
        ev_in.record(s_in)
        ev_out.record(s_out)
        cap.wait_event(ev_in)
        cap.wait_event(ev_out)

    g_e2e = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
    for buf in (0, 1):
        with torch.cuda.graph(g_e2e[buf]):
            round_with_copies(buf)
    for r in range(2):                                # buffer 0 holds round 0's inputs after these
        g_e2e[r % 2].replay()
    e2e_rounds = max(1, min(args.steps, 5000) // NS)
    e2e_steps = e2e_rounds * NS
    step.runs.zero_()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    te = time_loop(torch, lambda k: g_e2e[k % 2].replay(), e2e_rounds)
    te = max_over_ranks(te, world)
    n_esc_e = int(step.runs.item())
    device_ok(fl, "the end-to-end steps")
    assert np.array_equal(hres.numpy(), step.gates.cpu().numpy()), "read-back differs from the device rows"
    e2e_val = job_rate(e2e_steps * step.bytes_d4 + n_esc_e * step.bytes_res, world, te) / 1e9

    extra = None
    if world == 1 and not args.no_extra:
        extra = {"cfg1_in_pass_share_decision": in_pass_measurement(torch, fl, step, peak),
                 "cfg1_verified_speculation_k4": spec_measurement(torch, fl, step, peak)}
        extra.update(extra_measurements(torch, fl, peak))
        device_ok(fl, "the per-configuration measurements")

    if rank != 0:
        return 0
    cpu = cpu_baseline() if world == 1 else None
    tr = traffic_record("plane_gemv_batched_d4_decode_step")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8 codes x s8 activation digits -> s32 (31-bit per-group fixed-point x), fp32 scales/accumulate",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1, "weight_bytes_per_step_d4": step.bytes_d4,
                   "weight_bytes_per_escalation": step.bytes_res, "escalated_steps": n_esc,
                   "gate_thresholds": {"entropy": step.tau_h, "margin": step.tau_m,
                                       "escalating_sets": f"{step.NESC} of {step.NSETS}"},
                   "l2": "inputs larger than L2 (316.6 MB of weights read per step vs 126 MB L2)",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "tokens_per_s": tok_s, "hbm_frac": value / world / peak, "peak_gbs": peak, "peak_kind": peak_kind,
        "hbm_frac_of_8tbs_spec": value / world / SPEC_HBM_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": tr["bytes_per_launch"] if tr else None,
                     "kernel": "plane_gemv_kernel (fl_gemv_batched_gate, 197 problems, D4, logit gate fused)",
                     "us_per_launch": tk * 1e6, "bytes_per_launch": step.bytes_d4, **spread,
                     "frac_statistic": "achieved and frac use us_per_launch, the mean over back-to-back "
                                       "graph replays of the launch; frac_p50 uses the median of 100 "
                                       "replays each bracketed by its own events (graph-launch overhead "
                                       "included)",
                     "frac_of_8tbs_spec": achieved / SPEC_HBM_GBS,
                     # plane GEMV launches per step (the D4 pass plus the escalated steps' residual
                     # pass, both full reads of the store) x time per launch / step time
                     "share_of_step": (1 + n_esc / args.steps) * tk / (t / args.steps) if t > 0 else None},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": step.h2d_bytes,
                "d2h_bytes_per_step": 32, "steps": e2e_steps,
                "tokens_per_s": job_rate(e2e_steps, world, te)},
        "gpu_launches": 2 * args.steps,  # D4 pass + conditional residual pass (returns at once when not needed)
        "device_status": status,
        "parity_sample": parity,
        "timed_graphs": f"{args.steps // NS} x {NS}-step graph + 1 x {rem}-step graph",
        "clocks": clk.summary(),
        "kernels": extra,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_shard(args, rank, world, local_rank):
    """The decode step with the read split over the ranks (strong scaling: the step's total work is
    fixed; each rank reads its byte-balanced share of every layer's blocks, x replicated). Per step:
    one batched D4 pass over the rank's block ranges that also reduces the rank's share of the
    head's logits to the gate's partial (the vocabulary is split with the head's blocks); one
    all-gather of the partials and the merge on the device, identical on every rank; the D4->D8
    residual pass over the rank's ranges (partial fused too), run or skipped on the device by the
    merged escalate flag; its partials gathered and merged again; one all-gather of the output
    rows. Device time with CUDA events, max over ranks."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from variable_precision_weight_b200 import fl, shard, synth

    torch.cuda.set_device(local_rank)
    if not dist.is_initialized():   # one rank launched without torchrun
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29531")
        dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(2000)                       # every rank builds the same model
    shapes = synth.qwen3_step_shapes()
    layers, lv_host, to8 = [], [], []
    for _, o, i in shapes:
        layers.append((plane_layer(torch, fl, o, i, gen), o, i,
                       torch.full((o // 64,), 2, dtype=torch.uint8, device="cuda")))
        lv_host.append(np.full(o // 64, 2, np.uint8))
        to8.append(torch.full((o // 64,), 4, dtype=torch.uint8, device="cuda"))
    plans = shard.plan(lv_host, [i for _, _, i in shapes], world)
    rows, total = shard.rank_rows(plans, rank)
    counts = [shard.rank_rows(plans, r)[1] for r in range(world)]
    NS, NESC = 8, 2
    tot_in = sum(i for _, _, i in shapes)
    xs = torch.empty((NS, tot_in), dtype=torch.int16, device="cuda")
    for j in range(NS):
        xs[j].copy_(torch.from_numpy(synth.bf16_normal((tot_in,), 3000, j).view("int16")))
    # as wide as the largest rank's rows, so the row exchange sends it with no copy
    y_local = torch.zeros(max(counts), dtype=torch.float32, device="cuda")
    y_all = torch.zeros(world * max(counts), dtype=torch.float32, device="cuda")
    p_all = torch.zeros(world * fl.GATE_PARTIAL_BYTES, dtype=torch.uint8, device="cuda")
    prob_d4, prob_r = [], []
    for j in range(NS):
        lay, oi = [], 0
        for st, o, i, lv in layers:
            lay.append((st, o, i, lv, xs[j, oi:oi + i]))
            oi += i
        it4, placed = shard.local_items(lay, plans, rank, y_local)
        itr, _ = shard.local_items(lay, plans, rank, y_local, 1, to8)
        prob_d4.append(fl.gemv_problems(it4))
        prob_r.append(fl.gemv_problems(itr))
    n_items = len(placed)
    head = len(shapes) - 1
    h_idx, h_off, h_rows = next(((k, off, n) for k, (li, off, n) in enumerate(placed) if li == head), (0, 0, 0))
    h_first = 64 * plans[head][rank]
    assert h_rows > 0 and n_items == len(shapes), "every rank holds blocks of every layer at these shapes"
    part = torch.zeros(fl.GATE_PARTIAL_BYTES, dtype=torch.uint8, device="cuda")
    gates = torch.zeros(8, dtype=torch.int32, device="cuda")
    esc = gates[4:5].view(torch.uint8)[0:1]
    runs = torch.zeros(1, dtype=torch.int32, device="cuda")
    # each pass reduces the rank's head rows to the gate's partial in its own launch (the fused
    # gate in partial mode); the partials are gathered and merged into the step's gate
    gsz = fl.fl_gemv_gate_workspace_bytes(1)
    gws = torch.zeros(gsz, dtype=torch.uint8, device="cuda")
    spec_p = fl.gate_spec(h_idx, 0.0, 0.0, None, None, None, None, gws, gsz)
    tau = [1e30, -1.0]

    def merge():
        allp = shard.gather_partials(part, world, out=p_all)
        fl.fl_logit_gate_merge(allp, world, 1, tau[0], tau[1], gates[0:1].view(torch.float32),
                               gates[1:2].view(torch.float32), gates[2:4], esc)

    def d4(j):
        fl.fl_gemv_batched_gate_partial(prob_d4[j], n_items, 1, 0, spec_p, None, None, h_first, part)
        merge()

    def step(j):
        d4(j)
        fl.fl_gemv_batched_gate_partial(prob_r[j], n_items, 1, 1, spec_p, esc, runs, h_first, part)
        merge()
        shard.gather_rows(y_local, counts, out=y_all)

    # entropy threshold from the merged D4 gate so NESC of the NS input sets escalate
    H = []
    for j in range(NS):
        d4(j)
        H.append(float(gates[0:1].view(torch.float32).item()))
    h = sorted(H, reverse=True)
    tau[0] = 0.5 * (h[NESC - 1] + h[NESC])
    # one CUDA graph per input set (NCCL's collectives captured with the kernels), after one
    # eager pass of each so every communicator is set up before capture
    for j in range(NS):
        step(j)
    torch.cuda.synchronize()
    graphs = []
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        for j in range(NS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step(j)
            graphs.append(g)
    torch.cuda.current_stream().wait_stream(cap)
    torch.cuda.synchronize()
    clk = ClockSampler(local_rank)
    try:
        with clk:
            for k in range(args.warmup):
                graphs[k % NS].replay()
            runs.zero_()
            dist.barrier()
            torch.cuda.synchronize()
            clk.mark("before_timed")
            t = time_loop(torch, lambda k: graphs[k % NS].replay(), args.steps)
            clk.mark("after_timed")
        t = max_over_ranks(t, world)
    finally:
        torch.cuda.synchronize()
        del graphs      # graphs holding NCCL calls go before the process group does
    device_ok(fl, "the sharded steps")
    n_esc = int(runs.item())
    bytes_d4 = sum((o // 64) * plane_bytes(i, 2) for _, o, i in shapes)
    bytes_res = sum((o // 64) * (256 * (i // 128) + 2048 * (i // 128) * 2) for _, o, i in shapes)
    if rank != 0:
        return 0
    # every rank takes the same gate decision, so rank 0's count of residual passes is the job's
    value = (args.steps * bytes_d4 + n_esc * bytes_res) / t / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None,
            "dtype": "u8 codes x s8 activation digits -> s32 (31-bit per-group fixed-point x), fp32 scales/accumulate",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch": 1,
                       "parallelism": f"every layer's 64-row blocks split over {world} ranks by the bytes read",
                       "rows_per_rank": counts, "escalated_steps": n_esc, "input_sets": NS,
                       "l2": "weights (0.33 GB at D4) larger than L2; input sets rotate"},
            "tokens_per_s": args.steps / t, "clocks": clk.summary(),
            "gpu_launches": 4 * args.steps}   # D4 pass, residual pass (partials fused), 2 merges; NCCL's not counted
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.shard:
            return run_shard(args, rank, world, local_rank)
        return run_fl(args, rank, world, local_rank)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
