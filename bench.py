#!/usr/bin/env python
"""Benchmark of the trellis-coded FP4 hot path on B200.

One step = every step of the path over one batch on the 32-expert, hidden-2880 MoE layer
(per expert gate_up 5760x2880 and down 2880x2880; 2 bits/weight trellis streams, one UE8M0 scale
per 32 weights, seg_len 32), inputs resident in HBM:
  1. expansion of every expert into a resident packed MXFP4 tensor (HEPH serving mode 2):
     trellis_decode_to_mxfp4 on gate_up [32*5760][2880] and down [32*2880][2880];
  2. routing of one token (N(0,1) logits, top-4, softmax) and the fused-decode grouped MoE at
     batch 1 (HEPH serving mode 1): trellis_moe_route + trellis_grouped_moe;
  3. the batch-1 fused decode GEMV over every expert matrix of the layer: trellis_gemv on
     gate_up [32*5760][2880] and down [32*2880][2880] with bf16 N(0,1) activations.
Metric: decoded weights/s over the whole step (and HBM GB/s of the dominant kernel).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tcf4|reference]
With N > 1 it runs under torchrun, one independent replica of the step per GPU (weak scaling).
"""
import argparse
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

E, H, I, K_TOP, T = 32, 2880, 2880, 4, 1
SEG = 32
METRIC = "fused trellis-decode GEMV: decoded weights/s and HBM GB/s (% of B200 peak)"
UNIT = "decoded weights/s"
WORKLOAD = ("32-expert hidden-2880 MoE layer (gate_up 5760x2880 + down 2880x2880 per expert, 2-bit trellis, "
            "UE8M0/32, seg_len 32): expand all experts to MXFP4 + route and fused-decode grouped MoE at batch 1 "
            "(top-4) + batch-1 fused decode GEMV over every expert matrix")
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic per launch measured with ncu (dram__bytes_read.sum + dram__bytes_write.sum), per
# decoded weight, for the kernel as it is now; None when not yet measured for this kernel version.
# gemv: 153,369,088 bytes over the 530,841,600 weights of the gate_up launch; expand:
# 375,607,040 bytes over the same weights (profiles/k_mma_gemv_gate_up.md, profiles/k_expand_gate_up.md).
NCU_TRAFFIC_B_PER_WEIGHT = {"expand": 375607040 / 530841600, "gemv": 153748224 / 530841600}


def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples every 50 ms for one GPU while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index=0):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        self.t_start = time.time()

    def mark(self):
        return time.time()

    def stop(self, t0, t1):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        except Exception:
            return None
        finally:
            try:
                os.remove(self.path)
            except Exception:
                pass
        if not rows:
            return {"samples": 0}
        # nvidia-smi -lms writes one row per period from start; map rows to wall-clock times
        period = 0.05
        times = [self.t_start + i * period for i in range(len(rows))]
        inside = [r for r, t in zip(rows, times) if t0 - period <= t <= t1 + period]
        window = "timed"
        if not inside:
            inside = rows
            window = "whole run (timed region shorter than the sampling period)"
        def num(v):
            try:
                return float(v)
            except Exception:
                return None
        sm = [num(r[1]) for r in inside if num(r[1]) is not None]
        mx = [num(r[2]) for r in inside if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in inside for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside), "window": window,
                "power_w_max": max([num(r[3]) for r in inside if num(r[3]) is not None] or [0.0])}


# ----------------------------------------------------------------------------- the step

class Step:
    """Device buffers and the 9 launches of one step (all on the current stream)."""

    def __init__(self, seed, device):
        import trellis_coded_fp4_b200 as tc
        from trellis_coded_fp4_b200 import synth
        self.tc = tc
        self.layer = synth.moe_layer(E, H, I, seed=seed)
        lay = self.layer
        self.G = tc.TrellisMatrix.from_numpy(lay.gu_stream, lay.gu_scales, E * 2 * I, H, SEG, device)
        self.D = tc.TrellisMatrix.from_numpy(lay.dn_stream, lay.dn_scales, E * H, I, SEG, device)
        # expert views onto the same resident buffers
        gu = self.G.stream.view(E, -1)
        gus = self.G.scales.view(E, -1)
        dn = self.D.stream.view(E, -1)
        dns = self.D.scales.view(E, -1)
        self.M = tc.MoEWeights([tc.TrellisMatrix(gu[e], gus[e], 2 * I, H, SEG) for e in range(E)],
                               [tc.TrellisMatrix(dn[e], dns[e], H, I, SEG) for e in range(E)], H, I)
        nvar = 8  # rotating activations / logits
        self.x = [synth.activations(T, H, seed=seed, sub=i).to(device) for i in range(nvar)]
        self.xd = [synth.activations(T, I, seed=seed, sub=100 + i).to(device) for i in range(nvar)]
        self.logits = [synth.logits(T, E, seed=seed, sub=i).to(device) for i in range(nvar)]
        self.nibG = torch.empty((E * 2 * I, H // 2), dtype=torch.uint8, device=device)
        self.scG = torch.empty((E * 2 * I, H // 32), dtype=torch.uint8, device=device)
        self.nibD = torch.empty((E * H, I // 2), dtype=torch.uint8, device=device)
        self.scD = torch.empty((E * H, I // 32), dtype=torch.uint8, device=device)
        self.yG = torch.empty((T, E * 2 * I), dtype=torch.bfloat16, device=device)
        self.yD = torch.empty((T, E * H), dtype=torch.bfloat16, device=device)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        self.ids = torch.empty((T, K_TOP), dtype=torch.int32, device=device)
        self.wts = torch.empty((T, K_TOP), dtype=torch.float32, device=device)
        self.ws = torch.empty(self.M.workspace_bytes(T, K_TOP), dtype=torch.uint8, device=device)
        self.wsG = torch.empty(max(1, tc.gemv_workspace_bytes(self.G, T)), dtype=torch.uint8, device=device)
        self.wsD = torch.empty(max(1, tc.gemv_workspace_bytes(self.D, T)), dtype=torch.uint8, device=device)
        # expansion 2, route 1, grouped MoE 3 (the split of x, gate/up whose epilogue also splits h,
        # down), GEMV 2 x (split + product)
        self.launches_per_step = 2 + 1 + 3 + 4
        self.nG, self.nD = E * 2 * I * H, E * H * I
        self.moe_weights = K_TOP * (2 * I * H + H * I)  # distinct experts at T = 1: exactly k
        self.weights_per_step = self.nG + self.nD + self.moe_weights + self.nG + self.nD

    def run(self, i, ev=None, only=None):
        tc = self.tc
        v = i % len(self.x)
        if only is not None:
            calls = {"expand_gate_up": lambda: tc.decode_to_mxfp4(self.G, self.nibG, self.scG),
                     "expand_down": lambda: tc.decode_to_mxfp4(self.D, self.nibD, self.scD),
                     "route": lambda: tc.moe_route(self.logits[v], K_TOP, self.ids, self.wts),
                     "grouped_moe": lambda: tc.grouped_moe(self.M, self.x[v], self.ids, self.wts, self.out, self.ws),
                     "gemv_gate_up": lambda: tc.gemv(self.G, self.x[v], self.yG, self.wsG),
                     "gemv_down": lambda: tc.gemv(self.D, self.xd[v], self.yD, self.wsD)}
            if only == "grouped_moe":
                calls["route"]()
            calls[only]()
            return
        def mark(name):
            if ev is not None:
                e = torch.cuda.Event(enable_timing=True)
                e.record()
                ev.append((name, e))
        mark("expand_gate_up")
        tc.decode_to_mxfp4(self.G, self.nibG, self.scG)
        mark("expand_down")
        tc.decode_to_mxfp4(self.D, self.nibD, self.scD)
        mark("route")
        tc.moe_route(self.logits[v], K_TOP, self.ids, self.wts)
        mark("grouped_moe")
        tc.grouped_moe(self.M, self.x[v], self.ids, self.wts, self.out, self.ws)
        mark("gemv_gate_up")
        tc.gemv(self.G, self.x[v], self.yG, self.wsG)
        mark("gemv_down")
        tc.gemv(self.D, self.xd[v], self.yD, self.wsD)
        mark("end")

    # the next row beyond the step: products read straight from the resident MXFP4 tensors that the
    # step's expansion calls wrote (HEPH serving mode 2, consumer side)
    def mx_weights(self):
        tc = self.tc
        if not hasattr(self, "_mxG"):
            self._mxG = tc.Mxfp4Matrix(self.nibG, self.scG, E * 2 * I, H)
            self._mxD = tc.Mxfp4Matrix(self.nibD, self.scD, E * H, I)
            ng, sg, nd, sd = self.nibG.view(E, -1), self.scG.view(E, -1), self.nibD.view(E, -1), self.scD.view(E, -1)
            self._mxM = tc.Mxfp4MoEWeights([tc.Mxfp4Matrix(ng[e], sg[e], 2 * I, H) for e in range(E)],
                                           [tc.Mxfp4Matrix(nd[e], sd[e], H, I) for e in range(E)], H, I)
            self._mxws = torch.empty(max(1, self._mxM.workspace_bytes(T, K_TOP)), dtype=torch.uint8,
                                     device=self.nibG.device)
        return self._mxG, self._mxD, self._mxM

    def run_mx(self, name, i):
        tc = self.tc
        G, D, M = self.mx_weights()
        v = i % len(self.x)
        if name == "mxfp4_gemv_gate_up":
            tc.mxfp4_gemv(G, self.x[v], self.yG, self.wsG)
        elif name == "mxfp4_gemv_down":
            tc.mxfp4_gemv(D, self.xd[v], self.yD, self.wsD)
        else:
            tc.moe_route(self.logits[v], K_TOP, self.ids, self.wts)
            tc.mxfp4_grouped_moe(M, self.x[v], self.ids, self.wts, self.out, self._mxws)

    def mx_algo_bytes(self):
        def gemv(rows, cols):
            return rows * cols // 2 + rows * cols // 32 + 2 * cols * T + 2 * rows * T
        return {"mxfp4_gemv_gate_up": gemv(E * 2 * I, H), "mxfp4_gemv_down": gemv(E * H, I),
                "mxfp4_grouped_moe": K_TOP * (gemv(2 * I, H) + gemv(H, I))}

    # algorithmic bytes per call (what the method must move)
    def algo_bytes(self):
        def expand(rows, cols):
            return rows * cols // 4 + rows * cols // 2 + 2 * (rows * cols // 32)
        def gemv(rows, cols):
            return rows * cols // 4 + rows * cols // 32 + 2 * cols * T + 2 * rows * T
        moe = K_TOP * (gemv(2 * I, H) + gemv(H, I))
        return {"expand_gate_up": expand(E * 2 * I, H), "expand_down": expand(E * H, I),
                "route": 4 * T * E + 8 * T * K_TOP, "grouped_moe": moe,
                "gemv_gate_up": gemv(E * 2 * I, H), "gemv_down": gemv(E * H, I)}

    def weights(self):
        return {"expand_gate_up": self.nG, "expand_down": self.nD, "route": 0, "grouped_moe": self.moe_weights,
                "gemv_gate_up": self.nG, "gemv_down": self.nD}


def batch_sweep(step, device, n):
    """Fused decode GEMV and MXFP4 GEMV of the 184320 x 2880 gate_up matrix at T = 1 .. 32: CUDA-event
    time per call over n calls back to back after warm-up, algorithmic bytes (stream or nibbles, scales,
    activations and outputs) per second, and the fraction of the measured copy peak."""
    tc = step.tc
    peak, _ = measured_hbm_peak()
    G = step.G
    Gm = tc.Mxfp4Matrix(step.nibG, step.scG, G.rows, G.cols)
    tc.decode_to_mxfp4(G, step.nibG, step.scG)
    out = {"sweep": "gemv gate_up 184320x2880", "calls": n, "peak_gb_s": peak, "rows": []}
    for T in (1, 2, 4, 8, 16, 32):
        x = synth_activations(T, G.cols, device)
        y = torch.empty((T, G.rows), dtype=torch.bfloat16, device=device)
        row = {"T": T}
        for name, fn, w, wbytes in (("fused", tc.gemv, G, G.rows * G.cols // 4),
                                    ("mxfp4", tc.mxfp4_gemv, Gm, G.rows * G.cols // 2)):
            ws = torch.empty(max(1, tc.gemv_workspace_bytes(G, T)), dtype=torch.uint8, device=device)
            for _ in range(3):
                fn(w, x, y, ws)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(n):
                fn(w, x, y, ws)
            e1.record()
            torch.cuda.synchronize()
            us = 1e3 * e0.elapsed_time(e1) / n
            nbytes = wbytes + G.rows * G.cols // 32 + 2 * G.cols * T + 2 * G.rows * T
            gbs = nbytes / (us * 1e-6) / 1e9
            row[name] = {"us": round(us, 2), "gb_s": round(gbs, 1), "frac": round(gbs / peak, 3)}
        out["rows"].append(row)
    out["timeouts"] = tc.device_timeouts()
    return out


def synth_activations(T, cols, device):
    from trellis_coded_fp4_b200 import synth
    return synth.activations(T, cols, seed=synth.SEED_BASE + 90 + T).to(device)


def run_e2e(step, steps, device):
    """The same step through the public API with HOST buffers: every input (stream words, scales,
    activations, logits) is copied from pinned host memory and every output (MXFP4 nibbles and
    scales, GEMV outputs, MoE output) is copied back, inside the timed region."""
    lay = step.layer
    h_gu = torch.from_numpy(lay.gu_stream.view("int32").reshape(-1)).pin_memory()
    h_gus = torch.from_numpy(lay.gu_scales.reshape(-1)).pin_memory()
    h_dn = torch.from_numpy(lay.dn_stream.view("int32").reshape(-1)).pin_memory()
    h_dns = torch.from_numpy(lay.dn_scales.reshape(-1)).pin_memory()
    h_x = [x.cpu().pin_memory() for x in step.x]
    h_xd = [x.cpu().pin_memory() for x in step.xd]
    h_lg = [lg.cpu().pin_memory() for lg in step.logits]
    outs = [step.nibG, step.scG, step.nibD, step.scD, step.yG, step.yD, step.out]
    h_outs = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h2d = sum(t.numel() * t.element_size() for t in (h_gu, h_gus, h_dn, h_dns, h_x[0], h_xd[0], h_lg[0]))
    d2h = sum(t.numel() * t.element_size() for t in h_outs)

    def one(i):
        v = i % len(h_x)
        step.G.stream.copy_(h_gu, non_blocking=True)
        step.G.scales.copy_(h_gus, non_blocking=True)
        step.D.stream.copy_(h_dn, non_blocking=True)
        step.D.scales.copy_(h_dns, non_blocking=True)
        step.x[v].copy_(h_x[v], non_blocking=True)
        step.xd[v].copy_(h_xd[v], non_blocking=True)
        step.logits[v].copy_(h_lg[v], non_blocking=True)
        step.run(i)
        for o, h in zip(outs, h_outs):
            h.copy_(o, non_blocking=True)

    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        one(i)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return {"value": step.weights_per_step / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


# ----------------------------------------------------------------------------- CPU oracle sample

def oracle_sample(layer, x_bits, logits, stride):
    """Run the oracle on every `stride`-th row of each matrix the step touches, doing per row the
    work the step does (expand; multiply; MoE gate/up then down). Returns decoded weights."""
    import oracle
    n = 0
    gu_all = layer.gu_stream.reshape(E * 2 * I, H // 32, 2)
    gus_all = layer.gu_scales.reshape(E * 2 * I, H // 32)
    dn_all = layer.dn_stream.reshape(E * H, I // 32, 2)
    dns_all = layer.dn_scales.reshape(E * H, I // 32)
    for st, sc, rows, cols in ((gu_all, gus_all, E * 2 * I, H), (dn_all, dns_all, E * H, I)):
        sel = np.arange(0, rows, stride)
        oracle.expand_mxfp4(st[sel], sc[sel], len(sel), cols, SEG)
        oracle.gemv(st, sc, rows, cols, SEG, x_bits, row_ids=sel)
        n += 2 * len(sel) * cols
    ids, w = oracle.route(logits, K_TOP)
    for j in range(K_TOP):
        e = int(ids[0, j])
        ri = np.arange(0, I, stride)
        y, _ = oracle.gemv(layer.gu_stream[e], layer.gu_scales[e], 2 * I, H, SEG, x_bits,
                           row_ids=np.concatenate([ri, I + ri]))
        h = np.zeros((1, I), np.uint16)
        h[0, ri] = oracle.bf16_round_array(oracle.silu(y[0, :len(ri)]) * y[0, len(ri):])
        rn = np.arange(0, H, stride)
        oracle.gemv(layer.dn_stream[e], layer.dn_scales[e], H, I, SEG, h, row_ids=rn)
        n += 2 * len(ri) * H + len(rn) * I
    return n


def cpu_baseline(layer, seed, stride=16):
    from trellis_coded_fp4_b200 import synth
    xb = synth.bf16_bits(synth.activations(T, H, seed=seed))
    lg = synth.logits(T, E, seed=seed).numpy()
    t0 = time.perf_counter()
    n = oracle_sample(layer, xb, lg, stride)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": 1, "kind": "oracle", "seconds": dt,
            "sample": (f"every {stride}th row of each matrix the step touches (expansion and batch-1 GEMV of "
                       f"gate_up and down; MoE gate/up rows and down rows of the 4 routed experts), "
                       f"{n} decoded weights, single-threaded plain C oracle")}


# ----------------------------------------------------------------------------- arms

def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over all ranks (x itself on one process): replicas are timed by the slowest."""
    t = torch.tensor([x], device=device, dtype=torch.float64)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, weights_per_step: int, steps: int, ms_total: float) -> float:
    """Decoded weights/s of the whole job: every replica decodes weights_per_step per step."""
    return world * weights_per_step * steps / (ms_total * 1e-3)


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from trellis_coded_fp4_b200 import synth
    seed = synth.SEED_BASE + 1
    layer = synth.moe_layer(E, H, I, seed=seed)
    stride = 256
    xb = synth.bf16_bits(synth.activations(T, H, seed=seed))
    lg = synth.logits(T, E, seed=seed).numpy()
    for _ in range(args.warmup):
        oracle_sample(layer, xb, lg, stride)
    t0 = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        n += oracle_sample(layer, xb, lg, stride)
    dt = time.perf_counter() - t0
    value = n / dt
    sample = (f"every {stride}th row of each matrix the step touches, {n // max(args.steps, 1)} decoded weights "
              "per step, single-threaded plain C oracle")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample}, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)  # ~0.3 s timed: several clock samples
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tcf4", choices=["tcf4", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default=None,
                    help="run only this call of the step (e.g. gemv_gate_up), for profiling one kernel")
    ap.add_argument("--sweep", action="store_true",
                    help="batch sweep instead of the step: fused decode GEMV and MXFP4 GEMV of the gate_up "
                         "matrix at T = 1, 2, 4, 8, 16, 32 (one JSON line, not a bench line)")
    args = ap.parse_args()
    if args.impl == "reference":
        return reference_arm(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    from trellis_coded_fp4_b200 import build, synth
    build.build()
    seed = synth.SEED_BASE + 1 + rank
    step = Step(seed, device)
    if args.sweep:
        print(json.dumps(batch_sweep(step, device, max(10, args.steps // 10))))
        return 0
    if args.only is not None:  # profiling mode: a few launches of one call, no timing line
        for i in range(args.warmup + args.steps):
            step.run(i, only=args.only)
        torch.cuda.synchronize()
        print(json.dumps({"only": args.only, "launches": args.warmup + args.steps,
                          "timeouts": step.tc.device_timeouts()}))
        return 0

    for i in range(max(args.warmup, 3)):
        step.run(i)
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.15)
    # The step is timed with events at its two ends only: an event between two calls would sit
    # between their kernels in the stream and keep a call from overlapping its predecessor's tail
    # (the kernels are dependent launches).
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tw0 = time.time()
    start.record()
    for i in range(args.steps):
        step.run(i)
    end.record()
    torch.cuda.synchronize()
    tw1 = time.time()
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop(tw0, tw1)
    ms_total = max_over_ranks(start.elapsed_time(end), dist, device)
    ms_per_step = ms_total / args.steps

    # per-call durations from a second pass with an event before each call (on the launching
    # stream); these set the roofline of the dominant call and the shares
    events = []
    n_per = max(10, args.steps // 4)
    for i in range(n_per):
        step.run(i, events)
    torch.cuda.synchronize()
    per = {}
    for (name, e0), (_, e1) in zip(events[:-1], events[1:]):
        if name == "end":
            continue
        per.setdefault(name, []).append(e0.elapsed_time(e1))
    avg_us = {k: 1e3 * statistics.mean(v) for k, v in per.items()}
    algo = step.algo_bytes()
    wts = step.weights()
    peak, peak_kind = measured_hbm_peak()
    kernels = {}
    for k, us in avg_us.items():
        gbs = algo[k] / (us * 1e-6) / 1e9
        kernels[k] = {"avg_us": round(us, 3), "algo_bytes": algo[k], "gb_s": round(gbs, 1),
                      "frac_of_measured_hbm": round(gbs / peak, 4), "frac_of_8tbs": round(gbs / 8000.0, 4),
                      "decoded_weights_per_s": (wts[k] / (us * 1e-6)) if wts[k] else None,
                      "share": round(us / (1e3 * ms_per_step), 4), "calls": n_per}
    dom = max(avg_us, key=avg_us.get)
    dom_gbs = algo[dom] / (avg_us[dom] * 1e-6) / 1e9
    kind = "expand" if dom.startswith("expand") else ("gemv" if dom.startswith("gemv") else None)
    tpw = NCU_TRAFFIC_B_PER_WEIGHT.get(kind) if kind else None
    roofline = {"bound": "hbm", "achieved": round(dom_gbs, 1), "peak": peak, "unit": "GB/s",
                "frac": round(dom_gbs / peak, 4), "traffic": (tpw * wts[dom]) if tpw else None,
                "kernel": dom, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback 6650 GB/s"}

    value = job_value(world, step.weights_per_step, args.steps, ms_total)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": T, "top_k": K_TOP, "experts": E, "hidden": H,
                       "intermediate": I, "seg_len": SEG, "decoded_weights_per_step": step.weights_per_step,
                       "l2": "inputs larger than L2 (each step streams >900 MB of stream/MXFP4 bytes through L2)",
                       "parallelism": f"replicas x{world}",
                       "arithmetic": "decode: u32 bit logic; products: block-scaled MXFP4 tensor-core MMA (activations as "
                                     "six E2M1 terms per 32-block), fp32 accumulation"},
            "roofline": roofline, "kernels": kernels,
            "gpu_launches": step.launches_per_step * args.steps, "clocks": clocks}

    # the next row (outside the step): products from the resident MXFP4 tensors, each call timed on
    # its own with CUDA events after warm-up, inputs > L2 (the tensors are 423 MB)
    mx = {}
    for name, nbytes in step.mx_algo_bytes().items():
        for i in range(3):
            step.run_mx(name, i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_mx = max(10, args.steps // 4)
        e0.record()
        for i in range(n_mx):
            step.run_mx(name, i)
        e1.record()
        torch.cuda.synchronize()
        us = 1e3 * e0.elapsed_time(e1) / n_mx
        gbs = nbytes / (us * 1e-6) / 1e9
        mx[name] = {"avg_us": round(us, 3), "algo_bytes": nbytes, "gb_s": round(gbs, 1),
                    "frac_of_measured_hbm": round(gbs / peak, 4), "frac_of_8tbs": round(gbs / 8000.0, 4),
                    "calls": n_mx, "note": "includes route" if name == "mxfp4_grouped_moe" else ""}
    # the upstream encoder (D-weighted Viterbi): 296 rows of the gate_up matrix re-encoded from their
    # decoded values with random D, segments of 32 weights; compute-bound, timed over 3 calls
    enc_rows, enc_cols = 296, H
    gen = torch.Generator(device=device).manual_seed(seed)
    et = torch.randn(enc_rows, enc_cols, dtype=torch.float64, device=device, generator=gen)
    eD = torch.rand(enc_rows, enc_cols, dtype=torch.float64, device=device, generator=gen) + 0.1
    esc = step.G.scales[: enc_rows * (enc_cols // 32)]
    step.tc.encode(et, eD, esc, 32)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        step.tc.encode(et, eD, esc, 32)
    e1.record()
    torch.cuda.synchronize()
    enc_ms = e0.elapsed_time(e1) / 3
    encoder = {"ms_per_call": round(enc_ms, 3), "weights": enc_rows * enc_cols, "seg_len": 32,
               "weights_per_s": enc_rows * enc_cols / (enc_ms * 1e-3), "bound": "alu",
               "note": "2^16 candidate paths per weight, fp64 costs evaluated exactly (no fused operations)"}
    # the interleaved-packing repack of the gate_up stream (184320 x 2880: 133 MB read, 133 MB
    # written per call, more than L2 holds), back to back after warm-up
    rp_out = torch.empty_like(step.G.stream)
    rp_rows, rp_cols = step.G.rows, step.G.cols
    for _ in range(3):
        step.tc.repack_interleaved(step.G.stream, rp_rows, rp_cols, out=rp_out)
    torch.cuda.synchronize()
    n_rp = max(10, args.steps // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_rp):
        step.tc.repack_interleaved(step.G.stream, rp_rows, rp_cols, out=rp_out)
    e1.record()
    torch.cuda.synchronize()
    rp_us = 1e3 * e0.elapsed_time(e1) / n_rp
    rp_bytes = 16 * rp_rows * (rp_cols // 32)
    rp_gbs = rp_bytes / (rp_us * 1e-6) / 1e9
    repack = {"avg_us": round(rp_us, 3), "algo_bytes": rp_bytes, "gb_s": round(rp_gbs, 1),
              "frac_of_measured_hbm": round(rp_gbs / peak, 4), "frac_of_8tbs": round(rp_gbs / 8000.0, 4),
              "calls": n_rp, "bound": "hbm", "note": "8 bytes read + 8 written per 32-weight block"}
    del rp_out
    # the E5M3 block-scale variant: the gate_up stream (184320 x 2880) with E5M3 scale bytes of the
    # same binades as its UE8M0 ones and random mantissas, batch 1, on the CUDA-core kernel
    g5 = torch.Generator(device=device).manual_seed(seed + 5)
    m5 = torch.randint(0, 8, step.G.scales.shape, dtype=torch.int32, device=device, generator=g5)
    sc5 = (((step.G.scales.to(torch.int32) - 112) << 3) | m5).to(torch.uint8)
    W5 = step.tc.TrellisMatrix(step.G.stream, sc5, step.G.rows, step.G.cols, step.G.seg_len)
    y5 = torch.empty((T, W5.rows), dtype=torch.bfloat16, device=device)
    for i in range(3):
        step.tc.gemv_e5m3(W5, step.x[i % len(step.x)], out=y5)
    torch.cuda.synchronize()
    n5 = max(10, args.steps // 20)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n5):
        step.tc.gemv_e5m3(W5, step.x[i % len(step.x)], out=y5)
    e1.record()
    torch.cuda.synchronize()
    g5_us = 1e3 * e0.elapsed_time(e1) / n5
    g5_bytes = step.algo_bytes()["gemv_gate_up"]
    g5_gbs = g5_bytes / (g5_us * 1e-6) / 1e9
    e5m3 = {"avg_us": round(g5_us, 3), "algo_bytes": g5_bytes, "gb_s": round(g5_gbs, 1),
            "frac_of_measured_hbm": round(g5_gbs / peak, 4), "frac_of_8tbs": round(g5_gbs / 8000.0, 4),
            "decoded_weights_per_s": W5.rows * W5.cols / (g5_us * 1e-6), "calls": n5,
            "note": "CUDA-core kernel (a block-scaled MMA takes power-of-two scales only)"}
    del W5, sc5, m5, y5
    line["next_rows"] = {"mxfp4_consumer": mx, "encoder": encoder, "repack_interleaved": repack,
                         "gemv_e5m3_gate_up": e5m3,
                         "description": "products read straight from the resident MXFP4 tensors the step's "
                         "expansion wrote (HEPH serving mode 2), the D-weighted Viterbi encoder, the "
                         "interleaved-to-planar stream repack and the E5M3 block-scale GEMV; outside the "
                         "step and its value"}

    if rank == 0:
        line["e2e"] = run_e2e(step, args.e2e_steps, device)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(step.layer, seed)
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
