#!/usr/bin/env python
"""Benchmark of the batch-1 fused trellis-decode GEMV on B200, with every other row of the path.

Headline (the metric): one step = one batch-1 fused decode GEMV, y = W x, on the gate_up matrices
of all 32 experts of the hidden-2880 MoE layer stacked into one matrix (184320 x 2880, 2-bit
trellis stream, one UE8M0 scale per 32 weights, seg_len 32; bf16 N(0,1) activations, bf16 out),
through trellis_gemv_tiled (the activation split and the decode-MMA product: two launches), the
weights' UE8M0 scales held as scale tiles (the same bytes, rearranged once at load time by
trellis_make_scale_tiles, outside the timed region). Steps rotate over three distinct resident
matrices (450 MB, > 3x L2) and eight activation vectors, so no step finds its weights in L2.
value = decoded weights/s of the whole job; roofline = that call.

Extra rows, each timed on its own with CUDA events on the launching stream after warm-up:
  * gemv_gate_up_raw_scales: the headline call through trellis_gemv, scales in their [rows][cols/32]
    layout;
  * gemv_down: the same GEMV on the down matrices stacked (92160 x 2880), scale tiles;
  * expand: decode-only expansion of the whole layer into resident MXFP4 (gate_up + down);
  * moe_t1: routing + fused grouped MoE of the layer at batch 1, top-4 of 32;
  * moe_sweep: the same at T = 1, 2, 4, 8, 16, 32 with N(0,1) routing, and with every token on the
    same four experts (forced skew), with the kernel instance each call takes;
  * gemv_sweep: fused decode GEMV and MXFP4 GEMV of the gate_up stack at T = 1 .. 32;
  * single_2048: one 2048 x 2048 matrix at batch 1, back to back over 512 distinct matrices
    (576 MB) in a CUDA graph, and the single-call latency with L2 flushed before each call;
  * moe_7168: the 256-expert hidden-7168 layer (intermediate 2048, top-8, all 3.17 GB of experts
    resident) at T = 1, 8, 32;
  * mxfp4_consumer, encoder, repack_interleaved, gemv_e5m3_gate_up: the further rows.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tcf4|reference]
With N > 1 it runs under torchrun, one independent replica per GPU (weak scaling).
"""
import argparse
import concurrent.futures as cf
import json
import os
import platform
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

E, H, I, K_TOP = 32, 2880, 2880, 4
SEG = 32
ROT = 3     # distinct resident gate_up matrices the headline steps rotate over
NVAR = 8    # activation / logits variants
METRIC = "fused trellis-decode GEMV: decoded weights/s and HBM GB/s (% of B200 peak)"
UNIT = "decoded weights/s"
WORKLOAD = ("batch-1 fused trellis-decode GEMV on the gate_up matrices of all 32 experts of the hidden-2880 MoE "
            "layer stacked (184320 x 2880, 2-bit trellis, UE8M0 per 32, seg_len 32), bf16 N(0,1) x, bf16 y")
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0

# DRAM traffic of one launch of the product kernel on this workload, dram__bytes_read.sum +
# dram__bytes_write.sum (150,499,840 + 3,792,896 bytes) from
# `ncu --set full --clock-control none -k regex:k_mma -s 2 -c 1` of
# `python bench.py --only gemv_gate_up --warmup 2 --steps 1`, taken on the scale-tile kernel
# `k_mma<32, 0, 32, 0, 0, 1, 1, 1>` with the three-input-XOR decoders, the straight-line stage loop
# and the epilogue poller on sub-partition 3; set to None whenever that kernel changes, until taken
# again.
NCU_TRAFFIC_GEMV_GATE_UP = 154292736


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
        period = 0.05  # nvidia-smi -lms writes one row per period from its start
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


# ----------------------------------------------------------------------------- helpers

def gemv_bytes(rows, cols, T, bytes_per_weight=0.28125):
    """Algorithmic bytes of one product: weights (stream + scales, or nibbles + scales), x in, y out."""
    return int(rows * cols * bytes_per_weight) + 2 * cols * T + 2 * rows * T


def rate(nbytes, us, peak):
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"avg_us": round(us, 3), "algo_bytes": int(nbytes), "gb_s": round(gbs, 1),
            "frac_of_measured_hbm": round(gbs / peak, 4), "frac_of_8tbs": round(gbs / SPEC_HBM_GBS, 4)}


def time_calls(fn, n, warm=3):
    """Average CUDA-event time in microseconds of fn(i) over n calls back to back (after warm-up)."""
    for i in range(warm):
        fn(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        fn(i)
    e1.record()
    torch.cuda.synchronize()
    return 1e3 * e0.elapsed_time(e1) / n


def time_graph(fn, n, reps=5):
    """The n calls fn(0..n-1) captured once in a CUDA graph, replayed reps times: microseconds per
    call (launch overhead of the host excluded)."""
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(n):
                fn(i)
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / (reps * n)
    del g
    return us


def flush_l2(buf):
    buf.add_(1)  # read and write a buffer larger than L2


def rand_words(n_words, gen, device):
    """Uniform random 32-bit words (uniform 2-bit trellis symbols) as int32, on the device."""
    return torch.randint(-2 ** 31, 2 ** 31, (n_words,), dtype=torch.int64, device=device, generator=gen).to(torch.int32)


def rand_scales(n, lo, hi, gen, device):
    return torch.randint(lo, hi + 1, (n,), dtype=torch.int32, device=device, generator=gen).to(torch.uint8)


# ----------------------------------------------------------------------------- the 32-expert layer

class Layer:
    """The 32-expert hidden-2880 layer: stacked gate_up / down matrices (and per-expert views), plus
    ROT - 1 further random gate_up stacks for the headline rotation."""

    def __init__(self, seed, device):
        import trellis_coded_fp4_b200 as tc
        from trellis_coded_fp4_b200 import synth
        self.tc, self.device = tc, device
        self.layer = synth.moe_layer(E, H, I, seed=seed)
        lay = self.layer
        self.G = tc.TrellisMatrix.from_numpy(lay.gu_stream, lay.gu_scales, E * 2 * I, H, SEG, device)
        self.D = tc.TrellisMatrix.from_numpy(lay.dn_stream, lay.dn_scales, E * H, I, SEG, device)
        gen = torch.Generator(device=device).manual_seed(seed)
        self.Grot = [self.G] + [tc.TrellisMatrix(rand_words(self.G.stream.numel(), gen, device),
                                                 rand_scales(self.G.scales.numel(), 120, 126, gen, device),
                                                 self.G.rows, self.G.cols, SEG) for _ in range(ROT - 1)]
        # the scale tiles of every rotated matrix and of down, made once (load time)
        self.Trot = [tc.scale_tiles(g) for g in self.Grot]
        gu, gus = self.G.stream.view(E, -1), self.G.scales.view(E, -1)
        dn, dns = self.D.stream.view(E, -1), self.D.scales.view(E, -1)
        self.M = tc.MoEWeights([tc.TrellisMatrix(gu[e], gus[e], 2 * I, H, SEG) for e in range(E)],
                               [tc.TrellisMatrix(dn[e], dns[e], H, I, SEG) for e in range(E)], H, I)
        self.x = [synth.activations(1, H, seed=seed, sub=i).to(device) for i in range(NVAR)]
        self.xd = [synth.activations(1, I, seed=seed, sub=100 + i).to(device) for i in range(NVAR)]
        self.yG = torch.empty((1, E * 2 * I), dtype=torch.bfloat16, device=device)
        self.yD = torch.empty((1, E * H), dtype=torch.bfloat16, device=device)
        self.wsG = torch.empty(max(1, tc.gemv_workspace_bytes(self.G, 1)), dtype=torch.uint8, device=device)
        self.wsD = torch.empty(max(1, tc.gemv_workspace_bytes(self.D, 1)), dtype=torch.uint8, device=device)
        self.TD = tc.scale_tiles(self.D)
        self.launches_per_step = 2  # the activation split and the decode-MMA product

    def step(self, i):
        self.tc.gemv_tiled(self.Grot[i % ROT], self.Trot[i % ROT], self.x[i % NVAR], self.yG, self.wsG)

    def step_raw(self, i):
        self.tc.gemv(self.Grot[i % ROT], self.x[i % NVAR], self.yG, self.wsG)

    def run_only(self, name, i):
        """One call of one row (profiling mode)."""
        tc = self.tc
        if name == "gemv_gate_up":
            self.step(i)
        elif name == "gemv_gate_up_raw":
            self.step_raw(i)
        elif name == "gemv_down":
            tc.gemv_tiled(self.D, self.TD, self.xd[i % NVAR], self.yD, self.wsD)
        elif name == "expand_gate_up":
            self._expanded()
            tc.decode_to_mxfp4(self.G, self.nibG, self.scG)
        elif name == "grouped_moe":
            if not hasattr(self, "_moe1"):
                self._moe1 = self.moe_call(1)
            self._moe1(i)
        elif name.startswith("gemv_gate_up_t"):  # gemv_gate_up_t<T>: the tiled call at T tokens
            T = int(name[len("gemv_gate_up_t"):])
            if getattr(self, "_tT", None) != T:
                from trellis_coded_fp4_b200 import synth
                self._tT = T
                self._xT = synth.activations(T, H, seed=synth.SEED_BASE + 90 + T).to(self.device)
                self._yT = torch.empty((T, self.G.rows), dtype=torch.bfloat16, device=self.device)
                self._wsT = torch.empty(tc.gemv_workspace_bytes(self.G, T), dtype=torch.uint8, device=self.device)
            tc.gemv_tiled(self.G, self.Trot[0], self._xT, self._yT, self._wsT)
        elif name == "encoder":
            if not hasattr(self, "_enc"):
                g = torch.Generator(device=self.device).manual_seed(7)
                self._enc = encoder_inputs(self, 296, H, g, self.device)
            tc.encode(self._enc[0], self._enc[1], self._enc[2], 32)
        elif name == "gemv_e5m3":
            if not hasattr(self, "_W5"):
                g5 = torch.Generator(device=self.device).manual_seed(5)
                m5 = torch.randint(0, 8, self.G.scales.shape, dtype=torch.int32, device=self.device, generator=g5)
                sc5 = (((self.G.scales.to(torch.int32) - 112) << 3) | m5).to(torch.uint8)
                self._W5 = tc.TrellisMatrix(self.G.stream, sc5, self.G.rows, self.G.cols, SEG)
                self._ws5 = torch.empty(tc.gemv_e5m3_workspace_bytes(self._W5, 1), dtype=torch.uint8,
                                        device=self.device)
            tc.gemv_e5m3(self._W5, self.x[i % NVAR], out=self.yG, workspace=self._ws5)
        else:
            raise ValueError(name)

    def _expanded(self):
        if not hasattr(self, "nibG"):
            d = self.device
            self.nibG = torch.empty((E * 2 * I, H // 2), dtype=torch.uint8, device=d)
            self.scG = torch.empty((E * 2 * I, H // 32), dtype=torch.uint8, device=d)
            self.nibD = torch.empty((E * H, I // 2), dtype=torch.uint8, device=d)
            self.scD = torch.empty((E * H, I // 32), dtype=torch.uint8, device=d)
            self.tc.decode_to_mxfp4(self.G, self.nibG, self.scG)
            self.tc.decode_to_mxfp4(self.D, self.nibD, self.scD)

    def moe_call(self, T, skew=False, mx=False):
        """fn(i): routing of T tokens (N(0,1) logits, top-4) + the grouped MoE, on preallocated
        buffers; skew: every token on experts 0..3 with fixed random weights instead."""
        from trellis_coded_fp4_b200 import synth
        tc, d = self.tc, self.device
        xs = [synth.activations(T, H, seed=900 + T, sub=i).to(d) for i in range(NVAR)]
        lg = [synth.logits(T, E, seed=900 + T, sub=i).to(d) for i in range(NVAR)]
        ids = torch.empty((T, K_TOP), dtype=torch.int32, device=d)
        wts = torch.empty((T, K_TOP), dtype=torch.float32, device=d)
        out = torch.empty((T, H), dtype=torch.bfloat16, device=d)
        if mx:
            self._expanded()
            ng, sg, nd, sd = self.nibG.view(E, -1), self.scG.view(E, -1), self.nibD.view(E, -1), self.scD.view(E, -1)
            M = tc.Mxfp4MoEWeights([tc.Mxfp4Matrix(ng[e], sg[e], 2 * I, H) for e in range(E)],
                                   [tc.Mxfp4Matrix(nd[e], sd[e], H, I) for e in range(E)], H, I)
            run = tc.mxfp4_grouped_moe
        else:
            M, run = self.M, tc.grouped_moe
        ws = torch.empty(max(1, M.workspace_bytes(T, K_TOP)), dtype=torch.uint8, device=d)
        if skew:
            ids.copy_(torch.arange(K_TOP, dtype=torch.int32, device=d).repeat(T, 1))
            wts.copy_(torch.rand((T, K_TOP), generator=torch.Generator().manual_seed(T)).to(d))

        def fn(i):
            if not skew:
                tc.moe_route(lg[i % NVAR], K_TOP, ids, wts)
            run(M, xs[i % NVAR], ids, wts, out, ws)
        fn.ids_of = lambda i: (ids.clone() if skew else tc.moe_route(lg[i % NVAR], K_TOP)[0]).cpu().numpy()
        fn.keep = (M, xs, lg, ids, wts, out, ws)
        return fn


def moe_bytes(distinct, T, H_, I_, bpw=0.28125):
    return int(distinct * (2 * I_ * H_ + H_ * I_) * bpw) + 2 * T * H_ + 2 * T * H_


def moe_paths(ids, T):
    """The product-kernel instance a call takes and its routing groups (same rule as the library:
    up to 5 tokens per group on the 32-row B operand, else groups of up to 16 on the 96-row one)."""
    gmax = 5 if T <= 5 else 16
    cnt = np.bincount(ids.ravel(), minlength=E)
    groups = int(sum((c + gmax - 1) // gmax for c in cnt if c > 0))
    return {"instance": "32-row B, two MMA issuers" if gmax == 5 else "96-row B, 16-block stages",
            "distinct_experts": int((cnt > 0).sum()), "groups": groups, "max_tokens_per_expert": int(cnt.max())}


# ----------------------------------------------------------------------------- extra rows

def row_gemv_down(L, n, peak):
    us = time_calls(lambda i: L.tc.gemv_tiled(L.D, L.TD, L.xd[i % NVAR], L.yD, L.wsD), n)
    us_raw = time_calls(lambda i: L.tc.gemv(L.D, L.xd[i % NVAR], L.yD, L.wsD), n)
    return {**rate(gemv_bytes(E * H, I, 1), us, peak), "decoded_weights_per_s": E * H * I / (us * 1e-6),
            "shape": "92160 x 2880, T = 1, scale tiles", "raw_scales": rate(gemv_bytes(E * H, I, 1), us_raw, peak),
            "calls": n}


def row_gemv_raw(L, n, peak):
    us = time_calls(L.step_raw, n)
    return {**rate(gemv_bytes(L.G.rows, L.G.cols, 1), us, peak),
            "decoded_weights_per_s": L.G.rows * L.G.cols / (us * 1e-6),
            "what": "the headline call through trellis_gemv (scales in their [rows][cols/32] layout)", "calls": n}


def row_expand(L, n, peak):
    L._expanded()
    tc = L.tc
    exb = lambda rows, cols: rows * cols // 4 + rows * cols // 2 + 2 * (rows * cols // 32)  # noqa: E731

    def fn(i):
        tc.decode_to_mxfp4(L.G, L.nibG, L.scG)
        tc.decode_to_mxfp4(L.D, L.nibD, L.scD)
    us = time_calls(fn, n)
    us_g = time_calls(lambda i: tc.decode_to_mxfp4(L.G, L.nibG, L.scG), n)
    nb = exb(E * 2 * I, H) + exb(E * H, I)
    return {**rate(nb, us, peak), "decoded_weights_per_s": (E * 2 * I * H + E * H * I) / (us * 1e-6),
            "gate_up_only": rate(exb(E * 2 * I, H), us_g, peak),
            "what": "trellis_decode_to_mxfp4 of gate_up (184320 x 2880) then down (92160 x 2880); bit-exact "
                    "nibbles and scales (tests)", "calls": n}


def row_moe(L, T, n, peak, skew=False, mx=False):
    fn = L.moe_call(T, skew=skew, mx=mx)
    us = time_calls(fn, n)
    ids = [fn.ids_of(i) for i in range(1 if skew else NVAR)]
    paths = [moe_paths(a, T) for a in ids]
    distinct = statistics.mean(p["distinct_experts"] for p in paths)
    nb = moe_bytes(distinct, T, H, I, 0.53125 if mx else 0.28125)
    return {**rate(nb, us, peak), "T": T, "routing": "forced skew (experts 0-3)" if skew else "N(0,1) logits, top-4",
            "includes_route": not skew, "path": paths[0] if skew else
            {"instance": paths[0]["instance"], "distinct_experts_mean": distinct,
             "groups_mean": statistics.mean(p["groups"] for p in paths),
             "max_tokens_per_expert": max(p["max_tokens_per_expert"] for p in paths)}, "calls": n}


def row_gemv_sweep(L, n, peak):
    tc, d = L.tc, L.device
    L._expanded()
    G = L.G
    Gm = tc.Mxfp4Matrix(L.nibG, L.scG, G.rows, G.cols)
    from trellis_coded_fp4_b200 import synth
    out = []
    for T in (1, 2, 4, 8, 16, 32):
        x = synth.activations(T, G.cols, seed=synth.SEED_BASE + 90 + T).to(d)
        y = torch.empty((T, G.rows), dtype=torch.bfloat16, device=d)
        ws_f = torch.empty(max(1, tc.gemv_workspace_bytes(G, T)), dtype=torch.uint8, device=d)
        ws_m = torch.empty(max(1, tc.mxfp4_gemv_workspace_bytes(Gm, T)), dtype=torch.uint8, device=d)
        us_f = time_calls(lambda i: tc.gemv_tiled(G, L.Trot[0], x, y, ws_f), n)
        us_r = time_calls(lambda i: tc.gemv(G, x, y, ws_f), n)
        us_m = time_calls(lambda i: tc.mxfp4_gemv(Gm, x, y, ws_m), n)
        out.append({"T": T, "fused": rate(gemv_bytes(G.rows, G.cols, T), us_f, peak),
                    "fused_raw_scales": rate(gemv_bytes(G.rows, G.cols, T), us_r, peak),
                    "mxfp4": rate(gemv_bytes(G.rows, G.cols, T, 0.53125), us_m, peak)})
    return {"shape": "184320 x 2880", "calls": n, "rows": out}


def row_single_2048(L, peak, device):
    """2048 x 2048 at batch 1: 512 distinct matrices (576 MB, > 4x L2) back to back in a CUDA graph;
    and one call with L2 flushed before it (median of 20)."""
    tc = L.tc
    gen = torch.Generator(device=device).manual_seed(0x7CF40000)
    nmat, n = 512, 2048
    st = rand_words(nmat * n * (n // 32) * 2, gen, device).view(nmat, -1)
    sc = rand_scales(nmat * n * (n // 32), 120, 126, gen, device).view(nmat, -1)
    mats = [tc.TrellisMatrix(st[j], sc[j], n, n, SEG) for j in range(nmat)]
    from trellis_coded_fp4_b200 import synth
    x = synth.activations(1, n, seed=synth.SEED_BASE).to(device)
    y = torch.empty((1, n), dtype=torch.bfloat16, device=device)
    ws = torch.empty(max(1, tc.gemv_workspace_bytes(mats[0], 1)), dtype=torch.uint8, device=device)
    call = lambda i: tc.gemv(mats[i % nmat], x, y, ws)  # noqa: E731
    nb = gemv_bytes(n, n, 1)
    res = {"shape": "2048 x 2048, T = 1, seg_len 32", "matrices": nmat}
    try:
        res["graph"] = {**rate(nb, time_graph(call, nmat), peak), "note": "back to back, CUDA graph of 512 calls"}
    except Exception as ex:  # capture unavailable: host-launched back to back instead
        res["graph"] = {"error": str(ex)[:200]}
    res["stream"] = {**rate(nb, time_calls(call, nmat), peak), "note": "back to back, launched from the host"}
    flush = torch.empty(256 * 2 ** 20 // 4, dtype=torch.float32, device=device)
    lat = []
    for j in range(20):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call(j)
        e1.record()
        torch.cuda.synchronize()
        lat.append(1e3 * e0.elapsed_time(e1))
    res["cold_latency_us"] = {"median": round(statistics.median(lat), 3), "p10": round(float(np.percentile(lat, 10)), 3),
                              "p90": round(float(np.percentile(lat, 90)), 3)}
    del st, sc, mats, flush
    return res


def row_moe_7168(tc, peak, device, n):
    """256 experts, hidden 7168, intermediate 2048, top-8 of N(0,1) logits, T = 1, 8, 32; random
    2-bit streams and UE8M0 bytes in [118, 126] generated on the device (3.17 GB resident)."""
    from trellis_coded_fp4_b200 import synth
    E4, H4, I4, k4 = 256, 7168, 2048, 8
    gen = torch.Generator(device=device).manual_seed(0x7CF40004)
    gu = rand_words(E4 * 2 * I4 * (H4 // 32) * 2, gen, device).view(E4, -1)
    gus = rand_scales(E4 * 2 * I4 * (H4 // 32), 118, 126, gen, device).view(E4, -1)
    dn = rand_words(E4 * H4 * (I4 // 32) * 2, gen, device).view(E4, -1)
    dns = rand_scales(E4 * H4 * (I4 // 32), 118, 126, gen, device).view(E4, -1)
    M = tc.MoEWeights([tc.TrellisMatrix(gu[e], gus[e], 2 * I4, H4, SEG) for e in range(E4)],
                      [tc.TrellisMatrix(dn[e], dns[e], H4, I4, SEG) for e in range(E4)], H4, I4)
    rows = []
    for T in (1, 8, 32):
        xs = [synth.activations(T, H4, seed=0x7CF40004 + T, sub=i).to(device) for i in range(NVAR)]
        lg = [synth.logits(T, E4, seed=0x7CF40004 + T, sub=i).to(device) for i in range(NVAR)]
        ids = torch.empty((T, k4), dtype=torch.int32, device=device)
        wts = torch.empty((T, k4), dtype=torch.float32, device=device)
        out = torch.empty((T, H4), dtype=torch.bfloat16, device=device)
        ws = torch.empty(max(1, M.workspace_bytes(T, k4)), dtype=torch.uint8, device=device)

        def fn(i):
            tc.moe_route(lg[i % NVAR], k4, ids, wts)
            tc.grouped_moe(M, xs[i % NVAR], ids, wts, out, ws)
        us = time_calls(fn, n)
        distinct = statistics.mean(len(np.unique(tc.moe_route(lg[i], k4)[0].cpu().numpy())) for i in range(NVAR))
        nb = moe_bytes(distinct, T, H4, I4)
        rows.append({**rate(nb, us, peak), "T": T, "distinct_experts_mean": distinct, "includes_route": True,
                     "decoded_weights_per_s": distinct * 3 * H4 * I4 / (us * 1e-6)})
    del gu, gus, dn, dns, M
    return {"layer": "256 experts, hidden 7168, intermediate 2048, top-8, 3.17 GB resident", "calls": n, "rows": rows}


def row_mxfp4(L, n, peak):
    tc, d = L.tc, L.device
    L._expanded()
    Gm = tc.Mxfp4Matrix(L.nibG, L.scG, E * 2 * I, H)
    Dm = tc.Mxfp4Matrix(L.nibD, L.scD, E * H, I)
    wsg = torch.empty(max(1, tc.mxfp4_gemv_workspace_bytes(Gm, 1)), dtype=torch.uint8, device=d)
    wsd = torch.empty(max(1, tc.mxfp4_gemv_workspace_bytes(Dm, 1)), dtype=torch.uint8, device=d)
    ug = time_calls(lambda i: tc.mxfp4_gemv(Gm, L.x[i % NVAR], L.yG, wsg), n)
    ud = time_calls(lambda i: tc.mxfp4_gemv(Dm, L.xd[i % NVAR], L.yD, wsd), n)
    return {"mxfp4_gemv_gate_up": rate(gemv_bytes(E * 2 * I, H, 1, 0.53125), ug, peak),
            "mxfp4_gemv_down": rate(gemv_bytes(E * H, I, 1, 0.53125), ud, peak),
            "mxfp4_grouped_moe_t1": row_moe(L, 1, n, peak, mx=True), "calls": n}


def encoder_inputs(L, rows, cols, gen, device):
    """The encoder's workload: targets N(0, 2.5^2) times their block's scale, D uniform in [0.1, 10],
    the scales of the first rows of the gate_up stack."""
    esc = L.G.scales[: rows * (cols // 32)]
    sval = torch.pow(2.0, esc.to(torch.float64) - 127.0).repeat_interleave(32).view(rows, cols)
    et = torch.randn(rows, cols, dtype=torch.float64, device=device, generator=gen) * 2.5 * sval
    eD = torch.rand(rows, cols, dtype=torch.float64, device=device, generator=gen) * 9.9 + 0.1
    return et, eD, esc


def row_encoder(L, seed, device):
    tc = L.tc
    enc_rows, enc_cols = 296, H
    gen = torch.Generator(device=device).manual_seed(seed)
    et, eD, esc = encoder_inputs(L, enc_rows, enc_cols, gen, device)
    ms = time_calls(lambda i: tc.encode(et, eD, esc, 32), 3, warm=1) / 1e3
    return {"ms_per_call": round(ms, 3), "weights": enc_rows * enc_cols, "seg_len": 32,
            "weights_per_s": enc_rows * enc_cols / (ms * 1e-3), "bound": "alu",
            "note": "2^16 candidate paths per weight, fp64 costs evaluated exactly (no fused operations)"}


def row_repack(L, n, peak):
    tc = L.tc
    out = torch.empty_like(L.G.stream)
    us = time_calls(lambda i: tc.repack_interleaved(L.G.stream, L.G.rows, L.G.cols, out=out), n)
    res = {**rate(16 * L.G.rows * (L.G.cols // 32), us, peak), "calls": n, "bound": "hbm",
           "note": "8 bytes read + 8 written per 32-weight block"}
    del out
    return res


def row_e5m3(L, n, peak, seed):
    tc, d = L.tc, L.device
    g5 = torch.Generator(device=d).manual_seed(seed + 5)
    m5 = torch.randint(0, 8, L.G.scales.shape, dtype=torch.int32, device=d, generator=g5)
    sc5 = (((L.G.scales.to(torch.int32) - 112) << 3) | m5).to(torch.uint8)
    W5 = tc.TrellisMatrix(L.G.stream, sc5, L.G.rows, L.G.cols, L.G.seg_len)
    ws5 = torch.empty(max(1, tc.gemv_e5m3_workspace_bytes(W5, 1)), dtype=torch.uint8, device=d)
    us = time_calls(lambda i: tc.gemv_e5m3(W5, L.x[i % NVAR], out=L.yG, workspace=ws5), n)
    return {**rate(gemv_bytes(E * 2 * I, H, 1), us, peak), "decoded_weights_per_s": W5.rows * W5.cols / (us * 1e-6),
            "calls": n, "note": "E5M3 block scales of the same binades, batch 1; tensor cores, four block-scaled "
                                "MMAs per K-step (one per power of two of the scale)"}


# ----------------------------------------------------------------------------- end to end

def run_e2e(L, steps):
    """The headline metric through the public API with HOST buffers: every step copies the gate_up
    stream, its scale tiles and x from pinned host memory, runs trellis_gemv_tiled and copies y back."""
    lay = L.layer
    h_st = torch.from_numpy(lay.gu_stream.view("int32").reshape(-1)).pin_memory()
    h_sc = L.Trot[0].cpu().pin_memory()  # the scale tiles, as stored
    h_x = [x.cpu().pin_memory() for x in L.x]
    h_y = torch.empty(L.yG.shape, dtype=L.yG.dtype).pin_memory()
    h2d = h_st.numel() * 4 + h_sc.numel() + h_x[0].numel() * 2
    d2h = h_y.numel() * 2

    def one(i):
        L.G.stream.copy_(h_st, non_blocking=True)
        L.Trot[0].copy_(h_sc, non_blocking=True)
        L.x[i % NVAR].copy_(h_x[i % NVAR], non_blocking=True)
        L.tc.gemv_tiled(L.G, L.Trot[0], L.x[i % NVAR], L.yG, L.wsG)
        h_y.copy_(L.yG, non_blocking=True)
    us = time_calls(one, steps, warm=2)
    return {"value": L.G.rows * L.G.cols / (us * 1e-6), "unit": UNIT, "ms_per_step": us / 1e3,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


# ----------------------------------------------------------------------------- CPU oracle

def oracle_gemv_sample(layer, x_bits, stride, threads):
    """The oracle's batch-1 GEMV on every `stride`-th row of the stacked gate_up matrix, the rows
    split over `threads` threads (each call is one plain C loop; ctypes releases the GIL).
    Returns the decoded weights."""
    import oracle
    st = layer.gu_stream.reshape(E * 2 * I, H // 32, 2)
    sc = layer.gu_scales.reshape(E * 2 * I, H // 32)
    sel = np.arange(0, E * 2 * I, stride)
    parts = np.array_split(sel, threads)
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda r: oracle.gemv(st, sc, E * 2 * I, H, SEG, x_bits, row_ids=r), parts))
    return len(sel) * H


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return platform.processor() or "unknown"


def cpu_baseline(layer, seed):
    from trellis_coded_fp4_b200 import synth
    xb = synth.bf16_bits(synth.activations(1, H, seed=seed))
    ncores = len(os.sched_getaffinity(0))
    res = {}
    for name, stride, threads in (("single", 8, 1), ("all", 1, ncores)):
        t0 = time.perf_counter()
        n = oracle_gemv_sample(layer, xb, stride, threads)
        dt = time.perf_counter() - t0
        res[name] = {"value": n / dt, "cores": threads, "seconds": round(dt, 3), "weights": n, "stride": stride}
    a, s = res["all"], res["single"]
    return {"value": a["value"], "unit": UNIT, "cores": a["cores"], "kind": "oracle",
            "sample": (f"batch-1 GEMV of every {a['stride']}th row of the stacked gate_up matrix ({a['weights']} decoded "
                       f"weights), rows split over {a['cores']} threads of the plain C oracle"),
            "single_core": {"value": s["value"], "cores": 1,
                            "sample": f"every {s['stride']}th row ({s['weights']} weights), one thread"},
            "cpu_model": cpu_model()}


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
    """The oracle as it stands, on a bounded sample of the headline workload (every stride-th row of
    the stacked gate_up matrix per step, rows split over the host's cores; the stride is set from a
    first timed sample so that warm-up and steps together take about a minute); rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from trellis_coded_fp4_b200 import synth
    seed = synth.SEED_BASE + 1
    layer = synth.moe_layer(E, H, I, seed=seed)
    ncores = len(os.sched_getaffinity(0))
    xb = synth.bf16_bits(synth.activations(1, H, seed=seed))
    t0 = time.perf_counter()
    n0 = oracle_gemv_sample(layer, xb, 1024, ncores)
    rate0 = n0 / (time.perf_counter() - t0)
    budget_s = 60.0
    rows_per_step = rate0 * budget_s / H / max(1, args.steps + args.warmup)
    stride = int(max(64, min(E * 2 * I, np.ceil(E * 2 * I / max(rows_per_step, 1.0)))))
    for _ in range(args.warmup):
        oracle_gemv_sample(layer, xb, stride, ncores)
    t0 = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        n += oracle_gemv_sample(layer, xb, stride, ncores)
    dt = time.perf_counter() - t0
    value = n / dt
    sample = (f"every {stride}th row of the stacked gate_up matrix, {n // max(args.steps, 1)} decoded weights per "
              f"step, plain C oracle, rows split over {ncores} threads")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample}, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": ncores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)  # ~0.3 s timed: several clock samples
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="tcf4", choices=["tcf4", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="the headline only, without the extra rows")
    ap.add_argument("--only", default=None,
                    help="run only this call (gemv_gate_up, gemv_gate_up_raw, gemv_gate_up_t<T>, gemv_down, gemv_e5m3, "
                         "expand_gate_up, grouped_moe, encoder) warmup + "
                         "steps times, for profiling one kernel; prints no bench line")
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
    L = Layer(seed, device)
    if args.only is not None:
        for i in range(args.warmup + args.steps):
            L.run_only(args.only, i)
        torch.cuda.synchronize()
        print(json.dumps({"only": args.only, "launches": args.warmup + args.steps,
                          "timeouts": L.tc.device_timeouts()}))
        return 0

    warm = max(args.warmup, 3)
    for i in range(warm):
        L.step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.15)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tw0 = time.time()
    start.record()
    for i in range(args.steps):
        L.step(i)
    end.record()
    torch.cuda.synchronize()
    tw1 = time.time()
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop(tw0, tw1)
    ms_total = max_over_ranks(start.elapsed_time(end), dist, device)
    ms_per_step = ms_total / args.steps
    weights_per_step = L.G.rows * L.G.cols
    peak, peak_kind = measured_hbm_peak()
    nb = gemv_bytes(L.G.rows, L.G.cols, 1)
    achieved = nb / (ms_per_step * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": NCU_TRAFFIC_GEMV_GATE_UP,
                "kernel": "trellis_gemv_tiled: k_bsplit_gemv + k_mma (decode-MMA, scale tiles) on the 184320 x 2880 "
                          "gate_up stack, T = 1",
                "algo_bytes_per_launch": nb, "avg_us": round(ms_per_step * 1e3, 3),
                "frac_of_8tbs": round(achieved / SPEC_HBM_GBS, 4),
                "peak_source": (f"{peak_kind}: MEASURED_PEAKS.json hbm_gbs" if peak_kind == "measured"
                                else "fallback 6650 GB/s")}
    value = job_value(world, weights_per_step, args.steps, ms_total)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": warm,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u32 decode, f32 accumulate", "data": "synthetic",
            "config": {"workload": WORKLOAD, "rows": L.G.rows, "cols": L.G.cols, "tokens": 1, "seg_len": SEG,
                       "decoded_weights_per_step": weights_per_step,
                       "scales": "UE8M0 scale tiles (the same bytes as [rows][cols/32], rearranged once at load time)",
                       "l2": f"inputs larger than L2: steps rotate over {ROT} distinct resident matrices "
                             f"({ROT * nb / 1e6:.0f} MB) and {NVAR} activation vectors",
                       "parallelism": f"replicas x{world}",
                       "arithmetic": "decode: u32 bit logic; products: block-scaled MXFP4 tensor-core MMA "
                                     "(activations as six E2M1 terms per 32-block), fp32 accumulation, bf16 out"},
            "roofline": roofline, "gpu_launches": L.launches_per_step * args.steps, "clocks": clocks}

    if not args.no_rows:
        n = 200
        rows = {}
        rows["gemv_gate_up_raw_scales"] = row_gemv_raw(L, 1000, peak)
        rows["gemv_down"] = row_gemv_down(L, n, peak)
        rows["expand"] = row_expand(L, 100, peak)
        rows["moe_t1"] = row_moe(L, 1, n, peak)
        rows["moe_sweep"] = {"natural": [row_moe(L, T, 100, peak) for T in (1, 2, 4, 8, 16, 32)],
                             "skew": [row_moe(L, T, 100, peak, skew=True) for T in (1, 8, 16, 32)]}
        rows["gemv_sweep"] = row_gemv_sweep(L, 50, peak)
        rows["single_2048"] = row_single_2048(L, peak, device)
        rows["moe_7168"] = row_moe_7168(L.tc, peak, device, 50)
        rows["mxfp4_consumer"] = row_mxfp4(L, n, peak)
        rows["encoder"] = row_encoder(L, seed, device)
        rows["repack_interleaved"] = row_repack(L, n, peak)
        rows["gemv_e5m3_gate_up"] = row_e5m3(L, 50, peak, seed)
        rows["timeouts"] = L.tc.device_timeouts()
        line["rows"] = rows

    if rank == 0:
        line["e2e"] = run_e2e(L, args.e2e_steps)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(L.layer, seed)
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
