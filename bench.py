"""Benchmark of the merged-LoRA refiner hot path on B200.

One step is one pass of the whole path over the 2K workload (latent
37 x 24 x 90 x 160, 532,800 tokens, d = 7168, merged rank 576):

  lora_merge for the three layer shapes (d->d, d->3d, 4d->d)
  renoise(up) at sigma0 = 0.909
  lora_linear d->d,   euler_step 0.909 -> 0.857
  lora_linear d->3d,  euler_step 0.857 -> 0.667
  lora_linear 4d->d,  euler_step 0.667 -> 0

(each Euler step follows one stand-in transformer pass, as in the refine
loop).  `value` is tokens/s over the whole job (tokens of every rank divided
by the slowest rank's time); with N GPUs each rank runs its own copy of the
workload (weak scaling, no data-path collective).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

`--impl reference` times the FP64 CPU oracle on the host cores over a
bounded sample of tokens per step (the reference arm for this path).
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "lora_linear tokens/s + % bf16 TC peak at 2K grid; renoise/Euler HBM GB/s"
UNIT = "tokens/s"
WORKLOAD = "2k"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {
            "hbm_gbs": float(p["hbm_gbs"]),
            "bf16_tflops": float(p["bf16_tflops"]),
            "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
            "source": "measured",
        }
    except (OSError, KeyError, ValueError):
        return {
            "hbm_gbs": FALLBACK_HBM_GBS,
            "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": FALLBACK_BF16_TFLOPS_SUSTAINED,
            "source": "fallback",
        }


# ---------------------------------------------------------------------------
# Distributed plumbing: lora_gemm_b200.dist (one process per GPU; NCCL only
# for the barrier and the max over ranks).
# ---------------------------------------------------------------------------
def _dist():
    from lora_gemm_b200 import dist

    return dist


def barrier(world):
    _dist().barrier(world)


def max_over_ranks(value, world):
    return _dist().max_over_ranks(value, world)


# ---------------------------------------------------------------------------
# Clock sampling during the timed region.
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = torch.cuda.get_device_properties(device_index).uuid
            self.uuid = "GPU-" + str(uuid) if not str(uuid).startswith("GPU-") else str(uuid)
        except Exception:
            self.uuid = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
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
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None

        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, val in zip(names, r[6:10]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {
            "sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None,
            "reasons": sorted(reasons),
            "samples": len(rows),
            "power_w_max": max((num(r[4]) or 0.0) for r in rows),
        }


# ---------------------------------------------------------------------------
# Our arm.
# ---------------------------------------------------------------------------
def layer_flops(M, K, N, R):
    return 2.0 * M * (K * N + K * R + R * N)


class Problem:
    """Device-resident inputs and outputs of one 2K step."""

    def __init__(self, w, dev, tokens=None, noise_offset=0, lean=False, frames=None):
        """lean: every layer's activations are the first M x K values of one
        buffer drawn for the widest K, and every layer writes its output into
        the first M x N values of one buffer of the widest N (the 4K grid's
        step then holds ~123 GB instead of ~175 GB)."""
        import synth
        import lora_gemm_b200 as lg

        self.w = w
        if frames is not None:  # one clip split by frames: this rank's frames [f0, f1)
            f0, f1 = frames
            M = (f1 - f0) * w.height * w.width if tokens is None else tokens
        else:
            M = w.tokens if tokens is None else tokens
        self.M = M
        R = sum(synth.ADAPTER_RANKS)
        self.R = R
        self.layers = []
        x_by_k = {}
        if lean:
            k_max = max(K for K, _ in w.shapes)
            x_all = synth.activations(w, k_max, [K for K, _ in w.shapes].index(k_max), dev, M=M).view(-1)
            y_all = torch.empty(M * max(N for _, N in w.shapes), dtype=torch.bfloat16, device=dev)
        for i, (K, N) in enumerate(w.shapes):
            if K not in x_by_k:
                x_by_k[K] = x_all[:M * K].view(M, K) if lean else synth.activations(w, K, i, dev, M=M)
            As, Bs = synth.adapters(w, i, dev)
            L = {
                "K": K, "N": N, "x": x_by_k[K], "W": synth.weight(w, i, dev), "As": As, "Bs": Bs,
                "A_cat": torch.empty((R, K), dtype=torch.float32, device=dev),
                "B_cat": torch.empty((N, R), dtype=torch.float32, device=dev),
                "y": y_all[:M * N].view(M, N) if lean else torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                "ws": torch.empty(lg.lora_linear_workspace_size(M, K, N, R), dtype=torch.uint8, device=dev),
            }
            self.layers.append(L)
        self.up = synth.upscaled_latent(w, dev)
        self.v = [synth.velocity(w, k, dev) for k in range(3)]
        if frames is not None:
            self.up = self.up[frames[0]:frames[1]].contiguous()
            self.v = [v[frames[0]:frames[1]].contiguous() for v in self.v]
        self.x_lat = torch.empty_like(self.up)
        self.sigmas = [float(torch.tensor(s, dtype=torch.float32)) for s in synth.SIGMA_SCHEDULE]
        self.noise_offset = noise_offset  # this rank's slice of the Philox stream
        self.scales = synth.ADAPTER_SCALES


def run_step(P, ev=None):
    """One pass of the hot path on the current stream; ev collects (name, start, end) event pairs."""
    import lora_gemm_b200 as lg

    def rec(name, fn):
        if ev is None:
            fn()
            return
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        ev.append((name, s, e))

    for L in P.layers:
        rec("lora_merge", lambda L=L: lg.lora_merge(L["As"], L["Bs"], P.scales, L["A_cat"], L["B_cat"]))
    rec("renoise", lambda: lg.renoise(P.up, P.sigmas[0], P.w.seed, offset=P.noise_offset, out=P.x_lat))
    # Euler step k follows layer k; a workload with fewer layers than steps
    # (768P, tiny: one layer) runs the remaining steps after it.
    for k in range(len(P.sigmas) - 1):
        if k < len(P.layers):
            L = P.layers[k]
            rec(f"lora_linear{k}", lambda L=L: lg.lora_linear(L["x"], L["W"], L["A_cat"], L["B_cat"], y=L["y"],
                                                              workspace=L["ws"]))
        rec(f"euler{k}", lambda k=k: lg.euler_step(P.x_lat, P.v[k], P.sigmas[k], P.sigmas[k + 1]))


def run_mxfp8(P, args, world, peaks):
    """The same step with the linear layers as MXFP8 GEMMs (lg_lora_linear_mxfp8):
    W is quantized once (model load), each distinct x once per step inside
    the timed region (it comes from the previous op in a real forward), the
    LoRA path stays bf16.  Reported beside the bf16 headline, not instead of it."""
    import lora_gemm_b200 as lg

    wq = [lg.mx_quantize(L["W"]) for L in P.layers]
    xq = {}
    for L in P.layers:
        if id(L["x"]) not in xq:
            xq[id(L["x"])] = lg.mx_quantize(L["x"])
    first_use = {}
    for k, L in enumerate(P.layers):
        first_use.setdefault(id(L["x"]), k)

    def step(ev=None):
        def rec(name, fn):
            if ev is None:
                fn()
                return
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            ev.append((name, s, e))

        for L in P.layers:
            rec("lora_merge", lambda L=L: lg.lora_merge(L["As"], L["Bs"], P.scales, L["A_cat"], L["B_cat"]))
        rec("renoise", lambda: lg.renoise(P.up, P.sigmas[0], P.w.seed, offset=P.noise_offset, out=P.x_lat))
        for k in range(len(P.sigmas) - 1):
            if k < len(P.layers):
                L = P.layers[k]
                if first_use[id(L["x"])] == k:
                    q = xq[id(L["x"])]
                    rec("quantize", lambda L=L, q=q: lg.mx_quantize(L["x"], codes=q[0], scales=q[1]))
                rec(f"lin{k}", lambda k=k, L=L: lg.lora_linear_mxfp8(L["x"], xq[id(L["x"])], wq[k], L["A_cat"],
                                                                      L["B_cat"], y=L["y"], workspace=L["ws"]))
            rec(f"euler{k}", lambda k=k: lg.euler_step(P.x_lat, P.v[k], P.sigmas[k], P.sigmas[k + 1]))

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    ev = []
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step(ev)
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    status = lg.get_last_device_error()
    if status != lg.LG_OK:
        raise SystemExit(f"device error during the MXFP8 steps: {lg.status_string(status)}")
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    per = {}
    for name, s, e in ev:
        per.setdefault(name, []).append(s.elapsed_time(e))
    flops = [layer_flops(P.M, L["K"], L["N"], P.R) for L in P.layers]
    lin_ms = [statistics.mean(per[f"lin{k}"]) for k in range(len(P.layers))]
    tflops = sum(flops) / (sum(lin_ms) * 1e-3) / 1e12
    fp8_peak = 2.0 * peaks["bf16_tflops_sustained"]
    q_ms = sum(per["quantize"]) / args.steps
    cublas = _cublas_mxfp8_context(P, xq, wq, world)
    del xq, wq
    return {
        "value": round(_dist().whole_job_rate(P.M, world, args.steps, ms), 1), "unit": UNIT,
        "ms_per_step": round(ms / args.steps, 3),
        "lora_linear_mxfp8": {
            "per_layer_ms": [round(t, 4) for t in lin_ms],
            "per_layer_tflops": [round(f / (t * 1e-3) / 1e12, 1) for f, t in zip(flops, lin_ms)],
            "tflops": round(tflops, 1),
            "peak": round(fp8_peak, 1),
            "peak_kind": "fp8 dense, derived: measured bf16 sustained x 2 (the nominal fp8 / bf16 ratio)",
            "frac": round(tflops / fp8_peak, 4),
        },
        "quantize_x_ms_per_step": round(q_ms, 4),
        "cublas_mxfp8_base_term": cublas,
        "note": "W quantized once outside the timed steps; x quantized inside; LoRA path bf16",
    }


def _cublas_mxfp8_context(P, xq, wq, world):
    """Context for the MXFP8 layers: cuBLAS's block-scaled MXFP8 GEMM
    (torch._scaled_mm) on the same codes and scales -- the scale layout
    lg_mx_quantize writes is the one cuBLAS takes -- computing the base term
    deq(x) deq(W)^T alone, without the LoRA term, per layer shape."""
    try:
        layers = []
        for k, L in enumerate(P.layers):
            a, sa = xq[id(L["x"])]
            b, sb = wq[k]
            A8, B8 = a.view(torch.float8_e4m3fn), b.view(torch.float8_e4m3fn)
            SA, SB = sa.view(torch.float8_e8m0fnu), sb.view(torch.float8_e8m0fnu)
            ms = _time_calls(lambda: torch._scaled_mm(A8, B8.t(), scale_a=SA, scale_b=SB, out_dtype=torch.bfloat16),
                             2, world)
            layers.append({"ms": round(ms, 4), "tflops": round(2.0 * P.M * L["K"] * L["N"] / (ms * 1e-3) / 1e12, 1)})
        torch.cuda.empty_cache()
        return {"per_layer": layers, "what": "torch._scaled_mm, E4M3 codes with E8M0 block scales (1 x 32), "
                                             "base term only (no LoRA), bf16 output"}
    except Exception as e:  # an older torch or cuBLAS without MXFP8
        return {"unavailable": f"{type(e).__name__}: {str(e)[:200]}"}


def _time_calls(fn, reps, world):
    """Mean ms of fn over reps calls (one untimed call first), CUDA events on
    the current stream, max over ranks."""
    fn()
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(reps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    return max_over_ranks(t0.elapsed_time(t1) / reps, world)


def run_elementwise_isolated(P, args, world, peaks):
    """renoise and euler_step timed alone: 100 back-to-back launches each,
    rotating over 4 buffer sets (408 MB, more than L2 holds), captured in one
    CUDA graph (so the binding's per-call host work cannot leave the GPU idle
    between launches of a few tens of microseconds) with CUDA events around
    its replay.  The in-step figures come from the bench step."""
    import lora_gemm_b200 as lg

    hbm = peaks["hbm_gbs"]
    n = P.up.numel()
    sets = 4
    ups = [P.up.clone() for _ in range(sets)]
    xs = [torch.empty_like(P.up) for _ in range(sets)]
    vs = [P.v[i % len(P.v)].clone() for i in range(sets)]
    s0, s1 = P.sigmas[0], P.sigmas[1]
    out = {}
    for name, per_elem, fn in (
            ("renoise", 8.0, lambda i: lg.renoise(ups[i], s0, P.w.seed, offset=P.noise_offset, out=xs[i])),
            ("euler_step", 12.0, lambda i: lg.euler_step(xs[i], vs[i], s0, s1))):
        for i in range(sets):
            fn(i)
        torch.cuda.synchronize()
        launches = 100
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for k in range(launches):
                fn(k % sets)
        graph.replay()
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        del graph
        ms = max_over_ranks(e0.elapsed_time(e1) / launches, world)
        gbs = per_elem * n / (ms * 1e-3) / 1e9
        out[name] = {"launches": launches, "ms": round(ms, 5), "gbs": round(gbs, 1),
                     "frac_of_measured_hbm": round(gbs / hbm, 4)}
    out["note"] = (f"{sets} rotating buffer sets ({sets * 2 * 4 * n / 1e6:.0f} MB) so that no launch finds its data "
                   f"in L2; the {launches} launches replayed from one CUDA graph")
    del ups, xs, vs
    status = lg.get_last_device_error()
    if status != lg.LG_OK:
        raise SystemExit(f"device error during the isolated elementwise runs: {lg.status_string(status)}")
    return out


def run_ic_routes(P, args, world, peaks, routes=None):
    """The IC sampler routes (up3, up4, hf8: re-noise at the route's start and
    one Euler step per rung of HyperFlow's shift-12 ladder) on the workload's
    latent, with the step's velocity stand-ins (or the given {name: ladder}
    routes).  The linear layers of each rung are those of the main step and
    are not repeated here.  L2 is flushed (a 256 MiB write) before every
    timed route; only the route is timed."""
    import lora_gemm_b200 as lg

    hbm = peaks["hbm_gbs"]
    n = P.up.numel()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=P.up.device)
    out = {}
    if routes is None:
        routes = {route: lg.shift_ladder(s0) for route, s0 in lg.IC_ROUTES.items()}
    for route, lad in routes.items():

        def f(lad=lad):
            lg.renoise(P.up, lad[0], P.w.seed, offset=P.noise_offset, out=P.x_lat)
            for k in range(len(lad) - 1):
                lg.euler_step(P.x_lat, P.v[k % len(P.v)], lad[k], lad[k + 1])

        f()
        times = []
        for _ in range(max(args.steps, 5)):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = max_over_ranks(statistics.median(times), world)
        nbytes = 8.0 * n + 12.0 * n * (len(lad) - 1)
        out[route] = {"sigmas": [round(x, 6) for x in lad], "euler_steps": len(lad) - 1, "ms": round(ms, 4),
                      "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                      "frac_of_measured_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)}
    del flush
    status = lg.get_last_device_error()
    if status != lg.LG_OK:
        raise SystemExit(f"device error during the IC routes: {lg.status_string(status)}")
    out["note"] = (f"algorithmic bytes 8 + 12 per step per latent element; the {4 * n / 1e6:.0f} MB latent stays "
                   "partly in L2 between the steps of a route, so long routes can pass the HBM copy rate")
    return out


def _time_alternating(f, g, reps, world):
    """Median ms of f and of g over reps rounds of f then g (one untimed call
    of each first), CUDA events around every call on the current stream, max
    over ranks.  Alternating keeps both forms under the same clock and power
    state."""
    f()
    g()
    torch.cuda.synchronize()
    barrier(world)
    tf, tg = [], []
    for _ in range(reps):
        for fn, acc in ((f, tf), (g, tg)):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            acc.append(e0.elapsed_time(e1))
    return max_over_ranks(statistics.median(tf), world), max_over_ranks(statistics.median(tg), world)


def run_library_ab(P, args, world, peaks):
    """Each layer of the step against the unfused library composition of the
    same arithmetic, timed alternately (medians, CUDA events on the current
    stream): cuBLAS bf16 y = x W^T, cuBLAS h = x A_cat^T written to HBM
    (bf16, [M, R]), cuBLAS y += h B_cat^T, with the factors' bf16 copies made
    by torch inside the timed call (the fused call makes its own inside too).
    Context for the fusion: the fused kernel saves the h round trip (2 M R
    bytes each way) and the separate passes."""
    import lora_gemm_b200 as lg

    out = []
    h = torch.empty((P.M, P.R), dtype=torch.bfloat16, device=P.up.device)
    reps = 3
    for k, L in enumerate(P.layers):
        x, W, A, B, y, ws = L["x"], L["W"], L["A_cat"], L["B_cat"], L["y"], L["ws"]

        def fused():
            lg.lora_linear(x, W, A, B, y=y, workspace=ws)

        def unfused():
            A16 = A.to(torch.bfloat16)
            B16 = B.to(torch.bfloat16)
            torch.matmul(x, W.t(), out=y)
            torch.matmul(x, A16.t(), out=h)
            y.addmm_(h, B16.t())

        f_ms, u_ms = _time_alternating(fused, unfused, reps, world)
        fl = layer_flops(P.M, L["K"], L["N"], P.R)
        out.append({"k_n": [L["K"], L["N"]], "fused_ms": round(f_ms, 3), "unfused_cublas_ms": round(u_ms, 3),
                    "fused_tflops": round(fl / (f_ms * 1e-3) / 1e12, 1),
                    "unfused_tflops": round(fl / (u_ms * 1e-3) / 1e12, 1),
                    "fused_speedup": round(u_ms / f_ms, 3)})
    del h
    torch.cuda.empty_cache()
    status = lg.get_last_device_error()
    if status != lg.LG_OK:
        raise SystemExit(f"device error during the library A/B: {lg.status_string(status)}")
    return {"per_layer": out, "reps": reps,
            "note": "fused lg_lora_linear against cuBLAS x W^T + cuBLAS h = x A^T (h in HBM) + cuBLAS y += h B^T, "
                    "calls alternating, medians; algorithmic FLOPs 2 M (K N + K R + R N) for both"}


def run_fusions(P, args, world, peaks):
    """Epilogue fusions beside the step, each against its unfused form:

    * projection_euler: the step's last projection (d -> C channels, rank R)
      with the Euler update and the bf16 copy of the new latent fused
      (lg_lora_linear_euler), on all of the workload's whole frames; unfused:
      lg_lora_linear with W padded to 32 rows, the velocity permuted into the
      latent's layout by torch, lg_euler_step and a torch bf16 cast.
    * swiglu_mxfp8: the MLP's input projection d -> 2 ffn with SwiGLU and the
      MXFP8 quantizer fused (lg_lora_linear_swiglu_mxfp8) on a quarter of the
      tokens (the unfused form holds the [M, 2 ffn] intermediate); unfused:
      lg_lora_linear_mxfp8, torch silu(gate) * up in bf16, lg_mx_quantize.
    Fused and unfused calls alternate; each figure is a median.
    """
    import lora_gemm_b200 as lg
    import synth

    w, dev, R = P.w, P.up.device, P.R
    reps = max(args.steps, 5)
    out = {}
    L0 = P.layers[0]
    K = L0["K"]
    # Projection + Euler over whole frames of the layer-0 activations.
    T = w.height * w.width
    frames = P.M // T
    if frames > 0 and K == w.d:
        Kp, C = synth.proj_out_shape(w)
        M = frames * T
        x = L0["x"][:M]
        W = synth.weight(w, synth.PROJ_OUT_LAYER, dev, shape=(Kp, C))
        As, Bs = synth.adapters(w, synth.PROJ_OUT_LAYER, dev, shape=(Kp, C))
        A_cat, B_cat = lg.lora_merge(As, Bs, P.scales)
        z = torch.zeros((frames, C, T), dtype=torch.float32, device=dev)
        zb = torch.empty_like(z, dtype=torch.bfloat16)
        ws = torch.empty(lg.lora_linear_euler_workspace_size(M, K, C, R), dtype=torch.uint8, device=dev)
        s0, s1 = P.sigmas[1], P.sigmas[2]
        Cp = 32
        Wp = torch.zeros((Cp, K), dtype=torch.bfloat16, device=dev)
        Wp[:C] = W
        Bp = torch.zeros((Cp, R), dtype=torch.float32, device=dev)
        Bp[:C] = B_cat
        y = torch.empty((M, Cp), dtype=torch.bfloat16, device=dev)
        wsp = torch.empty(lg.lora_linear_workspace_size(M, K, Cp, R), dtype=torch.uint8, device=dev)

        def unfused():
            lg.lora_linear(x, Wp, A_cat, Bp, y=y, workspace=wsp)
            v = y.view(frames, T, Cp)[:, :, :C].permute(0, 2, 1).float().contiguous()
            lg.euler_step(z, v, s0, s1)
            zb.copy_(z)

        fused_ms, unfused_ms = _time_alternating(
            lambda: lg.lora_linear_euler(x, W, A_cat, B_cat, z, s0, s1, T, z_bf16=zb, workspace=ws), unfused,
            reps, world)
        fl = layer_flops(M, K, C, R)
        peak = peaks["bf16_tflops_sustained"]
        out["projection_euler"] = {
            "workload": f"{w.name} last projection: {M} tokens ({frames} frames x {T} cells), d = {K} -> "
                        f"{C} channels, rank {R}, FP32 latent + bf16 copy",
            "fused_ms": round(fused_ms, 4), "unfused_ms": round(unfused_ms, 4),
            "speedup": round(unfused_ms / fused_ms, 3),
            "tflops": round(fl / (fused_ms * 1e-3) / 1e12, 1), "peak": peak,
            "frac": round(fl / (fused_ms * 1e-3) / 1e12 / peak, 4),
            "peak_kind": f"bf16_tflops_sustained ({peaks['source']}); algorithmic FLOPs with N = {C}",
        }
        del W, As, Bs, A_cat, B_cat, z, zb, ws, Wp, Bp, y, wsp
    # SwiGLU + MXFP8 on a quarter of the tokens.
    Km, N2 = synth.mlp_in_shape(w)
    Mq = (P.M // 4) // 128 * 128 if P.M >= 512 else P.M
    if K == Km and Mq > 0:
        F = N2 // 2
        x = L0["x"][:Mq]
        W2 = synth.weight(w, synth.MLP_IN_LAYER, dev, shape=(Km, N2))
        wq = lg.mx_quantize(W2)
        del W2
        As, Bs = synth.adapters(w, synth.MLP_IN_LAYER, dev, shape=(Km, N2))
        A_cat, B_cat = lg.lora_merge(As, Bs, P.scales)
        del As, Bs
        xq = lg.mx_quantize(x)
        q = (torch.empty((Mq, F), dtype=torch.uint8, device=dev),
             torch.empty(lg.mx_scale_bytes(Mq, F), dtype=torch.uint8, device=dev))
        ws = torch.empty(lg.lora_linear_workspace_size(Mq, Km, N2, R), dtype=torch.uint8, device=dev)
        y = torch.empty((Mq, N2), dtype=torch.bfloat16, device=dev)

        def unfused():
            lg.lora_linear_mxfp8(x, xq, wq, A_cat, B_cat, y=y, workspace=ws)
            s = torch.nn.functional.silu(y[:, :F]) * y[:, F:]
            lg.mx_quantize(s, codes=q[0], scales=q[1])

        fused_ms, unfused_ms = _time_alternating(
            lambda: lg.lora_linear_swiglu_mxfp8(x, xq, wq, A_cat, B_cat, out=q, workspace=ws), unfused, reps, world)
        fl = layer_flops(Mq, Km, N2, R)
        peak = 2.0 * peaks["bf16_tflops_sustained"]
        out["swiglu_mxfp8"] = {
            "workload": f"{w.name} MLP input projection: {Mq} tokens (a quarter of the grid), d = {Km} -> 2 x {F} "
                        f"(gate, up), rank {R}, MXFP8 output",
            "fused_ms": round(fused_ms, 4), "unfused_ms": round(unfused_ms, 4),
            "speedup": round(unfused_ms / fused_ms, 3),
            "tflops": round(fl / (fused_ms * 1e-3) / 1e12, 1), "peak": round(peak, 1),
            "frac": round(fl / (fused_ms * 1e-3) / 1e12 / peak, 4),
            "peak_kind": "fp8 dense, derived: measured bf16 sustained x 2 (the nominal fp8 / bf16 ratio)",
        }
        del wq, A_cat, B_cat, xq, q, ws, y
    torch.cuda.empty_cache()
    status = lg.get_last_device_error()
    if status != lg.LG_OK:
        raise SystemExit(f"device error during the fusion runs: {lg.status_string(status)}")
    return out


def bytes_per_kernel(P):
    n = P.up.numel()
    M = P.M
    merge = sum(4 * P.R * (L["K"] + L["N"]) * 2 for L in P.layers)  # read adapters, write merged
    return {"renoise": 8.0 * n, "euler": 12.0 * n, "lora_merge": merge / len(P.layers),
            "lora_linear_min_bytes": [2.0 * (M * L["K"] + L["N"] * L["K"] + M * L["N"]) + 4.0 * P.R * (L["K"] + L["N"])
                                      for L in P.layers]}


def time_steps(P, args, world, rank, dev):
    """W untimed steps, then K steps bracketed by a barrier and a device
    synchronize on both sides, timed with CUDA events (max over ranks), the
    SM clocks sampled meanwhile.  Returns (ms, per-op event times, launches,
    clock record)."""
    import lora_gemm_b200 as lg

    for _ in range(args.warmup):
        run_step(P)
    torch.cuda.synchronize()
    if lg.get_last_device_error() != lg.LG_OK:
        raise SystemExit("device error during warm-up")

    clocks = ClockSampler(dev.index) if rank == 0 else None
    if clocks:
        clocks.start()
    ev = []
    launches0 = lg.launch_count()
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for _ in range(args.steps):
        run_step(P, ev)
    t_end.record()
    torch.cuda.synchronize()
    barrier(world)
    launches = lg.launch_count() - launches0
    clk = clocks.stop() if clocks else None
    status = lg.get_last_device_error()
    if status != lg.LG_OK:
        raise SystemExit(f"device error during timed steps: {lg.status_string(status)}")
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    per = {}
    for name, s, e in ev:
        per.setdefault(name, []).append(s.elapsed_time(e))
    return elapsed_ms, per, launches, clk


def kernel_report(P, per, peaks):
    """Per-kernel figures of timed steps: the linear layers against the bf16
    peaks, re-noise, Euler and merge against HBM."""
    M = P.M
    flops = [layer_flops(M, L["K"], L["N"], P.R) for L in P.layers]
    lin_ms = [statistics.mean(per[f"lora_linear{k}"]) for k in range(len(P.layers))]
    achieved_tflops = sum(flops) / (sum(lin_ms) * 1e-3) / 1e12
    peak_t = peaks["bf16_tflops_sustained"]
    bpk = bytes_per_kernel(P)
    ren_ms = statistics.mean(per["renoise"])
    eul_ms = statistics.mean([t for k in range(3) for t in per[f"euler{k}"]])
    mer_ms = statistics.mean(per["lora_merge"])
    hbm = peaks["hbm_gbs"]

    def gbs(b, ms):
        return b / (ms * 1e-3) / 1e9

    kernels = {
        "lora_linear": {
            "per_layer_ms": [round(t, 4) for t in lin_ms],
            "per_layer_tflops": [round(f / (t * 1e-3) / 1e12, 1) for f, t in zip(flops, lin_ms)],
            "tflops": round(achieved_tflops, 1),
            "frac_of_measured_sustained": round(achieved_tflops / peak_t, 4),
            "frac_of_measured_burst": round(achieved_tflops / peaks["bf16_tflops"], 4),
            "frac_of_spec_2250": round(achieved_tflops / 2250.0, 4),
            "tokens_per_s_per_layer": [round(M / (t * 1e-3), 1) for t in lin_ms],
            "note": "time includes the bf16 conversion of the merged factors inside the call",
        },
        "renoise": {"ms": round(ren_ms, 5), "gbs": round(gbs(bpk["renoise"], ren_ms), 1),
                    "frac_of_measured_hbm": round(gbs(bpk["renoise"], ren_ms) / hbm, 4),
                    "frac_of_8000": round(gbs(bpk["renoise"], ren_ms) / 8000.0, 4)},
        "euler_step": {"ms": round(eul_ms, 5), "gbs": round(gbs(bpk["euler"], eul_ms), 1),
                       "frac_of_measured_hbm": round(gbs(bpk["euler"], eul_ms) / hbm, 4),
                       "frac_of_8000": round(gbs(bpk["euler"], eul_ms) / 8000.0, 4)},
        "lora_merge": {"ms": round(mer_ms, 5), "gbs": round(gbs(bpk["lora_merge"], mer_ms), 1)},
    }
    return kernels, flops, achieved_tflops


def run_ours(args, rank, world, local):
    import lora_gemm_b200 as lg
    import synth

    peaks = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    w = synth.WORKLOADS[args.workload]
    if args.scaling == "strong":
        # One clip split by latent frames; the noise offset is the global index
        # of the rank's first latent element.
        frames = _dist().frame_shard(w.frames, rank, world)
        _, (e0, _) = _dist().clip_shard(w.frames, w.channels, w.height, w.width, rank, world)
        P = Problem(w, dev, tokens=args.tokens, noise_offset=e0, frames=frames)
    else:
        P = Problem(w, dev, tokens=args.tokens, noise_offset=_dist().noise_offset(rank, w.latent_numel))
    torch.cuda.synchronize()

    elapsed_ms, per, launches, clk = time_steps(P, args, world, rank, dev)
    M = P.M
    if args.scaling == "strong":
        # the whole clip's tokens over the slowest rank's time
        value = (w.tokens if args.tokens is None else _dist().sum_over_ranks(M, world)) * args.steps / (
            elapsed_ms * 1e-3)
    else:
        value = _dist().whole_job_rate(M, world, args.steps, elapsed_ms)

    # Dominant kernel: lora_linear (tensor-bound).
    kernels, flops, achieved_tflops = kernel_report(P, per, peaks)
    peak_t = peaks["bf16_tflops_sustained"]
    traffic = load_traffic(w.name, M)
    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 3),
        "higher_is_better": True,
        "scaling": args.scaling,
        "vs_baseline": None,
        "dtype": "bf16",
        "dtype_detail": "bf16 x, W and factor copies on the tensor cores with FP32 accumulate; FP32 latent",
        "data": "synthetic (seeded torch draws shaped like the pages' 2K grid; no weights)",
        "config": {
            "workload": w.name,
            "latent": list(w.latent_shape),
            "tokens": M,
            "tokens_override": args.tokens is not None,
            "d": w.d,
            "layers_k_n": [list(s) for s in w.shapes],
            "rank": P.R,
            "adapter_ranks": list(synth.ADAPTER_RANKS),
            "schedule": list(synth.SIGMA_SCHEDULE),
            "parallelism": (f"replicas x{world} (weak scaling, no collective)" if args.scaling == "weak" else
                            f"one clip split by latent frames over {world} ranks (strong scaling, no collective)"),
            "l2": "no explicit flush: lora_linear inputs (7.6-30.5 GB) exceed L2, and each elementwise kernel's "
                  "inputs were last touched before >= 364 MB of other traffic",
        },
        "roofline": {
            "bound": "tensor",
            "kernel": "k_lora_linear",
            "achieved": round(achieved_tflops, 1),
            "peak": peak_t,
            "peak_kind": f"bf16_tflops_sustained ({peaks['source']})",
            "unit": "TFLOP/s",
            "frac": round(achieved_tflops / peak_t, 4),
            "frac_is_of": "the measured sustained bf16 rate (a cuBLAS GEMM looped for seconds under the 1 kW cap), "
                          "the right denominator for a kernel inside a step of hundreds of ms",
            "frac_of_measured_burst": round(achieved_tflops / peaks["bf16_tflops"], 4),
            "frac_of_spec_2250": round(achieved_tflops / 2250.0, 4),
            "sm_mhz_median": (clk or {}).get("sm_mhz"),
            "traffic": traffic,
            "algorithmic_flops_per_token": sum(f / M for f in flops),
        },
        "kernels": kernels,
        "clocks": clk,
        "gpu_launches": int(launches),
        "launches_per_step": int(launches) // max(args.steps, 1),
    }
    if not args.no_mxfp8:
        result["mxfp8"] = run_mxfp8(P, args, world, peaks)
    if not args.no_fusions:
        result["library_ab"] = run_library_ab(P, args, world, peaks)
        result["fusions"] = run_fusions(P, args, world, peaks)
        result["ic_routes"] = run_ic_routes(P, args, world, peaks)
        result["elementwise_isolated"] = run_elementwise_isolated(P, args, world, peaks)
    if not args.no_e2e:
        result["e2e"] = run_e2e(P, args, world)
        # Hand the pinned buffers back to the host (torch keeps them cached).
        torch._C._host_emptyCache()
    del P
    torch.cuda.empty_cache()
    names = [n for n in args.workloads.split(",") if n and n != w.name] if args.workloads else []
    if names:
        result["workloads"] = run_workloads(names, args, world, rank, dev, peaks)
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, target_s=args.cpu_seconds)
    return result


def run_workloads(names, args, world, rank, dev, peaks):
    """The other grids of the pages, each as its own step (merge, re-noise,
    its layers, three Euler steps) timed like the headline, with its own
    clock record.  Inputs are held lean (one activation buffer of the widest
    K, one output buffer of the widest N) so the 4K step fits one GPU.  The
    4K grid also sweeps its re-noise start over the main schedule's 0.909 and
    the IC routes' 0.835 (up3) and 0.923 (up4) on the same latent."""
    import lora_gemm_b200 as lg
    import synth

    out = {}
    for name in names:
        w = synth.WORKLOADS[name]
        # The inputs of a grid are allocated before anything is timed; a device
        # without room for them (the 4K step holds ~123 GB) records that and
        # moves on.  The ranks agree first (max over ranks of a failure flag),
        # so that all of them skip the grid when any one is short of memory and
        # every rank runs the same collectives.
        P, err = None, None
        try:
            if args.scaling == "strong":
                frames = _dist().frame_shard(w.frames, rank, world)
                _, (e0, _) = _dist().clip_shard(w.frames, w.channels, w.height, w.width, rank, world)
                P = Problem(w, dev, noise_offset=e0, lean=True, frames=frames)
            else:
                P = Problem(w, dev, noise_offset=_dist().noise_offset(rank, w.latent_numel), lean=True)
        except torch.cuda.OutOfMemoryError as e:
            err = f"device memory: {str(e).splitlines()[0][:160]}"
        if max_over_ranks(1.0 if err else 0.0, world) > 0.0:
            del P
            torch.cuda.empty_cache()
            out[name] = {"unavailable": err or "device memory on another rank"}
            continue
        torch.cuda.synchronize()
        # Enough timed steps for >= 1.5 s under the clock sampler (200 ms period).
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run_step(P)
        e1.record()
        torch.cuda.synchronize()
        one_ms = max_over_ranks(e0.elapsed_time(e1), world)
        wargs = argparse.Namespace(**vars(args))
        wargs.steps = max(args.steps, min(2000, int(1500.0 / max(one_ms, 1e-3)) + 1))
        ms, per, launches, clk = time_steps(P, wargs, world, rank, dev)
        kernels, flops, tflops = kernel_report(P, per, peaks)
        rec = {
            "latent": list(w.latent_shape), "tokens": P.M, "d": w.d, "layers_k_n": [list(x) for x in w.shapes],
            "tokens_per_s": round(w.tokens * wargs.steps / (ms * 1e-3) if args.scaling == "strong"
                                  else _dist().whole_job_rate(P.M, world, wargs.steps, ms), 1),
            "ms_per_step": round(ms / wargs.steps, 3), "steps": wargs.steps, "warmup": args.warmup,
            "kernels": kernels, "clocks": clk, "gpu_launches": int(launches),
            "inputs": "lean: layer activations are views of one buffer of the widest K, outputs share one buffer",
        }
        if len(w.sigma_starts) > 1:
            sched = [float(torch.tensor(x, dtype=torch.float32)) for x in synth.SIGMA_SCHEDULE]
            routes = {}
            for s0 in w.sigma_starts:
                s32 = float(torch.tensor(s0, dtype=torch.float32))
                routes[f"{s0}"] = sched if s32 == sched[0] else lg.shift_ladder(s32)
            rec["sigma_sweep"] = run_ic_routes(P, args, world, peaks, routes=routes)
        out[name] = rec
        del P
        torch.cuda.empty_cache()
    return out


def load_traffic(workload, tokens):
    """DRAM bytes per lora_linear launch from the committed ncu summary, or None
    when the summary is missing, was taken on a different kernel source, or
    was scaled to another workload or token count."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "lora_linear_traffic.json")
    src = os.path.join(ROOT, "lora_gemm_b200", "csrc", "lg_lora_linear.cu")
    try:
        with open(path) as f:
            t = json.load(f)
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except (OSError, ValueError):
        return None
    if t.get("kernel_source_sha256") != digest or workload != "2k" or t.get("scaled_to_tokens") != tokens:
        return None
    return t.get("traffic_bytes_per_launch")


def run_e2e(P, args, world):
    """The same step through the public API with host buffers: every step
    copies its inputs (activations, upscaled latent, velocities) from pinned
    host memory and reads its results (y of each layer, the final latent)
    back, all inside the timed region.  Copies run on two copy streams beside
    the compute stream, ordered by events: an input is copied in as soon as
    its device buffer is free (the previous step's last use of it is done),
    an op waits only for its own inputs, and an output is copied out as soon
    as the op that writes it is done (and is not overwritten before that copy
    ends).  Host->device, device->host and compute overlap within and across
    steps, as a serving loop would run them.  (Double-buffering the
    activations on the device gave no further gain: the step is then bound by
    the host link, ~41 GB/s each way with both directions busy.)"""
    import lora_gemm_b200 as lg

    compute = torch.cuda.current_stream()
    s_in = torch.cuda.Stream()
    s_out = torch.cuda.Stream()

    def pinned(t):
        return torch.empty(t.shape, dtype=t.dtype, pin_memory=True)

    # Inputs in the order their device buffers are released by a step (one
    # copy stream serialises them, so a copy never waits behind a later
    # release); outputs in the order they are produced.
    last_use = {}
    for k, L in enumerate(P.layers):
        last_use[id(L["x"])] = k
    inputs = [P.up]
    for k in range(len(P.sigmas) - 1):
        if k < len(P.layers) and last_use[id(P.layers[k]["x"])] == k:
            inputs.append(P.layers[k]["x"])
        inputs.append(P.v[k])
    outputs = [L["y"] for L in P.layers] + [P.x_lat]
    h2d = sum(t.numel() * t.element_size() for t in inputs)
    d2h = sum(t.numel() * t.element_size() for t in outputs)

    # Pinned host buffers, within this rank's share of the host's memory (the
    # ranks of a node share it): separate input and output buffers when they
    # fit, else one pool that the outputs overwrite after the inputs were read
    # from it (same copies, same timing; later steps then read back earlier
    # results as their inputs), else no end-to-end figure.
    def padded(t):
        return (t.numel() * t.element_size() + 4095) // 4096 * 4096

    need_in, need_out = sum(padded(t) for t in inputs), sum(padded(t) for t in outputs)
    # Every rank reads the free memory before any rank pins, and all take the
    # most restrictive choice, so that they run the same collectives.
    barrier(world)
    choice = int(max_over_ranks(float(host_buffer_choice(need_in, need_out, _host_budget())), world))
    if choice == 0:
        host_mode = "separate"
        host_in = {id(t): pinned(t) for t in inputs}
        host_out = {id(t): pinned(t) for t in outputs}
    elif choice == 1:
        host_mode = "shared pool (host memory)"
        pool = torch.empty(max(need_in, need_out), dtype=torch.uint8, pin_memory=True)

        def carve(ts):
            views, off = {}, 0
            for t in ts:
                n = t.numel() * t.element_size()
                views[id(t)] = pool[off:off + n].view(t.dtype).view(t.shape)
                off += padded(t)
            return views

        host_in, host_out = carve(inputs), carve(outputs)
    else:
        return {"unavailable": f"host memory: the step's pinned buffers need {max(need_in, need_out) / 1e9:.0f} GB "
                               "per rank even shared, more than a rank's share of the node's free memory"}
    for t in inputs:
        host_in[id(t)].copy_(t)

    arrived = {}    # input -> event: this step's copy-in is done
    released = {}   # input -> event: the previous step's last use of its device buffer is done
    copied = {}     # output -> event: the previous copy-out is done

    def ev(stream):
        e = torch.cuda.Event()
        e.record(stream)
        return e

    def copy_in():
        with torch.cuda.stream(s_in):
            for t in inputs:
                if id(t) in released:
                    s_in.wait_event(released[id(t)])
                t.copy_(host_in[id(t)], non_blocking=True)
                arrived[id(t)] = ev(s_in)

    def use(t):
        compute.wait_event(arrived[id(t)])
        return t

    def release(t):
        released[id(t)] = ev(compute)

    def write(t):
        if id(t) in copied:
            compute.wait_event(copied[id(t)])

    def copy_out(t):
        done = ev(compute)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            host_out[id(t)].copy_(t, non_blocking=True)
            copied[id(t)] = ev(s_out)

    def step():
        copy_in()
        for L in P.layers:
            lg.lora_merge(L["As"], L["Bs"], P.scales, L["A_cat"], L["B_cat"])
        up = use(P.up)
        write(P.x_lat)
        lg.renoise(up, P.sigmas[0], P.w.seed, offset=P.noise_offset, out=P.x_lat)
        release(P.up)
        for k in range(len(P.sigmas) - 1):
            if k < len(P.layers):
                L = P.layers[k]
                x = use(L["x"])
                write(L["y"])
                lg.lora_linear(x, L["W"], L["A_cat"], L["B_cat"], y=L["y"], workspace=L["ws"])
                if last_use[id(L["x"])] == k:
                    release(L["x"])
                copy_out(L["y"])
            v = use(P.v[k])
            lg.euler_step(P.x_lat, v, P.sigmas[k], P.sigmas[k + 1])
            release(P.v[k])
        copy_out(P.x_lat)

    def join():
        compute.wait_stream(s_in)
        compute.wait_stream(s_out)

    step()
    join()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 5))
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    s_in.wait_stream(compute)
    s_out.wait_stream(compute)
    for _ in range(steps):
        step()
    join()
    e.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e), world)
    # Every step computes the same outputs from the same inputs: what came
    # back to the host must equal what the device holds (sampled rows).
    for t in outputs:
        rows = torch.arange(0, t.shape[0], max(1, t.shape[0] // 97), device=t.device)
        if not torch.equal(host_out[id(t)][rows.cpu()], t[rows].cpu()):
            raise RuntimeError("e2e: a copied-out result differs from the device result")
    return {"value": round(_dist().whole_job_rate(P.M, world, steps, ms), 1), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": round(ms / steps, 3), "host_buffers": host_mode,
            "overlap": "host->device, compute and device->host on three streams, ordered by events per buffer"}


def host_buffer_choice(need_in, need_out, budget):
    """0: separate pinned input and output buffers; 1: one pool shared by
    both; 2: no end-to-end figure.  budget None means unknown (assume room)."""
    if budget is None or need_in + need_out <= budget:
        return 0
    return 1 if max(need_in, need_out) <= budget else 2


def _host_budget():
    """Bytes of host memory this rank may pin: 80 % of what the kernel reports
    available, split among the ranks of this node; None if unknown."""
    try:
        with open("/proc/meminfo") as f:
            avail = next(int(line.split()[1]) * 1024 for line in f if line.startswith("MemAvailable"))
    except (OSError, StopIteration, ValueError):
        return None
    local = int(os.environ.get("LOCAL_WORLD_SIZE", "1") or 1)
    return 0.8 * avail / max(local, 1)


# ---------------------------------------------------------------------------
# The FP64 oracle on the host cores.
# ---------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        n = [d.get("num_threads", 1) for d in info if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


class OracleStep:
    """The whole path for a sample of `tokens` tokens of the workload, in FP64 on the CPU."""

    def __init__(self, w, tokens):
        import numpy as np

        import synth

        self.w = w
        self.tokens = tokens
        self.np = np
        g = np.random.default_rng(w.seed)
        self.layers = []
        for K, N in w.shapes:
            x = g.standard_normal((tokens, K)).astype(np.float32).astype(np.float64)
            W = g.standard_normal((N, K)) * K ** -0.5
            As = [(g.standard_normal((r, K)) * K ** -0.5).astype(np.float32) for r in synth.ADAPTER_RANKS]
            Bs = [(g.standard_normal((N, r)) * synth.B_STD).astype(np.float32) for r in synth.ADAPTER_RANKS]
            self.layers.append((x, W, As, Bs))
        n = tokens * w.channels
        self.n = n
        self.up = g.standard_normal(n).astype(np.float32)
        self.v = [g.standard_normal(n).astype(np.float32) for _ in range(3)]
        self.scales = synth.ADAPTER_SCALES

    def run(self):
        from oracle import flow, lora, noise

        eps = noise.normal(self.w.seed, 0, self.n)
        z = flow.renoise(self.up, eps, flow.SCHEDULE[0])
        for k, (x, W, As, Bs) in enumerate(self.layers):
            A_cat, B_cat = lora.lora_merge(As, Bs, self.scales)
            lora.lora_linear(x, W, A_cat, B_cat)
            z = flow.euler_step(z, self.v[k], flow.SCHEDULE[k], flow.SCHEDULE[k + 1])
        return z


def _oracle_tokens_for(w, seconds, cap):
    """Tokens whose OracleStep takes about `seconds`: a fixed cost (the
    merge, per-layer setup) plus a per-token cost, fitted from two probes."""
    times = []
    for n in (32, 256):
        probe = OracleStep(w, n)
        probe.run()
        t0 = time.perf_counter()
        probe.run()
        times.append(time.perf_counter() - t0)
    per_token = max((times[1] - times[0]) / 224.0, 1e-7)
    fixed = max(times[0] - 32 * per_token, 0.0)
    return int(max(32, min(cap, (seconds - fixed) / per_token)))


def cpu_baseline(w, target_s=15.0):
    tokens = _oracle_tokens_for(w, target_s, 16384)
    step = OracleStep(w, tokens)
    t0 = time.perf_counter()
    step.run()
    dt = time.perf_counter() - t0
    return {"value": round(tokens / dt, 2), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{tokens} tokens of the {w.name} workload through merge, renoise, the three layers and "
                      f"three Euler steps in FP64 ({dt:.1f} s)"}


def run_reference(args, rank, world):
    import synth

    w = synth.WORKLOADS[args.workload]
    per_step_s = getattr(args, "reference_seconds", 90.0) / max(1, args.steps + args.warmup)
    tokens = _oracle_tokens_for(w, per_step_s, 12288)
    step = OracleStep(w, tokens)
    for _ in range(args.warmup):
        step.run()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step.run()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = tokens * args.steps / total
    sample = (f"{tokens} tokens of the {w.name} workload per step through merge, renoise, the three layers "
              f"and three Euler steps in FP64 on the host CPU")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "latent": list(w.latent_shape), "tokens": w.tokens, "d": w.d,
                   "layers_k_n": [list(s) for s in w.shapes], "rank": sum(synth.ADAPTER_RANKS),
                   "parallelism": "host CPU (rank 0 only)"},
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-mxfp8", action="store_true")
    ap.add_argument("--no-fusions", action="store_true", help="skip the fused-epilogue comparisons, the IC routes and the isolated elementwise runs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="weak: every rank runs the whole workload; strong: one clip split by latent frames")
    ap.add_argument("--workloads", default="768p,1080p,4k",
                    help="other grids timed after the headline, comma-separated ('' for none)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=90.0,
                    help="CPU seconds the oracle arm spends over all its warm-up and timed steps")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the token count of the linear layers (profiling runs only)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    rank, world, local = _dist().init(args.gpus, backend="nccl")
    try:
        result = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        _dist().destroy(world)


if __name__ == "__main__":
    main()
