#!/usr/bin/env python
"""Benchmark of the B200 int4 MoE layer (libmoe), one JSON line on stdout (rank 0).

Headline workload (default): the 16384-token prefill of a 40-layer stack, processed as four
4096-token chunks per layer (chunk-major: each chunk passes through layers 0..39), Zipf(1.2)
routing skew, synthetic random-init weights of the 256-expert int4 layer.  value = MoE-layer
tokens/s = tokens x layers / step time.  A second measurement on the same line ("decode") times
batch-1 decode over 40 distinct layers replayed as one CUDA graph (us per token per layer).

Timing: W untimed warm-up steps, then K steps between CUDA events on the launching stream,
bracketed by a barrier + synchronize, max over ranks.  Every layer's weights (457 MB) exceed the
126 MB L2, so no flush is needed between steps.  Per-kernel durations for the roofline come from
events the library records around each of its launches in a separate profiled pass of K steps.

Multi-GPU (torchrun): every rank runs its own replica on its own tokens (the layer shards by
tokens with no exchange), value = all ranks' tokens / max-over-ranks time ("scaling": "weak").

--impl reference: the CPU oracle (test infrastructure) timed as it stands on the host cores over a
bounded token sample of the same workload; rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import re
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill16k_zipf",
                    choices=["prefill16k_zipf", "prefill4k_zipf", "prefill512", "decode"])
    ap.add_argument("--layers", type=int, default=None, help="override the stack depth (quick runs)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the prefill512 / prefill4k_zipf fractions")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target oracle sample time")
    ap.add_argument("--ablations", action="store_true",
                    help="also time the pages' two prefill ablations (host-synchronised routing, fp16 "
                         "weights dequantised once into HBM) against the product path")
    return ap.parse_args()


# ------------------------------------------------------------------------------------------ dist
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend):
        import torch
        import torch.distributed as dist
        if self.world > 1:
            import datetime
            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        import torch.distributed as dist
        dev = torch.device("cuda", self.local) if torch.cuda.is_available() else torch.device("cpu")
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ---------------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [v.strip() for v in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = max((num(r[2]) for r in rows if num(r[2]) is not None), default=None)
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        # "under load": samples drawing more than idle power
        loaded = [s for s, pw in zip(sm, power) if pw is not None and pw > 250] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------------------- stacks
def build_stack(shape, n_layers, max_tokens, decode_max_tokens, keep_host_layer0=False, flags=0):
    import torch
    from bit_grouped_expert_router_b200 import _lib as M
    from bit_grouped_expert_router_b200 import synth
    layers, host0 = [], None
    for l in range(n_layers):
        w = synth.make_layer(shape, l, device="cuda")
        if l == 0 and keep_host_layer0:
            host0 = {k: (v.cpu() if v is not None else None) for k, v in w.items()}
        layers.append(M.Layer.from_shape(w, shape, max_tokens=max_tokens, decode_max_tokens=decode_max_tokens,
                                         flags=flags))
        del w
    torch.cuda.synchronize()
    return layers, host0


def timed(fn, steps, warmup, dist):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        fn()
    e1.record(s)
    torch.cuda.synchronize()
    dist.barrier()
    ms = e0.elapsed_time(e1) / steps
    return dist.max(ms)


def profile_pass(layers, fn, steps):
    import torch
    for L in layers:
        L.profile(True)
    for _ in range(steps):
        fn()
    torch.cuda.synchronize()
    tot = {}
    for L in layers:
        for k, (ms, n) in L.profile_read().items():
            a = tot.setdefault(k, [0.0, 0])
            a[0] += ms
            a[1] += n
        L.profile(False)
    return {k: {"avg_us": 1000.0 * v[0] / v[1], "launches": v[1], "total_ms": v[0]} for k, v in tot.items()}


# ---------------------------------------------------------------------------------------- prefill
def gemm_flops(shape):
    rows = shape.T * shape.k + (shape.T if shape.has_shared else 0)
    return 2.0 * rows * 2 * shape.I * shape.H, 2.0 * rows * shape.I * shape.H


def tile_stats(layers, xs, shape, prof, clk):
    """Tile fill and executed k-steps of the grouped GEMMs over every (layer, chunk) call of a step,
    from the library's own routing (moe_route's bucket offsets).  The tile height follows the
    library's launch-shape rule (256-token tiles when T*k > 64*E, else 128).  fill = bucket rows /
    (tiles x tile height); a k-step is one 64-deep slice of the contraction for one 128-row
    m-tile, so cycles_per_kstep = launch time x SM clock x SMs / k-steps."""
    import torch
    tile_rows = 256 if shape.T * shape.k > 64 * shape.E else 128
    tiles, rows, calls = 0, 0, 0
    for l, L in enumerate(layers):
        for x in xs[l]:
            off = L.route(x)["offsets"].to(torch.int64)
            cnt = off[1:] - off[:-1]
            tiles += int(((cnt + tile_rows - 1) // tile_rows).sum())
            rows += int(cnt.sum())
            if shape.has_shared:
                tiles += (shape.T + tile_rows - 1) // tile_rows
                rows += shape.T
            calls += 1
    tiles_per_call = tiles / calls
    ks_gu = tiles_per_call * (2 * shape.I // 128) * (shape.H // 64)
    ks_dn = tiles_per_call * (shape.H // 128) * (shape.I // 64)
    out = {"tile_rows": tile_rows, "tiles_per_launch": round(tiles_per_call, 1),
           "tile_fill": round(rows / (tiles * tile_rows), 4),
           "ksteps_per_launch": {"gemm_gateup": round(ks_gu), "gemm_down": round(ks_dn)}}
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    mhz = (clk or {}).get("sm_mhz")
    if mhz:
        out["cycles_per_kstep"] = {
            k: round(prof[k]["avg_us"] * mhz * sms / n) for k, n in (("gemm_gateup", ks_gu), ("gemm_down", ks_dn))}
    return out


def run_prefill(args, dist, peaks, peak_src):
    import torch
    from bit_grouped_expert_router_b200 import synth
    shape = synth.WORKLOADS[args.workload]
    n_layers = args.layers or shape.layers
    chunks = shape.chunks
    layers, host0 = build_stack(shape, n_layers, shape.T, 16, keep_host_layer0=True)
    xs = [[synth.make_x(shape, l, c, device="cuda") for c in range(chunks)] for l in range(n_layers)]
    out = torch.empty((shape.T, shape.H), dtype=torch.bfloat16, device="cuda")

    def step():
        for c in range(chunks):
            for l in range(n_layers):
                layers[l].forward(xs[l][c], out=out)

    tokens_per_step = shape.T * chunks * n_layers  # layer-tokens
    clocks = ClockSampler(torch.cuda.current_device())
    # warm-up outside the sampled window, then the timed region with clocks sampled
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks.start()
    ms = timed(step, args.steps, 0, dist)
    clk = clocks.stop()
    for L in layers:
        assert L.status() == 0, "device status after the timed region"
    value = dist.world * tokens_per_step / (ms / 1000.0)

    prof = profile_pass(layers, step, args.steps)
    f_gu, f_dn = gemm_flops(shape)
    peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])  # fp16 dense == bf16 dense
    roof = None
    if "gemm_gateup" in prof:
        a = f_gu / (prof["gemm_gateup"]["avg_us"] * 1e-6) / 1e12
        roof = {"bound": "tensor", "kernel": "gemm_gateup (tcgen05 grouped GEMM + SwiGLU)",
                "achieved": round(a, 1), "peak": peak_tf, "unit": "TFLOP/s", "frac": round(a / peak_tf, 4),
                "traffic": profiled_traffic("gemm_gateup"), "peak_source": f"{peak_src} bf16 sustained (fp16 dense rate = bf16 dense rate)",
                "flops_per_launch": f_gu}
    gg = None
    if "gemm_gateup" in prof and "gemm_down" in prof:
        t = (prof["gemm_gateup"]["avg_us"] + prof["gemm_down"]["avg_us"]) * 1e-6
        a = (f_gu + f_dn) / t / 1e12
        gg = {"achieved_tflops": round(a, 1), "frac_of_peak": round(a / peak_tf, 4),
              "us_per_chunk": round(t * 1e6, 1)}
        gg.update(tile_stats(layers, xs, shape, prof, clk))
    res = dict(value=value, ms=ms, clocks=clk, roofline=roof, kernels=prof, grouped_gemm=gg,
               launches=len(prof) * chunks * n_layers * args.steps, shape=shape, n_layers=n_layers,
               tokens_per_step=tokens_per_step)

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    if not args.no_e2e:
        xh = [[xs[l][c].cpu().pin_memory() for c in range(chunks)] for l in range(n_layers)]
        # one stream per prompt chunk, each chunk through the layers in order (chunked prefill);
        # chunk c enters layer l after chunk c - 1 has left it (one event per layer handle, so a
        # handle's workspace is never used by two streams at once): a wavefront in which one
        # chunk's PCIe copies overlap the other chunks' kernels.  One pinned output per chunk.
        side = [torch.cuda.Stream() for _ in range(chunks)]
        done = [torch.cuda.Event() for _ in range(n_layers)]
        oh = [torch.empty((shape.T, shape.H), dtype=torch.bfloat16).pin_memory() for _ in side]

        def step_host():
            cur = torch.cuda.current_stream()
            for s in side:
                s.wait_stream(cur)
            for l in range(n_layers):
                for c in range(chunks):
                    side[c].wait_event(done[l])   # (not yet recorded: no wait)
                    layers[l].forward_host_async(xh[l][c], oh[c], side[c])
                    done[l].record(side[c])
            for s in side:
                cur.wait_stream(s)
        ms_e2e = timed(step_host, max(1, args.steps // 2), 1, dist)
        bytes_io = shape.T * shape.H * 2 * chunks * n_layers
        res["e2e"] = {"value": dist.world * tokens_per_step / (ms_e2e / 1000.0), "unit": "tokens/s",
                      "h2d_bytes_per_step": bytes_io, "d2h_bytes_per_step": bytes_io,
                      "ms_per_step": round(ms_e2e, 3),
                      "api": "moe_forward_host_async (pinned host buffers, one stream per chunk, layer order kept)"}
        del xh
    res["host0"] = host0
    res["x0"] = xs[0][0].cpu()
    for L in layers:
        L.close()
    del xs
    torch.cuda.empty_cache()
    return res


def decode_gemv_only(shape, xs, reps, hbm, peak_src):
    """The expert GEMV kernels alone: batch-1 decode through the multi-kernel chain (router, top-k,
    gate/up GEMV, down GEMV) on 8 distinct layers; bytes = the k+1 experts' packed weights."""
    import torch
    from bit_grouped_expert_router_b200 import _lib as M
    from bit_grouped_expert_router_b200 import synth
    n = min(8, len(xs))
    layers = []
    for l in range(n):
        w = synth.make_layer(shape, l, device="cuda")
        layers.append(M.Layer.from_shape(w, shape, max_tokens=16, decode_max_tokens=16,
                                         flags=M.MOE_FLAG_DECODE_UNFUSED))
        del w
    outs = [torch.empty((1, shape.H), dtype=torch.bfloat16, device="cuda") for _ in range(n)]

    def step():
        for l in range(n):
            layers[l].forward(xs[l], out=outs[l])

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    torch.cuda.synchronize()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    chain_us = e0.elapsed_time(e1) * 1000.0 / (reps * n)
    del g
    prof = profile_pass(layers, step, reps)
    for L in layers:
        assert L.status() == 0
        L.close()
    nexp = shape.k + 1
    b = nexp * ((shape.I // 64) * (shape.H // 64) + (shape.H // 128) * (shape.I // 64)) * 4608
    t = (prof["gemv_gateup"]["avg_us"] + prof["gemv_down"]["avg_us"]) * 1e-6
    a = b / t / 1e9
    return {"kernels": "gemv_gateup + gemv_down of the multi-kernel chain (per-kernel events, eager: "
                       "includes the host's launch gaps, an upper bound on their time)",
            "us": round(t * 1e6, 3), "bytes": b, "achieved": round(a, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(a / hbm, 4), "peak_source": f"{peak_src} hbm_gbs",
            "chain_us_per_layer_in_graph": round(chain_us, 3),
            "chain_kernels_us_eager": {k: round(v["avg_us"], 2) for k, v in prof.items()}}


def small_batch_decode(shape, reps, hbm, peak_src):
    """Decode batches of T = 1..16 tokens through both paths of the same 8 distinct layers: the
    sparse GEMV path (a handle with decode_max_tokens = 16) and the grouped-GEMM prefill path (a
    handle with decode_max_tokens = 0), each pass over the 8 layers replayed as one CUDA graph.
    Per T: us per layer call for each path, the GEMV path's HBM fraction (algorithmic bytes = the
    experts that receive a token + router + shared gate + x/out) and where the GEMM path wins."""
    import torch
    from bit_grouped_expert_router_b200 import _lib as M
    from bit_grouped_expert_router_b200 import synth
    n = 8
    gemv, gemm, xs = [], [], []
    for l in range(n):
        w = synth.make_layer(shape, l, device="cuda")
        gemv.append(M.Layer.from_shape(w, shape, max_tokens=16, decode_max_tokens=16))
        gemm.append(M.Layer.from_shape(w, shape, max_tokens=16, decode_max_tokens=0))
        del w
        xs.append(synth.make_x(shape, l, 0, device="cuda", T=16))
    expert_bytes = (shape.I // 64) * (shape.H // 64) * 4608 + (shape.H // 128) * (shape.I // 64) * 4608

    def graph_us(layers, T):
        outs = [torch.empty((T, shape.H), dtype=torch.bfloat16, device="cuda") for _ in range(n)]

        def step():
            for l in range(n):
                layers[l].forward(xs[l][:T], out=outs[l])

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            step()
        torch.cuda.synchronize()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1000.0 / (reps * n)

    rows, crossover = {}, None
    for T in (1, 2, 4, 8, 16):
        u_gemv, u_gemm = graph_us(gemv, T), graph_us(gemm, T)
        active = statistics.mean(int(torch.unique(gemv[l].route(xs[l][:T])["idx"]).numel()) + 1
                                 for l in range(n))
        b = active * expert_bytes + shape.E * shape.H * 4 + shape.H * 4 + 2 * T * shape.H * 2
        rows[str(T)] = {"gemv_us_per_layer": round(u_gemv, 2), "gemm_us_per_layer": round(u_gemm, 2),
                        "gemv_us_per_token_layer": round(u_gemv / T, 2), "active_experts_mean": active,
                        "gemv_hbm_frac": round(b / (u_gemv * 1e-6) / 1e9 / hbm, 4)}
        if crossover is None and u_gemm < u_gemv:
            crossover = T
    for L in gemv + gemm:
        assert L.status() == 0
        L.close()
    return {"layers": n, "timing": "CUDA graph of one pass over the layers, events", "per_T": rows,
            "gemm_path_faster_from_T": crossover, "peak_source": f"{peak_src} hbm_gbs"}


def run_configs(args, dist, peaks, peak_src):
    """The other prefill configurations' roofline fractions: prefill512 (HBM-bound: algorithmic
    bytes = weights of the experts that receive a token + router + shared gate + x/out, over the
    whole-layer time) and prefill4k_zipf (tensor-bound: MoE FLOPs over the two GEMMs' time), each
    on 4 distinct layers (1.8 GB of weights, well above L2)."""
    import torch
    from bit_grouped_expert_router_b200 import synth
    out = {}
    expert_bytes = None
    for name in ("prefill512", "prefill4k_zipf"):
        shape = synth.WORKLOADS[name]
        n = 4
        layers, _ = build_stack(shape, n, shape.T, 16)
        xs = [synth.make_x(shape, l, 0, device="cuda") for l in range(n)]
        expert_bytes = (shape.I // 64) * (shape.H // 64) * 4608 + (shape.H // 128) * (shape.I // 64) * 4608

        def step():
            for l in range(n):
                layers[l].forward(xs[l])

        reps = max(args.steps, 5)
        ms = timed(step, reps, 3, dist) / n
        prof = profile_pass(layers, step, reps)
        active = []
        for l in range(n):
            idx = layers[l].route(xs[l])["idx"]
            active.append(int(torch.unique(idx).numel()) + (1 if shape.has_shared else 0))
        for L in layers:
            assert L.status() == 0
            L.close()
        f_gu, f_dn = gemm_flops(shape)
        t_gemm = (prof["gemm_gateup"]["avg_us"] + prof["gemm_down"]["avg_us"]) * 1e-6
        bytes_alg = statistics.mean(active) * expert_bytes + shape.E * shape.H * 4 + shape.H * 4 + 2 * shape.T * shape.H * 2
        hbm, tf = peaks["hbm_gbs"], peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
        out[name] = {"tokens": shape.T, "layer_us": round(ms * 1000, 2),
                     "layer_tokens_per_s": round(shape.T / (ms / 1000), 1),
                     "active_experts_mean": statistics.mean(active),
                     "hbm_frac_whole_layer": round(bytes_alg / (ms / 1000) / 1e9 / hbm, 4),
                     "algorithmic_bytes": int(bytes_alg),
                     "gemm_tflops": round((f_gu + f_dn) / t_gemm / 1e12, 1),
                     "gemm_tensor_frac": round((f_gu + f_dn) / t_gemm / 1e12 / tf, 4),
                     "kernels_us": {k: round(v["avg_us"], 1) for k, v in prof.items()},
                     "peaks": f"{peak_src}: hbm_gbs {hbm}, bf16 sustained {tf} TFLOP/s"}
        del xs
        torch.cuda.empty_cache()
    return out


def run_ep_single(args):
    """The expert-parallel layer (bit_grouped_expert_router_b200.ep) with one rank, beside
    moe_forward on the same layer and 4096-token chunk: eager calls, CUDA events around whole
    forward calls (the EP forward reads its all-to-all split sizes back to the host once per call)."""
    import torch
    from bit_grouped_expert_router_b200 import _lib as M
    from bit_grouped_expert_router_b200 import synth
    from bit_grouped_expert_router_b200.ep import Exchange, ExpertParallelLayer, LibraryShard
    shape = synth.WORKLOADS["prefill16k_zipf"]
    w = synth.make_layer(shape, 0, device="cuda")
    x = synth.make_x(shape, 0, 0, device="cuda")
    full = M.Layer.from_shape(w, shape, max_tokens=shape.T, decode_max_tokens=16)
    shard = LibraryShard(w, shape.H, shape.I, shape.E, shape.k, shape.has_shared, 0, 1, max_tokens=shape.T)
    ep = ExpertParallelLayer(shard, Exchange(None, 1))
    del w

    def time_us(fn, reps=max(args.steps, 5)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1000.0 / reps

    out = torch.empty((shape.T, shape.H), dtype=torch.bfloat16, device="cuda")
    t_full = time_us(lambda: full.forward(x, out=out))
    t_ep = time_us(lambda: ep.forward(x))
    diff = (ep.forward(x).float() - full.forward(x).float()).abs().max().item()
    assert full.status() == 0
    for L in (shard.router, shard.experts, shard.shared):
        assert L.status() == 0
    full.close()
    shard.close()
    return {"ranks": 1, "tokens": shape.T, "moe_forward_us": round(t_full, 1), "ep_forward_us": round(t_ep, 1),
            "max_abs_diff_vs_moe_forward": round(diff, 4),
            "note": "one rank: route, dispatch plan, row gather, routing-supplied expert forward, shared "
                    "expert, combine; the all-to-all is a local copy"}


def run_ablations(args, dist):
    """The pages' prefill levers, each against the product path on the same 4 layers (eager calls,
    CUDA events): GPU-resident routing vs a host round trip between routing and the expert GEMMs
    (MOE_FLAG_HOST_SYNC_ROUTING), and 4-bit weights rebuilt inside the grouped GEMM vs fp16
    weights dequantised once into HBM (MOE_FLAG_DEQUANT_TO_HBM).  us per layer call."""
    import torch
    from bit_grouped_expert_router_b200 import _lib as M
    from bit_grouped_expert_router_b200 import synth
    out = {}
    variants = (("product", 0), ("host_sync_routing", M.MOE_FLAG_HOST_SYNC_ROUTING),
                ("fp16_weights_in_hbm", M.MOE_FLAG_DEQUANT_TO_HBM))
    for name in ("prefill16k_zipf", "prefill512"):
        shape = synth.WORKLOADS[name]
        n = 4
        xs = [synth.make_x(shape, l, 0, device="cuda") for l in range(n)]
        row = {}
        for vname, flags in variants:
            layers, _ = build_stack(shape, n, shape.T, 16, flags=flags)

            def step():
                for l in range(n):
                    layers[l].forward(xs[l])

            reps = max(args.steps, 5)
            row[vname] = round(timed(step, reps, 3, dist) * 1000.0 / n, 2)
            prof = profile_pass(layers, step, reps)
            row[vname + "_gemm_us"] = round(prof["gemm_gateup"]["avg_us"] + prof["gemm_down"]["avg_us"], 2)
            for L in layers:
                assert L.status() == 0
                L.close()
            del layers
            torch.cuda.empty_cache()
        for vname, _ in variants[1:]:
            row[vname + "_vs_product"] = round(row[vname] / row["product"], 4)
        out[name] = row
        del xs
    out["unit"] = "us per layer call (eager), and the two grouped GEMMs' kernel time"
    return out


def run_decode(args, dist, peaks, peak_src):
    import torch
    from bit_grouped_expert_router_b200 import synth
    shape = synth.WORKLOADS["decode"]
    n_layers = args.layers or shape.layers
    layers, _ = build_stack(shape, n_layers, 16, 16)
    xs = [synth.make_x(shape, l, 0, device="cuda") for l in range(n_layers)]
    outs = [torch.empty((1, shape.H), dtype=torch.bfloat16, device="cuda") for _ in range(n_layers)]

    def eager():
        for l in range(n_layers):
            layers[l].forward(xs[l], out=outs[l])

    def graph_ms():
        eager()
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            eager()
        torch.cuda.synchronize()
        t = timed(g.replay, max(args.steps, 20) * 5, args.warmup, dist)
        del g
        return t

    ms = graph_ms()
    us_layer = ms * 1000.0 / n_layers
    prof = profile_pass(layers, eager, max(args.steps, 20))
    expert_bytes = (shape.I // 64) * (shape.H // 64) * 4608 + (shape.H // 128) * (shape.I // 64) * 4608
    nexp = shape.k + 1
    hbm = peaks["hbm_gbs"]
    roof = None
    if "decode_fused" in prof:
        # one launch per layer: the graph-timed time per layer is the launch's duration (the
        # eager profile below adds the host's launch gaps)
        b = nexp * expert_bytes + shape.E * shape.H * 4 + shape.H * 4 + 2 * shape.H * 2
        a = b / (us_layer * 1e-6) / 1e9
        roof = {"bound": "hbm", "kernel": "decode_fused_kernel (one launch per layer, timed in the graph)",
                "achieved": round(a, 1), "peak": hbm, "unit": "GB/s", "frac": round(a / hbm, 4),
                "traffic": profiled_traffic("decode_fused", "decode_fused_decode_2layers.md", "decode_fused.cu"),
                "bytes_per_token": b, "peak_source": f"{peak_src} hbm_gbs"}
    elif "gemv_gateup" in prof and "gemv_down" in prof:
        b_gu = nexp * (shape.I // 64) * (shape.H // 64) * 4608 + shape.H * 2
        b_dn = nexp * (shape.H // 128) * (shape.I // 64) * 4608 + shape.H * 2
        t = (prof["gemv_gateup"]["avg_us"] + prof["gemv_down"]["avg_us"]) * 1e-6
        a = (b_gu + b_dn) / t / 1e9
        roof = {"bound": "hbm", "kernel": "sparse GEMV gate/up + down (eager, profiled)",
                "achieved": round(a, 1), "peak": hbm, "unit": "GB/s", "frac": round(a / hbm, 4),
                "traffic": None, "bytes_per_token": b_gu + b_dn,
                "peak_source": f"{peak_src} hbm_gbs"}
    layer_bytes = nexp * expert_bytes + shape.E * shape.H * 4 + shape.H * 4 + 2 * shape.H * 2
    for L in layers:
        assert L.status() == 0
        L.close()
    gemv_only = decode_gemv_only(shape, xs, max(args.steps, 20), hbm, peak_src)
    try:   # a measurement beside the decode line: must never cost the line itself
        small = small_batch_decode(shape, max(args.steps, 20), hbm, peak_src)
    except Exception as e:   # noqa: BLE001
        small = {"error": f"{type(e).__name__}: {e}"[:300]}
    return {"metric": DECODE_METRIC,
            "value": round(us_layer, 3), "unit": "us/token/layer", "higher_is_better": False,
            "whole_layer_hbm_frac": round(layer_bytes / (us_layer * 1e-6) / 1e9 / hbm, 4),
            "whole_layer_bytes": layer_bytes, "roofline": roof, "kernels": prof,
            "gemv_kernels_only": gemv_only, "small_batch": small,
            "gpu_launches_per_step": (1 if "decode_fused" in prof else 4) * n_layers}


# ------------------------------------------------------------------------------------ ncu traffic
def kernel_code_hash(main="gemm.cu"):
    """sha256 (16 hex digits) of a kernel's code: csrc/<main>, common.cuh and kernels.h with
    comments and whitespace removed, concatenated (comment edits keep the hash)."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    h = hashlib.sha256()
    for f in (main, "common.cuh", "kernels.h"):
        with open(os.path.join(here, "bit_grouped_expert_router_b200", "csrc", f)) as fh:
            src = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", " ", src).strip().encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, summary="grouped_gemm_prefill16k_zipf_1layer.md", main="gemm.cu"):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu summary, or None when
    the kernel code changed since that capture (the summary records kernel_code_hash())."""
    here = os.path.dirname(os.path.abspath(__file__))
    prof = os.path.join(here, "profiles", summary)
    if not os.path.exists(prof):
        return None
    text = open(prof).read()
    m = re.search(r"kernel_sources_sha256_16: ([0-9a-f]{16})", text)
    t = re.search(r"traffic_bytes_per_launch %s: (\d+)" % re.escape(kernel), text)
    if not m or not t or m.group(1) != kernel_code_hash(main):
        return None
    return int(t.group(1))


# ------------------------------------------------------------------------------------ CPU oracle
def cpu_baseline(host0, x0, shape, target_s):
    import oracle
    ol = oracle.OracleLayer.from_shape(host0, shape)
    # batches of 32 tokens until the target time is spent (or the chunk is used up)
    total_n, t0 = 0, time.perf_counter()
    while total_n < shape.T and time.perf_counter() - t0 < target_s:
        b = min(32, shape.T - total_n)
        ol.forward(x0, tokens=list(range(total_n, total_n + b)))
        total_n += b
    total_t = time.perf_counter() - t0
    return {"value": round(total_n / total_t, 3), "unit": "tokens/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{total_n} tokens of layer 0, chunk 0 through one MoE layer (fp64 oracle, "
                      f"{total_t:.1f} s); per-layer tokens/s comparable to value"}


def prefill_metric(shape, n_layers):
    return (f"MoE-layer prefill tokens/s ({shape.T * shape.chunks}-token prompt in {shape.T}-token chunks, "
            f"{n_layers} layers; also decode us/token/layer)")


DECODE_METRIC = "MoE-layer decode us/token/layer (batch 1, 40 distinct layers, one CUDA graph)"


def prefill_config(args, shape, n_layers):
    return {"workload": args.workload, "tokens": shape.T * shape.chunks, "chunk": shape.T,
            "layers": n_layers, "H": shape.H, "I": shape.I, "E": shape.E, "k": shape.k,
            "shared_expert": shape.has_shared, "zipf_s": shape.zipf_s,
            "weights": "int4 g64 asymmetric, bf16 scale/bias (repacked fp16)",
            "l2": "inputs larger than L2: 457 MB of weights per layer, 40 distinct layers",
            "decode_workload": "decode (T=1, 40 layers, CUDA graph)"}


def run_reference(args, dist):
    """The oracle as the reference arm: rank 0 only, bounded token sample per step."""
    if dist.rank != 0:
        return
    import torch
    import oracle
    from bit_grouped_expert_router_b200 import synth
    shape = synth.WORKLOADS[args.workload]
    w = synth.make_layer(shape, 0)
    x = synth.make_x(shape, 0, 0)
    ol = oracle.OracleLayer.from_shape(w, shape)
    # 32 tokens per step for prefill, as cpu_baseline times them, so the oracle's OpenMP loop over
    # tokens keeps every host core busy and the two CPU figures of one run agree
    per_step = 32 if shape.T > 1 else 1
    t_tok = []
    for i in range(args.warmup + args.steps):
        tok = [(i * per_step + j) % shape.T for j in range(per_step)]
        t0 = time.perf_counter()
        ol.forward(x, tokens=tok)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            t_tok.append(dt)
    ms = 1000.0 * sum(t_tok) / len(t_tok)
    n_layers = args.layers or shape.layers
    if args.workload == "decode":
        value, unit, hib, metric = ms * 1000.0 / per_step, "us/token/layer", False, DECODE_METRIC
        config = {"workload": "decode", "T": 1, "H": shape.H, "I": shape.I, "E": shape.E, "k": shape.k,
                  "layers": n_layers}
    else:
        # per-layer tokens/s: the same unit as the GPU arm's layer-tokens/s
        value, unit, hib, metric = per_step / (ms / 1000.0), "tokens/s", True, prefill_metric(shape, n_layers)
        config = prefill_config(args, shape, n_layers)
    sample = f"{per_step} tokens of layer 0 per step through one MoE layer (fp64 CPU oracle)"
    line = {"impl": "reference", "metric": metric, "value": round(value, 4), "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": hib,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded random-init weights and activations)",
            "config": config,
            "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": oracle.max_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    del torch


def main():
    args = parse_args()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    import torch
    dist.init("nccl")
    torch.cuda.set_device(dist.local)
    peaks, peak_src = load_peaks()
    from bit_grouped_expert_router_b200 import build as B
    B.build()

    line = None
    if args.workload == "decode":
        d = run_decode(args, dist, peaks, peak_src)
        line = {"metric": DECODE_METRIC, "value": d["value"] / dist.world, "unit": d["unit"],
                "higher_is_better": False, "roofline": d["roofline"], "decode_detail": d}
    else:
        r = run_prefill(args, dist, peaks, peak_src)
        shape = r["shape"]
        line = {"metric": prefill_metric(shape, r["n_layers"]),
                "value": round(r["value"], 1), "unit": "tokens/s", "higher_is_better": True,
                "ms_per_step": round(r["ms"], 3), "roofline": r["roofline"], "grouped_gemm": r["grouped_gemm"],
                "kernels": r["kernels"], "gpu_launches": r["launches"], "clocks": r["clocks"]}
        if "e2e" in r:
            line["e2e"] = r["e2e"]
        if dist.world == 1 and dist.rank == 0 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(r["host0"], r["x0"], shape, args.cpu_seconds)
        if not args.no_decode:
            d = run_decode(args, dist, peaks, peak_src)
            line["decode"] = d
        if not args.no_configs and dist.world == 1:
            line["other_configs"] = run_configs(args, dist, peaks, peak_src)
        if args.ablations and dist.world == 1:
            line["ablations"] = run_ablations(args, dist)
        if not args.no_configs and dist.world == 1:
            try:   # a measurement beside the line: must never cost the line itself
                line["expert_parallel"] = run_ep_single(args)
            except Exception as e:   # noqa: BLE001
                line["expert_parallel"] = {"error": f"{type(e).__name__}: {e}"[:300]}
        line["config"] = prefill_config(args, shape, r["n_layers"])
    base = {"n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp16", "data": "synthetic (seeded random-init weights and activations)"}
    for k, v in base.items():
        line.setdefault(k, v)
    line.setdefault("gpu_launches", None)
    if dist.rank == 0:
        print(json.dumps(line, default=str), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
