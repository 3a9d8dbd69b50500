#!/usr/bin/env python
"""Benchmark of the DF-SSM batch-1 decode hot path on B200.

One step = 64 decode tokens (batch 1) through the 48-layer Mamba-2-1.3B-shaped DF-SSM stack (1-bit
scaffold + int8 LoRA in_proj/out_proj, conv shift register, SSM state update), on synthetic seeded
inputs.  The per-step working set (weights ~177 MB + SSM state 96 MiB) is larger than the 126 MB L2,
so no explicit L2 flush is needed between steps.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle on the same workload instead.
Multi-GPU (torchrun): independent replicas, one per GPU ("scaling": "weak"), no data-path collective.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 decode tokens/s (48-layer 1.3B shape); scaffold GEMV % of HBM peak"
N_TOKENS = 64
WORKLOAD = ("DF-SSM Mamba-2-1.3B-shape decode: 48 layers, d_model 2048, d_inner 4096, 64 heads x 64, "
            "d_state 128, batch 1, 64 tokens per step")

# B200 HBM3e nominal bandwidth (GB/s), reported beside the measured copy bandwidth.
NOMINAL_HBM_GBS = 8000.0

# Algorithmic bytes (weights + state read/write) per layer per token at batch 1.
BYTES_IN_PROJ = 8512 * 2048 // 8 + 8512 * 4 + (16 * 2048 + 8512 * 16) + (16 * 4 + 8512 * 4)
BYTES_OUT_PROJ = 2048 * 4096 // 8 + 2048 * 4 + (16 * 4096 + 2048 * 16) + (16 * 4 + 2048 * 4)
BYTES_LAYER = (BYTES_IN_PROJ + BYTES_OUT_PROJ + 4352 * 5 * 4 + 4352 * 3 * 4 * 2
               + 64 * 64 * 128 * 4 * 2 + 64 * 3 * 4 + (2048 + 4096) * 4)
BYTES_TOKEN = 48 * BYTES_LAYER


def peaks_bf16():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ reference arm

class OracleDecode:
    """The CPU oracle running the decode workload's 64-token stream (48 layers, batch 1) from the same
    zero starting state as the GPU arm; each call advances it by whole tokens."""

    def __init__(self):
        import oracle
        from bit_quantized_mamba_b200 import inputs
        self.model = inputs.decode_model(seed=3)
        self.layers = [dict(l, in_proj=oracle.Linear.from_dict(l["in_proj"]),
                            out_proj=oracle.Linear.from_dict(l["out_proj"])) for l in self.model["layers"]]
        self.conv, self.ssm = inputs.zero_states(1, 48)
        self.t = 0

    def run(self, n_tokens: int, budget_s: float | None = None):
        """Decode up to n_tokens next tokens of the stream (stopping after budget_s seconds, at least one
        token); returns (tokens, seconds)."""
        import numpy as np
        import oracle
        done = 0
        t0 = time.perf_counter()
        while done < n_tokens:
            h = np.ascontiguousarray(self.model["emb"][self.t % N_TOKENS])
            for i, ol in enumerate(self.layers):
                oracle.layer_decode(ol, h, self.conv[i], self.ssm[i])
            self.t += 1
            done += 1
            if budget_s is not None and time.perf_counter() - t0 > budget_s:
                break
        return done, time.perf_counter() - t0


def host_cores():
    return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, rank):
    """The reference arm: the CPU oracle on the same 64-token stream from the same zero starting state
    (states carried from step to step as on the GPU), one token per step so that the run stays within a
    few minutes, on all host cores."""
    if rank != 0:
        return
    import oracle
    threads = host_cores()
    oracle.set_threads(threads)
    dec = OracleDecode()
    tokens_per_step = 1
    per = []
    for i in range(args.warmup + args.steps):
        n, dt = dec.run(tokens_per_step)
        if i >= args.warmup:
            per.append(dt / n)
    sec_per_token = sum(per) / len(per)
    value = 1.0 / sec_per_token
    sample = (f"tokens {args.warmup}..{args.warmup + args.steps - 1} of the 64-token stream (tokens "
              f"0..{args.warmup - 1} untimed), one token x 48 layers per step, states carried from zero")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec_per_token * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic", "config": {"workload": WORKLOAD, "batch": 1,
                                        "tokens_per_step": tokens_per_step},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------- our arm

# DRAM traffic of one decode_kernel launch (dram__bytes_read.sum + dram__bytes_write.sum, one ncu capture
# of the fourth launch of `bench.py --ncu --warmup 3`: 280.51 MB + 53.51 MB), valid only for the kernel
# source it was measured on; reported as null once that source changes.
TRAFFIC_MEASURED = {"sha": "57db9d3cbb95", "bytes": 334_023_680}


def src_sha(*names):
    h = hashlib.sha1()
    for n in names:
        with open(os.path.join(ROOT, "bit_quantized_mamba_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    from bit_quantized_mamba_b200 import build, dfssm, inputs, replicas

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if rank == 0 or not build.up_to_date():
        build.build()
    if world > 1:
        dist.barrier()

    def barrier():
        replicas.barrier(world)

    def max_over_ranks(x: float) -> float:
        return replicas.max_over_ranks(x, world, dev)

    # ---- model, states, embeddings (seeded; identical replica on every rank)
    model = inputs.decode_model(seed=3)
    dims = dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1)
    layers = [dfssm.Layer.from_host(l, dev) for l in model["layers"]]
    conv, ssm = inputs.zero_states(1, 48)
    conv_d = [torch.from_numpy(conv[i]).to(dev) for i in range(48)]
    ssm_d = [torch.from_numpy(ssm[i]).to(dev) for i in range(48)]
    stack = dfssm.LayerStack(layers, dims, conv_d, ssm_d)
    emb_host = torch.from_numpy(np.ascontiguousarray(model["emb"].reshape(N_TOKENS, 2048))).pin_memory()
    emb = emb_host.to(dev)
    h = torch.zeros((1, 2048), dtype=torch.float32, device=dev)
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LAYER_DECODE, 1, 2048, 4096), dev)
    stream = torch.cuda.Stream(device=dev)

    if args.ncu:  # launch list / kernel capture: eager tokens, no graph, nothing else
        for t in range(args.warmup + 1):
            h.copy_(emb[t:t + 1])
            dfssm.layer_decode(stack, h, ws)
        torch.cuda.synchronize()
        return

    def decode_step():
        for t in range(N_TOKENS):
            h.copy_(emb[t:t + 1], non_blocking=True)
            dfssm.layer_decode(stack, h, ws, stream=torch.cuda.current_stream())

    # capture one step (64 tokens) into a CUDA graph; run eagerly if capture is refused
    with torch.cuda.stream(stream):
        decode_step()  # untimed warm-up of every kernel before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(graph, stream=stream):
            decode_step()
        torch.cuda.synchronize()
        run_step = graph.replay
        engine_mode = "CUDA graph of 64 per-token launches"
    except Exception as exc:  # noqa: BLE001
        torch.cuda.synchronize()
        graph = None
        engine_mode = f"eager per-token launches (graph capture failed: {type(exc).__name__})"

        def run_step():
            with torch.cuda.stream(stream):
                decode_step()

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    barrier()
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    with torch.cuda.stream(stream):
        start.record()
        for _ in range(args.steps):
            run_step()
        end.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    ms = start.elapsed_time(end)
    ms = max_over_ranks(ms)
    ms_per_step = ms / args.steps
    value = replicas.whole_job_rate(N_TOKENS * args.steps, world, ms / 1e3)

    # ---- end to end through the public API: pinned host embeddings in, final hidden state out
    out_host = torch.empty((1, 2048), dtype=torch.float32).pin_memory()
    e2e_steps = args.steps

    def e2e_step():
        emb.copy_(emb_host, non_blocking=True)
        for t in range(N_TOKENS):
            h.copy_(emb[t:t + 1], non_blocking=True)
            dfssm.layer_decode(stack, h, ws, stream=torch.cuda.current_stream())
        out_host.copy_(h, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(e2e_steps):
            e2e_step()
        e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = replicas.whole_job_rate(N_TOKENS * e2e_steps, world, e2e_ms / 1e3)

    # ---- scaffold GEMV sweep: 48 in_proj / out_proj copies through dfssm_linear_decode, captured in
    # a CUDA graph (48 calls = 96 kernels, PDL-chained); L2 flushed before each timed replay
    hbm, peak_kind = peaks()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    mws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LINEAR_MULTI, 0, 0, 0), dev)
    gemv = {}
    if not args.no_extras:
        for which, data_fn, nbytes in (("in_proj", inputs.in_proj_stack, BYTES_IN_PROJ),
                                       ("out_proj", inputs.out_proj_stack, BYTES_OUT_PROJ)):
            data = data_fn()
            lins = [dfssm.Linear.from_host(l, dev) for l in data["linears"]]
            xd = torch.from_numpy(data["x"]).to(dev)
            for B in (1, 4, 16):
                y = torch.empty((B, lins[0].d_out), dtype=torch.float32, device=dev)
                gws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LINEAR_DECODE, B, lins[0].d_in,
                                                           lins[0].d_out), dev)
                xb = xd[:B].contiguous()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    for L in lins:  # warm every launch configuration before capture
                        dfssm.linear_decode(L, xb, y, gws, stream=torch.cuda.current_stream())
                    torch.cuda.synchronize()
                    with torch.cuda.graph(g, stream=stream):
                        for L in lins:
                            dfssm.linear_decode(L, xb, y, gws, stream=torch.cuda.current_stream())
                tot, reps = 0.0, 10
                with torch.cuda.stream(stream):
                    for r in range(reps + 2):
                        flush.fill_(r & 0xFF)
                        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        a.record()
                        g.replay()
                        b.record()
                        b.synchronize()
                        if r >= 2:
                            tot += a.elapsed_time(b)
                del g
                us_per_call = tot / reps / len(lins) * 1e3
                gbs = nbytes / (us_per_call * 1e-6) / 1e9
                gemv[f"{which}_B{B}"] = {"us_per_call": round(us_per_call, 3), "GB_s": round(gbs, 1),
                                         "frac_of_measured_hbm": round(gbs / hbm, 3)}
                # the same 48 copies in one dfssm_linear_decode_multi launch (shared input x)
                ys = [torch.empty((B, L.d_out), dtype=torch.float32, device=dev) for L in lins]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    dfssm.linear_decode_multi(lins, xb, ys, ws=mws, stream=torch.cuda.current_stream())
                    torch.cuda.synchronize()
                    with torch.cuda.graph(g, stream=stream):
                        dfssm.linear_decode_multi(lins, xb, ys, ws=mws, stream=torch.cuda.current_stream())
                tot, reps = 0.0, 10
                with torch.cuda.stream(stream):
                    for r in range(reps + 2):
                        flush.fill_(r & 0xFF)
                        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        a.record()
                        g.replay()
                        b.record()
                        b.synchronize()
                        if r >= 2:
                            tot += a.elapsed_time(b)
                del g, ys
                us_all = tot / reps * 1e3
                gbs = nbytes * len(lins) / (us_all * 1e-6) / 1e9
                gemv[f"{which}_B{B}_multi"] = {"us_per_48_copies": round(us_all, 3), "GB_s": round(gbs, 1),
                                               "frac_of_measured_hbm": round(gbs / hbm, 3)}
            del lins

    # ---- prefill (2048 tokens) on tcgen05 int8, and the int8 LM head on the last token
    prefill = {}
    if not args.no_extras:
        pdata = inputs.prefill(seed=4, m=2048)
        int8_peak = 2.0 * peaks_bf16()  # int8 dense = 2x bf16 dense (nominal ratio)
        for which, xkey in (("in_proj", "x_in"), ("out_proj", "x_out")):
            L = dfssm.Linear.from_host(pdata[which], dev)
            xin = torch.from_numpy(pdata[xkey]).to(dev)
            M = xin.shape[0]
            yp = torch.empty((M, L.d_out), dtype=torch.float32, device=dev)
            pws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LINEAR_PREFILL, M, L.d_in, L.d_out), dev)
            with torch.cuda.stream(stream):
                for r in range(3):
                    dfssm.linear_prefill(L, xin, yp, pws, stream=torch.cuda.current_stream())
                torch.cuda.synchronize()
                tot, reps = 0.0, 10
                for r in range(reps):
                    flush.fill_(r & 0xFF)
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    dfssm.linear_prefill(L, xin, yp, pws, stream=torch.cuda.current_stream())
                    b.record()
                    b.synchronize()
                    tot += a.elapsed_time(b)
            ms = tot / reps
            tops = 2.0 * M * L.d_out * L.d_in / (ms * 1e-3) / 1e12
            prefill[which] = {"ms_per_call": round(ms, 4), "int8_TOPS": round(tops, 1),
                              "frac_of_int8_peak": round(tops / int8_peak, 3)}
        W = torch.from_numpy(pdata["lm_w"]).to(dev)
        srow = torch.from_numpy(pdata["lm_s"]).to(dev)
        xl = torch.from_numpy(pdata["x_in"][-1].copy()).to(dev)
        logits = torch.empty(W.shape[0], dtype=torch.float32, device=dev)
        lws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LM_HEAD, 1, W.shape[1], W.shape[0]), dev)
        with torch.cuda.stream(stream):
            for r in range(3):
                dfssm.lm_head(W, srow, xl, logits, ws=lws, stream=torch.cuda.current_stream())
            torch.cuda.synchronize()
            tot, reps = 0.0, 10
            for r in range(reps):
                flush.fill_(r & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                dfssm.lm_head(W, srow, xl, logits, ws=lws, stream=torch.cuda.current_stream())
                b.record()
                b.synchronize()
                tot += a.elapsed_time(b)
        ms = tot / reps
        lm_bytes = W.numel() + 4 * W.shape[0]
        prefill["lm_head"] = {"ms_per_call": round(ms, 4),
                              "GB_s": round(lm_bytes / (ms * 1e-3) / 1e9, 1),
                              "frac_of_measured_hbm": round(lm_bytes / (ms * 1e-3) / 1e9 / hbm, 3)}
        prefill["int8_peak_TOPS"] = round(int8_peak, 1)
        prefill["int8_peak_kind"] = "measured bf16 burst x 2 (nominal int8/bf16 ratio)"
        del W
    # ---- layer prefill: a 2048-token prompt through the 48 layers (in_proj GEMM, conv and SSM over the
    # prompt, out_proj GEMM), states continuing from the bench's decode
    prefill_layers = {}
    if not args.no_extras:
        Mp = 2048
        hp0 = torch.from_numpy(inputs.normal(np.random.default_rng(11), (Mp, 2048))).to(dev)
        hp = hp0.clone()
        pws_l = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LAYER_PREFILL, Mp, 2048, 4096), dev)
        with torch.cuda.stream(stream):
            dfssm.layer_prefill(stack, hp, pws_l, stream=torch.cuda.current_stream())
            torch.cuda.synchronize()
            tot = 0.0
            reps = 2
            for r in range(reps):
                hp.copy_(hp0)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                dfssm.layer_prefill(stack, hp, pws_l, stream=torch.cuda.current_stream())
                b.record()
                b.synchronize()
                tot += a.elapsed_time(b)
        pms = tot / reps
        prefill_layers = {"prompt_tokens": Mp, "layers": 48, "ms_per_prompt": round(pms, 3),
                          "tokens_per_s": round(Mp / (pms * 1e-3), 1),
                          "kernels_per_layer": 10}
        del pws_l, hp, hp0

    # ---- greedy generation: embedding + the 48 layers + final RMSNorm / int8 LM head / argmax per token,
    # 64 tokens captured in one CUDA graph (the bench's stack, the tied 50288 x 2048 matrix of seed 5)
    generate = {}
    if not args.no_extras:
        gm = inputs.generation_model(seed=5, n_layers=0)
        GW = torch.from_numpy(gm["emb_w"]).to(dev)
        Gs = torch.from_numpy(gm["emb_s"]).to(dev)
        Gn = torch.from_numpy(gm["final_norm_w"]).to(dev)
        V = GW.shape[0]
        toks = torch.zeros(N_TOKENS + 1, dtype=torch.int32, device=dev)
        toks[0] = gm["first_token"]
        gws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_GENERATE, V, 2048, 4096), dev)
        with torch.cuda.stream(stream):
            dfssm.generate(stack, GW, Gs, Gn, toks, ws=gws, stream=torch.cuda.current_stream())
        torch.cuda.synchronize()
        ggraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ggraph, stream=stream):
            dfssm.generate(stack, GW, Gs, Gn, toks, ws=gws, stream=torch.cuda.current_stream())
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for _ in range(2):
                ggraph.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 3
            a.record()
            for _ in range(reps):
                ggraph.replay()
            b.record()
        torch.cuda.synchronize()
        g_us = a.elapsed_time(b) * 1e3 / (reps * N_TOKENS)
        # the head alone (final norm + LM head + greedy choice), L2 flushed before each call
        hidden = torch.from_numpy(inputs.normal(np.random.default_rng(9), (2048,))).to(dev)
        hws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_HEAD_GREEDY, 1, 2048, V), dev)
        lg = torch.empty(V, dtype=torch.float32, device=dev)
        tk = torch.empty(1, dtype=torch.int32, device=dev)
        with torch.cuda.stream(stream):
            for _ in range(3):
                dfssm.head_greedy(GW, Gs, hidden, Gn, lg, token=tk, ws=hws, stream=torch.cuda.current_stream())
            torch.cuda.synchronize()
            tot = 0.0
            for r in range(10):
                flush.fill_(r & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                dfssm.head_greedy(GW, Gs, hidden, Gn, lg, token=tk, ws=hws, stream=torch.cuda.current_stream())
                b.record()
                b.synchronize()
                tot += a.elapsed_time(b)
        head_us = tot * 1e3 / 10
        head_bytes = GW.numel() + 4 * V + 2 * 4 * 2048
        generate = {"tokens_per_s": round(1e6 / g_us, 1), "us_per_token": round(g_us, 2),
                    "kernels_per_token": 3, "engine": "CUDA graph of 64 dfssm_generate steps",
                    "head_us_per_call": round(head_us, 2),
                    "head_GB_s": round(head_bytes / (head_us * 1e-6) / 1e9, 1),
                    "head_frac_of_measured_hbm": round(head_bytes / (head_us * 1e-6) / 1e9 / hbm, 3),
                    "last_token": int(toks[-1].item())}
        ggraph = None
        del GW
    state_field = measure_state_field(dev, flush, hbm) if not args.no_extras else {}
    del flush
    torch.cuda.synchronize()

    # roofline: the dominant (and only) kernel of the step is the fused decode kernel, one launch per
    # token; its algorithmic bytes are the weights and state a token moves (BYTES_TOKEN).
    us_tok = ms_per_step * 1e3 / N_TOKENS
    achieved = BYTES_TOKEN / (us_tok * 1e-6) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4),
                "frac_of_nominal_8TBs": round(achieved / NOMINAL_HBM_GBS, 4),
                "traffic": (TRAFFIC_MEASURED["bytes"]
                            if src_sha("decode_fused.cu", "common.cuh") == TRAFFIC_MEASURED["sha"] else None),
                "kernel": "dfssm::fused::decode_kernel (one cooperative launch per token, 48 layers)",
                "bytes_per_launch": BYTES_TOKEN, "peak_kind": peak_kind}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1, "tokens_per_step": N_TOKENS,
                   "l2": "inputs larger than L2 (177 MB weights + 96 MiB SSM state per step)",
                   "engine": engine_mode},
        "us_per_token": ms_per_step * 1e3 / N_TOKENS,
        "algorithmic_GB_s": BYTES_TOKEN * N_TOKENS / (ms_per_step * 1e-3) / 1e9,
        "roofline": roofline,
        "scaffold_gemv": gemv,
        "prefill": prefill,
        "prefill_layers": prefill_layers,
        "generate": generate,
        "state_field": state_field,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": N_TOKENS * 2048 * 4,
                "d2h_bytes_per_step": 2048 * 4},
        "gpu_launches": args.steps * N_TOKENS,
        "clocks": clocks,
    }

    # CPU baseline: the oracle on a bounded sample of the same workload (rank 0, N = 1 only), on all host
    # cores and on one
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        cores = host_cores()
        oracle.set_threads(cores)
        n, dt = OracleDecode().run(N_TOKENS, budget_s=args.cpu_budget)
        oracle.set_threads(1)
        n1, dt1 = OracleDecode().run(N_TOKENS, budget_s=args.cpu_budget)
        oracle.set_threads(cores)
        line["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "cpu_model": cpu_model(),
                                "sample": f"first {n} token(s) of the 64-token decode, 48 layers, from the "
                                          f"zero state, on {cores} threads",
                                "single_thread": {"value": n1 / dt1, "unit": "tokens/s", "cores": 1,
                                                  "sample": f"first {n1} token(s), 1 thread"}}
        vnni = vnni_engine_rate(cores)
        if vnni is not None:
            line["cpu_baseline"]["vnni_engine"] = vnni
        line["cpu_baseline"]["state_field_encode"] = field_cpu_times(cores)
    if rank == 0:
        print(json.dumps(line), flush=True)
    graph = None


def vnni_engine_rate(cores, n_tokens=8):
    """The host-CPU engine (libdfssm_cpu, AVX-512 VNNI scaffold GEMV; bit-identical to the oracle) on the
    first tokens of the same 48-layer decode, all host cores; None when the CPU lacks VNNI."""
    import numpy as np
    import torch
    from bit_quantized_mamba_b200 import build, dfssm, inputs
    build.build_cpu()
    if not dfssm.cpu_available():
        return None
    dfssm.cpu_set_threads(cores)
    model = inputs.decode_model(seed=3, n_layers=48, n_tokens=n_tokens)
    conv, ssm = inputs.zero_states(1, 48)
    layers = [dfssm.Layer.from_host(x, "cpu") for x in model["layers"]]
    stack = dfssm.LayerStack(layers, dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1),
                             [torch.from_numpy(conv[i]) for i in range(48)],
                             [torch.from_numpy(ssm[i]) for i in range(48)])
    h = torch.from_numpy(np.array(model["emb"][0], dtype=np.float32))
    dfssm.cpu_layer_decode(stack, h)  # first token: page-in, not timed
    t0 = time.perf_counter()
    for t in range(1, n_tokens):
        h = torch.from_numpy(np.array(model["emb"][t], dtype=np.float32))
        dfssm.cpu_layer_decode(stack, h)
    dt = time.perf_counter() - t0
    return {"value": (n_tokens - 1) / dt, "unit": "tokens/s", "cores": cores, "kind": "vnni_engine",
            "sample": f"tokens 1..{n_tokens - 1} of the 64-token decode, 48 layers, on {cores} threads"}


FIELD_ROWS = 48 * 64 * 64   # the 48-layer Mamba-2-1.3B SSM state at batch 1: 196,608 rows of d_state 128
FIELD_N = 128


def measure_state_field(dev, flush, hbm, reps=10):
    """Density-field encode, readout and in-place round trip of the whole 48-layer SSM state (technical
    summary §2.D), each call timed alone with CUDA events on its stream, L2 flushed before each.
    Algorithmic bytes per row: encode 4N read + N/2 + 4 written; readout N/2 + 4 read + 4N written;
    round trip 4N read + 4N written."""
    import torch
    from bit_quantized_mamba_b200 import dfssm, inputs
    state = torch.from_numpy(inputs.ssm_state_rows(seed=77, rows=FIELD_ROWS, d_state=FIELD_N)).to(dev)
    work = state.clone()
    field = torch.empty((FIELD_ROWS, FIELD_N // 8), dtype=torch.int32, device=dev)
    scale = torch.empty(FIELD_ROWS, dtype=torch.float32, device=dev)
    out = torch.empty_like(state)
    per_row = {"encode": 4 * FIELD_N + FIELD_N // 2 + 4, "decode": 4 * FIELD_N + FIELD_N // 2 + 4,
               "roundtrip": 8 * FIELD_N}
    calls = {"encode": lambda st: dfssm.state_field_encode(state, field, scale, stream=st),
             "decode": lambda st: dfssm.state_field_decode(field, scale, FIELD_N, out, stream=st),
             "roundtrip": lambda st: dfssm.state_field_roundtrip(work, stream=st)}
    res = {"rows": FIELD_ROWS, "d_state": FIELD_N, "bits_per_value": 4,
           "kernels": "dfssm::field_encode_kernel, dfssm::field_decode_kernel (one launch per call)"}
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        st = torch.cuda.current_stream()
        for name, fn in calls.items():
            for _ in range(3):
                work.copy_(state)
                fn(st)
            tot = 0.0
            for r in range(reps):
                work.copy_(state)
                flush.fill_(r & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(st)
                fn(st)
                b.record(st)
                b.synchronize()
                tot += a.elapsed_time(b)
            us = tot * 1e3 / reps
            gbs = per_row[name] * FIELD_ROWS / (us * 1e-6) / 1e9
            res[name] = {"us_per_call": round(us, 2), "GB_s": round(gbs, 1),
                         "frac_of_measured_hbm": round(gbs / hbm, 3),
                         "bytes_per_call": per_row[name] * FIELD_ROWS}
    torch.cuda.synchronize()
    return res


def field_cpu_times(cores):
    """The density-field encode of the same 48-layer state on the host: the oracle (cell-by-cell
    sigma-delta loop) and the host-CPU engine, best of three, all cores."""
    import oracle
    import torch
    from bit_quantized_mamba_b200 import build, dfssm, inputs
    S = inputs.ssm_state_rows(seed=77, rows=FIELD_ROWS, d_state=FIELD_N)

    def best(fn):
        ts = []
        for _ in range(3):
            t0 = time.perf_counter()
            fn()
            ts.append(time.perf_counter() - t0)
        return round(min(ts) * 1e6, 1)

    res = {"rows": FIELD_ROWS, "d_state": FIELD_N, "cores": cores,
           "oracle_us_per_call": best(lambda: oracle.field_encode(S))}
    build.build_cpu()
    if dfssm.cpu_available():
        dfssm.cpu_set_threads(cores)
        St = torch.from_numpy(S)
        res["cpu_engine_us_per_call"] = best(lambda: dfssm.cpu_state_field_encode(St))
    return res


def run_field_only(args):
    """Only the density-field measurement, printed as one JSON object (no decode line)."""
    import torch
    from bit_quantized_mamba_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    hbm, peak_kind = peaks()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    res = measure_state_field(dev, flush, hbm)
    res["peak"], res["peak_kind"] = hbm, peak_kind
    print(json.dumps({"state_field": res}), flush=True)


def run_field_profile(args):
    """Eager density-field encodes of the 48-layer state for an ncu capture (no timing is reported)."""
    import torch
    from bit_quantized_mamba_b200 import build, dfssm, inputs
    build.build()
    dev = torch.device("cuda", 0)
    state = torch.from_numpy(inputs.ssm_state_rows(seed=77, rows=FIELD_ROWS, d_state=FIELD_N)).to(dev)
    field = torch.empty((FIELD_ROWS, FIELD_N // 8), dtype=torch.int32, device=dev)
    scale = torch.empty(FIELD_ROWS, dtype=torch.float32, device=dev)
    out = torch.empty_like(state)
    for _ in range(args.warmup + 1):
        dfssm.state_field_encode(state, field, scale)
        dfssm.state_field_decode(field, scale, FIELD_N, out)
    torch.cuda.synchronize()


def run_prefill_profile(args):
    """Eager prefill calls for an ncu launch list (no timing is reported)."""
    import torch
    from bit_quantized_mamba_b200 import build, dfssm, inputs
    build.build()
    dev = torch.device("cuda", 0)
    p = inputs.prefill(seed=4, m=2048, vocab=16)
    L = dfssm.Linear.from_host(p["in_proj"], dev)
    x = torch.from_numpy(p["x_in"]).to(dev)
    y = torch.empty((x.shape[0], L.d_out), dtype=torch.float32, device=dev)
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LINEAR_PREFILL, x.shape[0], L.d_in, L.d_out), dev)
    for _ in range(args.warmup + 1):
        dfssm.linear_prefill(L, x, y, ws)
    torch.cuda.synchronize()


def run_gemv_profile(args):
    """Eager dfssm_linear_decode_multi calls over the 48 in_proj copies (batch --gemv-batch), for ncu."""
    import torch
    from bit_quantized_mamba_b200 import build, dfssm, inputs
    build.build()
    dev = torch.device("cuda", 0)
    data = inputs.in_proj_stack()
    lins = [dfssm.Linear.from_host(l, dev) for l in data["linears"]]
    B = args.gemv_batch
    x = torch.from_numpy(data["x"][:B].copy()).to(dev)
    ys = [torch.empty((B, L.d_out), dtype=torch.float32, device=dev) for L in lins]
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LINEAR_MULTI, 0, 0, 0), dev)
    for _ in range(args.warmup + 1):
        dfssm.linear_decode_multi(lins, x, ys, ws=ws)
    torch.cuda.synchronize()


def run_layer_prefill_profile(args):
    """Eager 2048-token prompts through one layer of the 1.3B shape (dfssm_layer_prefill), for ncu."""
    import numpy as np
    import torch
    from bit_quantized_mamba_b200 import build, dfssm, inputs
    build.build()
    dev = torch.device("cuda", 0)
    m = inputs.decode_model(seed=3, n_layers=1, n_tokens=1)
    dims = dict(d_model=2048, nheads=64, headdim=64, d_state=128, ngroups=1)
    conv, ssm = inputs.zero_states(1, 1)
    stack = dfssm.LayerStack([dfssm.Layer.from_host(m["layers"][0], dev)], dims,
                             [torch.from_numpy(conv[0]).to(dev)], [torch.from_numpy(ssm[0]).to(dev)])
    h0 = torch.from_numpy(inputs.normal(np.random.default_rng(11), (2048, 2048))).to(dev)
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_LAYER_PREFILL, 2048, 2048, 4096), dev)
    for _ in range(args.warmup + 1):
        h = h0.clone()
        dfssm.layer_prefill(stack, h, ws)
    torch.cuda.synchronize()


def run_head_profile(args):
    """Eager final-norm + LM-head + greedy calls over the 50288 x 2048 tied matrix, for ncu."""
    import numpy as np
    import torch
    from bit_quantized_mamba_b200 import build, dfssm, inputs
    build.build()
    dev = torch.device("cuda", 0)
    gm = inputs.generation_model(seed=5, n_layers=0)
    W = torch.from_numpy(gm["emb_w"]).to(dev)
    s_row = torch.from_numpy(gm["emb_s"]).to(dev)
    nw = torch.from_numpy(gm["final_norm_w"]).to(dev)
    h = torch.from_numpy(inputs.normal(np.random.default_rng(9), (2048,))).to(dev)
    ws = dfssm.workspace(dfssm.workspace_size(dfssm.OP_HEAD_GREEDY, 1, 2048, W.shape[0]), dev)
    for _ in range(args.warmup + 1):
        dfssm.head_greedy(W, s_row, h, nw, ws=ws)
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle decode per CPU-baseline leg (all cores, then one core)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the GEMV sweep, prefill and LM-head measurements")
    ap.add_argument("--ncu-prefill", action="store_true",
                    help="profiling mode: run the 2048-token in_proj prefill --warmup + 1 times and exit")
    ap.add_argument("--ncu-gemv", action="store_true",
                    help="profiling mode: the 48-copy in_proj multi-linear decode --warmup + 1 times and exit")
    ap.add_argument("--gemv-batch", type=int, default=1, choices=[1, 4, 16],
                    help="token count of the --ncu-gemv profiling mode")
    ap.add_argument("--ncu-layer-prefill", action="store_true",
                    help="profiling mode: a 2048-token prompt through one layer --warmup + 1 times and exit")
    ap.add_argument("--ncu-head", action="store_true",
                    help="profiling mode: the final norm + LM head + greedy choice --warmup + 1 times and exit")
    ap.add_argument("--field-only", action="store_true",
                    help="time only the density-field encode / readout / round trip and print them")
    ap.add_argument("--ncu-field", action="store_true",
                    help="profiling mode: density-field encode + readout of the 48-layer state --warmup + 1 "
                         "times and exit")
    ap.add_argument("--ncu", action="store_true",
                    help="profiling mode: decode --warmup tokens then one more token, eagerly, and exit")
    args = ap.parse_args()
    profiling = (args.ncu or args.ncu_gemv or args.ncu_prefill or args.ncu_layer_prefill or args.ncu_head
                 or args.ncu_field)
    if args.warmup < 3 and not profiling:
        args.warmup = 3
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.ncu_prefill:
        run_prefill_profile(args)
        return
    if args.ncu_gemv:
        run_gemv_profile(args)
        return
    if args.ncu_layer_prefill:
        run_layer_prefill_profile(args)
        return
    if args.ncu_head:
        run_head_profile(args)
        return
    if args.ncu_field:
        run_field_profile(args)
        return
    if args.field_only:
        run_field_only(args)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
