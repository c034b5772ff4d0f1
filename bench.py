#!/usr/bin/env python
"""Throughput of the BitLinear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of the "square" workload
(one BitLinear 2048 -> 2048, 4096 tokens per GPU, bf16 X / dY, fp32 latent W):
weight quantisation (absmean + ternary round + 2-bit pack), RMSNorm + int8 activation
quantisation, the int8 x ternary contraction, the straight-through backward (grad
input GEMM, RMSNorm backward, grad weight GEMM), and a 16-token decode GEMV over the
freshly packed weights.  With N > 1 GPUs each rank holds its own 4096 tokens (weak
scaling) and the weight gradient is summed over ranks with an NCCL all-reduce.

Prints one JSON line (rank 0).  Inputs are synthetic and seeded (bit_ternary_qat_b200.synth).
L2 is flushed (a 512 MB write) before every timed step; each step is timed with CUDA
events on the launching stream, the per-rank sum is max-reduced over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

T_TOK, D_IN, D_OUT = 4096, 2048, 2048
DECODE_B = 16
METRIC = "BitLinear fwd+bwd tokens/s & % of TC peak; packed-ternary GEMV HBM GB/s"
WORKLOAD = "square: BitLinear 2048->2048, 4096 tokens/GPU, bf16 X/dY, fp32 W; quant+fwd+bwd+16-token decode GEMV"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-gemv", action="store_true", help="skip the decode-GEMV side measurement")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only-gemv", action="store_true", help="run only the decode-GEMV measurement (profiling)")
    ap.add_argument("--only-mem", action="store_true",
                    help="run each HBM-bound kernel of the step (and the optimizer step) once on 7B-MLP-sized "
                         "inputs larger than L2 (profiling)")
    ap.add_argument("--only-packed", action="store_true",
                    help="run only the packed-weight linear at 16 tokens on the 28672 x 8192 weight (profiling)")
    ap.add_argument("--next", action="store_true",
                    help="time the fused optimizer step and the quantiser variants back to back; one JSON object, "
                         "not the bench line")
    ap.add_argument("--table", action="store_true",
                    help="time every configuration's full step (single, square, mlp7b, layer7b, decode) and the "
                         "oracle on a bounded sample of each; one JSON object, not the bench line")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


# sources of the dominant kernel (the tcgen05 GEMMs): the committed DRAM counters apply
# while these files are unchanged
GEMM_SOURCES = ("gemm_tc.cuh", "common.cuh")


def kernel_src_hash() -> str:
    h = hashlib.sha256()
    cdir = os.path.join(ROOT, "bit_ternary_qat_b200", "csrc")
    for f in GEMM_SOURCES:
        with open(os.path.join(cdir, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str):
    """DRAM bytes per launch of a kernel from the committed ncu summary, if it was taken on
    the current kernel sources; otherwise None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("src_sha") != kernel_src_hash():
            return None
        v = d.get("kernels", {}).get(kernel_key, {}).get("dram_bytes_per_launch")
        return None if v is None else float(v)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.strip().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ------------------------------------------------------------------------------------

def oracle_step(ora, li, t_s: int):
    """The oracle's pass over the hot path on the first t_s tokens (weight quantisation
    over the full W).  Returns seconds."""
    X = li.X[:t_s].float().numpy()
    dY = li.dY[:t_s].float().numpy()
    W = li.W.numpy()
    t0 = time.perf_counter()
    gamma, wq = ora.quant_weight(W)
    packed = ora.pack(wq)
    r = ora.rmsnorm_rinv(X, 1e-6)
    xq, s, xdq = ora.act_quant(X, r, None)
    acc = ora.int_gemm(xq, wq)
    ora.linear_epilogue(acc, gamma, s)
    xdq_b = ora.bf16_bits_to_f32(ora.round_bf16(xdq))
    dxh = ora.grad_input_hat(dY, wq, gamma)
    ora.rmsnorm_backward(X, r, None, dxh)
    ora.grad_weight(dY, xdq_b)
    b = min(DECODE_B, t_s)
    ora.gemv(packed, gamma, W.shape[1], xq[:b], s[:b])
    return time.perf_counter() - t0


def cpu_baseline(target_s: float = 12.0):
    """The oracle on the square workload, repeated until about `target_s` seconds of CPU work."""
    import oracle as ora
    from bit_ternary_qat_b200 import synth
    ora.build()
    li = synth.workload_inputs("square")[0]
    t_s = 64
    dt = oracle_step(ora, li, t_s)
    while dt < target_s / 4 and t_s < T_TOK:
        t_s = min(T_TOK, t_s * 4)
        dt = oracle_step(ora, li, t_s)
    steps, tot = 1, dt
    while tot < target_s:
        tot += oracle_step(ora, li, t_s)
        steps += 1
    return {"value": steps * t_s / tot, "unit": "tokens/s", "cores": ora.num_threads(), "kind": "oracle",
            "sample": f"{steps} oracle step(s) on {t_s} of the {T_TOK} tokens of the square workload "
                      f"(weight quantisation over the full 2048x2048 W included), {tot:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle as ora
    from bit_ternary_qat_b200 import synth
    ora.build()
    li = synth.workload_inputs("square")[0]
    t_s = 256
    for _ in range(args.warmup):
        oracle_step(ora, li, t_s)
    tot = 0.0
    for _ in range(args.steps):
        tot += oracle_step(ora, li, t_s)
    value = t_s * args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "tokens_per_step": t_s},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle", "cores": ora.num_threads(),
                         "sample": f"each step: the oracle on {t_s} of {T_TOK} tokens (full weight quantisation)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------
# the CUDA path
# ------------------------------------------------------------------------------------

def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    import bit_ternary_qat_b200 as bl
    from bit_ternary_qat_b200 import build as blbuild, dp, synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.only_gemv or args.table or args.next or args.only_packed or args.only_mem:
        blbuild.build()
        bl.load()
        flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
        if args.only_mem:
            print(json.dumps({"memory_kernels": mem_once(bl, torch, dev)}), flush=True)
        elif args.only_packed:
            print(json.dumps({"linear_packed": packed_once(bl, torch, dev)}), flush=True)
        elif args.next:
            print(json.dumps({"next": next_measure(bl, torch, dev, flush, peaks())}), flush=True)
        elif args.table:
            print(json.dumps({"table": table_measure(bl, torch, dev, flush, peaks())}), flush=True)
        else:
            print(json.dumps({"decode_gemv": gemv_measure(bl, torch, dev, flush, peaks())}), flush=True)
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    if rank == 0:
        blbuild.build()
    if world > 1:
        dist.barrier()
    bl.load()

    # ---------------------------------------------------------------- inputs (HBM resident)
    wl = synth.WORKLOADS["square"]
    gen = synth.generator(wl.seed)
    W_h = synth.normal((D_OUT, D_IN), synth.W_STD, gen)                  # same W on every rank
    gen_r = synth.generator(wl.seed * 1000 + rank)                       # rank's own tokens
    X_h = synth.normal((T_TOK, D_IN), 1.0, gen_r).to(torch.bfloat16)
    dY_h = synth.normal((T_TOK, D_OUT), synth.DY_STD_BF16, gen_r).to(torch.bfloat16)
    W, X, dY = W_h.to(dev), X_h.to(dev), dY_h.to(dev)

    f32, bf16, i8, u8 = torch.float32, torch.bfloat16, torch.int8, torch.uint8
    bufs = dict(
        gamma=torch.empty(1, dtype=f32, device=dev), wq_i8=torch.empty(D_OUT, D_IN, dtype=i8, device=dev),
        wq_bf16=torch.empty(D_OUT, D_IN, dtype=bf16, device=dev),
        packed=torch.empty(D_OUT, D_IN // 4, dtype=u8, device=dev),
        xq=torch.empty(T_TOK, D_IN, dtype=i8, device=dev), sx=torch.empty(T_TOK, dtype=f32, device=dev),
        rinv=torch.empty(T_TOK, dtype=f32, device=dev), xdq=torch.empty(T_TOK, D_IN, dtype=bf16, device=dev),
        y=torch.empty(T_TOK, D_OUT, dtype=bf16, device=dev), dX=torch.empty(T_TOK, D_IN, dtype=f32, device=dev),
        dW=torch.empty(D_OUT, D_IN, dtype=f32, device=dev), dg=torch.empty(D_IN, dtype=f32, device=dev),
        ydec=torch.empty(DECODE_B, D_OUT, dtype=f32, device=dev),
        ws=bl.workspace(T_TOK, D_OUT, D_IN, dev))
    flush = torch.empty(512 * 1024 * 1024, dtype=u8, device=dev)        # > 126 MB L2

    # names of the timed pieces, in step order (each is one public call)
    PIECES = ["quant_weight", "act_quant", "linear_i8", "grad_input", "rmsnorm_bwd", "grad_weight",
              "allreduce_dW", "decode_gemv"]

    def step(ev=None, inputs=None, dom_ev=None):
        b = bufs
        Wi, Xi, dYi = inputs if inputs is not None else (W, X, dY)
        rec = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        if dom_ev is not None:      # bracket only the dominant kernel (grad-input GEMM)
            rec = (lambda i: dom_ev[i - 3].record() if i in (3, 4) else None)
        rec(0)
        bl.bitlinear_quant_weight(Wi, ws=b["ws"], out=b)
        rec(1)
        bl.bitlinear_act_quant(Xi, apply_rmsnorm=True, out=b)
        rec(2)
        bl.bitlinear_linear(b["xq"], b["sx"], b["wq_i8"], b["gamma"], y=b["y"])
        rec(3)
        bl.bitlinear_grad_input(dYi, b["wq_bf16"], b["gamma"], dXhat=b["dX"])
        rec(4)
        bl.bitlinear_rmsnorm_backward(Xi, b["rinv"], b["dX"], ws=b["ws"], dg=b["dg"])
        rec(5)
        bl.bitlinear_backward_weight(dYi, b["xdq"], dW=b["dW"])
        rec(6)
        dp.allreduce_weight_grad(b["dW"])
        rec(7)
        bl.ternary_gemv(b["packed"], b["gamma"], D_IN, b["xq"][:DECODE_B], b["sx"][:DECODE_B], y=b["ydec"])
        rec(8)

    # The timed step runs the forward as one call (bitlinear_forward_qat: quantisation of W and
    # X, then the GEMM) and the backward pieces; after the grad-input GEMM the RMSNorm
    # backward and the decode GEMV go to a second stream and run beside the weight-gradient
    # GEMM (its persistent CTAs leave room for the RMSNorm blocks).  Measured against other
    # orders (weight quantisation beside activation quantisation as well, the weight-gradient
    # GEMM first): this one is the fastest; the calls before the fork keep their
    # programmatic-dependent-launch overlap.
    ovs = torch.cuda.Stream(device=dev)

    def step_overlap(dom_ev=None, inputs=None, with_tail=True):
        b = bufs
        Wi, Xi, dYi = inputs if inputs is not None else (W, X, dY)
        main = torch.cuda.current_stream(dev)
        # weight + activation quantisation and the forward GEMM in one call
        bl.bitlinear_forward_qat(Xi, Wi, ws=b["ws"], out=b)
        if dom_ev is not None:
            dom_ev[0].record()
        bl.bitlinear_grad_input(dYi, b["wq_bf16"], b["gamma"], dXhat=b["dX"])
        if dom_ev is not None:
            dom_ev[1].record()
        ovs.wait_stream(main)
        with torch.cuda.stream(ovs):
            bl.bitlinear_rmsnorm_backward(Xi, b["rinv"], b["dX"], ws=b["ws"], dg=b["dg"])
            if with_tail:
                bl.ternary_gemv(b["packed"], b["gamma"], D_IN, b["xq"][:DECODE_B], b["sx"][:DECODE_B],
                                y=b["ydec"])
        bl.bitlinear_backward_weight(dYi, b["xdq"], dW=b["dW"])
        if with_tail:
            dp.allreduce_weight_grad(b["dW"])
        main.wait_stream(ovs)

    def sync_all():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
            torch.cuda.synchronize()

    # ---------------------------------------------------------------- warm-up
    for _ in range(max(3, args.warmup)):
        step()
    sync_all()
    assert bl.check_device_status() == 0

    # ---------------------------------------------------------------- CUDA graphs of one step
    # The step is 9 library calls; replaying it as a captured graph removes the Python /
    # ctypes launch overhead from the device timeline.  The timed graph holds the kernels
    # alone (consecutive kernels overlap their launch with the previous kernel's drain); a
    # second graph with event nodes between the calls times every piece, in a separate loop
    # whose time does not enter the step time.
    gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(9)]
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()
        step_overlap(with_tail=(world == 1))
    torch.cuda.current_stream(dev).wait_stream(side)
    sync_all()

    def capture(ev, dom_ev=None):
        if world == 1:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                if ev is None:
                    step_overlap(dom_ev)
                else:
                    step(ev)
            return [g], (lambda: g.replay())
        # the NCCL all-reduce stays outside the graphs
        rec = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        g1, g2 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        b = bufs
        if ev is None:
            with torch.cuda.graph(g1):
                step_overlap(dom_ev, with_tail=False)
            with torch.cuda.graph(g2):
                bl.ternary_gemv(b["packed"], b["gamma"], D_IN, b["xq"][:DECODE_B], b["sx"][:DECODE_B],
                                y=b["ydec"])

            def rp0():
                g1.replay()
                dp.allreduce_weight_grad(bufs["dW"])
                g2.replay()
            return [g1, g2], rp0
        with torch.cuda.graph(g1):
            rec(0)
            bl.bitlinear_quant_weight(W, ws=b["ws"], out=b); rec(1)
            bl.bitlinear_act_quant(X, apply_rmsnorm=True, out=b); rec(2)
            bl.bitlinear_linear(b["xq"], b["sx"], b["wq_i8"], b["gamma"], y=b["y"]); rec(3)
            bl.bitlinear_grad_input(dY, b["wq_bf16"], b["gamma"], dXhat=b["dX"]); rec(4)
            bl.bitlinear_rmsnorm_backward(X, b["rinv"], b["dX"], ws=b["ws"], dg=b["dg"]); rec(5)
            bl.bitlinear_backward_weight(dY, b["xdq"], dW=b["dW"]); rec(6)
        with torch.cuda.graph(g2):
            rec(7)
            bl.ternary_gemv(b["packed"], b["gamma"], D_IN, b["xq"][:DECODE_B], b["sx"][:DECODE_B], y=b["ydec"])
            rec(8)

        def rp():
            g1.replay()
            dp.allreduce_weight_grad(bufs["dW"])
            g2.replay()
        return [g1, g2], rp

    dom_ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    launches_before_capture = bl.launch_count()
    graphs, replay = capture(None)                 # the timed step: kernels only
    kernels_per_step = bl.launch_count() - launches_before_capture
    graphs_dom, replay_dom = capture(None, dom_ev)  # the same step, events around the grad-input GEMM
    graphs_pc, replay_pc = capture(gev)            # sequential, events between all calls
    for _ in range(max(3, args.warmup)):
        replay()
        replay_dom()
        replay_pc()
    sync_all()
    assert bl.check_device_status() == 0

    # ---------------------------------------------------------------- timed region
    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    gpu_uuid = None
    try:
        gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_uuid = str(local)
    clk = ClockSampler(gpu_uuid) if rank == 0 else None
    sync_all()
    if clk:
        clk.start()
        time.sleep(0.3)
    for i in range(K):
        flush.zero_()                       # evict L2 (outside the timed events)
        ev_s[i].record()
        replay()
        ev_e[i].record()
    sync_all()
    # roofline: K more timed steps of the same work with two event nodes around the
    # grad-input GEMM (event nodes cost the step its launch overlap at that point, so they
    # stay out of the steps that give the value)
    dom_ms = []
    for i in range(K):
        flush.zero_()
        replay_dom()
        torch.cuda.synchronize()
        dom_ms.append(dom_ev[0].elapsed_time(dom_ev[1]))
    sync_all()
    clocks = clk.stop() if clk else None
    launches = kernels_per_step * K
    per_step = [a.elapsed_time(b) for a, b in zip(ev_s, ev_e)]
    tot_ms = sum(per_step)
    t = torch.tensor([tot_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    tot_ms = float(t.item())
    # piece breakdown (same step with event nodes between the calls; not part of the value)
    pieces = {p: [] for p in PIECES}
    for i in range(K):
        flush.zero_()
        replay_pc()
        torch.cuda.synchronize()
        for j, p in enumerate(PIECES):
            pieces[p].append(gev[j].elapsed_time(gev[j + 1]))
    sync_all()
    piece_ms = {p: statistics.mean(v) for p, v in pieces.items()}
    # the grad-input GEMM back to back (20 launches per graph, one event pair): its duration
    # without an event node's lost launch overlap, reported beside the roofline
    g_b2b = torch.cuda.CUDAGraph()
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        bl.bitlinear_grad_input(dY, bufs["wq_bf16"], bufs["gamma"], dXhat=bufs["dX"])
    torch.cuda.current_stream(dev).wait_stream(side)
    with torch.cuda.graph(g_b2b):
        for _ in range(20):
            bl.bitlinear_grad_input(dY, bufs["wq_bf16"], bufs["gamma"], dXhat=bufs["dX"])
    g_b2b.replay()
    b2b = []
    for i in range(5):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g_b2b.replay()
        e1.record()
        torch.cuda.synchronize()
        b2b.append(e0.elapsed_time(e1) / 20)
    b2b_ms = statistics.median(b2b)
    assert bl.check_device_status() == 0
    del graphs, graphs_dom, graphs_pc, g_b2b

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        W_p, X_p, dY_p = W_h.pin_memory(), X_h.pin_memory(), dY_h.pin_memory()
        W_d, X_d, dY_d = torch.empty_like(W), torch.empty_like(X), torch.empty_like(dY)
        dW_p = torch.empty(D_OUT, D_IN, dtype=f32).pin_memory()
        g_p = torch.empty(1, dtype=f32).pin_memory()
        h2d = W_p.numel() * 4 + X_p.numel() * 2 + dY_p.numel() * 2
        d2h = dW_p.numel() * 4 + 4
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(2):
            W_d.copy_(W_p, non_blocking=True); X_d.copy_(X_p, non_blocking=True); dY_d.copy_(dY_p, non_blocking=True)
            step_overlap(inputs=(W_d, X_d, dY_d))
            dW_p.copy_(bufs["dW"], non_blocking=True); g_p.copy_(bufs["gamma"], non_blocking=True)
        sync_all()
        for i in range(K):
            flush.zero_()
            es[i][0].record()
            W_d.copy_(W_p, non_blocking=True); X_d.copy_(X_p, non_blocking=True); dY_d.copy_(dY_p, non_blocking=True)
            step_overlap(inputs=(W_d, X_d, dY_d))
            dW_p.copy_(bufs["dW"], non_blocking=True); g_p.copy_(bufs["gamma"], non_blocking=True)
            es[i][1].record()
        sync_all()
        e2e_ms = torch.tensor([sum(a.elapsed_time(b) for a, b in es)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
        e2e = {"value": T_TOK * world * K / (float(e2e_ms.item()) * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    # ---------------------------------------------------------------- decode GEMV (28672 x 8192)
    gemv = None
    if not args.no_gemv and rank == 0:
        gemv = gemv_measure(bl, torch, dev, flush, peaks())

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    # ---------------------------------------------------------------- roofline of the dominant kernel
    pk = peaks()
    gemm_flops = 2.0 * T_TOK * D_OUT * D_IN
    gemm_pieces = {"linear_i8": "int8", "grad_input": "bf16", "grad_weight": "bf16"}
    # the grad-input GEMM, timed by the two event nodes around it inside the timed graph
    dom = "grad_input"
    dom_ms = statistics.mean(dom_ms)
    achieved = gemm_flops / (dom_ms * 1e-3) / 1e12
    if gemm_pieces[dom] == "bf16":
        peak, peak_note = pk["bf16_sust"], f"bf16 sustained ({pk['src']})"
    else:
        peak, peak_note = 2.0 * pk["bf16_sust"], f"int8 = 2 x bf16 sustained ({pk['src']}; nominal 4.5/2.25 ratio)"
    kernel_names = {"linear_i8": "tc_gemm2_kernel<int8,K,K,linear> (2-SM, 256x256)",
                    "grad_input": "tc_gemm2_kernel<bf16,K,MN,scale_f32> (2-SM, 256x256)",
                    "grad_weight": "tc_gemm2_kernel<bf16,MN,MN,f32> (2-SM, 256x256)"}
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": ncu_traffic(dom), "kernel": kernel_names[dom], "peak_kind": peak_note,
                "launch_ms": dom_ms,
                "back_to_back": {"launch_ms": b2b_ms, "achieved": gemm_flops / (b2b_ms * 1e-3) / 1e12,
                                 "frac": gemm_flops / (b2b_ms * 1e-3) / 1e12 / peak,
                                 "how": "20 launches of the GEMM in one CUDA graph, one event pair, median of 5"}}

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline()

    value = T_TOK * world * K / (tot_ms * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": tot_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "s8+bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_gpu": T_TOK, "d_in": D_IN, "d_out": D_OUT,
                   "decode_batch": DECODE_B, "parallelism": f"dp{world}",
                   "l2": "flushed before every timed step (512 MB write)"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "timing": ("each step replays a CUDA graph of the step's library calls (RMSNorm backward and decode "
                   "GEMV on a second stream beside the weight-gradient GEMM) with no event node inside; the "
                   "roofline's grad-input GEMM time comes from K further timed steps of the same graph with "
                   "two event nodes around that GEMM, and pieces_ms from a sequential graph with events "
                   "between all calls; gpu_launches = kernels per step x steps"),
        "clocks": clocks,
        "pieces_ms": {k: round(v, 5) for k, v in piece_ms.items()},
        "gemm_tflops": {p: gemm_flops / (piece_ms[p] * 1e-3) / 1e12 for p in gemm_pieces},
        "decode_gemv": gemv,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def gemv_measure(bl, torch, dev, flush, pk):
    """Decode GEMV on the 28672 x 8192 packed weight at batch 1, 4, 16.

    Four copies of the packed weight (235 MB, above the 126 MB L2) are cycled, so every launch
    reads a matrix that 176 MB of other weights have passed through L2 since its last use;
    `reps` back-to-back launches, captured in one CUDA graph, sit between one pair of CUDA
    events, so the per-launch time carries neither the event floor of a lone launch nor the
    host's per-call cost.
    """
    from bit_ternary_qat_b200 import synth
    N, K = 28672, 8192
    copies = 4
    W, _ = synth.decode_inputs(1, N, K)
    q = bl.bitlinear_quant_weight(W.to(dev), want_i8=False, want_bf16=False)
    del W
    packs = [q["packed"]] + [q["packed"].clone() for _ in range(copies - 1)]
    out = {}
    reps = 40
    for B in (1, 4, 16):
        _, x = synth.decode_inputs(B, 16, K, seed=40 + B)
        aq = bl.bitlinear_act_quant(x.to(dev), apply_rmsnorm=False, want_xdq=False)
        y = torch.empty(B, N, dtype=torch.float32, device=dev)
        for i in range(2 * copies):
            bl.ternary_gemv(packs[i % copies], q["gamma"], K, aq["xq"], aq["sx"], y=y)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(reps):
                bl.ternary_gemv(packs[i % copies], q["gamma"], K, aq["xq"], aq["sx"], y=y)
        graph.replay()
        samples = []
        for _ in range(5):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            torch.cuda.synchronize()
            samples.append(a.elapsed_time(b) / reps)
        del graph
        ms = statistics.median(samples)
        nbytes = N * K // 4 + B * K + 4 * B + 4 * B * N + 4
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[f"B{B}"] = {"us": ms * 1e3, "GB/s": gbs, "frac_hbm": gbs / pk["hbm"],
                        "int_ops_T": 2.0 * B * N * K / (ms * 1e-3) / 1e12}
    out["hbm_peak_GBs"] = pk["hbm"]
    out["workload"] = ("decode: packed W 28672x8192 (58.7 MB), int8 x [B x 8192]; 4 weight copies cycled "
                       "(inputs larger than L2), 40 launches in one CUDA graph per event pair, median of 5")
    return out


def mem_once(bl, torch, dev):
    """One call each of the activation quantiser (8192 x 11008 bf16, RMSNorm fused), the weight
    quantiser (11008 x 4096 fp32), the RMSNorm backward (8192 x 11008) and the optimizer step
    with re-quantisation (11008 x 4096): every input is larger than L2 (a small case for a
    profiler capture; about 2 GB on the device)."""
    from bit_ternary_qat_b200 import synth
    gen = synth.generator(5)
    T, K, N = 8192, 11008, 4096
    X = synth.normal((T, K), 1.0, gen).to(torch.bfloat16).to(dev)
    a = bl.bitlinear_act_quant(X)
    dX = synth.normal((T, K), 1e-2, gen).to(dev)
    ws = bl.workspace(T, N, K, dev)
    bl.bitlinear_rmsnorm_backward(X, a["rinv"], dX, ws=ws, dg=torch.empty(K, device=dev))
    del X, dX, a
    W = synth.normal((K, N), 0.02, gen).to(dev)
    q = bl.bitlinear_quant_weight(W, ws=ws)
    dW = synth.normal((K, N), 1e-3, gen).to(dev)
    m, v = torch.zeros_like(W), torch.zeros_like(W)
    step = torch.zeros(1, dtype=torch.int32, device=dev)
    bl.bitlinear_optimizer_step(W, dW, m, v, step, requantize=True, ws=ws, out=q)
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    return {"act_quant": f"{T}x{K} bf16", "rmsnorm_backward": f"{T}x{K}", "quant_weight": f"{K}x{N}",
            "optimizer_step": f"{K}x{N} with re-quantisation"}


def packed_once(bl, torch, dev):
    """Three launches of the packed-weight linear, 16 tokens x the 28672 x 8192 decode weight
    (a small case for a profiler capture); returns the last launch's event time."""
    from bit_ternary_qat_b200 import synth
    N, K, T = 28672, 8192, 16
    W, _ = synth.decode_inputs(1, N, K)
    q = bl.bitlinear_quant_weight(W.to(dev), want_i8=False, want_bf16=False)
    del W
    xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, device=dev, generator=torch.Generator(dev).manual_seed(1))
    sx = torch.full((T,), 50.0, device=dev)
    y = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(8 * T * N * 4, dtype=torch.uint8, device=dev)
    ms = 0.0
    for _ in range(3):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        bl.bitlinear_linear_packed(xq, sx, q["packed"], q["gamma"], K, y=y, ws=ws)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
    assert bl.check_device_status() == 0
    return {"us_last": ms * 1e3, "shape": f"T={T} K={K} N={N}"}


def next_measure(bl, torch, dev, flush, pk):
    """The fused optimizer step and the quantiser variants, each launched `reps` times back to
    back in one CUDA graph between one pair of CUDA events (median of 5, L2 flushed before each
    replay).  Every input set is larger than the 126 MB L2 or cycled over copies that are.
    Bytes are algorithmic: each tensor read once and each output written once."""
    from bit_ternary_qat_b200 import synth
    out = {}

    def timed(calls, reps):
        for c in calls:
            c()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(reps):
                calls[i % len(calls)]()
        graph.replay()
        torch.cuda.synchronize()
        samples = []
        for _ in range(5):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            torch.cuda.synchronize()
            samples.append(a.elapsed_time(b) / reps)
        del graph
        assert bl.check_device_status() == 0
        return statistics.median(samples) * 1e3

    def hbm_row(us, nbytes, note):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us": us, "GB/s": gbs, "frac_hbm": gbs / pk["hbm"], "bytes": nbytes, "note": note}

    gen = synth.generator(77)
    # optimizer step: 7B-MLP-shaped weight (4 x 180 MB of fp32 state), and the square weight
    # cycled over 4 copies (4 x 67 MB)
    for name, (N, K), copies in (("optimizer_11008x4096", (11008, 4096), 1), ("optimizer_2048x2048", (2048, 2048), 4)):
        n = N * K
        sets = []
        for _ in range(copies):
            W = synth.normal((N, K), 0.3, gen).clamp_(-1, 1).to(dev)
            sets.append(dict(W=W, dW=synth.normal((N, K), 1e-3, gen).to(dev), m=torch.zeros_like(W),
                             v=torch.zeros_like(W), step=torch.zeros(1, dtype=torch.int32, device=dev),
                             q=dict(gamma=torch.empty(1, dtype=torch.float32, device=dev),
                                    wq_i8=torch.empty(N, K, dtype=torch.int8, device=dev),
                                    wq_bf16=torch.empty(N, K, dtype=torch.bfloat16, device=dev),
                                    packed=torch.empty(N, K // 4, dtype=torch.uint8, device=dev))))
        ws = bl.workspace(1, N, K, dev)
        for requant in (True, False):
            calls = [(lambda S=S, rq=requant: bl.bitlinear_optimizer_step(
                S["W"], S["dW"], S["m"], S["v"], S["step"], requantize=rq, ws=ws, out=S["q"] if rq else None))
                for S in sets]
            us = timed(calls, 8)
            per = 31.25 if requant else 28.0
            out[name + ("_requantize" if requant else "")] = hbm_row(
                us, n * per, f"reads dW, W, m, v; writes W, m, v{', int8 + bf16 + 2-bit codes' if requant else ''} "
                             f"({per} B per weight); {copies} state cop{'ies' if copies > 1 else 'y'}")
        del sets, ws
        torch.cuda.empty_cache()

    # weight quantisers on the 11008 x 4096 fp32 weight (180 MB): default, per-row, tau = 0.7
    N, K = 11008, 4096
    W = synth.student_t3((N, K), 0.02, gen).to(dev)
    ws = bl.workspace(1, N, K, dev)
    q = dict(gamma=torch.empty(1, dtype=torch.float32, device=dev),
             wq_i8=torch.empty(N, K, dtype=torch.int8, device=dev),
             wq_bf16=torch.empty(N, K, dtype=torch.bfloat16, device=dev),
             packed=torch.empty(N, K // 4, dtype=torch.uint8, device=dev))
    qr = dict(q, gamma_rows=torch.empty(N, dtype=torch.float32, device=dev))
    nb = N * K * 7.25
    out["quant_weight_11008x4096"] = hbm_row(timed([lambda: bl.bitlinear_quant_weight(W, ws=ws, out=q)], 8), nb,
                                             "per-tensor gamma (two launches)")
    out["quant_weight_rows_11008x4096"] = hbm_row(timed([lambda: bl.bitlinear_quant_weight_rows(W, out=qr)], 8), nb,
                                                  "per-row gamma (one launch)")
    out["quant_weight_tau_11008x4096"] = hbm_row(
        timed([lambda: bl.bitlinear_quant_weight_tau(W, 0.7, ws=ws, out=q)], 8), nb, "tau = 0.7 gamma (two launches)")
    wq_i8 = q["wq_i8"]
    del W
    # activation quantisers on X [8192 x 11008] bf16 (180 MB), RMSNorm fused, X_dq written
    T = 8192
    X = synth.normal((T, 11008), 1.0, gen).to(torch.bfloat16).to(dev)
    a = dict(xq=torch.empty(T, 11008, dtype=torch.int8, device=dev), sx=torch.empty(T, device=dev),
             rinv=torch.empty(T, device=dev), xdq=torch.empty(T, 11008, dtype=torch.bfloat16, device=dev))
    wsa = bl.workspace(T, 16, 11008, dev)
    nb = T * 11008 * 5 + T * 8
    out["act_quant_8192x11008"] = hbm_row(timed([lambda: bl.bitlinear_act_quant(X, out=a)], 8), nb,
                                          "per-token scale (one launch)")
    out["act_quant_tensor_8192x11008"] = hbm_row(
        timed([lambda: bl.bitlinear_act_quant_tensor(X, ws=wsa, out=a)], 8), nb,
        "per-tensor scale (two launches; X read twice)")
    del X, a
    # int8 GEMM with the per-tensor and the per-row epilogue: 8192 tokens, 4096 -> 11008
    xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, device=dev)
    sx = torch.full((T,), 50.0, device=dev)
    gr = torch.rand(N, device=dev) * 0.02 + 0.01
    y = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
    ops = 2.0 * T * N * K
    us_t = timed([lambda: bl.bitlinear_linear(xq, sx, wq_i8, q["gamma"], y=y)], 10)
    us_r = timed([lambda: bl.bitlinear_linear_rows(xq, sx, wq_i8, gr, y=y)], 10)
    out["linear_8192x4096x11008"] = {"us": us_t, "TOPS": ops / (us_t * 1e-6) / 1e12, "note": "gamma / s_t epilogue"}
    out["linear_rows_8192x4096x11008"] = {"us": us_r, "TOPS": ops / (us_r * 1e-6) / 1e12,
                                          "note": "fl(gamma_n / s_t) per element epilogue"}
    del xq, y
    # packed-weight tensor-core linear vs the int8-code linear and the decode GEMV, few tokens
    for (T, N, K) in ((16, 28672, 8192), (64, 11008, 4096), (256, 11008, 4096)):
        Wd = synth.normal((N, K), 0.02, gen).to(dev)
        qd = bl.bitlinear_quant_weight(Wd)
        del Wd
        # weight copies cycled so that each operand's copies together exceed 3 x L2
        c8 = max(1, int(-(-3 * 128 * 2 ** 20 // (N * K))))
        cp = max(1, int(-(-3 * 128 * 2 ** 20 // (N * K // 4))))
        i8s = [qd["wq_i8"]] + [qd["wq_i8"].clone() for _ in range(c8 - 1)]
        pks = [qd["packed"]] + [qd["packed"].clone() for _ in range(cp - 1)]
        xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, device=dev)
        sx = torch.full((T,), 50.0, device=dev)
        y = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
        ws_p = torch.empty(8 * T * N * 4, dtype=torch.uint8, device=dev)
        us_p = timed([lambda i=i: bl.bitlinear_linear_packed(xq, sx, pks[i], qd["gamma"], K, y=y, ws=ws_p)
                      for i in range(cp)], 2 * cp)
        us_8 = timed([lambda i=i: bl.bitlinear_linear(xq, sx, i8s[i], qd["gamma"], y=y) for i in range(c8)], 2 * c8)
        row = {"packed_us": us_p, "int8_us": us_8,
               "packed_weight_GBs": N * K / 4 / (us_p * 1e-6) / 1e9,
               "packed_frac_hbm": (N * K / 4 + T * K + 2 * T * N) / (us_p * 1e-6) / 1e9 / pk["hbm"],
               "int8_frac_hbm": (N * K + T * K + 2 * T * N) / (us_8 * 1e-6) / 1e9 / pk["hbm"],
               "weight_copies": {"int8": c8, "packed": cp}}
        if T <= 16:
            y32 = torch.empty(T, N, dtype=torch.float32, device=dev)
            row["gemv_us"] = timed([lambda i=i: bl.ternary_gemv(pks[i], qd["gamma"], K, xq, sx, y=y32)
                                    for i in range(cp)], 2 * cp)
        out[f"linear_packed_T{T}_{K}x{N}"] = row
        del i8s, pks, qd, xq, y, ws_p
        torch.cuda.empty_cache()
    out["hbm_peak_GBs"] = pk["hbm"]
    return out


def table_measure(bl, torch, dev, flush, pk, steps: int = 5):
    """Every configuration's step -- for each of its layers: weight quantisation, activation
    quantisation, forward GEMM, grad-input GEMM, RMSNorm backward, weight-gradient GEMM --
    captured in one CUDA graph and timed with CUDA events after an L2 flush (median of
    `steps`); tokens/s = T / step time.  Plus the oracle on a bounded token sample of each
    layer (full weight quantisation), extrapolated linearly in tokens."""
    import oracle as ora
    from bit_ternary_qat_b200 import synth
    ora.build()
    out = {}
    for name in ("single", "square", "mlp7b", "layer7b"):
        wl = synth.WORKLOADS[name]
        lis = synth.workload_inputs(name)
        T = lis[0].X.shape[0]
        dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
        maxK = max(li.X.shape[1] for li in lis)
        maxN = max(li.W.shape[0] for li in lis)
        ws = bl.workspace(T, maxN, maxK, dev)
        dev_layers = []
        for li in lis:
            N, K = li.W.shape
            dev_layers.append(dict(
                W=li.W.to(dev), X=li.X.to(dev), dY=li.dY.to(dev), N=N, K=K,
                q=dict(gamma=torch.empty(1, dtype=torch.float32, device=dev),
                       wq_i8=torch.empty(N, K, dtype=torch.int8, device=dev),
                       wq_bf16=torch.empty(N, K, dtype=torch.bfloat16, device=dev),
                       packed=torch.empty(N, K // 4, dtype=torch.uint8, device=dev))))
        shared = dict(xq=torch.empty(T * maxK, dtype=torch.int8, device=dev),
                      xdq=torch.empty(T * maxK, dtype=dt, device=dev),
                      sx=torch.empty(T, dtype=torch.float32, device=dev),
                      rinv=torch.empty(T, dtype=torch.float32, device=dev),
                      y=torch.empty(T * maxN, dtype=dt, device=dev),
                      dX=torch.empty(T * maxK, dtype=torch.float32, device=dev),
                      dW=torch.empty(maxN * maxK, dtype=torch.float32, device=dev),
                      dg=torch.empty(maxK, dtype=torch.float32, device=dev))

        def step():
            for L in dev_layers:
                N, K = L["N"], L["K"]
                a = dict(xq=shared["xq"][:T * K].view(T, K), xdq=shared["xdq"][:T * K].view(T, K),
                         sx=shared["sx"], rinv=shared["rinv"])
                bl.bitlinear_quant_weight(L["W"], ws=ws, out=L["q"])
                bl.bitlinear_act_quant(L["X"], apply_rmsnorm=True, out=a)
                bl.bitlinear_linear(a["xq"], a["sx"], L["q"]["wq_i8"], L["q"]["gamma"],
                                    out_dtype=dt, y=shared["y"][:T * N].view(T, N))
                dX = shared["dX"][:T * K].view(T, K)
                bl.bitlinear_grad_input(L["dY"], L["q"]["wq_bf16"], L["q"]["gamma"], dXhat=dX)
                bl.bitlinear_rmsnorm_backward(L["X"], a["rinv"], dX, ws=ws, dg=shared["dg"][:K])
                bl.bitlinear_backward_weight(L["dY"], a["xdq"], dW=shared["dW"][:N * K].view(N, K))

        for _ in range(2):
            step()
        torch.cuda.synchronize()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        ms = []
        for _ in range(steps):
            flush.zero_()
            a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_ev.record()
            graph.replay()
            b_ev.record()
            torch.cuda.synchronize()
            ms.append(a_ev.elapsed_time(b_ev))
        del graph
        assert bl.check_device_status() == 0
        t = statistics.median(ms)
        ops_fwd = sum(2.0 * T * L["N"] * L["K"] for L in dev_layers)
        # oracle: bounded token sample per layer, extrapolated linearly in tokens
        t_s = min(T, 64 if T <= 4096 else 16)
        cpu_s = 0.0
        for li in lis:
            full = oracle_step(ora, li, t_s)
            wq_only = oracle_weight_quant_s(ora, li)
            cpu_s += wq_only + (full - wq_only) * (T / t_s)
        out[name] = {"tokens": T, "layers": [f"{L['K']}->{L['N']}" for L in dev_layers], "dtype": wl.dtype,
                     "ms_per_step": t, "tokens_per_s": T / (t * 1e-3),
                     "step_tops_all_gemms": 3 * ops_fwd / (t * 1e-3) / 1e12,
                     "oracle": {"tokens_per_s": T / cpu_s, "cores": ora.num_threads(),
                                "sample": f"{t_s} of {T} tokens per layer, full weight quantisation, "
                                          f"extrapolated linearly in tokens" if t_s < T else "full step"}}
        print(json.dumps({name: out[name]}), flush=True)
        del dev_layers, shared, ws
        torch.cuda.empty_cache()
    out["decode"] = gemv_measure(bl, torch, dev, flush, pk)
    # oracle decode GEMV at batch 1 on the packed 28672 x 8192 weight (quantisation not timed)
    W, x = synth.decode_inputs(1)
    gamma, wq = ora.quant_weight(W.numpy())
    packed = ora.pack(wq)
    xq, s_b, _ = ora.act_quant(x.numpy(), None, None)
    t0 = time.perf_counter()
    ora.gemv(packed, gamma, 8192, xq, s_b)
    dt_s = time.perf_counter() - t0
    out["decode"]["oracle_B1"] = {"us": dt_s * 1e6, "GB/s": (28672 * 8192 // 4) / dt_s / 1e9,
                                  "cores": ora.num_threads()}
    return out


def oracle_weight_quant_s(ora, li) -> float:
    W = li.W.numpy()
    t0 = time.perf_counter()
    gamma, wq = ora.quant_weight(W)
    ora.pack(wq)
    return time.perf_counter() - t0


if __name__ == "__main__":
    main()
