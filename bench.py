#!/usr/bin/env python
"""Throughput of the BitLinear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path over the seven projections of a 7B-shaped
transformer layer (q, k, v, o 4096 -> 4096; gate, up 4096 -> 11008; down 11008 -> 4096),
16384 tokens per GPU, bf16 X / dY, fp32 latent W.  For every projection: weight
quantisation (absmean + ternary round + 2-bit pack), RMSNorm + int8 activation
quantisation, the int8 x ternary contraction, the straight-through backward (grad-input
GEMM, RMSNorm backward, weight-gradient GEMM) and a 16-token decode GEMV over the freshly
packed codes.  With N > 1 GPUs each rank holds its own 16384 tokens (weak scaling) and each
projection's weight gradient is summed over ranks with an NCCL all-reduce that overlaps
the next projection's work.

Prints one JSON line (rank 0).  Inputs are synthetic and seeded (bit_ternary_qat_b200.synth;
rank 0 draws exactly the parity tests' layer7b inputs).  L2 is flushed (a 512 MB write)
before every timed step; each step is timed with CUDA events on the launching stream and
the sum over steps is max-reduced over ranks.  The roofline denominators are the measured
peaks of MEASURED_PEAKS.json (HBM copy, cuBLAS bf16 burst) and, for int8, the library's own
tcgen05 kind::i8 peak loop timed at the start of the run.
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

WORKLOAD_NAME = "layer7b"
T_TOK = 16384
DECODE_B = 16
METRIC = "BitLinear fwd+bwd tokens/s & % of TC peak; packed-ternary GEMV HBM GB/s"
WORKLOAD = ("layer7b: the 7 projections of a 7B-shaped layer (q,k,v,o 4096->4096; gate,up 4096->11008; "
            "down 11008->4096), 16384 tokens/GPU, bf16 X/dY, fp32 W; per projection quant+fwd+bwd and a "
            "16-token decode GEMV")
PIECES = ["quant_weight", "act_quant", "linear_i8", "grad_input", "rmsnorm_bwd", "grad_weight", "decode_gemv"]
CPU_SAMPLE_TOKENS = 16


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="skip the decode-GEMV and other-configuration records")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only-gemv", action="store_true", help="run only the decode-GEMV measurement (profiling)")
    ap.add_argument("--only-mem", action="store_true",
                    help="run each HBM-bound kernel of the step (and the optimizer step) once on 7B-MLP-sized "
                         "inputs larger than L2 (profiling)")
    ap.add_argument("--only-packed", action="store_true",
                    help="run three launches of the packed-weight linear only (profiling); see --packed-case")
    ap.add_argument("--packed-case", default="16,28672,8192",
                    help="tokens,d_out,d_in of --only-packed (default: 16 tokens on the 28672 x 8192 weight)")
    ap.add_argument("--only-gemm", choices=["linear_i8", "grad_input", "grad_weight"], default=None,
                    help="run three launches of one GEMM of the step at 16384 tokens (profiling)")
    ap.add_argument("--gemm-shape", choices=["q", "gate", "down"], default="gate",
                    help="projection shape for --only-gemm: q 4096->4096, gate 4096->11008, down 11008->4096")
    ap.add_argument("--only-peak", action="store_true", help="run only the tensor-pipe peak probe")
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
    """DRAM bytes per launch of a kernel of the step, from the committed ncu summary, if it
    was taken on the current kernel sources; otherwise None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("src_sha") != kernel_src_hash() or d.get("workload") != WORKLOAD_NAME:
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
        sm, smax, power, reasons = [], [], [], set()
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
            try:
                power.append(float(parts[3]))
            except ValueError:
                pass
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
               "samples": len(sm)}
        if power:
            out["power_w_max"] = max(power)
        return out


def gpu_id_of(torch, dev) -> str:
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(dev.index or 0)


# ------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ------------------------------------------------------------------------------------

def oracle_step(ora, li, t_s: int):
    """The oracle's pass over the hot path on the first t_s tokens of one layer (weight
    quantisation over the full W).  Returns (seconds, seconds of the weight quantisation)."""
    X = li.X[:t_s].float().numpy()
    dY = li.dY[:t_s].float().numpy()
    W = li.W.numpy()
    t0 = time.perf_counter()
    gamma, wq = ora.quant_weight(W)
    packed = ora.pack(wq)
    t_wq = time.perf_counter() - t0
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
    return time.perf_counter() - t0, t_wq


def oracle_workload_step(ora, lis, t_s: int):
    """One oracle step over every layer of the workload on a t_s-token sample.  Returns
    (measured seconds, seconds extrapolated to the full token count): per layer, the weight
    quantisation once plus the token-proportional rest scaled by T / t_s."""
    meas, extra = 0.0, 0.0
    for li in lis:
        T = li.X.shape[0]
        full, wq = oracle_step(ora, li, t_s)
        meas += full
        extra += wq + (full - wq) * (T / t_s)
    return meas, extra


def cpu_baseline(target_s: float = 12.0):
    """The oracle on the layer7b workload, 16 tokens per projection per step (full weight
    quantisation), repeated until about `target_s` seconds of CPU work, extrapolated to
    16384 tokens."""
    import oracle as ora
    from bit_ternary_qat_b200 import synth
    ora.build()
    lis = synth.workload_inputs(WORKLOAD_NAME)
    steps, meas, extra = 0, 0.0, 0.0
    while meas < target_s:
        m, e = oracle_workload_step(ora, lis, CPU_SAMPLE_TOKENS)
        meas += m
        extra += e
        steps += 1
    return {"value": T_TOK * steps / extra, "unit": "tokens/s", "cores": ora.num_threads(), "kind": "oracle",
            "sample": f"{steps} oracle step(s), each: every projection's full weight quantisation and "
                      f"{CPU_SAMPLE_TOKENS} of its {T_TOK} tokens (fwd + bwd + decode GEMV), {meas:.1f} s measured; "
                      f"tokens/s extrapolated linearly in tokens (weight quantisation once per projection)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle as ora
    from bit_ternary_qat_b200 import synth
    ora.build()
    lis = synth.workload_inputs(WORKLOAD_NAME)
    for _ in range(args.warmup):
        oracle_workload_step(ora, lis, CPU_SAMPLE_TOKENS)
    meas, extra = 0.0, 0.0
    for _ in range(args.steps):
        m, e = oracle_workload_step(ora, lis, CPU_SAMPLE_TOKENS)
        meas += m
        extra += e
    value = T_TOK * args.steps / extra
    sample = (f"each step: every projection's full weight quantisation and {CPU_SAMPLE_TOKENS} of its {T_TOK} "
              f"tokens (fwd + bwd + decode GEMV), {meas / args.steps:.2f} s measured per step; tokens/s "
              f"extrapolated linearly in tokens (weight quantisation once per projection)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * extra / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "tokens_per_gpu": T_TOK,
                                        "sampled_tokens_per_step": CPU_SAMPLE_TOKENS},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle", "cores": ora.num_threads(),
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------
# tensor-pipe peak (the library's own tcgen05 loop; denominator of the int8 GEMMs)
# ------------------------------------------------------------------------------------

def probe_tensor_peaks(bl, torch, dev, iters: int = 20000, reps: int = 5):
    """Each of kind::i8 / kind::f16 x cta_group::1 / ::2: one short warm-up launch, then `reps`
    timed launches (about 5 ms each); the best rate of each is its burst peak in TFLOP/s (or
    TOPS for int8)."""
    out = {}
    for kind in ("int8", "bf16"):
        for pair in (False, True):
            bl.mma_peak_probe(kind, pair, max(1, iters // 4))
            torch.cuda.synchronize()
            rates = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                ops = bl.mma_peak_probe(kind, pair, iters)
                b.record()
                torch.cuda.synchronize()
                rates.append(ops / (a.elapsed_time(b) * 1e-3) / 1e12)
            out[f"{kind}_{'cta_pair' if pair else 'cta'}"] = max(rates)
    # the warp-level IMMA of the decode GEMV (mma.sync m16n8k32 int8)
    bl.mma_peak_probe("imma_sync", False, max(1, iters // 8))
    torch.cuda.synchronize()
    rates = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        ops = bl.mma_peak_probe("imma_sync", False, iters // 2)
        b.record()
        torch.cuda.synchronize()
        rates.append(ops / (a.elapsed_time(b) * 1e-3) / 1e12)
    out["imma_sync"] = max(rates)
    assert bl.check_device_status() == 0
    out["int8"] = max(out["int8_cta"], out["int8_cta_pair"])
    out["bf16"] = max(out["bf16_cta"], out["bf16_cta_pair"])
    out["how"] = (f"tcgen05.mma loop from fixed pseudo-random shared-memory operands into TMEM, no global "
                  f"traffic; {iters} x 4 instructions per CTA (or pair) per launch, best of {reps} launches; "
                  f"imma_sync: mma.sync m16n8k32 u8 x s8 from registers, 16 warps x 8 chains per SM")
    return out


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
    if (args.only_gemv or args.table or args.next or args.only_packed or args.only_mem or args.only_gemm
            or args.only_peak):
        blbuild.build()
        bl.load()
        if args.only_peak:
            print(json.dumps({"tensor_peaks": probe_tensor_peaks(bl, torch, dev)}), flush=True)
            return
        if args.only_gemm:
            print(json.dumps({"gemm": gemm_once(bl, torch, dev, args.only_gemm, args.gemm_shape)}), flush=True)
            return
        flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
        if args.only_mem:
            print(json.dumps({"memory_kernels": mem_once(bl, torch, dev)}), flush=True)
        elif args.only_packed:
            T_, N_, K_ = (int(v) for v in args.packed_case.split(","))
            print(json.dumps({"linear_packed": packed_once(bl, torch, dev, T_, N_, K_)}), flush=True)
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
    pk = peaks()
    f32, bf16, i8, u8 = torch.float32, torch.bfloat16, torch.int8, torch.uint8

    # ---------------------------------------------------------------- tensor-pipe peaks
    clk_probe = ClockSampler(gpu_id_of(torch, dev)) if rank == 0 else None
    if clk_probe:
        clk_probe.start()
        time.sleep(0.3)
    tpk = probe_tensor_peaks(bl, torch, dev)
    if clk_probe:
        tpk["clocks"] = clk_probe.stop()

    # ---------------------------------------------------------------- inputs (HBM resident)
    lis = synth.workload_inputs(WORKLOAD_NAME)          # rank 0: the parity tests' inputs
    if rank > 0:                                        # same W; the rank's own tokens
        gen_r = synth.generator(synth.WORKLOADS[WORKLOAD_NAME].seed * 1000 + rank)
        for li in lis:
            li.X = synth.normal(tuple(li.X.shape), 1.0, gen_r).to(bf16)
            li.dY = synth.normal(tuple(li.dY.shape), synth.DY_STD_BF16, gen_r).to(bf16)
    maxK = max(li.W.shape[1] for li in lis)
    maxN = max(li.W.shape[0] for li in lis)
    T = T_TOK
    shared = dict(
        gamma=torch.empty(1, dtype=f32, device=dev), wq_i8=torch.empty(maxN * maxK, dtype=i8, device=dev),
        wq_bf16=torch.empty(maxN * maxK, dtype=bf16, device=dev),
        packed=torch.empty(maxN * maxK // 4, dtype=u8, device=dev),
        xq=torch.empty(T * maxK, dtype=i8, device=dev), sx=torch.empty(T, dtype=f32, device=dev),
        rinv=torch.empty(T, dtype=f32, device=dev), xdq=torch.empty(T * maxK, dtype=bf16, device=dev),
        y=torch.empty(T * maxN, dtype=bf16, device=dev), dX=torch.empty(T * maxK, dtype=f32, device=dev),
        dg=torch.empty(maxK, dtype=f32, device=dev), ydec=torch.empty(DECODE_B * maxN, dtype=f32, device=dev))
    ws = bl.workspace(T, maxN, maxK, dev)
    layers = []
    for li in lis:
        N, K = li.W.shape
        fo = dict(gamma=shared["gamma"], wq_i8=shared["wq_i8"][:N * K].view(N, K),
                  wq_bf16=shared["wq_bf16"][:N * K].view(N, K), packed=shared["packed"][:N * K // 4].view(N, K // 4),
                  y=shared["y"][:T * N].view(T, N), xq=shared["xq"][:T * K].view(T, K), sx=shared["sx"],
                  rinv=shared["rinv"], xdq=shared["xdq"][:T * K].view(T, K))
        layers.append(dict(name=li.shape.name, N=N, K=K, W=li.W.to(dev), X=li.X.to(dev), dY=li.dY.to(dev),
                           dW=torch.empty(N, K, dtype=f32, device=dev), fo=fo,
                           dX=shared["dX"][:T * K].view(T, K), dg=shared["dg"][:K],
                           ydec=shared["ydec"][:DECODE_B * N].view(DECODE_B, N)))
    flush = torch.empty(512 * 1024 * 1024, dtype=u8, device=dev)        # > 126 MB L2
    ovs = torch.cuda.Stream(device=dev)

    # One projection's step.  The forward is one call (bitlinear_forward_qat: the weight
    # quantiser's |W| sums, the ternary codes, the activation quantiser, the int8 GEMM); after
    # the grad-input GEMM the RMSNorm backward and the decode GEMV go to a second stream and
    # run beside the weight-gradient GEMM.  `dom` maps a GEMM's name to the two events that
    # bracket it.
    def layer_step(L, dom=None, inputs=None):
        fo = L["fo"]
        Wi, Xi, dYi = inputs if inputs is not None else (L["W"], L["X"], L["dY"])
        main = torch.cuda.current_stream(dev)
        bl.bitlinear_forward_qat(Xi, Wi, ws=ws, out=fo)
        if dom is not None and "grad_input" in dom:
            dom["grad_input"][0].record()
        bl.bitlinear_grad_input(dYi, fo["wq_bf16"], fo["gamma"], dXhat=L["dX"])
        if dom is not None and "grad_input" in dom:
            dom["grad_input"][1].record()
        ovs.wait_stream(main)
        with torch.cuda.stream(ovs):
            bl.bitlinear_rmsnorm_backward(Xi, fo["rinv"], L["dX"], ws=ws, dg=L["dg"])
            bl.ternary_gemv(fo["packed"], fo["gamma"], L["K"], fo["xq"][:DECODE_B], fo["sx"][:DECODE_B],
                            y=L["ydec"])
        if dom is not None and "grad_weight" in dom:
            dom["grad_weight"][0].record()
        bl.bitlinear_backward_weight(dYi, fo["xdq"], dW=L["dW"])
        if dom is not None and "grad_weight" in dom:
            dom["grad_weight"][1].record()
        main.wait_stream(ovs)

    # The same work as separate sequential calls with an event before each (piece times).
    def layer_pieces(L, ev):
        fo = L["fo"]
        q = dict(gamma=fo["gamma"], wq_i8=fo["wq_i8"], wq_bf16=fo["wq_bf16"], packed=fo["packed"])
        a = dict(xq=fo["xq"], sx=fo["sx"], rinv=fo["rinv"], xdq=fo["xdq"])
        ev[0].record()
        bl.bitlinear_quant_weight(L["W"], ws=ws, out=q)
        ev[1].record()
        bl.bitlinear_act_quant(L["X"], apply_rmsnorm=True, out=a)
        ev[2].record()
        bl.bitlinear_linear(fo["xq"], fo["sx"], fo["wq_i8"], fo["gamma"], y=fo["y"])
        ev[3].record()
        bl.bitlinear_grad_input(L["dY"], fo["wq_bf16"], fo["gamma"], dXhat=L["dX"])
        ev[4].record()
        bl.bitlinear_rmsnorm_backward(L["X"], fo["rinv"], L["dX"], ws=ws, dg=L["dg"])
        ev[5].record()
        bl.bitlinear_backward_weight(L["dY"], fo["xdq"], dW=L["dW"])
        ev[6].record()
        bl.ternary_gemv(fo["packed"], fo["gamma"], L["K"], fo["xq"][:DECODE_B], fo["sx"][:DECODE_B], y=L["ydec"])

    def sync_all():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
            torch.cuda.synchronize()

    # ---------------------------------------------------------------- warm-up (eager)
    for _ in range(max(3, args.warmup)):
        for L in layers:
            layer_step(L)
        for L in layers:
            dp.allreduce_weight_grad(L["dW"])
    sync_all()
    assert bl.check_device_status() == 0

    # ---------------------------------------------------------------- CUDA graphs
    # One GPU: the whole step (7 projections) is one graph.  N GPUs: one graph per projection,
    # and after each replay its dW is all-reduced asynchronously (NCCL stays outside the
    # graphs) while the next projection's graph runs.
    launches_before = bl.launch_count()
    if world == 1:
        g_all = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_all):
            for L in layers:
                layer_step(L)
        graphs = [g_all]

        def replay():
            g_all.replay()
    else:
        graphs = []
        for L in layers:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                layer_step(L)
            graphs.append(g)

        def replay():
            works = []
            for g, L in zip(graphs, layers):
                g.replay()
                works.append(dist.all_reduce(L["dW"], op=dist.ReduceOp.SUM, async_op=True))
            for w in works:
                w.wait()
    kernels_per_step = bl.launch_count() - launches_before
    # sequential pieces with events between the calls (piece times; not part of the value)
    pev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(8)] for _ in layers]
    g_pc = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_pc):
        for L, ev in zip(layers, pev):
            layer_pieces(L, ev)
        pev[-1][7].record()
    for _ in range(max(3, args.warmup)):
        replay()
        g_pc.replay()
    sync_all()
    assert bl.check_device_status() == 0

    # ---------------------------------------------------------------- timed region
    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    clk = ClockSampler(gpu_id_of(torch, dev)) if rank == 0 else None
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
    clocks = clk.stop() if clk else None
    per_step = [a.elapsed_time(b) for a, b in zip(ev_s, ev_e)]
    t = torch.tensor([sum(per_step)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    tot_ms = float(t.item())

    # ---------------------------------------------------------------- piece times
    pieces = {p: [[] for _ in layers] for p in PIECES}
    for i in range(K):
        flush.zero_()
        g_pc.replay()
        torch.cuda.synchronize()
        for li, ev in enumerate(pev):
            nxt = pev[li + 1][0] if li + 1 < len(pev) else pev[-1][7]
            for j, p in enumerate(PIECES):
                end = ev[j + 1] if j + 1 < 7 else nxt
                pieces[p][li].append(ev[j].elapsed_time(end))
    sync_all()
    piece_ms = {p: [statistics.mean(v) for v in per_layer] for p, per_layer in pieces.items()}

    # ---------------------------------------------------------------- dominant kernel, live in the step
    ops_gemm = [2.0 * T * L["N"] * L["K"] for L in layers]
    dom = max(("grad_input", "grad_weight"), key=lambda p: sum(piece_ms[p]))
    # both backward GEMMs bracketed in the same replays: the dominant one gives the roofline,
    # the other is reported beside it
    gemm_names = ("grad_input", "grad_weight")
    dev_ev = [{nm: (torch.cuda.Event(enable_timing=True, external=True),
                    torch.cuda.Event(enable_timing=True, external=True)) for nm in gemm_names} for _ in layers]
    g_dom = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.graph(g_dom):
        for L, evs in zip(layers, dev_ev):
            layer_step(L, dom=evs)
    g_dom.replay()
    torch.cuda.synchronize()
    inst_ms = {nm: [[] for _ in layers] for nm in gemm_names}
    for i in range(K):
        flush.zero_()
        g_dom.replay()
        torch.cuda.synchronize()
        for li, evs in enumerate(dev_ev):
            for nm in gemm_names:
                inst_ms[nm][li].append(evs[nm][0].elapsed_time(evs[nm][1]))
    dom_ms = inst_ms[dom]
    dom_layer_ms = [statistics.mean(v) for v in dom_ms]
    in_step = {nm: sum(statistics.mean(v) for v in inst_ms[nm]) for nm in gemm_names}
    assert bl.check_device_status() == 0
    del graphs, g_pc, g_dom

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        host = [dict(W=li.W.pin_memory(), X=li.X.pin_memory(), dY=li.dY.pin_memory()) for li in lis]
        dW_h = [torch.empty(L["N"], L["K"], dtype=f32).pin_memory() for L in layers]
        g_h = torch.empty(len(layers), dtype=f32).pin_memory()
        h2d = sum(h["W"].numel() * 4 + h["X"].numel() * 2 + h["dY"].numel() * 2 for h in host)
        d2h = sum(d.numel() * 4 for d in dW_h) + 4 * len(layers)

        # Copies run on their own streams so that PCIe traffic overlaps the compute: every
        # projection's inputs go host -> device on one stream (each projection has its own
        # device buffers), a projection's compute waits only for its own inputs, and its dW goes
        # device -> host on a third stream as soon as it is final (PCIe is full duplex).
        # gamma is copied to a per-projection device slot on the compute stream before the next
        # projection overwrites it, and read back with the gradients.
        h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        g_dev = torch.empty(len(layers), dtype=f32, device=dev)

        def e2e_step():
            main = torch.cuda.current_stream(dev)
            start = torch.cuda.Event()
            start.record(main)
            h2d_s.wait_event(start)
            d2h_s.wait_event(start)
            ready = []
            with torch.cuda.stream(h2d_s):
                for L, h in zip(layers, host):
                    L["W"].copy_(h["W"], non_blocking=True)
                    L["X"].copy_(h["X"], non_blocking=True)
                    L["dY"].copy_(h["dY"], non_blocking=True)
                    e = torch.cuda.Event()
                    e.record(h2d_s)
                    ready.append(e)
            for li, L in enumerate(layers):
                main.wait_event(ready[li])
                layer_step(L)
                g_dev[li:li + 1].copy_(L["fo"]["gamma"])
                dp.allreduce_weight_grad(L["dW"])
                done = torch.cuda.Event()
                done.record(main)
                d2h_s.wait_event(done)
                with torch.cuda.stream(d2h_s):
                    dW_h[li].copy_(L["dW"], non_blocking=True)
            d2h_s.wait_stream(main)
            with torch.cuda.stream(d2h_s):
                g_h.copy_(g_dev, non_blocking=True)
            main.wait_stream(d2h_s)

        e2e_step()
        sync_all()
        ke = max(1, min(K, 10))
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(ke)]
        for i in range(ke):
            flush.zero_()
            es[i][0].record()
            e2e_step()
            es[i][1].record()
        sync_all()
        e2e_ms = torch.tensor([sum(a.elapsed_time(b) for a, b in es)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
        e2e = {"value": T * world * ke / (float(e2e_ms.item()) * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": ke,
               "how": "pinned host -> device copies of every projection's W, X, dY on a copy stream, each "
                      "projection's eager library calls as soon as its inputs have landed, device -> host copies "
                      "of its dW on a second copy stream as soon as it is final, gamma read back at the end; "
                      "CUDA events around each step on the compute stream, which joins both copy streams"}
        del host, dW_h

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    # ---------------------------------------------------------------- roofline of the dominant kernel
    bf16_peak = pk["bf16"]
    int8_peak = tpk["int8"]
    dom_ms_tot = sum(dom_layer_ms)
    achieved = sum(ops_gemm) / (dom_ms_tot * 1e-3) / 1e12
    kernel_names = {"linear_i8": "tc_gemm2_kernel<int8,K,K,linear> (2-SM, 256x256)",
                    "grad_input": "tc_gemm2_kernel<bf16,K,MN,scale_f32> (2-SM, 256x256)",
                    "grad_weight": "tc_gemm2_kernel<bf16,MN,MN,f32> (2-SM, 256x256)"}
    roofline = {"bound": "tensor", "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": achieved / bf16_peak, "traffic": ncu_traffic(dom), "kernel": kernel_names[dom],
                "peak_kind": f"bf16 dense, cuBLAS burst ({pk['src']})",
                "launch_ms": dom_ms_tot / len(layers), "launches_per_step": len(layers),
                "flop_per_launch": sum(ops_gemm) / len(layers),
                "per_layer_ms": {L["name"]: round(v, 5) for L, v in zip(layers, dom_layer_ms)},
                "frac_of_probe_bf16": achieved / tpk["bf16"],
                "in_step": {nm: {"ms_per_step": in_step[nm],
                                 "achieved": sum(ops_gemm) / (in_step[nm] * 1e-3) / 1e12,
                                 "frac": sum(ops_gemm) / (in_step[nm] * 1e-3) / 1e12 / bf16_peak}
                            for nm in gemm_names},
                "how": "two event nodes around this GEMM of every projection inside K further replays of the "
                       "timed step's graph (L2 flushed before each; the grad-input GEMM is bracketed in the same "
                       "replays, `in_step`); achieved = its FLOPs / its time, summed over the projections"}

    # every kernel of the step against its roofline (sequential piece times)
    def bytes_of(p, L):
        N, K = L["N"], L["K"]
        if p == "act_quant":
            return T * K * 2 + T * K + T * K * 2 + 8 * T
        if p == "quant_weight":
            return N * K * 4 + N * K + N * K * 2 + N * K // 4
        if p == "rmsnorm_bwd":
            return T * K * 4 + T * K * 2 + T * K * 4 + 4 * T
        if p == "decode_gemv":
            return N * K // 4 + DECODE_B * K + 4 * DECODE_B * N + 4 * DECODE_B
        return None
    kernels = {}
    for p in PIECES:
        ms = sum(piece_ms[p])
        rec = {"ms_per_step": ms, "share_of_pieces": ms / sum(sum(v) for v in piece_ms.values())}
        if p in ("linear_i8", "grad_input", "grad_weight"):
            rate = sum(ops_gemm) / (ms * 1e-3) / 1e12
            pkv = int8_peak if p == "linear_i8" else bf16_peak
            rec.update({"achieved": rate, "unit": "TOPS" if p == "linear_i8" else "TFLOP/s", "peak": pkv,
                        "frac": rate / pkv,
                        "peak_kind": "int8 measured (own tcgen05 kind::i8 loop)" if p == "linear_i8"
                        else f"bf16 dense, cuBLAS burst ({pk['src']})"})
        else:
            nb = sum(bytes_of(p, L) for L in layers)
            rate = nb / (ms * 1e-3) / 1e9
            rec.update({"achieved": rate, "unit": "GB/s", "peak": pk["hbm"], "frac": rate / pk["hbm"],
                        "bytes_per_step": nb})
        rec["per_layer_ms"] = {L["name"]: round(v, 5) for L, v in zip(layers, piece_ms[p])}
        kernels[p] = rec

    sub = None
    if not args.no_sub:
        sub = {"decode_gemv": gemv_measure(bl, torch, dev, flush, pk, imma_peak=tpk["imma_sync"]),
               "hbm_kernels_b2b": hbm_b2b_measure(bl, torch, dev, flush, pk),
               "configs": configs_measure(bl, torch, dev, flush)}

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline()

    value = T * world * K / (tot_ms * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": tot_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "s8+bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_gpu": T,
                   "layers": {L["name"]: f"{L['K']}->{L['N']}" for L in layers},
                   "decode_batch": DECODE_B, "parallelism": f"dp{world}",
                   "l2": "flushed before every timed step (512 MB write); every projection's inputs exceed L2"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(kernels_per_step * K),
        "timing": ("each step replays CUDA graph(s) of the step's library calls (per projection: forward_qat, "
                   "grad-input GEMM, then RMSNorm backward and decode GEMV on a second stream beside the "
                   "weight-gradient GEMM) with no event node inside; the roofline's GEMM times come from K "
                   "further replays with event nodes around that GEMM, and `kernels` from a sequential graph "
                   "with events between all calls; gpu_launches = kernels per step x steps"),
        "clocks": clocks,
        "tensor_peaks": tpk,
        "kernels": kernels,
        "sub": sub,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()



def timed_b2b(bl, torch, flush, calls, reps):
    """`reps` launches cycling over `calls`, captured in one CUDA graph between one pair of CUDA
    events (median of 5 replays, L2 flushed before each): microseconds per launch."""
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


def hbm_b2b_measure(bl, torch, dev, flush, pk):
    """The HBM-bound kernels of the step at the 7B layer's sizes (16384 tokens; d_in 4096 and
    11008; weights 4096 x 4096 and 11008 x 4096), each launched back to back over input copies
    that together exceed L2, so every launch reads from HBM; bytes are algorithmic (each tensor
    read once, each output written once)."""
    from bit_ternary_qat_b200 import synth
    gen = synth.generator(91)
    T = 16384
    out = {}

    def row(us, nbytes, note):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us": us, "GB/s": gbs, "frac_hbm": gbs / pk["hbm"], "bytes": nbytes, "note": note}

    for K, copies in ((4096, 3), (11008, 2)):
        Xs = [synth.normal((T, K), 1.0, gen).to(torch.bfloat16).to(dev) for _ in range(copies)]
        a = dict(xq=torch.empty(T, K, dtype=torch.int8, device=dev), sx=torch.empty(T, device=dev),
                 rinv=torch.empty(T, device=dev), xdq=torch.empty(T, K, dtype=torch.bfloat16, device=dev))
        us = timed_b2b(bl, torch, flush, [lambda X=X: bl.bitlinear_act_quant(X, out=a) for X in Xs], 4 * copies)
        out[f"act_quant_{T}x{K}"] = row(us, T * K * 5 + 8 * T, "RMSNorm + per-token int8 codes + bf16 X_dq")
        ws = bl.workspace(T, 16, K, dev)
        dg = torch.empty(K, device=dev)
        dXs = [synth.normal((T, K), 1e-2, gen).to(dev) for _ in range(2 if K == 4096 else 1)]
        Xb = Xs[:len(dXs)]
        us = timed_b2b(bl, torch, flush, [lambda X=X, d=d: bl.bitlinear_rmsnorm_backward(X, a["rinv"], d, ws=ws, dg=dg)
                                          for X, d in zip(Xb, dXs)], 4 * len(dXs))
        out[f"rmsnorm_bwd_{T}x{K}"] = row(us, T * K * 10 + 4 * T, "reads fp32 dX_hat and bf16 X, writes fp32 dX "
                                                                    "(plus the dg partial rows and their sum)")
        del Xs, dXs, a, ws
        torch.cuda.empty_cache()
    for (N, K), copies in (((4096, 4096), 4), ((11008, 4096), 2)):
        Ws = [synth.normal((N, K), 0.02, gen).to(dev) for _ in range(copies)]
        ws = bl.workspace(1, N, K, dev)
        q = dict(gamma=torch.empty(1, dtype=torch.float32, device=dev),
                 wq_i8=torch.empty(N, K, dtype=torch.int8, device=dev),
                 wq_bf16=torch.empty(N, K, dtype=torch.bfloat16, device=dev),
                 packed=torch.empty(N, K // 4, dtype=torch.uint8, device=dev))
        us = timed_b2b(bl, torch, flush, [lambda W=W: bl.bitlinear_quant_weight(W, ws=ws, out=q) for W in Ws],
                       4 * copies)
        rec = row(us, int(N * K * 7.25), "two launches: |W| partial sums, then codes (int8 + bf16 + 2-bit); "
                                        "W is read twice (the second read hits L2 only when W fits there)")
        rec["frac_hbm_both_reads"] = (N * K * 11.25) / (us * 1e-6) / 1e9 / pk["hbm"]
        out[f"quant_weight_{N}x{K}"] = rec
        del Ws, ws, q
        torch.cuda.empty_cache()
    out["hbm_peak_GBs"] = pk["hbm"]
    return out

def configs_measure(bl, torch, dev, flush, steps: int = 5):
    """The other training configurations' full steps (single, square, mlp7b): per layer weight
    quantisation, activation quantisation, forward GEMM, grad-input GEMM, RMSNorm backward,
    weight-gradient GEMM, all in one CUDA graph; L2 flushed before each replay; median of
    `steps`."""
    from bit_ternary_qat_b200 import synth
    out = {}
    for name in ("single", "square", "mlp7b"):
        ms, T, layers = step_graph_ms(bl, torch, dev, flush, name, steps)
        out[name] = {"ms_per_step": ms, "tokens_per_s": T / (ms * 1e-3), "layers": layers,
                     "dtype": synth.WORKLOADS[name].dtype}
    return out


def step_graph_ms(bl, torch, dev, flush, name, steps):
    from bit_ternary_qat_b200 import synth
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
    layers = [f"{L['K']}->{L['N']}" for L in dev_layers]
    del dev_layers, shared, ws
    torch.cuda.empty_cache()
    return statistics.median(ms), T, layers


def gemm_once(bl, torch, dev, which: str, shape: str = "gate"):
    """Three launches of one GEMM of the step on one projection's shape at 16384 tokens (q
    4096 -> 4096, gate 4096 -> 11008, down 11008 -> 4096): a small case for a profiler capture
    (at most about 1.5 GB on the device)."""
    T = 16384
    K, N = {"q": (4096, 4096), "gate": (4096, 11008), "down": (11008, 4096)}[shape]
    g = torch.Generator(device=dev).manual_seed(1)
    gamma = torch.full((1,), 0.02, device=dev)
    if which == "linear_i8":
        xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, device=dev, generator=g)
        wq = torch.randint(-1, 2, (N, K), dtype=torch.int8, device=dev, generator=g)
        sx = torch.full((T,), 50.0, device=dev)
        y = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
        call = lambda: bl.bitlinear_linear(xq, sx, wq, gamma, y=y)  # noqa: E731
    elif which == "grad_input":
        dY = (torch.randn(T, N, device=dev, generator=g) * 1e-2).to(torch.bfloat16)
        wq = torch.randint(-1, 2, (N, K), device=dev, generator=g).to(torch.bfloat16)
        dX = torch.empty(T, K, dtype=torch.float32, device=dev)
        call = lambda: bl.bitlinear_grad_input(dY, wq, gamma, dXhat=dX)  # noqa: E731
    else:
        dY = (torch.randn(T, N, device=dev, generator=g) * 1e-2).to(torch.bfloat16)
        xdq = (torch.randn(T, K, device=dev, generator=g)).to(torch.bfloat16)
        dW = torch.empty(N, K, dtype=torch.float32, device=dev)
        call = lambda: bl.bitlinear_backward_weight(dY, xdq, dW=dW)  # noqa: E731
    ms = 0.0
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
    assert bl.check_device_status() == 0
    return {"which": which, "shape": f"T={T} K={K} N={N}", "ms_last": ms,
            "tflops_last": 2.0 * T * N * K / (ms * 1e-3) / 1e12}


def gemv_measure(bl, torch, dev, flush, pk, imma_peak=None):
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
        rec = {"us": ms * 1e3, "GB/s": gbs, "frac_hbm": gbs / pk["hbm"],
               "int_ops_T": 2.0 * B * N * K / (ms * 1e-3) / 1e12}
        if imma_peak:
            # the MMAs run 8 batch columns per n-tile (one n-tile up to B = 8, two beyond)
            mma_ops = 2.0 * (8 if B <= 8 else 16) * N * K
            rec["imma_bound_us"] = mma_ops / (imma_peak * 1e12) * 1e6
            rec["frac_imma"] = rec["imma_bound_us"] / rec["us"]
        out[f"B{B}"] = rec
    # per-launch fixed cost vs streaming rate: the same launches on a weight twice as tall
    # (57344 x 8192, 117 MB; 2 copies cycled): marginal rate = the extra 58.7 MB / the extra time
    W2, _ = synth.decode_inputs(1, 2 * N, K, seed=44)
    q2 = bl.bitlinear_quant_weight(W2.to(dev), want_i8=False, want_bf16=False)
    del W2
    packs2 = [q2["packed"], q2["packed"].clone()]
    for B in (1, 4, 16):
        _, x = synth.decode_inputs(B, 16, K, seed=40 + B)
        aq = bl.bitlinear_act_quant(x.to(dev), apply_rmsnorm=False, want_xdq=False)
        y = torch.empty(B, 2 * N, dtype=torch.float32, device=dev)
        for i in range(4):
            bl.ternary_gemv(packs2[i % 2], q2["gamma"], K, aq["xq"], aq["sx"], y=y)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(reps):
                bl.ternary_gemv(packs2[i % 2], q2["gamma"], K, aq["xq"], aq["sx"], y=y)
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
        us2 = statistics.median(samples) * 1e3
        rec = out[f"B{B}"]
        extra = us2 - rec["us"]
        rec["us_2x_rows"] = us2
        rec["marginal_GB/s"] = (N * K // 4) / (extra * 1e-6) / 1e9 if extra > 0 else None
        rec["marginal_frac_hbm"] = rec["marginal_GB/s"] / pk["hbm"] if rec["marginal_GB/s"] else None
        rec["fixed_us"] = rec["us"] - extra

    def graph_us(call, flush_first=True):
        """us per launch of `reps` launches call(0..reps-1) in one CUDA graph, median of 5."""
        for i in range(8):
            call(i)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(reps):
                call(i)
        graph.replay()
        samples = []
        for _ in range(5):
            if flush_first:
                flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            torch.cuda.synchronize()
            samples.append(a.elapsed_time(b) / reps)
        del graph
        return statistics.median(samples) * 1e3

    # the read-only ceiling of the same bytes, read the same way and chained the same way (the
    # library's read probe: no arithmetic), on the same weight copies and the 2x-tall ones
    sink = torch.zeros(4, dtype=torch.int32, device=dev)
    wbytes = N * K // 4
    ceiling = {}
    for pat in ("gemv", "coalesced"):
        u1 = graph_us(lambda i: bl.read_peak_probe(packs[i % copies], pat, sink))
        u2 = graph_us(lambda i: bl.read_peak_probe(packs2[i % 2], pat, sink))
        ceiling[pat] = {"us": u1, "GB/s": wbytes / (u1 * 1e-6) / 1e9, "frac_hbm": wbytes / (u1 * 1e-6) / 1e9 / pk["hbm"],
                        "marginal_GB/s": wbytes / ((u2 - u1) * 1e-6) / 1e9 if u2 > u1 else None,
                        "fixed_us": 2 * u1 - u2}
    assert bl.check_device_status() == 0
    out["read_ceiling"] = ceiling
    for B in (1, 4, 16):
        out[f"B{B}"]["frac_of_read_ceiling"] = ceiling["gemv"]["us"] / out[f"B{B}"]["us"]
    del packs2, q2

    # the GEMV's loop with the weight resident in L2 (one 4736- or 14208-row weight, 9.7 or
    # 29.1 MB, reused by every launch): the marginal time per 28672 rows is its
    # instruction-bound rate, to set beside the streaming rate above
    small = {}
    for n in (4736, 14208):
        Wn, _ = synth.decode_inputs(1, n, K, seed=45)
        small[n] = bl.bitlinear_quant_weight(Wn.to(dev), want_i8=False, want_bf16=False)
        del Wn
    for B in (1, 4, 16):
        _, x = synth.decode_inputs(B, 16, K, seed=40 + B)
        aq = bl.bitlinear_act_quant(x.to(dev), apply_rmsnorm=False, want_xdq=False)
        t = {}
        for n in (4736, 14208):
            y = torch.empty(B, n, dtype=torch.float32, device=dev)
            qn = small[n]
            t[n] = graph_us(lambda i: bl.ternary_gemv(qn["packed"], qn["gamma"], K, aq["xq"], aq["sx"], y=y),
                            flush_first=False)
        out[f"B{B}"]["l2_resident_us_per_28672_rows"] = (t[14208] - t[4736]) / (14208 - 4736) * N
    del small
    out["hbm_peak_GBs"] = pk["hbm"]
    out["imma_peak_T"] = imma_peak
    out["workload"] = ("decode: packed W 28672x8192 (58.7 MB), int8 x [B x 8192]; 4 weight copies cycled "
                       "(inputs larger than L2), 40 launches in one CUDA graph per event pair, median of 5; "
                       "marginal rate and fixed cost from the same launches on a 57344x8192 weight (2 copies); "
                       "read_ceiling: the library's read probe on the same copies (the GEMV's partition and a "
                       "coalesced one, no arithmetic); l2_resident: the GEMV on 4736- and 14208-row weights "
                       "reused by every launch")
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


def packed_once(bl, torch, dev, T=16, N=28672, K=8192):
    """Three launches of the packed-weight linear, T tokens x an N x K weight (a small case for a
    profiler capture); returns the last launch's event time."""
    from bit_ternary_qat_b200 import synth
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
    for (T, N, K) in ((16, 28672, 8192), (64, 28672, 8192), (256, 28672, 8192), (32, 11008, 4096),
                      (64, 11008, 4096), (128, 11008, 4096), (256, 11008, 4096), (64, 4096, 4096),
                      (256, 4096, 4096)):
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
               "speedup_vs_int8": us_8 / us_p,
               "kernel": "ternary_gemv" if T <= 16 else "tc_gemm_packed2 (CTA pairs)",
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
            full, wq_only = oracle_step(ora, li, t_s)
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


if __name__ == "__main__":
    main()
