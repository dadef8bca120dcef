#!/usr/bin/env python3
"""GPTQ layer-quantization benchmark.

One step = the whole hot path for one linear layer of 4096 x 4096 with n = 2048
bf16 calibration tokens, 4-bit asymmetric, group 128, lambda = 0.01 * mean(diag H):
  H = 2 X^T X (tensor cores) -> U = upper Cholesky factor of (H + lambda I)^-1 ->
  GPTQ column loop with 128-column lazy blocks and 3xTF32 trailing updates,
  writing packed int32 codes, fp16 scales and packed zeros.
Inputs are seeded synthetic data (package ``inputs``: lognormal channel scales with
0.5 % hot channels for X, N(0, 0.02^2) weights with 0.1 % outliers), resident in HBM
when timing starts; W is restored from a pristine copy and the L2 is flushed (256 MB
write) before every step, outside the per-step CUDA events.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
       python bench.py --workload stack7b [--steps K] [--warmup W]
       python bench.py --workload dqgemm [--steps K] [--warmup W]   (dequantizing GEMM on the output)
The stack7b workload times one block of the 7B-shaped stack (q, k, v, o 4096 x 4096;
gate, up 11008 x 4096; down 4096 x 11008; n = 2048 tokens each, 4-bit g128) per step;
every block has the same shapes, so the 32-block stack time is 32 times that.
With N > 1 (torchrun, one rank per GPU) every rank quantizes its own independent
layer (weak scaling, no collective on the data path); the reported time is the max
over ranks.  Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/layer & weights quantized/s at 4096×4096 n=2048 4b g128; % of roofline"
UNIT = "weights/s"
D_OUT, D_IN, N_TOK, BITS, GROUP, SYM = 4096, 4096, 2048, 4, 128, False
WORKLOAD = "attn 4096x4096, n=2048 bf16 tokens, 4-bit asym g128"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- clocks during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle leg

def oracle_layer_time(layer) -> tuple[float, str, int]:
    """Seconds for the fp64 oracle to quantize the whole layer: H = 2 X^T X, U = chol(Hd^-1)
    (explicit inverse, then Cholesky) and the lazy-block column loop over every row.
    Measured, not extrapolated."""
    import numpy as np

    from oracle import gptq_oracle as O

    X = layer.X.astype(np.float64)
    t0 = time.perf_counter()
    H = O.hessian(X)
    t1 = time.perf_counter()
    Hd, _ = O.damp(H, 0.01)
    U = O.hinv_upper_cholesky(Hd)
    t2 = time.perf_counter()
    O.gptq(layer.W, U, BITS, GROUP, SYM, 128)
    t3 = time.perf_counter()
    sample = (f"the whole {layer.d_out}x{layer.d_in} layer, measured: H=2X^T X, U=chol(Hd^-1) and the column loop "
              f"over all {layer.d_out} rows (fp64 numpy/LAPACK); H {t1 - t0:.2f}s U {t2 - t1:.2f}s "
              f"column loop {t3 - t2:.2f}s")
    return t3 - t0, sample, len(os.sched_getaffinity(0))


def bench_config(world: int, desc_act: int) -> dict:
    """The workload description both arms print (the same dict in each)."""
    return {"workload": WORKLOAD, "d_out": D_OUT, "d_in": D_IN, "n": N_TOK, "bits": BITS, "group_size": GROUP,
            "sym": SYM, "damp_rel": 0.01, "desc_act": desc_act,
            "l2": "flushed (256 MB write) before every step, outside the step events",
            "parallelism": f"{world} independent layers, one per GPU"}


def max_over_ranks(ms: float, dist, device) -> float:
    """The job's time: the slowest rank's (identity without a process group)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank_step: float, steps: int, total_ms: float) -> float:
    """Units all ranks processed per second over the (max-over-ranks) timed region."""
    return world * units_per_rank_step * steps / (total_ms / 1e3)


def layer_seed(rank: int) -> int:
    """Each rank quantizes its own independent layer (weak scaling)."""
    return rank


def run_reference(args, rank: int, world: int) -> None:
    """The reference arm: the fp64 CPU oracle, as it stands, on the machine's host cores; every
    step quantizes the whole layer.  Under torchrun only rank 0 runs it."""
    if rank != 0:
        return
    from post_weight_quantization_14_b200 import inputs as I

    layer = I.make_layer("attn", seed=0)
    for _ in range(args.warmup):
        oracle_layer_time(layer)
    secs = []
    sample, cores = "", 0
    for _ in range(args.steps):
        s_, sample, cores = oracle_layer_time(layer)
        secs.append(s_)
    ms = 1e3 * sum(secs) / len(secs)
    value = D_OUT * D_IN / (ms / 1e3)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(world, args.desc_act),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "step_s": secs}
    print(json.dumps(line), flush=True)


def relaunch_command(argv: list[str], n: int, port: int) -> list[str]:
    """bench.py --gpus N started without torchrun: the same command as N ranks, one per GPU."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s_:
        s_.bind(("127.0.0.1", 0))
        return s_.getsockname()[1]


def rank_probe(world: int, rank: int) -> None:
    """--rank-probe: every rank joins a gloo group and reports its rank (a check of the
    launch plumbing that needs no GPU)."""
    import datetime

    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    t = torch.tensor([float(rank)])
    dist.all_reduce(t)
    if rank == 0:
        print(json.dumps({"rank_probe": True, "world": dist.get_world_size(), "rank_sum": float(t.item())}),
              flush=True)
    dist.barrier()
    dist.destroy_process_group()


# ---------------------------------------------------------------- GPU leg

CHOL_KERNELS = ("chol_dag", "damp_copy", "diag_mean", "perm_invert", "damp_copy_perm")
QUANT_KERNELS = ("colloop", "trailing_update", "trailing_update_sb", "up_prep", "ut_split", "pack_zeros", "row_params",
                 "gather_cols", "unpermute_codes")
ACT_KERNELS = ("act_sum", "act_rank", "act_perm")   # activation ordering (--desc-act 1 or 2)
# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu --set full capture of this
# workload, for kernels whose launches all do the same work and whose code has not changed since the capture
# (the kernel's ncu summary under profiles/); the column loop and the generic GEMM changed after theirs.
TRAFFIC_PER_LAUNCH = {"chol_dag": 39034112 + 311716096}
# Sum of the stage bounds for this layer: Hessian 21.0 us (bf16), factor + invert 168.1 us and
# trailing updates 244.3 us (3xTF32 at a third of bf16 x 1.1/2.25), column loop 11.6 us (HBM).
# The trailing updates here run as bf16x3 products (a third of bf16, 122 us at that rate); the
# bound keeps the 3xTF32 figure it was set with.
END_TO_END_BOUND_MS = 0.445


def measure_tf32_tflops(dev) -> float | None:
    """Dense TF32 tensor-core throughput of this GPU, measured the way the bf16 peak is: a
    cuBLAS fp32 GEMM with TF32 allowed, 8192^3 (2 N^3 flops), best of 5, CUDA events."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    try:
        torch.backends.cuda.matmul.allow_tf32 = True
        n = 8192
        a = torch.randn((n, n), device=dev, dtype=torch.float32)
        b = torch.randn((n, n), device=dev, dtype=torch.float32)
        for _ in range(2):
            torch.matmul(a, b)
        best = None
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        del a, b
        return 2.0 * n ** 3 / (best / 1e3) / 1e12
    except Exception:
        return None
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def kernel_rooflines(kernel_ms: dict, launches: dict, hbm: float, bf16: float, peak_kind: str,
                     tf32: float | None = None) -> dict:
    """Achieved vs peak per kernel class, from algorithmic work and measured per-step time.

    Algorithmic work:
      trailing_update  2 * d_out * (d_in - e) * 128 flops per launch, summed over the layer; bf16x3
      chol_dag         2/3 d_in^3 flops (factor + triangular inverse) per launch; 3xTF32
      hessian_syrk     n * d_in * (d_in + 1) flops; bf16
      colloop          W read once + codes + scales/zeros written, bytes; HBM
    tf32 peak = measured bf16 x 1.1/2.25 (nominal ratio); 3xTF32 peak = a third of it.
    """
    B = 128
    d_out, d_in, n = D_OUT, D_IN, N_TOK
    tf32x3 = (tf32 if tf32 else bf16 * (1.1 / 2.25)) / 3.0
    tf32_kind = "cuBLAS TF32 measured in this run" if tf32 else f"{peak_kind} bf16 x 1.1/2.25"
    sm_fp32 = 128 * 2 * 1.965e9 / 1e12            # one SM, TFLOP/s at max clock
    out = {}
    def add(name, bound, work, unit, peak, note):
        ms = kernel_ms.get(name)
        if not ms:
            return
        scale = 1e9 if unit == "GB/s" else 1e12
        ach = work / (ms / 1e3) / scale
        out[name] = {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
                     "traffic": TRAFFIC_PER_LAUNCH.get(name), "launches": launches.get(name), "note": note}
    trailing = sum(2.0 * d_out * (d_in - (b + 1) * B) * B for b in range(d_in // B) if (b + 1) * B < d_in)
    tr_ms = kernel_ms.get("trailing_update", 0) + kernel_ms.get("trailing_update_sb", 0)
    if tr_ms:
        ach = trailing / (tr_ms / 1e3) / 1e12
        bf16x3 = bf16 / 3.0   # three bf16 products per product of the 16-bit operand splits
        out["trailing_update"] = {"bound": "tensor", "achieved": ach, "peak": bf16x3, "unit": "TFLOP/s",
                                  "frac": ach / bf16x3, "traffic": None,
                                  "launches": launches.get("trailing_update", 0) + launches.get("trailing_update_sb", 0),
                                  "note": f"all trailing updates (per block and per superblock, {tr_ms:.3f} ms); "
                                          f"bf16x3 (bf16 {peak_kind} / 3)"}
    add("hessian_syrk", "tensor", 1.0 * n * d_in * (d_in + 1), "TFLOP/s", bf16, f"bf16 {peak_kind} burst")
    col_bytes = 4.0 * d_out * d_in + BITS / 8 * d_out * d_in + (2 + BITS / 8) * d_out * (d_in // GROUP)
    add("colloop", "hbm", col_bytes, "GB/s", hbm, f"HBM {peak_kind}; latency chain of d_in rounding steps per row")
    add("chol_dag", "tensor", (2.0 / 3.0) * d_in ** 3, "TFLOP/s", tf32x3,
        f"Cholesky d^3/3 + triangular inverse d^3/3 flops in one persistent launch; 3xTF32 ({tf32_kind} / 3); "
        "its time is bounded below by the chain of 128x128 diagonal blocks")
    return out


def run_stack(args) -> None:
    """One step = the seven layers of block 0 of the 7B-shaped stack, end to end on the device."""
    import numpy as np
    import torch

    from post_weight_quantization_14_b200 import gptq as G
    from post_weight_quantization_14_b200 import inputs as I

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    layers = []
    for index in range(7):
        ly = I.make_stack_layer(0, index)
        cfg = G.make_config(ly.spec.bits, ly.spec.group_size, ly.spec.sym, 128, ly.spec.damp_rel)
        W0 = torch.from_numpy(ly.W).to(dev)
        X = torch.from_numpy(ly.X_bits.view(np.int16)).to(dev).view(torch.bfloat16)
        bufs = G.LayerBuffers(ly.d_out, ly.d_in, ly.n, torch.bfloat16, cfg, dev)
        layers.append((ly, W0, torch.empty_like(W0), X, bufs))
    stream = torch.cuda.current_stream()
    # --shared-input: q, k, v read one input and gate, up another (as in a transformer
    # block), so each group takes one H and one U; the group's first layer's X is used.
    groups = [[0, 1, 2], [3], [4, 5], [6]] if args.shared_input else [[i] for i in range(7)]
    shared = {}
    if args.shared_input:
        for grp in groups:
            if len(grp) > 1:
                ly0 = layers[grp[0]][0]
                cfg = G.make_config(ly0.spec.bits, ly0.spec.group_size, ly0.spec.sym, 128, ly0.spec.damp_rel)
                shared[grp[0]] = G.SharedInputBuffers([layers[i][0].d_out for i in grp], ly0.d_in, ly0.n,
                                                      torch.bfloat16, cfg, dev)

    def step(marks=None):
        for gi, grp in enumerate(groups):
            for i in grp:
                layers[i][2].copy_(layers[i][1])
            if marks:
                marks[gi][0].record(stream)
            if len(grp) == 1:
                ly, W0, W, X, bufs = layers[grp[0]]
                G.quantize_layer(W, X, buffers=bufs)
            else:
                G.quantize_layers_shared_input([layers[i][2] for i in grp], layers[grp[0]][3],
                                               buffers=shared[grp[0]])
            if marks:
                marks[gi][1].record(stream)

    for _ in range(args.warmup):
        step()
    G.gptq_sync_status()
    marks = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in groups]
             for _ in range(args.steps)]
    torch.cuda.synchronize()
    for m in marks:
        step(m)
    torch.cuda.synchronize()
    G.gptq_sync_status()
    per_layer = {"+".join(layers[i][0].name.split(".")[-1] for i in grp):
                 statistics.median(m[gi][0].elapsed_time(m[gi][1]) for m in marks) for gi, grp in enumerate(groups)}
    block_ms = sum(per_layer.values())
    weights = sum(ly.d_out * ly.d_in for ly, *_rest in layers)
    print(json.dumps({"metric": "7B-shaped stack end-to-end quantize time (32 blocks x 7 layers)",
                      "value": 32 * block_ms / 1e3, "unit": "s", "higher_is_better": False, "n_gpus": 1,
                      "steps": args.steps, "warmup": args.warmup, "dtype": "f32", "data": "synthetic",
                      "config": {"workload": "stack7b: one block per step (block 0 seeds), x32 blocks",
                                 "n": 2048, "bits": 4, "group_size": 128, "sym": False,
                                 "shared_input": bool(args.shared_input)},
                      "block_ms": block_ms, "layer_ms": per_layer,
                      "weights_per_s": 32 * weights / (32 * block_ms / 1e3)}), flush=True)


def run_dqgemm(args) -> None:
    """Dequantizing GEMM Y = X W_hat^T on the packed output of the quantizer (4096 x 4096
    attention layer, 4-bit asym g128, quantized once by this library): prefill with the
    layer's 2048 bf16 tokens (timed, tensor roofline) and a 16-token decode batch (HBM
    roofline over the packed weights).  X is larger than nothing in L2 can hide for the
    prefill; the L2 is flushed before every timed step anyway."""
    import numpy as np
    import torch

    from post_weight_quantization_14_b200 import gptq as G
    from post_weight_quantization_14_b200 import inputs as I

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    layer = I.make_layer("attn", seed=0)
    cfg = G.make_config(BITS, GROUP, SYM, 128, 0.01)
    W = torch.from_numpy(layer.W).to(dev)
    X = torch.from_numpy(layer.X_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    q = G.quantize_layer(W, X, buffers=G.LayerBuffers(D_OUT, D_IN, N_TOK, torch.bfloat16, cfg, dev))
    G.gptq_sync_status()
    Y = torch.empty((N_TOK, D_OUT), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(Xm, Ym, steps):
        for _ in range(args.warmup):
            G.gptq_dequant_gemm(Xm, q.qweight, q.scales, q.qzeros, D_OUT, D_IN, cfg, Ym)
        G.gptq_sync_status()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in evs:
            flush.fill_(1)
            a.record(stream)
            G.gptq_dequant_gemm(Xm, q.qweight, q.scales, q.qzeros, D_OUT, D_IN, cfg, Ym)
            b.record(stream)
        torch.cuda.synchronize()
        G.gptq_sync_status()
        return [a.elapsed_time(b) for a, b in evs]

    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    ms = timed(X, Y, args.steps)
    X16 = X[:16].contiguous()
    Y16 = torch.empty((16, D_OUT), dtype=torch.float32, device=dev)
    ms16 = timed(X16, Y16, args.steps)
    clocks = sampler.stop()
    t = sum(ms) / len(ms)
    t16 = statistics.median(ms16)
    flops = 2.0 * N_TOK * D_OUT * D_IN
    hbm, bf16, _, peak_kind = peaks()
    packed_bytes = q.qweight.numel() * 4 + q.scales.numel() * 2 + q.qzeros.numel() * 4
    bytes16 = packed_bytes + 16 * D_IN * 2 + 16 * D_OUT * 4

    # end to end through the C ABI: X from pinned host memory in, Y back to pinned host memory
    X_host = torch.from_numpy(layer.X_bits.view(np.int16)).pin_memory()
    Y_host = torch.empty((N_TOK, D_OUT), dtype=torch.float32).pin_memory()
    Xd = torch.empty(X_host.shape, dtype=torch.int16, device=dev)
    e2e_steps = max(3, min(args.steps, 20))
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(e2e_steps):
        Xd.copy_(X_host, non_blocking=True)
        G.gptq_dequant_gemm(Xd.view(torch.bfloat16), q.qweight, q.scales, q.qzeros, D_OUT, D_IN, cfg, Y)
        Y_host.copy_(Y, non_blocking=True)
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ea.elapsed_time(eb) / e2e_steps

    cpu = None
    if not args.no_cpu_baseline:
        from oracle import gptq_oracle as O
        Xs = layer.X[:64].astype(np.float64)
        qw, sc, qz = q.qweight.cpu().numpy(), q.scales.cpu().numpy(), q.qzeros.cpu().numpy()
        t0 = time.perf_counter()
        O.dequant_gemm(Xs, qw, sc, qz, D_OUT, D_IN, BITS, GROUP, SYM)
        secs = time.perf_counter() - t0
        cpu = {"value": 2.0 * 64 * D_OUT * D_IN / secs / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
               "kind": "oracle", "sample": "64 of the 2048 tokens (fp64 dequantization + matmul)"}

    print(json.dumps({
        "metric": "dequant-GEMM Y = X W_hat^T on the packed 4-bit g128 format, 2048 x 4096 x 4096",
        "value": flops / (t / 1e3) / 1e12, "unit": "TFLOP/s", "higher_is_better": True, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 x int4 -> f32", "data": "synthetic",
        "config": {"workload": "dqgemm: attn 4096x4096 quantized 4-bit asym g128, X = its 2048 bf16 tokens",
                   "M": N_TOK, "N": D_OUT, "K": D_IN, "l2": "flushed (256 MB write) before every step"},
        "roofline": {"bound": "tensor", "achieved": flops / (t / 1e3) / 1e12, "peak": bf16, "unit": "TFLOP/s",
                     "frac": flops / (t / 1e3) / 1e12 / bf16, "traffic": None, "peak_kind": peak_kind},
        "decode16": {"ms": t16, "bytes": bytes16, "achieved_gbs": bytes16 / (t16 / 1e3) / 1e9, "peak_gbs": hbm,
                     "frac": bytes16 / (t16 / 1e3) / 1e9 / hbm},
        "e2e": {"value": flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": X_host.numel() * 2, "d2h_bytes_per_step": Y_host.numel() * 4,
                "steps": e2e_steps},
        "cpu_baseline": cpu, "gpu_launches": 2 * args.steps, "clocks": clocks,
        "step_ms_min": min(ms), "step_ms_median": statistics.median(ms)}), flush=True)


def run_gptq2d(args) -> None:
    """GPTQ-2D two-sided rounding (GPTQ-2D summary, method steps 1-3): a batch of 148
    problems of 128 x 128 (one CTA per problem, one per SM), fp64, sharing U_left and
    U_right; X ~ 3 N(0, 1).  Roofline: fp64 FMA issue (148 SMs x 64 fp64 FMA per clock x
    1965 MHz) over the algorithmic flops (the dot product of each entry with its column of
    U_left, i + 1 terms, and the push of its error along its row, n - j terms)."""
    import numpy as np
    import torch

    from post_weight_quantization_14_b200 import gptq as G

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    m = n = 128
    batch = 148
    rng = np.random.default_rng(11)

    def spd(k):
        a = rng.standard_normal((k, k)) + 2.0 * np.eye(k)
        return a.T @ a + 0.1 * np.eye(k)

    def upper_factor_of_inverse(h):   # U with U^T U = h^-1 (plain numpy; inputs only)
        return np.linalg.cholesky(np.linalg.inv(h)).T.copy()

    UL = upper_factor_of_inverse(spd(m))
    UR = upper_factor_of_inverse(spd(n))
    X = rng.standard_normal((batch, m, n)) * 3.0
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    Xd, ULd, URd = t(X), t(UL), t(UR)
    Z = torch.empty((batch, m, n), dtype=torch.int32, device=dev)
    ws = torch.empty(G.lib().gptq_2d_workspace_bytes(m, n, batch), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        G.gptq_2d_round(Xd, ULd, URd, Z, workspace=ws)
    G.gptq_sync_status()
    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        flush.fill_(1)
        a.record(stream)
        G.gptq_2d_round(Xd, ULd, URd, Z, workspace=ws)
        b.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    G.gptq_sync_status()
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    fma = batch * (n * m * (m + 1) / 2 + m * n * (n + 1) / 2)
    achieved = 2.0 * fma / (ms / 1e3) / 1e12
    peak = 148 * 64 * 2 * 1.965e9 / 1e12

    # end to end: X in from pinned host memory, Z back to pinned host memory
    X_host = torch.from_numpy(X).pin_memory()
    Z_host = torch.empty((batch, m, n), dtype=torch.int32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(e2e_steps):
        Xd.copy_(X_host, non_blocking=True)
        G.gptq_2d_round(Xd, ULd, URd, Z, workspace=ws)
        Z_host.copy_(Z, non_blocking=True)
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ea.elapsed_time(eb) / e2e_steps

    cpu = None
    if not args.no_cpu_baseline:
        from oracle import gptq_oracle as O
        t0 = time.perf_counter()
        O.gptq2d_antidiagonal(X[0], UL, UR)
        secs = time.perf_counter() - t0
        cpu = {"value": 1.0 / secs, "unit": "problems/s", "cores": os.cpu_count(), "kind": "oracle",
               "sample": "one of the 148 problems (the oracle's anti-diagonal route, fp64 numpy)"}
    line = {"metric": "GPTQ-2D two-sided rounding of 148 problems of 128 x 128 (fp64)", "value": batch / (ms / 1e3),
            "unit": "problems/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "gptq2d: 148 problems of 128x128, X ~ 3 N(0,1), shared U_left, U_right",
                       "l2": "flushed (256 MB write) before every step, outside the step events"},
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "traffic": None, "note": "fp64 FMA issue: 148 SMs x 64 FMA/clock x 1965 MHz (derived); the "
                                                  "kernel walks 255 anti-diagonals with a CTA barrier after each"},
            "cpu_baseline": cpu,
            "e2e": {"value": batch / (e2e_ms / 1e3), "unit": "problems/s", "h2d_bytes_per_step": int(X.nbytes),
                    "d2h_bytes_per_step": int(batch * m * n * 4)},
            "gpu_launches": 2 * args.steps, "clocks": clocks}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="attn", choices=["attn", "stack7b", "dqgemm", "gptq2d"])
    ap.add_argument("--shared-input", action="store_true",
                    help="stack7b: q/k/v and gate/up share one H and U per group (one input each)")
    ap.add_argument("--desc-act", type=int, default=0, choices=[0, 1, 2],
                    help="activation ordering: 0 natural column order, 1 ascending, 2 descending sum of |x|")
    ap.add_argument("--timeline", default="",
                    help="write the per-launch timeline of the instrumented steps (JSON) to this file")
    ap.add_argument("--rank-probe", action="store_true",
                    help="launch check only: the ranks join a gloo group and rank 0 reports the world size")
    args = ap.parse_args()

    world_env = os.environ.get("WORLD_SIZE")
    if args.gpus > 1 and world_env is None:
        # started without torchrun: become N ranks, one per GPU, and return their status
        cmd = relaunch_command(sys.argv[1:], args.gpus, free_port())
        env = dict(os.environ, MASTER_ADDR="127.0.0.1")
        sys.exit(subprocess.call(cmd, env=env))
    world = int(world_env or "1")
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}\n")
        sys.exit(2)
    if args.rank_probe:
        rank_probe(world, rank)
        return
    if args.workload == "stack7b":
        run_stack(args)
        return
    if args.workload == "gptq2d":
        return run_gptq2d(args)
    if args.workload == "dqgemm":
        run_dqgemm(args)
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_gpu(args, world, rank, local)


def run_gpu(args, world: int, rank: int, local: int) -> None:
    import numpy as np
    import torch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from post_weight_quantization_14_b200 import gptq as G
    from post_weight_quantization_14_b200 import inputs as I

    layer = I.make_layer("attn", seed=layer_seed(rank))
    cfg = G.make_config(BITS, GROUP, SYM, 128, 0.01, args.desc_act)
    W0 = torch.from_numpy(layer.W).to(dev)
    W = torch.empty_like(W0)
    X = torch.from_numpy(layer.X_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    bufs = G.LayerBuffers(D_OUT, D_IN, N_TOK, torch.bfloat16, cfg, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(marks=None):
        # the three stages of G.quantize_layer, with optional events between them
        G.gptq_hessian_accumulate(X, bufs.H, accumulate=False, workspace=bufs.ws)
        if cfg.desc_act:
            G.gptq_act_sum_accumulate(X, bufs.act)
            G.gptq_act_order(bufs.act, cfg.desc_act, bufs.perm, bufs.rank)
        if marks:
            marks[0].record(stream)
        # enqueued without host synchronisation (errors are read once after the timed steps)
        G.gptq_prepare_hinv_async(bufs.H, bufs.U, cfg.damp_rel, workspace=bufs.ws, lam=bufs.lam,
                                  perm=bufs.perm if cfg.desc_act else None)
        if marks:
            marks[1].record(stream)
        if cfg.desc_act:
            G.gptq_quantize_layer_act_order(W, bufs.U, bufs.perm, cfg, bufs.qweight, bufs.scales, bufs.qzeros,
                                            bufs.g_idx, bufs.err_sq, workspace=bufs.ws)
        else:
            G.gptq_quantize_layer(W, bufs.U, cfg, bufs.qweight, bufs.scales, bufs.qzeros, bufs.err_sq,
                                  workspace=bufs.ws)

    for _ in range(args.warmup):
        W.copy_(W0)
        step()
    G.gptq_sync_status()

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    marks = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for (a, b), m in zip(evs, marks):
        W.copy_(W0)
        flush.fill_(1)
        a.record(stream)
        step(m)
        b.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    G.gptq_sync_status()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    # stage times of the timed steps (events between the three C-ABI calls)
    stage_timed = {"hessian": statistics.median(a.elapsed_time(m[0]) for (a, _), m in zip(evs, marks)),
                   "prepare_hinv": statistics.median(m[0].elapsed_time(m[1]) for m in marks),
                   "quantize": statistics.median(m[1].elapsed_time(b) for (_, b), m in zip(evs, marks))}
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, D_OUT * D_IN, args.steps, total_ms)

    # per-kernel times (instrumented steps; every launch bracketed by CUDA events on its stream)
    G.gptq_timing_enable(True)
    G.gptq_timing_report()
    reps = 3
    for _ in range(reps):  # instrumented steps (not part of the timed region)
        W.copy_(W0)
        flush.fill_(1)
        step()
    kt = G.gptq_timing_report()
    timeline = G.gptq_timing_timeline()
    G.gptq_timing_enable(False)
    if args.timeline:
        with open(args.timeline, "w") as f:
            json.dump(timeline, f)
    launches_per_step = sum(c for c, _ in kt.values()) / reps
    kernel_ms = {k: ms / reps for k, (c, ms) in kt.items()}
    kernel_launches = {k: c // reps for k, (c, ms) in kt.items()}

    hbm, bf16, bf16_sus, peak_kind = peaks()
    tf32 = measure_tf32_tflops(dev)
    roof_all = kernel_rooflines(kernel_ms, kernel_launches, hbm, bf16, peak_kind, tf32)
    stage_ms = {"hessian": kernel_ms.get("hessian_syrk", 0) + kernel_ms.get("transpose_x", 0)
                + sum(kernel_ms.get(k, 0) for k in ACT_KERNELS),
                "prepare_hinv": sum(v for k, v in kernel_ms.items() if k in CHOL_KERNELS),
                "quantize": sum(kernel_ms.get(k, 0) for k in QUANT_KERNELS)}
    dom = max((k for k in roof_all), key=lambda k: kernel_ms.get(k, 0) + (kernel_ms.get("trailing_update_sb", 0)
                                                                         if k == "trailing_update" else 0))
    roofline = dict(roof_all[dom])
    roofline["kernel"] = dom
    roofline["share_of_step"] = kernel_ms[dom] / max(1e-9, sum(kernel_ms.values()))

    # end-to-end through the public API with host buffers (pinned), copies inside the timed region.
    # Layers are pipelined: layer i+1's inputs go up on one copy stream and layer i-1's outputs
    # come down on another while layer i computes; two sets of device buffers alternate, and
    # events order every reuse (inputs after the compute that read them, outputs after the
    # copy that read them).
    W_host = torch.from_numpy(layer.W).pin_memory()
    X_host = torch.from_numpy(layer.X_bits.view(np.int16)).pin_memory()
    slots = []
    for _ in range(2):
        b_ = G.LayerBuffers(D_OUT, D_IN, N_TOK, torch.bfloat16, cfg, dev)
        slots.append(dict(
            bufs=b_, W=torch.empty_like(W0), X=torch.empty(X_host.shape, dtype=torch.int16, device=dev),
            qw=torch.empty(b_.qweight.shape, dtype=torch.int32).pin_memory(),
            sc=torch.empty(b_.scales.shape, dtype=torch.float16).pin_memory(),
            qz=torch.empty(b_.qzeros.shape, dtype=torch.int32).pin_memory(),
            gi=torch.empty((D_IN,), dtype=torch.int32).pin_memory(),
            ev_in=torch.cuda.Event(), ev_done=torch.cuda.Event(), ev_out=torch.cuda.Event()))
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e2e_steps = max(3, min(args.steps, 30))

    def h2d(sl, after=None):
        with torch.cuda.stream(up):
            if after is not None:
                up.wait_event(after)
            sl["W"].copy_(W_host, non_blocking=True)
            sl["X"].copy_(X_host, non_blocking=True)
            sl["ev_in"].record(up)

    def e2e_run(nsteps):
        h2d(slots[0])
        pending_out = [False, False]
        for i_ in range(nsteps):
            sl = slots[i_ % 2]
            if i_ + 1 < nsteps:   # next layer's inputs, once the layer that last read that slot is done
                nxt = slots[(i_ + 1) % 2]
                h2d(nxt, nxt["ev_done"] if i_ >= 1 else None)
            stream.wait_event(sl["ev_in"])
            if pending_out[i_ % 2]:
                stream.wait_event(sl["ev_out"])   # that slot's previous outputs have been copied out
            q = G.quantize_layer(sl["W"], sl["X"].view(torch.bfloat16), buffers=sl["bufs"])
            sl["ev_done"].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(sl["ev_done"])
                sl["qw"].copy_(q.qweight, non_blocking=True)
                sl["sc"].copy_(q.scales, non_blocking=True)
                sl["qz"].copy_(q.qzeros, non_blocking=True)
                if cfg.desc_act:
                    sl["gi"].copy_(q.g_idx, non_blocking=True)
                sl["ev_out"].record(down)
            pending_out[i_ % 2] = True
        for sl in slots:
            stream.wait_event(sl["ev_out"])

    e2e_run(2)   # warm the second set of buffers and the copy streams
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    up.wait_event(ea)
    e2e_run(e2e_steps)
    eb.record(stream)
    torch.cuda.synchronize()
    G.gptq_sync_status()
    e2e_ms = max_over_ranks(ea.elapsed_time(eb), dist, dev)
    e2e_value = job_throughput(world, D_OUT * D_IN, e2e_steps, e2e_ms)
    h2d_bytes = W_host.numel() * 4 + X_host.numel() * 2
    d2h_bytes = (slots[0]["qw"].numel() * 4 + slots[0]["sc"].numel() * 2 + slots[0]["qz"].numel() * 4
                 + (D_IN * 4 if cfg.desc_act else 0))
    # the last layer's outputs as they reached the host equal the device-timed path's
    last = slots[(e2e_steps - 1) % 2]
    e2e_outputs_match = bool(torch.equal(last["qw"], bufs.qweight.cpu()) and torch.equal(last["sc"], bufs.scales.cpu())
                             and torch.equal(last["qz"], bufs.qzeros.cpu()))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, sample, cores = oracle_layer_time(layer)
        cpu = {"value": D_OUT * D_IN / secs, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": bench_config(world, args.desc_act),
                "roofline": roofline,
                "roofline_by_kernel": roof_all,
                "peaks": {"hbm_gbs": hbm, "bf16_tflops": bf16, "kind": peak_kind, "tf32_tflops_measured": tf32,
                          "tf32x3_tflops": (tf32 / 3.0) if tf32 else None},
                "e2e_roofline": {"bound_ms": END_TO_END_BOUND_MS, "frac": END_TO_END_BOUND_MS / ms_per_step},
                "stage_ms": stage_timed,
                "stage_ms_instrumented": stage_ms,
                "kernel_ms_per_step": kernel_ms,
                "kernel_launches_per_step": kernel_launches,
                "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d_bytes,
                        "d2h_bytes_per_step": d2h_bytes, "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                        "pipelined": "layer i+1 H2D and layer i-1 D2H on two copy streams beside layer i",
                        "outputs_match_device_path": e2e_outputs_match},
                "gpu_launches": int(round(launches_per_step * args.steps)),
                "clocks": clocks,
                "step_ms_min": min(step_ms), "step_ms_median": statistics.median(step_ms)}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
