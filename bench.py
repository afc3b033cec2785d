#!/usr/bin/env python
"""Benchmark: one CCQ W2A16 MoE FFN layer, decode-sized (32 tokens, hidden 8192, 64 experts of
gate/up 8192x3584x2 and down 3584x8192, all CCQ W2 group 64, top-8 uniform routing with softmax
weights from N(0,1) logits, SiLU-gated, BF16 activations).

A step is one full layer forward through the C ABI (routing, activation packing, gate/up matmul
with the SiLU gate, group sums, down matmul with routing weights, top-k combine) over one batch.
`value` is whole-job tokens/s (every rank runs its own replica of the layer: the path has no
exchange step), timed with CUDA events over exactly --steps steps after --warmup steps, max over
ranks.  `--impl reference` times the CPU oracle on a bounded sample of the same workload.

Launch: python bench.py --gpus N --steps K --warmup W  (N > 1: under torch.distributed.run).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

T, H, I, E, TOPK = 32, 8192, 3584, 64, 8
DISTINCT = 2          # 4-bit-scale format: experts encoded on the host, the rest device copies of them
NOMINAL_HBM_GBS = 8000.0
METRIC = "W2A16 MoE layer tokens/s; packed-weight HBM GB/s (% of 8 TB/s), 1 B200"
WORKLOAD = "moe_ffn_decode_T32_H8192_I3584_E64_top8_ccq_w2_g64"
SCALES = "fp32"       # group scale storage: fp32 (the benchmark format) or q4 (CCQ's 2.06-bpw form)
CODES = "ccq"         # codes: ccq (code cluster), std (plain WINT2-Standard fields, CCQ Table 4), or the
                      # Algorithm 2 formats w275 ((4,3,2), 2.75 bpw) and w25 (hybrid, 2.5 bpw)
EMB_CODES = {"w275": (5, 22), "w25": (6, 20)}  # format constant, code bytes per 64 weights


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-small", action="store_true",
                    help="8 tokens over 16 experts (same tokens per expert, 442 MB of weights): for ncu captures")
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "gemm", "stack"],
                    help="decode: 32 tokens, uniform routing (the headline line); prefill: 4096 tokens, "
                         "Zipf(1.1) routing, 1%% of channels x20 (tcgen05 path, tensor roofline); gemm: one "
                         "dense 8192x8192 W2 linear at --m tokens; stack: 8 MoE layers (2 W4 + 6 W2) at --m tokens")
    ap.add_argument("--m", type=int, default=0, help="tokens for --workload gemm (default 1) / stack (default 32)")
    ap.add_argument("--scales", default="fp32", choices=["fp32", "q4"],
                    help="W2 group scales: fp32 (default) or 4-bit x per-channel super scale (2.06 bpw)")
    ap.add_argument("--codes", default="ccq", choices=["ccq", "std", "w275", "w25"],
                    help="codes: ccq (code cluster, default), std (plain 2-bit WINT2-Standard fields, the "
                         "comparison format of CCQ Table 4), w275 ((4,3,2), 2.75 bpw) or w25 (hybrid "
                         "(3,3,2)+(3,4,2), 2.5 bpw), the last two with the scale in the codes (Algorithm 2); "
                         "all but ccq take --scales fp32 only")
    ap.add_argument("--shape", default="8192x8192",
                    help="--workload gemm: input x output size KxN (CCQ Table 4: 4096x4096, 4096x1024, "
                         "8192x8192, 8192x1024)")
    args = ap.parse_args()
    global T, E, WORKLOAD, SCALES, CODES
    SCALES = args.scales
    CODES = args.codes
    if CODES != "ccq" and SCALES != "fp32":
        ap.error("--scales q4 applies to --codes ccq only")
    if args.workload == "prefill":
        T = 4096
        WORKLOAD = "moe_ffn_prefill_T4096_zipf1.1_H8192_I3584_E64_top8_ccq_w2_g64"
    if args.profile_small:
        T, E = (8, 16) if args.workload == "decode" else (512, 16)
    if SCALES == "q4":
        WORKLOAD = WORKLOAD.replace("ccq_w2_g64", "ccq_w2_g64_q4scale")
    if CODES == "std":
        WORKLOAD = WORKLOAD.replace("ccq_w2_g64", "std_w2_g64")
    if CODES == "w275":
        WORKLOAD = WORKLOAD.replace("ccq_w2_g64", "ccq_w275_432_g64")
    if CODES == "w25":
        WORKLOAD = WORKLOAD.replace("ccq_w2_g64", "ccq_w25_hybrid_g64")
    return args


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def replica_seed(base: int, rank: int) -> int:
    """Seed of a rank's replica inputs (every rank times its own copy of the layer)."""
    return base + 17 * rank


def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's time: the job's time for replicas that run concurrently."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's step time."""
    return world * tokens / (ms_per_step * 1e-3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        # the timed region is seconds of back-to-back steps under the power cap: the sustained
        # figure is the matching denominator (the burst one is reported beside it)
        return float(d["bf16_tflops_sustained"]), "measured bf16_tflops_sustained", float(d["bf16_tflops"])
    return 1400.0, "fallback (sustained)", 1590.0


# DRAM bytes (read + write) per touched expert of the fused decode launch, from the ncu capture of
# the same kernel on the 16-expert small case (profiles/decode_gemm_w2_moe_decode_T8_E16_full.md:
# 459.4 MB over 16 experts); each expert's weights cost the same bytes at any expert count, so the
# full workload's traffic is this times the touched experts.  Retake the capture (and update this
# figure) whenever the kernel changes.
FUSED_DECODE_DRAM_BYTES_PER_EXPERT = 459_449_856 / 16


def config_dict():
    prefill = WORKLOAD.startswith("moe_ffn_prefill")
    return {
        "workload": WORKLOAD,
        "tokens": T, "hidden": H, "intermediate": I, "experts": E, "topk": TOPK,
        "weight_format": ("WINT2-Standard plain 2-bit fields, 4 weights/byte, fp32 group-64 scales"
                          if CODES == "std" else
                          "CCQ (4,3,2), 22 one-byte codes per 64 weights, 4-bit scale in the last code x fp32 "
                          "per-channel super scale (2.75 bpw)" if CODES == "w275" else
                          "CCQ hybrid (3,3,2)+(3,4,2), ten 16-bit words per 64 weights, 13-bit scale in the last "
                          "word x fp32 per-channel super scale (2.5 bpw)" if CODES == "w25" else
                          "CCQ (6,4,3) code cluster, 4 weights/byte, " + (
                              "4-bit group-64 scales x fp32 per-channel super scale (2.06 bpw)" if SCALES == "q4"
                              else "fp32 group-64 scales")),
        "routing": ("Zipf(1.1) expert popularity, top-8 by Gumbel-max; " if prefill else "uniform distinct top-8, ")
                   + "softmax of N(0,1) logits",
        "activations": "BF16 N(0,1)" + (", 1% of channels x20" if prefill else ""),
        "weights": (f"N(0,0.02) encoded by ccq_encode_host_q4 for {DISTINCT} experts, copied to all {E}"
                    if SCALES == "q4" else
                    f"N(0,0.02) per expert (seeded device RNG), all {E} quantized by ccq_quantize_std_device"
                    if CODES == "std" else
                    f"N(0,0.02) (seeded device RNG) encoded by ccq_encode_emb_device for {DISTINCT} experts, "
                    f"copied to all {E}" if CODES in EMB_CODES else
                    f"N(0,0.02) per expert (seeded device RNG), all {E} encoded by ccq_encode_device"),
        "l2": "inputs larger than L2: ~1.74 GB of packed weights touched per step vs 126 MB L2",
        "parallelism": "replicas",
    }


# ------------------------------------------------------------------------------------------------
# inputs
# ------------------------------------------------------------------------------------------------
def make_layer_device(ccq, torch, device, seed_base: int = 3100):
    """Every expert its own N(0, 0.02) weights (seeded device RNG), encoded by ccq_encode_device
    (or, for the WINT2-Standard codes, quantized by ccq_quantize_std_device)."""
    std = CODES == "std"
    if CODES in EMB_CODES:
        fmt, gb = EMB_CODES[CODES]

        def stack_emb(n, k, seed):
            codes = torch.empty((E * n, k // 64 * gb), dtype=torch.uint8, device=device)
            sup = torch.empty((E * n,), dtype=torch.float32, device=device)
            g = torch.Generator(device=device)
            # the exhaustive code search costs seconds per expert: DISTINCT experts are encoded and
            # copied into every slot (each slot its own memory; decode cost does not depend on values)
            for e in range(E):
                if e < DISTINCT:
                    g.manual_seed(seed + e)
                    w = torch.randn((n, k), generator=g, device=device, dtype=torch.float32) * 0.02
                    c, su = ccq.ccq_encode_emb_device(fmt, w)
                else:
                    d = e % DISTINCT
                    c, su = codes[d * n:(d + 1) * n], sup[d * n:(d + 1) * n]
                codes[e * n:(e + 1) * n].copy_(c)
                sup[e * n:(e + 1) * n].copy_(su)
            return ccq.CcqWeight(fmt, n, k, codes, None, experts=E, device=device, super_scale=sup)

        return stack_emb(2 * I, H, seed_base), stack_emb(H, I, seed_base + 100)

    def stack(n, k, seed):
        codes = torch.empty((E * n, k // 4), dtype=torch.uint8, device=device)
        scales = torch.empty((E * n, k // 64), dtype=torch.float32, device=device)
        alpha = None if std else torch.empty((E * n,), dtype=torch.float32, device=device)
        beta = None if std else torch.empty((E * n,), dtype=torch.float32, device=device)
        ws = None if std else ccq.workspace(ccq._lib.ccq_encode_device_workspace_size(n, k), device)
        g = torch.Generator(device=device)
        for e in range(E):
            g.manual_seed(seed + e)
            w = torch.randn((n, k), generator=g, device=device, dtype=torch.float32) * 0.02
            if std:
                c, s = ccq.ccq_quantize_std_device(w)
            else:
                c, s, a, b = ccq.ccq_encode_device(w, 64, 0, ws=ws)
                alpha[e * n:(e + 1) * n].copy_(a)
                beta[e * n:(e + 1) * n].copy_(b)
            codes[e * n:(e + 1) * n].copy_(c)
            scales[e * n:(e + 1) * n].copy_(s)
        fmt = ccq.CCQ_FMT_W2_STD_G64 if std else ccq.CCQ_FMT_W2_CCQ_G64
        return ccq.CcqWeight(fmt, n, k, codes, scales, alpha, beta, experts=E, device=device)

    return stack(2 * I, H, seed_base), stack(H, I, seed_base + 100)


def make_layer(ccq, torch, device):
    import synth

    q4 = SCALES == "q4"
    if not q4:
        return make_layer_device(ccq, torch, device)

    def enc(rows, cols, seed):
        w = synth.weights_normal(rows, cols, seed)
        if q4:
            c, sq, sup, a, b, _ = ccq.ccq_encode_host_q4(w, 64, 0, 0)
            return c, sq, a, b, sup
        c, s, a, b, _ = ccq.ccq_encode_host(w, 64, 0, 0)
        return c, s, a, b, None

    parts13 = [enc(2 * I, H, 3100 + e) for e in range(DISTINCT)]
    parts2 = [enc(H, I, 3200 + e) for e in range(DISTINCT)]

    def stack(parts, n, k):
        codes = torch.empty((E * n, k // 4), dtype=torch.uint8, device=device)
        scales = (torch.empty((E * n, k // 128), dtype=torch.uint8, device=device) if q4 else
                  torch.empty((E * n, k // 64), dtype=torch.float32, device=device))
        alpha = torch.empty((E * n,), dtype=torch.float32, device=device)
        beta = torch.empty((E * n,), dtype=torch.float32, device=device)
        sup = torch.empty((E * n,), dtype=torch.float32, device=device) if q4 else None
        dev = [tuple(None if a is None else torch.from_numpy(a).to(device) for a in p) for p in parts]
        for e in range(E):
            c, s, a, b, su = dev[e % len(dev)]
            codes[e * n:(e + 1) * n].copy_(c)
            scales[e * n:(e + 1) * n].copy_(s)
            alpha[e * n:(e + 1) * n].copy_(a)
            beta[e * n:(e + 1) * n].copy_(b)
            if q4:
                sup[e * n:(e + 1) * n].copy_(su)
        if q4:
            return ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64_Q4SCALE, n, k, codes, None, alpha, beta, experts=E,
                                 device=device, scale_q4=scales, super_scale=sup)
        return ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, n, k, codes, scales, alpha, beta, experts=E, device=device)

    W13 = stack(parts13, 2 * I, H)
    W2 = stack(parts2, H, I)
    return W13, W2


def touched_bytes(ids):
    """Algorithmic packed-weight bytes of one step: codes + scales + per-row constants (alpha, beta;
    q4: and the super scale; std: none) of the touched experts."""
    if CODES == "std":
        per13 = 2 * I * (H // 4) + 2 * I * (H // 64) * 4
        per2 = H * (I // 4) + H * (I // 64) * 4
    elif CODES in EMB_CODES:
        gb = EMB_CODES[CODES][1]
        per13 = 2 * I * ((H // 64) * gb + 4)
        per2 = H * ((I // 64) * gb + 4)
    elif SCALES == "q4":
        per13 = 2 * I * (H // 4) + 2 * I * (H // 128) + 2 * I * 12
        per2 = H * (I // 4) + H * (I // 128) + H * 12
    else:
        per13 = 2 * I * (H // 4) + 2 * I * (H // 64) * 4 + 2 * I * 8
        per2 = H * (I // 4) + H * (I // 64) * 4 + H * 8
    ne = len(set(int(v) for v in np.asarray(ids).ravel()))
    return ne * per13, ne * per2, ne


# ------------------------------------------------------------------------------------------------
# clocks
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # raw nvidia-smi samples; the JSON line carries their summary
        log_dir = os.environ.get("CCQ_BENCH_LOG_DIR", os.path.join(ROOT, "bench_logs"))
        self.path = os.path.join(log_dir, f"clocks_rank{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the same layer
# ------------------------------------------------------------------------------------------------
_ORACLE_INPUTS = None


def _oracle_inputs():
    global _ORACLE_INPUTS
    if _ORACLE_INPUTS is None:
        import synth

        x = synth.activations(T, H, 3302)
        ids, rw = synth.routing_uniform(T, E, TOPK, 3303)
        w13 = synth.w2_format_random(2 * I, H, 3304)
        w2 = synth.w2_format_random(H, I, 3305)
        _ORACLE_INPUTS = (synth.bf16_bits(x), ids, rw, w13, w2)
    return _ORACLE_INPUTS


def oracle_sample(n_experts: int = 1, row_frac: float = 1.0):
    """Time the oracle on `n_experts` experts of the decode layer: decode their weights (the first
    `row_frac` of the rows of each projection) and run every (token, expert) pair routed to them
    through the fp64 expert FFN on those rows; scale to the whole layer by the touched-expert count
    and 1/row_frac."""
    import oracle

    xb, ids, rw, (c13, s13, a13, b13), (c2, s2, a2, b2) = _oracle_inputs()
    touched = sorted(set(int(v) for v in ids.ravel()))
    rg = max(1, int(round(row_frac * I)))   # gate rows, and the same number of up rows
    r2 = max(16, int(round(row_frac * H)))  # down rows
    g13 = np.concatenate([np.arange(rg), I + np.arange(rg)])
    r13 = 2 * rg
    pairs = 0
    t0 = time.perf_counter()
    for e in touched[:n_experts]:
        d13 = oracle.dequant_w2(c13[g13], s13[g13], a13[g13], b13[g13])
        d2 = oracle.dequant_w2(c2[:r2], s2[:r2], a2[:r2], b2[:r2])
        toks = [t for t in range(T) if e in ids[t]]
        pairs += len(toks)
        gu = oracle.gemm_f64(xb[toks], d13)                       # gate | up rows of the slice
        h = oracle.silu_f64(gu[:, :r13 // 2]) * gu[:, r13 // 2:]
        hb = oracle.bf16_bits(h.astype(np.float32))
        out = oracle.gemm_f64(hb, np.ascontiguousarray(d2[:, :r13 // 2]))
        del out
    dt = time.perf_counter() - t0
    frac = min(1.0, (r13 * H + r2 * I) / (3.0 * I * H))  # share of the expert's weights sampled
    layer_s = dt * len(touched) / n_experts / frac
    cores = os.cpu_count() or 1
    sample = (f"{n_experts} of {len(touched)} touched experts, {100 * frac:.1f}% of their weight rows "
              f"({pairs} of {T * TOPK} token-expert pairs): oracle decode + fp64 expert FFN, "
              f"scaled by touched experts and rows")
    return T / layer_s, cores, sample, dt


# ------------------------------------------------------------------------------------------------
# reference arm (the oracle, on host cores)
# ------------------------------------------------------------------------------------------------
def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle

    oracle.build()
    # size each step so the whole run takes about 90 s of host time
    _, _, _, dt_full = oracle_sample(1, 0.05)
    per_step = 90.0 / max(1, args.warmup + args.steps)
    frac = float(min(1.0, max(0.002, 0.05 * per_step / max(dt_full, 1e-6))))
    vals = []
    for i in range(args.warmup + args.steps):
        v, cores, sample, dt = oracle_sample(1, frac)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * T / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------
def run_ours(args, rank, world, local):
    import torch

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        pg = dist
    import extreme_bit_weight_b200 as ccq
    import synth

    # CPU baseline first (rank 0, N = 1 only), before any large GPU allocation
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        oracle.build()
        v, cores, sample, dt = oracle_sample(16)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}

    W13, W2 = make_layer(ccq, torch, device)
    prefill = args.workload == "prefill"
    x_host = synth.activations(T, H, replica_seed(3002, rank), outlier_frac=0.01 if prefill else 0.0)
    if prefill:
        ids_np, rw_np = synth.routing_zipf(T, E, TOPK, replica_seed(3003, rank), s=1.1)
    else:
        ids_np, rw_np = synth.routing_uniform(T, E, TOPK, replica_seed(3003, rank))
    x = x_host.to(device)
    ids = torch.from_numpy(ids_np).to(device)
    rw = torch.from_numpy(rw_np).to(device)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    ws = ccq.workspace(ccq.ccq_moe_workspace_size(T, TOPK, H, I, E), device)
    stream = torch.cuda.current_stream(device)

    def step():
        ccq.ccq_moe_w2a16_forward(W13, W2, x, ids, rw, y=y, ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    assert ccq.ccq_check_device_error(ws, stream) == ccq.CCQ_OK

    # ---- device-timed region: exactly K steps, events around every step's kernels ----
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ccq.CCQ_MOE_TRACE_POINTS)] for _ in range(K)]
    for row in evs:  # torch creates an event on its first record; libccq re-records the same handles
        for ev in row:
            ev.record(stream)
    clocks = ClockSampler(local)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(device)
    clocks.start()
    time.sleep(0.3)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(K):
        ccq.ccq_moe_w2a16_forward_traced(W13, W2, x, ids, rw, y, ws, evs[k], stream=stream)
    stop.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    if pg:
        pg.barrier()
    total_ms = start.elapsed_time(stop)
    gemm1_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    gemm2_ms = statistics.mean(e[4].elapsed_time(e[5]) for e in evs)
    # the decode path may run both projections as one launch: then events 3, 4, 5 are recorded
    # back to back and the "down" interval is only event overhead
    fused = (not prefill) and gemm2_ms < 0.02 * gemm1_ms
    total_ms = max_over_ranks(total_ms, pg, device)
    ms_per_step = total_ms / K
    value = job_tokens_per_s(world, T, ms_per_step)

    # ---- end to end: pinned host inputs in, result out, through the same public call ----
    xp = x_host.pin_memory()
    idp = torch.from_numpy(ids_np).pin_memory()
    rwp = torch.from_numpy(rw_np).pin_memory()
    yp = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    K2 = max(1, min(K, 500))

    def e2e_step():
        x.copy_(xp, non_blocking=True)
        ids.copy_(idp, non_blocking=True)
        rw.copy_(rwp, non_blocking=True)
        step()
        yp.copy_(y, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(device)
    if pg:
        pg.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(K2):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = a.elapsed_time(b) / K2
    e2e_ms = max_over_ranks(e2e_ms, pg, device)
    h2d = xp.numel() * 2 + idp.numel() * 4 + rwp.numel() * 4
    d2h = yp.numel() * 2

    b13, b2, ne = touched_bytes(ids_np)
    hbm, src = peaks()
    ach13 = b13 / (gemm1_ms * 1e-3) / 1e9
    layer_gbs = (b13 + b2) / (ms_per_step * 1e-3) / 1e9
    valid_pairs = int(np.sum(ids_np >= 0))
    flops13 = 2.0 * valid_pairs * (2 * I) * H
    flops2 = 2.0 * valid_pairs * H * I
    roofline_tensor = None
    if prefill:
        tf, tsrc, tf_burst = tensor_peak()
        ach_tf = flops13 / (gemm1_ms * 1e-3) / 1e12
        roofline_tensor = {"bound": "tensor", "kernel": "tc_gemm_w2_kernel (gate/up, SiLU epilogue)",
                           "achieved": ach_tf, "peak": tf, "peak_source": tsrc,
                           "unit": "TFLOP/s", "frac": ach_tf / tf, "frac_of_burst": ach_tf / tf_burst,
                           "traffic": None,
                           "launch_ms": gemm1_ms, "algorithmic_flops_per_launch": flops13,
                           "down_kernel": {"achieved": flops2 / (gemm2_ms * 1e-3) / 1e12, "launch_ms": gemm2_ms,
                                           "algorithmic_flops_per_launch": flops2},
                           "layer_tflops": (flops13 + flops2) / (ms_per_step * 1e-3) / 1e12}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(),
        "packed_weight_gbs": layer_gbs, "packed_weight_pct_of_8tbs": 100.0 * layer_gbs / NOMINAL_HBM_GBS,
        "touched_experts": ne,
        "roofline": roofline_tensor or (
            {"bound": "hbm", "kernel": "decode_gemm_w2_kernel (fused MoE: gate/up + SiLU, then down)",
             "achieved": (b13 + b2) / (gemm1_ms * 1e-3) / 1e9, "peak": hbm, "peak_source": f"{src} hbm_gbs (copy)",
             "unit": "GB/s", "frac": (b13 + b2) / (gemm1_ms * 1e-3) / 1e9 / hbm,
             "traffic": FUSED_DECODE_DRAM_BYTES_PER_EXPERT * ne if (SCALES, CODES) == ("fp32", "ccq") else None,
             "traffic_source": "ncu dram__bytes_read+write of the 16-expert capture, scaled by touched experts",
             "launch_ms": gemm1_ms, "algorithmic_bytes_per_launch": b13 + b2} if fused else
            {"bound": "hbm", "kernel": "decode_gemm_w2_kernel (gate/up, SiLU epilogue)",
             "achieved": ach13, "peak": hbm, "peak_source": f"{src} hbm_gbs (copy)", "unit": "GB/s",
             "frac": ach13 / hbm, "traffic": None, "launch_ms": gemm1_ms,
             "algorithmic_bytes_per_launch": b13,
             "down_kernel": {"achieved": b2 / (gemm2_ms * 1e-3) / 1e9, "launch_ms": gemm2_ms,
                             "algorithmic_bytes_per_launch": b2}}),
        "cpu_baseline": cpu,
        "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        # our kernels per step: route, pack, matmul(s), [group sums], combine
        "gpu_launches": (4 if fused else 6) * K,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()


# ------------------------------------------------------------------------------------------------
# side workloads: the dense linear and the mixed W4/W2 layer stack (reported per M, not headline)
# ------------------------------------------------------------------------------------------------
def _timed(torch, device, stream, step, K, W):
    for i in range(W):
        step(i)
    torch.cuda.synchronize(device)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(K):
        step(W + i)
    b.record(stream)
    torch.cuda.synchronize(device)
    return a.elapsed_time(b) / K, clocks.stop()


def run_gemm(args, rank, world, local):
    """y = x W^T at M tokens, K x N from --shape (default 8192 x 8192), CCQ W2 g64 or the
    WINT2-Standard codes.  The weight (21.04 MB at 8192 x 8192) is smaller than L2, so the timed
    calls rotate over enough device copies to exceed twice the L2 size."""
    import torch

    import extreme_bit_weight_b200 as ccq
    import synth

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    M = args.m or 1
    KD, ND = (int(v) for v in args.shape.lower().split("x"))
    w = synth.weights_normal(ND, KD, 4100)
    if CODES == "std":
        c, sc = (t.cpu().numpy() for t in ccq.ccq_quantize_std_device(torch.from_numpy(w).to(device)))
        per_copy = c.nbytes + sc.nbytes
        mk = lambda: ccq.CcqWeight(ccq.CCQ_FMT_W2_STD_G64, ND, KD, c, sc, device=device)
    elif CODES in EMB_CODES:
        fmt = EMB_CODES[CODES][0]
        c, su = (t.cpu().numpy() for t in ccq.ccq_encode_emb_device(fmt, torch.from_numpy(w).to(device)))
        per_copy = c.nbytes + su.nbytes
        mk = lambda: ccq.CcqWeight(fmt, ND, KD, c, None, device=device, super_scale=su)
    elif SCALES == "q4":
        c, sq, sup, al, be, _ = ccq.ccq_encode_host_q4(w, 64, 0, 0)
        per_copy = c.nbytes + sq.nbytes + sup.nbytes + al.nbytes + be.nbytes
        mk = lambda: ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64_Q4SCALE, ND, KD, c, None, al, be, device=device,
                                   scale_q4=sq, super_scale=sup)
    else:
        c, sc, al, be, _ = ccq.ccq_encode_host(w, 64, 0, 0)
        per_copy = c.nbytes + sc.nbytes + al.nbytes + be.nbytes
        mk = lambda: ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, ND, KD, c, sc, al, be, device=device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    R = max(2, -(-2 * l2 // per_copy))
    Ws = [mk() for _ in range(R)]
    x = synth.activations(M, KD, 4101).to(device)
    y = torch.empty((M, ND), dtype=torch.bfloat16, device=device)
    ws = ccq.workspace(max(ccq.ccq_gemm_workspace_size(Ws[0], M), 256), device)
    stream = torch.cuda.current_stream(device)
    ms, clk = _timed(torch, device, stream, lambda i: ccq.ccq_w2a16_gemm(Ws[i % R], x, y=y, ws=ws, stream=stream),
                     args.steps, args.warmup)
    # the same calls captured once in a CUDA graph (one call per weight copy) and replayed: the
    # device time of a call without the host's per-call cost, as a serving loop that captures
    # its decode step would see it
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for i in range(R):
            ccq.ccq_w2a16_gemm(Ws[i], x, y=y, ws=ws, stream=side)
    stream.wait_stream(side)
    g_ms, _ = _timed(torch, device, stream, lambda i: graph.replay(), max(3, args.steps // R), 3)
    graph_us = 1000.0 * g_ms / R
    # end to end: pinned host x in, y out, every call
    xp = x.cpu().pin_memory()
    yp = torch.empty((M, ND), dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(x)

    def e2e(i):
        xd.copy_(xp, non_blocking=True)
        ccq.ccq_w2a16_gemm(Ws[i % R], xd, y=y, ws=ws, stream=stream)
        yp.copy_(y, non_blocking=True)

    e2e_ms, _ = _timed(torch, device, stream, e2e, max(1, args.steps // 4), 3)
    hbm, src = peaks()
    tf, tsrc, tf_burst = tensor_peak()
    flops = 2.0 * M * ND * KD
    tensor = M >= 33  # the tcgen05 kernel's range
    gbs = per_copy / (ms * 1e-3) / 1e9
    roof = ({"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": tf, "peak_source": tsrc,
             "unit": "TFLOP/s", "frac": flops / (ms * 1e-3) / 1e12 / tf} if tensor else
            {"bound": "hbm", "achieved": gbs, "peak": hbm, "peak_source": f"{src} hbm_gbs (copy)", "unit": "GB/s",
             "frac": gbs / hbm})
    roof.update({"kernel": "whole ccq_w2a16_gemm call (" + ("activation packing, tcgen05 kernel, split-K reduce"
                                                            if tensor else
                 "activation packing, decode kernel, split-K reduce") + ")", "traffic": None,
                 "algorithmic_bytes_per_call": per_copy, "algorithmic_flops_per_call": flops})
    fmt_tag = ("std_w2_g64" if CODES == "std" else "ccq_w275_432_g64" if CODES == "w275" else
               "ccq_w25_hybrid_g64" if CODES == "w25" else "ccq_w2_g64" + ("_q4scale" if SCALES == "q4" else ""))
    line = {"metric": f"W2A16 dense linear tokens/s (K={KD}, N={ND})", "value": M / (ms * 1e-3), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "us_per_call": 1000.0 * ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"dense_gemm_M{M}_K{KD}_N{ND}_{fmt_tag}",
                       "m": M, "k": KD, "n": ND,
                       "weights": "N(0,0.02) " + ("quantized by ccq_quantize_std_device" if CODES == "std" else
                                                  "encoded by ccq_encode_emb_device" if CODES in EMB_CODES else
                                                  "encoded by ccq_encode_host" + ("_q4" if SCALES == "q4" else "")),
                       "l2": f"{R} rotating weight copies ({R * per_copy / 1e6:.0f} MB) vs {l2 / 1e6:.0f} MB L2"},
            "packed_weight_gbs": gbs, "roofline": roof,
            "graph": {"us_per_call": graph_us, "value": M / (graph_us * 1e-6), "unit": "tokens/s",
                      "packed_weight_gbs": per_copy / (graph_us * 1e-6) / 1e9,
                      "note": f"{R} calls (one per weight copy) captured in one CUDA graph, replayed"},
            "e2e": {"value": M / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": x.numel() * 2,
                    "d2h_bytes_per_step": y.numel() * 2},
            "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_stack(args, rank, world, local):
    """Eight MoE layers of the decode layer's shape: layers 0-1 with W4 per-channel experts, 2-7 with
    CCQ W2 g64; fresh uniform top-8 routing per layer; x_{l+1} = MoE_l(x_l).  A step is the whole
    stack at M tokens."""
    import torch

    import extreme_bit_weight_b200 as ccq
    import synth

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    M = args.m or 32
    parts = {}

    def w4_layer(seed):
        def q(rows, cols, sd):
            c, s = ccq.ccq_quantize_w4_host(synth.weights_normal(rows, cols, sd))
            return torch.from_numpy(c).to(device), torch.from_numpy(s).to(device)

        if "w4" not in parts:
            parts["w4"] = ([q(2 * I, H, seed + e) for e in range(DISTINCT)], [q(H, I, seed + 50 + e) for e in range(DISTINCT)])
        p13, p2 = parts["w4"]

        def stack(pp, n, k):
            codes = torch.empty((E * n, k // 2), dtype=torch.uint8, device=device)
            scales = torch.empty((E * n,), dtype=torch.float32, device=device)
            for e in range(E):
                codes[e * n:(e + 1) * n].copy_(pp[e % len(pp)][0])
                scales[e * n:(e + 1) * n].copy_(pp[e % len(pp)][1])
            return ccq.CcqWeight(ccq.CCQ_FMT_W4_PER_CHANNEL, n, k, codes, scales, experts=E, device=device)

        return stack(p13, 2 * I, H), stack(p2, H, I)

    def clone(w):  # a layer of its own memory with the same contents
        cp = lambda t: None if t is None else t.clone()
        return ccq.CcqWeight(w.fmt, w.n, w.k, cp(w.codes), cp(w.scales), cp(w.alpha), cp(w.beta),
                             experts=w.experts, device=device, scale_q4=cp(w.scale_q4),
                             super_scale=cp(w.super_scale))

    w2_first = make_layer(ccq, torch, device)
    layers = ([w4_layer(4200) for _ in range(2)] + [w2_first] +
              [(clone(w2_first[0]), clone(w2_first[1])) for _ in range(5)])
    routes = []
    for l in range(8):
        ids_np, rw_np = synth.routing_uniform(M, E, TOPK, 4300 + l)
        routes.append((ids_np, torch.from_numpy(ids_np).to(device), torch.from_numpy(rw_np).to(device)))
    xs = [synth.activations(M, H, 4400).to(device)] + [torch.empty((M, H), dtype=torch.bfloat16, device=device)
                                                       for _ in range(8)]
    ws = ccq.workspace(ccq.ccq_moe_workspace_size(M, TOPK, H, I, E), device)
    stream = torch.cuda.current_stream(device)

    def step(_):
        for l, (w13, w2) in enumerate(layers):
            ccq.ccq_moe_w2a16_forward(w13, w2, xs[l], routes[l][1], routes[l][2], y=xs[l + 1], ws=ws, stream=stream)

    ms, clk = _timed(torch, device, stream, step, args.steps, args.warmup)
    assert ccq.ccq_check_device_error(ws, stream) == ccq.CCQ_OK
    # algorithmic bytes and flops of one step (touched experts of every layer)
    per_w4 = 2 * I * (H // 2) + 2 * I * 4 + H * (I // 2) + H * 4
    per_w2 = sum(touched_bytes(np.zeros((1, 1), dtype=np.int32))[:2])
    nbytes = 0
    for l in range(8):
        ne = len(set(int(v) for v in routes[l][0].ravel()))
        nbytes += ne * (per_w4 if l < 2 else per_w2)
    flops = 8 * 6.0 * M * TOPK * H * I
    hbm, src = peaks()
    tf, tsrc, _ = tensor_peak()
    tensor = M * TOPK / E >= 28  # the tcgen05 kernel's range
    roof = ({"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": tf, "peak_source": tsrc,
             "unit": "TFLOP/s", "frac": flops / (ms * 1e-3) / 1e12 / tf} if tensor else
            {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm, "peak_source": f"{src} hbm_gbs (copy)",
             "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / hbm})
    roof.update({"kernel": "whole 8-layer stack", "traffic": None, "algorithmic_bytes_per_step": nbytes,
                 "algorithmic_flops_per_step": flops})
    line = {"metric": "W2A16/W4A16 8-layer MoE stack tokens/s", "value": M / (ms * 1e-3), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"moe_stack_8layers_M{M}_H8192_I3584_E64_top8_w4x2_w2x6", "m": M,
                       "weights": f"W4: N(0,0.02) quantized by ccq_quantize_w4_host for {DISTINCT} experts, copied "
                                  f"to all {E}; W2: all {E} experts encoded by ccq_encode_device, layers 3-7 "
                                  f"device copies of layer 2",
                       "l2": f"{nbytes / 1e9:.2f} GB of packed weights touched per step vs 126 MB L2"},
            "roofline": roof, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.workload in ("gemm", "stack"):
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the oracle on the "
                                  "decode MoE layer only"}), flush=True)
            return
        (run_gemm if args.workload == "gemm" else run_stack)(args, rank, world, local)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
