"""Benchmark of the DeepSeek-V4 hybrid CSA/HCA attention hot path on B200.

One step = one V4-Flash CSA prefill layer over one sequence of 8192 tokens (bf16, H=64,
c=512, m=4, H_I=64, c_I=128, k=512, w=128, per-head sink):
    compress(main) -> compress(index keys) -> index scores + top-k -> hybrid attention,
all through the library's C ABI (libdsv4.so) on the current stream, inputs resident
in HBM. The L2 is flushed (256 MiB write) before every step, outside the step's events.

Prints one JSON line (rank 0). `--impl reference` times the fp64 CPU oracle instead
(a bounded sample of the same workload on the host cores).

Multi-GPU: the layer has no exchange step at this size, so N GPUs run N independent
replicas (weak scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "flash_csa_prefill"
METRIC = "prefill tokens/s per CSA/HCA layer"
# nominal B200 figures, reported beside the measured denominators: dense bf16 tensor rate and
# the HGX HBM3e bandwidth
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 7700.0
UNIT = "tokens/s"

# DRAM traffic of the attention kernel per launch, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the hash of the attention
# sources it was measured on; reported as null once those sources change.
ATTN_TRAFFIC = {"sources_sha1": "bf087f975892cb2814b868345dd23be8dc40e9c6",
                "bytes_per_launch": 562_292_992 + 496_906_752}
ATTN_SOURCES = ("attn_common.cuh", "attn_tc.cu", "dsv4_common.cuh", "rope.cuh", "tc_common.cuh")


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of the ranks' values (per-rank device times -> the job's time); the value
    itself on one rank. Every rank calls it at the same point."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Units all ranks processed (the same number on each: weak scaling) per second of the
    slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


def _attn_sources_sha1() -> str:
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "compressed_sparse_mqa_dsv4_b200", "csrc")
    for f in ATTN_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def attention_flops(n: int, m: int, k: int, w: int, H: int, c: int) -> float:
    """4*H*c*sum_t N_t with N_t = min(k, floor((t+1)/m)) + min(w, t+1)."""
    tot = 0
    for t in range(n):
        tot += min(k, (t + 1) // m) + min(w, t + 1)
    return 4.0 * H * c * tot


def hca_attention_flops(n: int, m: int, w: int, H: int, c: int) -> float:
    """Dense read: 4*H*c*sum_t (floor((t+1)/m) + min(w, t+1))."""
    tot = 0
    for t in range(n):
        tot += (t + 1) // m + min(w, t + 1)
    return 4.0 * H * c * tot


def index_flops(n: int, m: int, HI: int, cI: int) -> float:
    return 2.0 * HI * cI * sum((t + 1) // m for t in range(n))


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi sampling (200 ms) while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        hi = max(sm)
        loaded = [s for s in sm if s >= 0.5 * hi] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- CUDA arm


def run_cuda(args, rank: int, world: int):
    import torch
    import compressed_sparse_mqa_dsv4_b200 as dsv4
    from workloads import Generator, preset

    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    s = preset(WORKLOAD)
    E = s.n // s.m
    gen = Generator(args.seed + rank)
    C, Z, bias = gen.compressor_inputs(s, "main")
    CI, ZI, biasI = gen.compressor_inputs(s, "index")
    qI, w = gen.index_queries(s)
    Q = gen.queries(s)
    local = gen.local_kv(s)
    sink = gen.sink(s)
    host = dict(C=C, Z=Z, bias=bias, CI=CI, ZI=ZI, biasI=biasI, qI=qI, w=w, Q=Q, local=local,
                sink=sink)
    d = {k: v.to(dev) for k, v in host.items()}
    off = torch.zeros(1, dtype=torch.int64, device=dev)
    pos0 = torch.zeros(1, dtype=torch.int32, device=dev)
    pool = torch.empty(1, E, s.c, dtype=torch.bfloat16, device=dev)
    KI = torch.empty(1, E, s.c_I, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(1, s.n, s.k, dtype=torch.int32, device=dev)
    counts = torch.empty(1, s.n, dtype=torch.int32, device=dev)
    ws = torch.empty(dsv4.dsv4_index_topk_workspace_size(1, s.n, E, s.k), dtype=torch.uint8,
                     device=dev)
    Out = torch.empty_like(d["Q"])
    lse = torch.empty(1, s.n, s.H, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ev = {}

    def step(inp, record=None):
        if record is not None:
            record[0].record(stream)
        dsv4.dsv4_compress(inp["C"], inp["Z"], inp["bias"], s.m, True, out=pool)
        dsv4.dsv4_compress(inp["CI"], inp["ZI"], inp["biasI"], s.m, True, out=KI)
        if record is not None:
            record[1].record(stream)
        dsv4.dsv4_index_topk(inp["qI"], inp["w"], KI.view(E, s.c_I), off, pos0, s.m, s.k, E,
                             idx=idx, counts=counts, workspace=ws)
        if record is not None:
            record[2].record(stream)
        dsv4.dsv4_hybrid_sparse_attn(inp["Q"], pool.view(E, s.c), off, idx, counts,
                                     inp["local"], pos0, s.m, s.w, inp["sink"], O=Out, lse=lse)
        if record is not None:
            record[3].record(stream)

    launches_per_step = 2 + 2 * math.ceil(s.n * ((E + 3) // 4 * 4) * 4 / ws.numel()) + 1

    for _ in range(args.warmup):
        flush.zero_()
        step(d)
    dsv4.dsv4_check_errors()

    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(d, recs[i])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    dsv4.dsv4_check_errors()
    step_ms = [r[0].elapsed_time(r[3]) for r in recs]
    comp_ms = [r[0].elapsed_time(r[1]) for r in recs]
    index_ms = [r[1].elapsed_time(r[2]) for r in recs]
    attn_ms = [r[2].elapsed_time(r[3]) for r in recs]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(s.B * s.n * args.steps, world, total_ms)

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the region
    pinned = {k: v.pin_memory() for k, v in host.items()}
    out_host = torch.empty(Out.shape, dtype=Out.dtype, pin_memory=True)
    lse_host = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_host.numel() * out_host.element_size() + lse_host.numel() * lse_host.element_size()
    e2e_steps = max(1, min(args.steps, 5))
    dd = {k: torch.empty_like(v) for k, v in d.items()}

    def e2e_step():
        for k2, v in pinned.items():
            dd[k2].copy_(v, non_blocking=True)
        step(dd)
        out_host.copy_(Out, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_throughput(s.B * s.n * e2e_steps, world, e2e_ms)

    # ---- roofline of the dominant kernel (attention, tensor-core bound by algorithm)
    peaks, peak_src = _peaks()
    flops = attention_flops(s.n, s.m, s.k, s.w, s.H, s.c)
    attn_avg = sum(attn_ms) / len(attn_ms)
    achieved = flops / (attn_avg / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = None
    if ATTN_TRAFFIC["sources_sha1"] == _attn_sources_sha1():
        traffic = ATTN_TRAFFIC["bytes_per_launch"]
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)/sqrt(dim) activations, N(0,1) gate logits)",
        "config": {"workload": "flash_csa_prefill: V4-Flash CSA layer prefill, bf16, B=1, "
                               "n=8192, H=64, c=512, m=4 (2048 entries), H_I=64, c_I=128, "
                               "k=512, w=128, sink",
                   "tokens_per_step": s.B * s.n, "parallelism": f"replicas x{world}",
                   "l2": "flushed (256 MiB write) before every step, outside the step events"},
        "breakdown_ms": {"compress": round(statistics.mean(comp_ms), 4),
                         "index_topk": round(statistics.mean(index_ms), 4),
                         "attention": round(attn_avg, 4)},
        "roofline": {"kernel": "hybrid_sparse_attn", "bound": "tensor",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_flops_per_launch": flops,
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "frac_of_nominal": round(achieved / NOMINAL_BF16_TFLOPS, 4),
                     "index_topk_tflops": round(index_flops(s.n, s.m, s.H_I, s.c_I) /
                                                (statistics.mean(index_ms) / 1e3) / 1e12, 1)},
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "clocks": clk.summary(),
        "gpu_launches": launches_per_step * args.steps,
    }
    if not args.no_decode:
        res["decode"] = run_decode(args, dev, stream)
    if not args.no_layers:
        res["other_layers"] = {nm: run_layer(args, dev, stream, nm)
                               for nm in ("flash_hca_prefill", "pro_csa_prefill")}
        res["other_layers"]["chunk_prefill"] = run_chunk(args, dev, stream)
    if not args.no_decode:
        try:                                          # last, so that it cannot cost the line
            res["decode"]["state_update"] = run_decode_state(args, dev, stream)
        except Exception as e:                        # noqa: BLE001
            res["decode"]["state_update"] = {"error": str(e)[:300]}
    return res


# ----------------------------------------------------------------------------- decode


def run_decode(args, dev, stream):
    """Batched decode (one query per sequence at t = L - 1): 64 sequences with context
    lengths uniform in [131072, 1048576], V4-Flash shapes, layers alternating CSA (indexer
    top-k over all completed entries, then attention over k + w rows) and HCA (dense read of
    floor(L/128) entries + window). Pools are bf16 and resident in HBM; the two CSA and the
    two HCA layers of a step read the same pools (each pool is far larger than L2, and L2 is
    flushed before every step). Returns the decode record for the JSON line."""
    import torch
    import compressed_sparse_mqa_dsv4_b200 as dsv4
    from workloads import DECODE_BATCH as D
    B, H, c, k, w, HI, cI = D["B"], D["H"], D["c"], D["k"], D["w"], D["H_I"], D["c_I"]
    g = torch.Generator(device="cpu").manual_seed(args.seed + 1)
    L = torch.randint(D["L_lo"], D["L_hi"] + 1, (B,), generator=g)
    E4, E128 = (L // D["m_csa"]).tolist(), (L // D["m_hca"]).tolist()
    off4 = torch.tensor([0] + torch.cumsum(torch.tensor(E4), 0)[:-1].tolist(), dtype=torch.int64, device=dev)
    off128 = torch.tensor([0] + torch.cumsum(torch.tensor(E128), 0)[:-1].tolist(), dtype=torch.int64,
                          device=dev)
    pos0 = (L - 1).to(torch.int32).to(dev)
    gd = torch.Generator(device=dev).manual_seed(args.seed + 2)

    def normal(shape, std):
        t = torch.empty(*shape, dtype=torch.bfloat16, device=dev)
        return t.normal_(0.0, std, generator=gd)

    KI = normal((sum(E4), cI), cI ** -0.5)
    pool4 = normal((sum(E4), c), c ** -0.5)
    pool128 = normal((sum(E128), c), c ** -0.5)
    qI = normal((B, 1, HI, cI), cI ** -0.5)
    wI = torch.rand(B, 1, HI, device=dev, generator=gd)
    Q = normal((B, 1, H, c), c ** -0.5)
    local = normal((B, w, c), c ** -0.5)
    sink = torch.randn(H, device=dev, generator=gd)
    maxE = max(E4)
    ws = torch.empty(dsv4.dsv4_index_topk_workspace_size(B, 1, maxE, k), dtype=torch.uint8, device=dev)
    aws = torch.empty(max(1, dsv4.dsv4_hybrid_sparse_attn_workspace_size(B, 1, H, c)), dtype=torch.uint8,
                      device=dev)
    idx = torch.empty(B, 1, k, dtype=torch.int32, device=dev)
    cnt = torch.empty(B, 1, dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    lse = torch.empty(B, 1, H, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def layer_csa():
        dsv4.dsv4_index_topk(qI, wI, KI, off4, pos0, D["m_csa"], k, maxE, idx=idx, counts=cnt, workspace=ws)
        dsv4.dsv4_hybrid_sparse_attn(Q, pool4, off4, idx, cnt, local, pos0, D["m_csa"], w, sink, O=O,
                                     lse=lse, workspace=aws)

    def layer_hca():
        dsv4.dsv4_hybrid_sparse_attn(Q, pool128, off128, None, None, local, pos0, D["m_hca"], w, None,
                                     O=O, lse=lse, workspace=aws)

    def step():
        for kind in D["layers"]:
            (layer_csa if kind == "csa" else layer_hca)()

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    dsv4.dsv4_check_errors()
    steps = max(1, min(args.steps, 10))
    ts = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    dsv4.dsv4_check_errors()
    ms = statistics.median(ts)
    # algorithmic bytes: index keys + query/weights/indices, selected + window rows, Q and O
    b_csa = sum(e * cI * 2 for e in E4) + B * HI * (cI * 2 + 4) + B * k * 4 \
        + sum(min(k, e) + w for e in E4) * c * 2 + 2 * B * H * c * 2
    b_hca = sum(e + w for e in E128) * c * 2 + 2 * B * H * c * 2
    nbytes = sum(b_csa if kind == "csa" else b_hca for kind in D["layers"])
    peaks, src = _peaks()
    peak = float(peaks["hbm_gbs"])
    gbps = nbytes / (ms / 1e3) / 1e9

    # the same step with the CSA layers' main pool in the production FP8 entry format (448 FP8
    # + 64 bf16 channels, 604 bytes per entry): the selected entries are read in that format
    codes, scales, rope = dsv4.dsv4_quantize_main_kv(pool4.view(-1, c))
    fws = torch.empty(dsv4.dsv4_hybrid_sparse_attn_fp8_workspace_size(B, H, c, k), dtype=torch.uint8,
                      device=dev)

    def layer_csa_fp8():
        dsv4.dsv4_index_topk(qI, wI, KI, off4, pos0, D["m_csa"], k, maxE, idx=idx, counts=cnt, workspace=ws)
        dsv4.dsv4_hybrid_sparse_attn_fp8(Q, codes, scales, rope, off4, idx, cnt, local, pos0, D["m_csa"], w,
                                         sink, O=O, lse=lse, workspace=fws)

    def step_fp8():
        for kind in D["layers"]:
            (layer_csa_fp8 if kind == "csa" else layer_hca)()

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step_fp8()
    dsv4.dsv4_check_errors()
    ts8 = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step_fp8()
        e1.record(stream)
        torch.cuda.synchronize()
        ts8.append(e0.elapsed_time(e1))
    dsv4.dsv4_check_errors()
    ms8 = statistics.median(ts8)
    row8 = (c - 64) + 4 * ((c - 64) // 64) + 64 * 2
    b_csa8 = sum(e * cI * 2 for e in E4) + B * HI * (cI * 2 + 4) + B * k * 4 \
        + sum(min(k, e) for e in E4) * row8 + B * w * c * 2 + 2 * B * H * c * 2
    nbytes8 = sum(b_csa8 if kind == "csa" else b_hca for kind in D["layers"])
    # and with the index keys in their production format too: FP4 (e2m1 + one E4M3 scale per
    # 16, 72 bytes per key), expanded inside the score kernel
    kc, ks = dsv4.dsv4_quantize_fp4(KI)
    qc, qs = dsv4.dsv4_quantize_fp4(qI.reshape(-1, cI))
    qc = qc.view(B, 1, HI, cI // 2)
    ws4 = torch.empty(dsv4.dsv4_index_topk_workspace_size_ex(dsv4.FP4, B, 1, HI, cI, maxE, k, kc.shape[0]),
                      dtype=torch.uint8, device=dev)

    def layer_csa_prod():
        dsv4.dsv4_index_topk(qc, wI, kc, off4, pos0, D["m_csa"], k, maxE, qI_scales=qs, KI_scales=ks,
                             c_I=cI, idx=idx, counts=cnt, workspace=ws4)
        dsv4.dsv4_hybrid_sparse_attn_fp8(Q, codes, scales, rope, off4, idx, cnt, local, pos0, D["m_csa"], w,
                                         sink, O=O, lse=lse, workspace=fws)

    def step_prod():
        for kind in D["layers"]:
            (layer_csa_prod if kind == "csa" else layer_hca)()

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step_prod()
    dsv4.dsv4_check_errors()
    tsp = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step_prod()
        e1.record(stream)
        torch.cuda.synchronize()
        tsp.append(e0.elapsed_time(e1))
    dsv4.dsv4_check_errors()
    msp = statistics.median(tsp)
    key4 = cI // 2 + cI // 16
    b_csap = sum(e * key4 for e in E4) + B * HI * (cI // 2 + cI // 16 + 4) + B * k * 4 \
        + sum(min(k, e) for e in E4) * row8 + B * w * c * 2 + 2 * B * H * c * 2
    nbytesp = sum(b_csap if kind == "csa" else b_hca for kind in D["layers"])
    production = {"what": "the same step with both CSA pools in their production formats: main entries "
                          f"FP8 ({row8} bytes) and index keys FP4 (e2m1 + E4M3 per 16 = {key4} bytes, "
                          "expanded to f16 inside the score kernel); HCA pools bf16",
                  "ms_per_step": round(msp, 4), "bytes_per_step": nbytesp,
                  "achieved_gbs": round(nbytesp / (msp / 1e3) / 1e9, 1),
                  "frac": round(nbytesp / (msp / 1e3) / 1e9 / peak, 4), "steps": steps,
                  "csa_index_key_bytes": {"bf16": int(sum(E4)) * cI * 2, "fp4": int(sum(E4)) * key4}}
    packed = {"what": "the same step with the CSA layers' compressed main pool stored as FP8 entries "
                      f"(448 FP8 + 64 bf16 channels + 7 fp32 scales = {row8} bytes per entry; index keys "
                      "and the HCA pools bf16)",
              "ms_per_step": round(ms8, 4), "bytes_per_step": nbytes8,
              "achieved_gbs": round(nbytes8 / (ms8 / 1e3) / 1e9, 1),
              "frac": round(nbytes8 / (ms8 / 1e3) / 1e9 / peak, 4), "steps": steps,
              "csa_main_pool_bytes": {"bf16": int(sum(E4)) * c * 2, "fp8_entries": int(sum(E4)) * row8}}
    return {"workload": f"batched decode: B={B}, one query per sequence, L ~ U[{D['L_lo']}, {D['L_hi']}] "
                        f"(seeded), H={H}, c={c}, k={k}, w={w}, H_I={HI}, c_I={cI}, layers "
                        f"{'/'.join(D['layers'])} (CSA m=4, HCA m'=128), bf16 pools in HBM",
            "ms_per_step": round(ms, 4), "bytes_per_step": nbytes, "achieved_gbs": round(gbps, 1),
            "peak_gbs": peak, "frac": round(gbps / peak, 4), "peak_source": f"{src} hbm_gbs",
            "frac_of_nominal": round(gbps / NOMINAL_HBM_GBS, 4),
            "steps": steps, "l2": "flushed (256 MiB write) before every step", "packed_pools": packed,
            "production_pools": production}


def run_decode_state(args, dev, stream):
    """Per-token state updates of the batched decode step ("CSA And HCA: Definition, State,
    And Cost Model", s7 steps 1-4) for the same 64 sequences and 4 layers: the ring slot
    write in every layer, the main and index-key compressor states of the CSA layers and the
    main compressor state of the HCA layers, appending the entries that complete at this
    token (L mod m == 0) to the pools. Timed apart from the decode step above."""
    import torch
    import compressed_sparse_mqa_dsv4_b200 as dsv4
    from workloads import DECODE_BATCH as D
    B, c, w, cI = D["B"], D["c"], D["w"], D["c_I"]
    m4, m128 = D["m_csa"], D["m_hca"]
    g = torch.Generator(device="cpu").manual_seed(args.seed + 1)
    L = torch.randint(D["L_lo"], D["L_hi"] + 1, (B,), generator=g)
    E4, E128 = (L // m4).tolist(), (L // m128).tolist()
    off4 = torch.tensor([0] + torch.cumsum(torch.tensor(E4), 0)[:-1].tolist(), dtype=torch.int64,
                        device=dev)
    off128 = torch.tensor([0] + torch.cumsum(torch.tensor(E128), 0)[:-1].tolist(),
                          dtype=torch.int64, device=dev)
    pos = (L - 1).to(torch.int32).to(dev)
    gd = torch.Generator(device=dev).manual_seed(args.seed + 4)

    def normal(*shape):
        return torch.empty(*shape, dtype=torch.bfloat16, device=dev).normal_(0.0, 1.0, generator=gd)

    pool4, KI, pool128 = normal(sum(E4), c), normal(sum(E4), cI), normal(sum(E128), c)
    local = normal(B, w, c)
    tail4 = normal(*dsv4.decode_tail_shape(B, c, m4, True))
    tailI = normal(*dsv4.decode_tail_shape(B, cI, m4, True))
    tail128 = normal(*dsv4.decode_tail_shape(B, c, m128, False))
    kv, C4, Z4 = normal(B, c), normal(B, 2 * c), normal(B, 2 * c)
    CI, ZI, C128, Z128 = normal(B, 2 * cI), normal(B, 2 * cI), normal(B, c), normal(B, c)
    b4 = torch.randn(2, m4, c, device=dev, generator=gd) * 0.1
    bI = torch.randn(2, m4, cI, device=dev, generator=gd) * 0.1
    b128 = torch.randn(1, m128, c, device=dev, generator=gd) * 0.1
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step_separate():
        for kind in D["layers"]:
            dsv4.dsv4_ring_write(kv, local, pos)
            if kind == "csa":
                dsv4.dsv4_compress_decode(C4, Z4, b4, tail4, pool4, off4, pos, m4, True)
                dsv4.dsv4_compress_decode(CI, ZI, bI, tailI, KI, off4, pos, m4, True)
            else:
                dsv4.dsv4_compress_decode(C128, Z128, b128, tail128, pool128, off128, pos, m128,
                                          False)

    # the same jobs in one launch (every layer's ring slot and compressor states). Jobs of one
    # launch run concurrently and must not write the same memory, so each layer of this
    # synthetic step gets its own ring, states and pools (the pools' contents are not read)
    jobs = []
    first = {}
    for kind in D["layers"]:
        own = kind in first
        first[kind] = True
        jobs.append(dsv4.decode_ring_job(kv, local if not jobs else torch.empty_like(local)))
        if kind == "csa":
            jobs.append(dsv4.decode_compress_job(C4, Z4, b4, tail4.clone() if own else tail4,
                                                 torch.empty_like(pool4) if own else pool4, off4, m4, True))
            jobs.append(dsv4.decode_compress_job(CI, ZI, bI, tailI.clone() if own else tailI,
                                                 torch.empty_like(KI) if own else KI, off4, m4, True))
        else:
            jobs.append(dsv4.decode_compress_job(C128, Z128, b128, tail128.clone() if own else tail128,
                                                 torch.empty_like(pool128) if own else pool128, off128,
                                                 m128, False))

    def step_one_launch():
        dsv4.dsv4_decode_state(jobs, pos)

    # the same launch emitting into the production pool formats: CSA main entries quantised to
    # the FP8 entry format (448 FP8 channels + 7 scales + 64 bf16 RoPE channels), CSA index
    # keys to FP4 (e2m1 + one E4M3 scale per 16); HCA entries stay bf16
    rd = 64
    jobs_q = []
    for kind in D["layers"]:
        jobs_q.append(dsv4.decode_ring_job(kv, torch.empty_like(local)))
        if kind == "csa":
            rows = int(sum(E4))
            jobs_q.append(dsv4.decode_compress_fp8_job(
                C4, Z4, b4, tail4.clone(), torch.empty(rows, c - rd, dtype=torch.uint8, device=dev),
                torch.empty(rows, (c - rd) // 64, device=dev),
                torch.empty(rows, rd, dtype=torch.bfloat16, device=dev), off4, m4, True, rd))
            jobs_q.append(dsv4.decode_compress_fp4_job(
                CI, ZI, bI, tailI.clone(), torch.empty(rows, cI // 2, dtype=torch.uint8, device=dev),
                torch.empty(rows, cI // 16, dtype=torch.uint8, device=dev), off4, m4, True))
        else:
            jobs_q.append(dsv4.decode_compress_job(C128, Z128, b128, tail128.clone(),
                                                   torch.empty_like(pool128), off128, m128, False))

    def step_production():
        dsv4.dsv4_decode_state(jobs_q, pos)

    def timed(step):
        for _ in range(3):
            step()
        dsv4.dsv4_check_errors()
        ts = []
        for _ in range(max(1, min(args.steps, 10))):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        dsv4.dsv4_check_errors()
        return statistics.median(ts), len(ts)

    ms_one, n_one = timed(step_one_launch)
    ms_sep, _ = timed(step_separate)
    ms_q, _ = timed(step_production)
    launches = sum(3 if kind == "csa" else 2 for kind in D["layers"])
    return {"what": "ring writes + compressor states of the 4 layers for one token of each of "
                    f"the {B} sequences (entries completing at this token appended), all "
                    f"{len(jobs)} jobs in one dsv4_decode_state launch",
            "ms_per_step": round(ms_one, 4), "launches_per_step": 1,
            "separate_calls": {"ms_per_step": round(ms_sep, 4), "launches_per_step": launches},
            "production_pools": {"what": "the same single launch emitting CSA main entries as FP8 "
                                         "entries and CSA index keys as FP4",
                                 "ms_per_step": round(ms_q, 4), "launches_per_step": 1},
            "emitting_sequences": {"csa": int((L % m4 == 0).sum()), "hca": int((L % m128 == 0).sum())},
            "steps": n_one, "l2": "flushed (256 MiB write) before every step"}


# ----------------------------------------------------------------------------- other layers


def run_layer(args, dev, stream, name):
    """One full prefill layer of another configuration, inputs drawn on the device:
    flash_hca_prefill (B=2, n=65536, HCA m'=128 dense read + window) or pro_csa_prefill
    (n=131072, H=128, k=1024, indexer operands quantised to FP4 inside the step)."""
    import torch
    import compressed_sparse_mqa_dsv4_b200 as dsv4
    from workloads import Generator, preset
    s = preset(name)
    g = Generator(args.seed + 3, device=dev.type)
    E = s.n // s.m
    C, Z, bias = g.compressor_inputs(s, "main")
    Q = g.queries(s)
    local = g.local_kv(s)
    sink = g.sink(s)
    off = torch.arange(s.B, dtype=torch.int64, device=dev) * E
    pos0 = torch.zeros(s.B, dtype=torch.int32, device=dev)
    pool = torch.empty(s.B, E, s.c, dtype=torch.bfloat16, device=dev)
    O = torch.empty_like(Q)
    lse = torch.empty(s.B, s.n, s.H, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    extra = {}
    if s.kind == "csa":
        CI, ZI, biasI = g.compressor_inputs(s, "index")
        qI, w = g.index_queries(s)
        KI = torch.empty(s.B, E, s.c_I, dtype=torch.bfloat16, device=dev)
        qc = torch.empty(s.B * s.n * s.H_I, s.c_I // 2, dtype=torch.uint8, device=dev)
        qs = torch.empty(s.B * s.n * s.H_I, s.c_I // 16, dtype=torch.uint8, device=dev)
        kc = torch.empty(s.B * E, s.c_I // 2, dtype=torch.uint8, device=dev)
        ks = torch.empty(s.B * E, s.c_I // 16, dtype=torch.uint8, device=dev)
        idx = torch.empty(s.B, s.n, s.k, dtype=torch.int32, device=dev)
        cnt = torch.empty(s.B, s.n, dtype=torch.int32, device=dev)
        ws = torch.empty(dsv4.dsv4_index_topk_workspace_size_ex(dsv4.FP4, s.B, s.n, s.H_I, s.c_I, E, s.k,
                                                                s.B * E), dtype=torch.uint8, device=dev)

    def step(rec):
        rec[0].record(stream)
        dsv4.dsv4_compress(C, Z, bias, s.m, s.kind == "csa", out=pool)
        if s.kind == "csa":
            dsv4.dsv4_compress(CI, ZI, biasI, s.m, True, out=KI)
            dsv4.dsv4_quantize_fp4(qI.view(-1, s.c_I), qc, qs)
            dsv4.dsv4_quantize_fp4(KI.view(-1, s.c_I), kc, ks)
            rec[1].record(stream)
            dsv4.dsv4_index_topk(qc.view(s.B, s.n, s.H_I, s.c_I // 2), w, kc, off, pos0, s.m, s.k, E,
                                 qI_scales=qs, KI_scales=ks, c_I=s.c_I, idx=idx, counts=cnt,
                                 workspace=ws)
            rec[2].record(stream)
            dsv4.dsv4_hybrid_sparse_attn(Q, pool.view(-1, s.c), off, idx, cnt, local, pos0, s.m, s.w,
                                         sink, O=O, lse=lse)
        else:
            rec[1].record(stream)
            rec[2].record(stream)
            dsv4.dsv4_hybrid_sparse_attn(Q, pool.view(-1, s.c), off, None, None, local, pos0, s.m, s.w,
                                         sink, O=O, lse=lse)
        rec[3].record(stream)

    for _ in range(2):
        flush.zero_()
        step([torch.cuda.Event(enable_timing=True) for _ in range(4)])
    dsv4.dsv4_check_errors()
    steps = 3
    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        step(recs[i])
    torch.cuda.synchronize()
    dsv4.dsv4_check_errors()
    ms = statistics.median([r[0].elapsed_time(r[3]) for r in recs])
    t_pre = statistics.median([r[0].elapsed_time(r[1]) for r in recs])
    t_idx = statistics.median([r[1].elapsed_time(r[2]) for r in recs])
    t_att = statistics.median([r[2].elapsed_time(r[3]) for r in recs])
    peaks, src = _peaks()
    peak = float(peaks["bf16_tflops"])
    attn_fl = s.B * attention_flops(s.n, s.m, s.k if s.kind == "csa" else 0, s.w, s.H, s.c) \
        if s.kind == "csa" else s.B * hca_attention_flops(s.n, s.m, s.w, s.H, s.c)
    rec = {"workload": f"{name}: B={s.B}, n={s.n}, H={s.H}, c={s.c}, m={s.m}, w={s.w}"
                       + (f", k={s.k}, H_I={s.H_I}, c_I={s.c_I}, FP4 indexer" if s.kind == "csa" else ", dense"),
           "tokens_per_s": round(s.B * s.n / (ms / 1e3), 1), "ms_per_step": round(ms, 3),
           "breakdown_ms": {"compress_quantize": round(t_pre, 3), "index_topk": round(t_idx, 3),
                            "attention": round(t_att, 3)},
           "attention_tflops": round(attn_fl / (t_att / 1e3) / 1e12, 1),
           "attention_frac": round(attn_fl / (t_att / 1e3) / 1e12 / peak, 4), "steps": steps}
    if s.kind == "csa":
        ifl = s.B * index_flops(s.n, s.m, s.H_I, s.c_I)
        rec["index_tflops"] = round(ifl / (t_idx / 1e3) / 1e12, 1)
    return rec


def run_chunk(args, dev, stream):
    """Chunked prefill with a start position (pypto-lib PR #834's workload: 128 tokens at
    start position 896), V4-Flash CSA shapes: the chunk's compressors with their one-block
    halo, its local-window ring, index top-k over the prefix's and the chunk's entries, and
    attention. The prefix [0, 896) is compressed before the timed region (it is the cache
    the chunk extends). Every call goes through the library's public Python API."""
    import torch
    import compressed_sparse_mqa_dsv4_b200 as dsv4
    from compressed_sparse_mqa_dsv4_b200 import cp
    from workloads import Generator, preset
    p0, nq = 896, 128
    n = p0 + nq
    s = preset(WORKLOAD, n=n)
    g = Generator(args.seed + 5, device=dev.type)
    C, Z, bias = g.compressor_inputs(s, "main")
    CI, ZI, biasI = g.compressor_inputs(s, "index")
    qI, w = g.index_queries(s)
    Q, local, sink = g.queries(s), g.local_kv(s), g.sink(s)
    E, m = n // s.m, s.m
    pool = torch.empty(1, E, s.c, dtype=torch.bfloat16, device=dev)
    KI = torch.empty(1, E, s.c_I, dtype=torch.bfloat16, device=dev)
    dsv4.dsv4_compress(C[:, :p0].contiguous(), Z[:, :p0].contiguous(), bias, m, True, out=pool[:, :p0 // m])
    dsv4.dsv4_compress(CI[:, :p0].contiguous(), ZI[:, :p0].contiguous(), biasI, m, True, out=KI[:, :p0 // m])
    sl = slice(p0, n)
    Cc, Zc, CIc, ZIc = (x[:, sl].contiguous() for x in (C, Z, CI, ZI))
    Ch, Zh, CIh, ZIh = (x[:, p0 - m:p0].contiguous() for x in (C, Z, CI, ZI))
    Qc, qIc, wc, lc = (x[:, sl].contiguous() for x in (Q, qI, w, local))
    lh = local[:, p0 - s.w + 1:p0].contiguous()
    pos0 = torch.full((1,), p0, dtype=torch.int32, device=dev)
    off = torch.zeros(1, dtype=torch.int64, device=dev)
    ws = torch.empty(dsv4.dsv4_index_topk_workspace_size(1, nq, E, s.k), dtype=torch.uint8, device=dev)
    idx = torch.empty(1, nq, s.k, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, nq, dtype=torch.int32, device=dev)
    O = torch.empty_like(Qc)
    lse = torch.empty(1, nq, s.H, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(rec):
        rec[0].record(stream)
        cp.compress_range(Cc, Zc, bias, m, True, p0, Ch, Zh, out=pool[:, p0 // m:])
        cp.compress_range(CIc, ZIc, biasI, m, True, p0, CIh, ZIh, out=KI[:, p0 // m:])
        ring, _ = cp.window_ring(lc, p0, s.w, lh)
        rec[1].record(stream)
        dsv4.dsv4_index_topk(qIc, wc, KI.view(E, s.c_I), off, pos0, m, s.k, E, idx=idx, counts=cnt,
                             workspace=ws)
        rec[2].record(stream)
        dsv4.dsv4_hybrid_sparse_attn(Qc, pool.view(E, s.c), off, idx, cnt, ring, pos0, m, s.w, sink,
                                     O=O, lse=lse)
        rec[3].record(stream)

    for _ in range(3):
        flush.zero_()
        step([torch.cuda.Event(enable_timing=True) for _ in range(4)])
    dsv4.dsv4_check_errors()
    steps = 10
    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        step(recs[i])
    torch.cuda.synchronize()
    dsv4.dsv4_check_errors()
    ms = statistics.median([r[0].elapsed_time(r[3]) for r in recs])
    return {"workload": f"chunk_prefill: V4-Flash CSA layer, {nq} tokens at start position {p0} "
                        f"(B=1, H={s.H}, c={s.c}, m={m}, H_I={s.H_I}, c_I={s.c_I}, k={s.k}, w={s.w}, "
                        f"sink; prefix entries compressed before the timed region)",
            "tokens_per_s": round(nq / (ms / 1e3), 1), "ms_per_step": round(ms, 4),
            "breakdown_ms": {
                "compress_and_ring": round(statistics.median([r[0].elapsed_time(r[1]) for r in recs]), 4),
                "index_topk": round(statistics.median([r[1].elapsed_time(r[2]) for r in recs]), 4),
                "attention": round(statistics.median([r[2].elapsed_time(r[3]) for r in recs]), 4)},
            "steps": steps, "l2": "flushed (256 MiB write) before every step",
            "context": "the pages quote 609.6 us (sparse attention) and 488.7 us (indexer) for this "
                       "workload on an Ascend a2a3 device"}


# ----------------------------------------------------------------------------- oracle arm
#
# The fp64 oracle runs the layer on the host cores: both compressors in the parent process,
# then every query's index scores, TopK and attention spread over a pool of worker processes
# (started with "spawn", one BLAS thread each), reading the inputs from shared memory.

_OW = {}


def _bf16_bits(t):
    """A bf16 tensor's raw 16-bit patterns as a numpy uint16 array (no arithmetic)."""
    import torch
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bits_to_f64(bits):
    """Exact fp64 value of bf16 bit patterns (the pattern is the top half of an fp32)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _oracle_worker_init(shm_names, shapes, small):
    from multiprocessing import shared_memory
    _OW.clear()
    _OW["shm"] = [shared_memory.SharedMemory(name=nm) for nm in shm_names]
    _OW["Q"] = np.ndarray(shapes[0], dtype=np.uint16, buffer=_OW["shm"][0].buf)
    _OW["qI"] = np.ndarray(shapes[1], dtype=np.uint16, buffer=_OW["shm"][1].buf)
    _OW.update(small)


def _oracle_worker_run(q_range):
    """Index scores, TopK and attention of the queries t in [q0, q1) (fp64 oracle)."""
    import oracle as O
    q0, q1 = q_range
    s = _OW["s"]
    for t in range(q0, q1):
        sc = O.index_scores_query(_bits_to_f64(_OW["qI"][t]), _OW["w"][t], _OW["KI"], t, s["m"])
        idx, cnt = O.topk_select(sc, s["k"])
        A = O.candidates(_OW["pool"], idx, cnt, _OW["local"], s["n"], t, s["w"])
        O.attend_query(_bits_to_f64(_OW["Q"][t]), A, _OW["sink"], None)
    return q1 - q0


class OracleRunner:
    """The oracle over the whole flash_csa_prefill layer on `workers` host processes."""

    def __init__(self, seed: int, workers: int = 0):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        from workloads import Generator, preset
        s = preset(WORKLOAD)
        g = Generator(seed)
        self.s = s
        self.C, self.Z, self.bias = g.compressor_inputs(s, "main")
        self.CI, self.ZI, self.biasI = g.compressor_inputs(s, "index")
        qI, w = g.index_queries(s)
        Q, local, sink = g.queries(s), g.local_kv(s), g.sink(s)
        self.workers = workers or min(os.cpu_count() or 1, 64)
        self.shm = []
        shapes = []
        for arr in (_bf16_bits(Q[0]), _bf16_bits(qI[0])):
            sh = shared_memory.SharedMemory(create=True, size=max(arr.nbytes, 1))
            np.ndarray(arr.shape, dtype=np.uint16, buffer=sh.buf)[...] = arr
            self.shm.append(sh)
            shapes.append(arr.shape)
        self.small = dict(w=w[0].double().numpy(), local=_bits_to_f64(_bf16_bits(local[0])),
                          sink=sink.double().numpy(),
                          s=dict(m=s.m, k=s.k, n=s.n, w=s.w))
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        # the workers get the compressed pools once (the same values every step recomputes)
        import oracle as O
        small = dict(self.small, pool=O.compress(self.C, self.Z, self.bias, s.m, True)[0],
                     KI=O.compress(self.CI, self.ZI, self.biasI, s.m, True)[0])
        try:
            self.procs = mp.get_context("spawn").Pool(
                self.workers, initializer=_oracle_worker_init,
                initargs=([sh.name for sh in self.shm], shapes, small))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.procs.map(_oracle_worker_run, [(0, 1)] * self.workers)    # every worker is up

    def step(self):
        """One pass over the layer; returns (seconds, compress seconds, queries seconds)."""
        import oracle as O
        s = self.s
        t0 = time.perf_counter()
        O.compress(self.C, self.Z, self.bias, s.m, True)
        O.compress(self.CI, self.ZI, self.biasI, s.m, True)
        t1 = time.perf_counter()
        chunk = 16
        ranges = [(q, min(q + chunk, s.n)) for q in range(0, s.n, chunk)]
        done = sum(self.procs.map(_oracle_worker_run, ranges, chunksize=1))
        t2 = time.perf_counter()
        assert done == s.n
        return t2 - t0, t1 - t0, t2 - t1

    def close(self):
        if self.procs is not None:
            self.procs.close()
            self.procs.join()
        for sh in self.shm:
            sh.close()
            sh.unlink()


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    runner = OracleRunner(args.seed)
    try:
        for _ in range(min(args.warmup, 1)):
            runner.step()
        times = [runner.step() for _ in range(args.steps)]
    finally:
        runner.close()
    total = sum(t[0] for t in times)
    value = runner.s.n * args.steps / total
    sample = (f"the whole layer each step: both compressors over all {runner.s.n} tokens in one "
              f"process ({statistics.mean(t[1] for t in times):.2f} s), then index top-k and "
              f"attention of all {runner.s.n} queries over {runner.workers} worker processes "
              f"({statistics.mean(t[2] for t in times):.2f} s)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": min(args.warmup, 1),
        "ms_per_step": round(total / args.steps * 1e3, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": "flash_csa_prefill: V4-Flash CSA layer prefill, bf16 inputs, "
                               "B=1, n=8192, H=64, c=512, m=4, H_I=64, c_I=128, k=512, w=128, "
                               "sink", "parallelism": f"host processes x{runner.workers} (rank 0 only)"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": runner.workers,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the batched-decode measurement")
    ap.add_argument("--no-layers", action="store_true",
                    help="skip the HCA-prefill, V4-Pro (FP4 indexer) and chunked-prefill records")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus and "RANK" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_cuda(args, rank, world)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                runner = OracleRunner(args.seed)
                try:
                    sec, tc, tq = runner.step()
                finally:
                    runner.close()
                res["cpu_baseline"] = {
                    "value": round(runner.s.n / sec, 3), "unit": UNIT, "cores": runner.workers,
                    "kind": "oracle",
                    "sample": f"fp64 oracle, one pass over the whole layer: both compressors over "
                              f"all {runner.s.n} tokens in one process ({tc:.2f} s), then index "
                              f"top-k and attention of all {runner.s.n} queries over "
                              f"{runner.workers} worker processes ({tq:.2f} s)"}
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
