#!/usr/bin/env python
"""Benchmark of the FP8 grouped matmul hot path on B200.

One step = the three passes of one MoE expert-MLP layer on one batch:
forward gmm (lhs quantized inside the call), dlhs gmm and tgmm drhs, on the
Mixtral-like workload (G=8, M=16384 = 8192 tokens x top-2, K=4096,
N=28672 = merged 2 x 14336, static per-tensor lhs scale, rhs pre-quantized
E4M3 with per-(g, n) scales).  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs under torchrun: N independent replicas (the path has no exchange
step; each rank draws its own batch), weak scaling, time = max over ranks.
--impl reference times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 grouped-GEMM TFLOP/s (fwd, dlhs, drhs) and % of B200 dense FP8 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)
# the GEMM kernel sources a traffic record was captured from (one-CTA and pair tiles)
GEMM_SRCS = [os.path.join(ROOT, "moe_fp8_grouped_b200", "csrc", f) for f in ("gemm_tc.cu", "gemm_pair.cu")]


def gemm_src_hash() -> str:
    h = hashlib.sha256()
    for f in GEMM_SRCS:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mixtral")
    ap.add_argument("--m-override", type=int, default=None,
                    help="fewer rows (same routing recipe), for profiler captures of a small case")
    ap.add_argument("--n-override", type=int, default=None,
                    help="fewer output columns, for profiler captures of a small case")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--separate-backward", action="store_true",
                    help="run dlhs and drhs as two calls (gmm_dlhs, tgmm_drhs) instead of gmm_backward, which "
                         "quantizes dout once for both")
    ap.add_argument("--tiles", default="auto", choices=["auto", "one_cta", "cta_pairs", "cta_pairs_narrow"],
                    help="GEMM tile choice (gmm_set_tiles): automatic, 128-row tiles on one CTA, or 256-row tiles "
                         "over CTA pairs")
    ap.add_argument("--no-forward-shapes", dest="forward_shapes", action="store_false",
                    help="skip the forward measurement on the DeepSeek-V3 and EP-shrunk shapes that the default "
                         "(Mixtral, one GPU) run adds to its line")
    ap.add_argument("--rhs-blocks", action="store_true",
                    help="block-wise weight scales: forward codes with [G, K/128, N] scales, dlhs codes with "
                         "[G, N/128, K] scales (two weight copies, made outside the timed step)")
    return ap.parse_args()


L2_BYTES = 126 * 2 ** 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, src, region_s: float, bf16_family: bool, clocks=None):
    """The tensor peak a kernel timed inside a region of region_s seconds is
    held to: the burst cuBLAS bf16 figure while the SM clock stays near its
    maximum, the sustained (power-capped) one when the median SM clock sampled
    during the region fell below 90 % of the maximum; without clock samples,
    burst for regions under 2 s.  x2 (the nominal dense fp8 / bf16 ratio,
    4.5 / 2.25 PFLOP/s) for fp8."""
    mhz = clocks.get("sm_mhz") if clocks else None
    mx = clocks.get("sm_max_mhz") if clocks else None
    if mhz and mx:
        sustained = mhz < 0.9 * mx
        why = f"median SM clock {mhz:.0f} of {mx:.0f} MHz over the timed region ({region_s:.2f} s)"
    else:
        sustained = region_s >= 2.0
        why = f"timed region {region_s:.2f} s, no clock samples"
    v = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"] * (1.0 if bf16_family else FP8_OVER_BF16)
    desc = (f"{src} bf16 {'sustained' if sustained else 'burst'} cuBLAS"
            + ("" if bf16_family else f" x {FP8_OVER_BF16} (nominal fp8/bf16 ratio)") + f"; {why}")
    return v, desc


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time (every rank takes part; world == 1: unchanged)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step_per_rank: float, world: int, steps: int, ms: float) -> float:
    """Whole-job throughput: the FLOPs every rank did over the slowest rank's time."""
    return world * flops_per_step_per_rank * steps / (ms / 1e3) / 1e12


def algorithmic_bytes(M, K, N, G, G_ne, rule):
    """Bytes each pass must move: its inputs once and its outputs once (bf16
    activations, E4M3 weights with fp32 [G, N] scales, dynamic block scales,
    bf16 fwd / dlhs outputs, fp32 dW; bf16 weights for the bf16 family)."""
    wb = 2 if rule == "none" else 1
    wsc = 0 if rule == "none" else 4 * G * N
    lsc = 4 * M * K // 128 if rule == "dynamic" else 0
    gsc = 0 if rule == "none" else 4 * M * N // 128
    return {"fwd": 2 * M * K + lsc + wb * G_ne * K * N + wsc + 2 * M * N,
            "dlhs": 2 * M * N + gsc + wb * G_ne * K * N + wsc + 2 * M * K,
            "drhs": 2 * M * K + 2 * M * N + 4 * G * K * N,
            # merged gate|up forward with SwiGLU fused: the [M, N/2] bf16 result only
            "fwd_swiglu": 2 * M * K + lsc + wb * G_ne * K * N + wsc + M * N}


def needs_l2_flush(w):
    """True when one step's operands (lhs, dout, weights) could stay in L2
    (126 MB) from one step to the next."""
    op_bytes = w.M * w.K * 2 + w.M * w.N * 2 + w.G * w.K * w.N * (2 if w.rule == "none" else 1)
    return op_bytes < 4 * L2_BYTES


def step_config(w, args, world):
    """The config of one bench step for workload w under these arguments (the
    same dict on both arms)."""
    separate = w.name == "ep_separate"
    parts = 2 if separate else 1
    Np = w.N // parts
    bf16_family = w.rule == "none"
    fused_bwd = not args.separate_backward
    keep_lhs = w.rule == "static" and not bf16_family
    blocks = bool(args.rhs_blocks)
    flush_l2 = needs_l2_flush(w)
    return config_of(w, {"parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                         "calls_per_pass": parts,
                         "backward": ("gmm_backward (dout quantized once for dlhs and drhs)" if fused_bwd
                                      else "gmm_dlhs + tgmm_drhs"),
                         "lhs_codes": ("gmm_fwd_keep_lhs hands the forward's E4M3 lhs codes to the tgmm"
                                       if keep_lhs else "the tgmm quantizes lhs itself"),
                         "rhs_scales": ("block-wise: fwd [G, K/128, N], dlhs [G, N/128, K]" if blocks
                                        else "per channel [G, N]"),
                         "tiles": args.tiles,
                         **({"l2": "flushed before every step (256 MiB write outside the timed events; "
                                   "the operands would fit in L2 across steps)"} if flush_l2 else {}),
                         **({"workload": f"ep_separate: G={w.G} M={w.M} K={w.K}, two N={Np} calls per pass "
                                         f"(W0, W1 apart), lhs rule {w.rule}, fwd+dlhs+drhs"}
                            if separate else {})})


def config_of(w, extra=None):
    cfg = {"workload": f"{w.name}: G={w.G} M={w.M} K={w.K} N={w.N}, lhs rule {w.rule}, fwd+dlhs+drhs",
           "G": w.G, "M": w.M, "K": w.K, "N": w.N, "lhs_rule": w.rule, "routing": w.routing,
           "out_dtypes": {"fwd": "bf16", "dlhs": "bf16", "drhs": "f32"},
           "l2": "not flushed: inputs larger than L2 (rhs codes and dout exceed 126 MB)"}
    if extra:
        cfg.update(extra)
    return cfg


# --------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
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
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    rows.append((float(p[1]), float(p[2]), float(p[3]), p[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------- our arm

def workload_key(w, blocks: bool) -> str:
    return f"{w.name}/G{w.G}/M{w.M}/K{w.K}/N{w.N}/{w.rule}" + ("/blockwise" if blocks else "")


def traffic_record(kernel: str, key: str):
    """DRAM bytes per launch from a committed ncu capture of this kernel on this
    workload, or None when there is none or the kernel source changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        src_hash = gemm_src_hash()
        for r in rec.get(kernel, []):
            if r.get("gemm_src_sha256_16") == src_hash and r.get("workload_key") == key:
                return r.get("bytes_per_launch")
    except Exception:
        pass
    return None


def run_ours(args):
    import torch
    import torch.distributed as dist

    import moe_fp8_grouped_b200 as gm
    from moe_fp8_grouped_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # ep_separate: the EP-shrunk workload as two separate N=256 calls per pass
    # (W0 and W1 apart) instead of one merged N=512 call
    gm.gmm_set_tiles(args.tiles)
    separate = args.workload == "ep_separate"
    w_named = synth.WORKLOADS[args.workload]
    w = synth.WORKLOADS["ep_merged" if separate else args.workload]
    if args.m_override:
        w = w_named = synth.with_rows(w, args.m_override)
    if args.n_override:
        w = w_named = synth.with_cols(w, args.n_override)
    inp = synth.make_inputs(w, seed=rank, device=str(dev))
    gs = inp.group_sizes.to(dev)
    rows_routed = int(inp.group_sizes.sum())
    G_ne = int((inp.group_sizes > 0).sum())
    s_static = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    M, K, N, G = w.M, w.K, w.N, w.G
    rule = w.rule
    bf16_family = rule == "none"
    parts = 2 if separate else 1
    Np = N // parts
    # weight quantization (or, for the bf16 family, nothing): outside the timed step
    blocks = bool(args.rhs_blocks)
    if blocks and (bf16_family or separate):
        raise SystemExit("--rhs-blocks needs an fp8 workload with one call per pass")
    if bf16_family:
        wparts = [(inp.w[:, :, i * Np:(i + 1) * Np].contiguous(), None) for i in range(parts)]
    elif blocks:
        wparts = [gm.gmm_quantize_rhs_blocks(inp.w, 0)]
    else:
        wparts = [gm.gmm_quantize_rhs(inp.w[:, :, i * Np:(i + 1) * Np].contiguous()) for i in range(parts)]
    codes, rscales = wparts[0]
    # dlhs weights: the same codes (per channel), or the copy block-wise along N
    dl_codes, dl_scales = gm.gmm_quantize_rhs_blocks(inp.w, 1) if blocks else (None, None)
    del inp.w
    lhs = inp.lhs
    douts = [inp.dout[:, i * Np:(i + 1) * Np].contiguous() for i in range(parts)]
    dout = douts[0]
    del inp.dout
    out = torch.empty((M, Np), dtype=torch.bfloat16, device=dev)
    dl = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((G, K, Np), dtype=torch.float32, device=dev)
    ws = torch.empty(max(gm.gmm_workspace_bytes(op, M, K, Np, G) for op in (0, 1, 2, 3)), dtype=torch.uint8,
                     device=dev)
    fused_bwd = not args.separate_backward
    # static rule: the forward hands its lhs codes to the backward (tgmm lhs re-laid out, not quantized again)
    keep_lhs = rule == "static" and not bf16_family
    lhs_codes = torch.empty((M, K), dtype=torch.uint8, device=dev) if keep_lhs else None
    sarg = s_static if rule == "static" else None
    grule = "none" if bf16_family else "dynamic"
    launches = [0]

    def step(lhs_, dout_, codes_, rscales_, gs_):
        for i in range(parts):
            c_, r_ = (codes_, rscales_) if i == 0 else wparts[i]
            d_ = dout_ if i == 0 else douts[i]
            if keep_lhs:
                gm.gmm_fwd_keep_lhs(lhs_, c_, r_, gs_, rule=rule, static_scale=sarg, out=out, ws=ws,
                                    lhs_codes=lhs_codes)
            else:
                gm.gmm_fwd(lhs_, c_, r_, gs_, rule=rule, static_scale=sarg, out=out, ws=ws)
            launches[0] += gm.last_launch_count()
            x_ = lhs_codes if keep_lhs else lhs_  # the tgmm's lhs operand
            if blocks:
                c_, r_ = dl_codes, dl_scales
            if fused_bwd:
                gm.gmm_backward(x_, d_, c_, r_, gs_, rule=rule, static_scale=sarg, dlhs=dl, drhs=dw, ws=ws)
                launches[0] += gm.last_launch_count()
            else:
                gm.gmm_dlhs(d_, c_, r_, gs_, out=dl, ws=ws, rule=grule)
                launches[0] += gm.last_launch_count()
                gm.tgmm_drhs(x_, d_, gs_, rule=rule, static_scale=sarg, out=dw, ws=ws)
                launches[0] += gm.last_launch_count()

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step(lhs, dout, codes, rscales, gs)
    st, bits = gm.gmm_read_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} bits {bits} after warm-up")
    barrier()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)  # let the sampler start before the timed region
    gm.profile_enable(True)
    launches[0] = 0
    # operands that could stay in L2 (126 MB) from one step to the next: flush
    # L2 between steps with a 256 MiB write outside the timed events
    flush_l2 = needs_l2_flush(w)
    barrier()
    if flush_l2:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in evs:
            flush.zero_()
            a.record()
            step(lhs, dout, codes, rscales, gs)
            b.record()
        barrier()
        local_ms = sum(a.elapsed_time(b) for a, b in evs)
        del flush
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            step(lhs, dout, codes, rscales, gs)
        e1.record()
        barrier()
        local_ms = e0.elapsed_time(e1)
    gm.profile_enable(False)
    prof = gm.profile_collect()
    clk = clocks.stop()
    ms = max_over_ranks(local_ms, world, dev)
    timed_launches = launches[0]

    flops_pass = 2.0 * rows_routed * K * Np  # one launch
    flops_step = 3 * parts * flops_pass
    value = job_tflops(flops_step, world, args.steps, ms)

    peaks, peak_src = load_peaks()
    peak_tc, peak_tc_src = tensor_peak(peaks, peak_src, ms / 1e3, bf16_family, clk)
    peak_bw = peaks["hbm_gbs"]
    bytes_pass = algorithmic_bytes(M, K, Np, G, G_ne, rule)
    passes = {}
    for name, key in (("fwd", "gemm_fwd"), ("dlhs", "gemm_dlhs"), ("drhs", "gemm_drhs")):
        n, tot = prof.get(key, (0, 0.0))
        if n:
            avg = tot / n
            tfl = flops_pass / (avg / 1e3) / 1e12
            gbs = bytes_pass[name] / (avg / 1e3) / 1e9
            floor_ms = max(flops_pass / (peak_tc * 1e12), bytes_pass[name] / (peak_bw * 1e9)) * 1e3
            passes[name] = {"gemm_ms": round(avg, 4), "gemm_tflops": round(tfl, 1), "gb_per_s": round(gbs, 1),
                            "frac_tensor": round(tfl / peak_tc, 4), "frac_hbm": round(gbs / peak_bw, 4),
                            "frac_roofline": round(floor_ms / avg, 4)}
    total_prof = sum(t for _, t in prof.values())
    kernels = {k: {"launches": n, "total_ms": round(t, 3), "share": round(t / total_prof, 4) if total_prof else None}
               for k, (n, t) in sorted(prof.items())}
    dom = max((k for k in prof if k.startswith("gemm_")), key=lambda k: prof[k][1])
    dn, dt = prof[dom]
    dname = dom.split("_")[1]
    tc_bound = flops_pass / (peak_tc * 1e12) >= bytes_pass[dname] / (peak_bw * 1e9)  # seconds at each peak
    if tc_bound:
        achieved = flops_pass / (dt / dn / 1e3) / 1e12
        roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak_tc, 1),
                    "unit": "TFLOP/s", "frac": round(achieved / peak_tc, 4),
                    "peak_source": peak_tc_src,
                    "algorithmic": f"2*sum(group_sizes)*K*N = {flops_pass:.4g} FLOP per launch"}
    else:
        achieved = bytes_pass[dname] / (dt / dn / 1e3) / 1e9
        roofline = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": round(peak_bw, 1),
                    "unit": "GB/s", "frac": round(achieved / peak_bw, 4),
                    "peak_source": f"{peak_src} HBM copy bandwidth",
                    "algorithmic": f"{bytes_pass[dname]:.4g} bytes per launch (operands in, results out)"}
    roofline["traffic"] = traffic_record(dom, workload_key(w, blocks))

    # merged gate|up workloads: the forward with SwiGLU fused into its
    # epilogue, timed on its own (not part of the step), with an L2 flush
    # (a 256 MiB write) before each call
    if w.merged and parts == 1 and not blocks:
        sw_out = torch.empty((M, N // 2), dtype=torch.bfloat16, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

        def swiglu_call():
            gm.gmm_fwd_swiglu(lhs, codes, rscales, gs, rule=rule, static_scale=sarg, out=sw_out, ws=ws)

        for _ in range(3):
            swiglu_call()
        barrier()
        gm.profile_enable(True)
        for _ in range(min(args.steps, 20)):
            flush.zero_()
            swiglu_call()
        barrier()
        gm.profile_enable(False)
        n, tot = gm.profile_collect().get("gemm_fwd_swiglu", (0, 0.0))
        if n:
            avg = tot / n
            tfl = flops_pass / (avg / 1e3) / 1e12
            gbs = bytes_pass["fwd_swiglu"] / (avg / 1e3) / 1e9
            floor_ms = max(flops_pass / (peak_tc * 1e12), bytes_pass["fwd_swiglu"] / (peak_bw * 1e9)) * 1e3
            passes["fwd_swiglu"] = {"gemm_ms": round(avg, 4), "gemm_tflops": round(tfl, 1),
                                    "gb_per_s": round(gbs, 1), "frac_tensor": round(tfl / peak_tc, 4),
                                    "frac_hbm": round(gbs / peak_bw, 4), "frac_roofline": round(floor_ms / avg, 4),
                                    "note": "gmm_fwd_swiglu: out[M, N/2] = silu(gate) * up of the merged "
                                            "product; timed apart from the step, L2 flushed per call"}
        del sw_out, flush

    # expert-parallel forward (ep_moe_fwd: row gather by expert, exchange,
    # gmm_fwd on the local experts, return and weighted combine) on the
    # EP-shrunk workload: M rows = T tokens x top-2; one rank, so the
    # exchange is the identity and the time is the data movement around the
    # gmm plus the gmm itself
    if w.name == "ep_merged" and parts == 1 and rule == "static" and world == 1 and not blocks:
        from moe_fp8_grouped_b200 import ep
        T, kk = M // 2, 2
        gen = torch.Generator(device=dev).manual_seed(1)
        ids = torch.stack([torch.randperm(G, generator=gen, device=dev)[:kk] for _ in range(T)]).to(torch.int32)
        wts = torch.softmax(torch.randn(T, kk, generator=gen, device=dev), dim=1)
        xq, _ = gm.gmm_quantize(lhs[:T].contiguous(), "static", axis=1, static_scale=s_static)
        for _ in range(3):
            ep.ep_moe_fwd(xq, s_static, ids, wts, codes, rscales)
        barrier()
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        evs = []
        for _ in range(min(args.steps, 20)):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            ep.ep_moe_fwd(xq, s_static, ids, wts, codes, rscales)
            b.record()
            evs.append((a, b))
        barrier()
        ep_ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
        # the same call captured as a CUDA graph (one rank: no host synchronization)
        try:
            graph = ep.EPForwardGraph(xq, s_static, ids, wts, codes, rscales)
        except RuntimeError as exc:  # capture refused by the runtime: report the eager time only
            graph, graph_err = None, str(exc).splitlines()[0]
        ep_graph_ms = None
        if graph is not None:
            barrier()
            evs = []
            for _ in range(min(args.steps, 20)):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                graph.replay()
                b.record()
                evs.append((a, b))
            barrier()
            ep_graph_ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
        passes["ep_moe_fwd"] = {"ms": round(ep_ms, 4), "tflops": round(flops_pass / (ep_ms / 1e3) / 1e12, 1),
                                "graph_ms": round(ep_graph_ms, 4) if ep_graph_ms else None,
                                "graph_tflops": (round(flops_pass / (ep_graph_ms / 1e3) / 1e12, 1)
                                                 if ep_graph_ms else None),
                                **({} if graph is not None else {"graph_error": graph_err}),
                                "gemm_fwd_ms": passes.get("fwd", {}).get("gemm_ms"),
                                "note": f"{T} tokens x top-{kk} over {G} experts, one rank: route (sort by "
                                        "expert), gather E4M3 rows, gmm_fwd, weighted combine (bf16 out); ms: "
                                        "eager calls (ids checked each call); graph_ms: the same kernels "
                                        "replayed from a CUDA graph; L2 flushed per call"}
        del flush, graph

    # end to end: pinned host buffers, copies inside the timed region.  Steps
    # are pipelined over three streams (upload, compute, download) with two
    # device buffer sets, so step i's download overlaps step i+1's upload and
    # compute; every step still uploads its inputs and downloads its results.
    e2e = None
    if args.e2e_steps > 0 and parts == 1 and not blocks:
        h_lhs, h_dout = lhs.cpu().pin_memory(), dout.cpu().pin_memory()
        h_codes, h_rs, h_gs = codes.cpu().pin_memory(), rscales.cpu().pin_memory(), inp.group_sizes.pin_memory()
        h_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        h_dl = [torch.empty(dl.shape, dtype=dl.dtype, pin_memory=True) for _ in range(2)]
        h_dw = [torch.empty(dw.shape, dtype=dw.dtype, pin_memory=True) for _ in range(2)]
        d_in = [(torch.empty_like(lhs), torch.empty_like(dout), torch.empty_like(codes), torch.empty_like(rscales),
                 torch.empty_like(gs)) for _ in range(2)]
        d_out = [(out if i == 0 else torch.empty_like(out), dl if i == 0 else torch.empty_like(dl),
                  dw if i == 0 else torch.empty_like(dw)) for i in range(2)]
        ws2 = [ws, torch.empty_like(ws)]
        e2e_codes = [lhs_codes, torch.empty_like(lhs_codes)] if keep_lhs else None
        h2d = sum(t.numel() * t.element_size() for t in (h_lhs, h_dout, h_codes, h_rs, h_gs))
        d2h = sum(t.numel() * t.element_size() for t in (h_out[0], h_dl[0], h_dw[0]))
        s_up, s_cmp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        Ev = lambda: torch.cuda.Event()  # noqa: E731
        up_done, cmp_done, down_done = [Ev(), Ev()], [Ev(), Ev()], [Ev(), Ev()]
        used_in = [False, False]
        used_out = [False, False]

        def e2e_step(i):
            b = i % 2
            a_lhs, a_dout, a_codes, a_rs, a_gs = d_in[b]
            o_out, o_dl, o_dw = d_out[b]
            with torch.cuda.stream(s_up):
                if used_in[b]:
                    s_up.wait_event(cmp_done[b])  # compute of step i-2 has read this input set
                a_lhs.copy_(h_lhs, non_blocking=True)
                a_dout.copy_(h_dout, non_blocking=True)
                a_codes.copy_(h_codes, non_blocking=True)
                a_rs.copy_(h_rs, non_blocking=True)
                a_gs.copy_(h_gs, non_blocking=True)
                up_done[b].record(s_up)
            used_in[b] = True
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(up_done[b])
                if used_out[b]:
                    s_cmp.wait_event(down_done[b])  # download of step i-2 has read this output set
                if keep_lhs:
                    gm.gmm_fwd_keep_lhs(a_lhs, a_codes, a_rs, a_gs, rule=rule, static_scale=sarg, out=o_out,
                                        ws=ws2[b], lhs_codes=e2e_codes[b])
                else:
                    gm.gmm_fwd(a_lhs, a_codes, a_rs, a_gs, rule=rule, static_scale=sarg, out=o_out, ws=ws2[b])
                launches[0] += gm.last_launch_count()
                a_x = e2e_codes[b] if keep_lhs else a_lhs
                if fused_bwd:
                    gm.gmm_backward(a_x, a_dout, a_codes, a_rs, a_gs, rule=rule, static_scale=sarg, dlhs=o_dl,
                                    drhs=o_dw, ws=ws2[b])
                    launches[0] += gm.last_launch_count()
                else:
                    gm.gmm_dlhs(a_dout, a_codes, a_rs, a_gs, out=o_dl, ws=ws2[b], rule=grule)
                    launches[0] += gm.last_launch_count()
                    gm.tgmm_drhs(a_x, a_dout, a_gs, rule=rule, static_scale=sarg, out=o_dw, ws=ws2[b])
                    launches[0] += gm.last_launch_count()
                cmp_done[b].record(s_cmp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(cmp_done[b])
                h_out[b].copy_(o_out, non_blocking=True)
                h_dl[b].copy_(o_dl, non_blocking=True)
                h_dw[b].copy_(o_dw, non_blocking=True)
                down_done[b].record(s_down)
            used_out[b] = True

        e2e_step(0)
        e2e_step(1)
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s_up)
        for i in range(args.e2e_steps):
            e2e_step(i)
        f1.record(s_down)
        barrier()
        ems = max_over_ranks(f0.elapsed_time(f1), world, dev)
        e2e = {"value": round(job_tflops(flops_step, world, args.e2e_steps, ems), 2), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(ems / args.e2e_steps, 3),
               "path": "per step: pinned host -> device copies of lhs, dout, rhs codes + scales, group sizes; "
                       "gmm_fwd(_keep_lhs) + gmm_backward (dlhs, drhs); device -> pinned host copies of out, dlhs, dW. Steps "
                       "pipelined over upload / compute / download streams with two device buffer sets."}

    # the forward on the HBM-bound shapes (DeepSeek-V3 up / down, EP-shrunk
    # merged), measured in the same process on one GPU: the shapes whose
    # forward throughput and HBM GB/s the metric asks for next to the step
    fwd_shapes = None
    if world == 1 and args.workload == "mixtral" and not args.m_override and not args.n_override \
            and args.forward_shapes:
        fwd_shapes = measure_forward_shapes(dev, ("dsv3_up", "dsv3_down", "ep_merged"), min(args.steps, 20), peaks,
                                            peak_src)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(w, args.cpu_seconds)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if bf16_family else "e4m3", "data": "synthetic",
        "config": step_config(w_named, args, world),
        "pct_peak": {"vs_nominal": round(value / world / (2250.0 if bf16_family else 4500.0) * 100, 2),
                     "vs_measured": round(value / world / peak_tc * 100, 2),
                     "peak": "dense bf16" if bf16_family else "dense fp8", "measured_peak": peak_tc_src},
        **({"forward_shapes": fwd_shapes} if fwd_shapes else {}),
        "passes": passes, "kernels": kernels, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": timed_launches, "clocks": clk,
    }
    print(json.dumps(line))


def measure_forward_shapes(dev, names, calls, peaks, peak_src):
    """gmm_fwd on each named workload (weights quantized outside the timed
    calls, a 256 MiB L2 flush before every call, outside its events): the whole
    call (group plan, lhs quantization, GEMM) and the GEMM kernel alone, as
    TFLOP/s, % of the nominal dense FP8 peak, algorithmic HBM GB/s and the
    fraction of the roofline max(FLOP / tensor peak, bytes / HBM peak)."""
    import torch

    import moe_fp8_grouped_b200 as gm
    from moe_fp8_grouped_b200 import synth

    res = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for name in names:
        w = synth.WORKLOADS[name]
        inp = synth.make_inputs(w, seed=0, device=str(dev))
        inp.dout = None
        gs = inp.group_sizes.to(dev)
        codes, rs = gm.gmm_quantize_rhs(inp.w)
        inp.w = None
        s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev) if w.rule == "static" else None
        out = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(gm.gmm_workspace_bytes(0, w.M, w.K, w.N, w.G), dtype=torch.uint8, device=dev)

        def call():
            gm.gmm_fwd(inp.lhs, codes, rs, gs, rule=w.rule, static_scale=s, out=out, ws=ws)

        for _ in range(3):
            call()
        st, bits = gm.gmm_read_device_status(ws)
        if st != 0:
            raise RuntimeError(f"{name}: device status {st} bits {bits}")
        clk = ClockSampler(dev.index if dev.index is not None else 0)
        clk.start()
        time.sleep(0.3)
        gm.profile_enable(True)
        evs = []
        for _ in range(calls):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            call()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        gm.profile_enable(False)
        prof = gm.profile_collect()
        clocks = clk.stop()
        call_ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
        n, tot = prof.get("gemm_fwd", (0, 0.0))
        gemm_ms = tot / n if n else None
        rows = int(inp.group_sizes.sum())
        G_ne = int((inp.group_sizes > 0).sum())
        flops = 2.0 * rows * w.K * w.N
        nbytes = algorithmic_bytes(w.M, w.K, w.N, w.G, G_ne, w.rule)["fwd"]
        peak_tc, tc_src = tensor_peak(peaks, peak_src, sum(a.elapsed_time(b) for a, b in evs) / 1e3, False, clocks)
        floor_ms = max(flops / (peak_tc * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e3

        def figures(t_ms):
            return {"ms": round(t_ms, 4), "tflops": round(flops / (t_ms / 1e3) / 1e12, 1),
                    "pct_nominal_fp8": round(flops / (t_ms / 1e3) / 1e12 / 4500.0 * 100, 2),
                    "gb_per_s": round(nbytes / (t_ms / 1e3) / 1e9, 1),
                    "frac_roofline": round(floor_ms / t_ms, 4)}

        res[name] = {"workload": f"{name}: G={w.G} M={w.M} K={w.K} N={w.N}, lhs rule {w.rule}, forward only",
                     "call": figures(call_ms), "gemm": figures(gemm_ms) if gemm_ms else None,
                     "bound": "hbm" if nbytes / (peaks["hbm_gbs"] * 1e9) > flops / (peak_tc * 1e12) else "tensor",
                     "roofline_ms": round(floor_ms, 4), "algorithmic_bytes": nbytes, "flop": flops,
                     "peak_tflops": round(peak_tc, 1), "peak_source": f"{tc_src}; HBM {peak_src} copy",
                     "clocks_sm_mhz": clocks.get("sm_mhz") if clocks else None,
                     "calls": calls, "l2": "flushed before every call (256 MiB write outside the events)"}
        del inp, gs, codes, rs, out, ws, s
        torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------ CPU (oracle) side

_SAMPLE_CACHE = {}


def _sample_group(w):
    """One expert of the workload for the oracle sample: its row count and its
    quantized weights (weight quantization is outside the timed passes)."""
    if w.name not in _SAMPLE_CACHE:
        import torch

        import oracle
        from moe_fp8_grouped_b200 import synth
        gen = torch.Generator().manual_seed(0)
        gs = synth.group_sizes(w, gen)
        S = int(gs[[g for g in range(w.G) if int(gs[g]) > 0][0]])
        W = (torch.randn((1, w.K, w.N), generator=gen) * 0.02).to(torch.bfloat16)
        _SAMPLE_CACHE[w.name] = (S,) + tuple(oracle.quantize_rhs(W))
    return _SAMPLE_CACHE[w.name]


def cpu_baseline_sample(w, budget_s: float, seed: int = 0):
    """Times the oracle on a bounded sample of the workload: batches of
    forward rows, dlhs rows and drhs (g, k) rows until ~budget_s of wall time.
    Returns TFLOP/s on the same FLOP count the GPU metric uses."""
    import numpy as np
    import torch

    import oracle

    S, qr, sr = _sample_group(w)
    gen = torch.Generator().manual_seed(1000 + seed)
    K, N = w.K, w.N
    rule = oracle.Q_STATIC if w.rule == "static" else oracle.Q_DYNAMIC
    s = 4.0 / 448.0
    nt = oracle.num_threads()
    S_drhs = min(S, 512)  # rows of the drhs sample group (bounded)
    x_g = torch.randn((S_drhs, K), generator=gen).to(torch.bfloat16)
    d_g = torch.randn((S_drhs, N), generator=gen).to(torch.bfloat16)
    flops = 0.0
    t_total = 0.0
    batches = 0
    while t_total < budget_s and batches < 1000:
        rows = nt
        lhs = torch.randn((rows, K), generator=gen).to(torch.bfloat16)
        dout = torch.randn((rows, N), generator=gen).to(torch.bfloat16)
        sizes = np.array([rows], np.int32)
        t0 = time.perf_counter()
        oracle.gmm_fwd(lhs, rule, s, qr, sr, sizes)
        oracle.gmm_dlhs(dout, qr, sr, sizes)
        oracle.tgmm_drhs(x_g, rule, s, d_g, np.array([S_drhs], np.int32), sel=list(range(nt)))
        t_total += time.perf_counter() - t0
        flops += 2.0 * rows * K * N * 2 + 2.0 * S_drhs * N * nt
        batches += 1
    return {"value": round(flops / t_total / 1e12, 6), "unit": UNIT, "cores": nt, "kind": "oracle",
            "sample": f"{batches} batches of {nt} fwd rows + {nt} dlhs rows (K={K}, N={N}) + {nt} drhs (g,k) rows "
                      f"over a {S_drhs}-row group; {t_total:.1f} s of oracle time; fp64 C loops, OpenMP over rows",
            "seconds": round(t_total, 2)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return  # only rank 0 runs the CPU reference
    from moe_fp8_grouped_b200 import synth
    w = synth.WORKLOADS[args.workload]
    per_step = max(1.0, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline_sample(w, per_step / 3)
    vals, secs = [], 0.0
    for i in range(args.steps):
        r = cpu_baseline_sample(w, per_step / 3, seed=i)
        vals.append(r["value"])
        secs += r["seconds"]
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": step_config(w, args, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": r["cores"], "kind": "oracle",
                         "sample": f"per step: {r['sample']}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
