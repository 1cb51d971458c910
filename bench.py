"""Benchmark of the NVFP4 GEMM + fused-epilogue hot path on B200.

One step = one DiT layer's projection path over M tokens, all on the GPU through the
C ABI (weights packed once beforehand, untimed):
  1. nvfp4_quantize(x)                    activations 16384 x 3072 bf16 -> NVFP4 (amax pass + quantise)
  2. gemm_nvfp4_rmsnorm(x, Wqkv)          N = 9216 (12 heads x 256 for each of Q, K, V),
                                          RMSNorm head_dim 256 on Q and K, V passed through
  3. gemm_nvfp4_swiglu(x, Wup) -> h       N = 2 x 12288 gate|up, SwiGLU, NVFP4 re-quantisation
                                          with a static scale (calibrated once, untimed)
  4. gemm_nvfp4_plain(h, Wdown)           K = 12288, N = 3072
value = GEMM FLOPs of the step (2MNK summed over the three GEMMs) / step time, TFLOP/s.
Separately timed (not in `value`): the unfused comparison (plain GEMM writes bf16, then a
separate RMSNorm / SwiGLU / quantise kernel), reported as fused-vs-unfused speedups.

Multi-GPU: one process per GPU (torchrun); every rank runs its own M-token batch, no
collective on the data path (weak scaling); time = max over ranks.

--impl reference times the CPU oracle (oracle/) on a bounded row sample of the same step.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "fused NVFP4 GEMM+epilogue TFLOPS and % of B200 FP4 peak; fused-vs-unfused speedup"
K_IN, N_QKV, N_NORM, HD, N_UP, K_DOWN = 3072, 9216, 6144, 256, 24576, 12288
EPS = 1e-6
FP4_PER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput (9 : 2.25 PFLOP/s)
FP4_DATASHEET_TFLOPS = 9000.0  # B200 dense FP4, the vendor's figure


def step_flops(M: int) -> dict:
    return {"qkv": 2 * M * N_QKV * K_IN, "up": 2 * M * N_UP * K_IN, "down": 2 * M * K_DOWN * K_IN}


def max_over_ranks(x: float, device) -> float:
    """The largest x over the ranks of the default process group (x itself with one rank).
    The whole job's time is its slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Work of all ranks per step over the slowest rank's time per step, in TFLOP/s."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def workload_desc(M: int) -> str:
    return (f"DiT layer projections at M={M} tokens: quantise x ({M}x{K_IN} bf16) -> QKV GEMM "
            f"N={N_QKV} + per-head RMSNorm hd{HD} on Q,K (V passthrough) -> FFN-up GEMM N={N_UP} "
            f"SwiGLU + NVFP4 re-quantisation -> FFN-down GEMM K={K_DOWN} N={K_IN}")


# DRAM bytes (read + write) per launch of the FFN-up fused GEMM at M=16384, from the ncu
# capture summarised in profiles/, keyed by a hash of the GEMM's device code: a value
# taken on another version of the kernel is not reported.
TRAFFIC_BY_SOURCE = {
    "923de5902a1b1c2e": 146.2e6,
}


def gemm_source_hash() -> str:
    """Hash of the GEMM's device sources with comments and blank space removed: the
    counters depend on the code, so a comment edit keeps the recorded traffic valid. (These
    sources hold no '//' inside string literals.)"""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "epilogues_nvfp4_quantize_b200", "csrc")
    for f in ("gemm.cuh", "ptx.cuh", "codec.cuh", "unfused.cuh"):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"], "bf16_sustained": p["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        self.path = os.path.join("/tmp", f"nvfp4_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", "50", "-i", str(self.gpu)], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, pw, reasons = [], 0.0, [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                s = float(parts[1].split()[0])
                mx = max(mx, float(parts[2].split()[0]))
                w = float(parts[3].split()[0])
            except ValueError:
                continue
            sm.append(s)
            pw.append(w)
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        loaded = [s for s, w in zip(sm, pw) if w > 0.5 * max(pw)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(pw)}


# ----------------------------------------------------------------------------------
# the CUDA arm
# ----------------------------------------------------------------------------------
class Layer:
    """Device-resident weights and activations of one DiT layer's projections."""

    def __init__(self, M: int, dev, seed: int):
        import torch
        import epilogues_nvfp4_quantize_b200 as ep
        import workloads as wk
        self.M, self.dev = M, dev
        T = ep.NVFP4Tensor
        self.x = wk.activations(M, K_IN, wk.outlier_count(K_IN), seed=seed).to(dev)
        std = 1.0 / np.sqrt(K_IN)
        w_qkv = wk.weights(N_QKV, K_IN, std, seed=seed, stream=11).to(dev)
        w_up = wk.weights(N_UP, K_IN, std, seed=seed, stream=12).to(dev)
        w_down = wk.weights(K_IN, K_DOWN, 1.0 / np.sqrt(K_DOWN), seed=seed, stream=13).to(dev)
        # weight packing (offline): quantise, SwiGLU interleave of the gate|up rows
        self.Wqkv, self.Wup, self.Wup_logical, self.Wdown = (T.empty(N_QKV, K_IN, dev), T.empty(N_UP, K_IN, dev),
                                                             T.empty(N_UP, K_IN, dev), T.empty(K_IN, K_DOWN, dev))
        ep.nvfp4_quantize(w_qkv, self.Wqkv)
        ep.nvfp4_quantize(w_up, self.Wup, interleave=True)
        ep.nvfp4_quantize(w_up, self.Wup_logical)
        ep.nvfp4_quantize(w_down, self.Wdown)
        wq = wk.norm_weight(HD, seed, 3)
        wkk = wk.norm_weight(HD, seed, 5)
        self.w_norm = torch.from_numpy(np.concatenate([np.tile(wq, N_NORM // 2 // HD),
                                                       np.tile(wkk, N_NORM // 2 // HD)]).astype(np.float32)).to(dev)
        del w_qkv, w_up, w_down
        self.ws = torch.empty(ep.quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
        self.xq = T.empty(M, K_IN, dev)
        self.qkv = torch.empty(M, N_QKV, dtype=torch.bfloat16, device=dev)
        self.h = T.empty(M, N_UP // 2, dev)
        self.out = torch.empty(M, K_IN, dtype=torch.bfloat16, device=dev)
        # static scale of the re-quantised FFN activations: calibrated once from a bf16
        # run of the fused SwiGLU GEMM (amax / 2688, derived by the library's quantiser)
        ep.nvfp4_quantize(self.x, self.xq, workspace=self.ws)
        hb = torch.empty(M, N_UP // 2, dtype=torch.bfloat16, device=dev)
        ep.gemm_nvfp4_swiglu(self.xq, self.Wup, hb, None)
        ep.nvfp4_quantize(hb, self.h, workspace=self.ws)
        torch.cuda.synchronize(dev)
        del hb

    def step(self, ev=None, x=None, qkv=None, out=None):
        """One step on the current torch stream; x/qkv/out default to the layer's buffers."""
        import epilogues_nvfp4_quantize_b200 as ep
        x = self.x if x is None else x
        qkv = self.qkv if qkv is None else qkv
        out = self.out if out is None else out
        ep.nvfp4_quantize(x, self.xq, workspace=self.ws)
        if ev is not None:
            ev[0].record()
        ep.gemm_nvfp4_rmsnorm(self.xq, self.Wqkv, self.w_norm, HD, N_NORM, EPS, qkv)
        if ev is not None:
            ev[1].record()
        ep.gemm_nvfp4_swiglu(self.xq, self.Wup, None, self.h)
        if ev is not None:
            ev[2].record()
        ep.gemm_nvfp4_plain(self.h, self.Wdown, out)

    # unfused comparison: GEMM -> bf16 in HBM -> separate op kernel(s)
    def alloc_unfused(self):
        import torch
        import epilogues_nvfp4_quantize_b200 as ep
        self.c_up = torch.empty(self.M, N_UP, dtype=torch.bfloat16, device=self.dev)
        self.y_up = torch.empty(self.M, N_UP // 2, dtype=torch.bfloat16, device=self.dev)
        self.h2 = ep.NVFP4Tensor(torch.empty_like(self.h.codes), torch.empty_like(self.h.sf), self.h.gscale,
                                 self.h.rows, self.h.cols)

    def unfused_qkv(self):
        import epilogues_nvfp4_quantize_b200 as ep
        ep.gemm_nvfp4_plain(self.xq, self.Wqkv, self.qkv)
        ep.rmsnorm_heads_bf16(self.qkv, self.w_norm, HD, N_NORM, EPS, self.qkv)

    def unfused_up(self):
        import epilogues_nvfp4_quantize_b200 as ep
        ep.gemm_nvfp4_plain(self.xq, self.Wup_logical, self.c_up)
        ep.swiglu_bf16(self.c_up, self.y_up)
        ep.nvfp4_quantize(self.y_up, self.h2, compute_amax=False)


def max_rel_err(got, ref) -> float:
    """max |g - o| / max(|o|, 1e-2 rms(o)): the bf16 output tolerance rule of the tests."""
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-2 * rms))) if ref.size else 0.0


def vendor_yardstick(layer, M, steps, torch, ep, flops):
    """cuBLASLt NVFP4 (torch._scaled_mm) at the FFN-up and FFN-down shapes on the step's own
    packed operands (the scale buffers already have the 128 x 4 tensor-core layout it
    expects). Never a product path: it shows how much of the tensor pipe a vendor GEMM
    without an epilogue gets on the same GPU."""
    out = {"what": "torch._scaled_mm (cuBLASLt) NVFP4, bf16 out, no epilogue, same operands"}
    try:
        f4, f8 = torch.float4_e2m1fn_x2, torch.float8_e4m3fn
        cases = {"ffn_up": (layer.xq, layer.Wup_logical, flops["up"]),
                 "ffn_down": (layer.h, layer.Wdown, flops["down"])}
        for name, (A, B, fl) in cases.items():
            a = A.codes.view(f4)
            b = B.codes.view(f4)
            sa = A.sf.view(f8).view(A.rows, A.cols // 16)
            sb = B.sf.view(f8).view(B.rows, B.cols // 16)
            D = torch.empty(A.rows, B.rows, dtype=torch.bfloat16, device=A.codes.device)
            t_v = time_loop(lambda: torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16), steps, 3, torch)
            t_o = time_loop(lambda: ep.gemm_nvfp4_plain(A, B, D), steps, 3, torch)
            out[name] = {"vendor_us": round(t_v * 1e3, 1), "vendor_tflops": round(fl / (t_v * 1e-3) / 1e12, 1),
                         "ours_plain_us": round(t_o * 1e3, 1), "ours_tflops": round(fl / (t_o * 1e-3) / 1e12, 1)}
            del D
    except Exception as e:  # the vendor path is optional context, never required
        out["error"] = f"{type(e).__name__}: {e}"[:200]
    return out


def time_loop(fn, steps, warmup, torch):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


def run_cuda(args):
    import torch
    import torch.distributed as dist
    import epilogues_nvfp4_quantize_b200 as ep
    from epilogues_nvfp4_quantize_b200.build import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    ep.load()

    M = args.M
    layer = Layer(M, dev, seed=rank)
    flops = step_flops(M)
    total_flops = sum(flops.values())

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---- warm-up; its outputs are the reference of the timed steps' outputs (same inputs,
    # deterministic kernels: every timed step must reproduce them bit for bit)
    for _ in range(args.warmup):
        layer.step()
    barrier()
    qkv_warm, out_warm = layer.qkv.clone(), layer.out.clone()
    ep.read_device_status()  # start the timed region with a clear status word

    # ---- timed region: K back-to-back steps (inputs x + weights exceed the L2)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    n0 = ep.launch_count()
    with ClockSampler(local) as clk:
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for i in range(K):
            ev_s[i].record()
            layer.step(ev[i])
            ev_e[i].record()
        stop.record()
        torch.cuda.synchronize(dev)
    launches = ep.launch_count() - n0
    # the timed steps checked themselves: no bounded wait gave up (device status word) and
    # the last step's outputs equal the warm-up's
    status = ep.read_device_status()
    output_ok = bool(torch.equal(layer.qkv, qkv_warm) and torch.equal(layer.out, out_warm))
    del qkv_warm, out_warm
    check_rows = np.sort(np.random.default_rng([7, M]).choice(M, size=min(64, M), replace=False))
    sel = torch.from_numpy(check_rows).to(dev)
    last_qkv = layer.qkv[sel].float().cpu().numpy().astype(np.float64)
    last_out = layer.out[sel].float().cpu().numpy().astype(np.float64)
    ms_total = max_over_ranks(start.elapsed_time(stop), dev)
    ms_step = ms_total / K
    per = {"quantize_x": [], "qkv_rmsnorm": [], "up_swiglu_requant": [], "down_plain": []}
    for i in range(K):
        per["quantize_x"].append(ev_s[i].elapsed_time(ev[i][0]))
        per["qkv_rmsnorm"].append(ev[i][0].elapsed_time(ev[i][1]))
        per["up_swiglu_requant"].append(ev[i][1].elapsed_time(ev[i][2]))
        per["down_plain"].append(ev[i][2].elapsed_time(ev_e[i]))
    avg = {k: sum(v) / len(v) for k, v in per.items()}
    value = whole_job_tflops(total_flops, world, ms_step)
    clocks = clk.summary()

    pk = peaks()
    fp4_peak = pk["bf16"] * FP4_PER_BF16
    up_tflops = flops["up"] / (avg["up_swiglu_requant"] * 1e-3) / 1e12
    kernels = {
        "quantize_x": {"us": avg["quantize_x"] * 1e3,
                       "gbs": (M * K_IN * 2 + M * K_IN * (0.5 + 1 / 16)) / (avg["quantize_x"] * 1e-3) / 1e9},
        "qkv_rmsnorm": {"us": avg["qkv_rmsnorm"] * 1e3,
                        "tflops": flops["qkv"] / (avg["qkv_rmsnorm"] * 1e-3) / 1e12},
        "up_swiglu_requant": {"us": avg["up_swiglu_requant"] * 1e3, "tflops": up_tflops},
        "down_plain": {"us": avg["down_plain"] * 1e3,
                       "tflops": flops["down"] / (avg["down_plain"] * 1e-3) / 1e12},
    }
    for k in ("qkv_rmsnorm", "up_swiglu_requant", "down_plain"):
        kernels[k]["pct_fp4_peak"] = 100.0 * kernels[k]["tflops"] / fp4_peak

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": workload_desc(M), "M": M, "K": K_IN, "N_qkv": N_QKV, "N_up": N_UP,
                   "K_down": K_DOWN, "head_dim": HD, "global_batch_tokens": M * world,
                   "parallelism": f"dp{world} (independent token batches, no collective)",
                   "l2": "no flush: per-step inputs (x 100.7 MB + packed weights 75 MB) exceed the 126 MB L2"},
        "roofline": {"bound": "tensor",
                     "kernel": ("gemm_nvfp4_pair_kernel<EPI_SWIGLU>" if M > 128 else
                                "gemm_nvfp4_kernel<EPI_SWIGLU>") + " (FFN-up, SwiGLU + NVFP4 re-quantisation)",
                     "achieved": round(up_tflops, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(up_tflops / fp4_peak, 4),
                     "traffic": args.traffic if args.traffic is not None else
                     (TRAFFIC_BY_SOURCE.get(gemm_source_hash()) if M == 16384 else None),
                     "peak_source": f"{pk['source']} bf16 {pk['bf16']} TFLOP/s x {FP4_PER_BF16} (nominal dense "
                                    f"FP4:BF16 ratio), burst figure",
                     "frac_of_sustained": round(up_tflops / (pk["bf16_sustained"] * FP4_PER_BF16), 4)},
        "kernels": kernels,
        "gpu_launches": launches,
        "clocks": clocks,
        "status_ok": status == 0,
        "output_ok": output_ok,
    }
    result["roofline"]["peak_datasheet"] = FP4_DATASHEET_TFLOPS
    result["roofline"]["frac_of_datasheet"] = round(up_tflops / FP4_DATASHEET_TFLOPS, 4)
    for k in ("qkv_rmsnorm", "up_swiglu_requant", "down_plain"):
        kernels[k]["pct_fp4_datasheet"] = round(100.0 * kernels[k]["tflops"] / FP4_DATASHEET_TFLOPS, 2)
    kernels["quantize_x"]["pct_hbm"] = round(100.0 * kernels["quantize_x"]["gbs"] / pk["hbm_gbs"], 1)
    # the same call alone, back to back: in the step it follows the FFN-down GEMM, whose
    # dirty bf16 output in L2 is written back to HBM while x streams in
    t_q = time_loop(lambda: ep.nvfp4_quantize(layer.x, layer.xq, workspace=layer.ws), 100, 5, torch)
    q_gbs = (M * K_IN * 2 + M * K_IN * (0.5 + 1 / 16)) / (t_q * 1e-3) / 1e9
    kernels["quantize_x"]["alone"] = {"us": round(t_q * 1e3, 2), "gbs": round(q_gbs, 1),
                                      "pct_hbm": round(100.0 * q_gbs / pk["hbm_gbs"], 1),
                                      "how": "100 calls back to back after the timed steps"}

    # ---- unfused comparison (separately timed, same step shapes)
    if not args.no_unfused:
        layer.alloc_unfused()
        barrier()
        t_fused_qkv = time_loop(lambda: ep.gemm_nvfp4_rmsnorm(layer.xq, layer.Wqkv, layer.w_norm, HD, N_NORM, EPS,
                                                              layer.qkv), args.cmp_steps, 3, torch)
        t_unf_qkv = time_loop(layer.unfused_qkv, args.cmp_steps, 3, torch)
        t_fused_up = time_loop(lambda: ep.gemm_nvfp4_swiglu(layer.xq, layer.Wup, None, layer.h), args.cmp_steps, 3,
                               torch)
        t_unf_up = time_loop(layer.unfused_up, args.cmp_steps, 3, torch)
        # the unfused path's op kernels alone, with the HBM bytes each must move
        t_rms = time_loop(lambda: ep.rmsnorm_heads_bf16(layer.qkv, layer.w_norm, HD, N_NORM, EPS, layer.qkv),
                          args.cmp_steps, 3, torch)
        t_swi = time_loop(lambda: ep.swiglu_bf16(layer.c_up, layer.y_up), args.cmp_steps, 3, torch)
        t_rq = time_loop(lambda: ep.nvfp4_quantize(layer.y_up, layer.h2, compute_amax=False), args.cmp_steps, 3,
                         torch)
        b_rms = M * N_NORM * 2 * 2                           # read + write the normalised bf16 columns
        b_swi = M * N_UP * 2 + M * (N_UP // 2) * 2           # read gate|up, write the product
        b_rq = M * (N_UP // 2) * (2 + 0.5 + 1 / 16)         # read bf16, write codes + scales
        op_kernels = {
            "rmsnorm_heads_bf16": {"us": round(t_rms * 1e3, 1), "gbs": round(b_rms / (t_rms * 1e-3) / 1e9, 1)},
            "swiglu_bf16": {"us": round(t_swi * 1e3, 1), "gbs": round(b_swi / (t_swi * 1e-3) / 1e9, 1)},
            "nvfp4_quantize_static": {"us": round(t_rq * 1e3, 1), "gbs": round(b_rq / (t_rq * 1e-3) / 1e9, 1)},
            "hbm_peak_gbs": pk["hbm_gbs"],
        }
        result["unfused"] = {
            "qkv": {"fused_us": t_fused_qkv * 1e3, "unfused_us": t_unf_qkv * 1e3,
                    "speedup": t_unf_qkv / t_fused_qkv},
            "ffn_up": {"fused_us": t_fused_up * 1e3, "unfused_us": t_unf_up * 1e3,
                       "speedup": t_unf_up / t_fused_up},
            "note": "unfused = plain NVFP4 GEMM writing bf16, then rmsnorm_heads_bf16 (in place) / "
                    "swiglu_bf16 + nvfp4_quantize (static scale); same kernels' library",
            "op_kernels": op_kernels,
        }
        del layer.c_up, layer.y_up
        torch.cuda.empty_cache()

    # ---- pointwise epilogues (bias, ReLU, cast, NVFP4 output) on the FFN-down GEMM
    if not args.no_unfused:
        bias = torch.randn(K_IN, device=dev, dtype=torch.float32) * 0.01
        d32 = torch.empty(M, K_IN, dtype=torch.float32, device=dev)
        dq = ep.NVFP4Tensor.empty(M, K_IN, dev)
        dq.gscale.fill_(float(layer.out.float().abs().max().item()) / 2688)
        red_ptrs = torch.tensor([d32.data_ptr()], dtype=torch.int64, device=dev)
        barrier()
        cases = {
            "plain_bf16": lambda: ep.gemm_nvfp4_plain(layer.h, layer.Wdown, layer.out),
            "bias_relu_bf16": lambda: ep.gemm_nvfp4_pointwise(layer.h, layer.Wdown, layer.out, bias=bias, relu=True),
            "bias_f32": lambda: ep.gemm_nvfp4_pointwise(layer.h, layer.Wdown, d32, bias=bias),
            "bias_relu_nvfp4_only": lambda: ep.gemm_nvfp4_pointwise(layer.h, layer.Wdown, None, bias=bias, relu=True,
                                                                   Dq=dq),
            # the row-parallel down GEMM with its reduction fused in, into this GPU's own block
            # (world size 1): atomic float32 additions instead of the f32 TMA stores above
            "reduce_rows_f32": lambda: ep.gemm_nvfp4_reduce_rows_f32(layer.h, layer.Wdown, red_ptrs, M, K_IN),
        }
        pw = {}
        for name, fn in cases.items():
            t = time_loop(fn, args.cmp_steps, 3, torch)
            pw[name] = {"us": round(t * 1e3, 1), "tflops": round(flops["down"] / (t * 1e-3) / 1e12, 1)}
        pw["shape"] = f"M={M} K={K_DOWN} N={K_IN} (FFN-down)"
        result["pointwise"] = pw
        del d32, dq

    # ---- MXFP4 with the block Hadamard transform: same GEMM shapes, E8M0 scales per 32
    if not args.no_unfused:
        T = ep.NVFP4Tensor
        xm = ep.mxfp4_quantize(layer.x, T.empty_mx(M, K_IN, dev), hadamard=True)
        w_up_bf16 = torch.randn(N_UP, K_IN, device=dev, dtype=torch.bfloat16) * (1.0 / K_IN ** 0.5)
        wm = ep.mxfp4_quantize(w_up_bf16, T.empty_mx(N_UP, K_IN, dev), hadamard=True)
        c_mx = torch.empty(M, N_UP, dtype=torch.bfloat16, device=dev)
        c_nv = torch.empty(M, N_UP, dtype=torch.bfloat16, device=dev)
        barrier()
        t_mx = time_loop(lambda: ep.gemm_mxfp4_plain(xm, wm, c_mx), args.cmp_steps, 3, torch)
        t_nv = time_loop(lambda: ep.gemm_nvfp4_plain(layer.xq, layer.Wup_logical, c_nv), args.cmp_steps, 3, torch)
        t_q = time_loop(lambda: ep.mxfp4_quantize(layer.x, xm, hadamard=True), args.cmp_steps, 3, torch)
        result["mxfp4"] = {
            "shape": f"M={M} K={K_IN} N={N_UP} (FFN-up, bf16 out, no epilogue op)",
            "gemm_us": round(t_mx * 1e3, 1), "gemm_tflops": round(flops["up"] / (t_mx * 1e-3) / 1e12, 1),
            "nvfp4_same_shape_us": round(t_nv * 1e3, 1),
            "quantize_hadamard_us": round(t_q * 1e3, 1),
            "quantize_gbs": round(layer.x.numel() * (2 + 0.5 + 1 / 32) / (t_q * 1e-3) / 1e9, 1),
        }
        del xm, wm, c_mx, c_nv, w_up_bf16

    # ---- vendor yardstick: cuBLASLt's NVFP4 GEMM (torch._scaled_mm, no epilogue, bf16 out)
    # on this step's own operands, against this library's plain GEMM of the same shapes
    if not args.no_unfused:
        result["yardstick"] = vendor_yardstick(layer, M, args.cmp_steps, torch, ep, flops)

    # ---- a small-batch step (serving): eager launches vs one CUDA-graph replay
    if not args.no_unfused:
        small = Layer(1024, dev, seed=rank + 100)
        barrier()
        t_eager = time_loop(small.step, args.cmp_steps, 3, torch)
        gs = torch.cuda.Stream(dev)
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            small.step()
        torch.cuda.current_stream().wait_stream(gs)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            small.step()
        t_graph = time_loop(graph.replay, args.cmp_steps, 3, torch)
        fl_small = sum(step_flops(1024).values())
        result["small_batch_graph"] = {
            "M": 1024, "eager_us": round(t_eager * 1e3, 1), "graph_us": round(t_graph * 1e3, 1),
            "eager_tflops": round(fl_small / (t_eager * 1e-3) / 1e12, 1),
            "graph_tflops": round(fl_small / (t_graph * 1e-3) / 1e12, 1),
        }
        del graph, small
        torch.cuda.empty_cache()

    # ---- fake quantisation (quantization-aware distillation forward), HBM-bound
    if not args.no_unfused:
        y_fq = torch.empty_like(layer.x)
        g_fq = torch.empty(1, dtype=torch.float32, device=dev)
        barrier()
        t_fq = time_loop(lambda: ep.nvfp4_fake_quantize(layer.x, y=y_fq, gscale=g_fq, workspace=layer.ws),
                         args.cmp_steps, 3, torch)
        t_fq_static = time_loop(lambda: ep.nvfp4_fake_quantize(layer.x, y=y_fq, gscale=g_fq, compute_amax=False),
                                args.cmp_steps, 3, torch)
        fq_bytes = layer.x.numel() * 4  # read x, write y (bf16)
        result["fake_quant"] = {
            "shape": list(layer.x.shape),
            "amax_us": round(t_fq * 1e3, 2), "static_us": round(t_fq_static * 1e3, 2),
            "amax_gbs": round(fq_bytes / (t_fq * 1e-3) / 1e9, 1),
            "static_gbs": round(fq_bytes / (t_fq_static * 1e-3) / 1e9, 1),
            "hbm_peak_gbs": pk["hbm_gbs"],
            "note": "algorithmic bytes = 2 B read + 2 B written per element; with amax the kernel "
                    "reads x twice",
        }
        del y_fq

    # ---- end to end through the public API with host buffers: every step copies its input
    # from pinned host memory and its outputs (QKV and FFN-down) back. Steps are pipelined
    # over three streams (host->device, compute, device->host) with two device buffer sets,
    # so the copies of neighbouring steps overlap this step's kernels (PCIe is full duplex).
    if not args.no_e2e:
        import workloads as wk
        n_e2e = max(2, min(K // 2, 60))
        # two different inputs alternate, so a step that read or returned a stale buffer
        # would fail the output check; each input's outputs computed eagerly beforehand
        x_host = [layer.x.cpu().pin_memory(),
                  wk.activations(M, K_IN, wk.outlier_count(K_IN), seed=rank + 1000).pin_memory()]
        ref_out = []
        for xb in x_host:
            layer.step(x=xb.to(dev))
            ref_out.append((layer.qkv.cpu(), layer.out.cpu()))
        qkv_host = [torch.empty(layer.qkv.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        out_host = [torch.empty(layer.out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_dev = [layer.x, torch.empty_like(layer.x)]
        qkv_dev = [layer.qkv, torch.empty_like(layer.qkv)]
        out_dev = [layer.out, torch.empty_like(layer.out)]
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        started = [False, False]

        def e2e_steps(n, start_ev=None, stop_ev=None):
            if start_ev is not None:
                start_ev.record(s_in)
                s_cmp.wait_event(start_ev)
                s_out.wait_event(start_ev)
            for i in range(n):
                b = i & 1
                with torch.cuda.stream(s_in):
                    if started[b]:
                        s_in.wait_event(ev_cmp[b])  # the compute of step i-2 has read x_dev[b]
                    x_dev[b].copy_(x_host[b], non_blocking=True)
                    ev_in[b].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[b])
                    if started[b]:
                        s_cmp.wait_event(ev_out[b])  # step i-2's outputs have left the device
                    layer.step(x=x_dev[b], qkv=qkv_dev[b], out=out_dev[b])
                    ev_cmp[b].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[b])
                    qkv_host[b].copy_(qkv_dev[b], non_blocking=True)
                    out_host[b].copy_(out_dev[b], non_blocking=True)
                    ev_out[b].record(s_out)
                started[b] = True
            if stop_ev is not None:
                s_in.wait_stream(s_out)
                s_in.wait_stream(s_cmp)
                stop_ev.record(s_in)

        barrier()
        e2e_steps(3)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps(n_e2e, e0, e1)
        torch.cuda.synchronize(dev)
        t_e2e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dev)
        ok = all(torch.equal(qkv_host[b], ref_out[b][0]) and torch.equal(out_host[b], ref_out[b][1])
                 for b in (0, 1))
        result["e2e"] = {"value": round(whole_job_tflops(total_flops, world, t_e2e), 2), "unit": "TFLOP/s",
                         "h2d_bytes_per_step": int(x_host[0].numel() * 2),
                         "d2h_bytes_per_step": int((qkv_host[0].numel() + out_host[0].numel()) * 2),
                         "ms_per_step": round(t_e2e, 4), "steps": n_e2e,
                         "pipelined": "3 streams (h2d, compute, d2h), 2 device buffer sets",
                         "inputs": "two different host inputs, alternating",
                         "output_check": ok}
        del ref_out
        del x_dev[1], qkv_dev[1], out_dev[1]

    if rank == 0 and world == 1 and not args.no_cpu:
        # the oracle checks the last timed step on seeded rows (the FFN activations
        # re-quantised with the same static scale as the GPU's), then is timed as the CPU
        # baseline
        ol = OracleLayer(M)
        ol.Gh = np.float32(layer.h.gscale.item())
        qkv_o, out_o = ol.step(check_rows)
        e_qkv = max_rel_err(last_qkv, qkv_o)
        # the FFN-down output comes from re-quantised activations, whose codes may differ
        # from the oracle's where the bf16 inputs differ: judged per element against
        # 2e-2 |o| + 2e-2 rms(o), and normwise
        rms_o = float(np.sqrt(np.mean(out_o * out_o)))
        out_over = int(np.sum(np.abs(last_out - out_o) > 2e-2 * np.abs(out_o) + 2e-2 * rms_o))
        out_norm = float(np.linalg.norm(last_out - out_o) / max(np.linalg.norm(out_o), 1e-300))
        result["oracle_check"] = {"rows": len(check_rows), "qkv_max_rel": round(e_qkv, 5), "qkv_tolerance": 2e-2,
                                  "out_elements_over": out_over, "out_normwise": round(out_norm, 6),
                                  "ok": bool(e_qkv <= 2e-2 and out_over == 0 and out_norm <= 1e-3)}
        result["cpu_baseline"] = cpu_baseline(M, rows=args.cpu_rows, layer=ol)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))
    if not (result["status_ok"] and result["output_ok"]):
        raise SystemExit(f"timed steps failed their self-check: status_ok={result['status_ok']} "
                         f"output_ok={result['output_ok']}")


# ----------------------------------------------------------------------------------
# the CPU oracle arm
# ----------------------------------------------------------------------------------
class OracleLayer:
    """The oracle's pieces of the same step; weight packing done once (model load)."""

    def __init__(self, M: int, seed: int = 0):
        from oracle import nvfp4_oracle as o
        import workloads as wk
        self.o = o
        self.M = M
        self.x = wk.activations(M, K_IN, wk.outlier_count(K_IN), seed=seed).float().numpy()
        std = 1.0 / np.sqrt(K_IN)
        t0 = time.perf_counter()
        self.Bqkv = o.dequantize(*o.quantize_fp32_order(wk.weights(N_QKV, K_IN, std, seed=seed, stream=11).float().numpy()))
        self.Bup = o.dequantize(*o.quantize_fp32_order(wk.weights(N_UP, K_IN, std, seed=seed, stream=12).float().numpy()))
        self.Bdown = o.dequantize(*o.quantize_fp32_order(
            wk.weights(K_IN, K_DOWN, 1.0 / np.sqrt(K_DOWN), seed=seed, stream=13).float().numpy()))
        self.pack_s = time.perf_counter() - t0
        wq, wkk = wk.norm_weight(HD, seed, 3), wk.norm_weight(HD, seed, 5)
        self.w = np.concatenate([np.tile(wq, N_NORM // 2 // HD), np.tile(wkk, N_NORM // 2 // HD)])
        self.Gx = o.global_scale(self.x)
        self.Gh = None

    def step(self, rows):
        o = self.o
        xs = self.x[rows]
        qa, sa, _ = o.quantize_fp32_order(xs, self.Gx)
        a = o.dequantize(qa, sa, self.Gx)
        qkv = o.bf16_round(o.rmsnorm_heads(o.gemm(a, self.Bqkv), self.w, HD, N_NORM, EPS))
        h = o.bf16_round(o.swiglu(o.gemm(a, self.Bup)))
        if self.Gh is None:
            self.Gh = np.float32(np.abs(h).max() / 2688)
        qh, sh, _ = o.requantize(h, self.Gh)
        out = o.bf16_round(o.gemm(o.dequantize(qh, sh, self.Gh), self.Bdown))
        return qkv, out


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:  # pragma: no cover
        return os.cpu_count()


def _timed_rows(layer, sample, chunk=1024):
    """Seconds for the oracle step over `sample`, run in row chunks so memory stays bounded."""
    t0 = time.perf_counter()
    for i in range(0, len(sample), chunk):
        layer.step(sample[i:i + chunk])
    return time.perf_counter() - t0


def cpu_baseline(M: int, rows: int = 0, target_s: float = 10.0, layer=None):
    """The oracle timed on a bounded sample of the step's rows. rows=0 sizes the sample by time:
    a 256-row probe, then enough rows for about `target_s` seconds of CPU work (at most M). One
    core is timed the same way with a third of the target. `layer`: an OracleLayer of M rows
    (built here when None)."""
    layer = OracleLayer(M) if layer is None else layer
    rng = np.random.default_rng(0)
    order = rng.permutation(M)

    def pick(n):
        return np.sort(order[:n])

    def sized(budget):
        probe = min(256, M)
        d = _timed_rows(layer, pick(probe))
        if rows:
            n = min(rows, M)
        else:
            n = min(M, max(probe, int(probe * budget / max(d, 1e-6)) // 64 * 64))
        if n == probe:
            return n, d
        return n, _timed_rows(layer, pick(n))

    n, dt = sized(target_s)
    fl = sum(step_flops(n).values())
    out = {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{n} random rows of the M={M} step (quantise, fp64 GEMMs, RMSNorm, SwiGLU, requant, "
                     f"down GEMM) in {dt:.2f} s; weight packing ({layer.pack_s:.1f} s, once per model) excluded",
           "host_threads": os.cpu_count()}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            n1, d1 = sized(target_s / 3) if not rows else (max(8, n // 4), _timed_rows(layer, pick(max(8, n // 4))))
        out["one_core"] = {"value": round(sum(step_flops(n1).values()) / d1 / 1e12, 6), "unit": "TFLOP/s",
                           "sample": f"{n1} rows in {d1:.2f} s"}
    except ImportError:  # pragma: no cover
        pass
    return out


# ----------------------------------------------------------------------------------
# the M sweep: fused vs unfused, cold and warm L2
# ----------------------------------------------------------------------------------
def run_sweep(args):
    """Fused vs unfused for M in {1024, 4096, 8192, 16384} x {QKV hd128, QKV hd256, FFN-up
    with NVFP4 re-quantisation}. Each run is timed alone with CUDA events: cold (a 512 MB
    buffer written before each run, primary) and warm (no scrub). 10 warm-ups, then the
    median of --sweep-runs runs."""
    import torch
    import epilogues_nvfp4_quantize_b200 as ep
    import workloads as wk
    from epilogues_nvfp4_quantize_b200.build import build

    build()
    ep.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T = ep.NVFP4Tensor
    scrub = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    pk = peaks()
    fp4_peak = pk["bf16"] * FP4_PER_BF16

    def median_us(fn, cold, runs):
        for _ in range(10):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(runs)]
        for e0, e1 in evs:
            if cold:
                scrub.fill_(1)
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize(dev)
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs) * 1e3

    rows = []
    n_launch0 = ep.launch_count()
    for wl in wk.sweep():
        inp = wk.make_inputs(wl)
        a, b = inp["a"].to(dev), inp["b"].to(dev)
        M, K, N = wl.M, wl.K, wl.N
        A = T.empty(M, K, dev)
        ep.nvfp4_quantize(a, A)
        if wl.op == "rmsnorm":
            B = T.empty(N, K, dev)
            ep.nvfp4_quantize(b, B)
            w = torch.from_numpy(inp["w"]).to(dev)
            D = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

            def fused():
                ep.gemm_nvfp4_rmsnorm(A, B, w, wl.head_dim, wl.n_norm_cols, wl.eps, D)

            def unfused():
                ep.gemm_nvfp4_plain(A, B, D)
                ep.rmsnorm_heads_bf16(D, w, wl.head_dim, wl.n_norm_cols, wl.eps, D)
        else:
            nh = N // 2
            Bi, Bl = T.empty(N, K, dev), T.empty(N, K, dev)
            ep.nvfp4_quantize(b, Bi, interleave=True)
            ep.nvfp4_quantize(b, Bl)
            Dq = T.empty(M, nh, dev)
            hb = torch.empty(M, nh, dtype=torch.bfloat16, device=dev)
            ep.gemm_nvfp4_swiglu(A, Bi, hb, None)
            ep.nvfp4_quantize(hb, Dq)  # static scale of the re-quantised output, calibrated once
            del hb
            Dq2 = T(torch.empty_like(Dq.codes), torch.empty_like(Dq.sf), Dq.gscale, M, nh)
            C = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            Y = torch.empty(M, nh, dtype=torch.bfloat16, device=dev)

            def fused():
                ep.gemm_nvfp4_swiglu(A, Bi, None, Dq)

            def unfused():
                ep.gemm_nvfp4_plain(A, Bl, C)
                ep.swiglu_bf16(C, Y)
                ep.nvfp4_quantize(Y, Dq2, compute_amax=False)
        r = {"workload": wl.name, "M": M, "op": wl.op, "head_dim": wl.head_dim}
        for mode, cold in (("cold", True), ("warm", False)):
            tf, tu = median_us(fused, cold, args.sweep_runs), median_us(unfused, cold, args.sweep_runs)
            r[mode] = {"fused_us": round(tf, 2), "unfused_us": round(tu, 2), "speedup": round(tu / tf, 3),
                       "fused_tflops": round(wl.flops / (tf * 1e-6) / 1e12, 1),
                       "pct_fp4_peak": round(100.0 * wl.flops / (tf * 1e-6) / 1e12 / fp4_peak, 1)}
        rows.append(r)
        print(json.dumps(r), flush=True)
        del A, a, b
        torch.cuda.empty_cache()
    status = ep.read_device_status()
    print(json.dumps({"sweep": "fused vs unfused", "runs": args.sweep_runs, "warmup": 10,
                      "fp4_peak_tflops": round(fp4_peak, 1), "peak_source": pk["source"],
                      "launches": ep.launch_count() - n_launch0, "device_status": status}), flush=True)
    if status != 0:
        raise SystemExit(f"device status {status}")


# ----------------------------------------------------------------------------------
# the named configurations: fused vs unfused, each timed alone
# ----------------------------------------------------------------------------------
def run_configs(args):
    """The five named problems (the tiny QK-norm case, SwiGLU at M=1024, the 1K-image QKV
    block, the 1K-image FFN block's up GEMM with re-quantisation and its down GEMM), each
    timed alone like the sweep: cold L2 (a 512 MB buffer written before each run), 10
    warm-ups, median of --sweep-runs runs, fused against the plain GEMM plus separate op
    kernels. cpu_baseline per problem: the oracle on a row sample (all rows of the tiny
    case), with B's packing done before timing, extrapolated linearly in M."""
    import torch
    import epilogues_nvfp4_quantize_b200 as ep
    import workloads as wk
    from oracle import nvfp4_oracle as o
    from epilogues_nvfp4_quantize_b200.build import build

    build()
    ep.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T = ep.NVFP4Tensor
    scrub = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    pk = peaks()
    fp4_peak = pk["bf16"] * FP4_PER_BF16
    cores = _blas_threads()

    def median_us(fn, runs):
        for _ in range(10):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(runs)]
        for e0, e1 in evs:
            scrub.fill_(1)
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize(dev)
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs) * 1e3

    def oracle_s(wl, a, b, w=None, sample=256):
        rows = None if wl.M <= sample else np.sort(np.random.default_rng(0).choice(wl.M, size=sample,
                                                                                    replace=False))
        bq = o.quantized_operand(b)  # weight packing, once per model: not timed
        t0 = time.perf_counter()
        if wl.op == "rmsnorm":
            o.problem_rmsnorm(a, b, w, wl.head_dim, wl.n_norm_cols, wl.eps, rows=rows, b_quant=bq)
        elif wl.op == "swiglu":
            ref = o.problem_swiglu(a, b, rows=rows, b_quant=bq)
            if wl.requant:
                o.requantize(ref, np.float32(np.abs(ref).max() / 2688))
        else:
            o.problem_plain(a, b, rows=rows, b_quant=bq)
        t = time.perf_counter() - t0
        n = wl.M if rows is None else len(rows)
        return t * wl.M / n, n

    n_launch0 = ep.launch_count()
    down_a = None
    for name, wl in (("1", wk.qk_norm_tiny()), ("2", wk.swiglu_1024()), ("3", wk.qkv(4096, 256)),
                     ("4a", wk.ffn_up(4096, True)), ("4b", wk.ffn_down(4096))):
        inp = wk.make_inputs(wl)
        a_cpu, b_cpu = inp["a"], inp["b"]
        a, b = a_cpu.to(dev), b_cpu.to(dev)
        M, K, N = wl.M, wl.K, wl.N
        A = T.empty(M, K, dev)
        ep.nvfp4_quantize(a, A)
        w_cpu = None
        if wl.op == "rmsnorm":
            B = T.empty(N, K, dev)
            ep.nvfp4_quantize(b, B)
            w_cpu = inp["w"]
            w = torch.from_numpy(w_cpu).to(dev)
            D = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

            def fused():
                ep.gemm_nvfp4_rmsnorm(A, B, w, wl.head_dim, wl.n_norm_cols, wl.eps, D)

            def unfused():
                ep.gemm_nvfp4_plain(A, B, D)
                ep.rmsnorm_heads_bf16(D, w, wl.head_dim, wl.n_norm_cols, wl.eps, D)
        elif wl.op == "swiglu":
            nh = N // 2
            Bi, Bl = T.empty(N, K, dev), T.empty(N, K, dev)
            ep.nvfp4_quantize(b, Bi, interleave=True)
            ep.nvfp4_quantize(b, Bl)
            C = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            Y = torch.empty(M, nh, dtype=torch.bfloat16, device=dev)
            if wl.requant:
                Dq = T.empty(M, nh, dev)
                ep.gemm_nvfp4_swiglu(A, Bi, Y, None)
                ep.nvfp4_quantize(Y, Dq)  # static scale of the re-quantised output, calibrated once
                Dq2 = T(torch.empty_like(Dq.codes), torch.empty_like(Dq.sf), Dq.gscale, M, nh)
                down_a = Dq  # the down GEMM's A, as in the FFN block

                def fused():
                    ep.gemm_nvfp4_swiglu(A, Bi, None, Dq)

                def unfused():
                    ep.gemm_nvfp4_plain(A, Bl, C)
                    ep.swiglu_bf16(C, Y)
                    ep.nvfp4_quantize(Y, Dq2, compute_amax=False)
            else:
                D = torch.empty(M, nh, dtype=torch.bfloat16, device=dev)

                def fused():
                    ep.gemm_nvfp4_swiglu(A, Bi, D, None)

                def unfused():
                    ep.gemm_nvfp4_plain(A, Bl, C)
                    ep.swiglu_bf16(C, Y)
        else:
            B = T.empty(N, K, dev)
            ep.nvfp4_quantize(b, B)
            Ad = down_a if down_a is not None else A
            D = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

            def fused():
                ep.gemm_nvfp4_plain(Ad, B, D)

            unfused = None  # a plain GEMM has no op to split off
        tf = median_us(fused, args.sweep_runs)
        tu = median_us(unfused, args.sweep_runs) if unfused is not None else None
        t_cpu, n_rows = oracle_s(wl, a_cpu, b_cpu, w_cpu)
        r = {"config": name, "workload": wl.name, "gflop": round(wl.flops / 1e9, 2), "fused_us": round(tf, 2),
             "fused_tflops": round(wl.flops / (tf * 1e-6) / 1e12, 1),
             "pct_fp4_peak": round(100.0 * wl.flops / (tf * 1e-6) / 1e12 / fp4_peak, 1),
             "unfused_us": None if tu is None else round(tu, 2),
             "speedup": None if tu is None else round(tu / tf, 3),
             "cpu_baseline": {"seconds": round(t_cpu, 2), "cores": cores, "kind": "oracle",
                              "sample": "all rows" if n_rows == M else f"{n_rows} rows, scaled to M={M}"}}
        print(json.dumps(r), flush=True)
        torch.cuda.empty_cache()
    status = ep.read_device_status()
    print(json.dumps({"configs": "fused vs unfused, cold L2", "runs": args.sweep_runs, "warmup": 10,
                      "fp4_peak_tflops": round(fp4_peak, 1), "peak_source": pk["source"],
                      "launches": ep.launch_count() - n_launch0, "device_status": status}), flush=True)
    if status != 0:
        raise SystemExit(f"device status {status}")


def run_quantize_only(args):
    """The activation quantiser alone on the step's x (M x 3072 bf16), with the amax pass and
    with a static scale, timed with CUDA events two ways: each call after a 256 MB buffer is
    written (so L2 starts with other data, as in the step; median of `steps` calls), and at
    least 200 calls back to back with nothing in between (their mean). One JSON line."""
    import torch
    import epilogues_nvfp4_quantize_b200 as ep
    import workloads as wk
    from epilogues_nvfp4_quantize_b200.build import build

    build()
    ep.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    M = args.M
    x = wk.activations(M, K_IN, wk.outlier_count(K_IN), seed=0).to(dev)
    xq = ep.NVFP4Tensor.empty(M, K_IN, dev)
    ws = torch.empty(ep.quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
    scrub = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)

    def timed(fn, n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i, (e0, e1) in enumerate(evs):
            scrub.fill_(i & 255)
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize(dev)
        return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs) * 1e3

    def loop(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n * 1e3

    n = max(args.steps, 1)
    for _ in range(args.warmup):
        ep.nvfp4_quantize(x, xq, workspace=ws)
    t_amax = timed(lambda: ep.nvfp4_quantize(x, xq, workspace=ws), n)
    t_static = timed(lambda: ep.nvfp4_quantize(x, xq, compute_amax=False), n)
    n_loop = max(200, n)  # long enough for the back-to-back steady state
    l_amax = loop(lambda: ep.nvfp4_quantize(x, xq, workspace=ws), n_loop)
    l_static = loop(lambda: ep.nvfp4_quantize(x, xq, compute_amax=False), n_loop)
    status = ep.read_device_status()
    algo = M * K_IN * (2 + 0.5 + 1 / 16)

    def gbs(t):
        return round(algo / (t * 1e-6) / 1e9, 1)

    print(json.dumps({"quantize": f"{M}x{K_IN} bf16", "calls": n, "amax_us": round(t_amax, 2),
                      "static_us": round(t_static, 2), "amax_gbs": gbs(t_amax), "static_gbs": gbs(t_static),
                      "back_to_back": {"calls": n_loop, "amax_us": round(l_amax, 2), "static_us": round(l_static, 2),
                                       "amax_gbs": gbs(l_amax), "static_gbs": gbs(l_static)},
                      "hbm_peak_gbs": peaks()["hbm_gbs"], "device_status": status}))
    if status != 0:
        raise SystemExit(f"device status {status}")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    layer = OracleLayer(args.M)
    rng = np.random.default_rng(1)
    rows = args.ref_rows
    for _ in range(args.warmup):
        layer.step(np.sort(rng.choice(args.M, size=rows, replace=False)))
    t = 0.0
    for _ in range(args.steps):
        sample = np.sort(rng.choice(args.M, size=rows, replace=False))
        t0 = time.perf_counter()
        layer.step(sample)
        t += time.perf_counter() - t0
    fl = sum(step_flops(rows).values())
    value = fl * args.steps / t / 1e12
    cores = _blas_threads()
    out = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(t / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": workload_desc(args.M), "M": args.M,
                      "sample_rows_per_step": rows, "parallelism": "cpu oracle, rank 0 only"},
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                            "sample": f"{rows} random rows of the M={args.M} step per step; weight packing "
                                      f"({layer.pack_s:.1f} s) done once before timing"},
           "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=600)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--M", type=int, default=16384, help="tokens per GPU per step")
    ap.add_argument("--cmp-steps", type=int, default=10, help="steps of each fused/unfused comparison loop")
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="rows of the oracle sample in cpu_baseline (0: as many as about 10 s of CPU work takes)")
    ap.add_argument("--ref-rows", type=int, default=64, help="rows per step of the --impl reference arm")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the FFN-up kernel from an ncu capture of this kernel")
    ap.add_argument("--sweep", action="store_true",
                    help="fused vs unfused over M in {1024, 4096, 8192, 16384} x {QKV hd128, hd256, FFN-up}")
    ap.add_argument("--sweep-runs", type=int, default=50)
    ap.add_argument("--configs", action="store_true",
                    help="time the five named problems fused vs unfused (cold L2), with the oracle's time")
    ap.add_argument("--no-unfused", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--quantize-only", action="store_true",
                    help="time the activation quantiser alone on the step's x (median of --steps calls)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.configs:
        run_configs(args)
    elif args.quantize_only:
        run_quantize_only(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
