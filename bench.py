"""Benchmark of the INT8 attention forward hot path on B200.

One step = the whole path on one batch of synthetic fp16 input already in HBM:
per-token quantisation of Q and K, per-head quantisation of V (codes in V's
own layout, on a side stream beside Q's and K's, as intfa_forward does), and
the fused INT8 attention kernel (V_hat tiles read N-major).  The metric is INT8 attention TOPS:
4 B H L^2 d ops (halved when causal) per step / step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...    # the CPU oracle, timed on host cores
    python bench.py --method index ...      # the IndexSoftmax variant (IntAttention
                                            # sections 3.1-3.2): per-tensor Q/K/V
                                            # quantisation + the two-pass LUT kernel

N > 1 runs under torchrun, one rank per GPU, each rank the full workload on
its own GPU (independent replicas: the path has no exchange step); the time
is the max over ranks and the value the ops of all ranks over that time.
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

METRIC = "INT8 attention fwd TOPS and % of B200 dense INT8 tensor peak"
UNIT = "TOPS"
DEFAULT_WORKLOAD = "attn_B4_H32_L4096_d128_causal"
# Nominal dense ratio INT8 : BF16 on B200 (4.5 POPS : 2.25 PFLOP/s).
I8_PER_BF16 = 2.0
FALLBACK_BF16_TFLOPS = 1590.0


def kernel_sources_sha(method: str = "online") -> str:
    """Hash of the dominant kernel's sources (the attention kernel of `method`;
    "online-fused-q" is the same kernel with Q quantised inside it)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int8_quantized_attention_token_b200", "csrc")
    files = {"online": ("attention.cu", "ptx.cuh", "quant_math.cuh"),
             "online-fused-q": ("attention.cu", "ptx.cuh", "quant_math.cuh"),
             "index": ("index_attention.cu", "ptx.cuh"),
             "decode": ("decode.cu", "ptx.cuh", "quant_math.cuh")}[method]
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            m = json.load(f)
        return {"bf16_burst": float(m["bf16_tflops"]), "bf16_sustained": float(m["bf16_tflops_sustained"]),
                "hbm_gbs": float(m["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"bf16_burst": FALLBACK_BF16_TFLOPS, "bf16_sustained": 1400.0, "hbm_gbs": 6650.0,
                "source": "fallback"}


def traffic_for(workload: str, method: str = "online"):
    """DRAM bytes per attention launch from the committed ncu summary, if it was
    taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)
        e = t.get(workload if method == "online" else f"{workload}:{method}")
        if e and e.get("kernel_sha") == kernel_sources_sha(method):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms; only the
    samples that arrive inside the timed window are kept."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def stop(self, t_begin=None, t_end=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.lines:
            if t_begin is not None and not (t_begin <= ts <= t_end + 0.1):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(x: float, device=None) -> float:
    """The max of x over all ranks of the default process group (x itself
    when there is none): every timing is reported as the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------- GPU arm ---

def run_gpu(args):
    import torch
    import torch.distributed as dist

    from int8_quantized_attention_token_b200 import intfa
    from int8_quantized_attention_token_b200.workloads import by_name, make_workload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = by_name(args.workload)
    B, H, L, d = w.B, w.H, w.L, w.d
    Qh, Kh, Vh = make_workload(w)
    Q, K, V = Qh.to(dev), Kh.to(dev), Vh.to(dev)
    BH = B * H
    ld = intfa.intfa_vt_ld(L)
    Qq = torch.empty(B, H, L, d, dtype=torch.int8, device=dev)
    Kq = torch.empty_like(Qq)
    Vt = torch.empty(BH, d, ld, dtype=torch.int8, device=dev)   # V_hat^T for the variant kernels
    Vr = torch.empty(B, H, L, d, dtype=torch.int8, device=dev)   # V_hat, untransposed
    sQ = torch.empty(B, H, L, dtype=torch.float32, device=dev)
    sK = torch.empty_like(sQ)
    sV = torch.empty(BH, dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, intfa.lib().intfa_quantize_per_tensor_workspace_size(BH)), dtype=torch.uint8, device=dev)
    O = torch.empty(B, H, L, d, dtype=torch.float16, device=dev)
    stream = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)   # V's quantiser, as in intfa_forward
    fork, join = torch.cuda.Event(), torch.cuda.Event()
    V3 = V.reshape(BH, L, d)

    fused_q = args.q_path == "fused"
    index = args.method == "index"
    if index:   # per-tensor Q and K codes and one scale per head
        sQh = torch.empty(BH, dtype=torch.float32, device=dev)
        sKh = torch.empty(BH, dtype=torch.float32, device=dev)
        Q3, K3 = Q.reshape(BH, L, d), K.reshape(BH, L, d)
        Qq3, Kq3 = Qq.reshape(BH, L, d), Kq.reshape(BH, L, d)

    def step_index(ev=None):
        # per-tensor quantisation of Q, K and V (transposed), then the
        # IndexSoftmax kernel (IntAttention sections 3.1-3.2)
        intfa.intfa_quantize_per_tensor(Q3, False, Qq3, sQh, ws, stream=stream)
        intfa.intfa_quantize_per_tensor(K3, False, Kq3, sKh, ws, stream=stream)
        intfa.intfa_quantize_per_tensor(V3, True, Vt, sV, ws, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        intfa.intfa_index_attention_fwd(Qq, Kq, Vt.reshape(B, H, d, ld), sQh.reshape(B, H), sKh.reshape(B, H),
                                        sV.reshape(B, H), w.causal, args.index_c, args.index_b, O, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    blk = args.scale_block
    if blk > 1:   # one Q / K scale per block of blk tokens (group-wise quantisation)
        if L % blk:
            raise SystemExit("--scale-block must divide L")
        sQb = torch.empty(BH * L // blk, dtype=torch.float32, device=dev)
        sKb = torch.empty_like(sQb)
        Qg, Kg = Q.reshape(BH * L // blk, blk, d), K.reshape(BH * L // blk, blk, d)
        Qqg, Kqg = Qq.reshape(BH * L // blk, blk, d), Kq.reshape(BH * L // blk, blk, d)
        wsb = torch.empty(max(1, intfa.lib().intfa_quantize_per_tensor_workspace_size(BH * L // blk)),
                          dtype=torch.uint8, device=dev)

    def step_blocks(ev=None):
        intfa.intfa_quantize_per_tensor(Qg, False, Qqg, sQb, wsb, stream=stream)
        intfa.intfa_quantize_per_tensor(Kg, False, Kqg, sKb, wsb, stream=stream)
        intfa.intfa_quantize_per_tensor(V3, True, Vt, sV, ws, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        intfa.intfa_attention_fwd_blockscale(Qq, Kq, Vt.reshape(B, H, d, ld), sQb.reshape(B, H, -1),
                                             sKb.reshape(B, H, -1), sV.reshape(B, H), w.causal, blk, O,
                                             stream=stream)
        if ev is not None:
            ev[1].record(stream)

    def step(ev=None):
        if index:
            return step_index(ev)
        if blk > 1:
            return step_blocks(ev)
        # a1 (K; and Q unless fused), a2 (V), then a3-a9 in the attention kernel
        plain = not fused_q and args.p_levels == 127 and args.lsum != "codes"
        if plain:   # the path of intfa_forward: V_hat untransposed, its quantiser
            # on a side stream beside Q's and K's, joined before the attention
            fork.record(stream)
            side.wait_event(fork)
            intfa.intfa_quantize_per_tensor(V3, False, Vr.reshape(BH, L, d), sV, ws, stream=side)
            intfa.intfa_quantize_per_token(Q, Qq, sQ, stream=stream)
            intfa.intfa_quantize_per_token(K, Kq, sK, stream=stream)
            join.record(side)
            stream.wait_event(join)
        else:
            if not fused_q:
                intfa.intfa_quantize_per_token(Q, Qq, sQ, stream=stream)
            intfa.intfa_quantize_per_token(K, Kq, sK, stream=stream)
            intfa.intfa_quantize_per_tensor(V3, True, Vt, sV, ws, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        if plain:
            intfa.intfa_attention_fwd_vrows(Qq, Kq, Vr, sQ, sK, sV.reshape(B, H), w.causal, O, stream=stream)
        elif fused_q:   # Q quantised per token inside the attention kernel
            intfa.intfa_attention_fwd_q16(Q, Kq, Vt.reshape(B, H, d, ld), sK, sV.reshape(B, H), w.causal, O,
                                          s_Q=sQ, stream=stream)
        elif args.p_levels != 127:   # UINT8 P codes RNE(255 p)
            intfa.intfa_attention_fwd_pcodes(Qq, Kq, Vt.reshape(B, H, d, ld), sQ, sK, sV.reshape(B, H), w.causal,
                                             p_levels=args.p_levels, lsum_codes=args.lsum == "codes", O=O,
                                             stream=stream)
        elif args.lsum == "codes":   # row sum from the P codes
            intfa.intfa_attention_fwd_codesum(Qq, Kq, Vt.reshape(B, H, d, ld), sQ, sK, sV.reshape(B, H), w.causal,
                                              O, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    # one kernel each: quantise Q (unless fused), K and V (both phases of the
    # per-head quantiser in one kernel), and the attention kernel
    kernels_per_step = 3 if (fused_q and not index and blk == 1) else 4

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if intfa.intfa_device_status(clear=True) != 0:
        raise RuntimeError("a kernel timed out during warm-up")

    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    h0 = time.perf_counter()
    t0.record(stream)
    for i in range(args.steps):
        step(attn_ev[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    h1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    time.sleep(0.1)
    clk = clocks.stop(h0, h1)
    elapsed_ms = t0.elapsed_time(t1)
    attn_ms = [a.elapsed_time(b) for a, b in attn_ev]
    if intfa.intfa_device_status(clear=True) != 0:
        raise RuntimeError("a kernel timed out during the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, dev)

    ms_per_step = elapsed_ms / args.steps
    value = w.ops * world * args.steps / (elapsed_ms * 1e-3) / 1e12
    attn_mean = sum(attn_ms) / len(attn_ms)

    # The same K-step region timed again, back to back, until about a second
    # of device time has passed (at most 50 regions): evidence that the
    # headline region above is typical, with clocks sampled over all of them.
    # Every rank runs the same number of regions (from the max-over-ranks time).
    repeats = None
    if not args.no_repeats:
        nreg = int(max(1, min(50, 1000.0 // max(elapsed_ms, 1e-3))))
        reg_ms = []
        rclocks = ClockSampler(local)
        rclocks.start()
        time.sleep(0.3)
        r_h0 = time.perf_counter()
        for _ in range(nreg):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            r0.record(stream)
            for _ in range(args.steps):
                step()
            r1.record(stream)
            torch.cuda.synchronize(dev)
            reg_ms.append(max_over_ranks(r0.elapsed_time(r1), dev) / args.steps)
        r_h1 = time.perf_counter()
        time.sleep(0.1)
        rclk = rclocks.stop(r_h0, r_h1)
        if intfa.intfa_device_status(clear=True) != 0:
            raise RuntimeError("a kernel timed out during the repeated regions")
        repeats = {"regions": nreg, "steps_each": args.steps,
                   "ms_per_step_median": round(statistics.median(reg_ms), 5),
                   "ms_per_step_min": round(min(reg_ms), 5), "ms_per_step_max": round(max(reg_ms), 5),
                   "clocks": rclk}
    achieved = w.ops / (attn_mean * 1e-3) / 1e12
    pk = peaks()
    peak = pk["bf16_burst"] * I8_PER_BF16

    # End to end through the host-buffer entry point: pinned fp16 in, fp16 out.
    e2e = None
    if not args.no_e2e and (index or blk > 1):
        # the same step with the fp16 inputs copied from pinned host memory
        # and O copied back, inside the timed region
        Qp, Kp, Vp = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory()
        Op = torch.empty(B, H, L, d, dtype=torch.float16).pin_memory()

        def e2e_step():
            Q.copy_(Qp, non_blocking=True)
            K.copy_(Kp, non_blocking=True)
            V.copy_(Vp, non_blocking=True)
            step()
            Op.copy_(O, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        e_steps = max(3, min(args.steps, 10))
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        nbytes = B * H * L * d * 2
        e2e = {"value": w.ops * world * e_steps / (e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "steps": e_steps, "ms_per_step": e_ms / e_steps,
               "api": ("intfa_quantize_per_tensor x3 + intfa_index_attention_fwd" if index else
                       "intfa_quantize_per_tensor x3 + intfa_attention_fwd_blockscale") + " with pinned host copies"}
    elif not args.no_e2e:
        Qp, Kp, Vp = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory()
        Op = torch.empty(B, H, L, d, dtype=torch.float16).pin_memory()
        wsh = torch.empty(intfa.intfa_forward_host_workspace_size(B, H, L, d), dtype=torch.uint8, device=dev)
        for _ in range(2):
            intfa.intfa_forward_host(Qp, Kp, Vp, w.causal, Op, wsh, stream=stream)
        torch.cuda.synchronize(dev)
        e_steps = max(3, min(args.steps, 10))
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            intfa.intfa_forward_host(Qp, Kp, Vp, w.causal, Op, wsh, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = e0.elapsed_time(e1)
        e_ms = max_over_ranks(e_ms, dev)
        nbytes = B * H * L * d * 2
        e2e = {"value": w.ops * world * e_steps / (e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "steps": e_steps, "ms_per_step": e_ms / e_steps,
               "api": "intfa_forward_host (pinned host fp16 Q/K/V in, O out)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, budget_s=args.cpu_seconds, method=args.method,
                           c=args.index_c, b=args.index_b, blk=blk, lcodes=args.lsum == "codes",
                           p_levels=args.p_levels)

    configs = None
    if rank == 0 and not args.no_configs and args.method == "online" and not fused_q and blk == 1 \
            and args.lsum == "p" and args.p_levels == 127:
        configs = measure_configs(intfa, dev, stream, peak, local)

    sha_method = "online-fused-q" if fused_q else args.method
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic (seeded N(0,1) fp16 Q/K/V)",
            "config": {**w.as_dict(), "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2 (fp16 Q/K/V 3x128 MiB read per step)",
                       "method": args.method,
                       **({"scale_block": blk} if blk > 1 else {}),
                       **({"lsum": "codes"} if args.lsum == "codes" else {}),
                       **({"p_levels": args.p_levels} if args.p_levels != 127 else {}),
                       **({"index_c": args.index_c, "index_b": args.index_b} if index else {})},
            "pct_of_int8_peak": round(100.0 * value / world / peak, 2),
            "roofline": {"bound": "tensor",
                         "kernel": ("attn_index_kernel<%d>" % d) if index else
                                   ("attn_fwd_kernel<%d, Q quantised in-kernel>" % d if fused_q else "attn_fwd_kernel<%d>" % d),
                         "achieved": round(achieved, 2),
                         "peak": round(peak, 1), "unit": UNIT, "frac": round(achieved / peak, 4),
                         "traffic": traffic_for(w.name, sha_method),
                         "peak_note": f"{pk['source']} bf16 burst {pk['bf16_burst']} TFLOP/s x {I8_PER_BF16} "
                                      "(nominal dense INT8:BF16 ratio)",
                         "frac_of_sustained": round(achieved / (pk["bf16_sustained"] * I8_PER_BF16), 4),
                         "attn_ms": round(attn_mean, 5), "ops_per_launch": w.ops,
                         **({"ops_note": "the method's two contractions counted once; the kernel "
                                         "computes Q K^T twice (row-max pass and table pass)"} if index else {})},
            "kernels_ms_per_step": {"attention": round(attn_mean, 5),
                                    "quantisation": round(ms_per_step - attn_mean, 5),
                                    "q_path": args.q_path},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": kernels_per_step * args.steps,
            "clocks": clk, "kernel_sha": kernel_sources_sha(sha_method),
            "repeats": repeats,
            "configs": configs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_configs(intfa, dev, stream, peak, gpu_index, launches=25):
    """intfa_attention_fwd_vrows alone on each of the five synthetic workloads, in
    this process: inputs quantised once, then `launches` launches each timed
    with its own CUDA events on the launching stream, L2 flushed (a 256 MiB
    write) between launches outside the timed pairs; clocks sampled while the
    workload runs.  Returns {name: {attn_ms, TOPS, frac, clocks}}."""
    import torch

    from int8_quantized_attention_token_b200.workloads import WORKLOADS, make_workload
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = {}
    for w in WORKLOADS:
        Qh, Kh, Vh = make_workload(w)
        B, H, L, d = Qh.shape
        Q, K, V = Qh.to(dev), Kh.to(dev), Vh.to(dev)
        Qq, sQ = intfa.intfa_quantize_per_token(Q, stream=stream)
        Kq, sK = intfa.intfa_quantize_per_token(K, stream=stream)
        Vr, sV = intfa.intfa_quantize_per_tensor(V.reshape(B * H, L, d), False, stream=stream)
        Vr, sV = Vr.reshape(B, H, L, d), sV.reshape(B, H)
        O = torch.empty_like(Q)
        for _ in range(3):
            intfa.intfa_attention_fwd_vrows(Qq, Kq, Vr, sQ, sK, sV, w.causal, O, stream=stream)
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
        clocks = ClockSampler(gpu_index)
        clocks.start()
        time.sleep(0.2)
        h0 = time.perf_counter()
        for a, b in ev:
            flush.fill_(1)
            a.record(stream)
            intfa.intfa_attention_fwd_vrows(Qq, Kq, Vr, sQ, sK, sV, w.causal, O, stream=stream)
            b.record(stream)
        torch.cuda.synchronize(dev)
        h1 = time.perf_counter()
        clk = clocks.stop(h0, h1)
        if intfa.intfa_device_status(clear=True) != 0:
            raise RuntimeError(f"a kernel timed out while timing {w.name}")
        ms = sum(a.elapsed_time(b) for a, b in ev) / launches
        tops = w.ops / (ms * 1e-3) / 1e12
        out[w.name] = {"attn_ms": round(ms, 5), "TOPS": round(tops, 2), "frac": round(tops / peak, 4),
                       "launches": launches, "clocks": clk}
        del Q, K, V, Qq, Kq, Vr, O
    del flush
    return out


# ------------------------------------------------------------- decode ---

def run_decode(args):
    """One query per head against a resident INT8 key / value cache
    (intfa_decode_fwd: split-KV partial kernel + merge).  HBM-bound: the
    roofline is the cache bytes read per call over the call's time."""
    import numpy as np
    import torch

    from int8_quantized_attention_token_b200 import intfa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    B, H, L, d = (int(x) for x in args.decode_shape.split(","))
    BH = B * H
    # auto: about 2048 CTAs (seven waves of two CTAs per SM), measured best at
    # B8 H32 L32768 d128 (8 ranges: 92% of HBM; 3: 86%, 16: 91%, 48: 83%)
    splits = args.splits if args.splits > 0 else max(1, min(-(-L // 128), round(2048 / BH)))
    g = torch.Generator().manual_seed(0)
    q = torch.randn(B, H, d, generator=g).half()
    K = torch.randn(B, H, L, d, generator=g).half()
    V = torch.randn(B, H, L, d, generator=g).half()
    Kq, sK = intfa.intfa_quantize_per_token(K.to(dev))
    Vq, sV = intfa.intfa_quantize_per_tensor(V.to(dev).reshape(BH, L, d), transpose=False)
    Vq, sV = Vq.reshape(B, H, L, d), sV.reshape(B, H)
    qd = q.to(dev)
    O = torch.empty(B, H, d, dtype=torch.float16, device=dev)
    ws = torch.empty(int(intfa.lib().intfa_decode_workspace_size(B, H, d, splits)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # a buffer larger than L2, written between timed calls: the cache (2 GB at
    # the default shape) exceeds L2 anyway, the flush keeps small shapes honest
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def call():
        intfa.intfa_decode_fwd(qd, Kq, sK, Vq, sV, splits, O, ws, stream=stream)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    if intfa.intfa_device_status(clear=True) != 0:
        raise RuntimeError("a kernel timed out during warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    h0 = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record(stream)
        call()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    h1 = time.perf_counter()
    time.sleep(0.1)
    clk = clocks.stop(h0, h1)
    if intfa.intfa_device_status(clear=True) != 0:
        raise RuntimeError("a kernel timed out during the timed region")
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    ms = max_over_ranks(ms, dev)
    ops = 4.0 * d * BH * L
    cache_bytes = BH * L * (2 * d + 4)
    io_bytes = BH * d * 2 * 2 + BH * splits * (d + 2) * 4 * 2
    gbs = (cache_bytes + io_bytes) / (ms * 1e-3) / 1e9
    pk = peaks()

    e2e = None
    if not args.no_e2e:   # the query from pinned host memory, O back to the host
        qp = q.pin_memory()
        Op = torch.empty(B, H, d, dtype=torch.float16).pin_memory()
        e_steps = max(3, min(args.steps, 20))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            qd.copy_(qp, non_blocking=True)
            call()
            Op.copy_(O, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev) / e_steps
        e2e = {"value": ops * world / (e_ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": BH * d * 2,
               "d2h_bytes_per_step": BH * d * 2, "steps": e_steps, "ms_per_step": e_ms,
               "api": "intfa_decode_fwd with the query copied from pinned host memory and O copied back"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        cores = len(os.sched_getaffinity(0))
        oracle.set_threads(cores)
        nblk = -(-L // 128)
        split_len = -(-nblk // splits) * 128
        t, n = 0.0, 0
        while t < args.cpu_seconds and n < BH:
            b, h = n // H, n % H
            t0 = time.perf_counter()
            qq, sq = oracle.quantize_per_token(q[b, h].float().numpy()[None, :])
            kq, sk = oracle.quantize_per_token(K[b, h].float().numpy())
            vq, sv = oracle.quantize_per_tensor(V[b, h].float().numpy(), 1)
            oracle.decode(qq[0], float(sq[0]), kq, sk, vq, float(sv[0]), 128, split_len)
            t += time.perf_counter() - t0
            n += 1
        cpu = {"value": round(4.0 * d * L * n / t / 1e12, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{n} of {BH} heads (quantise the query and the head's cache, decode), {t:.1f} s, "
                         "single-threaded (the decode oracle has no thread loop)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(ops * world / (ms * 1e-3) / 1e12, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic (seeded N(0,1) fp16 q/K/V)",
            "config": {"workload": f"decode_B{B}_H{H}_L{L}_d{d}", "B": B, "H": H, "L": L, "d": d, "splits": splits,
                       "method": "decode", "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "256 MiB buffer written between timed calls; cache of %.2f GB" % (cache_bytes / 1e9)},
            "roofline": {"bound": "hbm", "kernel": f"decode_partial_kernel<{d}> + decode_combine_kernel<{d}>",
                         "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / pk["hbm_gbs"], 4), "traffic": None,
                         "peak_note": f"{pk['source']} HBM copy bandwidth",
                         "bytes_per_call": cache_bytes + io_bytes},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps, "clocks": clk,
            "kernel_sha": kernel_sources_sha("decode"),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------- CPU arm ---

def oracle_sample(w, heads, threads=None, method="online", c=6.6, b=5, blk=1, lcodes=False, p_levels=127):
    """Run the oracle's whole path (quantise, block-wise online attention; or
    for method "index" per-tensor quantisation and IndexSoftmax attention) on
    `heads` full (b, h) heads of the workload; returns (seconds, ops, cores)."""
    import numpy as np

    import oracle
    from int8_quantized_attention_token_b200.workloads import make_workload

    cores = len(os.sched_getaffinity(0)) if threads is None else threads
    oracle.set_threads(cores)
    Q, K, V = make_workload(w)
    t = 0.0
    for (bi, h) in heads:
        q, k, v = (X[bi, h].float().numpy() for X in (Q, K, V))
        t0 = time.perf_counter()
        if method == "index":
            Qq, sQ = oracle.quantize_per_tensor(q, 1)
            Kq, sK = oracle.quantize_per_tensor(k, 1)
            Vq, sV = oracle.quantize_per_tensor(v, 1)
            oracle.index_attention_rows(Qq, Kq, Vq, float(sQ[0]), float(sK[0]), float(sV[0]), w.causal, c, b)
        elif blk > 1:   # one scale per block of blk tokens
            n = w.L // blk
            Qq, sQ = oracle.quantize_per_tensor(q.reshape(n, blk * w.d), n)
            Kq, sK = oracle.quantize_per_tensor(k.reshape(n, blk * w.d), n)
            Vq, sV = oracle.quantize_per_tensor(v, 1)
            oracle.attention_online_rows(Qq.reshape(w.L, w.d), Kq.reshape(w.L, w.d), Vq, np.repeat(sQ, blk),
                                         np.repeat(sK, blk), float(sV[0]), w.causal, 128)
        else:
            Qq, sQ = oracle.quantize_per_token(q)
            Kq, sK = oracle.quantize_per_token(k)
            Vq, sV = oracle.quantize_per_tensor(v, 1)
            oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, float(sV[0]), w.causal, 128, lsum_codes=lcodes,
                                         p_levels=p_levels)
        t += time.perf_counter() - t0
    ops = w.ops / (w.B * w.H) * len(heads)
    return t, ops, oracle.get_threads()


def cpu_baseline(w, budget_s=15.0, method="online", c=6.6, b=5, blk=1, lcodes=False, p_levels=127):
    t1, ops1, cores = oracle_sample(w, [(0, 0)], method=method, c=c, b=b, blk=blk, lcodes=lcodes,
                                    p_levels=p_levels)
    n = max(1, min(w.B * w.H - 1, int(budget_s / max(t1, 1e-3)) - 1))
    heads = [((i + 1) // w.H % w.B, (i + 1) % w.H) for i in range(n)]
    t, ops, cores = oracle_sample(w, heads, method=method, c=c, b=b, blk=blk, lcodes=lcodes, p_levels=p_levels)
    t += t1
    ops += ops1
    what = ("per-tensor quantise + IndexSoftmax attention" if method == "index" else
            f"per-{blk}-token-block quantise + online attention" if blk > 1 else "quantise + online attention")
    return {"value": round(ops / t / 1e12, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n + 1} of {w.B * w.H} heads at full L={w.L} ({what}), "
                      f"{t:.1f} s on {cores} threads"}


def oracle_rows_step(w, head, rows, data):
    """One reference step: the oracle's whole path for one head (quantise Q, K,
    V; block-wise online attention) on a contiguous run of query rows.  Returns
    (seconds, ops): ops = 4 d per visible (query, key) pair."""
    import numpy as np

    import oracle

    Q, K, V = data
    b, h = head
    q, k, v = (X[b, h].float().numpy() for X in (Q, K, V))
    t0 = time.perf_counter()
    Qq, sQ = oracle.quantize_per_token(q)
    Kq, sK = oracle.quantize_per_token(k)
    Vq, sV = oracle.quantize_per_tensor(v, 1)
    oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, float(sV[0]), w.causal, 128,
                                 int(rows[0]), int(rows[-1]) + 1)
    t = time.perf_counter() - t0
    visible = (np.asarray(rows) + 1) if w.causal else np.full(len(rows), w.L)
    return t, 4.0 * w.d * float(visible.sum())


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    import oracle
    from int8_quantized_attention_token_b200.workloads import by_name, make_workload
    w = by_name(args.workload)
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    data = make_workload(w)
    heads = [(i // w.H % w.B, i % w.H) for i in range(w.B * w.H)]
    rng = np.random.default_rng(0)
    # size each step so that the whole run takes about args.ref_seconds
    cal = min(w.L, 256)
    t_cal, _ = oracle_rows_step(w, heads[0], np.arange(w.L - cal, w.L), data)
    per_row = t_cal / cal
    n_rows = int(max(1, min(w.L, args.ref_seconds / max(args.steps, 1) / max(per_row, 1e-6))))
    tt, ops_total = 0.0, 0.0
    for i in range(args.steps):
        r0 = int(rng.integers(0, w.L - n_rows + 1))
        rows = np.arange(r0, r0 + n_rows)
        t, ops = oracle_rows_step(w, heads[i % len(heads)], rows, data)
        tt += t
        ops_total += ops
    value = ops_total / tt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tt / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) fp16 Q/K/V)", "config": w.as_dict(),
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": oracle.get_threads(),
                             "kind": "oracle",
                             "sample": f"per step: one head of the workload quantised, {n_rows} consecutive query "
                                       f"rows (random start) of it through the block-wise online attention; {args.steps} steps, "
                                       f"{tt:.1f} s"},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="libintfa", choices=["libintfa", "reference"])
    ap.add_argument("--q-path", default="separate", choices=["fused", "separate"],
                    help="quantise Q in its own pass (default, faster) or inside the attention kernel")
    ap.add_argument("--method", default="online", choices=["online", "index", "decode"],
                    help="online: the INT8 FlashAttention path (default); index: the IndexSoftmax variant; "
                         "decode: one query per head against an INT8 cache")
    ap.add_argument("--decode-shape", default="8,32,32768,128", help="decode: B,H,L,d")
    ap.add_argument("--splits", type=int, default=0, help="decode: key ranges per head (0: auto)")
    ap.add_argument("--index-c", type=float, default=6.6, help="IndexSoftmax clip threshold c")
    ap.add_argument("--index-b", type=int, default=5, help="IndexSoftmax table bits b")
    ap.add_argument("--lsum", default="p", choices=["p", "codes"],
                    help="online method: row sum from the unquantised p (default) or from the P codes")
    ap.add_argument("--p-levels", type=int, default=127, choices=[127, 255],
                    help="online method: P codes RNE(127 p) as INT8 (default) or RNE(255 p) as UINT8")
    ap.add_argument("--scale-block", type=int, default=1,
                    help="online method: one Q / K scale per block of this many tokens (1 = per token)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-repeats", action="store_true",
                    help="skip re-timing the K-step region for about a second after the headline region")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload attention timings of the five synthetic configs")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl != "reference":
        raise SystemExit("--warmup must be >= 3")
    if (args.scale_block != 1 or args.lsum != "p" or args.p_levels != 127) and \
            (args.method != "online" or args.q_path != "separate"):
        raise SystemExit("--scale-block / --lsum / --p-levels apply to the online method with the separate Q pass")
    if args.scale_block != 1 and (args.lsum != "p" or args.p_levels != 127):
        raise SystemExit("--scale-block and --lsum codes / --p-levels 255 are separate variants")
    if args.impl == "reference":
        run_reference(args)
    elif args.method == "decode":
        run_decode(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
