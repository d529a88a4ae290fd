#!/usr/bin/env python
"""Benchmark: SageBwd INT8 attention forward + backward on B200.

One step = the whole hot path on one batch: the quantization prologue (QK-norm, K-smoothing,
INT8 codes), the forward kernel and the three backward stages, on synthetic bf16 inputs that
are resident in HBM.  Metric: effective tensor-core TOPS over the step, counting the seven
attention GEMMs (FlashAttention convention, causal half not credited).  Each step is timed with
CUDA events on the launching stream; when an input tensor is smaller than 4x the 126 MB L2,
L2 is flushed (a 512 MiB buffer written) before every step, outside the timed events.

Roofline denominators are measured in the same run on the same GPU: the tensor cores' INT8
(kind::i8) and 16-bit (kind::f16) throughput from the library's own back-to-back tcgen05 MMA
loop (sage_mma_peak), weighted by each kernel's mix of INT8 and 16-bit GEMMs.

Multi-GPU (torchrun): every (batch, head) is independent and the operator has no weights, so
each rank runs its own full-size batch with no collective on the data path (weak scaling); the
harness takes the maximum elapsed time over ranks.  The end-to-end leg streams one global batch
from host memory, split across the ranks in contiguous batch ranges.

``--impl reference`` times the CPU oracle (the plain restatement of the method the tests
check the kernels against) on a bounded sample of the same workload.
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

METRIC = "attention fwd+bwd effective TOPS at 1 B200 and % of INT8/FP16 TC roofline"
METRIC_FP4 = "NVFP4 Q-Attn fwd+bwd effective TOPS at 1 B200 and % of FP4/16-bit TC roofline"
L2_BYTES = 126 * 2 ** 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="sage", choices=["sage", "reference"])
    ap.add_argument("--workload", default="sweep8192")
    ap.add_argument("--B", type=int, default=0, help="override the batch (small profiling runs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--chunks", type=int, default=16,
                    help="batch slices of the end-to-end host-buffer pipeline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-peaks", action="store_true",
                    help="skip the tensor-core peak loop (profiling runs; no roofline fraction)")
    ap.add_argument("--variant", default="int8", choices=["int8", "nvfp4"],
                    help="int8: the SageBwd step (default); nvfp4: the NVFP4 Q-Attn fwd+bwd step")
    ap.add_argument("--cp", type=int, default=0,
                    help="context parallelism: the workload's sequence in this many chunks, the "
                         "ranks as threads on one GPU (cp.LocalRing), beside the single-sequence "
                         "step")
    return ap.parse_args()


def peaks():
    """cuBLAS bf16 and HBM copy figures from MEASURED_PEAKS.json (driver-measured): context for
    the tensor cores, and the HBM roofline of the prologue."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        m = json.load(open(path))
        return {"bf16_burst": m["bf16_tflops"], "bf16_sustained": m["bf16_tflops_sustained"],
                "hbm_gbs": m["hbm_gbs"], "basis": "measured"}
    return {"bf16_burst": 1590.0, "bf16_sustained": 1400.0, "hbm_gbs": 6650.0,
            "basis": "fallback"}


def traffic_per_launch(kernel: str, src: str):
    """DRAM bytes per full launch from profiles/traffic.txt, if the kernel source still matches
    the one the counters were taken on (else None)."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()[:16]
    for line in open(path):
        f = line.split()
        if len(f) >= 3 and f[0] == kernel and f[1] == sha:
            return float(f[2]) * 1e9
    return None


def mixed_peak(p_a: float, p_b: float, n_a: int, n_b: int) -> float:
    """Peak of a mix of equal-size GEMMs at two rates: total ops over total minimum time."""
    n = n_a + n_b
    return 1.0 / (n_a / n / p_a + (n_b / n / p_b if n_b else 0.0))


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", uuid], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit()
                else None, "reasons": reasons, "samples": len(rows)}


def uuid_of(dev) -> str:
    import torch

    return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)


def measure_tc_peaks(dev, dtype16: str, seconds: float = 0.6) -> dict:
    """The tensor cores' own INT8 (kind::i8) and 16-bit (kind::f16) throughput on this GPU, now:
    one CTA per SM issuing back-to-back 128 x 256 MMAs from shared memory (sage_mma_peak), timed
    with CUDA events while nvidia-smi samples the SM clock.  Returns TOPS per kind (median of
    three launches) with the median SM clock seen."""
    import torch

    from fwd_bwd_b200 import ops

    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    kind16 = 2 if dtype16 == "bf16" else 1
    fills = {0: torch.randint(-127, 128, (49152,), generator=g, device=dev).to(torch.int8),
             kind16: torch.randn(24576, generator=g, device=dev).to(
                 torch.bfloat16 if kind16 == 2 else torch.float16)}
    out = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for kind in (0, kind16):
        groups = 2000
        ops.mma_peak(kind, nsm, groups, fills[kind])
        e0.record()
        ops.mma_peak(kind, nsm, groups, fills[kind])
        e1.record()
        torch.cuda.synchronize(dev)
        groups = max(1000, int(groups * (seconds / 3) * 1e3 / e0.elapsed_time(e1)))
        sampler = ClockSampler(uuid_of(dev))
        time.sleep(0.25)
        rates = []
        for _ in range(3):
            e0.record()
            ops.mma_peak(kind, nsm, groups, fills[kind])
            e1.record()
            torch.cuda.synchronize(dev)
            rates.append(ops.mma_peak_ops(kind, nsm, groups)
                         / (e0.elapsed_time(e1) * 1e-3) / 1e12)
        clk = sampler.stop() or {}
        if ops.device_status(dev) != 0:
            raise RuntimeError("the tensor-core peak loop reported a timeout")
        out["i8" if kind == 0 else "f16"] = {"tops": statistics.median(rates),
                                             "sm_mhz": clk.get("sm_mhz"),
                                             "reasons": clk.get("reasons")}
    return out


def cpu_baseline(w, n_heads: int):
    """Time the oracle (as it stands) on the first n_heads heads of the workload."""
    from threadpoolctl import threadpool_info

    import oracle.sage_oracle as O
    from fwd_bwd_b200.inputs import make_inputs

    x = make_inputs(w, heads=range(n_heads))
    args = [x[n + "_f32"] for n in ("q", "k", "v", "do")]
    t0 = time.perf_counter()
    O.sage_attention(*args, causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth,
                     q_block=w.q_block, k_block=w.k_block, dtype=w.dtype, qsmooth=w.qsmooth)
    dt = time.perf_counter() - t0
    ops = w.ops() / (w.B * w.H) * n_heads
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
            "seconds": dt,
            "sample": f"{n_heads} of {w.B * w.H} heads (flattened b*H+h = 0..{n_heads - 1}) of "
                      f"the workload, prologue+fwd+bwd, numpy oracle"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    times = []
    res = None
    for s in range(args.warmup + args.steps):
        res = cpu_baseline(w, 1)
        if s >= args.warmup:
            times.append(res["seconds"])
    sec = statistics.mean(times)
    ops = w.ops() / (w.B * w.H)
    val = ops / sec / 1e12
    cb = dict(res, value=val)
    cb.pop("seconds", None)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8+f64", "data": "synthetic",
            "config": config_of(w), "cpu_baseline": cb,
            "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline_fp4(w, n_heads: int):
    """Time the NVFP4 oracle (as it stands) on the first n_heads heads: prologue + forward +
    backward."""
    from threadpoolctl import threadpool_info

    import oracle.nvfp4_oracle as F
    from fwd_bwd_b200.inputs import make_inputs

    x = make_inputs(w, heads=range(n_heads))
    t0 = time.perf_counter()
    F.qattn_attention(x["q_f32"], x["k_f32"], x["v_f32"], x["do_f32"], causal=w.causal,
                      qknorm=w.qknorm, ksmooth=w.ksmooth, dtype=w.dtype)
    dt = time.perf_counter() - t0
    ops = w.ops() / (w.B * w.H) * n_heads
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
            "sample": f"{n_heads} of {w.B * w.H} heads (flattened b*H+h = 0..{n_heads - 1}) of "
                      f"the workload, NVFP4 prologue+forward+backward, numpy oracle"}


def l2_policy(w) -> tuple:
    """(flush, label): flush L2 before each step unless every input is >= 4x L2."""
    tensor = w.B * w.H * w.N * w.d * 2
    if tensor >= 4 * L2_BYTES:
        return False, f"no flush: every input tensor ({tensor / 2 ** 20:.0f} MiB) exceeds 4x L2"
    return True, (f"L2 flushed before every step (input tensors {tensor / 2 ** 20:.0f} MiB "
                  f"< 4x L2)")


def config_of(w):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "io_dtype": w.dtype, "q_block": w.q_block, "k_block": w.k_block,
            "qknorm": w.qknorm, "ksmooth": w.ksmooth, "qsmooth": w.qsmooth,
            "l2": l2_policy(w)[1]}


def timed_steps(step, nev: int, steps: int, dev, flush_buf=None):
    """Run `steps` steps, each bracketed by its own CUDA events (`step(ev)` records ev[1..]);
    L2 is flushed between steps (outside the events) when `flush_buf` is given.  Returns the
    per-step event lists."""
    import torch

    stream = torch.cuda.current_stream(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(steps)]
    for s in range(steps):
        if flush_buf is not None:
            flush_buf.add_(1)
        evs[s][0].record(stream)
        step(evs[s])
    return evs


def run_cp(args, w):
    """Context parallelism on one GPU: the workload's sequence cut into `args.cp` chunks whose
    ranks run as threads (cp.LocalRing; device-to-device copies stand in for the NVLink
    transfers), timed beside the single-sequence step of the same workload in the same run.
    Each step is bracketed by CUDA events on the launching thread's stream, recorded after every
    rank's stream has drained, so the ranks' host-side launch overhead is inside the time."""
    import statistics

    import torch

    from fwd_bwd_b200 import cp, ops
    from fwd_bwd_b200.inputs import make_inputs_fast

    W = args.cp
    if w.N % (128 * W) != 0 or w.qsmooth:
        raise SystemExit(f"--cp {W}: N must split into chunks of a multiple of 128 tokens, "
                         "without Q-smoothing")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = ops.Config(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                     k_block=w.k_block)
    x = make_inputs_fast(w, device=str(dev))
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    n = w.N // W
    per_rank = [tuple(t[:, :, r * n:(r + 1) * n].contiguous() for t in (q, k, v, do)) + (cfg,)
                for r in range(W)]
    ring = cp.LocalRing(W, dev)

    def ring_step():
        ring.run(lambda comm, *a: cp.forward_backward(*a, comm=comm), per_rank)

    def single_step():
        qb = ops.quant_prologue(q, k, v, cfg)
        o, lse = ops.attn_fwd(qb, q, cfg)
        ops.attn_bwd(q, k, v, qb, o, lse, do, cfg)

    def median_ms(step):
        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            e0, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
            e0.record()
            step()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    single_ms = median_ms(single_step)
    ring_ms = median_ms(ring_step)
    assert ops.device_status() == 0
    tops = w.ops() / (ring_ms * 1e-3) / 1e12
    elems = w.B * w.H * n * w.d
    line = {
        "metric": "attention fwd+bwd effective TOPS through the context-parallel ring "
                  "(ranks emulated on 1 B200)",
        "value": tops, "unit": "TOPS", "n_gpus": 1, "cp_ranks": W, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ring_ms,
        "single_sequence_ms": single_ms, "ring_over_single_sequence": ring_ms / single_ms,
        "higher_is_better": True, "dtype": "int8+bf16", "data": "synthetic",
        # bytes each rank sends per ring step: INT8 K and V codes (forward); K codes, raw
        # 16-bit V and the float32 dK / dV accumulators (backward); block scales excluded
        "ring_bytes_per_rank_step": {"forward": 2 * elems, "backward": 11 * elems},
        "config": dict(config_of(w), transport="cp.LocalRing: the ranks as threads on one GPU, "
                       "device-to-device copies in place of NVLink"),
    }
    print(json.dumps(line), flush=True)


def run_nvfp4(args, w):
    """The NVFP4 Q-Attn step: NVFP4 prologue (with the sequence views) + forward + backward
    (preprocess, main kernel, dQ finalize)."""
    import torch

    from fwd_bwd_b200 import nvfp4, ops
    from fwd_bwd_b200.inputs import make_inputs_fast

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--variant nvfp4 runs on one GPU")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    cfg = ops.Config(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth)
    x = make_inputs_fast(w, device=str(dev))
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    fb = nvfp4.Fp4Bufs.empty(tuple(q.shape), cfg, dev, seq=True)
    ws = torch.empty(nvfp4.workspace_bytes(cfg, q), dtype=torch.uint8, device=dev)
    wsb = torch.empty(nvfp4.bwd_workspace_bytes(cfg, q), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    stream = torch.cuda.current_stream(dev)
    # prologue: (K statistics: 2 when ksmooth) + amax + quantization; forward 1; backward 3
    launches_per_step = 2 * int(w.ksmooth) + 2 + 1 + 3
    flush, _ = l2_policy(w)
    flush_buf = torch.empty(2 ** 27, dtype=torch.float32, device=dev) if flush else None

    def step(ev):
        nvfp4.quant_prologue(q, k, cfg, out=fb, workspace=ws)
        ev[1].record(stream)
        nvfp4.attn_fwd(fb, v, cfg, o=o, lse=lse)
        ev[2].record(stream)
        for stage in range(3):  # preprocess, main kernel, dQ finalize
            nvfp4.attn_bwd(q, k, v, fb, o, lse, do, cfg, dq=dq, dk=dk, dv=dv, workspace=wsb,
                           stage=stage)
            ev[3 + stage].record(stream)

    for _ in range(args.warmup):
        step([torch.cuda.Event(enable_timing=True) for _ in range(6)])
    torch.cuda.synchronize(dev)
    tc = None if args.no_peaks else measure_tc_peaks(dev, w.dtype)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(uuid_of(dev))
    time.sleep(0.3)
    evs = timed_steps(step, 6, args.steps, dev, flush_buf)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if ops.device_status(dev) != 0:
        raise RuntimeError("device status reports a kernel timeout in the timed region")
    mean = lambda a, b: statistics.mean(e[a].elapsed_time(e[b]) for e in evs)  # noqa: E731
    ms = mean(0, 5)
    stages = {"prologue": mean(0, 1), "fwd": mean(1, 2), "bwd_preprocess": mean(2, 3),
              "bwd": mean(3, 4), "dq_finalize": mean(4, 5)}
    value = w.ops() / (ms * 1e-3) / 1e12
    kern = {"fp4::attn_fwd_kernel": (stages["fwd"], w.ops("fwd"), 1, 1),
            "fp4::bwd::attn_bwd_kernel": (stages["bwd"], w.ops("bwd"), 3, 2)}
    kernels = {}
    for name, (kms, kops, n4, n16) in kern.items():
        ach = kops / (kms * 1e-3) / 1e12
        kernels[name] = {"ms": round(kms, 4), "tops": round(ach, 2)}
        if tc is not None:
            # NVFP4 GEMMs at 4x the measured 16-bit rate (the nominal dense ratio 9 : 2.25
            # POPS), 16-bit GEMMs at the measured rate; equal op counts per GEMM
            pk = mixed_peak(4.0 * tc["f16"]["tops"], tc["f16"]["tops"], n4, n16)
            kernels[name].update(peak=round(pk, 1), frac=round(ach / pk, 4))
    top = max(kernels, key=lambda n: kernels[n]["ms"])
    src = {"fp4::attn_fwd_kernel": "fwd_bwd_b200/csrc/nvfp4.cuh",
           "fp4::bwd::attn_bwd_kernel": "fwd_bwd_b200/csrc/nvfp4_bwd.cuh"}[top]
    traffic = (traffic_per_launch(top, src) if w.name == "sweep8192" and w.B == 32 else None)
    roofline = {"bound": "tensor", "kernel": top, "achieved": kernels[top]["tops"],
                "unit": "TFLOP/s", "traffic": traffic}
    if tc is not None:
        p16 = tc["f16"]["tops"]
        roofline.update(peak=kernels[top]["peak"], frac=kernels[top]["frac"],
                        peak_note=f"measured in this run: own tcgen05 kind::f16 loop "
                                  f"{p16:.0f} TOPS; NVFP4 = 4x that (nominal ratio), weighted "
                                  f"by the kernel's GEMM mix (fwd 1 NVFP4 : 1 16-bit, bwd "
                                  f"3 : 2)")
    e2e = None
    if not args.no_e2e:
        hin = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t)
               for t in (q, k, v, do)]
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (dq, dk, dv)]
        qd, kd, vd, dod = (torch.empty_like(t) for t in (q, k, v, do))

        def host_step():
            for h, d_ in zip(hin, (qd, kd, vd, dod)):
                d_.copy_(h, non_blocking=True)
            nvfp4.quant_prologue(qd, kd, cfg, out=fb, workspace=ws)
            nvfp4.attn_fwd(fb, vd, cfg, o=o, lse=lse)
            nvfp4.attn_bwd(qd, kd, vd, fb, o, lse, dod, cfg, dq=dq, dk=dk, dv=dv,
                           workspace=wsb)
            for h, d_ in zip(hout, (dq, dk, dv)):
                h.copy_(d_, non_blocking=True)
            torch.cuda.synchronize(dev)

        host_step()
        w0 = time.perf_counter()
        for _ in range(args.steps):
            host_step()
        e_ms = (time.perf_counter() - w0) * 1e3 / args.steps
        e2e = {"value": w.ops() / (e_ms * 1e-3) / 1e12, "unit": "TOPS",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hin),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in hout),
               "note": "one stream, copies not overlapped with the kernels"}
    line = {"metric": METRIC_FP4, "value": value, "unit": "TOPS", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4+bf16", "data": "synthetic",
            "config": dict(config_of(w), variant="nvfp4 fwd+bwd"),
            "stages_ms": {kk: round(vv, 4) for kk, vv in stages.items()},
            "kernels": kernels, "tensor_peaks": tc, "roofline": roofline, "clocks": clocks,
            "e2e": e2e, "gpu_launches": launches_per_step * args.steps}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_fp4(w, 2)
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    from fwd_bwd_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    if args.B > 0:
        w = w.replace(B=args.B)
    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.variant == "nvfp4":
        run_nvfp4(args, w)
        return
    if args.cp > 0:
        run_cp(args, w)
        return

    import torch
    import torch.distributed as dist

    from fwd_bwd_b200 import ops
    from fwd_bwd_b200.inputs import make_inputs_fast

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    cfg = ops.Config(causal=w.causal, qknorm=w.qknorm, ksmooth=w.ksmooth, q_block=w.q_block,
                     k_block=w.k_block, qsmooth=w.qsmooth)
    x = make_inputs_fast(w.replace(seed=w.seed + rank), device=str(dev))
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    prm = cfg.params(q)
    qb = ops.QuantBufs.empty(tuple(q.shape), cfg, dev)
    ws_pro = torch.empty(max(ops.workspace_bytes(prm, 0), 16), dtype=torch.uint8, device=dev)
    ws_bwd = torch.empty(ops.workspace_bytes(prm, 2), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 1 + 2 * (int(w.ksmooth) + int(w.qsmooth)) + 1 + 3
    flush, _ = l2_policy(w)
    flush_buf = torch.empty(2 ** 27, dtype=torch.float32, device=dev) if flush else None

    # events: [0] step start, [1] prologue done, [2] forward done, [3] preprocess done,
    # [4] backward kernel done, [5] step done
    def step(ev):
        ops.quant_prologue(q, k, v, cfg, out=qb, workspace=ws_pro)
        ev[1].record(stream)
        ops.attn_fwd(qb, q, cfg, o=o, lse=lse)
        ev[2].record(stream)
        ops.attn_bwd(q, k, v, qb, o, lse, do, cfg, dq, dk, dv, workspace=ws_bwd, stage=0)
        ev[3].record(stream)
        ops.attn_bwd(q, k, v, qb, o, lse, do, cfg, dq, dk, dv, workspace=ws_bwd, stage=1)
        ev[4].record(stream)
        ops.attn_bwd(q, k, v, qb, o, lse, do, cfg, dq, dk, dv, workspace=ws_bwd, stage=2)
        ev[5].record(stream)

    for _ in range(args.warmup):
        step([torch.cuda.Event(enable_timing=True) for _ in range(6)])
    torch.cuda.synchronize(dev)
    if ops.device_status(dev) != 0:
        raise RuntimeError("device status reports a kernel timeout during warm-up")
    tc = None if args.no_peaks else measure_tc_peaks(dev, w.dtype)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(uuid_of(dev))
    time.sleep(0.3)
    evs = timed_steps(step, 6, args.steps, dev, flush_buf)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    elapsed = sum(e[0].elapsed_time(e[5]) for e in evs)
    part = {name: statistics.mean(e[a].elapsed_time(e[b]) for e in evs)
            for name, a, b in (("prologue", 0, 1), ("fwd", 1, 2), ("bwd_pre", 2, 3),
                               ("bwd", 3, 4), ("dq_finalize", 4, 5))}
    if world > 1:
        t = torch.tensor([elapsed], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed = float(t.item())
    if ops.device_status(dev) != 0:
        raise RuntimeError("device status reports a kernel timeout in the timed region")
    ms = elapsed / args.steps
    total_ops = w.ops() * world
    value = total_ops / (ms * 1e-3) / 1e12

    # end to end through the C ABI's host-buffer call (sage_fwd_bwd_host): pinned host inputs
    # in, pinned host results out, the copies and their overlap with the kernels inside the
    # timed region.  One global batch of B entries is split across the ranks (contiguous batch
    # ranges, shard.head_range), so the pinned host memory per node stays that of one batch.
    e2e = None
    if not args.no_e2e:
        from fwd_bwd_b200.shard import head_range

        mine = head_range(w.B, world, rank)
        bsl = len(mine)
        hin = [torch.empty((bsl,) + tuple(t.shape[1:]), dtype=t.dtype,
                           pin_memory=True).copy_(t[mine.start:mine.stop]) for t in (q, k, v, do)]
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in hin]
        del q, k, v, do, o, dq, dk, dv, qb, ws_pro, ws_bwd, lse, x, flush_buf
        torch.cuda.empty_cache()
        pipe = ops.HostPipeline(hin[0], cfg, args.chunks, dev)
        ops.fwd_bwd_host(*hin, cfg, *hout, pipeline=pipe)  # warm-up
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        t0 = time.perf_counter()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(torch.cuda.current_stream(dev))
        for _ in range(args.steps):
            ops.fwd_bwd_host(*hin, cfg, *hout, pipeline=pipe)
        e1.record(torch.cuda.current_stream(dev))
        torch.cuda.synchronize(dev)
        wall_ms = (time.perf_counter() - t0) * 1e3
        # every call returns after the results reached host memory, so the events on the
        # default stream bracket the whole sequence; take the larger of event and wall time
        e_ms = max(e0.elapsed_time(e1), wall_ms)
        if world > 1:
            t = torch.tensor([e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        if ops.device_status(dev) != 0:
            raise RuntimeError("device status reports a kernel timeout in the e2e run")
        e2e = {"value": w.ops() / (e_ms / args.steps * 1e-3) / 1e12, "unit": "TOPS",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hin),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in hout),
               "chunks": args.chunks, "api": "sage_fwd_bwd_host",
               "global_batch": w.B, "batch_per_rank": bsl,
               "bytes_note": "per rank; one global batch split across the ranks"}

    pk = peaks()
    bwd_ops, fwd_ops = w.ops("bwd"), w.ops("fwd")
    kernels = {"attn_bwd_kernel": {"ms": part["bwd"], "tops": bwd_ops / (part["bwd"] * 1e-3) / 1e12},
               "attn_fwd_kernel": {"ms": part["fwd"], "tops": fwd_ops / (part["fwd"] * 1e-3) / 1e12}}
    roofline = {"bound": "tensor", "kernel": "attn_bwd_kernel", "unit": "TFLOP/s",
                "achieved": kernels["attn_bwd_kernel"]["tops"],
                "traffic": traffic_per_launch("attn_bwd_kernel", "fwd_bwd_b200/csrc/attn_bwd.cuh")
                if w.name == "sweep8192" and w.B == 32 else None}
    line_extra = {}
    if tc is not None:
        p8, p16 = tc["i8"]["tops"], tc["f16"]["tops"]
        mix = {"attn_bwd_kernel": (4, 1), "attn_fwd_kernel": (2, 0)}
        step_mhz = (clocks or {}).get("sm_mhz")
        for name, (a, b) in mix.items():
            pk_k = mixed_peak(p8, p16, a, b)
            kernels[name].update(peak=pk_k, frac=kernels[name]["tops"] / pk_k)
        p_all = mixed_peak(p8, p16, 6, 1)
        roofline.update(peak=kernels["attn_bwd_kernel"]["peak"],
                        frac=kernels["attn_bwd_kernel"]["frac"],
                        peak_note=f"measured in this run on this GPU: own tcgen05 loops "
                                  f"kind::i8 {p8:.0f} TOPS at {tc['i8']['sm_mhz']} MHz, "
                                  f"kind::f16 {p16:.0f} TOPS at {tc['f16']['sm_mhz']} MHz; "
                                  f"weighted 4:1 for the backward kernel's GEMMs")
        # the same peaks scaled to the SM clock the step ran at (the loops draw more power and
        # run at a lower clock than the attention kernels)
        if step_mhz and tc["i8"]["sm_mhz"] and tc["f16"]["sm_mhz"]:
            p8c = p8 * step_mhz / tc["i8"]["sm_mhz"]
            p16c = p16 * step_mhz / tc["f16"]["sm_mhz"]
            roofline["frac_at_step_clock"] = (kernels["attn_bwd_kernel"]["tops"]
                                              / mixed_peak(p8c, p16c, 4, 1))
            line_extra["frac_of_weighted_peak_at_step_clock"] = (
                value / world / mixed_peak(p8c, p16c, 6, 1))
        line_extra.update(frac_of_weighted_peak=value / world / p_all, weighted_peak_tops=p_all)
    # the prologue's HBM roofline: 9 algorithmic bytes per (token, channel) -- q, k, v read at
    # 2 bytes and their INT8 codes written at 1 byte
    pro_bytes = 9.0 * w.B * w.H * w.N * w.d
    pro_gbs = pro_bytes / (part["prologue"] * 1e-3) / 1e9
    prologue = {"ms": part["prologue"], "algorithmic_bytes": pro_bytes, "gbs": pro_gbs,
                "peak_gbs": pk["hbm_gbs"], "frac": pro_gbs / pk["hbm_gbs"],
                "peak_note": f"{pk['basis']} HBM copy bandwidth"}

    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8+bf16", "data": "synthetic", "config": config_of(w),
            **line_extra,
            "kernels": {n: {k_: round(v_, 4) for k_, v_ in d.items()}
                        for n, d in kernels.items()},
            "stages_ms": {n: round(v_, 4) for n, v_ in part.items()},
            "prologue": prologue, "tensor_peaks": tc,
            "cublas_bf16_tflops": {"burst": pk["bf16_burst"], "sustained": pk["bf16_sustained"],
                                   "basis": pk["basis"]},
            "roofline": roofline, "clocks": clocks, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, 4)
        line["cpu_baseline"].pop("seconds", None)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
