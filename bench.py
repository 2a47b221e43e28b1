#!/usr/bin/env python
"""Throughput of the wav2vec2-base CTC forward on the fixed 16 s window.

One step = one pass of the whole hot path over one 16 s clip (256000 samples,
799 frames): conv feature encoder -> projection -> positional conv -> 12
post-norm blocks -> CTC head -> per-frame argmax -> greedy CTC collapse, all
in the library's CUDA kernels, replayed as one CUDA graph.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  With N > 1 (launched by torchrun) every rank
runs an independent replica of the same workload (a single clip does not
shard); value = audio seconds processed by all ranks / max-over-ranks time.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "audio-sec/s (RTFx) of wav2vec2 CTC forward @16 s; % tensor-core & HBM roofline"
UNIT = "audio-sec/s"
WORKLOAD = ("c1: wav2vec2-base shape, random-init, fixed 16 s window (256000 samples at 16 kHz -> 799 frames), "
            "batch 1, tanh-GELU, fp16 operands / fp32 accumulation, norms and softmax")
N_SAMPLES = 256000
AUDIO_SEC = N_SAMPLES / 16000.0
TENSOR_CLASSES = {"conv_gemm", "proj_gemm", "posconv", "qkv_gemm", "attention", "out_gemm", "ffn1_gemm",
                  "ffn2_gemm", "lm_head_gemm"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="measure only the headline workload (c1), not c0/c2/c3/c4")
    return ap.parse_args()


def config_dict(n):
    return {"workload": WORKLOAD, "global_batch": n, "seq_len": N_SAMPLES, "frames": 799,
            "parallelism": f"replicas x{n}" if n > 1 else "single GPU",
            "l2": "flushed between timed steps (256 MiB write outside the timed events)"}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------------ clocks
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.idx)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
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
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_id(local_rank: int) -> str:
    """nvidia-smi identifier (UUID) of the CUDA device this rank uses."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(local_rank).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local_rank)


def clocks_bad(c):
    if not c:
        return False
    if set(c["reasons"]) & {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}:
        return True
    return c["sm_mhz"] < 0.5 * c["sm_max_mhz"] and "sw_power_cap" not in c["reasons"]


# --------------------------------------------------------------- traffic
def ncu_traffic(kernel_class):
    """Per-launch DRAM bytes of a kernel class from the committed ncu summary,
    or None if absent or if the kernel's source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_class)
    if not e:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != e["source_sha256"]:
        return None
    return e["dram_bytes_per_launch"]


# -------------------------------------------------------------------- ours
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    from speech_encoder_b200 import w2v as B
    from synth import inputs as S

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = S.workload("c1")
    shape = w.model
    pcm_np = w.calls[0][0]  # the full 16 s clip, [1, 256000]
    blob = S.pack_blob(shape, S.init_weights(shape, 0))
    model = B.Model(shape, blob, max_samples=N_SAMPLES, max_batch=1, use_cuda_graph=True)
    del blob
    T = B.w2v_num_frames(N_SAMPLES)
    pcm = torch.from_numpy(pcm_np).to(dev)
    logits = torch.empty((1, T, shape.vocab), dtype=torch.float32, device=dev)
    tokens = torch.empty((1, T), dtype=torch.int32, device=dev)
    ntok = torch.empty((1,), dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        B.w2v_forward(model.handle, pcm, N_SAMPLES, 1, logits, stream)
        B.w2v_ctc_greedy(model.handle, logits, 1, T, T, tokens, ntok, stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        step()
    model.sync()
    launches_per_step = B.w2v_last_launch_count(model.handle) + 2

    def timed_region():
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        clk = Clocks(gpu_id(local_rank))
        clk.start()
        for i in range(args.steps):
            flush.zero_()
            ev0[i].record(stream)
            step()
            ev1[i].record(stream)
        torch.cuda.synchronize()
        barrier()
        c = clk.stop()
        total = sum(a.elapsed_time(b) for a, b in zip(ev0, ev1))
        return total, c

    total_ms, clocks = timed_region()
    if clocks_bad(clocks):
        total_ms, clocks = timed_region()
    model.sync()
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([total_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    value = world * args.steps * AUDIO_SEC / (total_ms / 1000.0)

    # ---- per-kernel timing and roofline: each kernel class's launches of this
    # forward replayed back to back in a CUDA graph, CUDA events around the
    # replay on this stream, divided by the launch count (w2v_time_class).
    hbm_peak, tc_peak, peak_src = measured_peaks()
    per_class = {}
    for name in B.KERNEL_CLASSES:
        us, n, fl, by = B.w2v_time_class(model.handle, pcm, N_SAMPLES, 1, logits, name, reps=10, stream=stream)
        if n:
            per_class[name] = {"us": us, "launches": n, "flops": fl, "bytes": by}
    tot = sum(e["us"] * e["launches"] for e in per_class.values())
    kernels = {}
    for name, e in sorted(per_class.items(), key=lambda kv: -kv[1]["us"] * kv[1]["launches"]):
        k = {"us_per_launch": e["us"], "launches_per_step": e["launches"],
             "ms_per_step": e["us"] * e["launches"] / 1000.0, "share": e["us"] * e["launches"] / tot}
        if name in TENSOR_CLASSES:
            k["tflops"] = e["flops"] / (e["us"] * 1e-6) / 1e12
            k["frac_tensor"] = k["tflops"] / tc_peak
        else:
            k["gbs"] = e["bytes"] / (e["us"] * 1e-6) / 1e9
            k["frac_hbm"] = k["gbs"] / hbm_peak
        kernels[name] = k
    dom = max(per_class, key=lambda nm: per_class[nm]["us"] * per_class[nm]["launches"])
    e = per_class[dom]
    tensor = dom in TENSOR_CLASSES
    achieved = (e["flops"] / (e["us"] * 1e-6) / 1e12) if tensor else (e["bytes"] / (e["us"] * 1e-6) / 1e9)
    peak = tc_peak if tensor else hbm_peak
    roofline = {"kernel": dom, "bound": "tensor" if tensor else "hbm", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s" if tensor else "GB/s", "frac": achieved / peak, "traffic": ncu_traffic(dom),
                "peak_source": f"{peak_src} ({'bf16/fp16 dense burst' if tensor else 'HBM copy'})",
                "algorithmic_per_launch": e["flops"] if tensor else e["bytes"],
                "us_per_launch": e["us"], "launches_per_step": e["launches"]}
    gemm_us = sum(per_class[nm]["us"] * per_class[nm]["launches"] for nm in per_class if nm in TENSOR_CLASSES)
    gemm_fl = sum(per_class[nm]["flops"] * per_class[nm]["launches"] for nm in per_class if nm in TENSOR_CLASSES)
    tensor_frac_all = gemm_fl / (gemm_us * 1e-6) / 1e12 / tc_peak

    # ---- end to end through the public host-buffer entry point
    pcm_host = torch.from_numpy(pcm_np.copy()).pin_memory()
    tok_host = torch.empty((1, T), dtype=torch.int32).pin_memory()
    nt_host = torch.empty((1,), dtype=torch.int32).pin_memory()

    def e2e_step():
        B.w2v_transcribe(model.handle, pcm_host.numpy(), T, tok_host.numpy(), nt_host.numpy(), stream)

    for _ in range(max(args.warmup, 3)):
        e2e_step()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e0[i].record(stream)
        e2e_step()
        e1[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in zip(e0, e1))
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e = {"value": world * args.steps * AUDIO_SEC / (e2e_ms / 1000.0), "unit": UNIT,
           "h2d_bytes_per_step": int(pcm_host.numel() * 4),
           "d2h_bytes_per_step": int(tok_host.numel() * 4 + nt_host.numel() * 4)}
    model.close()

    # ---- the other workloads (one GPU only; the headline stays c1)
    extra = {}
    if world == 1 and not args.no_extra_configs:
        for name in ("c0", "c2", "c3", "c4"):
            extra[name] = measure_workload(name, max(5, min(args.steps, 20)), args.warmup, tc_peak, dev, flush)

    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f16", "data": "synthetic (seeded sinusoids + noise PCM, random-init weights)",
           "config": config_dict(world), "frames_per_s": value / AUDIO_SEC * T, "roofline": roofline,
           "tensor_frac_all_contractions": tensor_frac_all, "kernels": kernels, "e2e": e2e,
           "gpu_launches": launches_per_step * args.steps, "clocks": clocks}
    if extra:
        out["other_workloads"] = extra
    return out


# ------------------------------------------------------- the other workloads
OTHER_WORKLOADS = {
    "c0": "wav2vec2-base shape, random-init, batch 1, 1 s (16000 samples -> 49 frames), exact GELU",
    "c2": "wav2vec2-base shape, random-init, 16 clips of 10 s (160000 samples -> 499 frames each), exact GELU",
    "c3": "wav2vec2-large stable-layer-norm shape, random-init, batch 1, 16 s (256000 samples -> 799 frames), "
          "2341-token head, exact GELU",
    "c4": "wav2vec2-large stable-layer-norm shape, random-init, 8 true-length clips of 2-20 s (seeded lengths), "
          "exact GELU",
}


def contraction_flops(shape, n):
    """Algorithmic FLOPs (2 per multiply-add) of the tensor-core work of one
    clip of n samples: conv layers, projection, positional conv, QKV,
    attention, out-projection, FFN and CTC head."""
    ks, ss = (10, 3, 3, 3, 3, 2, 2), (5, 2, 2, 2, 2, 2, 2)
    T, t, fl = [], n, 0.0
    for k, st in zip(ks, ss):
        t = (t - k) // st + 1 if t >= k else 0
        T.append(t)
    fl += 2.0 * 10 * 512 * T[0]
    for i in range(1, 7):
        fl += 2.0 * T[i] * 512 * 512 * ks[i]
    Tf, d, F, V = T[6], shape.d_model, shape.d_ffn, shape.vocab
    fl += 2.0 * Tf * d * 512 + 2.0 * Tf * d * (d // 16) * 128
    fl += shape.n_layers * (2.0 * Tf * 3 * d * d + 4.0 * Tf * Tf * d + 2.0 * Tf * d * d + 4.0 * Tf * F * d)
    fl += 2.0 * Tf * V * d
    return fl


def measure_workload(name, steps, warmup, tc_peak, dev, flush, cpu_budget_s=10.0):
    """Device throughput of one of the other workloads (the clips as the
    workload lists them, forward + greedy CTC per step, L2 flushed between
    steps), the tensor fraction of its contractions, and the fp64 oracle on a
    bounded sample of the same workload on the host cores."""
    import numpy as np
    import torch

    from speech_encoder_b200 import w2v as B
    from synth import inputs as S
    w = S.workload(name)
    shape = w.model
    stream = torch.cuda.current_stream()
    blob = S.pack_blob(shape, S.init_weights(shape, 0))
    lens = [int(p.shape[1]) for p, _ in w.calls for _ in range(p.shape[0])]
    audio = sum(lens) / 16000.0
    frames = sum(B.w2v_num_frames(n) for n in lens)
    flops = sum(contraction_flops(shape, n) for n in lens)
    if name == "c4":
        model = B.Model(shape, blob, max_samples=max(lens), max_batch=len(lens), use_cuda_graph=False)
        pcm = torch.from_numpy(np.concatenate([p[0] for p, _ in w.calls])).to(dev)
        T = [B.w2v_num_frames(n) for n in lens]
        logits = torch.empty((sum(T), shape.vocab), dtype=torch.float32, device=dev)
        tokens = torch.empty((sum(T),), dtype=torch.int32, device=dev)
        ntok = torch.empty((len(T),), dtype=torch.int32, device=dev)

        def step():
            B.w2v_forward_varlen(model.handle, pcm, lens, logits, stream)
            B.w2v_ctc_greedy_varlen(model.handle, logits, T, tokens, ntok, stream)
        path = "varlen: 8 true-length clips in one launch set (w2v_forward_varlen + w2v_ctc_greedy_varlen)"
    else:
        p_np = w.calls[0][0]
        bsz, n = p_np.shape
        model = B.Model(shape, blob, max_samples=n, max_batch=bsz, use_cuda_graph=True)
        pcm = torch.from_numpy(p_np).to(dev)
        T = B.w2v_num_frames(n)
        logits = torch.empty((bsz, T, shape.vocab), dtype=torch.float32, device=dev)
        tokens = torch.empty((bsz, T), dtype=torch.int32, device=dev)
        ntok = torch.empty((bsz,), dtype=torch.int32, device=dev)

        def step():
            B.w2v_forward(model.handle, pcm, n, bsz, logits, stream)
            B.w2v_ctc_greedy(model.handle, logits, bsz, T, T, tokens, ntok, stream)
        path = f"w2v_forward batch {bsz} x {n} samples as one CUDA graph + w2v_ctc_greedy"
    del blob
    for _ in range(max(warmup, 3)):
        step()
    model.sync()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        e0[i].record(stream)
        step()
        e1[i].record(stream)
    torch.cuda.synchronize()
    model.sync()
    ms = sum(a.elapsed_time(b) for a, b in zip(e0, e1)) / steps
    out = {"workload": OTHER_WORKLOADS[name], "path": path, "audio_s_per_step": audio, "ms_per_step": ms,
           "audio_s_per_s": audio / (ms / 1000.0), "frames_per_s": frames / (ms / 1000.0),
           "contraction_gflop_per_step": flops / 1e9,
           "tensor_frac_of_step": flops / (ms * 1e-3) / 1e12 / tc_peak}
    if name != "c4":
        # per-class kernel times, as for the headline workload
        us_t, fl_t, per = 0.0, 0.0, {}
        bsz, n = w.calls[0][0].shape
        for cls in B.KERNEL_CLASSES:
            us, nl, fl, _ = B.w2v_time_class(model.handle, pcm, n, bsz, logits, cls, reps=5, stream=stream)
            if not nl:
                continue
            per[cls] = {"us_per_launch": round(us, 2), "launches_per_step": nl, "ms_per_step": round(us * nl / 1000, 4)}
            if cls in TENSOR_CLASSES:
                us_t += us * nl
                fl_t += fl * nl
                per[cls]["frac_tensor"] = round(fl / (us * 1e-6) / 1e12 / tc_peak, 4)
        out["tensor_frac_all_contractions"] = fl_t / (us_t * 1e-6) / 1e12 / tc_peak
        out["kernels"] = dict(sorted(per.items(), key=lambda kv: -kv[1]["ms_per_step"]))
    model.close()
    # the oracle on a bounded sample of the same workload (host cores)
    from oracle import w2v_oracle as O
    W64 = O.to_f64(S.init_weights(shape, 0))
    clips = [p[i] for p, _ in w.calls for i in range(p.shape[0])]
    clips.sort(key=len)
    t0, done, secs = time.perf_counter(), 0, 0.0
    for c in clips:
        z = O.forward(shape, W64, c)
        O.ctc_greedy(z, z.shape[0], 0)
        done += 1
        secs += len(c) / 16000.0
        if time.perf_counter() - t0 >= cpu_budget_s:
            break
    wall = time.perf_counter() - t0
    out["cpu_oracle"] = {"audio_s_per_s": secs / wall, "cores": blas_threads(),
                         "sample": f"{done} of {len(clips)} clip(s), shortest first, {secs:.1f} audio s in {wall:.1f} s"}
    return out


# ---------------------------------------------------------------- oracle arm
def oracle_sample(seconds_budget: float):
    """Times the fp64 oracle on the 16 s clip: full forward + CTC, repeated until
    the budget is used (at least once).  Returns (audio-sec/s, runs, wall)."""
    from oracle import w2v_oracle as O
    from synth import inputs as S
    w = S.workload("c1")
    W64 = O.to_f64(S.init_weights(w.model, 0))
    pcm = w.calls[0][0][0]
    runs, t0 = 0, time.perf_counter()
    while True:
        z = O.forward(w.model, W64, pcm)
        O.ctc_greedy(z, z.shape[0], 0)
        runs += 1
        if time.perf_counter() - t0 >= seconds_budget:
            break
    wall = time.perf_counter() - t0
    return runs * AUDIO_SEC / wall, runs, wall


# timed oracle work of the reference arm (seconds); tests shorten it
REFERENCE_BUDGET_S = float(os.environ.get("W2V_BENCH_REFERENCE_BUDGET_S", "90"))


def run_reference(args, world):
    from oracle import w2v_oracle as O
    from synth import inputs as S
    w = S.workload("c1")
    W64 = O.to_f64(S.init_weights(w.model, 0))
    pcm = w.calls[0][0][0]

    def step():
        z = O.forward(w.model, W64, pcm)
        O.ctc_greedy(z, z.shape[0], 0)

    # The oracle needs seconds per step: one warm-up step (BLAS thread start-up
    # is its only warm-up effect), then as many of the requested timed steps
    # as fit in REFERENCE_BUDGET_S, at least one, so that the run stays within
    # a few minutes whatever --steps / --warmup ask for.
    t0 = time.perf_counter()
    step()
    est = time.perf_counter() - t0
    warmup = 1
    steps = max(1, min(args.steps, int(REFERENCE_BUDGET_S // max(est, 1e-3))))
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = steps * AUDIO_SEC / total
    cores = blas_threads()
    sample = (f"{steps} timed step(s) of the {args.steps} requested (+{warmup} warm-up), each the full 16 s clip: "
              f"fp64 numpy forward + greedy CTC")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": 1000 * total / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded sinusoids + noise PCM, random-init weights)", "config": config_dict(world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args, world)), flush=True)
        return
    # The oracle baseline runs before any CUDA work (a BLAS thread pool and a
    # CUDA context in one process are fine, but this keeps the timing clean).
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, runs, wall = oracle_sample(10.0)
        cpu = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{runs} x the 16 s clip (fp64 numpy forward + greedy CTC), {wall:.1f} s wall"}
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    out = run_ours(args, rank, world, local_rank)
    out["cpu_baseline"] = cpu
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
