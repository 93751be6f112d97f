"""Benchmark of the attention hot path on B200; prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline: causal GQA prefill (batch 4, 32 query / 8 key-value heads, head_dim 128, 2048
queries and keys, bf16, fp32 accumulation), TFLOP/s over the unmasked (attended) pairs,
4*head_dim flops per pair. The same line carries the other workloads of the hot path, each
timed the same way: KV-cache decode (HBM GB/s), ALiBi/T5 bias attention (fp16), and
block-sparse masked attention (with its block classification pass).

Timing: W untimed warm-up steps, then K steps, each preceded by an L2 flush (a 256 MiB write)
and timed on the launching stream with CUDA events; the K steps are bracketed by a barrier and
torch.cuda.synchronize() and the max over ranks is taken. With N GPUs every rank runs its own
copy of the workload (independent batches; no collective on the data path): weak scaling.

--impl reference times the CPU float64 oracle (the slow reference program) on a bounded
sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import sdpa_inputs as si  # noqa: E402

FLUSH_BYTES = 256 << 20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def causal_pairs(Lq, Lk, offset=0):
    """Number of (query, key) pairs with key <= offset + query, key < Lk."""
    i = np.arange(Lq, dtype=np.int64)
    return int(np.clip(offset + i + 1, 0, Lk).sum())


# ---- distributed plumbing -------------------------------------------------------------------

def init_dist(n_gpus, backend=None):
    """Process group from the torchrun environment (one rank per GPU over NCCL; gloo when
    there is no GPU, which the CPU tests use)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group(backend, timeout=timeout)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world):
    """The largest x over the ranks (device times: the job takes as long as its slowest rank)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---- clocks ---------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---- timing ---------------------------------------------------------------------------------

def time_steps(step, steps, warmup, world, stream=None):
    """Device time (ms) of each of `steps` calls of step(), each after an L2 flush."""
    stream = stream or torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for s in range(steps):
        flush.zero_()
        starts[s].record(stream)
        step()
        ends[s].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    per = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    return per


# ---- workloads --------------------------------------------------------------------------------

def prefill_case(dev):
    w = si.CAUSAL_GQA_PREFILL
    q, k, v = si.qkv(w)
    flops = 4.0 * w.head_dim * w.batch * w.nheads * causal_pairs(w.q_len, w.kv_len)
    byts = (q.numel() + k.numel() + v.numel() + q.numel()) * 2
    return w, (q, k, v), flops, byts


def run_ours(args, rank, world, local):
    import head_scaled_dot_sdpa_b200 as sdpa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = _peaks()
    stream = torch.cuda.current_stream()
    result = {}

    # ---- headline: causal GQA prefill
    w, (q, k, v), flops, byts = prefill_case(dev)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty_like(qd)
    ws = sdpa.Workspace(dev)
    step = lambda: sdpa.sdpa_forward(qd, kd, vd, is_causal=True, out=out, workspace=ws)
    step()
    kernel = sdpa.last_kernel()
    with ClockSampler(local) as clk:
        per = time_steps(step, args.steps, args.warmup, world)
    ms = max_over_ranks(float(np.sum(per)), world) / args.steps
    status = sdpa.read_device_status(ws)
    value = flops * world / (ms * 1e-3) / 1e12
    kernel_tflops = flops / (float(np.mean(per)) * 1e-3) / 1e12

    # ---- e2e through the public API with host buffers (pinned), copies inside the timed region
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step():
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        sdpa.sdpa_forward(qd, kd, vd, is_causal=True, out=out, workspace=ws)
        oh.copy_(out, non_blocking=True)

    per_e2e = time_steps(e2e_step, args.steps, args.warmup, world)
    ms_e2e = max_over_ranks(float(np.sum(per_e2e)), world) / args.steps
    h2d = (q.numel() + k.numel() + v.numel()) * q.element_size()
    d2h = out.numel() * out.element_size()

    result.update({
        "metric": "prefill attention TFLOP/s (unmasked FLOPs)",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1), numpy PCG64)",
        "config": {"workload": w.name, "batch": w.batch, "q_len": w.q_len, "kv_len": w.kv_len,
                   "nheads": w.nheads, "nkvheads": w.nkvheads, "head_dim": w.head_dim,
                   "is_causal": True, "flops_per_step": flops,
                   "l2": "flushed before every timed step (256 MiB write)",
                   "parallelism": f"replica per GPU x{world} (independent batches)"},
        "kernel": kernel,
        "device_status": int(status),
        "roofline": {"bound": "tensor", "achieved": round(kernel_tflops, 2), "peak": peaks["bf16"],
                     "unit": "TFLOP/s", "frac": round(kernel_tflops / peaks["bf16"], 4),
                     "traffic": None, "peak_source": f"{peaks['source']} bf16 burst",
                     "frac_of_sustained": round(kernel_tflops / peaks["bf16_sustained"], 4)},
        "e2e": {"value": round(flops * world / (ms_e2e * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 4)},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    })
    del qd, kd, vd, out, qh, kh, vh, oh

    if not args.headline_only:
        result["other_workloads"] = other_workloads(args, dev, world, ws, peaks)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    return result


def other_workloads(args, dev, world, ws, peaks):
    """The other rows of the hot path, each timed like the headline. A workload that raises is
    reported as {"error": ...} so that the line with the headline is still printed."""
    runs = (("decode", "kv_cache_decode", lambda: decode_workload(args, dev, world, ws, peaks)),
            ("bias", "alibi_t5_bias", lambda: bias_workload(args, dev, world, ws, peaks)),
            ("block_sparse", "block_sparse_mask", lambda: block_sparse_workload(args, dev, world, ws, peaks)),
            ("packed", "packed_docs", lambda: packed_workload(args, dev, world, ws, peaks)),
            ("backward", "fused_gradient", lambda: backward_workload(args, dev, world, ws, peaks)),
            ("weights", "with_weights", lambda: weights_workload(args, dev, world, ws, peaks)),
            ("rope", "rotary_embedding", lambda: rope_workload(args, dev, world, peaks)),
            ("rope_prefill", "rope_prefill", lambda: rope_prefill_workload(args, dev, world, ws, peaks)))
    res = {}
    for key, name, run in runs:
        if key not in args.workloads:
            continue
        try:
            res[name] = run()
        except Exception as e:  # noqa: BLE001 - reported in the JSON line
            res[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
    return res


def decode_workload(args, dev, world, ws, peaks):
    """KV-cache decode: HBM GB/s over the bytes a step must move."""
    import dataclasses
    import head_scaled_dot_sdpa_b200 as sdpa

    w = si.KV_CACHE_DECODE
    if args.shrink > 1:
        w = dataclasses.replace(w, batch=max(1, w.batch // args.shrink))
    d = si.decode_inputs(w)
    qd, kn, vn = d["q"].to(dev), d["k_new"].to(dev), d["v_new"].to(dev)
    kc, vc = d["k_cache"].to(dev), d["v_cache"].to(dev)
    idx = d["index"].to(dev)
    out = torch.empty_like(qd)
    kl = d["kv_lengths"].numpy().astype(np.int64)
    byts = (int(kl.sum()) * w.nkvheads * w.head_dim * 2 * 2 + 2 * qd.numel() * 2 + 4 * kn.numel() * 2)
    step = lambda: sdpa.sdpa_decode_with_cache(qd, kn, vn, kc, vc, idx, out=out, workspace=ws)
    per = time_steps(step, args.steps, args.warmup, world)
    ms = max_over_ranks(float(np.mean(per)), world)
    gbs = byts / (ms * 1e-3) / 1e9
    return {"workload": w.name, "metric": "decode HBM GB/s", "value": round(gbs * world, 1),
            "unit": "GB/s", "ms_per_step": round(ms, 4), "bytes_per_step": byts, "batch": w.batch,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm"],
                         "unit": "GB/s", "frac": round(gbs / peaks["hbm"], 4)},
            "kernel": sdpa.last_kernel(), "gpu_launches_per_step": 4}


def bias_workload(args, dev, world, ws, peaks):
    """ALiBi/T5 bias attention (fp16, causal, additive bias broadcast over the batch). Its
    binding roof is HBM: the causal half of the bias (read once: both batch elements of a
    (head, query tile) share it through L2) plus Q, K, V read and O written."""
    import head_scaled_dot_sdpa_b200 as sdpa

    w = si.ALIBI_T5_BIAS
    q, k, v = [t.to(dev) for t in si.qkv(w)]
    bias = si.alibi_t5_bias(w).to(dev)
    out = torch.empty_like(q)
    pairs = causal_pairs(w.q_len, w.kv_len)
    flops = 4.0 * w.head_dim * w.batch * w.nheads * pairs
    step = lambda: sdpa.sdpa_forward(q, k, v, bias, is_causal=True, out=out, workspace=ws)
    per = time_steps(step, args.steps, args.warmup, world)
    ms = max_over_ranks(float(np.mean(per)), world)
    bias_bytes = w.nheads * pairs * 2
    byts = bias_bytes + 4 * q.numel() * 2
    gbs = byts / (ms * 1e-3) / 1e9
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": w.name, "value": round(tf * world, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "flops_per_step": flops, "bytes_per_step": byts,
            "bias_GBs": round(bias_bytes / (ms * 1e-3) / 1e9, 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm"], 4), "traffic": None,
                         "peak_source": f"{peaks['source']} HBM copy",
                         "tensor": {"achieved": round(tf, 2), "peak": peaks["bf16"], "unit": "TFLOP/s",
                                    "frac": round(tf / peaks["bf16"], 4)}},
            "kernel": sdpa.last_kernel(), "gpu_launches_per_step": 1}


def block_sparse_workload(args, dev, world, ws, peaks):
    """Block-sparse mask: the classification pass, then attention over the non-empty blocks."""
    import dataclasses
    import head_scaled_dot_sdpa_b200 as sdpa

    w = si.BLOCK_SPARSE
    if args.shrink > 1:
        w = dataclasses.replace(w, q_len=w.q_len // args.shrink, kv_len=w.kv_len // args.shrink)
    cls = si.block_classes(w)
    mask = si.mask_device(w, cls, dev)
    allowed = int(mask.sum(dtype=torch.int64).item())
    q, k, v = [t.to(dev) for t in si.qkv(w)]
    out = torch.empty_like(q)
    info = sdpa.build_block_mask_info(mask)
    step_c = lambda: sdpa.build_block_mask_info(mask)
    per_c = time_steps(step_c, args.steps, args.warmup, world)
    ms_c = max_over_ranks(float(np.mean(per_c)), world)
    step = lambda: sdpa.sdpa_forward(q, k, v, block_info=info, out=out, workspace=ws)
    per = time_steps(step, args.steps, args.warmup, world)
    ms = max_over_ranks(float(np.mean(per)), world)
    flops = 4.0 * w.head_dim * allowed
    # executed work: every (query, key) pair of the non-empty blocks (the diagonal forcing can
    # turn an empty block partial, so the classes are counted from the classification itself)
    n_blocks = int((info.arrays()["cls"] != 0).sum().item())
    exec_flops = 4.0 * w.head_dim * n_blocks * 128 * 128
    exec_tf = exec_flops / (ms * 1e-3) / 1e12
    cgbs = mask.numel() / (ms_c * 1e-3) / 1e9
    return {
        "workload": w.name, "q_len": w.q_len, "value": round(flops / (ms * 1e-3) / 1e12 * world, 2), "unit": "TFLOP/s (unmasked)",
        "ms_per_step": round(ms, 4), "flops_per_step": flops, "executed_flops_per_step": exec_flops,
        "executed_tflops": round(exec_tf, 2),
        "roofline": {"bound": "tensor", "achieved": round(exec_tf, 2), "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": round(exec_tf / peaks["bf16"], 4), "traffic": None,
                     "basis": "executed flops (non-empty 128x128 blocks)",
                     "peak_source": f"{peaks['source']} bf16 burst"},
        "classification": {"ms": round(ms_c, 4), "GB/s": round(cgbs, 1),
                           "roofline": {"bound": "hbm", "achieved": round(cgbs, 1), "peak": peaks["hbm"],
                                        "unit": "GB/s", "frac": round(cgbs / peaks["hbm"], 4)}},
        "kernel": sdpa.last_kernel(), "gpu_launches_per_step": 1}


def packed_workload(args, dev, world, ws, peaks):
    """Packed sequences: documents of 64 to 4096 positions one after the other, each attending
    causally to itself only (the segment scan and the attention kernel, every step)."""
    import head_scaled_dot_sdpa_b200 as sdpa

    w = si.PACKED_DOCS
    segs = si.packed_segments(w)
    q, k, v = [t.to(dev) for t in si.packed_qkv(w)]
    seg = torch.tensor(segs, dtype=torch.int32, device=dev)
    maxlen = max(segs)
    out = torch.empty_like(q)
    flops = 4.0 * w.head_dim * w.nheads * sum(causal_pairs(n, n) for n in segs)
    step = lambda: sdpa.sdpa_forward_packed(q, k, v, seg, maxlen=maxlen, is_causal=True, out=out, workspace=ws)
    per = time_steps(step, args.steps, args.warmup, world)
    ms = max_over_ranks(float(np.mean(per)), world)
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": w.name, "segments": len(segs), "maxlen": maxlen, "value": round(tf * world, 2),
            "unit": "TFLOP/s", "ms_per_step": round(ms, 4), "flops_per_step": flops,
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16"], "unit": "TFLOP/s",
                         "frac": round(tf / peaks["bf16"], 4)},
            "kernel": sdpa.last_kernel(), "gpu_launches_per_step": 2}


def backward_workload(args, dev, world, ws, peaks):
    """The fused gradient (dq, dk, dv, dscale) of the causal GQA prefill workload, given the row
    log-sum-exp the forward kept (sdpa_forward_lse, outside the timed region, as in a training
    step): 10*head_dim flops per attended pair (the logits recomputed, dout.v, and the dv, dq
    and dk products; the recomputation of the logits in both gradient kernels and the low parts
    of dx are not counted). Three launches: delta, dK/dV, dQ."""
    import head_scaled_dot_sdpa_b200 as sdpa

    w = si.CAUSAL_GQA_PREFILL
    q, k, v = [t.to(dev) for t in si.qkv(w)]
    dout = si.normal(si.rng_for(w.seed + 7), tuple(q.shape), w.dtype).to(dev)
    # the forward of the training step keeps the row log-sum-exp for the gradient
    out, lse = sdpa.sdpa_forward_lse(q, k, v, is_causal=True, workspace=ws)
    flops = 10.0 * w.head_dim * w.batch * w.nheads * causal_pairs(w.q_len, w.kv_len)
    step = lambda: sdpa.sdpa_backward(q, k, v, out, dout, is_causal=True, lse=lse, workspace=ws)
    per = time_steps(step, max(3, args.steps // 4), args.warmup, world)
    ms = max_over_ranks(float(np.mean(per)), world)
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": w.name + "_backward", "value": round(tf * world, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "flops_per_step": flops,
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16"], "unit": "TFLOP/s",
                         "frac": round(tf / peaks["bf16"], 5)},
            "kernel": sdpa.last_kernel(),
            "gpu_launches_per_step": {"backward_tcgen05": 3, "backward_mma": 2}.get(sdpa.last_kernel(), 3)}


def weights_workload(args, dev, world, ws, peaks):
    """scaled_dot_product_attention_with_weights with dropout (p = 0.1) on the causal GQA
    workload: the whole (batch, nheads, q_len, kv_len) weight array is written, so the step is
    bound by that write (plus reading Q, K, V and writing out). The tcgen05 path runs three
    kernels per step: the forward with the row log-sum-exp, the fill of the weights past each
    query tile's causal bound, and the weights pass."""
    import head_scaled_dot_sdpa_b200 as sdpa

    w = si.CAUSAL_GQA_PREFILL
    q, k, v = [t.to(dev) for t in si.qkv(w)]
    out = torch.empty_like(q)
    weights = torch.empty((w.batch, w.nheads, w.q_len, w.kv_len), dtype=q.dtype, device=dev)
    byts = weights.numel() * 2 + 2 * q.numel() * 2 + 2 * k.numel() * 2
    step = lambda: sdpa.sdpa_forward_with_weights(q, k, v, is_causal=True, drop_p=0.1, seed=1, out=out,
                                                  weights=weights, workspace=ws)
    per = time_steps(step, max(3, args.steps // 4), args.warmup, world)
    ms = max_over_ranks(float(np.mean(per)), world)
    gbs = byts / (ms * 1e-3) / 1e9
    return {"workload": w.name + "_with_weights_p0.1", "metric": "HBM GB/s", "value": round(gbs * world, 1),
            "unit": "GB/s", "ms_per_step": round(ms, 3), "bytes_per_step": byts,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm"], 4)},
            "kernel": sdpa.last_kernel(),
            "gpu_launches_per_step": 3 if sdpa.last_kernel() == "weights_tcgen05" else 1}


def rope_workload(args, dev, world, peaks):
    """Rotary embedding of the causal GQA workload's q and k (positions 0..2047 in each
    sequence): an elementwise pass, bound by reading and writing both arrays once."""
    import head_scaled_dot_sdpa_b200 as sdpa

    w = si.CAUSAL_GQA_PREFILL
    q, k, _ = [t.to(dev) for t in si.qkv(w)]
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    pos = torch.arange(w.q_len, dtype=torch.int32, device=dev).repeat(w.batch)
    byts = 2 * (q.numel() + k.numel()) * 2 + 2 * pos.numel() * 4

    def step():
        sdpa.sdpa_rope(q, pos, out=qo)
        sdpa.sdpa_rope(k, pos, out=ko)

    per = time_steps(step, args.steps, args.warmup, world)
    ms = max_over_ranks(float(np.mean(per)), world)
    gbs = byts / (ms * 1e-3) / 1e9
    return {"workload": w.name + "_rope_qk", "metric": "HBM GB/s", "value": round(gbs * world, 1), "unit": "GB/s",
            "ms_per_step": round(ms, 4), "bytes_per_step": byts,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm"], 4)},
            "kernel": "rope_kernel", "gpu_launches_per_step": 2}


def rope_prefill_workload(args, dev, world, ws, peaks):
    """The causal GQA prefill workload with the rotary embedding of q and k folded in
    (sdpa_forward_rope, positions 0..2047 in every sequence): the keys are rotated once into the
    workspace, a table kernel takes the query angles' cos / sin, and the attention kernel rotates
    each Q tile in shared memory. TFLOP/s on the same flop count as the headline."""
    import head_scaled_dot_sdpa_b200 as sdpa

    w = si.CAUSAL_GQA_PREFILL
    q, k, v = [t.to(dev) for t in si.qkv(w)]
    out = torch.empty_like(q)
    pos = torch.arange(w.q_len, dtype=torch.int32, device=dev).repeat(w.batch)
    flops = 4.0 * w.head_dim * w.batch * w.nheads * causal_pairs(w.q_len, w.kv_len)
    step = lambda: sdpa.sdpa_forward_rope(q, k, v, pos, pos, is_causal=True, out=out, workspace=ws)
    per = time_steps(step, args.steps, args.warmup, world)
    ms = max_over_ranks(float(np.mean(per)), world)
    tf = flops / (ms * 1e-3) / 1e12
    return {"workload": w.name + "_rope_fused", "value": round(tf * world, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "flops_per_step": flops,
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16"], "unit": "TFLOP/s",
                         "frac": round(tf / peaks["bf16"], 4), "traffic": None},
            "kernel": sdpa.last_kernel(), "gpu_launches_per_step": 3}


# ---- CPU oracle ---------------------------------------------------------------------------------

def _oracle_heads(q, k, v, heads, group):
    """Run the oracle on (b, h) heads of the causal GQA workload, one head per call."""
    import oracle
    qn, kn, vn = (t.float().numpy() for t in (q, k, v))
    flops = 0.0
    for b, h in heads:
        g = h // group
        oracle.sdpa_forward(qn[b:b + 1, :, h:h + 1], kn[b:b + 1, :, g:g + 1], vn[b:b + 1, :, g:g + 1],
                            is_causal=True)
        flops += 4.0 * q.shape[3] * causal_pairs(q.shape[1], k.shape[1])
    return flops


def cpu_baseline(budget_s=20.0):
    import oracle
    oracle.load()
    w = si.CAUSAL_GQA_PREFILL
    q, k, v = si.qkv(w)
    group = w.nheads // w.nkvheads
    all_heads = [(b, h) for b in range(w.batch) for h in range(w.nheads)]
    t0 = time.perf_counter()
    flops, done = 0.0, 0
    for chunk in range(0, len(all_heads), 8):
        flops += _oracle_heads(q, k, v, all_heads[chunk:chunk + 8], group)
        done += len(all_heads[chunk:chunk + 8])
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{done} of {len(all_heads)} (batch, head) rows of the causal GQA workload, float64, "
                      f"{dt:.1f} s wall"}


def run_reference(args, rank, world):
    """The slow reference program: the CPU oracle, timed per step on a bounded sample."""
    import oracle
    oracle.load()
    w = si.CAUSAL_GQA_PREFILL
    q, k, v = si.qkv(w)
    group = w.nheads // w.nkvheads
    heads = [(b, h) for b in range(w.batch) for h in range(w.nheads)]
    per_step = max(1, args.reference_heads)
    for s in range(args.warmup):
        _oracle_heads(q, k, v, heads[:per_step], group)
    times, flops = [], 0.0
    for s in range(args.steps):
        sel = [heads[(s * per_step + j) % len(heads)] for j in range(per_step)]
        t0 = time.perf_counter()
        flops = _oracle_heads(q, k, v, sel, group)
        times.append(time.perf_counter() - t0)
    ms = float(np.mean(times)) * 1e3
    value = flops / (ms * 1e-3) / 1e12
    return {
        "impl": "reference",
        "metric": "prefill attention TFLOP/s (unmasked FLOPs)",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), numpy PCG64)",
        "config": {"workload": w.name, "batch": w.batch, "q_len": w.q_len, "kv_len": w.kv_len,
                   "nheads": w.nheads, "nkvheads": w.nkvheads, "head_dim": w.head_dim, "is_causal": True,
                   "step": f"{per_step} (batch, head) rows of the workload per step"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
                         "kind": "oracle", "sample": f"{per_step} (batch, head) rows per step, float64"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--reference-heads", type=int, default=16)
    ap.add_argument("--workloads", default="prefill,decode,bias,block_sparse,packed,backward,weights,rope,rope_prefill",
                    help="comma list; without 'prefill' only the other workloads run (a profiling aid)")
    ap.add_argument("--shrink", type=int, default=1,
                    help="divide the decode batch and the block-sparse length by this (small ncu cases)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    args.workloads = set(x.strip() for x in args.workloads.split(",") if x.strip())
    rank, world, local = init_dist(args.gpus)
    try:
        if "prefill" in args.workloads:
            res = run_ours(args, rank, world, local)
        else:
            torch.cuda.set_device(local)
            import head_scaled_dot_sdpa_b200 as sdpa
            res = {"other_workloads": other_workloads(args, torch.device("cuda", local), world,
                                                      sdpa.Workspace(torch.device("cuda", local)), _peaks())}
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
