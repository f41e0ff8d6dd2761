#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet token mixer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    (N > 1: launched by torchrun, one rank per GPU, NCCL for barrier/max only)

One step = one prefill call over the Qwen3.8 Gated DeltaNet layer workload
(B = 1, T = 4096, 16 q/k heads, 128 value heads, d = 128, bf16 activations,
FP32 state, final state returned): conv + SiLU, q/k L2 norm, gates, gated
delta rule and gated RMSNorm, i.e. the whole hot path.  Every rank runs its
own independent sequence (weak scaling; sequences never interact, so there
is no data-path collective).  `value` = tokens of all ranks / max-over-ranks
device time.  Decode (256 sequences x 1 token, resident FP32 states) is timed
the same way and reported in the "decode" object.

The JSON line also carries the roofline of the dominant kernel (its own
CUDA-event time per launch against the measured peaks), an end-to-end number
through the public API with host buffers, the sampled SM clocks, and the CPU
oracle's throughput on a bounded sample of the same workload.
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

METRIC = "GDN prefill tokens/s at Qwen3.8 layer shape"
UNIT = "tokens/s"
CHUNK = 64  # chunk size fixed for the algorithmic FLOP count
# nominal dense tensor-core ratio tf32 : bf16 on B200 (1.1 : 2.25 PFLOP/s); the
# chunked prefill's products run as kind::tf32, so its own peak is the measured
# bf16 peak times this ratio
TF32_PER_BF16 = 1.1 / 2.25


# ----------------------------------------------------------------- work model


def prefill_flops_per_token(Hk, Hv, d, C=CHUNK):
    """Algorithmic FLOPs per token of the chunked form at a fixed chunk C:
    per value head 2C(d_k + d_v) (W and U~ products) + 6 d_k d_v (three state
    products) + 2 C d_v (intra-chunk output) + C^2 / 3 (triangular solve), plus
    per q/k head 4 C d_k (K K^T and Q K^T)."""
    return Hv * (2 * C * (2 * d) + 6 * d * d + 2 * C * d + C * C / 3.0) + Hk * 4 * C * d


def prefill_bytes(Hk, Hv, d, N, B, act_bytes=2, read_state=False, write_state=True):
    """Minimum HBM bytes of a fully fused prefill: pre-conv q|k|v, z, a, b read,
    y written, plus the FP32 states read/written."""
    conv_dim = (2 * Hk + Hv) * d
    per_tok = act_bytes * (conv_dim + Hv * d + 2 * Hv + Hv * d)
    st = 4 * Hv * d * d * B
    return per_tok * N + st * (int(read_state) + int(write_state))


def decode_bytes(Hk, Hv, d, B, act_bytes=2, K=4):
    """HBM bytes of one decode call: state read + write, the token's q|k|v, z,
    a, b read, y written, conv cache read (K-1 rows) and written (K-1 rows)."""
    conv_dim = (2 * Hk + Hv) * d
    per_seq = 2 * 4 * Hv * d * d + act_bytes * (conv_dim + 2 * Hv * d + 2 * Hv) \
        + 2 * act_bytes * (K - 1) * conv_dim
    return per_seq * B


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def _sha(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()[:16]


def traffic_of(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None
    when no capture exists or the kernel's sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    ent = json.load(open(p)).get(kernel)
    if not ent:
        return None
    try:
        if _sha(ent["sources"]) != ent["sources_sha"]:
            return None
    except OSError:
        return None
    return ent["bytes_per_launch"]


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """nvidia-smi samples (every 20 ms) of SM clock and throttle reasons; stop()
    keeps the samples whose host timestamps fall inside the timed window."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.out = None
        try:
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={uuid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.5)  # let the sampler start before the work it should see
        except Exception:
            self.proc = None

    @staticmethod
    def _ts(s):
        import datetime
        try:
            return datetime.datetime.strptime(s.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self, t0=None, t1=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        rows = [[x.strip() for x in line.split(",")] for line in open(self.out.name)]
        rows = [r for r in rows if len(r) >= 9]
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        inside = rows
        if t0 is not None:
            inside = [r for r in rows if (self._ts(r[0]) or 0) >= t0 - 0.02 and
                      (self._ts(r[0]) or 0) <= t1 + 0.02]
            if not inside:  # window shorter than the sampling period: nearest sample
                inside = [min(rows, key=lambda r: abs((self._ts(r[0]) or 0) - (t0 + t1) / 2))]
        num = lambda v: float(v) if v.replace(".", "", 1).isdigit() else None
        sm = [num(r[1]) for r in inside if num(r[1]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in inside:
            for name, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(rows[0][2]),
                "reasons": sorted(reasons), "samples": len(inside)}


# -------------------------------------------------------------- CPU oracle


def oracle_throughput(wl, inp, budget_s=10.0, max_tokens=None):
    """Tokens/s of the FP64 oracle over all heads of the first T' tokens of the
    workload's first sequence, T' grown until about `budget_s` of CPU time."""
    import oracle
    shape = oracle.Shape(wl.num_qk_heads, wl.num_v_heads, wl.head_dim)
    P = [inp[k].cpu() for k in ("conv_w", "A_log", "dt_bias", "norm_w")]
    T_full = inp["seqlens"][0]
    cap = min(T_full, max_tokens or T_full)
    Tp = min(64, cap)
    while True:
        x = {k: inp[k][:Tp].cpu() for k in ("qkv", "a", "b", "z")}
        t0 = time.perf_counter()
        oracle.layer(shape, x["qkv"], x["a"], x["b"], x["z"], *P)
        dt = time.perf_counter() - t0
        if dt >= budget_s * 0.5 or Tp >= cap:
            break
        Tp = min(cap, max(Tp * 2, int(Tp * budget_s / max(dt, 1e-3))))
    threads = min(wl.num_v_heads, oracle.default_threads())
    return Tp / dt, {"tokens": Tp, "seconds": dt, "threads": threads}


# ----------------------------------------------------------------- our arm


# ------------------------------------------------------------------ ranks
# One process per GPU, replicas only: every rank runs its own seeded copy of
# the workload and the ranks meet only for a barrier and the max of the times.

def rank_seed(base, rank):
    """Seed of this rank's synthetic inputs (distinct per rank)."""
    return base + 7919 * rank


def reduce_max(dist, x, device):
    """Max of the float x over all ranks (x itself without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_step, world, steps, max_ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_step * world * steps / (max_ms / 1e3)


def run_ours(args, rank, world, dev, dist):
    import torch

    import linear_attention_layer_causal_b200 as gdn
    from linear_attention_layer_causal_b200 import workloads as W

    pk = peaks()
    wl = W.QWEN38_PREFILL
    if args.seq_len != 4096:
        import dataclasses
        wl = dataclasses.replace(wl, seqlens=(args.seq_len,))
    cfg = gdn.Config.of(wl, args.algo)
    inp = W.make_prefill(wl, dev, seed=rank_seed(wl.seed, rank))
    P = [inp[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")]
    N, B = sum(inp["seqlens"]), len(inp["seqlens"])
    y = torch.empty((N, cfg.num_v_heads, cfg.head_dim), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((B, cfg.num_v_heads, cfg.head_dim, cfg.head_dim), device=dev)
    ws = torch.empty(max(gdn.prefill_workspace_size(cfg, B, N), 1), dtype=torch.uint8, device=dev)

    def step():
        gdn.prefill(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"], *P,
                    y=y, final_state=fs, workspace=ws)

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(dist, x, dev)

    window = {}

    def timed(fn, K):
        ev = lambda: torch.cuda.Event(enable_timing=True)
        kb, ke = [ev() for _ in range(K)], [ev() for _ in range(K)]
        start, end = ev(), ev()
        barrier()
        torch.cuda.synchronize()
        window["t0"] = time.time()
        start.record()
        for i in range(K):
            gdn.profile_next_call(kb[i], ke[i])
            fn()
        end.record()
        torch.cuda.synchronize()
        window["t1"] = time.time()
        barrier()
        total = start.elapsed_time(end)
        kern = [kb[i].elapsed_time(ke[i]) for i in range(K)]
        return total, sum(kern) / K

    if args.only == "decode":
        return run_decode(args, rank, world, dev, pk, timed, max_over_ranks)
    if args.only == "kda":
        return run_kda(args, rank, world, dev, pk, timed, max_over_ranks)
    clocks = ClockSampler(dev.index)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    total_ms, kern_ms = timed(step, args.steps)
    clk = clocks.stop(window["t0"], window["t1"])
    total_ms = max_over_ranks(total_ms)
    kern_ms_max = max_over_ranks(kern_ms)
    ms_per_step = total_ms / args.steps
    value = job_rate(N, world, args.steps, total_ms)

    flops = prefill_flops_per_token(cfg.num_qk_heads, cfg.num_v_heads, cfg.head_dim) * N
    byts = prefill_bytes(cfg.num_qk_heads, cfg.num_v_heads, cfg.head_dim, N, B)
    tf = flops / (kern_ms_max / 1e3) / 1e12
    gbs = byts / (kern_ms_max / 1e3) / 1e9
    kname = "chunk_prefill_kernel" if cfg.head_dim == 128 and cfg.algo != "serial" \
        else "recurrent_prefill_kernel"
    tf32_peak = round(pk["bf16_tflops"] * TF32_PER_BF16, 1)
    roof = {"kernel": kname, "bound": "tensor", "achieved": round(tf, 2),
            "peak": tf32_peak, "unit": "TFLOP/s", "frac": round(tf / tf32_peak, 4),
            "traffic": traffic_of(kname),
            "algorithmic_flops": flops, "kernel_ms": round(kern_ms_max, 4),
            "peak_source": pk["source"] + " burst bf16 x nominal tf32/bf16 ratio 1.1/2.25",
            "bf16_view": {"peak": pk["bf16_tflops"], "frac": round(tf / pk["bf16_tflops"], 4)},
            "hbm_view": {"achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / pk["hbm_gbs"], 4), "algorithmic_bytes": byts}}

    if args.only == "prefill":
        return {"metric": METRIC, "value": value, "unit": UNIT, "ms_per_step": ms_per_step,
                "roofline": roof, "clocks": clk}
    decode = run_decode(args, rank, world, dev, pk, timed, max_over_ranks)
    decode_k = run_decode_k(args, rank, world, dev, pk, timed, max_over_ranks)
    qwen35 = run_prefill_shape(args, rank, world, dev, pk, timed, max_over_ranks, "qwen35_prefill")
    long_ctx = run_long_context(args, rank, world, dev, pk, timed, max_over_ranks)
    kda = run_kda(args, rank, world, dev, pk, timed, max_over_ranks)

    # ---- end to end through the public API from pinned host buffers.  Every
    # step uploads its inputs, runs the layer and reads back y and the final
    # state; as a serving loop would, the steps are pipelined over three
    # streams with two device buffer sets, so that the upload of step i + 1
    # and the download of step i - 1 overlap the compute of step i.
    host = {k: inp[k].cpu().pin_memory() for k in ("qkv", "a", "b", "z")}
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    fs_host = [torch.empty(fs.shape, dtype=fs.dtype).pin_memory() for _ in range(2)]
    dev_in = [{k: torch.empty_like(inp[k]) for k in host} for _ in range(2)]
    dev_y = [y, torch.empty_like(y)]
    dev_fs = [fs, torch.empty_like(fs)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = y_host[0].numel() * y_host[0].element_size() + fs_host[0].numel() * fs_host[0].element_size()
    up, comp, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    step_no = [0]

    def e2e_step():
        i = step_no[0]
        b = i & 1
        step_no[0] += 1
        if i >= 2:
            up.wait_event(ev_comp[b])    # step i - 2 has read this input set
        with torch.cuda.stream(up):
            for k in host:
                dev_in[b][k].copy_(host[k], non_blocking=True)
        ev_in[b].record(up)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])   # step i - 2's outputs are downloaded
        d = dev_in[b]
        gdn.prefill(cfg, d["qkv"], d["a"], d["b"], d["z"], inp["cu_seqlens"], *P,
                    y=dev_y[b], final_state=dev_fs[b], workspace=ws, stream=comp)
        ev_comp[b].record(comp)
        down.wait_event(ev_comp[b])
        with torch.cuda.stream(down):
            y_host[b].copy_(dev_y[b], non_blocking=True)
            fs_host[b].copy_(dev_fs[b], non_blocking=True)
        ev_out[b].record(down)
        torch.cuda.current_stream().wait_event(ev_out[b])  # the timing events cover it

    for _ in range(args.warmup):
        e2e_step()
    etot, _ = timed(e2e_step, args.steps)
    etot = max_over_ranks(etot)
    e2e = {"value": job_rate(N, world, args.steps, etot), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "tf32", "data": "synthetic",
            "config": {"workload": "qwen38_prefill: Qwen3.8 GDN layer prefill, B=1 per GPU, "
                                   "T=4096, 16 q/k heads, 128 value heads, d=128, FP32 state",
                       "global_batch": world, "seq_len": N, "parallelism": f"replicas x{world}",
                       "arith": "bf16 activations in/out, tf32 tensor-core products with FP32 "
                                "accumulation, FP32 state and CUDA-core math",
                       "l2": "no flush: inputs of one step (~447 MB) exceed the 126 MB L2"},
            "roofline": roof, "decode": decode, "decode_k": decode_k, "qwen35_prefill": qwen35,
            "long_context": long_ctx, "kda": kda,
            "e2e": e2e,
            # chunked (16-bit activations): offsets, conv of q|k, Gram, inverses, chunk kernel
            "gpu_launches": (5 if kname == "chunk_prefill_kernel" else 2) * args.steps,
            "clocks": clk}
    return line


def decode_k_bytes(Hk, Hv, d, B, k, act_bytes=2, K=4, read_state=True, write_state=True, y=True):
    """HBM bytes of one multi-token call: the state read and/or written once for all
    k tokens, k tokens' q|k|v, a, b (and z, y when outputs are formed) and the conv
    cache (read, and written when the state is)."""
    conv_dim = (2 * Hk + Hv) * d
    st = 4 * Hv * d * d * (int(read_state) + int(write_state))
    tok = act_bytes * k * (conv_dim + 2 * Hv + (2 * Hv * d if y else 0))
    cache = act_bytes * (K - 1) * conv_dim * (1 + int(write_state))
    return (st + tok + cache) * B


def run_decode_k(args, rank, world, dev, pk, timed, max_over_ranks):
    """Multi-token decode at the Qwen3.8 shape: k = 2 tokens per sequence (the one
    draft of the MTP layer and the token after it) against resident states: plain
    multi-token decode (state updated by both), and the speculative pair -- verify
    (outputs of both, state read only) then commit (state advanced by the accepted
    tokens, here all of them)."""
    import torch

    import linear_attention_layer_causal_b200 as gdn
    from linear_attention_layer_causal_b200 import workloads as W
    dwl = W.QWEN38_DECODE
    cfg = gdn.Config.of(dwl)
    B, k = args.decode_batch, 2
    d = W.make_decode(dwl, dev, batch=B, seed=rank_seed(dwl.seed, rank) + 1, tokens=k)
    P = [d[x] for x in ("conv_w", "A_log", "dt_bias", "norm_w")]
    y = torch.empty((B, k, cfg.num_v_heads, cfg.head_dim), dtype=torch.bfloat16, device=dev)
    acc = torch.full((B,), k, dtype=torch.int32, device=dev)
    out = {"metric": "GDN multi-token decode tokens/s at Qwen3.8 layer shape", "unit": "tokens/s",
           "config": {"workload": dwl.name, "batch": B, "tokens_per_sequence": k}}
    Hk, Hv, D = cfg.num_qk_heads, cfg.num_v_heads, cfg.head_dim

    def multi():
        gdn.decode_multi(cfg, d["qkv"], d["a"], d["b"], d["z"], d["state"], d["conv_cache"], *P, y=y)

    def verify():
        gdn.decode_verify(cfg, d["qkv"], d["a"], d["b"], d["z"], d["state"], d["conv_cache"], *P, y=y)

    def commit():
        gdn.decode_commit(cfg, d["qkv"], d["a"], d["b"], d["state"], d["conv_cache"], acc, *P)

    for name, fn, nbytes in [
            ("multi", multi, decode_k_bytes(Hk, Hv, D, B, k)),
            ("verify", verify, decode_k_bytes(Hk, Hv, D, B, k, write_state=False)),
            ("commit", commit, decode_k_bytes(Hk, Hv, D, B, k, y=False))]:
        for _ in range(args.warmup):
            fn()
        tot, kern = timed(fn, args.steps)
        tot, kern = max_over_ranks(tot), max_over_ranks(kern)
        gbs = nbytes / (kern / 1e3) / 1e9
        out[name] = {"value": job_rate(B * k, world, args.steps, tot), "ms_per_step": tot / args.steps,
                     "roofline": {"kernel": "decode_multi_kernel", "bound": "hbm",
                                  "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": round(gbs / pk["hbm_gbs"], 4), "algorithmic_bytes": nbytes,
                                  "kernel_ms": round(kern, 4), "peak_source": pk["source"] + " copy"}}
    # a speculative step of k tokens: verify + commit
    out["value"] = job_rate(B * k, world, 1, out["verify"]["ms_per_step"] + out["commit"]["ms_per_step"])
    return out


def run_prefill_shape(args, rank, world, dev, pk, timed, max_over_ranks, name):
    """Prefill at another layer shape of the family (tokens/s and the chunk kernel's
    tensor roofline), e.g. the Qwen3.5-397B-A17B layer: 16 q/k heads, 64 value heads."""
    import torch

    import linear_attention_layer_causal_b200 as gdn
    from linear_attention_layer_causal_b200 import workloads as W
    wl = W.WORKLOADS[name]
    cfg = gdn.Config.of(wl)
    inp = W.make_prefill(wl, dev, seed=rank_seed(wl.seed, rank))
    P = [inp[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")]
    N, B = sum(inp["seqlens"]), len(inp["seqlens"])
    y = torch.empty((N, cfg.num_v_heads, cfg.head_dim), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((B, cfg.num_v_heads, cfg.head_dim, cfg.head_dim), device=dev)
    ws = torch.empty(max(gdn.prefill_workspace_size(cfg, B, N), 1), dtype=torch.uint8, device=dev)

    def step():
        gdn.prefill(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"], *P, y=y,
                    final_state=fs, initial_state=inp["initial_state"], workspace=ws)

    for _ in range(args.warmup):
        step()
    tot, kern = timed(step, args.steps)
    tot, kern = max_over_ranks(tot), max_over_ranks(kern)
    flops = prefill_flops_per_token(cfg.num_qk_heads, cfg.num_v_heads, cfg.head_dim) * N
    tf32_peak = round(pk["bf16_tflops"] * TF32_PER_BF16, 1)
    tf = flops / (kern / 1e3) / 1e12
    return {"metric": f"GDN prefill tokens/s, {wl.notes}", "unit": "tokens/s",
            "value": job_rate(N, world, args.steps, tot), "ms_per_step": tot / args.steps,
            "config": {"workload": name, "batch": B, "seq_len": N // B, "num_qk_heads": cfg.num_qk_heads,
                       "num_v_heads": cfg.num_v_heads},
            "roofline": {"kernel": "chunk_prefill_kernel", "bound": "tensor", "achieved": round(tf, 2),
                         "peak": tf32_peak, "unit": "TFLOP/s", "frac": round(tf / tf32_peak, 4),
                         "kernel_ms": round(kern, 4)}}


def run_long_context(args, rank, world, dev, pk, timed, max_over_ranks):
    """One 262,144-token sequence (the Qwen3.8 context window) at the Qwen3.8 and the
    Qwen3.5-397B layer shapes: tokens/s with the library's choice of segments per
    sequence and, where that choice splits the sequence, the single chain beside it."""
    import torch

    import linear_attention_layer_causal_b200 as gdn
    from linear_attention_layer_causal_b200 import workloads as W
    out = {}
    for name in ("qwen38_262k_prefill", "qwen35_262k_prefill"):
        wl = W.WORKLOADS[name]
        inp = W.make_prefill(wl, dev, seed=rank_seed(wl.seed, rank))
        P = [inp[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")]
        N, B = sum(inp["seqlens"]), len(inp["seqlens"])
        y = torch.empty((N, wl.num_v_heads, wl.head_dim), dtype=torch.bfloat16, device=dev)
        fs = torch.empty((B, wl.num_v_heads, wl.head_dim, wl.head_dim), device=dev)
        res = {"config": {"workload": name, "batch": B, "seq_len": N // B,
                          "num_qk_heads": wl.num_qk_heads, "num_v_heads": wl.num_v_heads}}
        for label, segs in (("auto", 0), ("single_chain", 1)):
            cfg = gdn.Config.of(wl, segments=segs)
            nseg = gdn.prefill_segments(cfg, B, N)
            if label == "single_chain" and res["auto"]["segments"] == 1:
                break
            ws = torch.empty(max(gdn.prefill_workspace_size(cfg, B, N), 1), dtype=torch.uint8,
                             device=dev)

            def step():
                gdn.prefill(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"], *P,
                            y=y, final_state=fs, workspace=ws)

            for _ in range(args.warmup):
                step()
            tot, kern = timed(step, args.steps)
            tot, kern = max_over_ranks(tot), max_over_ranks(kern)
            res[label] = {"segments": nseg, "value": job_rate(N, world, args.steps, tot),
                          "unit": "tokens/s", "ms_per_step": tot / args.steps,
                          "scan_ms": round(kern, 4)}
            del ws
        out[name] = res
        del inp, y, fs
        torch.cuda.empty_cache()
    return out


def kda_decode_bytes(H, d, B, act_bytes=2, K=4):
    """HBM bytes of one KDA decode call: state read + write, the token's q|k|v,
    zdec, gate and b read, y written, conv cache read and written (K-1 rows)."""
    conv_dim = 3 * H * d
    per_seq = 2 * 4 * H * d * d + act_bytes * (conv_dim + 3 * H * d + H) + 2 * act_bytes * (K - 1) * conv_dim
    return per_seq * B


# FP32 FMA peak of the CUDA cores (148 SMs x 128 FMA lanes x 2 FLOP x 1.965 GHz),
# the bound of the token-serial recurrences
FP32_CUDA_CORE_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_kda(args, rank, world, dev, pk, timed, max_over_ranks):
    """Kimi Delta Attention at the Kimi K3 layer shape (96 heads of dim 128): a
    prefill of one 4,096-token sequence (token-serial FP32 recurrence on the CUDA
    cores) and a decode of 256 sequences (state streamed through registers)."""
    import torch

    import linear_attention_layer_causal_b200 as gdn
    from linear_attention_layer_causal_b200 import workloads as W
    wl = W.KIMI_K3_KDA
    cfg = gdn.Config.of(wl)
    H, D = wl.num_v_heads, wl.head_dim
    N = args.seq_len
    inp = W.make_kda_prefill(wl, dev, seqlens=(N,), seed=rank_seed(wl.seed, rank))
    P = [inp[k] for k in ("conv_w", "A_log", "norm_w")]
    y = torch.empty((N, H, D), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, H, D, D), device=dev)
    ws = torch.empty(max(gdn.kda_prefill_workspace_size(cfg, 1, N), 1), dtype=torch.uint8, device=dev)

    def pstep():
        gdn.kda_prefill(cfg, inp["qkv"], inp["zdec"], inp["b"], inp["gate"], inp["cu_seqlens"], *P,
                        y=y, final_state=fs, workspace=ws)

    for _ in range(args.warmup):
        pstep()
    tot, kern = timed(pstep, args.steps)
    tot, kern = max_over_ranks(tot), max_over_ranks(kern)
    # per token and head: decay, k-projection, rank-1 update and q-projection of
    # the d x d state, one FMA (2 FLOP) each per element
    flops = 4 * 2 * H * D * D * N
    tf = flops / (kern / 1e3) / 1e12
    out = {"metric": "KDA prefill tokens/s and decode tokens/s, Kimi K3 layer shape", "unit": "tokens/s",
           "config": {"workload": wl.name, "num_heads": H, "head_dim": D},
           "prefill": {"value": job_rate(N, world, args.steps, tot), "ms_per_step": tot / args.steps,
                       "batch": 1, "seq_len": N,
                       "roofline": {"kernel": "kda_prefill_kernel", "bound": "alu", "achieved": round(tf, 2),
                                    "peak": round(FP32_CUDA_CORE_TFLOPS, 1), "unit": "TFLOP/s",
                                    "frac": round(tf / FP32_CUDA_CORE_TFLOPS, 4), "kernel_ms": round(kern, 4),
                                    "peak_source": "FP32 FMA lanes x clock (148 x 128 x 2 x 1.965 GHz)"}}}
    del inp, y, fs, ws
    B = args.decode_batch
    d = W.make_kda_decode(wl, dev, batch=B, seed=rank_seed(wl.seed, rank) + 1)
    Pd = [d[k] for k in ("conv_w", "A_log", "norm_w")]
    yd = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)

    def dstep():
        gdn.kda_decode(cfg, d["qkv"], d["zdec"], d["b"], d["gate"], d["state"], d["conv_cache"], *Pd, y=yd)

    for _ in range(args.warmup):
        dstep()
    tot, _ = timed(dstep, args.steps)
    tot = max_over_ranks(tot)
    ms = tot / args.steps
    nbytes = kda_decode_bytes(H, D, B)
    gbs = nbytes / (ms / 1e3) / 1e9
    out["decode"] = {"value": job_rate(B, world, args.steps, tot), "ms_per_step": ms, "batch": B,
                     "roofline": {"kernel": "kda_decode_kernel", "bound": "hbm", "achieved": round(gbs, 1),
                                  "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                                  "algorithmic_bytes": nbytes}}
    return out


def run_decode(args, rank, world, dev, pk, timed, max_over_ranks):
    """Decode: B sequences x 1 token against resident FP32 states (in place)."""
    import torch

    import linear_attention_layer_causal_b200 as gdn
    from linear_attention_layer_causal_b200 import workloads as W
    dwl = W.QWEN38_DECODE
    dcfg = gdn.Config.of(dwl)
    dB = args.decode_batch
    d = W.make_decode(dwl, dev, batch=dB, seed=rank_seed(dwl.seed, rank))
    DP = [d[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")]
    dy = torch.empty((dB, dcfg.num_v_heads, dcfg.head_dim), dtype=torch.bfloat16, device=dev)

    def dstep():
        gdn.decode(dcfg, d["qkv"], d["a"], d["b"], d["z"], d["state"], d["conv_cache"], *DP, y=dy)

    for _ in range(args.warmup):
        dstep()
    dtot, dkern = timed(dstep, args.steps)
    dtot, dkern = max_over_ranks(dtot), max_over_ranks(dkern)
    dbytes = decode_bytes(dcfg.num_qk_heads, dcfg.num_v_heads, dcfg.head_dim, dB)
    dgbs = dbytes / (dkern / 1e3) / 1e9
    return {"metric": "GDN decode tokens/s at Qwen3.8 layer shape", "unit": "tokens/s",
            "value": job_rate(dB, world, args.steps, dtot), "ms_per_step": dtot / args.steps,
            "config": {"workload": dwl.name, "batch": dB, "state_gib": 4 * dB * 128 ** 3 / 2 ** 30},
            "roofline": {"kernel": "decode_kernel", "bound": "hbm", "achieved": round(dgbs, 1),
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(dgbs / pk["hbm_gbs"], 4),
                         "traffic": traffic_of("decode_kernel"), "algorithmic_bytes": dbytes,
                         "kernel_ms": round(dkern, 4), "peak_source": pk["source"] + " copy"}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default="all", choices=["all", "prefill", "decode", "kda"],
                    help="run only one part (for profiling small cases)")
    ap.add_argument("--decode-batch", type=int, default=256)
    ap.add_argument("--seq-len", type=int, default=4096,
                    help="with --only prefill or kda: the prefill sequence length (profiling cases)")
    ap.add_argument("--algo", default="auto", choices=["auto", "chunked", "serial"],
                    help="prefill algorithm (auto = tensor-core chunks at head dim 128)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.seq_len != 4096 and args.only not in ("prefill", "kda"):
        ap.error("--seq-len applies to --only prefill or kda")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import datetime

    import torch
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    line = run_ours(args, rank, world, dev, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.only == "all":
        from linear_attention_layer_causal_b200 import workloads as W
        inp = W.make_prefill(W.QWEN38_PREFILL, "cpu")
        v, info = oracle_throughput(W.QWEN38_PREFILL, inp)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": info["threads"],
                                "kind": "oracle",
                                "sample": f"FP64 C oracle, all 128 value heads of the first "
                                          f"{info['tokens']} of 4096 tokens, "
                                          f"{info['seconds']:.1f} s"}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: rank 0 only, each step a bounded
    token sample of the same workload."""
    if rank != 0:
        return
    from linear_attention_layer_causal_b200 import workloads as W
    wl = W.QWEN38_PREFILL
    inp = W.make_prefill(wl, "cpu")
    # calibrate the sample so that one step takes about 3 s
    _, info = oracle_throughput(wl, inp, budget_s=3.0)
    Tp = info["tokens"]
    import oracle
    shape = oracle.Shape(wl.num_qk_heads, wl.num_v_heads, wl.head_dim)
    P = [inp[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")]
    x = {k: inp[k][:Tp] for k in ("qkv", "a", "b", "z")}
    run = lambda: oracle.layer(shape, x["qkv"], x["a"], x["b"], x["z"], *P)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = Tp * args.steps / dt
    sample = f"FP64 C oracle, all 128 value heads of the first {Tp} of 4096 tokens per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "qwen38_prefill: Qwen3.8 GDN layer prefill, B=1, T=4096",
                       "global_batch": 1, "seq_len": 4096, "parallelism": "cpu threads"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": info["threads"],
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
