#!/usr/bin/env python3
"""Benchmark: NSNQuant KV-cache encode + quantized decode attention on B200.

One step = the hot path over one batch of the Llama-3-8B layer workload
(8 sequences x 8 kv-heads x 4096 prompt tokens, head_dim 128, bf16, 2 bits
per coordinate): encode K, encode V (normalize-shift-normalize, Hadamard,
nearest-codeword VQ), then one decode-attention query per sequence over the
fresh quantized cache (32 query heads, GQA 4:1). `value` is KV tokens encoded
per second over the whole step, all ranks together (weak scaling: every rank
runs its own batch; no collective on the data path).

The same run also times decode attention alone at the 32k-context workload
(16 x 32 query heads / 8 kv-heads x 32768 tokens, 2 bit) and reports its HBM
GB/s under "attention".

  python bench.py [--gpus N --steps K --warmup W]          # CUDA path
  python bench.py --impl reference ...                     # the CPU oracle
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

import nsnq_synth as S  # noqa: E402

GOLDEN = os.path.join(ROOT, "tests", "golden")
METRIC = "KV tokens/s encoded and quantized decode-attn HBM GB/s (fraction of peak), 1 B200"
STEP_WORKLOAD = "encode-8x4096"
ATTN_WORKLOAD = "decode-16x32k-2b"
STEP_HQ = 32
L2_FLUSH_BYTES = 256 << 20


def load_codebook(g: int) -> np.ndarray:
    return np.fromfile(os.path.join(GOLDEN, f"codebook_g{g}.f32"), dtype="<f4").reshape(256, g)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


NOMINAL_HBM_GBS = 8000.0  # nominal B200 HBM3e bandwidth (8 TB/s), for the second fraction
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "roofline_traffic.json")


def measured_traffic(call: str):
    """DRAM bytes per launch of `call` from the committed ncu record, or None
    when the kernel sources changed since the capture (hash mismatch)."""
    import hashlib
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)[call]
        h = hashlib.sha256()
        for name in rec["sources"]:
            with open(os.path.join(ROOT, "attention_decode_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        return int(rec["bytes_per_launch"]) if h.hexdigest() == rec["source_sha256"] else None
    except (OSError, KeyError, ValueError):
        return None


def encode_bytes_per_token_head(sub: int, in_bytes: int = 2) -> int:
    """Algorithmic bytes of encode per token-head: input row, codes, (s1, s2)."""
    return 128 * in_bytes + 128 // sub + 8


def attn_bytes_per_token(ksub: int, vsub: int) -> int:
    """Algorithmic bytes of attention per (batch, kv-head, token): K and V codes plus scales."""
    return 128 // ksub + 128 // vsub + 16


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every ~2 ms (nvidia-smi
    polling as a fallback) while the timed regions run."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        import threading
        self.gpu = gpu_index
        self.rows = []  # (sm_mhz, max_mhz, set(reasons))
        self.stop = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        try:
            import pynvml as N
            N.nvmlInit()
            hdl = N.nvmlDeviceGetHandleByIndex(self.gpu)
            bits = {"hw_slowdown": N.nvmlClocksThrottleReasonHwSlowdown,
                    "hw_thermal_slowdown": N.nvmlClocksThrottleReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": N.nvmlClocksThrottleReasonSwThermalSlowdown,
                    "sw_power_cap": N.nvmlClocksThrottleReasonSwPowerCap}
            mx = N.nvmlDeviceGetMaxClockInfo(hdl, N.NVML_CLOCK_SM)
            while not self.stop.is_set():
                sm = N.nvmlDeviceGetClockInfo(hdl, N.NVML_CLOCK_SM)
                r = N.nvmlDeviceGetCurrentClocksThrottleReasons(hdl)
                self.rows.append((float(sm), float(mx), {k for k, v in bits.items() if r & v}))
                self.stop.wait(0.002)
            return
        except Exception:
            pass
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        while not self.stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={fields}",
                                      "--format=csv,noheader,nounits"], capture_output=True,
                                     text=True, timeout=5).stdout.strip()
                p = [x.strip() for x in out.split(",")]
                self.rows.append((float(p[0]), float(p[1]),
                                  {n for n, v in zip(self.NAMES, p[2:6]) if v.lower() == "active"}))
            except Exception:
                return
            self.stop.wait(0.1)

    def __enter__(self):
        self.thread.start()
        return self

    def __exit__(self, *exc):
        self.stop.set()
        self.thread.join(timeout=10)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        reasons = set()
        for r in self.rows:
            reasons |= r[2]
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.rows[-1][1],
                "reasons": sorted(reasons), "samples": len(self.rows)}


# ------------------------------------------------------------- reduction --
def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest value over all ranks (timings are reported as the max)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------- CUDA arm --
def run_cuda(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    from attention_decode_b200 import build as nbuild
    nbuild.build()
    import attention_decode_b200 as nsnq

    dev = torch.device("cuda", local)
    w = S.WORKLOADS[STEP_WORKLOAD]
    B, H, T, Hq = w.B, w.Hkv, w.T, STEP_HQ
    cb = nsnq.Codebook(torch.from_numpy(load_codebook(w.sub_dim)).to(dev))
    # Inputs: seeded synthetic K/V of the workload (ranks draw disjoint sequences).
    kx = S.to_io(S.keys(w), "bf16")
    vx = S.to_io(S.values(w), "bf16")
    qx = S.to_io(S.queries(S.Workload(**{**w.__dict__, "Hq": Hq}), step=rank), "bf16")
    host = {n: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
            for n, a in (("k", kx), ("v", vx), ("q", qx))}
    k = host["k"].to(dev)
    v = host["v"].to(dev)
    q = host["q"].to(dev)
    kc = nsnq.Cache.empty(B, H, T, w.sub_dim, device=dev)
    vc = nsnq.Cache.empty(B, H, T, w.sub_dim, device=dev)
    ws_e = torch.empty(nsnq.nsnq_encode_kv_workspace(B, H, T), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(max(256, nsnq.nsnq_attn_workspace(B, Hq, H, T)), dtype=torch.uint8, device=dev)
    seq = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(kin, vin, qin):
        nsnq.nsnq_encode_kv(kin, vin, cb, kc, vc, workspace=ws_e)
        nsnq.nsnq_attn_decode(qin, kc, vc, cb, cb, seq, T, Hkv=H, out=out, workspace=ws_a)

    LAUNCHES_PER_STEP = 2 + 2  # encode of K and V (pass 1, pass 2) + attention (split, combine)

    def barrier():
        if world > 1:
            dist.barrier()

    clk = ClockSampler(local).__enter__()
    time.sleep(0.3)
    for _ in range(args.warmup):
        step(k, v, q)
    torch.cuda.synchronize()

    # ---- timed device-resident steps (L2 flushed before each step) ----
    # (no event between the two calls: the attention kernel is a programmatic
    # dependent of the encode's last kernel and may start during its tail,
    # which a stream operation between them would prevent)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    if True:
        for i in range(args.steps):
            flush.zero_()
            e = ev[i]
            e[0].record(stream)
            nsnq.nsnq_encode_kv(k, v, cb, kc, vc, workspace=ws_e)
            nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, seq, T, Hkv=H, out=out, workspace=ws_a)
            e[1].record(stream)
        torch.cuda.synchronize()
    barrier()
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]

    # ---- the step's two calls timed apart (same steps again, an event
    #      between the calls): the encode roofline and the stage split ----
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e = ev[i]
        e[0].record(stream)
        nsnq.nsnq_encode_kv(k, v, cb, kc, vc, workspace=ws_e)
        e[1].record(stream)
        nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, seq, T, Hkv=H, out=out, workspace=ws_a)
        e[2].record(stream)
    torch.cuda.synchronize()
    barrier()
    enc_ms = [e[0].elapsed_time(e[1]) for e in ev]
    att_small_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * T * world
    value = tokens_per_step / (ms_per_step / 1e3)

    # ---- end to end: pinned host K/V/q in, the step's result (the attention
    #      output) out, through the public API; the quantized cache is device
    #      state and stays on the GPU. The batch goes over in two pieces on a
    #      copy stream (all but an eighth of the sequences, then the rest), and
    #      each piece is encoded and attended as soon as it has arrived (the
    #      shift and the attention are per sequence), so the host link and the
    #      kernels overlap and only the small last piece's work follows the
    #      last copy. Measured (8 sequences): 7 + 1 12.8 M KV tokens/s, 6 + 2
    #      12.4-12.6 M, 4 + 4 12.2 M; three or four pieces 11.0-11.6 M ----
    res_host = torch.empty(B, Hq, 128, dtype=torch.bfloat16).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    copy_stream = torch.cuda.Stream(device=dev)
    cut1 = B - max(1, B // 8) if B > 1 else B
    halves = [(0, cut1), (cut1, B)] if B > 1 else [(0, B)]
    arrived = [torch.cuda.Event() for _ in halves]
    cut = lambda c, b0, b1: nsnq.Cache(c.codes[b0:b1], c.scales[b0:b1], c.shift[b0:b1])
    parts = [(b0, b1, cut(kc, b0, b1), cut(vc, b0, b1)) for b0, b1 in halves]
    # (a smaller piece can need more workspace: more pass-1 chunks per head)
    ws_h = torch.empty(max(nsnq.nsnq_encode_kv_workspace(b1 - b0, H, T) for b0, b1 in halves),
                       dtype=torch.uint8, device=dev)

    def e2e_step():
        copy_stream.wait_stream(stream)
        with torch.cuda.stream(copy_stream):
            for (b0, b1, _, _), ev_ in zip(parts, arrived):
                k[b0:b1].copy_(host["k"][b0:b1], non_blocking=True)
                v[b0:b1].copy_(host["v"][b0:b1], non_blocking=True)
                ev_.record(copy_stream)
        q.copy_(host["q"], non_blocking=True)
        # each piece: encode, then attention over its own sequences, then its
        # rows of the result back to the host
        for (b0, b1, kh, vh), ev_ in zip(parts, arrived):
            stream.wait_event(ev_)
            nsnq.nsnq_encode_kv(k[b0:b1], v[b0:b1], cb, kh, vh, workspace=ws_h)
            nsnq.nsnq_attn_decode(q[b0:b1], kh, vh, cb, cb, seq[b0:b1], T, Hkv=H, out=out[b0:b1],
                                  workspace=ws_a)
            res_host[b0:b1].copy_(out[b0:b1], non_blocking=True)

    for _ in range(2):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    e2e_ms = 0.0
    for i in range(args.steps):
        flush.zero_()
        e0.record(stream)
        e2e_step()
        e1.record(stream)
        e1.synchronize()
        e2e_ms += e0.elapsed_time(e1)
    barrier()
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("k", "v", "q"))
    d2h = res_host.numel() * res_host.element_size()
    e2e = {"value": tokens_per_step / (e2e_ms / args.steps / 1e3), "unit": "KV tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "overlap": "K/V host copies in two pieces (7/8 and 1/8 of the sequences) on a copy stream; each piece encoded and attended on arrival"}

    # ---- roofline of the dominant call (encode), algorithmic bytes ----
    hbm, peak_kind = peaks()
    enc_bytes = 2 * B * H * T * encode_bytes_per_token_head(w.sub_dim)  # K and V
    enc_avg_ms = sum(enc_ms) / len(enc_ms)
    enc_gbs = enc_bytes / (enc_avg_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(enc_gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(enc_gbs / hbm, 4), "frac_vs_8tbs": round(enc_gbs / NOMINAL_HBM_GBS, 4), "peak_kind": peak_kind,
                "kernel": "nsnq_encode_kv (nsn_stats + nsn_encode_pruned over K and V, one call)",
                "algorithmic_bytes_per_launch": enc_bytes,
                "traffic": args.traffic if args.traffic is not None else measured_traffic("nsnq_encode_kv")}

    # ---- decode attention alone at the 32k workload ----
    attention = run_attention_bench(args, nsnq, dev, world, barrier, hbm, peak_kind)
    attention_variants = run_attention_variants(args, nsnq, dev, world, barrier, hbm)
    encode_1bit = run_encode1_bench(args, nsnq, dev, world, barrier, hbm, peak_kind, k)
    encode_tc_search = run_encode1_bench(args, nsnq, dev, world, barrier, hbm, peak_kind, k, sub=4)
    long_context = run_long_context_bench(args, nsnq, dev, world, barrier, hbm)
    serving = run_serving_bench(args, nsnq, dev, world, barrier, hbm)
    clk.__exit__(None, None, None)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "KV tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded K with outlier channels x LogNormal token scale, V ~ N(0,1))",
        "config": {"workload": "encode-8x4096 + decode (Llama-3-8B layer: B 8, Hkv 8, Hq 32, "
                               "T 4096, d 128, 2 bit/coord)",
                   "global_batch": B * world, "seq_len": T, "parallelism": f"replicas x{world}",
                   "l2": "flushed (256 MB write) before every timed step"},
        "stages_ms": {"encode_kv": round(enc_avg_ms, 4),
                      "attention_4k": round(sum(att_small_ms) / len(att_small_ms), 4)},
        "stages_timing": "the step's calls timed apart in a second loop over the same steps "
                         "(an event between them); value is timed without it",
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "roofline": roofline, "attention": attention, "attention_variants": attention_variants,
        "encode_1bit": encode_1bit, "encode_2bit_tc_search": encode_tc_search,
        "long_context": long_context, "serving": serving, "e2e": e2e,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_attention_bench(args, nsnq, dev, world, barrier, hbm, peak_kind):
    """Decode attention over a 32k-token 2-bit cache built by encoding seeded
    K/V of the workload's distribution (generated on the device)."""
    import torch
    import torch.distributed as dist
    w = S.WORKLOADS[ATTN_WORKLOAD]
    B, H, Hq, T = w.B, w.Hkv, w.Hq, w.T
    cb = nsnq.Codebook(torch.from_numpy(load_codebook(w.sub_dim)).to(dev))
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    kc = nsnq.Cache.empty(B, H, T, w.sub_dim, device=dev)
    vc = nsnq.Cache.empty(B, H, T, w.sub_dim, device=dev)
    chans, signs = w.kdist.channels(128)
    bias = torch.zeros(128, device=dev)
    bias[chans] = torch.tensor(signs, device=dev) * w.kdist.bias
    for b in range(B):  # one sequence at a time keeps the bf16 staging at 8 MB x 8
        z = torch.randn(1, H, T, 128, generator=gen, device=dev)
        s = torch.exp(w.kdist.sigma * torch.randn(1, H, T, 1, generator=gen, device=dev))
        x = ((z + bias) * s).to(torch.bfloat16)
        sub = nsnq.Cache(kc.codes[b:b + 1], kc.scales[b:b + 1], kc.shift[b:b + 1])
        nsnq.nsnq_encode(x, cb, sub)
        x = torch.randn(1, H, T, 128, generator=gen, device=dev).to(torch.bfloat16)
        sub = nsnq.Cache(vc.codes[b:b + 1], vc.scales[b:b + 1], vc.shift[b:b + 1])
        nsnq.nsnq_encode(x, cb, sub)
    q = torch.randn(B, Hq, 128, generator=gen, device=dev).to(torch.bfloat16)
    seq = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(nsnq.nsnq_attn_workspace(B, Hq, H, T), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, seq, T, Hkv=H, out=out, workspace=ws)
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, seq, T, Hkv=H, out=out, workspace=ws)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = [a.elapsed_time(b) for a, b in evs]
    avg = max_over_ranks(sum(ms) / len(ms), world, dev)
    nbytes = B * H * T * attn_bytes_per_token(w.sub_dim, w.sub_dim)
    gbs = nbytes / (avg / 1e3) / 1e9
    # the same caches read as keys quantized before RoPE (keys rotated in the kernel)
    for _ in range(args.warmup):
        nsnq.nsnq_attn_decode_rope(q, kc, vc, cb, cb, seq, T, Hkv=H, out=out, workspace=ws)
    barrier()
    torch.cuda.synchronize()
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        nsnq.nsnq_attn_decode_rope(q, kc, vc, cb, cb, seq, T, Hkv=H, out=out, workspace=ws)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ravg = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / len(evs), world, dev)
    rgbs = nbytes / (ravg / 1e3) / 1e9
    rope = {"ms_per_call": round(ravg, 4), "value": round(rgbs * world, 1), "unit": "GB/s",
            "roofline": {"bound": "hbm", "achieved": round(rgbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(rgbs / hbm, 4), "frac_vs_8tbs": round(rgbs / NOMINAL_HBM_GBS, 4), "peak_kind": peak_kind,
                         "kernel": "nsnq_attn_decode_rope (attn_rope_split + attn_combine)",
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": measured_traffic("nsnq_attn_decode_rope")}}
    return {"metric": "decode-attn HBM GB/s (algorithmic bytes)", "value": round(gbs * world, 1),
            "unit": "GB/s", "ms_per_call": round(avg, 4),
            "workload": "decode-16x32k-2b (B 16, Hq 32, Hkv 8, T 32768, d 128, 2 bit K and V)",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "frac_vs_8tbs": round(gbs / NOMINAL_HBM_GBS, 4), "peak_kind": peak_kind,
                         "kernel": "nsnq_attn_decode (attn_split + attn_combine)",
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": measured_traffic("nsnq_attn_decode")},
            "l2": "flushed before every call (cache 335 MB > L2 anyway)",
            "keys_before_rope": rope}


def _encoded_caches(nsnq, w, cb, dev, sub, packed, flags, seed):
    """K/V caches of the workload's shape and distributions, encoded on the
    device one sequence at a time (packed: double-quantized 4-bit s1 levels)."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    B, H, T = w.B, w.Hkv, w.T
    kc = nsnq.Cache.empty(B, H, T, sub, device=dev, packed=packed)
    vc = nsnq.Cache.empty(B, H, T, sub, device=dev, packed=packed)
    for b in range(B):
        for which, c in (("k", kc), ("v", vc)):
            nsnq.nsnq_encode(_device_kv(w, gen, dev, 1, T, which), cb, c.view(b, b + 1), flags=flags)
    return kc, vc


def run_attention_variants(args, nsnq, dev, world, barrier, hbm):
    """Decode attention at 16 x 32k over 1-bit caches, and over packed
    double-quantized caches (4-bit s1 levels, s2 alone, 4-bit codebook) at 1
    and 2 bit: 41 and 73 bytes per token instead of 48 and 80."""
    import torch
    w = S.WORKLOADS[ATTN_WORKLOAD]
    B, H, Hq, T = w.B, w.Hkv, w.Hq, w.T
    q = torch.randn(B, Hq, 128, generator=torch.Generator(device=dev).manual_seed(99), device=dev)
    q = q.to(torch.bfloat16)
    seq = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(nsnq.nsnq_attn_workspace(B, Hq, H, T), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    res = {}
    for name, sub, packed in (("1bit", 8, False), ("dq_packed_1bit", 8, True),
                              ("dq_packed_2bit", 4, True)):
        C = torch.from_numpy(load_codebook(sub)).to(dev)
        if packed:
            C = nsnq.codebook_quantize4(C)
        cb = nsnq.Codebook(C)
        flags = nsnq.ENCODE_DOUBLE_QUANT if packed else 0
        kc, vc = _encoded_caches(nsnq, w, cb, dev, sub, packed, flags, 4242 + sub)
        run = lambda: nsnq.nsnq_attn_decode(q, kc, vc, cb, cb, seq, T, Hkv=H, out=out,
                                             workspace=ws)
        for _ in range(args.warmup):
            run()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        for e0, e1 in evs:
            flush.zero_()
            e0.record(stream)
            run()
            e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        avg = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / len(evs), world, dev)
        per_tok = 2 * (128 // sub) + (9 if packed else 16)
        nbytes = B * H * T * per_tok
        gbs = nbytes / (avg / 1e3) / 1e9
        res[name] = {"ms_per_call": round(avg, 4), "bytes_per_token": per_tok,
                     "gbs": round(gbs * world, 1), "frac": round(gbs / hbm, 4)}
        del kc, vc
    res["dq_bytes_saved_per_token_head"] = 3.5
    res["workload"] = "decode-16x32k (B 16, Hq 32, Hkv 8, T 32768), caches encoded on the device"
    return res


def run_encode1_bench(args, nsnq, dev, world, barrier, hbm, peak_kind, x, sub=8):
    """Encode of the step's K tensor with every codeword scored on the tensor
    cores: at 1 bit (sub 8), or at 2 bits with the tensor-core search (sub 4,
    ENCODE_TC_SEARCH, no index: the comparison with the index walk)."""
    import torch
    B, H, T = x.shape[0], x.shape[1], x.shape[2]
    flags = nsnq.ENCODE_TC_SEARCH if sub == 4 else nsnq.ENCODE_DEFAULT
    cb = nsnq.Codebook(torch.from_numpy(load_codebook(sub)).to(dev), no_index=sub == 4)
    cache = nsnq.Cache.empty(B, H, T, sub, device=dev)
    ws = torch.empty(nsnq.nsnq_encode_workspace(B, H, T), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        nsnq.nsnq_encode(x, cb, cache, workspace=ws, flags=flags)
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        nsnq.nsnq_encode(x, cb, cache, workspace=ws, flags=flags)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    avg = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / len(evs), world, dev)
    nbytes = B * H * T * encode_bytes_per_token_head(sub)
    gbs = nbytes / (avg / 1e3) / 1e9
    what = ("1 bit/coord (g = 8), codewords scored on the tensor cores" if sub == 8 else
            "2 bits/coord (g = 4), all 256 codewords scored on the tensor cores (no index)")
    return {"metric": f"KV tokens/s encoded at {8 // sub} bit" + ("" if sub == 8 else "s, tensor-core search"),
            "value": round(B * T * world / (avg / 1e3), 1),
            "unit": "KV tokens/s (one tensor)", "ms_per_call": round(avg, 4),
            "workload": f"encode-8x4096 keys at {what}",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "frac_vs_8tbs": round(gbs / NOMINAL_HBM_GBS, 4), "peak_kind": peak_kind,
                         "kernel": f"nsnq_encode at {8 // sub} bit (nsn_stats + nsn_encode_tc)",
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": measured_traffic("nsnq_encode_1bit") if sub == 8 else None},
            "l2": "flushed before every call"}


def _device_kv(w, gen, dev, B, T, which):
    """Seeded K (outlier channels x LogNormal token scale) or V ~ N(0,1) of the
    workload's distribution, bf16 [B][Hkv][T][128], drawn on the device."""
    import torch
    z = torch.randn(B, w.Hkv, T, 128, generator=gen, device=dev)
    if which == "v":
        return z.to(torch.bfloat16)
    chans, signs = w.kdist.channels(128)
    bias = torch.zeros(128, device=dev)
    bias[chans] = torch.tensor(signs, device=dev) * w.kdist.bias
    s = torch.exp(w.kdist.sigma * torch.randn(B, w.Hkv, T, 1, generator=gen, device=dev))
    return ((z + bias) * s).to(torch.bfloat16)


def _median(xs):
    return statistics.median(xs) if xs else 0.0


def run_long_context_bench(args, nsnq, dev, world, barrier, hbm):
    """Long context (B 1, Hkv 8, Hq 32, T 131072, strong outliers, 2 bit):
    the prompt's K and V encoded (shift computed), then decode steps that each
    encode one new K/V token with the stored shift and attend over the cache."""
    import torch
    w = S.WORKLOADS["long-128k"]
    B, H, Hq, T, n_dec = w.B, w.Hkv, w.Hq, w.T, w.decode_steps
    cb = nsnq.Codebook(torch.from_numpy(load_codebook(w.sub_dim)).to(dev))
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321)
    k = _device_kv(w, gen, dev, B, T, "k")
    v = _device_kv(w, gen, dev, B, T, "v")
    kn = _device_kv(w, gen, dev, B, n_dec, "k")
    vn = _device_kv(w, gen, dev, B, n_dec, "v")
    q = torch.randn(n_dec, B, Hq, 128, generator=gen, device=dev).to(torch.bfloat16)
    cap = T + n_dec
    kc = nsnq.Cache.empty(B, H, cap, w.sub_dim, device=dev)
    vc = nsnq.Cache.empty(B, H, cap, w.sub_dim, device=dev)
    ws_e = torch.empty(nsnq.nsnq_encode_kv_workspace(B, H, T), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(nsnq.nsnq_attn_workspace(B, Hq, H, cap), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=dev)
    seqs = [torch.full((B,), T + i + 1, dtype=torch.int32, device=dev) for i in range(n_dec)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def prompt():
        nsnq.nsnq_encode_kv(k, v, cb, kc, vc, workspace=ws_e)

    for _ in range(max(1, args.warmup // 2)):
        prompt()
    barrier()
    torch.cuda.synchronize()
    p_ms = []
    for _ in range(3):
        flush.zero_()
        e0, e1 = ev(), ev()
        e0.record(stream)
        prompt()
        e1.record(stream)
        torch.cuda.synchronize()
        p_ms.append(e0.elapsed_time(e1))
    step_ms, att_ms = [], []
    for i in range(n_dec):
        flush.zero_()
        e0, e1, e2 = ev(), ev(), ev()
        e0.record(stream)
        nsnq.nsnq_encode_kv(kn[:, :, i:i + 1], vn[:, :, i:i + 1], cb, kc, vc, t_offset=T + i,
                            shift_mode=nsnq.SHIFT_GIVEN, workspace=ws_e)
        e1.record(stream)
        nsnq.nsnq_attn_decode(q[i], kc, vc, cb, cb, seqs[i], cap, Hkv=H, out=out, workspace=ws_a)
        e2.record(stream)
        torch.cuda.synchronize()
        step_ms.append(e0.elapsed_time(e2))
        att_ms.append(e1.elapsed_time(e2))
    # the same 64 steps captured once in a CUDA graph and replayed: the
    # device-side step latency without the per-call host overhead
    def decode_steps():
        for i in range(n_dec):
            nsnq.nsnq_encode_kv(kn[:, :, i:i + 1], vn[:, :, i:i + 1], cb, kc, vc, t_offset=T + i,
                                shift_mode=nsnq.SHIFT_GIVEN, workspace=ws_e)
            nsnq.nsnq_attn_decode(q[i], kc, vc, cb, cb, seqs[i], cap, Hkv=H, out=out,
                                  workspace=ws_a)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        decode_steps()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        decode_steps()
    graph.replay()
    torch.cuda.synchronize()
    g_ms = []
    for _ in range(3):
        flush.zero_()
        e0, e1 = ev(), ev()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        g_ms.append(e0.elapsed_time(e1) / n_dec)
    del graph
    barrier()
    pm = max_over_ranks(_median(p_ms), world, dev)
    sm = max_over_ranks(_median(step_ms), world, dev)
    am = max_over_ranks(_median(att_ms), world, dev)
    gm = max_over_ranks(_median(g_ms), world, dev)
    att_bytes = B * H * (T + n_dec // 2) * attn_bytes_per_token(w.sub_dim, w.sub_dim)
    enc_bytes = 2 * B * H * T * encode_bytes_per_token_head(w.sub_dim)
    return {"workload": "long-128k (B 1, Hkv 8, Hq 32, T 131072 prompt + 64 decode steps, strong "
                        "outlier K, 2 bit)",
            "prompt_encode_ms": round(pm, 4),
            "prompt_encode_tokens_per_s": round(B * T * world / (pm / 1e3), 1),
            "prompt_encode_gbs": round(enc_bytes / (pm / 1e3) / 1e9, 1),
            "decode_step_ms_median": round(sm, 4),
            "decode_step_ms_graph": round(gm, 4),
            "decode_attention_ms_median": round(am, 4),
            "decode_attention_gbs": round(att_bytes / (am / 1e3) / 1e9, 1),
            "decode_attention_frac": round(att_bytes / (am / 1e3) / 1e9 / hbm, 4),
            "steps": n_dec, "l2": "flushed before every timed call (graph: before each replay "
                                  "of the 64 steps)",
            "timing": "median over the steps of CUDA events around each step launched from "
                      "Python (host launch overhead included); graph: the 64 steps captured "
                      "once and replayed, total / 64"}


def run_serving_bench(args, nsnq, dev, world, barrier, hbm):
    """Serving mix (Hq 64, Hkv 8, 64 resident sequences x 8192 tokens, 2 bit):
    per step, the 2048-token prompts of 4 new sequences are encoded into 4
    spare cache slots and one decode query per resident sequence attends."""
    import torch
    w = S.WORKLOADS["serving-64x8k"]
    B, H, Hq, T = w.B, w.Hkv, w.Hq, w.T
    P, Tp = w.prefill_seqs, w.prefill_len
    cb = nsnq.Codebook(torch.from_numpy(load_codebook(w.sub_dim)).to(dev))
    gen = torch.Generator(device=dev)
    gen.manual_seed(5678)
    kc = nsnq.Cache.empty(B + P, H, T, w.sub_dim, device=dev)
    vc = nsnq.Cache.empty(B + P, H, T, w.sub_dim, device=dev)
    view = lambda c, b0, b1: nsnq.Cache(c.codes[b0:b1], c.scales[b0:b1], c.shift[b0:b1])
    ws_r = torch.empty(nsnq.nsnq_encode_kv_workspace(1, H, T), dtype=torch.uint8, device=dev)
    for b in range(B):  # resident sequences, one at a time
        nsnq.nsnq_encode_kv(_device_kv(w, gen, dev, 1, T, "k"), _device_kv(w, gen, dev, 1, T, "v"),
                            cb, view(kc, b, b + 1), view(vc, b, b + 1), workspace=ws_r)
    kp = _device_kv(w, gen, dev, P, Tp, "k")
    vp = _device_kv(w, gen, dev, P, Tp, "v")
    q = torch.randn(B, Hq, 128, generator=gen, device=dev).to(torch.bfloat16)
    seq = torch.full((B,), T, dtype=torch.int32, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=dev)
    ws_e = torch.empty(nsnq.nsnq_encode_kv_workspace(P, H, Tp), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(nsnq.nsnq_attn_workspace(B, Hq, H, T), dtype=torch.uint8, device=dev)
    kres, vres = view(kc, 0, B), view(vc, 0, B)
    kspare, vspare = view(kc, B, B + P), view(vc, B, B + P)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if evs: evs[0].record(stream)
        nsnq.nsnq_encode_kv(kp, vp, cb, kspare, vspare, workspace=ws_e)
        if evs: evs[1].record(stream)
        nsnq.nsnq_attn_decode(q, kres, vres, cb, cb, seq, T, Hkv=H, out=out, workspace=ws_a)
        if evs: evs[2].record(stream)

    for _ in range(args.warmup):
        step()
    barrier()
    torch.cuda.synchronize()
    rows = []
    for _ in range(max(args.steps, 5)):
        flush.zero_()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        step(evs)
        rows.append(evs)
    torch.cuda.synchronize()
    barrier()
    st = max_over_ranks(_median([e[0].elapsed_time(e[2]) for e in rows]), world, dev)
    en = max_over_ranks(_median([e[0].elapsed_time(e[1]) for e in rows]), world, dev)
    at = max_over_ranks(_median([e[1].elapsed_time(e[2]) for e in rows]), world, dev)
    att_bytes = B * H * T * attn_bytes_per_token(w.sub_dim, w.sub_dim)
    return {"workload": "serving-64x8k (Hq 64, Hkv 8, 64 x 8192-token 2-bit caches; per step "
                        "4 x 2048-token prompts encoded into spare slots + 64 decode queries)",
            "step_ms_median": round(st, 4), "encode_ms_median": round(en, 4),
            "encode_tokens_per_s": round(P * Tp * world / (en / 1e3), 1),
            "attention_ms_median": round(at, 4),
            "attention_gbs": round(att_bytes / (at / 1e3) / 1e9, 1),
            "attention_frac": round(att_bytes / (at / 1e3) / 1e9 / hbm, 4),
            "l2": "flushed before every timed step"}


# ------------------------------------------------------------ oracle arm --
def oracle_step_sample(n_seq: int = 1, n_heads: int = 8):
    """The oracle on a bounded sample of the step: n_seq sequences x n_heads
    kv-heads (K and V encode, dequant, attention for their query heads).
    Returns (seconds, tokens-equivalent processed)."""
    from oracle import oracle as O
    w = S.WORKLOADS[STEP_WORKLOAD]
    C = load_codebook(w.sub_dim)
    k = S.io_to_f64(S.to_io(S.keys(w, b0=0, b1=n_seq)[:, :n_heads], "bf16"), "bf16")
    v = S.io_to_f64(S.to_io(S.values(w, b0=0, b1=n_seq)[:, :n_heads], "bf16"), "bf16")
    G = STEP_HQ // w.Hkv
    q = S.io_to_f64(S.to_io(S.queries(S.Workload(**{**w.__dict__, "Hq": STEP_HQ}), B=n_seq)
                            [:, :n_heads * G], "bf16"), "bf16")
    t0 = time.perf_counter()
    ok, ov = O.encode(k, C), O.encode(v, C)
    Kh = O.dequant(ok["codes"], *O.stored(ok), C)
    Vh = O.dequant(ov["codes"], *O.stored(ov), C)
    O.attention(q, Kh, Vh)
    dt = time.perf_counter() - t0
    # tokens are counted over all kv-heads of the layer: scale by the sampled fraction
    tokens = n_seq * w.T * (n_heads / w.Hkv)
    return dt, tokens


def cpu_baseline(args):
    dt, tokens = oracle_step_sample(4, 8)
    return {"value": round(tokens / dt, 2), "unit": "KV tokens/s", "cores": 1, "kind": "oracle",
            "sample": "4 sequences x 8 kv-heads x 4096 tokens (K+V encode, dequant, attention of 32 "
                      f"query heads), single-threaded fp64 C, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import build as obuild
    obuild.build()
    for _ in range(args.warmup):
        oracle_step_sample(1, 1)
    times, toks = [], 0.0
    for _ in range(args.steps):
        dt, tokens = oracle_step_sample(1, 2)
        times.append(dt)
        toks = tokens
    avg = sum(times) / len(times)
    value = toks / avg
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "KV tokens/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(avg * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "encode-8x4096 + decode (Llama-3-8B layer: B 8, Hkv 8, Hq 32, "
                               "T 4096, d 128, 2 bit/coord)", "global_batch": 8, "seq_len": 4096,
                   "parallelism": "none (CPU oracle)"},
        "cpu_baseline": {"value": round(value, 2), "unit": "KV tokens/s", "cores": 1,
                         "kind": "oracle",
                         "sample": "per step: 1 sequence x 2 kv-heads x 4096 tokens (K+V encode, "
                                   "dequant, attention of 8 query heads), scaled to all 8 kv-heads"},
        "e2e": {"value": round(value, 2), "unit": "KV tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["nsnq", "reference"], default="nsnq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the roofline kernel from an ncu capture")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
