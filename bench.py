"""Benchmark: StiefAttention latent-KV decode on B200.

A step is one pass of the whole hot path for one decode step of a batch:
stief_compress_append of one new key/value token per (sequence, KV head) into
the latent cache, then stief_decode_attention over the grown cache, for every
layer of the workload.  Inputs are seeded synthetic data resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs the same per-GPU
workload on its own GPU (independent sequences: weak scaling); the step time is
the maximum over ranks.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import stief_inputs as si  # noqa: E402

METRIC = "decode attn tokens/s and achieved HBM GB/s (frac of peak) over latent KV cache"
DEFAULT_WORKLOAD = "llama3_8b_32k"
FLUSH_BYTES = 512 << 20  # > 126 MB L2: written between timed steps
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------- helpers

def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _kernel_source_hash() -> str:
    p = os.path.join(ROOT, "decode_attention_stief_b200", "csrc", "decode_kernels.cu")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def _traffic_per_launch(workload: str):
    """dram read+write bytes per split-kernel launch from a committed ncu capture, or None if
    absent or taken on a different version of the kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        e = t[workload]
        if e.get("source_sha256_16") != _kernel_source_hash():
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()

    def summary(self):
        if self.proc is None or self.path is None:
            return None
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), reasons=parts[4],
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- workload state

class Layer:
    """Device state of one attention layer: bases, latent cache, lengths."""

    def __init__(self, w: si.Workload, layer: int, rK: int, rV: int, L0: int, L_max: int,
                 seed: int, dev):
        self.rK, self.rV = rK, rV
        self.L_max = L_max
        P_K, P_V = si.bases_bf16(si.sub_seed(seed, 11, layer), w.Hkv, w.d, rK, rV)
        self.P_K, self.P_V = P_K.to(dev), P_V.to(dev)
        self.k_lat = si.latent_cache_torch(si.sub_seed(seed, 12, layer), w.B, w.Hkv, L_max, rK, 0, dev)
        self.v_lat = si.latent_cache_torch(si.sub_seed(seed, 13, layer), w.B, w.Hkv, L_max, rV, 1, dev)
        self.seq_lens = torch.full((w.B,), L0, dtype=torch.int32, device=dev)
        self.ws = None


def build_state(w: si.Workload, total_steps: int, seed: int, dev):
    """Per-layer caches holding w.L - 1 - warmup tokens so the first timed step attends w.L."""
    import decode_attention_stief_b200 as stief
    L_max = w.L + total_steps + 1
    layers = []
    for li, (rK, rV) in enumerate(w.layer_ranks()):
        lay = Layer(w, li, rK, rV, w.L - 1, L_max, seed, dev)
        lay.ws = stief.workspace_for(w.B, w.Hq, w.Hkv, rV, L_max, device=dev)
        layers.append(lay)
    return layers, L_max


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args, w: si.Workload):
    import decode_attention_stief_b200 as stief
    ws_n, rank, local = _dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if ws_n > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    seed = w.seed + 7919 * rank
    W, K = args.warmup, args.steps
    n_steps = W + K + args.decode_iters
    layers, L_max = build_state(w, n_steps + W + K, seed, dev)
    # rewind: lengths so that after W warm-up appends the first timed decode sees w.L tokens
    for lay in layers:
        lay.seq_lens.fill_(w.L - 1 - W)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 1)
    steps_total = W + K
    k_new = [torch.randn((w.B, w.Hkv, 1, w.d), generator=g, device=dev).to(torch.bfloat16)
             for _ in range(steps_total)]
    v_new = [torch.randn((w.B, w.Hkv, 1, w.d), generator=g, device=dev).to(torch.bfloat16)
             for _ in range(steps_total)]
    q = [torch.randn((w.B, w.Hq, w.d), generator=g, device=dev).to(torch.bfloat16)
         for _ in range(steps_total)]
    out = torch.empty((len(layers), w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, q_i, k_i, v_i):
        for li, lay in enumerate(layers):
            stief.stief_compress_append(k_i, v_i, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat,
                                        lay.seq_lens, dev_status=status)
            stief.stief_decode_attention(q_i, lay.P_K, lay.P_V, lay.k_lat, lay.v_lat,
                                         lay.seq_lens, out[li], lay.ws, max_seq_len=L_max,
                                         num_splits=args.splits, dev_status=status)

    def barrier():
        if ws_n > 1:
            torch.distributed.barrier()

    # ---- warm-up
    for i in range(W):
        step(i, q[i], k_new[i], v_new[i])
    torch.cuda.synchronize()

    # ---- timed region: K steps, L2 flushed before each, CUDA events around each
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    ctx_lens = []
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_id = cvd.split(",")[local].strip() if cvd else str(local)
    lay0 = layers[0]
    with ClockSampler(smi_id) as clk:
        # keep the GPU loaded (decode only, lengths unchanged) for ~0.6 s so the clock
        # samples bracketing the timed region are taken under load
        t_keep = time.perf_counter()
        while time.perf_counter() - t_keep < args.clock_window:
            for _ in range(20):
                stief.stief_decode_attention(q[0], lay0.P_K, lay0.P_V, lay0.k_lat, lay0.v_lat,
                                             lay0.seq_lens, out[0], lay0.ws, max_seq_len=L_max,
                                             dev_status=status)
            torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        t_wall0 = time.perf_counter()
        for j in range(K):
            i = W + j
            flush.zero_()
            evs[j][0].record(stream)
            step(i, q[i], k_new[i], v_new[i])
            evs[j][1].record(stream)
            ctx_lens.append(w.L + j)
        torch.cuda.synchronize()
        barrier()
        t_wall = time.perf_counter() - t_wall0
        time.sleep(0.25)  # one more sample after the timed region
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms_per_step = sum(step_ms) / K
    clocks = clk.summary()
    st = stief.stief_read_device_status(status)
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after the timed steps")

    # ---- decode kernel timing for the roofline (decode call alone, L2 flushed before each)
    dec_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.decode_iters)]
    L_dec = int(lay0.seq_lens[0].item())
    for j in range(args.decode_iters):
        flush.zero_()
        dec_evs[j][0].record(stream)
        stief.stief_decode_attention(q[0], lay0.P_K, lay0.P_V, lay0.k_lat, lay0.v_lat,
                                     lay0.seq_lens, out[0], lay0.ws, max_seq_len=L_max,
                                     num_splits=args.splits, dev_status=status)
        dec_evs[j][1].record(stream)
    torch.cuda.synchronize()
    dec_ms = sorted(a.elapsed_time(b) for a, b in dec_evs)
    dec_ms_mean = sum(dec_ms) / len(dec_ms)

    # ---- end to end through the public API with host buffers (pinned), copies timed
    h_q = [x.cpu().pin_memory() for x in q]
    h_k = [x.cpu().pin_memory() for x in k_new]
    h_v = [x.cpu().pin_memory() for x in v_new]
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    d_q = torch.empty_like(q[0])
    d_k = torch.empty_like(k_new[0])
    d_v = torch.empty_like(v_new[0])
    for lay in layers:   # rewind the lengths to replay the same context
        lay.seq_lens.fill_(w.L - 1 - W)
    for i in range(W):
        step(i, q[i], k_new[i], v_new[i])
    e2e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    for j in range(K):
        i = W + j
        flush.zero_()
        e2e_evs[j][0].record(stream)
        d_q.copy_(h_q[i], non_blocking=True)
        d_k.copy_(h_k[i], non_blocking=True)
        d_v.copy_(h_v[i], non_blocking=True)
        step(i, d_q, d_k, d_v)
        h_out.copy_(out, non_blocking=True)
        e2e_evs[j][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_evs) / K
    h2d = d_q.numel() * 2 + d_k.numel() * 2 + d_v.numel() * 2
    d2h = out.numel() * 2

    if ws_n > 1:
        t = torch.tensor([ms_per_step, e2e_ms, dec_ms_mean], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms_per_step, e2e_ms, dec_ms_mean = (float(x) for x in t.tolist())

    # ---- prefill compress (the prefill + batched decode workload): one 4096-token chunk
    # per layer through stief_compress_append (tcgen05 path), timed separately
    compress = None
    if w.name == "prefill_b64" and not args.no_prefill:
        compress = time_prefill_compress(args, len(layers), dev, flush, stream)

    # ---- numbers
    tokens_per_step = w.B * ws_n
    value = tokens_per_step / (ms_per_step / 1e3)
    bytes_per_dec = 2 * (lay0.rK + lay0.rV) * w.B * w.Hkv * L_dec
    achieved = bytes_per_dec / (dec_ms_mean / 1e3) / 1e9
    peak, peak_kind = _hbm_peak()
    step_bytes = sum(2 * (lay.rK + lay.rV) * w.B * w.Hkv for lay in layers) * (
        sum(ctx_lens) / len(ctx_lens))
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": ws_n,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "context": w.L,
            "layers": len(layers), "ranks": [list(r) for r in w.layer_ranks()][:4]
            + (["..."] if len(layers) > 4 else []),
            "step": "append 1 token per (sequence, KV head) + decode, every layer",
            "context_growth": "+1 token per step (first timed step attends context tokens)",
            "l2": f"flushed before every timed step ({FLUSH_BYTES >> 20} MiB write)",
            "parallelism": f"independent sequences per GPU x{ws_n}",
        },
        "hbm_gbs_step": round(step_bytes / (ms_per_step / 1e3) / 1e9, 1),
        "roofline": {
            "kernel": "stief_decode_kernel (stief_decode_attention)",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_kind": f"{peak_kind} hbm_gbs (copy bandwidth, burst)",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": _traffic_per_launch(w.name),
            "algorithmic_bytes": bytes_per_dec,
            "decode_us": round(dec_ms_mean * 1e3, 3),
            "decode_us_min": round(dec_ms[0] * 1e3, 3),
        },
        "e2e": {"value": round(tokens_per_step / (e2e_ms / 1e3), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * len(layers) * K,  # compress rows, length update, decode
        "clocks": clocks,
        "wall_s_timed_region": round(t_wall, 3),
    }
    if compress is not None:
        result["compress"] = compress
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if ws_n > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def time_prefill_compress(args, n_layers: int, dev, flush, stream):
    """Time stief_compress_append of one prefill chunk (B=1, Hkv=8, T=4096, ranks 64/64)
    for every layer; L2 flushed before each repetition.  Returns a summary dict."""
    import decode_attention_stief_b200 as stief
    c = si.PREFILL_CHUNK
    B, Hkv, T, d, rK, rV = c["B"], c["Hkv"], c["T"], c["d"], c["rK"], c["rV"]
    ks = [si.low_rank_rows_torch(si.sub_seed(c["seed"], 21, li), B * Hkv, T, d, dev).view(B, Hkv, T, d)
          for li in range(n_layers)]
    vs = [si.low_rank_rows_torch(si.sub_seed(c["seed"], 22, li), B * Hkv, T, d, dev).view(B, Hkv, T, d)
          for li in range(n_layers)]
    P_K, P_V = si.bases_bf16(c["seed"], Hkv, d, rK, rV)
    P_K, P_V = P_K.to(dev), P_V.to(dev)
    kl = [torch.empty((B, Hkv, T, rK), dtype=torch.bfloat16, device=dev) for _ in range(n_layers)]
    vl = [torch.empty((B, Hkv, T, rV), dtype=torch.bfloat16, device=dev) for _ in range(n_layers)]
    lens = torch.zeros((n_layers, B), dtype=torch.int32, device=dev)

    def chunk():
        for li in range(n_layers):
            stief.stief_compress_append(ks[li], vs[li], P_K, P_V, kl[li], vl[li], lens[li])

    for _ in range(args.warmup):
        lens.zero_()
        chunk()
    reps = max(3, min(args.steps, 20))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for r in range(reps):
        lens.zero_()
        flush.zero_()
        evs[r][0].record(stream)
        chunk()
        evs[r][1].record(stream)
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in evs)
    ms_med = ms[len(ms) // 2]
    bytes_moved = n_layers * B * Hkv * T * (2 * d * 2 + 2 * (rK + rV))
    flops = n_layers * B * Hkv * T * 2 * d * (rK + rV)
    peak, kind = _hbm_peak()
    return {"what": f"stief_compress_append of a {T}-token chunk, {Hkv} KV heads, ranks {rK}/{rV}, "
                    f"x{n_layers} layers (tcgen05 path), L2 flushed",
            "us_total": round(ms_med * 1e3, 2), "us_per_layer": round(ms_med * 1e3 / n_layers, 3),
            "algorithmic_bytes": bytes_moved,
            "GBs": round(bytes_moved / (ms_med / 1e3) / 1e9, 1),
            "frac_of_hbm_peak": round(bytes_moved / (ms_med / 1e3) / 1e9 / peak, 4),
            "TFLOPs": round(flops / (ms_med / 1e3) / 1e12, 2),
            "kernel_launches_per_layer": 2}


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_step(w: si.Workload, L: int):
    """A callable doing one oracle step of layer 0 at context L: append 1 token + decode."""
    import oracle
    rK, rV = w.layer_ranks()[0]
    rng = np.random.default_rng(w.seed)
    Pk = si.bf16_to_f64(si.to_bf16(si.bases(w.seed, w.Hkv, w.d, rK)))
    Pv = si.bf16_to_f64(si.to_bf16(si.bases(w.seed + 1, w.Hkv, w.d, rV)))
    kl = rng.standard_normal((w.B, w.Hkv, L + 1, rK))
    vl = rng.standard_normal((w.B, w.Hkv, L + 1, rV))
    kn = rng.standard_normal((w.B, w.Hkv, 1, w.d))
    vn = rng.standard_normal((w.B, w.Hkv, 1, w.d))
    qq = rng.standard_normal((w.B, w.Hq, w.d))
    lens = np.full(w.B, L, np.int32)

    def step():
        k2, v2, l2, _ = oracle.compress_append(kn, vn, Pk, Pv, kl, vl, lens)
        oracle.decode(qq, Pk, Pv, k2, v2, l2)
    return step


def _sample_context(w: si.Workload, seconds_per_step: float) -> int:
    """Context for one oracle step of about seconds_per_step (probed at <= 1024 tokens)."""
    probe_L = min(w.L, 1024)
    fn = _oracle_step(w, probe_L)
    t0 = time.perf_counter()
    fn()
    t_probe = time.perf_counter() - t0
    est_full = t_probe * w.L / probe_L
    if est_full <= seconds_per_step:
        return w.L
    return max(probe_L, int(w.L * seconds_per_step / est_full))


def _time_oracle(w: si.Workload, L_s: int, warmup: int, steps: int):
    fn = _oracle_step(w, L_s)
    for _ in range(warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(steps):
        fn()
    return (time.perf_counter() - t0) / steps


def _oracle_tokens_per_s(w: si.Workload, L_s: int, t_step: float) -> float:
    # cost is linear in context and in the number of layers
    return w.B / (t_step * (w.L / L_s) * len(w.layer_ranks()))


def cpu_baseline(w: si.Workload, budget_s: float = 20.0):
    """The fp64 oracle (as it stands) on host cores, on a bounded sample of one step:
    layer 0, all sequences and heads, append 1 token + decode, at a context shortened
    so one step takes about budget_s / 2; tokens/s scaled to the full context and layers."""
    import oracle
    threads = min(oracle.max_threads(), w.B * w.Hkv)
    L_s = _sample_context(w, budget_s / 2)
    t = _time_oracle(w, L_s, 0, 2)
    return {"value": round(_oracle_tokens_per_s(w, L_s, t), 4), "unit": "tokens/s",
            "cores": threads, "kind": "oracle",
            "sample": f"layer 0, all {w.B} sequences x {w.Hq} heads, append 1 + decode at "
                      f"context {L_s} (of {w.L}), 2 steps of {t:.2f} s; scaled "
                      f"x{w.L / L_s:.2f} to the context and x{len(w.layer_ranks())} layers"}


def run_reference(args, w: si.Workload):
    """The reference arm: the fp64 oracle on host cores, W warm-up + K timed steps, each a
    bounded sample (layer 0 at a shortened context) of the GPU arm's step."""
    ws_n, rank, _ = _dist_env()
    if rank != 0:
        return
    import oracle
    K, W = args.steps, args.warmup
    threads = min(oracle.max_threads(), w.B * w.Hkv)
    L_s = _sample_context(w, max(0.05, args.cpu_seconds / (K + W)))
    t = _time_oracle(w, L_s, W, K)
    value = _oracle_tokens_per_s(w, L_s, t)
    sample = (f"layer 0, all {w.B} sequences x {w.Hq} heads, append 1 + decode at context "
              f"{L_s} (of {w.L}); {K} timed steps of {t:.3f} s; scaled x{w.L / L_s:.2f} to "
              f"the context and x{len(w.layer_ranks())} layers")
    res = {
        "metric": METRIC, "impl": "reference", "value": round(value, 4), "unit": "tokens/s",
        "n_gpus": ws_n, "steps": K, "warmup": W,
        "ms_per_step": round(w.B / value * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
                   "context": w.L, "layers": len(w.layer_ranks())},
        "cpu_baseline": {"kind": "oracle", "cores": threads, "value": round(value, 4),
                         "unit": "tokens/s", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(si.WORKLOADS))
    ap.add_argument("--impl", default="stief", choices=["stief", "reference"])
    ap.add_argument("--decode-iters", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=30.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill-compress measurement of the prefill_b64 workload")
    ap.add_argument("--layers", type=int, default=0,
                    help="diagnostics: run only the first N layers of the workload")
    ap.add_argument("--splits", type=int, default=0,
                    help="diagnostics: force the decode split count (0 = automatic)")
    ap.add_argument("--clock-window", type=float, default=0.6,
                    help="seconds of untimed decode load before the timed region")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = si.WORKLOADS[args.workload]
    if args.layers > 0:
        import dataclasses
        w = dataclasses.replace(w, layers=min(args.layers, w.layers),
                                ranks=w.ranks[:args.layers] if w.ranks else None)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
